"""Parity of the CUDA megakernel (through the C ABI) against the CPU oracle.

Bar (element by element on the same seeded inputs): per-step logits
max|diff| <= 0.05 and cosine >= 0.9999; greedy tokens identical over the tiny
model's 16 steps; event counters, completion counts and the work-queue head
bit-exact after every step.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import persistent_megakernel_decode_03_b200 as mk
import synthetic as syn
from tests.gpu_util import (compare_logits, device_weights, fill_kv_context, fill_oracle_kv,
                            make_decoder)

pytestmark = pytest.mark.gpu

CFG1_SEED = 1


def names(cfg):
    return [s.name for s in syn.tensor_specs(cfg)]


def check_counters(dec):
    info = dec.info
    c, ev = mk.mk_state_read_counters(dec.state, info.n_events, dec.stream())
    thr = mk.mk_graph_export_thresholds(dec.graph)
    assert c.error == 0, (c.error, list(c.error_info))
    assert c.done == info.n_tasks * c.epoch
    assert c.queue_head == (info.n_tasks + info.n_sm) * c.epoch
    assert ev == [t * c.epoch for t in thr]


def test_generator_device_bits_equal_host_bits():
    cfg = syn.TINY
    specs, ts = device_weights(cfg, 77, gain_sigma=0.1)
    for s, t in list(zip(specs, ts))[:6]:
        host = syn.host_tensor(s, 77)
        dev = t.view(torch.int16).cpu().numpy().view(np.uint16)
        np.testing.assert_array_equal(dev, host)


@pytest.mark.parametrize("gain_sigma", [0.0, 0.1])
def test_tiny_every_position_and_greedy(gain_sigma):
    """Prompt of 39 tokens fed one step at a time, then 16 greedy steps: every
    step's logits against the oracle, identical greedy tokens, exact counters."""
    cfg = syn.TINY
    seed = syn.SEED_WEIGHTS + CFG1_SEED
    specs, ts = device_weights(cfg, seed, gain_sigma)
    host_w = syn.host_weights(cfg, seed, gain_sigma)
    prompt = syn.host_tokens(39, syn.SEED_PROMPT + CFG1_SEED, cfg.vocab)
    max_ctx = 64
    dec = make_decoder(cfg, ts, 1, max_ctx)
    orc = oracle.Model(cfg, host_w, max_ctx, names(cfg))
    tok_d = torch.zeros(1, dtype=torch.int32, device="cuda")
    pos_d = torch.zeros(1, dtype=torch.int32, device="cuda")
    tok = int(prompt[0])
    worst = (0.0, 1.0)
    for p in range(39 + 16):
        if p < 39:
            tok = int(prompt[p])
        tok_d.fill_(tok)
        pos_d.fill_(p)
        g = dec.step(tok_d, pos_d).cpu().numpy()[0]
        dec.check()
        ref = orc.decode_step(tok, p)["logits"]
        d, cos, ok = compare_logits(g, ref)
        worst = (max(worst[0], d), min(worst[1], cos))
        assert ok, f"position {p}: max|diff| {d:.3g} cos {cos:.7f}"
        if p >= 38:
            g_tok, o_tok = int(np.argmax(g)), oracle.argmax(ref)
            assert g_tok == o_tok, f"greedy token differs at step {p - 38}"
            tok = g_tok
        check_counters(dec)
    print(f"tiny gain_sigma={gain_sigma}: worst max|diff| {worst[0]:.3g}, worst cos {worst[1]:.8f}")
    dec.close()


def test_tiny_prefill_entry_point_then_decode():
    cfg = syn.TINY
    seed = syn.SEED_WEIGHTS + CFG1_SEED
    specs, ts = device_weights(cfg, seed)
    host_w = syn.host_weights(cfg, seed)
    prompt = syn.host_tokens(39, syn.SEED_PROMPT + CFG1_SEED, cfg.vocab)
    dec = make_decoder(cfg, ts, 1, 64)
    orc = oracle.Model(cfg, host_w, 64, names(cfg))
    last = dec.prefill(torch.tensor(prompt, dtype=torch.int32, device="cuda")).cpu().numpy()
    dec.check()
    for p, t in enumerate(prompt):
        ref = orc.decode_step(int(t), p)["logits"]
    d, cos, ok = compare_logits(last, ref)
    assert ok, (d, cos)
    # KV cache contents written by the prefill equal the oracle's (bf16 bits, up to rare 1-ulp)
    k_gpu = dec.k_pages[0].view(torch.int16).cpu().numpy().view(np.uint16)   # [pages][nkv][16][d]
    k_gpu = k_gpu.transpose(0, 2, 1, 3).reshape(-1, cfg.n_kv_heads, cfg.head_dim)[:39]
    diff = np.abs(k_gpu.astype(np.int32) - orc.k[0][:39].astype(np.int32))
    assert diff.max() <= 1 and (diff > 0).mean() < 0.01
    # continue decoding greedily from the prefill
    tok = int(np.argmax(last))
    tok_d = torch.tensor([tok], dtype=torch.int32, device="cuda")
    pos_d = torch.tensor([39], dtype=torch.int32, device="cuda")
    g = dec.step(tok_d, pos_d).cpu().numpy()[0]
    dec.check()
    ref = orc.decode_step(tok, 39)["logits"]
    assert compare_logits(g, ref)[2]
    check_counters(dec)
    dec.close()


def test_tiny_host_entry_point_matches_device_entry_point():
    cfg = syn.TINY
    specs, ts = device_weights(cfg, 5)
    dec_a = make_decoder(cfg, ts, 1, 32)
    dec_b = make_decoder(cfg, ts, 1, 32)
    out_host = np.zeros((1, cfg.vocab), dtype=np.float32)
    for p, t in enumerate([3, 14, 159, 265]):
        dec_a.step(torch.tensor([t], dtype=torch.int32, device="cuda"),
                   torch.tensor([p], dtype=torch.int32, device="cuda"))
        dec_b.step_host(np.array([t], dtype=np.int32), np.array([p], dtype=np.int32), out_host)
        np.testing.assert_array_equal(dec_a.logits.cpu().numpy()[0], out_host[0])
    dec_a.check()
    dec_b.check()


def test_repeat_runs_are_bit_identical():
    """No float atomics: the same inputs give the same bits, run after run."""
    cfg = syn.TINY
    specs, ts = device_weights(cfg, 9)
    outs = []
    for rep in range(3):
        dec = make_decoder(cfg, ts, 1, 48)
        for p, t in enumerate([11, 22, 33, 44, 55, 66, 77]):
            g = dec.step(torch.tensor([t], dtype=torch.int32, device="cuda"),
                         torch.tensor([p], dtype=torch.int32, device="cuda")).clone()
        dec.check()
        outs.append(g.cpu().numpy())
        dec.close()
    assert all(np.array_equal(outs[0], o) for o in outs[1:])


def test_tiny_moe_parity():
    cfg = syn.TINY_MOE
    seed = 4242
    specs, ts = device_weights(cfg, seed, 0.1)
    host_w = syn.host_weights(cfg, seed, 0.1)
    dec = make_decoder(cfg, ts, 1, 64)
    orc = oracle.Model(cfg, host_w, 64, names(cfg))
    toks = syn.host_tokens(24, 99, cfg.vocab)
    for p, t in enumerate(toks):
        g = dec.step(torch.tensor([int(t)], dtype=torch.int32, device="cuda"),
                     torch.tensor([p], dtype=torch.int32, device="cuda")).cpu().numpy()[0]
        dec.check()
        sel_g = np.array([mk.mk_state_read_buffer(dec.state, 3, l, cfg.top_k) for l in range(cfg.n_layers)])
        out = orc.decode_step(int(t), p)
        np.testing.assert_array_equal(sel_g.astype(np.int32), out["moe_sel"], err_msg=f"router, pos {p}")
        wts_g = np.array([mk.mk_state_read_buffer(dec.state, 4, l, cfg.top_k) for l in range(cfg.n_layers)])
        np.testing.assert_allclose(wts_g, out["moe_wts"], rtol=1e-4, atol=1e-6)
        d, cos, ok = compare_logits(g, out["logits"])
        assert ok, f"position {p}: max|diff| {d:.3g} cos {cos:.7f}"
        check_counters(dec)
    dec.close()


def test_position_zero_and_ragged_page_tail():
    """Position 0 (empty cache) and a position whose page is only partly filled."""
    cfg = syn.TINY
    specs, ts = device_weights(cfg, 31)
    host_w = syn.host_weights(cfg, 31)
    dec = make_decoder(cfg, ts, 1, 40)
    orc = oracle.Model(cfg, host_w, 40, names(cfg))
    for p in range(35):      # 35 = two full pages + a 3-token tail
        t = (p * 37) % cfg.vocab
        g = dec.step(torch.tensor([t], dtype=torch.int32, device="cuda"),
                     torch.tensor([p], dtype=torch.int32, device="cuda")).cpu().numpy()[0]
        ref = orc.decode_step(t, p)["logits"]
        assert compare_logits(g, ref)[2], p
    dec.check()
    dec.close()


def test_shuffled_pages_equal_contiguous_pages():
    cfg = syn.TINY
    specs, ts = device_weights(cfg, 12)
    max_ctx = 64
    pages = (max_ctx + 15) // 16
    perm = torch.tensor(syn.page_permutation(3 * pages, 7)[:pages], dtype=torch.int32, device="cuda")
    dec_c = make_decoder(cfg, ts, 1, max_ctx)
    dec_s = make_decoder(cfg, ts, 1, max_ctx, page_table=perm.view(1, pages), n_pages=3 * pages)
    for p in range(50):
        t = torch.tensor([(p * 13 + 1) % cfg.vocab], dtype=torch.int32, device="cuda")
        pp = torch.tensor([p], dtype=torch.int32, device="cuda")
        a = dec_c.step(t, pp).clone()
        b = dec_s.step(t, pp).clone()
        assert torch.equal(a, b), p
    dec_c.check()
    dec_s.check()


def test_timeout_is_reported_and_state_recovers():
    """A wait that nothing satisfies ends with MK_ERR_TIMEOUT; the next step is fine."""
    cfg = syn.TINY
    specs, ts = device_weights(cfg, 3)
    dec = make_decoder(cfg, ts, 1, 32)
    t = torch.tensor([5], dtype=torch.int32, device="cuda")
    p0 = torch.tensor([0], dtype=torch.int32, device="cuda")
    ref = dec.step(t, p0).clone()
    dec.check()
    mk.mk_state_set_timeout(dec.state, 50_000_000)           # 50 ms
    mk.mk_state_debug_wait_offset(dec.state, 1)
    dec.step(t, p0)
    assert dec.sync() == mk.MK_ERR_TIMEOUT
    mk.mk_state_debug_wait_offset(dec.state, 0)
    again = dec.step(t, p0).clone()
    assert dec.sync() == mk.MK_OK
    assert torch.equal(again, ref)


def test_invalid_token_and_position_are_reported_by_the_device():
    cfg = syn.TINY
    specs, ts = device_weights(cfg, 3)
    dec = make_decoder(cfg, ts, 1, 32)
    dec.step(torch.tensor([cfg.vocab + 5], dtype=torch.int32, device="cuda"),
             torch.tensor([0], dtype=torch.int32, device="cuda"))
    assert dec.sync() == mk.MK_ERR_INVALID_ARG
    dec.step(torch.tensor([1], dtype=torch.int32, device="cuda"),
             torch.tensor([32], dtype=torch.int32, device="cuda"))    # == max_ctx
    assert dec.sync() == mk.MK_ERR_INVALID_ARG
    dec.step(torch.tensor([1], dtype=torch.int32, device="cuda"),
             torch.tensor([0], dtype=torch.int32, device="cuda"))
    assert dec.sync() == mk.MK_OK


def test_host_argument_errors():
    cfg = syn.TINY
    specs, ts = device_weights(cfg, 3)
    dec = make_decoder(cfg, ts, 1, 32)
    t = torch.tensor([1], dtype=torch.int32, device="cuda")
    with pytest.raises(mk.MkError):
        mk.mk_decode_step(dec.state, t.data_ptr(), t.data_ptr(), 2, dec.kv, dec.logits.data_ptr(), 0)
    bad = mk.make_kv(dec.k_pages.data_ptr(), dec.v_pages.data_ptr(), dec.page_table.data_ptr(),
                     dec.n_pages, dec.max_pages, page_size=8)
    with pytest.raises(mk.MkError):
        mk.mk_decode_step(dec.state, t.data_ptr(), t.data_ptr(), 1, bad, dec.logits.data_ptr(), 0)


@pytest.mark.parametrize("n_ctx", [300])
def test_8b_full_size_synthetic_context(n_ctx):
    """8B-class shapes at full size: synthetic cache of n_ctx positions, then two
    decode steps, each compared element by element with the oracle."""
    cfg = syn.LLAMA8B
    seed = syn.SEED_WEIGHTS + 2
    specs, ts = device_weights(cfg, seed)
    max_ctx = 551
    dec = make_decoder(cfg, ts, 1, max_ctx)
    fill_kv_context(dec, cfg, 0, n_ctx, syn.SEED_KV + 2)
    host_w = syn.host_weights(cfg, seed)
    orc = oracle.Model(cfg, host_w, max_ctx, names(cfg))
    fill_oracle_kv(orc, cfg, 0, n_ctx, syn.SEED_KV + 2)
    toks = syn.host_tokens(2, syn.SEED_PROMPT + 2, cfg.vocab)
    for i, t in enumerate(toks):
        p = n_ctx + i
        g = dec.step(torch.tensor([int(t)], dtype=torch.int32, device="cuda"),
                     torch.tensor([p], dtype=torch.int32, device="cuda")).cpu().numpy()[0]
        dec.check()
        ref = orc.decode_step(int(t), p)["logits"]
        d, cos, ok = compare_logits(g, ref)
        print(f"8B step at position {p}: max|diff| {d:.3g} cos {cos:.8f}")
        assert ok, (p, d, cos)
        check_counters(dec)
    dec.close()


def test_prefill_with_many_one_stage_tiles_per_cta():
    """Prefill at 8B shapes (two layers, full 128256-row LM head): the prompt's
    non-final steps skip the LM head, so every CTA runs ~54 tiles of one ring
    stage each in a row, and its warps drift apart by more tasks than there
    are per-task reduction slots.  Last logits, KV contents and counters must
    still match."""
    cfg = dataclasses.replace(syn.LLAMA8B, n_layers=2)
    seed = syn.SEED_WEIGHTS + 2
    specs, ts = device_weights(cfg, seed)
    n = 6
    prompt = syn.host_tokens(n, syn.SEED_PROMPT + 2, cfg.vocab)
    dec = make_decoder(cfg, ts, 1, 64)
    last = dec.prefill(torch.tensor(prompt, dtype=torch.int32, device="cuda")).cpu().numpy()
    dec.check()
    check_counters(dec)
    orc = oracle.Model(cfg, syn.host_weights(cfg, seed), 64, names(cfg))
    for p, t in enumerate(prompt):
        ref = orc.decode_step(int(t), p)["logits"]
    d, cos, ok = compare_logits(last, ref)
    assert ok, (d, cos)
    dec.close()


@pytest.mark.parametrize("nq,nkv,hd", [(4, 4, 64), (8, 1, 64), (8, 2, 64), (4, 2, 128), (8, 8, 128), (8, 1, 128)],
                         ids=lambda v: str(v))
def test_head_layouts_every_kernel_variant(nq, nkv, hd):
    """MHA, GQA and MQA with head_dim 64 and 128: every (q heads per kv head,
    head_dim) variant of the kernel, small shapes, 20 steps against the oracle,
    with an odd vocabulary (a ragged last LM-head tile) and a 1-layer model."""
    cfg = dataclasses.replace(syn.TINY, name=f"heads-{nq}-{nkv}-{hd}", n_layers=1, hidden=256,
                              n_q_heads=nq, n_kv_heads=nkv, head_dim=hd, ffn=512, vocab=1000)
    seed = 7700 + nq * 100 + nkv * 10 + hd
    specs, ts = device_weights(cfg, seed, 0.1)
    host_w = syn.host_weights(cfg, seed, 0.1)
    dec = make_decoder(cfg, ts, 1, 64)
    orc = oracle.Model(cfg, host_w, 64, names(cfg))
    toks = syn.host_tokens(20, seed, cfg.vocab)
    for p, t in enumerate(toks):
        g = dec.step(torch.tensor([int(t)], dtype=torch.int32, device="cuda"),
                     torch.tensor([p], dtype=torch.int32, device="cuda")).cpu().numpy()[0]
        dec.check()
        ref = orc.decode_step(int(t), p)["logits"]
        d, cos, ok = compare_logits(g, ref)
        assert ok, (p, d, cos)
    check_counters(dec)
    dec.close()
