"""Parity of batched decode steps (tensor-core projection tiles) with the oracle.

A batched step is B independent single-sequence steps that share the weights, so
sequence b's logits must equal the oracle run on sequence b alone.  The contexts
are ragged: each sequence has its own cached length.  They live in one pool of
16-token pages, dealt to the sequences in a shuffled order, as under continuous
batching (Cohere page, section "Folyamatos batchkezelés, paged attention").
Tolerances are those of the batch-1 path: max |logit diff| <= 0.05 and cosine
>= 0.9999 per sequence and step.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import persistent_megakernel_decode_03_b200 as mk
import synthetic as syn
from tests.gpu_util import compare_logits, device_weights, fill_kv_context, fill_oracle_kv, make_decoder
from tests.test_gpu_parity import check_counters, names

pytestmark = pytest.mark.gpu


def _ragged_lengths(B, lo, hi, seed):
    rng = np.random.default_rng(seed)
    return [int(x) for x in rng.integers(lo, hi + 1, size=B)]


def _run_batched(cfg, seed, B, lens, n_steps, seed_off, greedy=False, batch=None, label=""):
    """Builds a batched decoder over shuffled pages, fills each sequence's context,
    and compares n_steps steps of every active sequence with its own oracle."""
    batch = B if batch is None else batch
    max_ctx = max(lens) + n_steps + 16
    max_pages = (max_ctx + 15) // 16
    total = B * max_pages
    perm = torch.tensor(syn.page_permutation(total, syn.SEED_KV + seed_off), dtype=torch.int32,
                        device="cuda").view(B, max_pages)
    specs, ts = device_weights(cfg, seed)
    dec = make_decoder(cfg, ts, B, max_ctx, page_table=perm, n_pages=total)
    host_w = syn.host_weights(cfg, seed)
    orcs = []
    for b in range(batch):
        fill_kv_context(dec, cfg, b, lens[b], syn.SEED_KV + seed_off)
        o = oracle.Model(cfg, host_w, max_ctx, names(cfg))
        fill_oracle_kv(o, cfg, b, lens[b], syn.SEED_KV + seed_off)
        orcs.append(o)
    toks = [int(t) for t in syn.host_tokens(batch, syn.SEED_PROMPT + seed_off, cfg.vocab)]
    pos = list(lens[:batch])
    worst = (0.0, 1.0)
    for step in range(n_steps):
        g = dec.step(torch.tensor(toks, dtype=torch.int32, device="cuda"),
                     torch.tensor(pos, dtype=torch.int32, device="cuda")).cpu().numpy()
        dec.check()
        nxt = []
        for b in range(batch):
            ref = orcs[b].decode_step(toks[b], pos[b])["logits"]
            d, cos, ok = compare_logits(g[b], ref)
            worst = (max(worst[0], d), min(worst[1], cos))
            assert ok, (label, step, b, pos[b], d, cos)
            if greedy:
                assert int(np.argmax(g[b])) == int(np.argmax(ref)), (label, step, b)
            nxt.append(int(np.argmax(ref)))
        check_counters(dec)
        toks = nxt
        pos = [p + 1 for p in pos]
    print(f"{label}: B={B} batch={batch} steps={n_steps} worst max|diff| {worst[0]:.3g} cos {worst[1]:.8f}")
    dec.close()


@pytest.mark.parametrize("B,steps", [(2, 16), (4, 16), (16, 6), (64, 3)], ids=lambda v: str(v))
def test_tiny_batched_parity_and_greedy(B, steps):
    """Tiny model, ragged contexts of 1..200 tokens: every sequence's logits and
    greedy tokens over the steps (N = 16 for B <= 16, 64 for B = 64; the tiny
    shapes give ragged tiles: 688 FFN rows, K = 688 for the down projection)."""
    lens = _ragged_lengths(B, 1, 200, 4100 + B)
    _run_batched(syn.TINY, syn.SEED_WEIGHTS + 40 + B, B, lens, steps, 40 + B, greedy=True,
                 label="tiny")


def test_partial_batch_leaves_inactive_rows_out():
    """A graph for 8 sequences stepping 5 of them: the 5 match the oracle and the
    counters stay exact (rows 5..7 are computed as zeros and never stored)."""
    lens = _ragged_lengths(8, 3, 120, 4200)
    _run_batched(syn.TINY, syn.SEED_WEIGHTS + 50, 8, lens, 4, 50, batch=5, label="partial")


def test_batched_repeat_runs_are_bit_identical():
    """The splits of a tile are added in split order by whichever CTA arrives last,
    so two runs of the same steps give the same bits."""
    cfg = syn.TINY
    seed = syn.SEED_WEIGHTS + 60
    B = 16
    lens = _ragged_lengths(B, 1, 150, 4300)
    outs = []
    for _ in range(2):
        specs, ts = device_weights(cfg, seed)
        dec = make_decoder(cfg, ts, B, 256)
        for b in range(B):
            fill_kv_context(dec, cfg, b, lens[b], syn.SEED_KV + 60)
        toks = torch.tensor(syn.host_tokens(B, syn.SEED_PROMPT + 60, cfg.vocab), dtype=torch.int32,
                            device="cuda")
        pos = torch.tensor(lens, dtype=torch.int32, device="cuda")
        res = []
        for _ in range(3):
            res.append(dec.step(toks, pos).clone())
            dec.check()
            pos = pos + 1
        outs.append(torch.stack(res).cpu())
        dec.close()
    assert torch.equal(outs[0].view(torch.int32), outs[1].view(torch.int32))


@pytest.mark.parametrize("B", [16, 64])
def test_8b_shapes_batched_ragged_contexts(B):
    """8B-class shapes (2 layers; full width, full 128256-row LM head) with
    contexts drawn uniformly from 512..8192 tokens in shuffled pages: the
    continuous-batching workload's tiles and split counts, one step."""
    cfg = dataclasses.replace(syn.LLAMA8B, n_layers=2)
    lens = _ragged_lengths(B, 512, 8192, 4400 + B)
    _run_batched(cfg, syn.SEED_WEIGHTS + 70, B, lens, 1, 70 + B, label="8b-2layer")


def test_8b_full_size_batch16():
    """All 32 layers of the 8B-class model at batch 16 over ragged 512..8192-token
    contexts, one step: every logit of every sequence against the oracle."""
    cfg = syn.LLAMA8B
    lens = _ragged_lengths(16, 512, 8192, 4500)
    _run_batched(cfg, syn.SEED_WEIGHTS + 80, 16, lens, 1, 80, label="8b-full")


@pytest.mark.parametrize("nq,nkv,hd", [(8, 1, 64), (4, 2, 128), (8, 8, 128)], ids=lambda v: str(v))
def test_batched_head_layouts(nq, nkv, hd):
    """Batched tiles with other head layouts: a K/V projection narrower than one
    128-row tile (MQA, head_dim 64), and an odd vocabulary (ragged last LM tile)."""
    cfg = dataclasses.replace(syn.TINY, name=f"bheads-{nq}-{nkv}-{hd}", n_layers=1, hidden=256,
                              n_q_heads=nq, n_kv_heads=nkv, head_dim=hd, ffn=512, vocab=1000)
    lens = _ragged_lengths(4, 1, 90, 4600 + nq + nkv + hd)
    _run_batched(cfg, 8800 + nq * 100 + nkv * 10 + hd, 4, lens, 5, 90 + nkv, greedy=True,
                 label=f"heads {nq}/{nkv}/{hd}")


# ---------------------------------------------------------------- batched prefill

def _prefill_case(cfg, seed, max_batch, n_prompt, n_decode, seed_off, label, greedy=True):
    """Prompt through a batched graph (up to max_batch tokens per launch), then
    decode steps of that sequence alone; every logit against the oracle run
    token by token, and the cached K bits of the prompt against the oracle's."""
    max_ctx = n_prompt + n_decode + 8
    specs, ts = device_weights(cfg, seed)
    dec = make_decoder(cfg, ts, max_batch, max_ctx)
    prompt = [int(t) for t in syn.host_tokens(n_prompt, syn.SEED_PROMPT + seed_off, cfg.vocab)]
    last = dec.prefill(torch.tensor(prompt, dtype=torch.int32, device="cuda")).cpu().numpy()
    dec.check()
    check_counters(dec)
    orc = oracle.Model(cfg, syn.host_weights(cfg, seed), max_ctx, names(cfg))
    for p, t in enumerate(prompt):
        ref = orc.decode_step(t, p)["logits"]
    d, cos, ok = compare_logits(last, ref)
    print(f"{label}: prefill of {n_prompt} tokens in launches of {max_batch}: max|diff| {d:.3g} cos {cos:.8f}")
    assert ok, (d, cos)
    # K of every prompt position in layer 0, sequence 0's pages: each element within one
    # bf16 step of its own value (2^-7 relative), plus 2^-10 of the row's scale for
    # elements near zero (the projection accumulates in another order than the
    # oracle's double, so a value may round to its neighbour); a misplaced row would be
    # off by the scale itself
    k = dec.k_pages[0].float().cpu().numpy()
    rows = dec.page_table[0].cpu().numpy()
    worst = 0.0
    for p in range(n_prompt):
        got = k[rows[p // 16], :, p % 16, :]
        ref_k = oracle.bf16_to_f64(orc.k[0][p])
        scale = float(np.sqrt(np.mean(ref_k ** 2)))
        bound = 2.0 ** -7 * np.abs(ref_k) + 2.0 ** -10 * scale
        ratio = float(np.max(np.abs(got - ref_k) / bound))
        worst = max(worst, ratio)
        assert ratio <= 1.0, (p, ratio)
    print(f"{label}: cached K of the prompt within {worst:.3g} of the bound")
    tok = int(np.argmax(ref))
    for i in range(n_decode):
        p = n_prompt + i
        g = dec.step(torch.tensor([tok], dtype=torch.int32, device="cuda"),
                     torch.tensor([p], dtype=torch.int32, device="cuda")).cpu().numpy()[0]
        dec.check()
        ref = orc.decode_step(tok, p)["logits"]
        d, cos, ok = compare_logits(g, ref)
        assert ok, (label, p, d, cos)
        if greedy:
            assert int(np.argmax(g)) == int(np.argmax(ref)), (label, p)
        tok = int(np.argmax(ref))
    check_counters(dec)
    dec.close()


@pytest.mark.parametrize("max_batch", [4, 16, 64], ids=lambda v: f"B{v}")
def test_tiny_batched_prefill_then_decode(max_batch):
    """The 39-token prompt of the tiny config as batch rows (launches of 4, 16 or
    64 tokens: 10, 3 or 1 launches), then 16 greedy decode steps."""
    _prefill_case(syn.TINY, syn.SEED_WEIGHTS + 90, max_batch, 39, 16, 90, f"tiny B{max_batch}")


def test_8b_shapes_batched_prefill():
    """8B-class shapes (2 layers): a 100-token prompt in launches of 64 and 36
    rows, then 2 decode steps."""
    cfg = dataclasses.replace(syn.LLAMA8B, n_layers=2)
    _prefill_case(cfg, syn.SEED_WEIGHTS + 91, 64, 100, 2, 91, "8b-2layer", greedy=False)


def test_prefill_into_one_slot_then_mixed_batch():
    """mk_prefill_seq into sequence slot 2 of a 4-row graph, then one batched step in
    which slot 2 continues its prompt and slots 0, 1, 3 start at position 0."""
    cfg = syn.TINY
    seed = syn.SEED_WEIGHTS + 92
    specs, ts = device_weights(cfg, seed)
    dec = make_decoder(cfg, ts, 4, 64)
    prompt = [int(t) for t in syn.host_tokens(20, syn.SEED_PROMPT + 92, cfg.vocab)]
    kv = mk.make_kv(dec.k_pages.data_ptr(), dec.v_pages.data_ptr(), dec.page_table.data_ptr(), dec.n_pages,
                    dec.max_pages)
    out = torch.empty(cfg.vocab, dtype=torch.float32, device="cuda")
    toks_d = torch.tensor(prompt, dtype=torch.int32, device="cuda")
    mk.mk_prefill_seq(dec.state, toks_d.data_ptr(), len(prompt), 0, 2, kv, out.data_ptr(), dec.stream())
    dec.check()
    host_w = syn.host_weights(cfg, seed)
    orcs = [oracle.Model(cfg, host_w, 64, names(cfg)) for _ in range(4)]
    for p, t in enumerate(prompt):
        ref = orcs[2].decode_step(t, p)["logits"]
    d, cos, ok = compare_logits(out.cpu().numpy(), ref)
    assert ok, (d, cos)
    step_toks = [3, 5, int(np.argmax(ref)), 7]
    pos = [0, 0, len(prompt), 0]
    g = dec.step(torch.tensor(step_toks, dtype=torch.int32, device="cuda"),
                 torch.tensor(pos, dtype=torch.int32, device="cuda")).cpu().numpy()
    dec.check()
    for b in range(4):
        ref = orcs[b].decode_step(step_toks[b], pos[b])["logits"]
        d, cos, ok = compare_logits(g[b], ref)
        assert ok, (b, d, cos)
    check_counters(dec)
    dec.close()
