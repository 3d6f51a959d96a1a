"""Tensor-parallel decode on the device, the ranks emulated on one GPU.

Each rank is a full megakernel state over its shard (its heads, FFN rows and
vocabulary rows); a step runs all ranks in ONE cooperative launch, each on
n_sm/n SMs, so the ranks' reduce tasks wait on tiles of kernels that are
guaranteed to be resident.  The pushes and flags are the multi-GPU path's own
code (plain stores and system-scope release/acquire; the peers' buffers are
this GPU's memory here).  Bar: the concatenated logits shards against the
oracle of the whole model (max|diff| <= 0.05, cosine >= 0.9999, the step's
argmax equal) and against the single-GPU megakernel (max|diff| <= 2e-3: only
the order of the fp32 additions differs); counters exact after every step.
"""
import numpy as np
import pytest
import torch

import oracle
import persistent_megakernel_decode_03_b200 as mk
import synthetic as syn
from persistent_megakernel_decode_03_b200.tp import EmulatedTP
from tests.gpu_util import compare_logits, desc_kwargs, device_weights, make_decoder

pytestmark = pytest.mark.gpu

TP_TINY = syn.ModelConfig("tiny-tp-2L-h512", 2, 512, 8, 4, 128, 1024, 2048)
LLAMA8B_2L = syn.ModelConfig("llama-8b-class-2L", 2, 4096, 32, 8, 128, 14336, 128256)


def names(cfg):
    return [s.name for s in syn.tensor_specs(cfg)]


def check_rank_counters(tpd):
    for r in tpd.ranks:
        info = mk.mk_graph_get_info(r.graph)
        c, ev = mk.mk_state_read_counters(r.state, info.n_events)
        thr = mk.mk_graph_export_thresholds(r.graph)
        assert c.error == 0, (r.rank, c.error, list(c.error_info))
        assert c.done == info.n_tasks * c.epoch
        per = info.n_sm // tpd.tp
        assert c.queue_head == (info.n_tasks + per) * c.epoch
        assert ev == [t * c.epoch for t in thr]


def run_steps(cfg, tp, n_steps, seed, max_ctx=64):
    kw = desc_kwargs(cfg)
    specs, ts = device_weights(cfg, seed)
    tpd = EmulatedTP(kw, ts, tp, max_ctx)
    dec = make_decoder(cfg, ts, 1, max_ctx)
    orc = oracle.Model(cfg, syn.host_weights(cfg, seed), max_ctx, names(cfg))
    prompt = syn.host_tokens(n_steps, syn.SEED_PROMPT + seed, cfg.vocab)
    tok_d = torch.zeros(1, dtype=torch.int32, device="cuda")
    pos_d = torch.zeros(1, dtype=torch.int32, device="cuda")
    worst_single, worst_oracle = 0.0, (0.0, 1.0)
    for p in range(n_steps):
        tok = int(prompt[p])
        tok_d.fill_(tok)
        pos_d.fill_(p)
        got = tpd.step(tok_d, pos_d).cpu().numpy()
        tpd.check()
        one = dec.step(tok_d, pos_d).cpu().numpy()[0]
        dec.check()
        d1 = float(np.max(np.abs(got.astype(np.float64) - one)))
        worst_single = max(worst_single, d1)
        assert d1 <= 2e-3, f"position {p}: tensor-parallel vs single-GPU max|diff| {d1:.3g}"
        ref = orc.decode_step(tok, p)["logits"]
        d, cos, ok = compare_logits(got, ref)
        worst_oracle = (max(worst_oracle[0], d), min(worst_oracle[1], cos))
        assert ok, f"position {p}: max|diff| {d:.3g} cos {cos:.7f}"
        assert int(np.argmax(got)) == oracle.argmax(ref)
        check_rank_counters(tpd)
    print(f"{cfg.name} tp={tp}: worst vs single {worst_single:.3g}, vs oracle {worst_oracle}")
    tpd.close()
    dec.close()


@pytest.mark.parametrize("tp", [2, 4])
def test_tp_tiny_every_position_against_oracle(tp):
    run_steps(TP_TINY, tp, 24, seed=syn.SEED_WEIGHTS + 41)


@pytest.mark.parametrize("tp", [2, 4])
def test_tp_8b_shapes_two_layers(tp):
    """8B-class layer shapes (hidden 4096, 32 q / 8 KV heads, FFN 14336, vocabulary
    128256), two layers, four steps: every step against the single-GPU megakernel
    and the oracle."""
    run_steps(LLAMA8B_2L, tp, 4, seed=syn.SEED_WEIGHTS + 42, max_ctx=32)


def test_tp_steps_are_bit_identical_across_runs():
    """The reduce adds the ranks' parts in rank order: two runs of the same steps give
    the same bits, and every rank's residual stream is the same (its logits shard
    is all that differs)."""
    cfg = TP_TINY
    kw = desc_kwargs(cfg)
    _, ts = device_weights(cfg, syn.SEED_WEIGHTS + 43)
    outs = []
    for _ in range(2):
        tpd = EmulatedTP(kw, ts, 2, 32)
        tok = torch.tensor([5], dtype=torch.int32, device="cuda")
        seq = []
        for p in range(6):
            pos = torch.tensor([p], dtype=torch.int32, device="cuda")
            seq.append(tpd.step(tok, pos).cpu().clone())
        tpd.check()
        x = [mk.mk_state_read_buffer(r.state, 1, cfg.n_layers - 1, cfg.hidden) for r in tpd.ranks]
        assert np.array_equal(x[0], x[1])
        outs.append(torch.stack(seq))
        tpd.close()
    assert torch.equal(outs[0], outs[1])
