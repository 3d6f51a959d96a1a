"""The kernel-per-operator baseline (mk_decode_step_per_op) computes the same step.

Each (operator, layer) run of the task list is its own launch, so the tiles are
those of the megakernel, without the cross-operator overlap.  Its logits must
equal the megakernel's bit for bit (every task reduces in the same order) and
the oracle's within the usual tolerance, and every task must have run once.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
import persistent_megakernel_decode_03_b200 as mk
import synthetic as syn
from tests.gpu_util import compare_logits, device_weights, fill_kv_context, make_decoder
from tests.test_gpu_parity import names

pytestmark = pytest.mark.gpu


def _per_op_case(cfg, seed, B, n_steps, ctx0, label):
    specs, ts = device_weights(cfg, seed)
    max_ctx = ctx0 + n_steps + 16
    mega = make_decoder(cfg, ts, B, max_ctx)
    base = make_decoder(cfg, ts, B, max_ctx)
    for dec in (mega, base):
        for b in range(B):
            fill_kv_context(dec, cfg, b, ctx0, syn.SEED_KV + 7)
    orcs = []
    host_w = syn.host_weights(cfg, seed)
    for b in range(B):
        o = oracle.Model(cfg, host_w, max_ctx, names(cfg))
        for l in range(cfg.n_layers):
            o.k[l][:ctx0] = syn.host_kv(cfg, syn.SEED_KV + 7, l, "k", b, 0, ctx0)
            o.v[l][:ctx0] = syn.host_kv(cfg, syn.SEED_KV + 7, l, "v", b, 0, ctx0)
        orcs.append(o)
    toks = [int(t) for t in syn.host_tokens(B, syn.SEED_PROMPT + 7, cfg.vocab)]
    out = torch.empty((B, cfg.vocab), dtype=torch.float32, device="cuda")
    for i in range(n_steps):
        pos = [ctx0 + i] * B
        td = torch.tensor(toks, dtype=torch.int32, device="cuda")
        pd = torch.tensor(pos, dtype=torch.int32, device="cuda")
        g_mega = mega.step(td, pd).cpu().numpy()
        mega.check()
        n = mk.mk_decode_step_per_op(base.state, td.data_ptr(), pd.data_ptr(), B, base.kv, out.data_ptr(),
                                     base.stream())
        torch.cuda.synchronize()
        base.check()
        g_base = out.cpu().numpy()
        assert n > 4 * cfg.n_layers
        assert np.array_equal(g_base.view(np.int32), g_mega.view(np.int32)), (label, i)
        c, ev = mk.mk_state_read_counters(base.state, base.info.n_events, base.stream())
        assert c.error == 0 and c.done == base.info.n_tasks
        assert ev == mk.mk_graph_export_thresholds(base.graph)
        for b in range(B):
            ref = orcs[b].decode_step(toks[b], pos[b])["logits"]
            d, cos, ok = compare_logits(g_base[b], ref)
            assert ok, (label, i, b, d, cos)
        toks = [int(np.argmax(g_mega[b])) for b in range(B)]
    print(f"{label}: {n} launches per step, logits equal to the megakernel's")
    mega.close()
    base.close()


def test_per_op_tiny_batch1():
    _per_op_case(syn.TINY, syn.SEED_WEIGHTS + 95, 1, 4, 20, "tiny B1")


def test_per_op_tiny_batched():
    _per_op_case(syn.TINY, syn.SEED_WEIGHTS + 96, 4, 3, 30, "tiny B4")


def test_per_op_8b_shapes():
    cfg = dataclasses.replace(syn.LLAMA8B, n_layers=2)
    _per_op_case(cfg, syn.SEED_WEIGHTS + 97, 1, 2, 100, "8b-2layer B1")
