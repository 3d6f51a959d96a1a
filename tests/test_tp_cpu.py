"""Tensor parallelism on the host: shard shapes, the planned per-rank task lists,
a multi-rank execution of those lists in the kernels' claim discipline, and the
rank group's host path over world_size-2 gloo (no GPU anywhere here).

The device path (the megakernel with the ranks emulated in one launch) is
checked against the oracle in test_gpu_tp.py.
"""
import os
import socket

import numpy as np
import pytest
import torch

import persistent_megakernel_decode_03_b200 as mk
import synthetic as syn
from persistent_megakernel_decode_03_b200 import tp as mtp
from tests import dataflow
from tests.test_abi_cpu import desc_of, shape_of

TP_TINY = syn.ModelConfig("tiny-tp-2L-h512", 2, 512, 8, 4, 128, 1024, 2048)
LLAMA8B_2L = syn.ModelConfig("llama-8b-class-2L", 2, 4096, 32, 8, 128, 14336, 128256)


def rank_plan(cfg, tp, rank, max_ctx=1024, n_sm=148):
    g = mk.mk_plan_taskgraph_tp(desc_of(cfg), tp, rank, max_ctx, n_sm)
    try:
        return mk.mk_graph_get_info(g), mk.mk_graph_export_tasks(g), mk.mk_graph_export_thresholds(g)
    finally:
        mk.mk_graph_destroy(g)


def local_shape(cfg, tp):
    s = shape_of(cfg)
    s.update(nq=cfg.n_q_heads // tp, nkv=cfg.n_kv_heads // tp, F=cfg.ffn // tp, V=cfg.vocab // tp)
    return s


@pytest.mark.parametrize("cfg,tp", [(TP_TINY, 2), (TP_TINY, 4), (LLAMA8B_2L, 2), (LLAMA8B_2L, 8)],
                         ids=lambda x: getattr(x, "name", str(x)))
def test_rank_graph_structure(cfg, tp):
    """Per layer: the rank's QKV rows are its heads', each O-/down-projection tile is
    followed by one reduce task over the same rows (together covering the hidden
    size once), the reduce tasks wait on no event, and the next operator waits on
    the reduce tasks' event."""
    info, tasks, thr = rank_plan(cfg, tp, tp - 1)
    nq, nkv, hd, H = cfg.n_q_heads // tp, cfg.n_kv_heads // tp, cfg.head_dim, cfg.hidden
    by = {}
    for i, t in enumerate(tasks):
        by.setdefault((t.op, t.layer), []).append(i)
    for l in range(cfg.n_layers):
        qkv = [tasks[i] for i in by[(mk.MK_OP_QKV, l)]]
        assert sorted((t.r0, t.r1) for t in qkv)[-1][1] == (nq + 2 * nkv) * hd
        assert sum(t.r1 - t.r0 for t in qkv) == (nq + 2 * nkv) * hd
        red = [tasks[i] for i in by[(mk.MK_OP_TP_REDUCE, l)]]
        for ph, op in ((0, mk.MK_OP_OPROJ), (1, mk.MK_OP_DOWN)):
            tiles = [(tasks[i].r0, tasks[i].r1) for i in by[(op, l)]]
            mine = [(t.r0, t.r1) for t in red if t.aux == ph]
            assert tiles == mine
            assert sum(r1 - r0 for r0, r1 in tiles) == H
            assert all(tasks[i].signal == mk.MK_NO_EVENT for i in by[(op, l)])
            last_tile = max(by[(op, l)])
            assert all(i > last_tile for i in by[(mk.MK_OP_TP_REDUCE, l)] if tasks[i].aux == ph)
        assert all(t.wait[0] == mk.MK_NO_EVENT and t.wait[1] == mk.MK_NO_EVENT for t in red)
        ev0 = {t.signal for t in red if t.aux == 0}
        assert len(ev0) == 1 and thr[ev0.pop()] == sum(1 for t in red if t.aux == 0)
        assert {tasks[i].wait[0] for i in by[(mk.MK_OP_GATEUP, l)]} == {red[0].signal}
    lm = [tasks[i] for i in by[(mk.MK_OP_LMHEAD, cfg.n_layers)]]
    assert sum(t.r1 - t.r0 for t in lm) == cfg.vocab // tp
    assert info.weight_bytes_per_step < syn.weight_bytes(cfg) / tp + 2 * cfg.vocab * cfg.hidden


def test_models_that_do_not_divide_are_refused():
    with pytest.raises(mk.MkError):
        rank_plan(syn.TINY_MOE, 2, 0)                        # MoE
    with pytest.raises(mk.MkError):
        rank_plan(TP_TINY, 8, 0)                             # 4 KV heads over 8 ranks
    with pytest.raises(mk.MkError):
        rank_plan(TP_TINY, 2, 2)                             # rank out of range
    odd = syn.ModelConfig("odd-vocab", 2, 512, 8, 4, 128, 1024, 2047)
    with pytest.raises(mk.MkError):
        rank_plan(odd, 2, 0)


@pytest.mark.parametrize("cfg,tp,workers", [(TP_TINY, 2, 2), (TP_TINY, 4, 1), (LLAMA8B_2L, 4, 3)],
                         ids=lambda x: getattr(x, "name", str(x)))
def test_ranks_run_together_in_claim_order_without_deadlock(cfg, tp, workers):
    """All ranks' lists executed together with few CTAs per rank, each taking its
    rank's tasks in list order and holding up to 3 at a time: every read finds its
    data written (events and flags suffice), nothing deadlocks, and every
    interleaving gives the same digests."""
    plans = [rank_plan(cfg, tp, r) for r in range(tp)]
    tasks = [p[1] for p in plans]
    thr = [p[2] for p in plans]
    ref = dataflow.run_tp(tasks, thr, local_shape(cfg, tp), tp, seed=0, workers=workers, ahead=3)
    for s in range(1, 4):
        out = dataflow.run_tp(tasks, thr, local_shape(cfg, tp), tp, seed=s, workers=workers, ahead=3)
        assert all((a == b).all() for a, b in zip(out, ref))


def test_claim_order_executor_catches_a_broken_rank_list():
    """The executor has teeth: a reduce task moved ahead of the projection tiles it
    waits for deadlocks a one-CTA rank; a GATEUP tile that no longer waits reads the
    residual before the reduce tasks wrote it."""
    tp = 2
    plans = [rank_plan(TP_TINY, tp, r) for r in range(tp)]
    tasks = [list(p[1]) for p in plans]
    thr = [p[2] for p in plans]
    shape = local_shape(TP_TINY, tp)
    # (1) rank 1: the first reduce task before the first O-projection tile
    t1 = list(tasks[1])
    i_red = next(i for i, t in enumerate(t1) if t.op == mk.MK_OP_TP_REDUCE)
    i_op = next(i for i, t in enumerate(t1) if t.op == mk.MK_OP_OPROJ)
    t1.insert(i_op, t1.pop(i_red))
    with pytest.raises(dataflow.Violation, match="deadlock"):
        dataflow.run_tp([tasks[0], t1], thr, shape, tp, seed=0, workers=1, ahead=1)
    # (2) rank 0: a GATEUP tile without its wait
    import copy
    t0 = [copy.copy(t) for t in tasks[0]]
    j = next(i for i, t in enumerate(t0) if t.op == mk.MK_OP_GATEUP)
    t0[j].wait[0] = mk.MK_NO_EVENT
    hit = False
    for s in range(20):
        try:
            dataflow.run_tp([t0, tasks[1]], thr, shape, tp, seed=s, workers=8, ahead=4)
        except dataflow.Violation as e:
            assert "unwritten" in str(e)
            hit = True
            break
    assert hit


def test_shards_reassemble_the_model():
    """Concatenating the ranks' shards gives back every weight (rows of wq/wk/wv,
    gate/up and the LM head; columns of wo and down); the embedding and the norms
    are whole on every rank."""
    cfg = TP_TINY
    kw = dict(n_layers=cfg.n_layers, hidden=cfg.hidden, n_q_heads=cfg.n_q_heads, n_kv_heads=cfg.n_kv_heads,
              head_dim=cfg.head_dim, ffn=cfg.ffn, vocab=cfg.vocab)
    specs = syn.tensor_specs(cfg)
    full = [torch.from_numpy(syn.host_tensor(s, 7).view(np.int16)).view(torch.bfloat16).reshape(s.shape)
            for s in specs]
    for tp in (2, 4):
        shards = [mtp.shard_weights(kw, full, tp, r) for r in range(tp)]
        for k, s in enumerate(specs):
            parts = [sh[k] for sh in shards]
            name = s.name.split(".")[-1]
            if name in ("wo", "w_down"):
                back = torch.cat(parts, dim=1)
            elif name in ("wq", "wk", "wv", "w_gate", "w_up", "lm_head"):
                back = torch.cat(parts, dim=0)
            else:
                assert all(torch.equal(p, full[k]) for p in parts)
                continue
            assert torch.equal(back, full[k]), s.name
        # rank r's q heads are exactly the q heads of its KV heads (grouped-query layout)
        hpg = cfg.n_q_heads // cfg.n_kv_heads
        for r in range(tp):
            kvh = list(mtp.kv_heads_of(kw, tp, r))
            assert kvh[0] * hpg * cfg.head_dim == r * (cfg.n_q_heads // tp) * cfg.head_dim


# ----------------------------------------------------------------------------- gloo, world size 2

def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _gloo_rank(rank: int, world: int, port: int, out_dir: str) -> None:
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=__import__("datetime").timedelta(seconds=60))
    try:
        cfg = TP_TINY
        kw = dict(n_layers=cfg.n_layers, hidden=cfg.hidden, n_q_heads=cfg.n_q_heads, n_kv_heads=cfg.n_kv_heads,
                  head_dim=cfg.head_dim, ffn=cfg.ffn, vocab=cfg.vocab)
        # (1) the IPC-handle exchange the one-process-per-GPU path uses (fake handle bytes)
        mine = bytes([rank + 1]) * mk.MK_TP_IPC_HANDLE_BYTES
        got = mtp.exchange_handles(mine)
        assert got == [bytes([q + 1]) * mk.MK_TP_IPC_HANDLE_BYTES for q in range(world)]
        # (2) this rank's host plan; rank 0 runs all ranks' lists together
        info, tasks, thr = rank_plan(cfg, world, rank)
        rows = [(t.op, t.layer, t.b, t.aux, t.r0, t.r1, tuple(t.wait), t.signal) for t in tasks]
        every = [None] * world
        dist.all_gather_object(every, (rows, list(thr)))
        # (3) the all-reduce the reduce tasks compute: the ranks' partial O-projections
        # of one layer (their shards of wo times their heads' attention output) summed
        # over the group equal the whole product
        specs = syn.tensor_specs(cfg)
        full = [torch.from_numpy(syn.host_tensor(s, 11).view(np.int16)).view(torch.bfloat16).reshape(s.shape)
                for s in specs]
        shard = mtp.shard_weights(kw, full, world, rank)
        wo_full = syn.bf16_bits_to_f32(syn.host_tensor(specs[5], 11)).reshape(specs[5].shape).astype(np.float64)
        o = np.random.default_rng(3).standard_normal(cfg.n_q_heads * cfg.head_dim)
        qs = cfg.n_q_heads // world * cfg.head_dim
        wo_mine = shard[5].float().numpy().astype(np.float64)
        part = torch.from_numpy(wo_mine @ o[rank * qs:(rank + 1) * qs])
        dist.all_reduce(part)
        err = float(np.max(np.abs(part.numpy() - wo_full @ o)))
        np.save(os.path.join(out_dir, f"rank{rank}.npy"), np.array([err]))
        if rank == 0:
            import pickle
            with open(os.path.join(out_dir, "plans.pkl"), "wb") as f:
                pickle.dump(every, f)
    finally:
        dist.destroy_process_group()


class _T:
    def __init__(self, row):
        self.op, self.layer, self.b, self.aux, self.r0, self.r1, w, self.signal = row
        self.wait = list(w)
        self.pointer_wait = mk.MK_NO_EVENT


def test_gloo_world_size_2_rank_group_host_path(tmp_path):
    import pickle
    import torch.multiprocessing as tmp
    world = 2
    tmp.spawn(_gloo_rank, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    for r in range(world):
        assert float(np.load(tmp_path / f"rank{r}.npy")[0]) < 1e-12
    every = pickle.load(open(tmp_path / "plans.pkl", "rb"))
    tasks = [[_T(row) for row in rows] for rows, _ in every]
    thr = [t for _, t in every]
    out = dataflow.run_tp(tasks, thr, local_shape(TP_TINY, world), world, seed=5, workers=2, ahead=2)
    assert len(out) == world and all(o.size == TP_TINY.vocab // world for o in out)
