"""Host-side checks of the C-ABI library: exports, task-graph planning, events.

No compute call is made here (there is no GPU); the task graph is planned on
the host with mk_plan_taskgraph and checked symbolically.
"""
import copy
import json
import os
import re

import pytest

import persistent_megakernel_decode_03_b200 as mk
import synthetic as syn
from tests import dataflow

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
GOLDEN = os.path.join(ROOT, "tests", "golden")


def desc_of(cfg, flags=0):
    return mk.make_desc(cfg.n_layers, cfg.hidden, cfg.n_q_heads, cfg.n_kv_heads, cfg.head_dim,
                        cfg.ffn, cfg.vocab, cfg.rms_eps, cfg.rope_theta, cfg.n_experts, cfg.top_k,
                        cfg.expert_ffn, cfg.moe_renorm, flags)


def declared_functions():
    src = open(os.path.join(ROOT, "include", "mk.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(mk_[a-z0-9_]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 20
    L = mk.lib()
    for n in names:
        assert hasattr(L, n), f"{n} declared in include/mk.h but not exported"
    assert set(mk.SYMBOLS) == set(names)
    assert "sm_100a" in mk.mk_version()


def test_wave_stats_matches_the_pages_example():
    g = json.load(open(os.path.join(GOLDEN, "wave_quantization.json")))
    waves, idle = mk.mk_wave_stats(g["n_tiles"], g["n_sm"])
    assert waves == g["waves"] and idle == g["idle_sms_in_second_wave"]
    assert g["n_tiles"] - (waves - 1) * g["n_sm"] == g["tiles_in_second_wave"]


def plan(cfg, max_batch=1, max_ctx=600, n_sm=148):
    gph = mk.mk_plan_taskgraph(desc_of(cfg), max_batch, max_ctx, n_sm)
    try:
        info = mk.mk_graph_get_info(gph)
        tasks = mk.mk_graph_export_tasks(gph)
        thr = mk.mk_graph_export_thresholds(gph)
    finally:
        mk.mk_graph_destroy(gph)
    return info, tasks, thr


def shape_of(cfg, B=1):
    return dict(L=cfg.n_layers, H=cfg.hidden, nq=cfg.n_q_heads, nkv=cfg.n_kv_heads,
                hd=cfg.head_dim, B=B, E=cfg.n_experts, topk=cfg.top_k, Fe=cfg.expert_ffn,
                F=cfg.ffn, V=cfg.vocab)


@pytest.mark.parametrize("cfg", [syn.TINY, syn.LLAMA8B, syn.MOE30B, syn.TINY_MOE],
                         ids=lambda c: c.name)
def test_plan_is_topological_and_thresholds_match_signals(cfg):
    info, tasks, thr = plan(cfg, max_ctx=8192 + 300)
    assert info.n_tasks == len(tasks) and info.n_events == len(thr)
    signalled = [0] * len(thr)
    last_signal = {}
    for i, t in enumerate(tasks):
        if t.signal != mk.MK_NO_EVENT:
            last_signal[t.signal] = i
    # router tiles signal once per layer (the last tile, after the top-k)
    groups = {}
    for i, t in enumerate(tasks):
        if t.op == mk.MK_OP_ROUTER:
            groups.setdefault(("r", t.layer), t.signal)
        elif t.signal != mk.MK_NO_EVENT:
            signalled[t.signal] += 1
    for sig in groups.values():
        signalled[sig] += 1
    assert signalled == thr
    for i, t in enumerate(tasks):
        for e in (t.wait[0], t.pointer_wait):
            if e != mk.MK_NO_EVENT:
                assert last_signal[e] < i, "a wait on a later task"


def test_plan_dependency_granularity_8b():
    info, tasks, thr = plan(syn.LLAMA8B, max_ctx=551)
    attn = [t for t in tasks if t.op == mk.MK_OP_ATTN and t.layer == 3]
    # each kv head waits on its own event (only its QKV tiles), not on the whole projection
    assert len({t.wait[0] for t in attn}) == syn.LLAMA8B.n_kv_heads
    qkv_tiles = [t for t in tasks if t.op == mk.MK_OP_QKV and t.layer == 3]
    # the threshold of a kv head's event counts exactly the QKV tiles over its
    # q, k and v rows
    nq, nkv, hd = syn.LLAMA8B.n_q_heads, syn.LLAMA8B.n_kv_heads, syn.LLAMA8B.head_dim
    hpg = nq // nkv
    for t in attn:
        g = t.aux
        spans = [(g * hpg * hd, (g + 1) * hpg * hd), (nq * hd + g * hd, nq * hd + (g + 1) * hd),
                 ((nq + nkv) * hd + g * hd, (nq + nkv) * hd + (g + 1) * hd)]
        mine = [q for q in qkv_tiles if any(a <= q.r0 and q.r1 <= b for a, b in spans)]
        assert sum(q.r1 - q.r0 for q in mine) == (hpg + 2) * hd
        assert thr[t.wait[0]] == len(mine)
        assert {q.signal for q in mine} == {t.wait[0]}
    # QKV tiles are listed one KV group at a time (q heads, then k, then v rows)
    first_row = [t.r0 for t in qkv_tiles]
    group_of = [r // (hpg * hd) if r < nq * hd else (r - nq * hd) // hd % nkv for r in first_row]
    assert group_of == sorted(group_of)
    # the dense GEMV operators cover the SMs at least once
    for op in (mk.MK_OP_QKV, mk.MK_OP_OPROJ, mk.MK_OP_GATEUP, mk.MK_OP_DOWN, mk.MK_OP_LMHEAD):
        n = sum(1 for t in tasks if t.op == op and t.layer in (0, 32))
        assert n >= 148, (mk.OP_NAMES[op], n)
    assert abs(info.weight_bytes_per_step / 1e9 - 15.0099) < 0.001


def test_plan_moe_expert_down_waits_only_for_its_slot():
    info, tasks, thr = plan(syn.MOE30B, max_ctx=8192 + 300)
    l5 = [t for t in tasks if t.layer == 5]
    gu = {}
    for t in l5:
        if t.op == mk.MK_OP_EXP_GATEUP:
            gu.setdefault(t.aux, set()).add(t.signal)
    for t in l5:
        if t.op == mk.MK_OP_EXP_DOWN:
            assert gu[t.aux] == {t.wait[0]}
            assert t.pointer_wait != mk.MK_NO_EVENT
    # active bytes: attention + router + 8 experts per layer, plus LM head and norms
    assert abs(info.weight_bytes_per_step / 1e9 - 6.0837) < 0.001


@pytest.mark.parametrize("cfg,orders", [(syn.TINY, 100), (syn.TINY_MOE, 100)], ids=lambda x: str(x))
def test_random_topological_orders_give_identical_bits(cfg, orders):
    info, tasks, thr = plan(cfg, max_ctx=128, n_sm=16)
    ref = dataflow.run(tasks, thr, shape_of(cfg), seed=0)
    for s in range(1, orders):
        out = dataflow.run(tasks, thr, shape_of(cfg), seed=s)
        assert (out["logits"] == ref["logits"]).all()


def test_random_orders_on_8b_shaped_graph():
    import dataclasses
    cfg = dataclasses.replace(syn.LLAMA8B, n_layers=2, vocab=4096, name="8b-2layer")
    info, tasks, thr = plan(cfg, max_ctx=600)
    ref = dataflow.run(tasks, thr, shape_of(cfg), seed=0)
    for s in (1, 2):
        assert (dataflow.run(tasks, thr, shape_of(cfg), seed=s)["logits"] == ref["logits"]).all()


def test_long_context_graph_wide_attention_random_orders():
    """Long contexts at batch 1: one attention task per split covers every KV head,
    merge tasks per q head combine the splits, and the O-projection waits on the
    merges; the graph runs in random valid orders with identical digests, and a
    dropped merge wait is caught."""
    cfg = syn.TINY
    info, tasks, thr = plan(cfg, max_ctx=40000, n_sm=16)
    attn = [t for t in tasks if t.op == mk.MK_OP_ATTN]
    merges = [t for t in tasks if t.op == mk.MK_OP_ATTN_MERGE]
    assert attn and all(t.aux == -1 for t in attn)
    assert len(merges) == cfg.n_layers * cfg.n_q_heads
    assert len(attn) == cfg.n_layers * info.attn_splits == cfg.n_layers * 16
    ref = dataflow.run(tasks, thr, shape_of(cfg), seed=0)
    for s in range(1, 20):
        assert (dataflow.run(tasks, thr, shape_of(cfg), seed=s)["logits"] == ref["logits"]).all()
    broken = [copy.copy(t) for t in tasks]
    victim = next(i for i, t in enumerate(broken) if t.op == mk.MK_OP_ATTN_MERGE)
    broken[victim].wait[0] = mk.MK_NO_EVENT
    caught = 0
    for s in range(40):
        try:
            dataflow.run(broken, thr, shape_of(cfg), seed=s)
        except dataflow.Violation:
            caught += 1
    assert caught > 0
    # short contexts keep one task per (KV head, split)
    info2, tasks2, _ = plan(cfg, max_ctx=600, n_sm=16)
    assert all(t.aux >= 0 for t in tasks2 if t.op == mk.MK_OP_ATTN)
    assert not any(t.op == mk.MK_OP_ATTN_MERGE for t in tasks2)


def test_executor_detects_a_missing_dependency():
    """Planting a mistake in the graph (dropping one wait) must be caught."""
    info, tasks, thr = plan(syn.TINY, max_ctx=128, n_sm=16)
    broken = [t for t in tasks]
    victim = next(i for i, t in enumerate(broken) if t.op == mk.MK_OP_OPROJ)
    broken[victim].wait[0] = mk.MK_NO_EVENT
    caught = 0
    for s in range(40):
        try:
            dataflow.run(broken, thr, shape_of(syn.TINY), seed=s)
        except dataflow.Violation:
            caught += 1
    assert caught > 0


def test_invalid_shapes_are_rejected_on_the_host():
    bad = desc_of(syn.TINY)
    bad.head_dim = 96
    with pytest.raises(mk.MkError) as e:
        mk.mk_plan_taskgraph(bad, 1, 64, 148)
    assert e.value.status == mk.MK_ERR_UNSUPPORTED
    with pytest.raises(mk.MkError):
        mk.mk_plan_taskgraph(desc_of(syn.TINY), 0, 64, 148)
    with pytest.raises(mk.MkError):
        mk.mk_plan_taskgraph(desc_of(syn.TINY), 1, 0, 148)


# ---------------------------------------------------------------- batched graphs

def _tile_groups(tasks):
    """Tensor-core tiles grouped by (op, layer, first row): one producer each."""
    groups = {}
    for i, t in enumerate(tasks):
        if t.op in mk.MM_OPS:
            groups.setdefault((t.op, t.layer, t.r0), []).append(i)
    return groups


@pytest.mark.parametrize("B", [2, 4, 16, 64])
@pytest.mark.parametrize("cfg", [syn.TINY, syn.LLAMA8B], ids=lambda c: c.name)
def test_batched_plan_is_topological_and_thresholds_match_signals(cfg, B):
    info, tasks, thr = plan(cfg, max_batch=B, max_ctx=8192 + 200)
    assert info.max_batch == B
    ops = {t.op for t in tasks}
    assert ops == {mk.MK_OP_NORM, mk.MK_OP_KVAPPEND, mk.MK_OP_ATTN, *mk.MM_OPS}, \
        "batched graphs use only tensor-core tiles"
    groups = _tile_groups(tasks)
    signalled = [0] * len(thr)
    for i, t in enumerate(tasks):
        if t.op not in mk.MM_OPS and t.signal != mk.MK_NO_EVENT:
            signalled[t.signal] += 1
        assert t.pointer_wait == mk.MK_NO_EVENT
    for key, idx in groups.items():
        splits = sorted(tasks[i].b for i in idx)
        assert splits == list(range(tasks[idx[0]].aux)), f"tile {key}: splits {splits}"
        sigs = {tasks[i].signal for i in idx}
        assert len(sigs) == 1
        sig = sigs.pop()
        if sig != mk.MK_NO_EVENT:
            signalled[sig] += 1                 # the last split signals once per tile
    assert signalled == thr
    last_signal = {}
    for i, t in enumerate(tasks):
        if t.signal != mk.MK_NO_EVENT:
            last_signal[t.signal] = i
    for i, t in enumerate(tasks):
        if t.wait[0] != mk.MK_NO_EVENT:
            assert last_signal[t.wait[0]] < i, "a wait on a later task"
    # tiles: 128 output rows (64 FFN rows for gate/up: their 64 gate and 64 up rows)
    for t in tasks:
        if t.op in mk.MM_OPS:
            assert t.r1 - t.r0 <= (64 if t.op == mk.MK_OP_MM_GATEUP else 128)
    # every output row of every projection is covered exactly once per layer
    qkv_rows = (cfg.n_q_heads + 2 * cfg.n_kv_heads) * cfg.head_dim
    for op, n in ((mk.MK_OP_MM_QKV, qkv_rows), (mk.MK_OP_MM_OPROJ, cfg.hidden),
                  (mk.MK_OP_MM_GATEUP, cfg.ffn), (mk.MK_OP_MM_DOWN, cfg.hidden)):
        rows = sorted((k[2], tasks[v[0]].r1) for k, v in groups.items() if k[0] == op and k[1] == 0)
        assert rows[0][0] == 0 and rows[-1][1] == n
        assert all(a[1] == b[0] for a, b in zip(rows, rows[1:]))
    norms = [t for t in tasks if t.op == mk.MK_OP_NORM and t.layer == 0 and t.aux == 0]
    assert sorted((t.r0, t.r1) for t in norms)[-1][1] == B


def test_batched_splits_fill_the_sms_8b():
    """Tiles x splits per projection keep >= 90% of the slots of their waves busy
    (8B shapes, 148 SMs), so no projection runs a mostly idle last wave."""
    info, tasks, thr = plan(syn.LLAMA8B, max_batch=16, max_ctx=8192 + 200)
    for op in mk.MM_OPS:
        n = sum(1 for t in tasks if t.op == op and t.layer == (syn.LLAMA8B.n_layers if op == mk.MK_OP_MM_LMHEAD else 0))
        waves = -(-n // 148)
        assert n / (waves * 148) >= 0.85, f"op {op}: {n} tasks"


@pytest.mark.parametrize("B", [4, 16])
def test_batched_random_topological_orders_give_identical_bits(B):
    info, tasks, thr = plan(syn.TINY, max_batch=B, max_ctx=128, n_sm=16)
    ref = dataflow.run(tasks, thr, shape_of(syn.TINY, B), seed=0)
    for s in range(1, 40):
        out = dataflow.run(tasks, thr, shape_of(syn.TINY, B), seed=s)
        assert (out["logits"] == ref["logits"]).all()


def test_batched_executor_detects_a_missing_dependency():
    """Dropping the waits of one O-projection tile must be caught in some order."""
    info, tasks, thr = plan(syn.TINY, max_batch=4, max_ctx=128, n_sm=16)
    victim = next(t for t in tasks if t.op == mk.MK_OP_MM_OPROJ)
    for t in tasks:
        if t.op == victim.op and t.layer == victim.layer and t.r0 == victim.r0:
            t.wait[0] = mk.MK_NO_EVENT
    caught = 0
    for s in range(40):
        try:
            dataflow.run(tasks, thr, shape_of(syn.TINY, 4), seed=s)
        except dataflow.Violation:
            caught += 1
    assert caught > 0


def test_batched_plan_rejections():
    with pytest.raises(mk.MkError) as e:
        mk.mk_plan_taskgraph(desc_of(syn.TINY), 65, 64, 148)
    assert e.value.status == mk.MK_ERR_UNSUPPORTED
    with pytest.raises(mk.MkError):
        mk.mk_plan_taskgraph(desc_of(syn.TINY_MOE), 4, 64, 148)


@pytest.mark.parametrize("cfg,B", [(syn.TINY, 1), (syn.LLAMA8B, 1), (syn.TINY_MOE, 1), (syn.MOE30B, 1),
                                   (syn.TINY, 4), (syn.LLAMA8B, 64)], ids=lambda v: str(v))
def test_each_operator_and_layer_is_one_contiguous_run(cfg, B):
    """The kernel-per-operator baseline launches each maximal run of one (operator,
    layer); that is one launch per operator and layer (per norm kind) only if no
    such key appears in two runs, and every wait must point into an earlier run."""
    info, tasks, thr = plan(cfg, max_batch=B, max_ctx=2048)
    runs, seen = [], set()
    for i, t in enumerate(tasks):
        key = (t.op, t.layer, t.aux if t.op == mk.MK_OP_NORM else 0)   # a layer's two norms differ in kind
        if not runs or runs[-1][0] != key:
            assert key not in seen, f"{key} appears in two runs"
            seen.add(key)
            runs.append((key, i))
    run_of = {}
    for r, (key, start) in enumerate(runs):
        end = runs[r + 1][1] if r + 1 < len(runs) else len(tasks)
        for i in range(start, end):
            run_of[i] = r
    signal_runs = {}
    for i, t in enumerate(tasks):
        if t.signal != mk.MK_NO_EVENT:
            signal_runs.setdefault(t.signal, set()).add(run_of[i])
    for i, t in enumerate(tasks):
        for e in (t.wait[0], t.pointer_wait):
            if e != mk.MK_NO_EVENT:
                assert max(signal_runs[e]) < run_of[i], (i, e)
    if B > 1:
        assert info.n_ops == 8
