"""Host-side checks of the C-ABI library: exports, task-graph planning, events.

No compute call is made here (there is no GPU); the task graph is planned on
the host with mk_plan_taskgraph and checked symbolically.
"""
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
