"""CPU executor of an exported task graph, in random valid orders (test support).

Each task is executed symbolically: it reads the tensor elements the kernel's
tile for that task reads and writes a 64-bit digest of (task, inputs) to the
elements it writes.  A task may run only when its events have reached their
thresholds (the kernel's rule).  Reading an element nobody has written yet,
or writing one twice, is a violation.  If the events are sufficient for every
read, every valid order produces the same final digests ("identical bits").

Read/write sets per operator mirror the megakernel's tiles:
  qkv      reads x_in[l] (all)                 writes qkv[l][rows]
  attn     reads qkv[l] rows of its kv head    writes part[l][b,g,s]
  oproj    reads part[l] (all), x_in[l][rows]  writes x_mid[l][rows] (merging the splits)
  gateup   reads x_mid[l] (all)                writes act[l][rows]
  down     reads act[l] (all), x_mid[l][rows]  writes x_in[l+1][rows]
  router   reads x_mid[l] (all)                writes rlog[l][rows]; the last tile reads
           rlog[l] (all) and writes sel[l]
  exp_gu   reads sel[l], x_mid[l] (all)        writes acte[l][k][rows]
  exp_dn   reads sel[l], acte[l][k] (all)      writes ypart[l][k][rows]
  lmhead   reads x_in[L] (all)                 writes logits[rows]
Long-context batch-1 graphs ("wide" attention, exported with aux = -1):
  attn     reads qkv[l] (all)                  writes part[l][b, g, s] for every kv head g
  attn_merge  q head r0: reads part[l][b, its kv head, all splits]   writes ao[l][r0]
  oproj    then reads ao[l] (all) instead of the partials
For MoE models x_in[l+1][i] is x_mid[l][i] combined with ypart[l][k][i] for all k
and the routing weights sel[l].

Tensor-parallel batch-1 graphs (run_tp: every rank's list, each rank its own tensors):
  oproj    reads part[l] (all)                 writes recv[q][r, l, 0][rows] on EVERY rank q
           (r = this rank) and raises flag[q][l, 0, rows] there
  down     reads act[l] (all)                  the same with phase 1
  tp_reduce  (aux = phase) runs once flag[r][l, aux, rows] == tp; reads recv[r][q, l, aux][rows]
           for every q and x_in[l][rows] (aux 0) or x_mid[l][rows] (aux 1); writes x_mid[l][rows]
           (aux 0) or x_in[l+1][rows] (aux 1)

Batched graphs (tensor-core tiles; x_in, x_mid hold B rows of H):
  norm     reads its batch rows [r0, r1) of x_in[l] (aux 0), x_mid[l] (aux 1)
           or x_in[L] (aux 2)              writes those rows of opq[l] / opf[l] / opl
  mm_*     split b of aux splits writes its partial; the last split to run reads
           every partial and the tile's inputs, writes the rows, and signals:
  mm_qkv   reads opq[l] (all)                  writes qkv[l][rows]
  mm_oproj reads part[l] (all), x_in[l][b, rows] for every b   writes x_mid[l][b, rows]
  mm_gu    reads opf[l] (all)                  writes act[l][rows]
  mm_down  reads act[l] (all), x_mid[l][b, rows]   writes x_in[l+1][b, rows]
  mm_lm    reads opl (all)                     writes logits[rows]
  kvappend reads qkv[l] (all)                  writes kv[l][its batch rows]; the layer's
           attention tasks then also read kv[l] (all rows)
"""
from __future__ import annotations

import random
from collections import defaultdict
from typing import Dict, List

import numpy as np

OP = {1: "qkv", 2: "attn", 3: "oproj", 4: "gateup", 5: "down", 6: "lmhead", 7: "router",
      8: "exp_gu", 9: "exp_dn", 10: "norm", 11: "mm_qkv", 12: "mm_oproj", 13: "mm_gu", 14: "mm_down",
      15: "mm_lm", 16: "kvappend", 17: "attn_merge", 18: "tp_reduce"}
NO_EVENT = 0xFFFFFFFF
M64 = (1 << 64) - 1


class Violation(AssertionError):
    pass


def _mix(a: int) -> int:
    a = (a + 0x9E3779B97F4A7C15) & M64
    a = ((a ^ (a >> 30)) * 0xBF58476D1CE4E5B9) & M64
    a = ((a ^ (a >> 27)) * 0x94D049BB133111EB) & M64
    return a ^ (a >> 31)


class Tensor:
    def __init__(self, n: int, ready: bool = False):
        self.val = np.zeros(n, dtype=np.uint64)
        self.ok = np.full(n, ready, dtype=bool)
        if ready:
            self.val[:] = np.arange(n, dtype=np.uint64) * np.uint64(2654435761)

    def read(self, lo: int, hi: int, who: str) -> int:
        if not self.ok[lo:hi].all():
            raise Violation(f"{who} read unwritten elements [{lo},{hi})")
        return int(self.val[lo:hi].sum(dtype=np.uint64))

    def write(self, lo: int, hi: int, digest: int, who: str) -> None:
        if self.ok[lo:hi].any():
            raise Violation(f"{who} wrote [{lo},{hi}) twice")
        self.ok[lo:hi] = True
        self.val[lo:hi] = (np.arange(lo, hi, dtype=np.uint64) * np.uint64(0x100000001B3)) ^ np.uint64(digest)


def run(tasks, thr: List[int], shape: dict, seed: int) -> Dict[str, np.ndarray]:
    """Executes all tasks once in a random valid order; returns final digests."""
    L, H, nq, nkv, hd = shape["L"], shape["H"], shape["nq"], shape["nkv"], shape["hd"]
    B, E, K, Fe, F, V = shape["B"], shape["E"], shape["topk"], shape["Fe"], shape["F"], shape["V"]
    hpg = nq // nkv
    qkv_rows = (nq + 2 * nkv) * hd
    moe = E > 0
    T: Dict[tuple, Tensor] = {}

    def t(*key) -> Tensor:
        return T[key]

    T[("x_in", 0)] = Tensor(B * H, ready=True)      # embedding rows: inputs of the step
    for l in range(L):
        T[("qkv", l)] = Tensor(qkv_rows)
        T[("part", l)] = Tensor(B * nkv * 4096)
        T[("ao", l)] = Tensor(nq)
        T[("x_mid", l)] = Tensor(B * H)
        if moe:
            T[("rlog", l)] = Tensor(E)
            T[("sel", l)] = Tensor(B * K)
            for k in range(K):
                T[("acte", l, k)] = Tensor(B * Fe)
                T[("ypart", l, k)] = Tensor(B * H)
        else:
            T[("act", l)] = Tensor(F)
            T[("x_in", l + 1)] = Tensor(B * H)
        T[("opq", l)] = Tensor(B * H)
        T[("opf", l)] = Tensor(B * H)
    T[("opl",)] = Tensor(B * H)
    has_append = any(tk.op == 16 for tk in tasks)
    for l in range(L):
        T[("kv", l)] = Tensor(B)
    T[("logits",)] = Tensor(V)
    mm_arrivals = defaultdict(int)
    wide = any(tk.op == 17 for tk in tasks)
    tasks_split = {tk.layer: tk.r1 for tk in tasks if tk.op == 2}
    router_arr = defaultdict(int)
    n_router = defaultdict(int)
    for tk in tasks:
        if tk.op == 7:
            n_router[tk.layer] += 1

    def read_xin(l: int, lo: int, hi: int, who: str) -> int:
        if l == 0 or not moe:
            return t("x_in", l).read(lo, hi, who)
        d = t("x_mid", l - 1).read(lo, hi, who) + t("sel", l - 1).read(0, B * K, who)
        for k in range(K):
            d += t("ypart", l - 1, k).read(lo, hi, who)
        return d & M64

    counters = [0] * len(thr)
    pending = [0] * len(tasks)
    waiters = defaultdict(list)
    for i, tk in enumerate(tasks):
        evs = {e for e in (tk.wait[0], tk.wait[1]) if e != NO_EVENT}
        pad = tk.pointer_wait
        if pad != NO_EVENT:
            evs.add(pad)
        pending[i] = len(evs)
        for e in evs:
            waiters[e].append(i)
    rng = random.Random(seed)
    ready = [i for i in range(len(tasks)) if pending[i] == 0]
    done = 0

    def signal(e: int) -> None:
        if e == NO_EVENT:
            return
        counters[e] += 1
        if counters[e] == thr[e]:
            for w in waiters[e]:
                pending[w] -= 1
                if pending[w] == 0:
                    ready.append(w)
        if counters[e] > thr[e]:
            raise Violation(f"event {e} signalled beyond its threshold")

    while ready:
        j = rng.randrange(len(ready))
        ready[j], ready[-1] = ready[-1], ready[j]
        i = ready.pop()
        tk = tasks[i]
        op, l, r0, r1 = OP[tk.op], tk.layer, tk.r0, tk.r1
        who = f"task {i} ({op} l{l} b{tk.b} aux{tk.aux} {r0}:{r1})"
        base = _mix(i + 1)
        if op == "qkv":
            d = read_xin(l, 0, H, who)
            t("qkv", l).write(r0, r1, _mix(base ^ d), who)
            signal(tk.signal)
        elif op == "attn" and tk.aux == -1:               # every kv head of split r0
            b = tk.b
            d = t("qkv", l).read(0, qkv_rows, who)
            for g in range(nkv):
                idx = (b * nkv + g) * 4096 + r0
                t("part", l).write(idx, idx + 1, _mix(base ^ d ^ g), who)
            signal(tk.signal)
        elif op == "attn_merge":
            g, b = r0 // hpg, tk.b
            lo = (b * nkv + g) * 4096
            d = t("part", l).read(lo, lo + tasks_split[l], who)
            t("ao", l).write(r0, r1, _mix(base ^ d), who)
            signal(tk.signal)
        elif op == "attn":
            g, b = tk.aux, tk.b
            qkv = t("qkv", l)
            d = qkv.read(g * hpg * hd, (g + 1) * hpg * hd, who)
            d += qkv.read(nq * hd + g * hd, nq * hd + (g + 1) * hd, who)
            d += qkv.read((nq + nkv) * hd + g * hd, (nq + nkv) * hd + (g + 1) * hd, who)
            if has_append:
                d += t("kv", l).read(0, B, who)
            idx = (b * nkv + g) * 4096 + r0            # r0 = split index
            t("part", l).write(idx, idx + 1, _mix(base ^ (d & M64)), who)
            signal(tk.signal)
        elif op == "oproj":
            n_split = tasks_split[l]
            d = read_xin(l, r0, r1, who)
            if wide:
                d += t("ao", l).read(0, nq, who)
            else:
                for bb in range(B):
                    for gg in range(nkv):
                        lo = (bb * nkv + gg) * 4096
                        d += t("part", l).read(lo, lo + n_split, who)
            t("x_mid", l).write(r0, r1, _mix(base ^ (d & M64)), who)
            signal(tk.signal)
        elif op == "gateup":
            d = t("x_mid", l).read(0, B * H, who)
            t("act", l).write(r0, r1, _mix(base ^ d), who)
            signal(tk.signal)
        elif op == "down":
            d = t("act", l).read(0, F, who) + t("x_mid", l).read(r0, r1, who)
            t("x_in", l + 1).write(r0, r1, _mix(base ^ (d & M64)), who)
            signal(tk.signal)
        elif op == "router":
            d = t("x_mid", l).read(0, B * H, who)
            t("rlog", l).write(r0, r1, _mix(base ^ d), who)
            router_arr[l] += 1
            if router_arr[l] == n_router[l]:
                d2 = t("rlog", l).read(0, E, who)
                t("sel", l).write(0, B * K, _mix(d2), who)
                signal(tk.signal)
        elif op == "exp_gu":
            d = t("sel", l).read(0, B * K, who) + t("x_mid", l).read(0, B * H, who)
            lo = tk.b * Fe
            t("acte", l, tk.aux).write(lo + r0, lo + r1, _mix(base ^ (d & M64)), who)
            signal(tk.signal)
        elif op == "exp_dn":
            d = t("sel", l).read(0, B * K, who) + t("acte", l, tk.aux).read(tk.b * Fe, (tk.b + 1) * Fe, who)
            lo = tk.b * H
            t("ypart", l, tk.aux).write(lo + r0, lo + r1, _mix(base ^ (d & M64)), who)
            signal(tk.signal)
        elif op == "lmhead":
            d = read_xin(L, 0, H, who)
            t("logits").write(r0, r1, _mix(base ^ d), who)
            signal(tk.signal)
        elif op == "kvappend":
            d = t("qkv", l).read(0, qkv_rows, who)
            t("kv", l).write(r0, r1, _mix(base ^ d), who)
            signal(tk.signal)
        elif op == "norm":
            src = {0: ("x_in", l), 1: ("x_mid", l), 2: ("x_in", L)}[tk.aux]
            dst = {0: ("opq", l), 1: ("opf", l), 2: ("opl",)}[tk.aux]
            d = T[src].read(r0 * H, r1 * H, who)
            T[dst].write(r0 * H, r1 * H, _mix(base ^ d), who)
            signal(tk.signal)
        elif op.startswith("mm_"):
            key = (op, l, r0)
            if ("mmp",) + key not in T:
                T[("mmp",) + key] = Tensor(tk.aux)
            T[("mmp",) + key].write(tk.b, tk.b + 1, _mix(base), who)
            mm_arrivals[key] += 1
            if mm_arrivals[key] == tk.aux:               # the last split finishes the tile
                d = T[("mmp",) + key].read(0, tk.aux, who)
                if op == "mm_qkv":
                    d += t("opq", l).read(0, B * H, who)
                    t("qkv", l).write(r0, r1, _mix(d & M64), who)
                elif op == "mm_oproj":
                    for bb in range(B):
                        for gg in range(nkv):
                            lo = (bb * nkv + gg) * 4096
                            d += t("part", l).read(lo, lo + tasks_split[l], who)
                    for bb in range(B):
                        dd = (d + t("x_in", l).read(bb * H + r0, bb * H + r1, who)) & M64
                        t("x_mid", l).write(bb * H + r0, bb * H + r1, _mix(dd), who)
                elif op == "mm_gu":
                    d += t("opf", l).read(0, B * H, who)
                    t("act", l).write(r0, r1, _mix(d & M64), who)
                elif op == "mm_down":
                    d += t("act", l).read(0, F, who)
                    for bb in range(B):
                        dd = (d + t("x_mid", l).read(bb * H + r0, bb * H + r1, who)) & M64
                        t("x_in", l + 1).write(bb * H + r0, bb * H + r1, _mix(dd), who)
                else:
                    d += t("opl").read(0, B * H, who)
                    t("logits").write(r0, r1, _mix(d & M64), who)
                signal(tk.signal)
        else:
            raise Violation(f"unknown op {tk.op}")
        done += 1
    if done != len(tasks):
        raise Violation(f"only {done} of {len(tasks)} tasks could run (deadlock)")
    for e, (c, th) in enumerate(zip(counters, thr)):
        if c != th:
            raise Violation(f"event {e}: counter {c} != threshold {th}")
    if not T[("logits",)].ok.all():
        raise Violation("logits not fully written")
    return {"logits": T[("logits",)].val.copy()}


def run_tp(rank_tasks, rank_thr, shape: dict, tp: int, seed: int, workers: int = 4, ahead: int = 2):
    """Executes the ranks' task lists together, the way the kernels claim them: each
    rank has `workers` CTAs taking tasks from its own list IN ORDER, each holding up
    to `ahead` claimed tasks and running only the oldest (a CTA finishes its tasks
    in claim order).  Every step picks a random (rank, CTA) that can move.  Raises
    Violation on a read of unwritten data, a double write, or a deadlock (tasks
    left, no CTA can move).  Returns each rank's logits digests."""
    L, H, nq, nkv, hd = shape["L"], shape["H"], shape["nq"], shape["nkv"], shape["hd"]
    F, V = shape["F"], shape["V"]
    hpg = nq // nkv
    qkv_rows = (nq + 2 * nkv) * hd
    rng = random.Random(seed)
    T = []
    for r in range(tp):
        d = {("x_in", 0): Tensor(H, ready=True)}
        for l in range(L):
            d[("qkv", l)] = Tensor(qkv_rows)
            d[("part", l)] = Tensor(nkv * 4096)
            d[("x_mid", l)] = Tensor(H)
            d[("act", l)] = Tensor(F)
            d[("x_in", l + 1)] = Tensor(H)
            for q in range(tp):
                for ph in range(2):
                    d[("recv", q, l, ph)] = Tensor(H)
        d[("logits",)] = Tensor(V)
        T.append(d)
    flags = [defaultdict(int) for _ in range(tp)]
    counters = [[0] * len(th) for th in rank_thr]
    splits = [{tk.layer: tk.r1 for tk in tasks if tk.op == 2} for tasks in rank_tasks]
    nxt = [0] * tp                                   # next unclaimed task of each rank
    held = [[[] for _ in range(workers)] for _ in range(tp)]
    done = [0] * tp

    def ready(r: int, i: int) -> bool:
        tk = rank_tasks[r][i]
        for e in (tk.wait[0], tk.wait[1]):
            if e != NO_EVENT and counters[r][e] < rank_thr[r][e]:
                return False
        if OP[tk.op] == "tp_reduce" and flags[r][(tk.layer, tk.aux, tk.r0)] < tp:
            return False
        return True

    def execute(r: int, i: int) -> None:
        tk = rank_tasks[r][i]
        t = T[r]
        op, l, r0, r1 = OP[tk.op], tk.layer, tk.r0, tk.r1
        who = f"rank {r} task {i} ({op} l{l} aux{tk.aux} {r0}:{r1})"
        base = _mix(i + 1)
        if op == "qkv":
            t[("qkv", l)].write(r0, r1, _mix(base ^ t[("x_in", l)].read(0, H, who)), who)
        elif op == "attn":
            g = tk.aux
            qkv = t[("qkv", l)]
            d = qkv.read(g * hpg * hd, (g + 1) * hpg * hd, who)
            d += qkv.read(nq * hd + g * hd, nq * hd + (g + 1) * hd, who)
            d += qkv.read((nq + nkv) * hd + g * hd, (nq + nkv) * hd + (g + 1) * hd, who)
            t[("part", l)].write(g * 4096 + r0, g * 4096 + r0 + 1, _mix(base ^ (d & M64)), who)
        elif op in ("oproj", "down"):
            ph = 0 if op == "oproj" else 1
            if ph == 0:
                d = 0
                for g in range(nkv):
                    d += t[("part", l)].read(g * 4096, g * 4096 + splits[r][l], who)
            else:
                d = t[("act", l)].read(0, F, who)
            for q in range(tp):
                T[q][("recv", r, l, ph)].write(r0, r1, _mix(base ^ (d & M64)), who)
                flags[q][(l, ph, r0)] += 1
                if flags[q][(l, ph, r0)] > tp:
                    raise Violation(f"{who}: flag raised beyond tp")
        elif op == "tp_reduce":
            d = 0
            for q in range(tp):
                d += t[("recv", q, l, tk.aux)].read(r0, r1, who)
            if tk.aux == 0:
                d += t[("x_in", l)].read(r0, r1, who)
                t[("x_mid", l)].write(r0, r1, _mix(d & M64), who)
            else:
                d += t[("x_mid", l)].read(r0, r1, who)
                t[("x_in", l + 1)].write(r0, r1, _mix(d & M64), who)
        elif op == "gateup":
            t[("act", l)].write(r0, r1, _mix(base ^ t[("x_mid", l)].read(0, H, who)), who)
        elif op == "lmhead":
            t[("logits",)].write(r0, r1, _mix(base ^ t[("x_in", L)].read(0, H, who)), who)
        else:
            raise Violation(f"{who}: not an operator of a tensor-parallel graph")
        e = tk.signal
        if e != NO_EVENT:
            counters[r][e] += 1
            if counters[r][e] > rank_thr[r][e]:
                raise Violation(f"{who}: event {e} signalled beyond its threshold")
        done[r] += 1

    total = sum(len(x) for x in rank_tasks)
    while sum(done) < total:
        moves = []
        for r in range(tp):
            for w in range(workers):
                h = held[r][w]
                if len(h) < ahead and nxt[r] < len(rank_tasks[r]):
                    moves.append((r, w, "claim"))
                if h and ready(r, h[0]):
                    moves.append((r, w, "run"))
        if not moves:
            raise Violation(f"deadlock: {sum(done)} of {total} tasks ran")
        r, w, kind = moves[rng.randrange(len(moves))]
        if kind == "claim":
            held[r][w].append(nxt[r])
            nxt[r] += 1
        else:
            execute(r, held[r][w].pop(0))
    for r in range(tp):
        for e, (c, th) in enumerate(zip(counters[r], rank_thr[r])):
            if c != th:
                raise Violation(f"rank {r} event {e}: counter {c} != threshold {th}")
        if not T[r][("logits",)].ok.all():
            raise Violation(f"rank {r}: logits not fully written")
    return [T[r][("logits",)].val.copy() for r in range(tp)]
