#!/usr/bin/env python
"""Decode throughput of the persistent megakernel on B200.

Default workload: an 8B-class dense decoder (32 layers, hidden 4096, 32/8
heads, head_dim 128, FFN 14336, vocab 128256; bf16 weights ~N(0, 0.02)),
batch 1, a 39-token prompt and 512 decode steps over a contiguous KV cache
(the workload of the MPK digest, section "MPK का मुख्य मूल्य").  One step =
one decode step = one launch of the megakernel.  Tokens are seeded synthetic
ids fed teacher-forced; positions cycle over 39..550.

Metric: decode tokens/s at batch 1, and its fraction of the HBM
speed-of-light bound  tokens/s_SoL = 8e12 B/s / (weight bytes + KV bytes per
step)  (Cohere page, section "A szűk keresztmetszet a memória-sávszélesség").

Multi-GPU: replicas only (each rank decodes its own sequence with its own full
weight copy; no collective on the data path); value = all ranks' tokens / the
slowest rank's device time.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "decode tokens/s at batch 1 and % of HBM speed-of-light (bytes/step ÷ peak)"
SOL_BW = 8.0e12            # nominal B200 HBM bandwidth used for the speed-of-light bound
PROMPT = 39
GEN = 512


# ----------------------------------------------------------------------------- arithmetic

def sol_tokens_per_s(bytes_per_step: float, bandwidth: float, batch: int = 1) -> float:
    """Speed-of-light decode rate: every step must read its bytes once at `bandwidth`."""
    return batch * bandwidth / bytes_per_step


def kv_read_bytes(cfg, positions, batch: int = 1) -> float:
    """Mean KV bytes read per step: (p+1) cached tokens x layers x (K,V) x heads x dim x 2 B,
    summed over the batch (`positions` lists every sequence's position of every step)."""
    per_tok = cfg.n_layers * 2 * cfg.n_kv_heads * cfg.head_dim * 2
    return batch * sum((p + 1) * per_tok for p in positions) / len(positions)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.out = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"], stdout=self.out,
                stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.out.close()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None

        def num(x):
            try:
                return float(x)
            except ValueError:
                return float("nan")
        mhz = [num(r[1]) for r in rows]
        mx = max(num(r[2]) for r in rows)
        power = [num(r[3]) for r in rows]
        loaded = [m for m, pw in zip(mhz, power) if pw > 250.0] or mhz
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows), "samples_under_load": len(loaded)}


# ----------------------------------------------------------------------------- workloads

def workload(name: str):
    import synthetic as syn
    if name == "llama8b":
        return dict(cfg=syn.LLAMA8B, seed=2, prompt=PROMPT, gen=GEN, ctx0=0,
                    desc="llama-8b-class dense decode, batch 1, 39-token prompt + 512 steps, "
                         "contiguous KV")
    if name == "tiny":
        return dict(cfg=syn.TINY, seed=1, prompt=PROMPT, gen=16, ctx0=0,
                    desc="tiny 2-layer decoder, batch 1, 39-token prompt + 16 steps")
    if name == "moe30b":
        return dict(cfg=syn.MOE30B, seed=3, prompt=8192, gen=256, ctx0=8192,
                    desc="30B-total/3.3B-active MoE decode, batch 1, 8192-token synthetic KV, "
                         "256 steps")
    if name == "long131k":
        return dict(cfg=syn.LLAMA8B, seed=5, prompt=131072, gen=64, ctx0=131072,
                    desc="llama-8b-class decode, batch 1, 131072-token synthetic paged KV "
                         "(shuffled 16-token pages), 64 steps")
    if name in BATCH_WORKLOADS:
        B = int(name[len("batch"):])
        lens = ragged_lengths(B, 512, 8192, 4700 + B)
        return dict(cfg=syn.LLAMA8B, seed=6, batch=B, lens=lens, prompt=lens[0], gen=128,
                    ctx0=max(lens),
                    desc=f"llama-8b-class continuous batching, batch {B}, ragged contexts "
                         f"U(512, 8192) in shuffled 16-token pages, 128 steps")
    raise SystemExit(f"unknown workload {name}")


BATCH_WORKLOADS = ("batch1", "batch4", "batch16", "batch64")


def ragged_lengths(B: int, lo: int, hi: int, seed: int):
    """Cached tokens per sequence, uniform on [lo, hi] (seeded)."""
    import numpy as np
    return [int(x) for x in np.random.default_rng(seed).integers(lo, hi + 1, size=B)]


def max_over_ranks(x: float, pg, device) -> float:
    """Largest value of x over all ranks (identity without a process group)."""
    if pg is None:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    pg.all_reduce(t, op=pg.ReduceOp.MAX)
    return float(t.item())


def replica_tokens_per_s(steps: int, world: int, slowest_ms: float, batch: int = 1) -> float:
    """Whole-job throughput of `world` independent replicas: every rank decodes
    `steps` steps of `batch` tokens; the job ends with the slowest rank."""
    return world * steps * batch / (slowest_ms / 1e3)


def dist_info():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


# ----------------------------------------------------------------------------- CPU oracle arm

def oracle_rate(W: dict, max_steps: int, budget_s: float, warmup: int = 1):
    """Times the CPU oracle on a bounded sample of the workload; returns (tok/s, steps, desc)."""
    import numpy as np
    import oracle
    import synthetic as syn
    cfg = W["cfg"]
    seed = syn.SEED_WEIGHTS + W["seed"]
    ctx = W["prompt"]
    cap = ctx + max_steps + warmup + 1
    specs = syn.tensor_specs(cfg)
    names = [s.name for s in specs]
    if cfg.is_moe:
        # experts are regenerated on demand (all 128 per layer do not fit host memory)
        by_name = {s.name: s for s in specs}
        experts = ("w_gate", "w_up", "w_down")
        host_w = {s.name: syn.host_tensor(s, seed) for s in specs
                  if not any(s.name.endswith(e) for e in experts)}
        expert_elems = cfg.expert_ffn * cfg.hidden

        def prov(l, e, which):
            s = by_name[f"layers.{l}.{experts[which]}"]
            return syn.host_bf16(expert_elems, seed, s.tensor_id, s.sigma, s.mean,
                                 offset=e * expert_elems)
        model = oracle.Model(cfg, host_w, cap, names, expert_provider=prov)
    else:
        model = oracle.Model(cfg, syn.host_weights(cfg, seed), cap, names)
    for l in range(cfg.n_layers):     # synthetic context standing in for the prompt
        model.k[l][:ctx] = syn.host_kv(cfg, syn.SEED_KV + W["seed"], l, "k", 0, 0, ctx)
        model.v[l][:ctx] = syn.host_kv(cfg, syn.SEED_KV + W["seed"], l, "v", 0, 0, ctx)
    toks = syn.host_tokens(warmup + max_steps, syn.SEED_PROMPT + W["seed"], cfg.vocab)
    for i in range(warmup):
        model.decode_step(int(toks[i]), ctx + i)
    t0 = time.perf_counter()
    n_done = 0
    while n_done < max_steps:
        model.decode_step(int(toks[warmup + n_done]), ctx + warmup + n_done)
        n_done += 1
        if time.perf_counter() - t0 > budget_s:
            break
    dt = time.perf_counter() - t0
    n = n_done
    sample = (f"{n} decode step(s) of the same model at positions {ctx + warmup}..{ctx + warmup + n - 1} "
              f"over a {ctx}-token synthetic context, after {warmup} warm-up step(s)")
    return n / dt, n, sample, oracle.num_threads()


def run_reference(args, W):
    rank, world, _ = dist_info()
    if rank != 0:
        return
    rate, n, sample, cores = oracle_rate(W, max(1, args.steps), budget_s=float(args.ref_budget),
                                         warmup=min(args.warmup, 1))
    line = {"impl": "reference", "metric": METRIC, "value": rate, "unit": "tokens/s",
            "n_gpus": world, "steps": n, "warmup": min(args.warmup, 1),
            "ms_per_step": 1000.0 / rate, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": W["desc"], "batch": W.get("batch", 1)},
            "cpu_baseline": {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": rate, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------------- GPU arm

def run_gpu(args, W):
    import numpy as np
    import torch
    import synthetic as syn
    import persistent_megakernel_decode_03_b200 as mk
    from persistent_megakernel_decode_03_b200.runner import Decoder

    rank, world, local = dist_info()
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    pg = None
    if world > 1:
        import torch.distributed as dist
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
        pg = dist
    cfg = W["cfg"]
    seed = syn.SEED_WEIGHTS + W["seed"]
    specs = syn.tensor_specs(cfg)
    ts = []
    for s in specs:
        t = torch.empty(s.shape, dtype=torch.bfloat16, device=dev)
        syn.dev_fill_tensor(t, s, seed)
        ts.append(t)
    n_steps_total = args.warmup + args.steps
    ctx0 = W["ctx0"]
    span = W["gen"]                       # positions cycle over [prompt, prompt + gen)
    max_ctx = W["prompt"] + span
    desc = dict(n_layers=cfg.n_layers, hidden=cfg.hidden, n_q_heads=cfg.n_q_heads,
                n_kv_heads=cfg.n_kv_heads, head_dim=cfg.head_dim, ffn=cfg.ffn, vocab=cfg.vocab,
                rms_eps=cfg.rms_eps, rope_theta=cfg.rope_theta, n_experts=cfg.n_experts,
                top_k=cfg.top_k, expert_ffn=cfg.expert_ffn, moe_renorm=cfg.moe_renorm)
    B = W.get("batch", 1)
    lens = W.get("lens", [W["prompt"]])
    if "lens" in W:
        max_ctx = max(lens) + span
    page_table = None
    n_pages = None
    if args.workload == "long131k" or "lens" in W:
        per_seq = (max_ctx + 15) // 16
        pages = B * per_seq
        perm = syn.page_permutation(pages, syn.SEED_KV + W["seed"])
        page_table = torch.tensor(perm, dtype=torch.int32, device=dev).view(B, per_seq)
        n_pages = pages
    dec = Decoder(desc, [t.data_ptr() for t in ts], B, max_ctx, page_table=page_table,
                  n_pages=n_pages, device=f"cuda:{local}")
    stream = torch.cuda.current_stream(dev)
    prompt_toks = torch.tensor(syn.host_tokens(W["prompt"], syn.SEED_PROMPT + W["seed"], cfg.vocab),
                               dtype=torch.int32, device=dev)
    if ctx0 > 0:
        for b in range(B):
            for l in range(cfg.n_layers):
                syn.dev_fill_kv_paged(dec.k_pages[l], dec.page_table[b], b, 0, lens[b], cfg, 16,
                                      syn.SEED_KV + W["seed"], syn.TID_K_BASE + l)
                syn.dev_fill_kv_paged(dec.v_pages[l], dec.page_table[b], b, 0, lens[b], cfg, 16,
                                      syn.SEED_KV + W["seed"], syn.TID_V_BASE + l)
    else:
        dec.prefill(prompt_toks)          # the 39-token prompt through the same megakernel
    dec.check()
    # step i feeds B tokens; sequence b is at position lens[b] + (i % span)
    gen_toks = syn.host_tokens(n_steps_total * B, syn.SEED_PROMPT + 100 + W["seed"], cfg.vocab)
    positions = [lens[b] + (i % span) for i in range(n_steps_total) for b in range(B)]
    toks_d = torch.tensor(gen_toks, dtype=torch.int32, device=dev)
    pos_d = torch.tensor(positions, dtype=torch.int32, device=dev)

    def launch(i):
        mk.mk_decode_step(dec.state, toks_d[i * B:].data_ptr(), pos_d[i * B:].data_ptr(), B, dec.kv,
                          dec.logits.data_ptr(), stream.cuda_stream)

    for i in range(args.warmup):
        launch(i)
    torch.cuda.synchronize(dev)
    st = dec.sync()
    if st != mk.MK_OK:
        raise SystemExit(f"warm-up failed: {mk.mk_last_error_string()}")
    events = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    clocks = ClockSampler(local)
    if pg:
        pg.barrier()
    torch.cuda.synchronize(dev)
    clocks.start()
    torch.cuda.nvtx.range_push("timed")
    events[0].record(stream)
    for k in range(args.steps):
        launch(args.warmup + k)
        events[k + 1].record(stream)
    torch.cuda.nvtx.range_pop()
    torch.cuda.synchronize(dev)
    clk = clocks.stop()
    if pg:
        pg.barrier()
    st = dec.sync()
    if st != mk.MK_OK:
        raise SystemExit(f"timed steps failed: {mk.mk_last_error_string()}")
    per = [events[k].elapsed_time(events[k + 1]) for k in range(args.steps)]
    total_ms = max_over_ranks(events[0].elapsed_time(events[-1]), pg, dev)
    timed_pos = positions[args.warmup * B:]
    info = dec.info
    bytes_step = float(info.weight_bytes_per_step) + kv_read_bytes(cfg, timed_pos, B)
    tok_s = replica_tokens_per_s(args.steps, world, total_ms, B)
    sol = sol_tokens_per_s(bytes_step, SOL_BW, B)
    peak, peak_kind = measured_peaks()
    launch_ms = statistics.mean(per)
    achieved = bytes_step / (launch_ms / 1e3) / 1e9

    # end to end through the host-buffer entry point: H2D of token+position, D2H of logits
    e2e = None
    if not args.no_e2e:
        k_e2e = args.steps                 # the same steps (positions) as the timed region
        tok_h = torch.tensor(gen_toks, dtype=torch.int32).pin_memory()
        pos_h = torch.tensor(positions, dtype=torch.int32).pin_memory()
        logits_h = torch.empty((B, cfg.vocab), dtype=torch.float32).pin_memory()
        torch.cuda.synchronize(dev)
        if pg:
            pg.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for k in range(k_e2e):
            i = args.warmup + k
            mk.mk_decode_step_host(dec.state, tok_h[i * B:].data_ptr(), pos_h[i * B:].data_ptr(), B,
                                   dec.kv, logits_h.data_ptr(), stream.cuda_stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), pg, dev)
        if dec.sync() != mk.MK_OK:
            raise SystemExit(f"e2e steps failed: {mk.mk_last_error_string()}")
        e2e = {"value": replica_tokens_per_s(k_e2e, world, e2e_ms, B), "unit": "tokens/s",
               "h2d_bytes_per_step": 8 * B, "d2h_bytes_per_step": 4 * cfg.vocab * B, "steps": k_e2e,
               "api": "mk_decode_step_host"}

    traffic = None
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tpath):
        with open(tpath) as f:
            tr = json.load(f)
        ent = tr.get(args.workload)
        if ent and ent.get("kernel_source_sha") == kernel_source_sha():
            # DRAM bytes of a smaller capture of the same kernel, as a ratio to its
            # algorithmic bytes (traffic grows with the weight and KV bytes streamed)
            traffic = ent["ratio_to_algorithmic"] * bytes_step
    line = {
        "metric": METRIC, "value": tok_s, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": total_ms / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
        "data": "synthetic",
        "config": {"workload": W["desc"], "batch": B, "weights": "bf16", "activations": "f32",
                   "kv_cache": "bf16", "positions": [min(timed_pos), max(timed_pos)],
                   "l2": "inputs larger than L2 (every step streams all weights)",
                   "parallelism": "replicas" if world > 1 else "single-gpu"},
        "sol_pct": 100.0 * tok_s / world / sol,
        "sol_tokens_per_s": sol,
        "bytes_per_step": bytes_step,
        "tiles": "tcgen05 projection tiles" if B > 1 else "CUDA-core GEMV tiles",
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                     "frac": achieved / peak, "traffic": traffic,
                     "peak_kind": f"{peak_kind} hbm_gbs (copy)",
                     "kernel": "mk::megakernel", "launch_ms": launch_ms},
        "gpu_launches": args.steps,
        "clocks": clk,
    }
    if e2e:
        line["e2e"] = e2e
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rate, n, sample, cores = oracle_rate(W, 3 if cfg.n_layers > 2 else 16, budget_s=25.0)
        line["cpu_baseline"] = {"value": rate, "unit": "tokens/s", "cores": cores, "kind": "oracle",
                                "sample": sample}
    if rank == 0:
        print(json.dumps(line), flush=True)
    dec.close()
    if pg:
        pg.barrier()
        pg.destroy_process_group()


def run_prefill(args, W):
    """Prompt processing (the step before the decode loop): the workload's 39-token
    prompt through mk_prefill on a batch-64 graph (tensor-core tiles, the prompt's
    tokens as batch rows: one launch), timed beside the batch-1 graph's
    token-by-token prefill (39 launches).  Prints one JSON line; not a decode line."""
    import torch
    import synthetic as syn
    from persistent_megakernel_decode_03_b200.runner import Decoder

    cfg = W["cfg"]
    seed = syn.SEED_WEIGHTS + W["seed"]
    ts = []
    for s in syn.tensor_specs(cfg):
        t = torch.empty(s.shape, dtype=torch.bfloat16, device="cuda")
        syn.dev_fill_tensor(t, s, seed)
        ts.append(t)
    desc = dict(n_layers=cfg.n_layers, hidden=cfg.hidden, n_q_heads=cfg.n_q_heads,
                n_kv_heads=cfg.n_kv_heads, head_dim=cfg.head_dim, ffn=cfg.ffn, vocab=cfg.vocab,
                rms_eps=cfg.rms_eps, rope_theta=cfg.rope_theta)
    n = PROMPT
    prompt = torch.tensor(syn.host_tokens(n, syn.SEED_PROMPT + W["seed"], cfg.vocab), dtype=torch.int32,
                          device="cuda")
    res = {}
    for name, mb in (("batched", 64), ("token_by_token", 1)):
        dec = Decoder(desc, [t.data_ptr() for t in ts], mb, n + 16)
        for _ in range(args.warmup):
            dec.prefill(prompt)
        torch.cuda.synchronize()
        dec.check()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        for _ in range(args.steps):
            dec.prefill(prompt)
        e1.record()
        torch.cuda.synchronize()
        dec.check()
        res[name] = e0.elapsed_time(e1) / args.steps
        dec.close()
    line = {"metric": "prompt tokens/s (prefill)", "value": n / (res["batched"] / 1e3), "unit": "tokens/s",
            "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_prefill": res["batched"],
            "token_by_token_ms_per_prefill": res["token_by_token"],
            "speedup_vs_token_by_token": res["token_by_token"] / res["batched"],
            "higher_is_better": True, "dtype": "f32", "data": "synthetic",
            "config": {"workload": W["desc"] + f"; {n}-token prompt", "prefill": "batched (one launch, batch-64 graph)"}}
    print(json.dumps(line), flush=True)


def run_per_op(args, W):
    """The same decode step as a kernel-per-operator baseline: one launch per
    (operator, layer) run of the task list, replayed as a CUDA graph, timed beside
    the megakernel on the same workload.  Prints one JSON line; not a decode line."""
    import torch
    import synthetic as syn
    import persistent_megakernel_decode_03_b200 as mk
    from persistent_megakernel_decode_03_b200.runner import Decoder

    cfg = W["cfg"]
    seed = syn.SEED_WEIGHTS + W["seed"]
    ts = []
    for s in syn.tensor_specs(cfg):
        t = torch.empty(s.shape, dtype=torch.bfloat16, device="cuda")
        syn.dev_fill_tensor(t, s, seed)
        ts.append(t)
    desc = dict(n_layers=cfg.n_layers, hidden=cfg.hidden, n_q_heads=cfg.n_q_heads,
                n_kv_heads=cfg.n_kv_heads, head_dim=cfg.head_dim, ffn=cfg.ffn, vocab=cfg.vocab,
                rms_eps=cfg.rms_eps, rope_theta=cfg.rope_theta)
    ctx = 300
    dec = Decoder(desc, [t.data_ptr() for t in ts], 1, ctx + 8)
    for l in range(cfg.n_layers):
        syn.dev_fill_kv_paged(dec.k_pages[l], dec.page_table[0], 0, 0, ctx, cfg, 16, syn.SEED_KV + 2,
                              syn.TID_K_BASE + l)
        syn.dev_fill_kv_paged(dec.v_pages[l], dec.page_table[0], 0, 0, ctx, cfg, 16, syn.SEED_KV + 2,
                              syn.TID_V_BASE + l)
    tok = torch.tensor([7], dtype=torch.int32, device="cuda")
    pos = torch.tensor([ctx], dtype=torch.int32, device="cuda")
    out = torch.empty((1, cfg.vocab), dtype=torch.float32, device="cuda")
    stream = torch.cuda.Stream()

    def timed(fn, reps):
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(reps):
                fn()
            e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    n_launch = [0]

    def per_op():
        n_launch[0] = mk.mk_decode_step_per_op(dec.state, tok.data_ptr(), pos.data_ptr(), 1, dec.kv,
                                               out.data_ptr(), stream.cuda_stream)

    def mega():
        mk.mk_decode_step(dec.state, tok.data_ptr(), pos.data_ptr(), 1, dec.kv, out.data_ptr(),
                          stream.cuda_stream)

    ms_direct = timed(per_op, args.steps)
    dec.check()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream, capture_error_mode="relaxed"):
        per_op()
    ms_graph = timed(graph.replay, args.steps)
    dec.check()
    del graph
    ms_mega = timed(mega, args.steps)
    dec.check()
    dec.close()
    line = {"metric": "decode step time: megakernel vs kernel-per-operator baseline (same tiles)",
            "unit": "ms", "higher_is_better": False, "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "megakernel_ms": ms_mega, "per_op_graph_ms": ms_graph, "per_op_direct_ms": ms_direct,
            "launches_per_step": n_launch[0], "speedup_vs_per_op_graph": ms_graph / ms_mega,
            "dtype": "f32", "data": "synthetic",
            "config": {"workload": W["desc"] + f"; batch 1 at position {ctx}"}}
    print(json.dumps(line), flush=True)


def run_generate(args, W):
    """Greedy generation (the loop after the hot path): 128 new tokens of the 8B
    model after its 39-token prompt, with mk_generate (each step's argmax taken
    inside the step by its last LM-head tiles, one launch per token, all enqueued
    at once) beside a host loop that copies each
    step's logits to the host, takes the argmax there and sends the token back.
    Prints one JSON line; not a decode line."""
    import numpy as np
    import torch
    import synthetic as syn
    import persistent_megakernel_decode_03_b200 as mk
    from persistent_megakernel_decode_03_b200.runner import Decoder

    cfg = W["cfg"]
    seed = syn.SEED_WEIGHTS + W["seed"]
    ts = []
    for s in syn.tensor_specs(cfg):
        t = torch.empty(s.shape, dtype=torch.bfloat16, device="cuda")
        syn.dev_fill_tensor(t, s, seed)
        ts.append(t)
    desc = dict(n_layers=cfg.n_layers, hidden=cfg.hidden, n_q_heads=cfg.n_q_heads,
                n_kv_heads=cfg.n_kv_heads, head_dim=cfg.head_dim, ffn=cfg.ffn, vocab=cfg.vocab,
                rms_eps=cfg.rms_eps, rope_theta=cfg.rope_theta)
    n = 128
    dec = Decoder(desc, [t.data_ptr() for t in ts], 1, PROMPT + n + 8)
    prompt = torch.tensor(syn.host_tokens(PROMPT, syn.SEED_PROMPT + W["seed"], cfg.vocab), dtype=torch.int32,
                          device="cuda")
    last = dec.prefill(prompt)
    first = int(torch.argmax(last).item())
    dec.check()
    stream = torch.cuda.current_stream().cuda_stream
    out = torch.zeros((n, 1), dtype=torch.int32, device="cuda")
    logits = torch.empty((1, cfg.vocab), dtype=torch.float32, device="cuda")
    first_d = torch.tensor([first], dtype=torch.int32, device="cuda")
    pos_d = torch.tensor([PROMPT], dtype=torch.int32, device="cuda")
    for _ in range(2):   # warm-up (the same positions are rewritten each time)
        mk.mk_generate(dec.state, first_d.data_ptr(), pos_d.data_ptr(), 1, n, dec.kv, out.data_ptr(),
                       logits.data_ptr(), stream)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    mk.mk_generate(dec.state, first_d.data_ptr(), pos_d.data_ptr(), 1, n, dec.kv, out.data_ptr(),
                   logits.data_ptr(), stream)
    torch.cuda.synchronize()
    t_dev = time.perf_counter() - t0
    dec.check()
    dev_tokens = out[:, 0].cpu().tolist()
    # host loop: step, logits to the host, argmax there, token back
    tok_h = torch.zeros(1, dtype=torch.int32).pin_memory()
    pos_h = torch.zeros(1, dtype=torch.int32).pin_memory()
    lg_h = torch.empty((1, cfg.vocab), dtype=torch.float32).pin_memory()
    host_tokens = []
    t0 = time.perf_counter()
    tok = first
    for i in range(n):
        tok_h[0] = tok
        pos_h[0] = PROMPT + i
        mk.mk_decode_step_host(dec.state, tok_h.data_ptr(), pos_h.data_ptr(), 1, dec.kv, lg_h.data_ptr(), stream)
        tok = int(np.argmax(lg_h.numpy()[0]))
        host_tokens.append(tok)
    t_host = time.perf_counter() - t0
    dec.check()
    dec.close()
    line = {"metric": "greedy generation tokens/s (wall clock, batch 1)", "value": n / t_dev, "unit": "tokens/s",
            "n_gpus": 1, "tokens": n, "device_loop_ms_per_token": 1e3 * t_dev / n,
            "host_loop_tokens_per_s": n / t_host, "host_loop_ms_per_token": 1e3 * t_host / n,
            "same_tokens": dev_tokens == host_tokens, "higher_is_better": True, "dtype": "f32",
            "data": "synthetic", "config": {"workload": W["desc"] + f"; greedy, {n} new tokens"}}
    print(json.dumps(line), flush=True)


def run_solo(args, W):
    """One operator kind's tiles alone (dependencies dropped), on the workload's shapes.

    Prints one JSON line: median launch time and the algorithmic bytes of that
    operator over all layers divided by it.  Evidence per tile type; not the
    metric."""
    import torch
    import synthetic as syn
    import persistent_megakernel_decode_03_b200 as mk
    from persistent_megakernel_decode_03_b200.runner import Decoder

    names = {v: k for k, v in mk.OP_NAMES.items()}
    if args.solo not in names:
        raise SystemExit(f"unknown operator {args.solo}")
    op = names[args.solo]
    cfg = W["cfg"]
    if cfg.is_moe:
        raise SystemExit("solo lists cover the dense operators")
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    seed = syn.SEED_WEIGHTS + W["seed"]
    ts = []
    for s in syn.tensor_specs(cfg):
        t = torch.empty(s.shape, dtype=torch.bfloat16, device=dev)
        syn.dev_fill_tensor(t, s, seed)
        ts.append(t)
    ctx = W["prompt"] + W["gen"] // 2
    max_ctx = W["prompt"] + W["gen"]
    desc = dict(n_layers=cfg.n_layers, hidden=cfg.hidden, n_q_heads=cfg.n_q_heads,
                n_kv_heads=cfg.n_kv_heads, head_dim=cfg.head_dim, ffn=cfg.ffn, vocab=cfg.vocab,
                rms_eps=cfg.rms_eps, rope_theta=cfg.rope_theta)
    dec = Decoder(desc, [t.data_ptr() for t in ts], 1, max_ctx, device="cuda:0")
    L, H, F, V, d = cfg.n_layers, cfg.hidden, cfg.ffn, cfg.vocab, cfg.head_dim
    nq, nkv = cfg.n_q_heads, cfg.n_kv_heads
    nbytes = {"qkv": 2 * (nq + 2 * nkv) * d * H * L, "attn": (ctx + 1) * L * 2 * nkv * d * 2,
              "oproj": 2 * H * nq * d * L, "gateup": 4 * F * H * L, "down": 2 * H * F * L,
              "lmhead": 2 * V * H}[args.solo]
    g = mk.mk_build_taskgraph_solo(dec.model, 1, max_ctx, op)
    st = mk.mk_state_create(g)
    info = mk.mk_graph_get_info(g)
    tok = torch.tensor([7], dtype=torch.int32, device=dev)
    pos = torch.tensor([ctx], dtype=torch.int32, device=dev)
    stream = torch.cuda.current_stream(dev)
    times = []
    for i in range(args.warmup + args.steps):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        mk.mk_decode_step(st, tok.data_ptr(), pos.data_ptr(), 1, dec.kv, dec.logits.data_ptr(),
                          stream.cuda_stream)
        e1.record(stream)
        torch.cuda.synchronize(dev)
        if i >= args.warmup:
            times.append(e0.elapsed_time(e1))
    if mk.mk_sync(st, stream.cuda_stream) != mk.MK_OK:
        raise SystemExit(f"solo run failed: {mk.mk_last_error_string()}")
    med = statistics.median(times)
    peak, peak_kind = measured_peaks()
    gbs = nbytes / (med / 1e3) / 1e9
    print(json.dumps({"solo": args.solo, "workload": W["desc"], "tasks": info.n_tasks,
                      "bytes_per_launch": nbytes, "median_us": med * 1e3, "achieved_gbs": gbs,
                      "peak_gbs": peak, "frac": gbs / peak, "peak_kind": peak_kind}), flush=True)
    mk.mk_state_destroy(st)
    mk.mk_graph_destroy(g)
    dec.close()


def run_trace(args, W):
    """Per-task timestamps of a few steps (the state's trace flag): for each operator,
    the time its tasks waited on their dependency events, summed per SM; and for a
    middle layer, when each operator's first task started and its last task ended.
    The gap between one operator's last end and the next one's first start is the
    boundary cost the persistent kernel pays.  Timestamps are the GPU's global
    timer (ns) taken by the consumer warps (claim seen, dependency met) and the
    epilogue warp (signalled).  Evidence for where a step's time goes; not the
    metric (tracing slows the step a little)."""
    import numpy as np
    import torch
    import synthetic as syn
    import persistent_megakernel_decode_03_b200 as mk
    from persistent_megakernel_decode_03_b200.runner import Decoder

    cfg = W["cfg"]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    seed = syn.SEED_WEIGHTS + W["seed"]
    ts = []
    for s in syn.tensor_specs(cfg):
        t = torch.empty(s.shape, dtype=torch.bfloat16, device=dev)
        syn.dev_fill_tensor(t, s, seed)
        ts.append(t)
    desc = dict(n_layers=cfg.n_layers, hidden=cfg.hidden, n_q_heads=cfg.n_q_heads,
                n_kv_heads=cfg.n_kv_heads, head_dim=cfg.head_dim, ffn=cfg.ffn, vocab=cfg.vocab,
                rms_eps=cfg.rms_eps, rope_theta=cfg.rope_theta, n_experts=cfg.n_experts, top_k=cfg.top_k,
                expert_ffn=cfg.expert_ffn, moe_renorm=cfg.moe_renorm, flags=mk.MK_FLAG_TRACE)
    n_steps = 4
    ctx = W["prompt"] + max(0, min(60, W["gen"] - n_steps - 1))
    dec = Decoder(desc, [t.data_ptr() for t in ts], 1, W["prompt"] + W["gen"], device="cuda:0")
    tok = torch.tensor([7], dtype=torch.int32, device=dev)
    ms = []
    for i in range(n_steps):
        pos = torch.tensor([ctx + i], dtype=torch.int32, device=dev)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        dec.step(tok, pos)
        e1.record()
        torch.cuda.synchronize(dev)
        ms.append(e0.elapsed_time(e1))
    dec.check()
    tasks = mk.mk_graph_export_tasks(dec.graph)
    tr = np.array(mk.mk_state_read_trace(dec.state, dec.info.n_tasks), dtype=np.uint64)
    tr = tr.reshape(-1, 4).astype(np.int64)        # seen, go, signalled (ns), CTA of the last step
    ops = np.array([t.op for t in tasks])
    layers = np.array([t.layer for t in tasks])
    t0 = tr[:, 0].min()
    n_cta = int(tr[:, 3].max()) + 1
    wait_us = (tr[:, 1] - tr[:, 0]) / 1e3
    out = {"trace": W["desc"], "position": ctx + len(ms) - 1, "step_ms_traced": ms[-1],
           "makespan_us": float(tr[:, 2].max() - t0) / 1e3, "ops": {}, "layer": {}}
    for op in sorted(set(ops.tolist())):
        m = ops == op
        out["ops"][mk.OP_NAMES[op]] = {"tasks": int(m.sum()), "dep_wait_us_per_sm": float(wait_us[m].sum() / n_cta),
                                       "mean_wait_us": float(wait_us[m].mean())}
    l = cfg.n_layers // 2
    for op in sorted(set(ops[layers == l].tolist())):
        m = (ops == op) & (layers == l)
        out["layer"][mk.OP_NAMES[op]] = {"first_go_us": float((tr[m, 1].min() - t0) / 1e3),
                                         "last_end_us": float((tr[m, 2].max() - t0) / 1e3),
                                         "median_go_to_end_us": float(np.median((tr[m, 2] - tr[m, 1]) / 1e3))}
    out["layer_index"] = l
    print(json.dumps(out), flush=True)
    dec.close()


def kernel_source_sha() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in ("megakernel.cu", "mk_internal.h", "graph.cpp"):
        with open(os.path.join(ROOT, "persistent_megakernel_decode_03_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=507)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["mk", "reference"], default="mk")
    ap.add_argument("--workload", default="llama8b",
                    choices=["llama8b", "tiny", "moe30b", "long131k", *BATCH_WORKLOADS])
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--layers", type=int, default=0,
                    help="profiling only: run the workload with its first N layers (not a bench line)")
    ap.add_argument("--solo", default="",
                    help="profiling only: time one operator kind's task list alone "
                         "(qkv, attn, oproj, gateup, down, lmhead) and print its GB/s")
    ap.add_argument("--generate", action="store_true",
                    help="time greedy generation with the device-side loop beside a host loop instead")
    ap.add_argument("--per-op", action="store_true",
                    help="time the kernel-per-operator baseline of the step beside the megakernel instead")
    ap.add_argument("--trace", action="store_true",
                    help="print the per-operator dependency waits and one layer's timeline from the kernel's task trace")
    ap.add_argument("--prefill", action="store_true",
                    help="time the 39-token prompt's prefill (batched vs token by token) instead")
    ap.add_argument("--ref-budget", type=float, default=120.0,
                    help="seconds of CPU time the reference arm may spend on timed steps")
    args = ap.parse_args(argv)
    if args.warmup < 3 and args.impl == "mk":
        raise SystemExit("at least 3 warm-up steps")
    W = workload(args.workload)
    if args.layers:
        import dataclasses
        W["cfg"] = dataclasses.replace(W["cfg"], n_layers=min(args.layers, W["cfg"].n_layers))
        W["desc"] += f" [first {W['cfg'].n_layers} layers only: profiling case]"
    if args.solo:
        run_solo(args, W)
    elif args.trace:
        run_trace(args, W)
    elif args.prefill:
        run_prefill(args, W)
    elif args.per_op:
        run_per_op(args, W)
    elif args.generate:
        run_generate(args, W)
    elif args.impl == "reference":
        run_reference(args, W)
    else:
        run_gpu(args, W)


if __name__ == "__main__":
    main()
