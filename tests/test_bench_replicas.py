"""The N > 1 bench path (replicas only) on CPU: two gloo ranks.

Each rank decodes its own sequence with its own weights; the only cross-rank
step is the maximum of the ranks' device times, taken after the timed region.
These tests run that reduction and the throughput arithmetic on two real
processes, and check that the reference arm does no work on ranks other than 0.
"""
import contextlib
import io
import os
import socket
import sys
from types import SimpleNamespace

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, times_ms, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    from datetime import timedelta
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        slowest = bench.max_over_ranks(times_ms[rank], dist, "cpu")
        value = bench.replica_tokens_per_s(100, world, slowest)
        out.put((rank, slowest, value))
    finally:
        dist.destroy_process_group()


def test_two_replicas_report_the_slowest_rank():
    world = 2
    times_ms = [420.0, 455.5]          # rank 1 is slower
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, times_ms, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # every rank sees the same slowest time; 2 ranks x 100 tokens over 455.5 ms
    for rank, slowest, value in res:
        assert slowest == 455.5
        assert value == pytest.approx(2 * 100 / 0.4555)


def test_single_process_needs_no_group():
    assert bench.max_over_ranks(3.25, None, "cpu") == 3.25
    assert bench.replica_tokens_per_s(507, 1, 2000.0) == pytest.approx(253.5)
    assert bench.replica_tokens_per_s(10, 4, 1000.0, batch=16) == pytest.approx(640.0)


def test_reference_arm_runs_on_rank_zero_only(monkeypatch):
    monkeypatch.setenv("RANK", "1")
    monkeypatch.setenv("WORLD_SIZE", "2")
    args = SimpleNamespace(steps=1, warmup=1, ref_budget=1.0)
    buf = io.StringIO()
    with contextlib.redirect_stdout(buf):
        bench.run_reference(args, bench.workload("tiny"))
    assert buf.getvalue() == ""
