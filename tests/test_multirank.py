"""The N > 1 path of bench.py on CPU: world size 2 over gloo.

bench.py runs one process per GPU as independent replicas (no collective on
the data path); ranks meet only to take the slowest rank's time, and the
reference arm runs on rank 0 alone.  These tests run that logic with two CPU
processes over gloo on 127.0.0.1.
"""
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

torch = pytest.importorskip("torch")
import bench  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        r, _, ws = bench.dist_env()
        t = bench.max_over_ranks(1.5 + rank, ws)          # rank 1 is the slow one
        dist.barrier()
        q.put((r, ws, t))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    ctx = torch.multiprocessing.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    for p in procs:
        if p.is_alive():
            p.kill()
    assert all(p.exitcode == 0 for p in procs)
    got = sorted(q.get(timeout=10) for _ in range(2))
    assert got == [(0, 2, 2.5), (1, 2, 2.5)]


def test_max_over_ranks_single_process_is_identity():
    assert bench.max_over_ranks(3.25, 1) == 3.25


def test_weak_scaling_aggregate():
    w = bench.WORKLOADS["hires16k"]
    one = bench.aggregate_tops(1, w.ops, 11.0)
    assert one == pytest.approx(w.ops / 11e-3 / 1e12)
    # two replicas in the time of the slower one: twice the work
    assert bench.aggregate_tops(2, w.ops, 11.0) == pytest.approx(2 * one)


def test_reference_arm_runs_on_rank_zero_only():
    class A:
        steps, warmup = 2, 3
    # rank 1 returns at once, without touching the oracle or the inputs
    assert bench.run_reference(A, bench.WORKLOADS["hires16k"], rank=1, world=2) is None
