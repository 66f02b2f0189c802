"""Replica plumbing of bench.py on CPU: two gloo ranks, each with its own
timings, agree on the maximum, and the job throughput counts both replicas'
work over the slowest rank's time."""

import os
import socket

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime
    import sys
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        mine = [1.0 + rank, 10.0 - rank, 5.0 * (rank + 1)]
        q.put((rank, bench.max_over_ranks(mine, world, "cpu")))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_two_ranks():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    got = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert got[0] == got[1] == [2.0, 10.0, 10.0]


def test_job_throughput_counts_every_replica():
    import bench
    one = bench.job_tflops(1, 1e12, 1.0)
    assert one == pytest.approx(1000.0)
    assert bench.job_tflops(4, 1e12, 1.0) == pytest.approx(4 * one)
    # a slower rank sets the job's time
    assert bench.job_tflops(2, 1e12, 2.0) == pytest.approx(one)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks([3.0, 4.0], 1, "cpu") == [3.0, 4.0]
