"""The multi-process path of bench.py on CPU: two gloo ranks agree on the slowest rank's time and
the job's throughput counts every replica's weights."""
import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank(rank, world, port, q):
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = [10.0, 12.5][rank]
        got = bench.max_over_ranks(ms, dist, "cpu")
        q.put((rank, got, bench.job_value(world, 1000, 4, got)))
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29500 + os.getpid() % 1000
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, ms, value in res:
        assert ms == 12.5
        assert value == pytest.approx(2 * 1000 * 4 / 12.5e-3)


def test_single_process_is_its_own_max():
    import importlib
    sys.path.insert(0, ROOT)
    bench = importlib.import_module("bench")
    assert bench.max_over_ranks(3.25, None, "cpu") == 3.25
