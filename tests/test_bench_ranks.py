"""The benchmark's multi-rank host logic on CPU: two gloo ranks, the time is
the max over ranks and the value the work of all ranks over that time."""
import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import bench
    w, r, _ = bench.dist_env()
    bench.init_dist("gloo", w)
    local_seconds = 0.25 + 0.5 * r          # rank 1 is the slow one
    slowest = bench.reduce_max(local_seconds, torch.device("cpu"))
    bench.barrier()
    value = bench.aggregate(1.0e12, w, slowest)
    q.put((r, w, slowest, value))
    dist.destroy_process_group()


def test_two_gloo_ranks_take_the_slowest_time():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = 29400 + os.getpid() % 1000
    procs = [ctx.Process(target=_rank, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = sorted(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r, w, slowest, value in out:
        assert w == 2
        assert slowest == pytest.approx(0.75)
        assert value == pytest.approx(2 * 1.0e12 / 0.75)


def test_single_process_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(1.5, torch.device("cpu")) == 1.5
    assert bench.aggregate(10.0, 1, 2.0) == 5.0
