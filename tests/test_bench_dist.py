"""Multi-process (gloo, world size 2, CPU) check of the benchmark's rank aggregation: every rank runs
its own replica, the job's time is the slowest rank's, and the value sums all ranks' work."""
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    sys.path.insert(0, ROOT)
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port), "RANK": str(rank),
                       "WORLD_SIZE": str(world), "LOCAL_RANK": str(rank)})
    import datetime

    import bench

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        local_ms = [120.0, 150.0][rank]
        value, slowest = bench.weak_scaling_value(1e12, 100, local_ms, world)
        assert bench.dist_info() == (world, rank, rank)
        q.put((rank, value, slowest))
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_weak_scaling_aggregation_two_ranks_gloo():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    res = sorted(q.get(timeout=10) for _ in range(2))
    for rank, value, slowest in res:
        assert slowest == 150.0  # max over ranks
        assert value == pytest.approx(2 * 1e12 * 100 / 0.150 / 1e12)  # both ranks' work / slowest time


def test_single_rank_value_is_local():
    sys.path.insert(0, ROOT)
    import bench

    value, slowest = bench.weak_scaling_value(2e12, 10, 50.0, 1)
    assert slowest == 50.0 and value == pytest.approx(2e12 * 10 / 0.05 / 1e12)
