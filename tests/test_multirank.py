"""The N > 1 path of bench.py on CPU: two gloo ranks (the path has no data
exchange; each rank runs a replica, and rank 0 reports the whole-job value
over the slowest rank's device time)."""
import os
import socket
import sys

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, local_ms, out):
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    import bench
    try:
        ms = bench.max_over_ranks(local_ms[rank], world, "cpu")
        out[rank] = (ms, bench.whole_job_value(world, 100, ms))
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("local_ms", [(12.5, 20.0), (30.0, 7.25)])
def test_two_ranks_take_the_slowest_time(local_ms):
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    port = _free_port()
    mp.start_processes(_rank, args=(world, port, local_ms, out), nprocs=world, join=True, start_method="spawn")
    slow = max(local_ms)
    for r in range(world):
        ms, value = out[r]
        assert ms == slow                                     # every rank sees the max
        assert value == pytest.approx(world * 100 / (slow / 1e3))   # units of all ranks / slowest time


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.5, 1, "cpu") == 3.5
    assert bench.whole_job_value(1, 50, 10.0) == pytest.approx(5000.0)
