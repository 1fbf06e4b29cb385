"""The N > 1 path of bench.py on CPU: two gloo ranks, each timing its own independent problem.
Checks the max-over-ranks reduction of step times and the whole-job throughput."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, results):
    import datetime
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        mine = [10.0 + rank, 5.0 - rank, 1.0 * (rank + 1)]      # per-rank step times (ms)
        got = bench.reduce_max_over_ranks(mine, world)
        value = bench.job_tflops(2.0e13, world, got[0])
        results[rank] = (got, value)
    finally:
        dist.destroy_process_group()


def test_two_ranks_reduce_and_aggregate():
    world = 2
    port = _free_port()
    manager = mp.Manager()
    results = manager.dict()
    mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
    for r in range(world):
        got, value = results[r]
        assert got == [11.0, 5.0, 2.0]                          # element-wise max over ranks
        assert value == pytest.approx(2 * 2.0e13 / 11e-3 / 1e12)


def test_single_rank_is_identity():
    import sys
    sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
    import bench
    assert bench.reduce_max_over_ranks([3.0, 1.0], 1) == [3.0, 1.0]
    assert bench.job_tflops(1e12, 1, 1000.0) == pytest.approx(1.0)
