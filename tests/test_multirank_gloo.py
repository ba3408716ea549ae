"""Multi-rank timing aggregation of bench.py on CPU ranks (gloo, world size 2).

bench.py --gpus N runs N replicas of the per-rank workload (weak scaling, no
collective on the data path); the reported time is the slowest rank's and the
value counts every rank's units.
"""

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
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank          # rank 1 is the slow one
        ms = bench.max_over_ranks(local_ms)
        rate = bench.whole_job_rate(1000.0, world, ms)
        dist.barrier()
        results[rank] = (ms, rate)
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2])
def test_max_over_ranks_and_whole_job_rate(world):
    port = _free_port()
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_worker, args=(world, port, results), nprocs=world, join=True)
        out = dict(results)
    slowest = 10.0 + 5.0 * (world - 1)
    for rank in range(world):
        ms, rate = out[rank]
        assert ms == slowest                               # every rank sees the max
        assert rate == pytest.approx(world * 1000.0 / (slowest * 1e-3))


def test_single_rank_is_identity():
    import bench
    assert bench.max_over_ranks(3.5) == 3.5
    assert bench.whole_job_rate(10.0, 1, 2.0) == pytest.approx(5000.0)
