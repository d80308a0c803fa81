"""Multi-process host logic of the benchmark on CPU (gloo, world size 2):
each rank runs its own batch (no data-path collective); the job's step time
is the max over ranks and its throughput counts every rank's work."""
import os
import socket
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, results):
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        bench._barrier(world)
        ms_local = 1.0 + rank            # rank 1 is the slow one
        ms, value = bench.job_throughput(ms_local, world, bench.FLOP_STEP)
        results[rank] = (ms, value)
        bench._barrier(world)
    finally:
        dist.destroy_process_group()


def test_weak_scaling_aggregation_two_ranks():
    world, port = 2, _free_port()
    with mp.Manager() as mgr:
        results = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, results), nprocs=world, join=True)
        results = dict(results)
    sys.path.insert(0, ROOT)
    import bench
    for rank in range(world):
        ms, value = results[rank]
        assert ms == 2.0                                   # slowest rank
        assert value == pytest.approx(world * bench.FLOP_STEP / 2e-3 / 1e12)


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    ms, value = bench.job_throughput(0.5, 1, bench.FLOP_STEP)
    assert ms == 0.5 and value == pytest.approx(bench.FLOP_STEP / 0.5e-3 / 1e12)
