"""Multi-process host logic of the replica benchmark (gloo, world size 2, CPU):
the timed region's max over ranks and the whole-job throughput."""
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


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    # rank r "took" 10 * (r + 1) ms for 5 steps of 1e12 units each
    ms = bench.max_over_ranks(10.0 * (rank + 1), dist, "cpu")
    value = bench.aggregate_throughput(1e12, 5, ms, world)
    out[rank] = (ms, value)
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_and_aggregate_with_two_gloo_ranks():
    world = 2
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    for r in range(world):
        ms, value = out[r]
        assert ms == 20.0                       # the slowest rank's time, on every rank
        assert value == pytest.approx(2 * 1e12 * 5 / 0.020)


def test_single_process_is_identity():
    import bench
    assert bench.max_over_ranks(3.5, None, "cpu") == 3.5
    assert bench.aggregate_throughput(2.0, 4, 1000.0, 1) == pytest.approx(8.0)
