"""Host logic of the replicated multi-GPU benchmark, exercised with two gloo ranks on the CPU:
the rank environment, the max-over-ranks of the per-rank device time, and the whole-job
aggregation (all ranks' query tokens over the slowest rank's time)."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      LOCAL_RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, lr, w = bench._dist_env()
        assert (r, lr, w) == (rank, rank, world)
        my_time = 1.0 + rank            # rank 1 is the slower replica
        t = bench.max_over_ranks(my_time, world, device="cpu")
        value = bench.aggregate(units_per_rank=64 * 10, max_time_s=t, world=world)
        out[rank] = (t, value)
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_aggregate():
    world, port = 2, _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    for rank in range(world):
        t, value = out[rank]
        assert t == 2.0                           # every rank sees the slowest time
        assert value == pytest.approx(64 * 10 * 2 / 2.0)


def test_single_process_is_identity():
    assert bench.max_over_ranks(3.5, 1) == 3.5
    assert bench.aggregate(100, 2.0, 1) == 50.0
