"""The multi-rank timing logic of bench.py (replicas, max over ranks) on two
gloo ranks on the CPU."""
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
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [10.0 + 5 * rank, 100.0 - rank]          # rank 1 is slower on the first timer
        out[rank] = bench.max_over_ranks(local, torch.device("cpu"))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0] == res[1] == [15.0, 100.0]


def test_weak_scaling_throughput():
    # 2 ranks x 32768 tokens x 10 steps in 1 s of the slowest rank
    assert bench.weak_scaling_throughput(2, 32768, 10, 1000.0) == pytest.approx(655360.0)
    assert bench.weak_scaling_throughput(1, 32768, 10, 2000.0) == pytest.approx(163840.0)
