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


def test_zero_fractions_of_a_step():
    """bench.zero_fractions on CPU tensors shaped and typed like a Layer's
    buffers: counts zero codes per projection input and non-positive gates."""
    from types import SimpleNamespace
    m, f, d = 4, 8, 16
    o8 = torch.ones((m, d), dtype=torch.int8)
    o8[:, ::2] = 0                                            # half zeros
    h8 = torch.zeros((m, f), dtype=torch.int8)
    h8[0, 0] = 5                                              # 31 of 32 zeros
    up = torch.full((m, f), 1.0, dtype=torch.bfloat16)
    gate = torch.tensor([[-1.0, 0.0, -0.0, 2.0] * 2] * m, dtype=torch.bfloat16)   # 3 of 4 zeroed by ReLU
    y_ug = torch.cat([up, gate], dim=1).view(torch.int16)
    qa = torch.zeros((m, d), dtype=torch.uint8)
    qf = torch.full((m, d), 3, dtype=torch.uint8)
    layer = SimpleNamespace(o8=o8, h8=h8, y_ug=y_ug, f=f, qa=qa, qf=qf, afmt="int4")
    z = bench.zero_fractions(torch, layer)
    assert z == {"o_input": 0.5, "down_input": round(31 / 32, 4), "gate_relu_zero": 0.75,
                 "qkv_input": 1.0, "upgate_input": 0.0, "down_groups_over_2of4": 0.0}
    layer.afmt = "fp4"
    assert set(bench.zero_fractions(torch, layer)) == {"o_input", "down_input", "gate_relu_zero",
                                                        "down_groups_over_2of4"}
    # two 128-row tiles of 8 columns: tile 0 has nonzeros in columns 0, 1, 3 (row 5)
    # and 6 (row 77), tile 1 in column 2 only (row 200), so 4 + 7 = 11 of the 16
    # (tile, column) pairs are all zero; row 5's first group of four holds three
    # nonzeros (1 of the 512 groups breaks 2:4)
    layer.h8 = torch.zeros((256, 8), dtype=torch.int8)
    layer.h8[5, 0], layer.h8[5, 1], layer.h8[5, 3] = -3, 1, 1
    layer.h8[77, 6] = 9
    layer.h8[200, 2] = 4
    z = bench.zero_fractions(torch, layer)
    assert z["down_all_zero_k_columns_per_128_rows"] == round(11 / 16, 4)
    assert z["down_groups_over_2of4"] == round(1 / 512, 4)
