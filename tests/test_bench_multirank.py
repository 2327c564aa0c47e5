"""Host-side multi-rank logic of bench.py on CPU (gloo, world size 2): the
step time is the max over ranks, the value is whole-job (weak scaling),
and the reference arm runs on rank 0 only."""

import os
import sys

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    sys.path.insert(0, ROOT)
    import bench
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 3.0], torch.device("cpu"))
        out[rank] = got
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo():
    world = 2
    port = 29500 + os.getpid() % 1000
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        for r in range(world):
            assert out[r] == [2.0, 10.0, 3.0]


def test_weak_scaling_value_and_single_rank_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.weak_scaling_value(4, 7e12, 7.0) == pytest.approx(4000.0)
    assert bench.max_over_ranks([5.0, 6.0], torch.device("cpu")) == [5.0, 6.0]


def test_reference_arm_only_on_rank0(monkeypatch, capsys):
    sys.path.insert(0, ROOT)
    import bench

    class Args:
        workload = "tiny"
        steps = 1
        warmup = 0

    assert bench.run_reference(Args(), rank=1, world=2) == 0
    assert capsys.readouterr().out == ""
