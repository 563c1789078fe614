"""The bench's multi-rank plumbing on CPU: two gloo ranks, each timing its
own replica of the work (weak scaling, no collective on the data path);
the job time is the max over ranks and only rank 0 reports."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        local_ms = 10.0 * (rank + 1)          # rank 1 is the slow one
        ms = bench.max_over_ranks(local_ms, world)
        value = bench.weak_scaling_value(65536.0, world, ms)
        out[rank] = (ms, value)
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_take_the_max():
    world = 2
    port = _free_port()
    with mp.Manager() as mgr:
        out = mgr.dict()
        mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0] == res[1]                   # every rank sees the same job time
    ms, value = res[0]
    assert ms == 20.0                          # the slowest rank's time
    assert value == pytest.approx(2 * 65536 / 0.020)


def test_reference_arm_only_rank0_reports(monkeypatch):
    """Under torchrun the reference arm runs on rank 0 only."""
    class A:
        steps, warmup = 1, 0
    assert bench.run_reference(A(), 2, 1) is None
