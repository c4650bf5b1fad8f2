"""Host logic of bench.py's replicated multi-GPU run, on CPU: two gloo ranks.

Under torchrun every rank runs its own batch (the path has no data-path
collective); the step time is the max over ranks and the reported value is
world * tokens / that time.  This checks both with world size 2 on CPU.
"""
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


def _rank_main(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 10.0 + 5.0 * rank              # rank 1 is the slower one
        step_ms = bench.reduce_max(local_ms, world, torch.device("cpu"))
        out[rank] = (step_ms, bench.aggregate_value(12800, world, step_ms))
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    world = 2
    port = _free_port()
    manager = mp.Manager()
    out = manager.dict()
    mp.spawn(_rank_main, args=(world, port, out), nprocs=world, join=True)
    assert out[0][0] == out[1][0] == 15.0
    assert out[0][1] == pytest.approx(2 * 12800 / 0.015)


def test_single_rank_is_identity():
    assert bench.reduce_max(7.5, 1, None) == 7.5
    assert bench.aggregate_value(100, 1, 10.0) == pytest.approx(1e4)
