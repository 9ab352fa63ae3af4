"""Host logic of the multi-GPU bench path, on CPU: two gloo ranks agree on
the slowest rank's time, and whole-job throughput is weak-scaled."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as tmp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local_ms = 100.0 + 37.0 * rank          # rank 1 is the slow one
        bench._barrier(dist)
        out[rank] = bench._max_over_ranks(dist, local_ms)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    world = 2
    out = tmp.get_context("spawn").Manager().dict()
    tmp.start_processes(_rank, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    assert dict(out) == {0: 137.0, 1: 137.0}


def test_weak_scaling_throughput_and_single_rank():
    assert bench._max_over_ranks(None, 12.5) == 12.5
    one = bench._throughput(1, 5e14, 1000.0)
    assert one == pytest.approx(500.0)
    assert bench._throughput(4, 5e14, 1000.0) == pytest.approx(4 * one)
