"""Host logic of the multi-GPU bench path, on CPU: two gloo ranks agree on
the slowest rank's time, split one layer by KV-head group so that every
query head is computed exactly once, and whole-job throughput adds up."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as tmp

import bench
from dynamic_sparse_attention_minf_b200 import layer
from dynamic_sparse_attention_minf_b200 import workloads as wl


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


def _shard_rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = wl.config(4)
        hq0, hq1, hk0, hk1 = layer.kv_group_slice(w, rank, world)
        lw = layer.local_workload(w, rank, world)
        mine = {"q": list(range(hq0, hq1)), "kv": list(range(hk0, hk1)), "patterns": lw.patterns,
                "Hq": lw.Hq, "Hkv": lw.Hkv}
        got = [None] * world
        dist.all_gather_object(got, mine)
        # useful work of the whole layer = sum over ranks; time = the slowest rank
        total = torch.tensor([1.0e14 * (rank + 1)], dtype=torch.float64)
        dist.all_reduce(total, op=dist.ReduceOp.SUM)
        out[rank] = (got, float(total.item()), bench._max_over_ranks(dist, 10.0 + rank))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_kv_group_partition_covers_every_head_once(world):
    out = tmp.get_context("spawn").Manager().dict()
    tmp.start_processes(_shard_rank, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    w = wl.config(4)
    for rank in range(world):
        got, total, slowest = out[rank]
        qs = sorted(h for g in got for h in g["q"])
        assert qs == list(range(w.Hq))                       # every query head exactly once
        kvs = sorted(h for g in got for h in g["kv"])
        assert kvs == list(range(w.Hkv))
        for g in got:                                        # whole GQA groups, local ids consistent
            assert all(h // w.group in g["kv"] for h in g["q"])
            assert g["Hq"] == len(g["q"]) == g["Hkv"] * w.group
            assert g["patterns"] == [w.patterns[h] for h in g["q"]]
        assert total == pytest.approx(1.0e14 * world * (world + 1) / 2)
        assert slowest == 10.0 + world - 1


def test_kv_group_slice_rejects_uneven_split():
    w = wl.config(4)
    with pytest.raises(ValueError):
        layer.kv_group_slice(w, 0, 3)
