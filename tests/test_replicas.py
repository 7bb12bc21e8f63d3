"""The multi-GPU bench runs independent replicas (the path does not shard):
its only cross-rank steps are a barrier and the max over ranks of the times.
Checked here with two gloo ranks on the CPU."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        t = 1.0 + rank  # rank 1 is the slower one
        out[rank] = bench.dist_max(t, world)
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def test_max_over_two_gloo_ranks():
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    ctx = mp.get_context("spawn")
    procs = [ctx.Process(target=_rank, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert out[0] == out[1] == 2.0


def test_replica_value_is_weak_scaling_aggregate():
    assert bench.replica_value(100.0, 2.0, 1) == 50.0
    assert bench.replica_value(100.0, 2.0, 4) == 200.0


def test_single_rank_needs_no_process_group():
    assert bench.dist_max(3.5, 1) == 3.5
    bench.barrier(1)
