"""The N > 1 host path of the benchmark on CPU: two gloo ranks, each timing
its own replica, report the maximum over ranks (the layer has no data-path
exchange; replicas are independent)."""
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
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # rank r "measured" (1 + r, 10 - r, 0.5 * r) ms
        got = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 0.5 * rank])
        out[rank] = got
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    for r in range(world):
        assert list(out[r]) == [2.0, 10.0, 0.5]


def test_max_over_ranks_without_group_is_identity():
    assert not (dist.is_available() and dist.is_initialized())
    assert bench.max_over_ranks([3.0, 4.0]) == [3.0, 4.0]
