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


# ------------------------------------------------- shared-table gradient exchange

def _partials(rank):
    g = torch.Generator().manual_seed(100 + rank)
    daq = torch.randn(129, 64, generator=g)
    db = torch.randn(12, 129, generator=g)
    return daq, db


def _ascending_sum(gathered):
    """CPU stand-in for the library's relpos_sum_partials (same order)."""
    acc = gathered[0].clone()
    for r in range(1, gathered.shape[0]):
        acc += gathered[r]
    return acc


def _exchange_worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from exact_relative_position_b200.data_parallel import reduce_table_grads
        daq, db = _partials(rank)
        got = reduce_table_grads([daq, None, db], sum_partials=_ascending_sum)
        assert got[1] is None and got[0] is daq and got[2] is db
        out[rank] = (daq.clone(), db.clone())
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_reduce_table_grads_two_gloo_ranks():
    world, port = 2, _free_port()
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    procs = [ctx.Process(target=_exchange_worker, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    want = [a + b for a, b in zip(_partials(0), _partials(1))]
    for r in range(world):
        for got, w in zip(out[r], want):
            assert torch.equal(got, w)                  # rank 0's partial first, then rank 1's
    assert all(torch.equal(a, b) for a, b in zip(out[0], out[1]))   # identical bits on every rank
