"""The data-parallel exchange on one GPU: the library's ascending-rank sum
against the same additions in PyTorch (bit-exact: the same fp32 adds in the
same order), its argument checks, and a two-way batch split whose exchanged
table gradients equal those of the unsplit batch and of the fp64 oracle."""
import numpy as np
import pytest
import torch
import torch.distributed as dist

import exact_relative_position_b200 as rp
from exact_relative_position_b200.data_parallel import reduce_table_grads
from synth import small_workload

from relpos_harness import lmap, run_oracle, relf

pytestmark = pytest.mark.gpu


def _ascending(p):
    acc = p[0].clone()
    for r in range(1, p.shape[0]):
        acc += p[r]
    return acc


@pytest.mark.parametrize("world,n", [(1, 5), (2, 33), (3, 1000), (8, 129 * 64 + 12 * 129 + 7), (5, 300001)])
def test_sum_partials_bit_exact(world, n):
    g = torch.Generator(device="cuda").manual_seed(world * 1000 + n)
    p = torch.randn(world, n, device="cuda", generator=g) * torch.logspace(-3, 3, n, device="cuda")
    want = _ascending(p)
    got = rp.sum_partials(p)
    assert torch.equal(got, want)
    # in place into row 0
    q = p.clone()
    rp.sum_partials(q, out=q[0])
    assert torch.equal(q[0], want)
    assert torch.equal(q[1:], p[1:])


def test_sum_partials_edge_cases():
    p = torch.empty(3, 0, device="cuda")
    assert rp.sum_partials(p).numel() == 0
    p = torch.randn(3, 64, device="cuda")
    with pytest.raises(rp.RelPosError):
        rp.sum_partials(p, out=p[1])                 # overlaps a row that is still to be read
    lib = rp.lib()
    assert lib.relpos_sum_partials(p.data_ptr(), 0, 64, p.data_ptr(), None) == -1   # world < 1
    assert lib.relpos_sum_partials(p.data_ptr(), 3, -1, p.data_ptr(), None) == -1   # n < 0
    assert lib.relpos_sum_partials(p.data_ptr() + 2, 3, 60, p[0].data_ptr(), None) == -1   # misaligned


def _grads(w, b0, b1):
    """Table gradients of batch elements b0 .. b1 - 1 through the library."""
    sl = lambda t: None if t is None else t[b0:b1].to("cuda").contiguous()
    dv = lambda t: None if t is None else t.to("cuda").contiguous()
    q, k, v, do = sl(w.q), sl(w.k), sl(w.v), sl(w.do)
    aq, ak, b = dv(w.aq), dv(w.ak), dv(w.b)
    o, lse = rp.relpos_attn_fwd(q, k, v, aq, ak, b, tau=w.tau, map=lmap(w), causal=w.causal)
    _, _, _, daq, dak, db = rp.relpos_attn_bwd(do, q, k, v, o, lse, aq, ak, b, tau=w.tau, map=lmap(w),
                                               causal=w.causal)
    return [daq, dak, db]


def test_batch_split_exchange_equals_whole_batch(tmp_path):
    # shared aQ / aK across the batch, bias per head: all three need the exchange
    w = small_workload(B=2, H=2, N=300, terms=("aQ", "aK", "b"), seed=7)
    whole = _grads(w, 0, 2)
    parts = [_grads(w, 0, 1), _grads(w, 1, 2)]
    # what two ranks would do: gather the partials in rank order, add ascending
    summed = [rp.sum_partials(torch.stack([a.reshape(-1), b.reshape(-1)])).view_as(a) for a, b in zip(*parts)]
    want = run_oracle(w)
    for name, got, full in zip(("daq", "dak", "db"), summed, whole):
        assert relf(got.double().cpu().numpy(), full.double().cpu().numpy()) <= 1e-5, name
        assert relf(got.double().cpu().numpy(), want[name]) <= 1e-2, name

    # the same through reduce_table_grads and NCCL, with a one-rank group
    dist.init_process_group("nccl", init_method=f"file://{tmp_path}/store", rank=0, world_size=1)
    try:
        mine = [t.clone() for t in parts[0]]
        reduce_table_grads(mine)
        torch.cuda.synchronize()
        for a, b in zip(mine, parts[0]):
            assert torch.equal(a, b)              # one rank: the sum is its own partial
    finally:
        dist.destroy_process_group()
    assert np.isfinite(summed[0].cpu().numpy()).all()
