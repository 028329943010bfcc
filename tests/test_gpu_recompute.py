"""Projection recomputed inside every tile (projection="recompute"; [digest]
ablation "projection precompute" and limitations section: storing the
identity map's projection is quadratic, recomputing it per tile keeps the
forward's memory linear).  The forward is compared with the fp64 oracle on
small and ragged cases of every map, with both masks, both dtypes, shared and
per-head tables and dropout, and on sampled rows of the 16K Transformer-XL
layer; the backward of a recomputing forward (which rebuilds Z^Q) is checked
in full on the small cases.
"""
import numpy as np
import pytest
import torch

import oracle as orc
from synth import make_workload, small_workload
from relpos_harness import (TOL_LSE_MAXABS, TOL_O_MAXABS, TOL_O_RELF, check_backward, check_forward, lmap, lse_err,
                            maxabs, omap, relf, run_oracle, to_dev)
import exact_relative_position_b200 as rp

pytestmark = pytest.mark.gpu

CASES = {
    "identity_520": dict(map_kind="identity", N=520, B=1, H=2, terms=("aQ", "b")),
    "identity_520_causal_aq": dict(map_kind="identity", N=520, B=2, H=2, terms=("aQ",), causal=True),
    "identity_777_bf16_per_head": dict(map_kind="identity", N=777, B=1, H=2, terms=("aQ", "b"),
                                       dtype=torch.bfloat16, per_head_tables=True, causal=True),
    "identity_1": dict(map_kind="identity", N=1, B=1, H=1, terms=("aQ", "b")),
    "identity_127_padding": dict(map_kind="identity", N=127, B=2, H=1, terms=("aQ", "b"), key_len=[127, 40]),
    "trunc16_300": dict(map_kind="truncated", clip=16, N=300, B=2, H=2, terms=("aQ",), key_len=[300, 211]),
    "trunc200_600": dict(map_kind="truncated", clip=200, N=600, B=1, H=3, terms=("aQ", "b"), per_head_tables=True),
    "t5_400_bias": dict(map_kind="t5", num_buckets=32, max_distance=128, bidirectional=1, N=400, B=1, H=2,
                        terms=("b",)),
    "log_1000": dict(map_kind="log", num_buckets=32, max_distance=128, N=1000, B=1, H=2, terms=("aQ", "b"),
                     causal=True),
}


def _run(w, projection, backward=True, out_f32=False, dropout=(0.0, 0, 0)):
    dev = to_dev(w)
    kw = dict(tau=w.tau, map=lmap(w), causal=w.causal, key_len=dev["key_len"], projection=projection,
              dropout_p=dropout[0], dropout_seed=dropout[1], dropout_offset=dropout[2])
    fws, bws = rp.workspace_size(dev["q"], dev["aq"], dev["ak"], dev["b"], w.tau, lmap(w), causal=w.causal,
                                 key_len=dev["key_len"], out_f32=out_f32, projection=projection)
    ws = torch.empty(max(fws, bws, 256), device="cuda", dtype=torch.uint8)
    o, lse = rp.relpos_attn_fwd(dev["q"], dev["k"], dev["v"], dev["aq"], dev["ak"], dev["b"], workspace=ws,
                                out_f32=out_f32, **kw)
    res = dict(o=o, lse=lse)
    if backward:
        g = rp.relpos_attn_bwd(dev["do"], dev["q"], dev["k"], dev["v"], o, lse, dev["aq"], dev["ak"], dev["b"],
                               workspace=ws, reuse_forward=True, **kw)
        res.update(zip(("dq", "dk", "dv", "daq", "dak", "db"), g))
    torch.cuda.synchronize()
    assert rp.check_workspace(ws) == 0
    return {k: (None if v is None else v.detach().double().cpu().numpy()) for k, v in res.items()}, fws


@pytest.mark.parametrize("case", sorted(CASES))
def test_recompute_matches_oracle(case):
    w = small_workload(**CASES[case])
    out_f32 = w.dtype == torch.bfloat16
    got, _ = _run(w, "recompute", out_f32=out_f32)
    want = run_oracle(w)
    check_forward(got, want, case)
    check_backward(got, want, case)
    # the same layer with the stored projection agrees to rounding
    ret, _ = _run(w, "retained", backward=False, out_f32=out_f32)
    assert relf(got["o"], ret["o"]) <= 1e-3


def test_recompute_with_dropout():
    w = small_workload(map_kind="identity", N=300, B=1, H=2, terms=("aQ", "b"), causal=True)
    drop = (0.125, 1234, 7)
    got, _ = _run(w, "recompute", dropout=drop)
    want = run_oracle(w, dropout=drop)
    check_forward(got, want, "recompute dropout")
    check_backward(got, want, "recompute dropout")


def test_recompute_rejects_key_side_term():
    w = small_workload(map_kind="identity", N=200, terms=("aQ", "aK"))
    dev = to_dev(w)
    with pytest.raises(rp.RelPosError, match="unsupported"):
        rp.relpos_attn_fwd(dev["q"], dev["k"], dev["v"], dev["aq"], dev["ak"], None, tau=w.tau, map=lmap(w),
                           projection="recompute")


def test_recompute_txl_identity_causal_n16384_sampled():
    """The 16K Transformer-XL layer with a linear-memory forward: O and LSE on
    sampled rows of the first and last head against the oracle (fp32 O)."""
    w = make_workload("txl_identity_causal_n16384")
    got, fws = _run(w, "recompute", backward=False, out_f32=True)
    assert fws < w.B * w.H * w.N * 64 * 4      # less than one fp32 copy of Q: no projection stored
    m = omap(w)
    rng = np.random.default_rng(3)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, 8191, 16256, 16383], rng.choice(w.N, 24, replace=False)]))
    f64 = lambda t: t.double().numpy()
    for h in (0, w.H - 1):
        O, L = orc.forward(w.q[:, h:h + 1], w.k[:, h:h + 1], w.v[:, h:h + 1], w.aq[h:h + 1], None,
                           w.b[h:h + 1], w.tau, m, causal=True, rows=rows)
        o = got["o"][0, h][rows]
        assert relf(o, O[0, 0]) <= TOL_O_RELF and maxabs(o, O[0, 0]) <= TOL_O_MAXABS, h
        assert lse_err(got["lse"][0, h][rows], L[0, 0]) <= TOL_LSE_MAXABS, h
