"""GPU parity on the five layer workloads at their full sizes, in the launch
configuration the benchmark times.

Small workloads are compared element by element with the full fp64 oracle.
At 8K/16K tokens the oracle evaluates sampled query rows (O, LSE, dQ) and
sampled key columns (dK, dV) of a few heads exactly, one by one, and the
table gradients element by element in full: every head's bias gradient of
the T5 layer, the shared daQ / daK of the Shaw layer summed over all twelve
heads, and the per-head daQ and db of the first and last Transformer-XL
head, each from the oracle's Eq. (4) sums over all query rows.
"""
import numpy as np
import pytest
import torch

import oracle as orc
from synth import make_workload
from relpos_harness import (TOL_GRAD_RELF, TOL_LSE_MAXABS, TOL_O_MAXABS, TOL_O_RELF, check_backward, check_forward,
                            lse_err, maxabs, omap, relf, run_library, run_oracle)

pytestmark = pytest.mark.gpu


def _f64(t):
    return None if t is None else t.double().numpy()


def _sample_rows(N, seed, k=24):
    rng = np.random.default_rng(seed)
    fixed = [0, 1, 127, 128, 129, N // 2, N - 129, N - 128, N - 2, N - 1]
    return np.unique(np.concatenate([fixed, rng.choice(N, size=k, replace=False)]))


def _table(t, h):
    if t is None:
        return None
    return t[h] if t.ndim == 3 else t


def _report(name, errs):
    print(f"{name}: " + " ".join(f"{k}={v:.2g}" for k, v in errs.items()))


def test_config_shaw_clip16_n256_full():
    w = make_workload("shaw_clip16_n256")
    got, want = run_library(w), run_oracle(w)
    o_rel, o_abs = check_forward(got, want, w.name)
    _report(w.name + " (full)", dict(o_relF=o_rel, o_maxabs=o_abs, lse_maxabs=lse_err(got["lse"], want["lse"]),
                                     **check_backward(got, want, w.name)))


def test_config_deberta_log256_n2048_full():
    w = make_workload("deberta_log256_n2048")
    got, want = run_library(w), run_oracle(w)
    o_rel, o_abs = check_forward(got, want, w.name)
    _report(w.name + " (full)", dict(o_relF=o_rel, o_maxabs=o_abs, lse_maxabs=lse_err(got["lse"], want["lse"]),
                                     **check_backward(got, want, w.name)))


def _sampled_check(w, got, heads, out_f32_note=""):
    m = omap(w)
    q, k, v, do = (_f64(getattr(w, n)) for n in ("q", "k", "v", "do"))
    aq, ak, b = _f64(w.aq), _f64(w.ak), _f64(w.b)
    kl = None if w.key_len is None else w.key_len.numpy()
    rows = _sample_rows(w.N, 1)
    cols = _sample_rows(w.N, 2)
    for bi in range(w.B):
        for h in heads:
            ref = orc.head_grads_sampled(q[bi, h], k[bi, h], v[bi, h], do[bi, h], _table(aq, h), _table(ak, h),
                                         None if b is None else b[h], w.tau, m, w.causal,
                                         None if kl is None else kl[bi], rows, cols)
            ctx = f"{w.name} b={bi} h={h}"
            o = got["o"][bi, h][rows]
            errs = dict(o_relF=relf(o, ref["o"][rows]), o_maxabs=maxabs(o, ref["o"][rows]),
                        lse_maxabs=lse_err(got["lse"][bi, h][rows], ref["lse"][rows]),
                        dq=relf(got["dq"][bi, h][rows], ref["dq"]), dk=relf(got["dk"][bi, h][cols], ref["dk"]),
                        dv=relf(got["dv"][bi, h][cols], ref["dv"]))
            _report(ctx + " (sampled rows)", errs)
            assert errs["o_relF"] <= TOL_O_RELF and errs["o_maxabs"] <= TOL_O_MAXABS, ctx
            assert errs["lse_maxabs"] <= TOL_LSE_MAXABS, ctx
            for n in ("dq", "dk", "dv"):
                assert errs[n] <= TOL_GRAD_RELF, ctx + " " + n


def _table_grads_full(w, heads):
    """Oracle table gradients of the whole workload, element by element: the
    Eq. (4) sums over every query row of each (batch, head) slice, accumulated
    block by block (oracle.head_table_grads).  Shared tables are summed over
    batch and heads in ascending order; per-head tables and the bias keep their
    head index (only `heads` are computed)."""
    m = omap(w)
    q, k, v, do = (_f64(getattr(w, n)) for n in ("q", "k", "v", "do"))
    aq, ak, b = _f64(w.aq), _f64(w.ak), _f64(w.b)
    kl = None if w.key_len is None else w.key_len.numpy()
    shared = {n: t is not None and t.ndim == 2 for n, t in (("daq", aq), ("dak", ak))}
    out = {}
    for h in heads:
        for bi in range(w.B):
            g = orc.head_table_grads(q[bi, h], k[bi, h], v[bi, h], do[bi, h], _table(aq, h), _table(ak, h),
                                     None if b is None else b[h], w.tau, m, w.causal,
                                     None if kl is None else kl[bi])
            for n, val in g.items():
                key = n if shared.get(n) else (n, h)
                out[key] = val if key not in out else out[key] + val
    return out


def _check_table_grads(got, want, ctx):
    for key, ref in want.items():
        name, h = (key, None) if isinstance(key, str) else key
        g = got[name] if h is None else got[name][h]
        e_rel, e_abs = relf(g, ref), maxabs(g, ref)
        print(f"{ctx} {name}{'' if h is None else f'[h={h}]'}: relF={e_rel:.3g} maxabs={e_abs:.3g} "
              f"(max |ref| {np.abs(ref).max():.3g})")
        assert e_rel <= TOL_GRAD_RELF, (ctx, key, e_rel)


def test_config_t5_bucket32_n8192_sampled():
    w = make_workload("t5_bucket32_n8192")
    got = run_library(w)
    _sampled_check(w, got, heads=[0, w.H - 1])
    # every head's bias gradient, element by element
    _check_table_grads(got, _table_grads_full(w, range(w.H)), w.name)


def test_config_shaw_clip64_n8192_sampled():
    w = make_workload("shaw_clip64_n8192")
    got = run_library(w)
    _sampled_check(w, got, heads=[0, w.H - 1])
    # the shared daQ / daK summed over all 12 heads, element by element
    _check_table_grads(got, _table_grads_full(w, range(w.H)), w.name)


def test_config_txl_identity_causal_n16384_sampled():
    w = make_workload("txl_identity_causal_n16384")
    got = run_library(w, out_f32=True)     # bf16 workload: O judged in fp32
    _sampled_check(w, got, heads=[0])
    # per-head daQ [32767, 64] and db [32767] of the first and last head in full
    _check_table_grads(got, _table_grads_full(w, [0, w.H - 1]), w.name)
