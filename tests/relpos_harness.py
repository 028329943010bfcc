"""Shared helpers of the GPU parity tests: run a synthetic workload through the
CUDA library (C ABI) and through the fp64 oracle, and compare.

Tolerances (fp16/bf16 inputs, fp32 accumulation): O relative Frobenius error
<= 2e-3 and max-abs <= 5e-3; every gradient relative Frobenius error <= 1e-2.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle as orc
import exact_relative_position_b200 as rp

TOL_O_RELF = 2e-3
TOL_O_MAXABS = 5e-3
TOL_GRAD_RELF = 1e-2
TOL_LSE_MAXABS = 2e-3


def omap(w):
    return orc.MapDesc(w.map_kind, w.clip, w.num_buckets, w.max_distance, w.bidirectional)


def lmap(w):
    return rp.RelPosMap(w.map_kind, w.clip, w.num_buckets, w.max_distance, w.bidirectional)


def to_dev(w, device="cuda"):
    d = lambda t: None if t is None else t.to(device).contiguous()
    return dict(q=d(w.q), k=d(w.k), v=d(w.v), do=d(w.do), aq=d(w.aq), ak=d(w.ak), b=d(w.b), key_len=d(w.key_len))


def run_library(w, backward=True, out_f32=False, dev=None, dropout=(0.0, 0, 0)):
    dev = dev or to_dev(w)
    dkw = dict(dropout_p=dropout[0], dropout_seed=dropout[1], dropout_offset=dropout[2])
    o, lse = rp.relpos_attn_fwd(dev["q"], dev["k"], dev["v"], dev["aq"], dev["ak"], dev["b"], tau=w.tau,
                                map=lmap(w), causal=w.causal, key_len=dev["key_len"], out_f32=out_f32, **dkw)
    res = dict(o=o, lse=lse)
    if backward:
        dq, dk, dv, daq, dak, db = rp.relpos_attn_bwd(dev["do"], dev["q"], dev["k"], dev["v"], o, lse, dev["aq"],
                                                      dev["ak"], dev["b"], tau=w.tau, map=lmap(w), causal=w.causal,
                                                      key_len=dev["key_len"], **dkw)
        res.update(dq=dq, dk=dk, dv=dv, daq=daq, dak=dak, db=db)
    torch.cuda.synchronize()
    return {k: (None if v is None else v.detach().double().cpu().numpy()) for k, v in res.items()}


def run_oracle(w, backward=True, dropout=(0.0, 0, 0)):
    kl = None if w.key_len is None else w.key_len.numpy()
    # the library receives the rate as float32: the oracle takes that value
    dkw = dict(dropout_p=float(np.float32(dropout[0])), dropout_seed=dropout[1], dropout_offset=dropout[2])
    if backward:
        return orc.backward(w.q, w.k, w.v, w.do, w.aq, w.ak, w.b, w.tau, omap(w), causal=w.causal, key_len=kl, **dkw)
    O, L = orc.forward(w.q, w.k, w.v, w.aq, w.ak, w.b, w.tau, omap(w), causal=w.causal, key_len=kl, **dkw)
    return dict(o=O, lse=L)


def relf(got, want):
    den = np.linalg.norm(want)
    return float(np.linalg.norm(got - want) / (den if den > 0 else 1.0))


def maxabs(got, want):
    return float(np.max(np.abs(got - want))) if got.size else 0.0


def lse_err(got, want):
    fin = np.isfinite(want)
    assert np.array_equal(np.isfinite(got), fin), "LSE finiteness differs (fully masked rows)"
    assert np.all(got[~fin] == want[~fin])
    return maxabs(got[fin], want[fin])


def check_forward(got, want, ctx=""):
    e_rel, e_abs = relf(got["o"], want["o"]), maxabs(got["o"], want["o"])
    assert e_rel <= TOL_O_RELF and e_abs <= TOL_O_MAXABS, f"{ctx} O relF={e_rel:.3g} maxabs={e_abs:.3g}"
    el = lse_err(got["lse"], want["lse"])
    assert el <= TOL_LSE_MAXABS, f"{ctx} LSE maxabs={el:.3g}"
    return e_rel, e_abs


def check_backward(got, want, ctx=""):
    errs = {}
    for n in ("dq", "dk", "dv", "daq", "dak", "db"):
        if want.get(n) is None:
            assert got.get(n) is None
            continue
        errs[n] = relf(got[n], want[n])
        assert errs[n] <= TOL_GRAD_RELF, f"{ctx} {n} relF={errs[n]:.3g}"
    return errs
