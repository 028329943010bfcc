"""Failure detection: a bounded wait in the fused kernels that runs out.

The host lowers the kernels' wait limit to 1 ns (relpos_set_wait_limit_ns),
so the first wait that does not succeed at once gives up.  The kernel then
flags the abort, drains the TMA loads and MMAs it issued, frees its tensor
memory and returns; the status word reports RELPOS_ERR_TIMEOUT.  Afterwards
the same context must run a normal call with a clean status and correct
results.  No GPU fault is involved: every wait is bounded.
"""
import pytest
import torch

from synth import make_workload
from relpos_harness import check_backward, check_forward, lmap, run_oracle, to_dev
import exact_relative_position_b200 as rp
from exact_relative_position_b200 import _binding as bd

pytestmark = pytest.mark.gpu


def _calls(w, dev, ws, projection="retained"):
    kw = dict(tau=w.tau, map=lmap(w), causal=w.causal, key_len=dev["key_len"], projection=projection)
    o, lse = rp.relpos_attn_fwd(dev["q"], dev["k"], dev["v"], dev["aq"], dev["ak"], dev["b"], workspace=ws, **kw)
    fwd_status = _status(ws)
    grads = rp.relpos_attn_bwd(dev["do"], dev["q"], dev["k"], dev["v"], o, lse, dev["aq"], dev["ak"], dev["b"],
                               workspace=ws, **kw)
    bwd_status = _status(ws)
    return o, lse, grads, fwd_status, bwd_status


def _status(ws):
    try:
        return rp.check_workspace(ws)
    except bd.RelPosError as e:
        assert "timed out" in str(e)
        return -5


@pytest.mark.parametrize("projection", ["retained", "recompute"])
def test_wait_limit_expiry_reports_timeout_then_recovers(projection):
    w = make_workload("shaw_clip16_n256")     # q.aQ only: both projection modes apply
    dev = to_dev(w)
    f, b = rp.workspace_size(dev["q"], dev["aq"], dev["ak"], dev["b"], w.tau, lmap(w), projection=projection)
    ws = torch.empty(max(f, b), device="cuda", dtype=torch.uint8)
    try:
        bd.set_wait_limit_ns(1)
        _, _, _, fwd_status, bwd_status = _calls(w, dev, ws, projection)
    finally:
        bd.set_wait_limit_ns(0)
    assert fwd_status == -5 and bwd_status == -5
    # same device, same workspace, default limit: clean status, correct results
    o, lse, (dq, dk, dv, daq, dak, db), fwd_status, bwd_status = _calls(w, dev, ws, projection)
    assert fwd_status == 0 and bwd_status == 0
    f64 = lambda t: None if t is None else t.double().cpu().numpy()
    got = dict(o=f64(o), lse=f64(lse), dq=f64(dq), dk=f64(dk), dv=f64(dv), daq=f64(daq), dak=f64(dak), db=f64(db))
    want = run_oracle(w)
    check_forward(got, want, "after timeout")
    check_backward(got, want, "after timeout")
