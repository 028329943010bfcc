"""relpos_attn_fwd_noalloc: the forward for callers that cannot allocate device
memory (a pool or another runtime owns the device and forbids outside
allocations, or an enqueue step must not allocate).  It runs in the library's
fixed 32 MiB scratch array instead of a caller workspace.

Checked through the C ABI against the ordinary workspace forward on two
calls in a row (the scratch array keeps the previous call's contents), with
the tolerances of the other parity tests, and for the clear rejection of
shapes whose workspace does not fit.  Kept in its own file, collected last.
"""
import numpy as np
import pytest
import torch

from synth import small_workload
from relpos_harness import TOL_LSE_MAXABS, TOL_O_MAXABS, TOL_O_RELF, lmap, lse_err, maxabs, relf, to_dev
import exact_relative_position_b200 as rp
from exact_relative_position_b200._binding import NOALLOC_MAX_WORKSPACE, RelPosError

pytestmark = pytest.mark.gpu


def _fwd(fn, w, dev, **extra):
    o, lse = fn(dev["q"], dev["k"], dev["v"], dev["aq"], dev["ak"], dev["b"], tau=w.tau, map=lmap(w),
                causal=w.causal, key_len=dev["key_len"], **extra)
    torch.cuda.synchronize()
    return o.double().cpu().numpy(), lse.double().cpu().numpy()


@pytest.mark.parametrize("first,second", [
    (dict(map_kind="log", num_buckets=32, max_distance=128, N=600, B=2, H=3, terms=("aQ", "aK", "b"),
          key_len=[600, 413], per_head_tables=True),
     dict(map_kind="truncated", clip=16, N=300, B=1, H=2, terms=("aQ",), causal=True)),
])
def test_noalloc_matches_workspace_forward_twice(first, second):
    for spec in (first, second):
        w = small_workload(**spec)
        dev = to_dev(w)
        f, _ = rp.workspace_size(dev["q"], dev["aq"], dev["ak"], dev["b"], w.tau, lmap(w), causal=w.causal,
                                 key_len=dev["key_len"])
        assert f <= NOALLOC_MAX_WORKSPACE
        ref_o, ref_l = _fwd(rp.relpos_attn_fwd, w, dev)
        for _ in range(2):
            o, lse = _fwd(rp._binding.relpos_attn_fwd_noalloc, w, dev)
            assert relf(o, ref_o) <= TOL_O_RELF and maxabs(o, ref_o) <= TOL_O_MAXABS
            assert lse_err(lse, ref_l) <= TOL_LSE_MAXABS


def test_noalloc_rejects_oversized_workspace():
    w = small_workload(map_kind="truncated", clip=64, N=8192, B=1, H=12, terms=("aQ", "aK"))
    dev = to_dev(w)
    f, _ = rp.workspace_size(dev["q"], dev["aq"], dev["ak"], dev["b"], w.tau, lmap(w))
    assert f > NOALLOC_MAX_WORKSPACE
    with pytest.raises(RelPosError, match="workspace"):
        _fwd(rp._binding.relpos_attn_fwd_noalloc, w, dev)
