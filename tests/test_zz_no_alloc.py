"""relpos_attn_fwd_noalloc: the forward for callers that cannot allocate device
memory (a pool or another runtime owns the device and forbids outside
allocations, or an enqueue step must not allocate).  It runs in the library's
fixed 32 MiB scratch array instead of a caller workspace.

Checked through the C ABI against the ordinary workspace forward on two
calls in a row (the scratch array keeps the previous call's contents): both
run the same deterministic kernels, so O and LSE must be equal bit for bit.
After a warm-up call a further call must leave the device's free memory
unchanged (the entry point's reason to exist), and its status word, read
with relpos_check_noalloc, must be clean; a call whose bounded wait runs out
must be reported there.  Shapes whose workspace does not fit are rejected.
Kept in its own file, collected last.
"""
import numpy as np
import pytest
import torch

from synth import small_workload
from relpos_harness import lmap, to_dev
import exact_relative_position_b200 as rp
from exact_relative_position_b200 import _binding as bd
from exact_relative_position_b200._binding import NOALLOC_MAX_WORKSPACE, RelPosError

pytestmark = pytest.mark.gpu


def _fwd(fn, w, dev, out, **extra):
    fn(dev["q"], dev["k"], dev["v"], dev["aq"], dev["ak"], dev["b"], tau=w.tau, map=lmap(w), causal=w.causal,
       key_len=dev["key_len"], o=out[0], lse=out[1], **extra)
    torch.cuda.synchronize()
    return out[0].cpu().numpy().copy(), out[1].cpu().numpy().copy()


def _outputs(w, dev):
    return (torch.empty(dev["q"].shape, device="cuda", dtype=dev["q"].dtype),
            torch.empty(dev["q"].shape[:3], device="cuda", dtype=torch.float32))


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
        ref_o, ref_l = _fwd(rp.relpos_attn_fwd, w, dev, _outputs(w, dev))
        out = _outputs(w, dev)
        _fwd(bd.relpos_attn_fwd_noalloc, w, dev, out)          # warm-up: modules loaded, scratch committed
        for _ in range(2):
            torch.cuda.synchronize()
            free0, _ = torch.cuda.mem_get_info()
            o, lse = _fwd(bd.relpos_attn_fwd_noalloc, w, dev, out)
            free1, _ = torch.cuda.mem_get_info()
            assert free1 == free0, "the no-allocation forward changed the device's free memory"
            assert bd.check_noalloc() == 0
            assert np.array_equal(o, ref_o) and np.array_equal(lse, ref_l)


def test_noalloc_reports_an_expired_wait():
    w = small_workload(map_kind="truncated", clip=16, N=300, B=1, H=2, terms=("aQ", "aK"))
    dev = to_dev(w)
    out = _outputs(w, dev)
    try:
        bd.set_wait_limit_ns(1)
        _fwd(bd.relpos_attn_fwd_noalloc, w, dev, out)
    finally:
        bd.set_wait_limit_ns(0)
    with pytest.raises(RelPosError, match="timed out"):
        bd.check_noalloc()
    ref = _fwd(rp.relpos_attn_fwd, w, dev, _outputs(w, dev))
    got = _fwd(bd.relpos_attn_fwd_noalloc, w, dev, out)
    assert bd.check_noalloc() == 0
    assert np.array_equal(got[0], ref[0]) and np.array_equal(got[1], ref[1])


def test_noalloc_rejects_oversized_workspace():
    w = small_workload(map_kind="truncated", clip=64, N=8192, B=1, H=12, terms=("aQ", "aK"))
    dev = to_dev(w)
    f, _ = rp.workspace_size(dev["q"], dev["aq"], dev["ak"], dev["b"], w.tau, lmap(w))
    assert f > NOALLOC_MAX_WORKSPACE
    with pytest.raises(RelPosError, match="workspace"):
        _fwd(bd.relpos_attn_fwd_noalloc, w, dev, _outputs(w, dev))
