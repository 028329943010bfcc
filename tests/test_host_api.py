"""Host-side checks of the C ABI (CPU only; no CUDA call is made).

The shared library must load and export every entry point the header
declares; the host planner's maps, saturation bounds and tile plan must
equal the oracle's bit for bit; argument validation must reject bad calls
before anything is launched; and the workspace must stay O(B H N R_reach)
(no N x N buffer) for the non-identity maps.
"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle as orc
from exact_relative_position_b200 import _binding as bd
from exact_relative_position_b200.build import build_library

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build_library()
    return bd.load_library()


def test_exports_every_declared_symbol(lib):
    hdr = open(os.path.join(ROOT, "include", "relpos_attn.h")).read()
    declared = set(re.findall(r"^\s*(?:int|int64_t|const char\*)\s+(relpos_\w+)\s*\(", hdr, re.M))
    assert len(declared) >= 11
    for name in declared:
        assert hasattr(lib, name), name
    assert set(bd.EXPORTS) == declared


MAPS = [
    ("truncated", dict(clip=16)), ("truncated", dict(clip=64)), ("truncated", dict(clip=0)),
    ("truncated", dict(clip=1000)), ("identity", {}),
    ("t5", dict(num_buckets=32, max_distance=128, bidirectional=1)),
    ("t5", dict(num_buckets=32, max_distance=128, bidirectional=0)),
    ("log", dict(num_buckets=256, max_distance=512)), ("log", dict(num_buckets=16, max_distance=64)),
    ("log_rev", dict(num_buckets=256, max_distance=512)), ("log_rev", dict(num_buckets=16, max_distance=64)),
]


def _maps(kind, kw):
    return orc.MapDesc(kind, **kw), bd.RelPosMap(kind, **kw)


@pytest.mark.parametrize("kind,kw", MAPS)
@pytest.mark.parametrize("N", [1, 2, 7, 50, 300, 2048])
def test_rows_and_bounds_match_oracle(lib, kind, kw, N):
    om, bm = _maps(kind, kw)
    assert bd.table_rows(bm, N) == orc.table_rows(om, N)
    assert bd.expanded_bounds(bm, N) == orc.expanded_bounds(om, N)


@pytest.mark.parametrize("kind,kw", MAPS)
@pytest.mark.parametrize("N", [1, 9, 130, 700])
def test_host_phi_bit_exact(lib, kind, kw, N):
    om, bm = _maps(kind, kw)
    got = bd.debug_phi(bm, N).numpy()
    assert np.array_equal(got, orc.phi_matrix(om, N))


@pytest.mark.parametrize("kind,kw", MAPS)
@pytest.mark.parametrize("N,causal,key_len", [(300, False, None), (1000, False, [1000, 613]),
                                              (700, True, None), (129, True, [129, 5]), (2048, False, [2000, 1843])])
def test_host_tile_plan_bit_exact(lib, kind, kw, N, causal, key_len):
    om, bm = _maps(kind, kw)
    B = 1 if key_len is None else len(key_len)
    cls, seg = bd.debug_tile_plan(bm, B, N, causal=causal, key_len=key_len)
    ocls, oseg = orc.tile_plan_rule(om, N, bd.TILE, causal, key_len, B)
    assert np.array_equal(cls.numpy(), ocls)
    assert np.array_equal(seg.numpy(), oseg)


def test_tile_plan_band_fraction_headline_shape(lib):
    # truncated clip 64 at N = 8192: only the three central tile diagonals are BAND
    cls, _ = bd.debug_tile_plan(bd.RelPosMap("truncated", clip=64), 1, 8192)
    c = cls.numpy()[0]
    nT = c.shape[0]
    band = np.argwhere(c == bd.TILE_BAND)
    assert np.all(np.abs(band[:, 1] - band[:, 0]) <= 1)
    assert len(band) == 3 * nT - 2


def _args(B=1, H=2, N=256, d=64, dtype=bd.F16, kind="truncated", clip=16, mask=0, aq=True, ak=True, b=True,
          per_head=0):
    a = bd.relpos_fwd_args()
    a.B, a.H, a.N, a.d = B, H, N, d
    a.dtype, a.out_dtype, a.tau = dtype, dtype, 0.125
    a.map = bd.RelPosMap(kind, clip=clip, num_buckets=32, max_distance=128).desc()
    a.mask, a.table_per_head = mask, per_head
    fake = 1 << 20   # never dereferenced: every call below fails validation first
    a.q = a.k = a.v = a.o = a.lse = fake
    a.aq = fake if aq else None
    a.ak = fake if ak else None
    a.b = fake if b else None
    return a


def test_validation_rejects_before_launch(lib):
    f, b = ctypes.c_size_t(), ctypes.c_size_t()
    assert lib.relpos_workspace_size(ctypes.byref(_args(d=32)), ctypes.byref(f), ctypes.byref(b)) == -2
    assert lib.relpos_workspace_size(ctypes.byref(_args(dtype=bd.F32)), ctypes.byref(f), ctypes.byref(b)) == -2
    assert lib.relpos_workspace_size(ctypes.byref(_args(N=0)), ctypes.byref(f), ctypes.byref(b)) == -1
    assert lib.relpos_workspace_size(ctypes.byref(_args(mask=8)), ctypes.byref(f), ctypes.byref(b)) == -2
    for bad_tau in (0.0, -0.125, float("nan"), float("inf")):
        a = _args()
        a.tau = bad_tau
        assert lib.relpos_workspace_size(ctypes.byref(a), ctypes.byref(f), ctypes.byref(b)) == -1, bad_tau
    assert lib.relpos_workspace_size(ctypes.byref(_args(kind="truncated", clip=-1)), ctypes.byref(f), ctypes.byref(b)) == -1
    a = _args()
    a.map.kind = 9
    assert lib.relpos_workspace_size(ctypes.byref(a), ctypes.byref(f), ctypes.byref(b)) == -2
    # null q
    a = _args()
    a.q = None
    assert lib.relpos_attn_fwd(ctypes.byref(a), 1 << 20, 1 << 30, None) == -1
    # key padding without key_len
    a = _args(mask=2)
    assert lib.relpos_attn_fwd(ctypes.byref(a), 1 << 20, 1 << 30, None) == -1
    # misaligned pointer
    a = _args()
    a.k = (1 << 20) + 2
    assert lib.relpos_attn_fwd(ctypes.byref(a), 1 << 20, 1 << 30, None) == -1
    # workspace too small / misaligned / null
    a = _args()
    assert lib.relpos_attn_fwd(ctypes.byref(a), 1 << 20, 16, None) == -3
    assert lib.relpos_attn_fwd(ctypes.byref(a), (1 << 20) + 8, 1 << 30, None) == -3
    assert lib.relpos_attn_fwd(ctypes.byref(a), None, 1 << 30, None) == -3
    # backward: missing gradient output for a present term
    g = bd.relpos_bwd_args()
    g.fwd = _args()
    g.dout = g.dq = g.dk = g.dv = 1 << 20
    g.daq = 1 << 20
    g.dak = None
    g.db = 1 << 20
    assert lib.relpos_attn_bwd(ctypes.byref(g), 1 << 20, 1 << 34, None) == -1
    assert lib.relpos_status_string(-3).decode().startswith("workspace")
    # debug projection: missing layout record, then a workspace that is too small
    lay = bd.relpos_projection_layout()
    assert lib.relpos_debug_projection(ctypes.byref(_args()), 1 << 20, 1 << 30, None, None) == -1
    assert lib.relpos_debug_projection(ctypes.byref(_args()), 1 << 20, 16, None, ctypes.byref(lay)) == -3


@pytest.mark.parametrize("key_len", [[8192 + 200, -1], [-5, 100000], [0, 8191]])
def test_tile_plan_clamps_out_of_range_key_lengths(lib, key_len):
    """A key length outside [0, N] masks as its clamped value would (the oracle's
    mask j >= key_len needs no clamp): the host plan equals the oracle's rule."""
    m, lm = _maps("truncated", dict(clip=64))
    N = 8192
    cls, seg = bd.debug_tile_plan(lm, 2, N, causal=False, key_len=key_len)
    want_cls, want_seg = orc.tile_plan_rule(m, N, 128, False, key_len=key_len, B=2)
    assert np.array_equal(cls.numpy(), want_cls) and np.array_equal(seg.numpy(), want_seg)


@pytest.mark.parametrize("kind,clip,N,B,H", [("truncated", 64, 8192, 1, 12), ("t5", 0, 8192, 1, 12),
                                            ("log", 0, 2048, 2, 12), ("truncated", 256, 16384, 1, 12)])
def test_workspace_has_no_n_by_n_buffer(lib, kind, clip, N, B, H):
    a = _args(B=B, H=H, N=N, kind=kind, clip=clip)
    if kind == "log":
        a.map = bd.RelPosMap("log", num_buckets=256, max_distance=512).desc()
    f, b = ctypes.c_size_t(), ctypes.c_size_t()
    assert lib.relpos_workspace_size(ctypes.byref(a), ctypes.byref(f), ctypes.byref(b)) == 0
    lo, hi = ctypes.c_int32(), ctypes.c_int32()
    lib.relpos_expanded_bounds(ctypes.byref(a.map), N, ctypes.byref(lo), ctypes.byref(hi))
    rexp = hi.value - lo.value + 1
    per_proj = B * H * N * ((rexp + 3) // 4 * 4) * 4
    # forward: Z^Q, Z^K plus small tables; backward adds dZ^Q, dZ^K, fp32 dQ/dK and split partials
    assert f.value <= 2 * per_proj + (8 << 20)
    assert b.value <= 4 * per_proj + 2 * B * H * N * 64 * 4 + B * H * N * 4 + (64 << 20)
    if rexp * 8 < N:   # short-reach maps: far below one fp32 N x N score matrix per head
        assert b.value < B * H * N * N * 4 / 4


def test_identity_grouped_projection_reach(lib):
    # identity map, causal, N = 16384: each 128-query group stores only its reachable
    # offsets (i0 + 128 columns), the quadratic projection the pages keep for this map
    N, H = 16384, 8
    a = _args(B=1, H=H, N=N, kind="identity", mask=1, ak=False)
    f, b = ctypes.c_size_t(), ctypes.c_size_t()
    assert lib.relpos_workspace_size(ctypes.byref(a), ctypes.byref(f), ctypes.byref(b)) == 0
    G = 128
    zq = H * sum(G * (g * G + G) for g in range(N // G)) * 4
    assert zq <= f.value <= zq + (32 << 20)


def test_recompute_projection_forward_workspace_is_linear(lib):
    """Projection recomputed per tile: the forward workspace of the identity map
    (the Transformer-XL layer, N = 16384, 8 heads, q.aQ and b) holds no
    projection at all, O(B H N) instead of the retained O(B H N^2); the
    backward, which rebuilds Z^Q, keeps its size.  The key-side term is not
    available in this mode, and an unknown mode is rejected."""
    N, B, H = 16384, 1, 8
    a = _args(B=B, H=H, N=N, kind="identity", ak=False, mask=1, per_head=1)
    f, b = ctypes.c_size_t(), ctypes.c_size_t()
    assert lib.relpos_workspace_size(ctypes.byref(a), ctypes.byref(f), ctypes.byref(b)) == 0
    f_ret, b_ret = f.value, b.value
    assert f_ret > B * H * N * N * 4 / 4          # retained: the quadratic Z^Q (causal: about half of N^2)
    a.projection = 1
    assert lib.relpos_workspace_size(ctypes.byref(a), ctypes.byref(f), ctypes.byref(b)) == 0
    assert f.value <= B * H * (2 * N - 1) * 4 + (4 << 20)   # expanded bias and group records only
    assert b.value == b_ret
    a.ak = 1 << 20
    assert lib.relpos_workspace_size(ctypes.byref(a), ctypes.byref(f), ctypes.byref(b)) == -2
    a = _args()
    a.projection = 2
    assert lib.relpos_workspace_size(ctypes.byref(a), ctypes.byref(f), ctypes.byref(b)) == -1


def test_packed_batch_argument_checks(lib):
    """A packed batch (cu_seqlens) needs total_tokens >= 1 and excludes the key
    padding flag (the sequence lengths already mask the keys); its workspace
    is the dense one of B sequences of N tokens."""
    f, b = ctypes.c_size_t(), ctypes.c_size_t()
    a = _args(B=3, N=517)
    assert lib.relpos_workspace_size(ctypes.byref(a), ctypes.byref(f), ctypes.byref(b)) == 0
    dense = (f.value, b.value)
    a.cu_seqlens, a.total_tokens = 1 << 20, 846
    assert lib.relpos_workspace_size(ctypes.byref(a), ctypes.byref(f), ctypes.byref(b)) == 0
    assert (f.value, b.value) == dense
    a.total_tokens = 0
    assert lib.relpos_workspace_size(ctypes.byref(a), ctypes.byref(f), ctypes.byref(b)) == -1
    a = _args(B=3, N=517, mask=2)
    a.cu_seqlens, a.total_tokens = 1 << 20, 846
    assert lib.relpos_workspace_size(ctypes.byref(a), ctypes.byref(f), ctypes.byref(b)) == -1
