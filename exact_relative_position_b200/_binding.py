"""ctypes binding of the C ABI in include/relpos_attn.h.

Argument marshalling only: every step of the computation runs in the CUDA
library.  Importing this module loads librelpos_b200.so and fails loudly if
it has not been built; there is no fallback path.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass
from typing import Optional

import torch

from .build import LIBPATH

RELPOS_OK = 0
STATUS = {0: "ok", -1: "invalid argument", -2: "unsupported", -3: "workspace", -4: "cuda error", -5: "timeout"}
MAP_KINDS = {"truncated": 0, "identity": 1, "t5": 2, "log": 3, "log_rev": 4}
MASK_CAUSAL, MASK_KEY_PADDING = 1, 2
PROJECTION_MODES = {"retained": 0, "recompute": 1}
F16, BF16, F32 = 0, 1, 2
TILE = 128
TILE_MASKED, TILE_CONST_LO, TILE_BAND, TILE_CONST_HI = 0, 1, 2, 3


class relpos_map_desc(ctypes.Structure):
    _fields_ = [("kind", ctypes.c_int32), ("clip", ctypes.c_int32), ("num_buckets", ctypes.c_int32),
                ("max_distance", ctypes.c_int32), ("bidirectional", ctypes.c_int32)]


class relpos_fwd_args(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("H", ctypes.c_int32), ("N", ctypes.c_int32), ("d", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("out_dtype", ctypes.c_int32), ("tau", ctypes.c_float),
                ("map", relpos_map_desc), ("mask", ctypes.c_int32), ("table_per_head", ctypes.c_int32),
                ("key_len", ctypes.c_void_p), ("q", ctypes.c_void_p), ("k", ctypes.c_void_p),
                ("v", ctypes.c_void_p), ("aq", ctypes.c_void_p), ("ak", ctypes.c_void_p),
                ("b", ctypes.c_void_p), ("o", ctypes.c_void_p), ("lse", ctypes.c_void_p),
                ("dropout_p", ctypes.c_float), ("dropout_offset", ctypes.c_uint32), ("dropout_seed", ctypes.c_uint64),
                ("projection", ctypes.c_int32), ("cu_seqlens", ctypes.c_void_p), ("total_tokens", ctypes.c_int32)]


class relpos_bwd_args(ctypes.Structure):
    _fields_ = [("fwd", relpos_fwd_args), ("dout", ctypes.c_void_p), ("dq", ctypes.c_void_p),
                ("dk", ctypes.c_void_p), ("dv", ctypes.c_void_p), ("daq", ctypes.c_void_p),
                ("dak", ctypes.c_void_p), ("db", ctypes.c_void_p), ("reuse_forward_workspace", ctypes.c_int32)]


class relpos_group_info(ctypes.Structure):
    _fields_ = [("e0", ctypes.c_int32), ("W", ctypes.c_int32), ("S", ctypes.c_int32), ("pad", ctypes.c_int32),
                ("base", ctypes.c_int64)]


class relpos_projection_layout(ctypes.Structure):
    _fields_ = [("E_lo", ctypes.c_int32), ("E_hi", ctypes.c_int32), ("R_exp", ctypes.c_int32),
                ("nT", ctypes.c_int32), ("grouped", ctypes.c_int32), ("pad", ctypes.c_int32),
                ("zq_offset", ctypes.c_int64), ("zk_offset", ctypes.c_int64), ("zq_head", ctypes.c_int64),
                ("zk_head", ctypes.c_int64), ("gq_offset", ctypes.c_int64), ("gk_offset", ctypes.c_int64)]


class relpos_phase_stat(ctypes.Structure):
    _fields_ = [("name", ctypes.c_char * 32), ("calls", ctypes.c_int32), ("kernels", ctypes.c_int32),
                ("total_ms", ctypes.c_float)]


EXPORTS = ["relpos_table_rows", "relpos_expanded_bounds", "relpos_workspace_size", "relpos_attn_fwd",
           "relpos_attn_bwd", "relpos_status_string", "relpos_last_cuda_error", "relpos_debug_phi",
           "relpos_debug_phi_device", "relpos_debug_tile_plan", "relpos_debug_tile_plan_device",
           "relpos_profile_start", "relpos_profile_stop", "relpos_kernel_launches", "relpos_attn_fwd_noalloc",
           "relpos_check_workspace", "relpos_sum_partials", "relpos_check_noalloc", "relpos_debug_projection",
           "relpos_set_wait_limit_ns"]


def load_library(path: str = LIBPATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise RuntimeError(f"CUDA library {path} is not built; run `python -m exact_relative_position_b200.build`")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER
    sig = {
        "relpos_table_rows": [P(relpos_map_desc), ctypes.c_int32, P(ctypes.c_int32)],
        "relpos_expanded_bounds": [P(relpos_map_desc), ctypes.c_int32, P(ctypes.c_int32), P(ctypes.c_int32)],
        "relpos_workspace_size": [P(relpos_fwd_args), P(ctypes.c_size_t), P(ctypes.c_size_t)],
        "relpos_attn_fwd": [P(relpos_fwd_args), ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p],
        "relpos_attn_bwd": [P(relpos_bwd_args), ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p],
        "relpos_status_string": [ctypes.c_int],
        "relpos_last_cuda_error": [],
        "relpos_debug_phi": [P(relpos_map_desc), ctypes.c_int32, ctypes.c_void_p],
        "relpos_debug_phi_device": [P(relpos_map_desc), ctypes.c_int32, ctypes.c_void_p, ctypes.c_void_p],
        "relpos_debug_tile_plan": [P(relpos_map_desc), ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p],
        "relpos_debug_tile_plan_device": [P(relpos_map_desc), ctypes.c_int32, ctypes.c_int32, ctypes.c_int32,
                                          ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p],
    }
    sig["relpos_profile_start"] = []
    sig["relpos_profile_stop"] = [P(relpos_phase_stat), ctypes.c_int32, P(ctypes.c_int32)]
    sig["relpos_kernel_launches"] = []
    sig["relpos_attn_fwd_noalloc"] = [P(relpos_fwd_args), ctypes.c_void_p]
    sig["relpos_check_workspace"] = [ctypes.c_void_p, ctypes.c_void_p, P(ctypes.c_int32)]
    sig["relpos_sum_partials"] = [ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
    sig["relpos_check_noalloc"] = [ctypes.c_void_p, P(ctypes.c_int32)]
    sig["relpos_debug_projection"] = [P(relpos_fwd_args), ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                                      P(relpos_projection_layout)]
    sig["relpos_set_wait_limit_ns"] = [ctypes.c_uint64]
    for name, args in sig.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = ctypes.c_char_p if name == "relpos_status_string" else ctypes.c_int
    lib.relpos_kernel_launches.restype = ctypes.c_int64
    return lib


_LIB: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    global _LIB
    if _LIB is None:
        _LIB = load_library()
    return _LIB


class RelPosError(RuntimeError):
    pass


def _check(status: int, what: str):
    if status != RELPOS_OK:
        msg = lib().relpos_status_string(status).decode()
        extra = ""
        if status == -4:
            extra = f" (cudaError {lib().relpos_last_cuda_error()})"
        raise RelPosError(f"{what}: {msg}{extra}")


@dataclass(frozen=True)
class RelPosMap:
    """Offset map phi: kind in {'truncated', 'identity', 't5', 'log'}."""
    kind: str
    clip: int = 0
    num_buckets: int = 0
    max_distance: int = 0
    bidirectional: int = 1

    def desc(self) -> relpos_map_desc:
        return relpos_map_desc(MAP_KINDS[self.kind], self.clip, self.num_buckets, self.max_distance,
                               self.bidirectional)


def table_rows(m: RelPosMap, N: int) -> int:
    r = ctypes.c_int32()
    _check(lib().relpos_table_rows(ctypes.byref(m.desc()), N, ctypes.byref(r)), "relpos_table_rows")
    return r.value


def expanded_bounds(m: RelPosMap, N: int):
    lo, hi = ctypes.c_int32(), ctypes.c_int32()
    _check(lib().relpos_expanded_bounds(ctypes.byref(m.desc()), N, ctypes.byref(lo), ctypes.byref(hi)),
           "relpos_expanded_bounds")
    return lo.value, hi.value


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else t.data_ptr()


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.float16:
        return F16
    if dt == torch.bfloat16:
        return BF16
    raise RelPosError(f"unsupported dtype {dt}")


def _shape(q, cu_seqlens=None, max_seqlen=None):
    """(B, H, N, d): q is [B, H, N, d], or packed [T, H, d] with cu_seqlens [B + 1]
    and max_seqlen = N (the longest sequence)."""
    if cu_seqlens is None:
        return tuple(q.shape)
    if q.dim() != 3 or max_seqlen is None:
        raise RelPosError("a packed batch needs q as [total_tokens, H, d] and max_seqlen")
    if not cu_seqlens.is_cuda or cu_seqlens.dtype != torch.int32 or cu_seqlens.dim() != 1:
        raise RelPosError("cu_seqlens must be an int32 CUDA tensor [B + 1]")
    T, H, d = q.shape
    return cu_seqlens.numel() - 1, H, int(max_seqlen), d


def _lse_shape(q, cu_seqlens=None, max_seqlen=None):
    B, H, N, _ = _shape(q, cu_seqlens, max_seqlen)
    return (B, H, N) if cu_seqlens is None else (H, q.shape[0])


def _fwd_args(q, k, v, aq, ak, b, tau, m: RelPosMap, causal, key_len, out_f32, o=None, lse=None,
              dropout=(0.0, 0, 0), projection="retained", cu_seqlens=None, max_seqlen=None):
    B, H, N, d = _shape(q, cu_seqlens, max_seqlen)
    for name, t in (("q", q), ("k", k), ("v", v)):
        if not t.is_cuda or not t.is_contiguous() or t.shape != q.shape or t.dtype != q.dtype:
            raise RelPosError(f"{name} must be a contiguous CUDA tensor shaped and typed like q")
    per_head = 0
    for t in (aq, ak):
        if t is not None:
            if not t.is_cuda or not t.is_contiguous() or t.dtype != q.dtype:
                raise RelPosError("aq/ak must be contiguous CUDA tensors of q's dtype")
            per_head = 1 if t.dim() == 3 else 0
    if b is not None and (not b.is_cuda or not b.is_contiguous() or b.dtype != torch.float32):
        raise RelPosError("b must be a contiguous float32 CUDA tensor [H, R]")
    mask = (MASK_CAUSAL if causal else 0) | (MASK_KEY_PADDING if key_len is not None else 0)
    a = relpos_fwd_args()
    a.B, a.H, a.N, a.d = B, H, N, d
    a.dtype = _dtype_code(q.dtype)
    a.out_dtype = F32 if out_f32 else a.dtype
    a.tau = float(tau)
    a.map = m.desc()
    a.mask = mask
    a.table_per_head = per_head
    a.key_len = _ptr(key_len)
    a.q, a.k, a.v = q.data_ptr(), k.data_ptr(), v.data_ptr()
    a.aq, a.ak, a.b = _ptr(aq), _ptr(ak), _ptr(b)
    a.o, a.lse = _ptr(o), _ptr(lse)
    a.dropout_p, a.dropout_seed, a.dropout_offset = float(dropout[0]), int(dropout[1]), int(dropout[2])
    if projection not in PROJECTION_MODES:
        raise RelPosError(f"projection must be one of {sorted(PROJECTION_MODES)}")
    a.projection = PROJECTION_MODES[projection]
    if cu_seqlens is not None:
        a.cu_seqlens, a.total_tokens = cu_seqlens.data_ptr(), q.shape[0]
    return a


def workspace_size(q, aq, ak, b, tau, m: RelPosMap, causal=False, key_len=None, out_f32=False,
                   projection="retained", cu_seqlens=None, max_seqlen=None):
    a = _fwd_args(q, q, q, aq, ak, b, tau, m, causal, key_len, out_f32, projection=projection,
                  cu_seqlens=cu_seqlens, max_seqlen=max_seqlen)
    f, bw = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().relpos_workspace_size(ctypes.byref(a), ctypes.byref(f), ctypes.byref(bw)), "relpos_workspace_size")
    return f.value, bw.value


def _stream(dev) -> int:
    return torch.cuda.current_stream(dev).cuda_stream


def relpos_attn_fwd(q, k, v, aq=None, ak=None, b=None, *, tau: float, map: RelPosMap, causal: bool = False,
                    key_len=None, out_f32: bool = False, workspace=None, o=None, lse=None,
                    dropout_p: float = 0.0, dropout_seed: int = 0, dropout_offset: int = 0,
                    projection: str = "retained", cu_seqlens=None, max_seqlen=None):
    """Forward through the C ABI.  Returns (O, LSE); O is float32 when out_f32.
    Attention dropout with rate dropout_p (rounded up to a multiple of 1/256) uses
    the Philox mask of (seed, offset); the backward needs the same three values.  projection="recompute" projects
    q.aQ inside every tile instead of storing Z^Q (linear forward memory).
    Packed variable-length batch: q, k, v [T, H, d] with cu_seqlens (int32
    CUDA [B + 1]) and max_seqlen; LSE is then [H, T]."""
    if o is None:
        o = torch.empty(q.shape, device=q.device, dtype=torch.float32 if out_f32 else q.dtype)
    if lse is None:
        lse = torch.empty(_lse_shape(q, cu_seqlens, max_seqlen), device=q.device, dtype=torch.float32)
    if key_len is not None:
        key_len = key_len.to(device=q.device, dtype=torch.int32).contiguous()
    a = _fwd_args(q, k, v, aq, ak, b, tau, map, causal, key_len, out_f32, o, lse,
                  (dropout_p, dropout_seed, dropout_offset), projection, cu_seqlens, max_seqlen)
    f, bw = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().relpos_workspace_size(ctypes.byref(a), ctypes.byref(f), ctypes.byref(bw)), "relpos_workspace_size")
    if workspace is None or workspace.numel() < f.value:
        workspace = torch.empty(max(f.value, 256), device=q.device, dtype=torch.uint8)
    _check(lib().relpos_attn_fwd(ctypes.byref(a), workspace.data_ptr(), workspace.numel(), _stream(q.device)),
           "relpos_attn_fwd")
    return o, lse


def relpos_attn_bwd(dout, q, k, v, o, lse, aq=None, ak=None, b=None, *, tau: float, map: RelPosMap,
                    causal: bool = False, key_len=None, workspace=None, grads=None, reuse_forward: bool = False,
                    dropout_p: float = 0.0, dropout_seed: int = 0, dropout_offset: int = 0,
                    projection: str = "retained", cu_seqlens=None, max_seqlen=None):
    """Backward through the C ABI.  Returns (dq, dk, dv, daq, dak, db).

    reuse_forward: `workspace` is the one the forward with these same arguments
    ran in and still holds its tables and projections, so the backward reads
    them instead of recomputing them."""
    if key_len is not None:
        key_len = key_len.to(device=q.device, dtype=torch.int32).contiguous()
    out_f32 = o.dtype == torch.float32
    if not dout.is_contiguous() or dout.dtype != q.dtype or dout.shape != q.shape:
        raise RelPosError("dout must be contiguous, shaped and typed like q")
    a = _fwd_args(q, k, v, aq, ak, b, tau, map, causal, key_len, out_f32, o, lse,
                  (dropout_p, dropout_seed, dropout_offset), projection, cu_seqlens, max_seqlen)
    g = relpos_bwd_args()
    g.fwd = a
    if grads is None:
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        daq = None if aq is None else torch.empty(aq.shape, device=q.device, dtype=torch.float32)
        dak = None if ak is None else torch.empty(ak.shape, device=q.device, dtype=torch.float32)
        db = None if b is None else torch.empty(b.shape, device=q.device, dtype=torch.float32)
    else:
        dq, dk, dv, daq, dak, db = grads
    g.dout, g.dq, g.dk, g.dv = dout.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr()
    g.daq, g.dak, g.db = _ptr(daq), _ptr(dak), _ptr(db)
    f, bw = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().relpos_workspace_size(ctypes.byref(a), ctypes.byref(f), ctypes.byref(bw)), "relpos_workspace_size")
    if workspace is None or workspace.numel() < bw.value:
        if reuse_forward:
            raise RelPosError("reuse_forward needs the forward's workspace, at least the backward's size")
        workspace = torch.empty(max(bw.value, 256), device=q.device, dtype=torch.uint8)
    g.reuse_forward_workspace = 1 if reuse_forward else 0
    _check(lib().relpos_attn_bwd(ctypes.byref(g), workspace.data_ptr(), workspace.numel(), _stream(q.device)),
           "relpos_attn_bwd")
    return dq, dk, dv, daq, dak, db


def debug_phi(m: RelPosMap, N: int):
    out = torch.empty((N, N), dtype=torch.int32)
    _check(lib().relpos_debug_phi(ctypes.byref(m.desc()), N, out.data_ptr()), "relpos_debug_phi")
    return out


def debug_phi_device(m: RelPosMap, N: int, device="cuda"):
    out = torch.empty((2 * N - 1,), dtype=torch.int32, device=device)
    _check(lib().relpos_debug_phi_device(ctypes.byref(m.desc()), N, out.data_ptr(), _stream(out.device)),
           "relpos_debug_phi_device")
    return out


def debug_tile_plan(m: RelPosMap, B: int, N: int, causal=False, key_len=None):
    nT = (N + TILE - 1) // TILE
    cls = torch.empty((B, nT, nT), dtype=torch.int32)
    seg = torch.empty((B, nT, 4), dtype=torch.int32)
    mask = (MASK_CAUSAL if causal else 0) | (MASK_KEY_PADDING if key_len is not None else 0)
    kl = None if key_len is None else torch.as_tensor(key_len, dtype=torch.int32).contiguous()
    _check(lib().relpos_debug_tile_plan(ctypes.byref(m.desc()), B, N, mask, _ptr(kl), cls.data_ptr(), seg.data_ptr()),
           "relpos_debug_tile_plan")
    return cls, seg


def debug_tile_plan_device(m: RelPosMap, B: int, N: int, causal=False, key_len=None, device="cuda"):
    nT = (N + TILE - 1) // TILE
    cls = torch.empty((B, nT, nT), dtype=torch.int32, device=device)
    seg = torch.empty((B, nT, 4), dtype=torch.int32, device=device)
    mask = (MASK_CAUSAL if causal else 0) | (MASK_KEY_PADDING if key_len is not None else 0)
    kl = None if key_len is None else torch.as_tensor(key_len, dtype=torch.int32).to(device).contiguous()
    _check(lib().relpos_debug_tile_plan_device(ctypes.byref(m.desc()), B, N, mask, _ptr(kl), cls.data_ptr(),
                                               seg.data_ptr(), _stream(cls.device)), "relpos_debug_tile_plan_device")
    return cls, seg


def profile_start():
    _check(lib().relpos_profile_start(), "relpos_profile_start")


def profile_stop():
    """Returns {phase: (calls, kernels, total_ms)} collected since profile_start()."""
    arr = (relpos_phase_stat * 16)()
    n = ctypes.c_int32()
    _check(lib().relpos_profile_stop(arr, 16, ctypes.byref(n)), "relpos_profile_stop")
    return {arr[i].name.decode(): (arr[i].calls, arr[i].kernels, arr[i].total_ms) for i in range(min(n.value, 16))}


def kernel_launches() -> int:
    return int(lib().relpos_kernel_launches())


NOALLOC_MAX_WORKSPACE = 32 << 20


def relpos_attn_fwd_noalloc(q, k, v, aq=None, ak=None, b=None, *, tau: float, map: RelPosMap, causal: bool = False,
                            key_len=None, out_f32: bool = False, o=None, lse=None, projection: str = "retained"):
    """Forward through relpos_attn_fwd_noalloc: the library's fixed 32 MiB scratch
    array replaces the workspace, so the call needs no device allocation for it."""
    if o is None:
        o = torch.empty(q.shape, device=q.device, dtype=torch.float32 if out_f32 else q.dtype)
    if lse is None:
        lse = torch.empty(_lse_shape(q), device=q.device, dtype=torch.float32)
    if key_len is not None:
        key_len = key_len.to(device=q.device, dtype=torch.int32).contiguous()
    a = _fwd_args(q, k, v, aq, ak, b, tau, map, causal, key_len, out_f32, o, lse, projection=projection)
    _check(lib().relpos_attn_fwd_noalloc(ctypes.byref(a), _stream(q.device)), "relpos_attn_fwd_noalloc")
    return o, lse


def check_noalloc(device=None) -> int:
    """Synchronises the current stream and returns the device status word of the
    last relpos_attn_fwd_noalloc on this device (0 = ok); raises RelPosError on a
    timeout."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    st = ctypes.c_int32()
    _check(lib().relpos_check_noalloc(_stream(dev), ctypes.byref(st)), "relpos_check_noalloc")
    return st.value


def set_wait_limit_ns(ns: int) -> None:
    """Limit of the fused kernels' bounded waits for later launches (0 = the
    default 2 s).  Only for tests of the timeout path."""
    _check(lib().relpos_set_wait_limit_ns(int(ns)), "relpos_set_wait_limit_ns")


def debug_projection(q, k, aq=None, ak=None, b=None, *, tau: float, map: RelPosMap, causal: bool = False,
                     key_len=None):
    """relpos_debug_projection: runs the table expansion and the projections only.

    Returns (layout, workspace, groups_q, groups_k): the layout record, the
    workspace tensor holding Z^Q / Z^K at the recorded offsets, and the group
    records of each side as [nT, 4] int32 (e0, W, S, pad) plus [nT] int64 bases."""
    if key_len is not None:
        key_len = key_len.to(device=q.device, dtype=torch.int32).contiguous()
    a = _fwd_args(q, k, q, aq, ak, b, tau, map, causal, key_len, False)
    f, bw = ctypes.c_size_t(), ctypes.c_size_t()
    _check(lib().relpos_workspace_size(ctypes.byref(a), ctypes.byref(f), ctypes.byref(bw)), "relpos_workspace_size")
    ws = torch.zeros(max(f.value, 256), device=q.device, dtype=torch.uint8)
    lay = relpos_projection_layout()
    _check(lib().relpos_debug_projection(ctypes.byref(a), ws.data_ptr(), ws.numel(), _stream(q.device),
                                         ctypes.byref(lay)), "relpos_debug_projection")

    def groups(off):
        raw = ws[off:off + 24 * lay.nT].cpu()
        ints = raw.view(torch.int32).reshape(lay.nT, 6)
        return ints[:, :4].clone(), raw.view(torch.int64).reshape(lay.nT, 3)[:, 2].clone()

    return lay, ws, groups(lay.gq_offset), groups(lay.gk_offset)


def check_workspace(workspace) -> int:
    """Synchronises the current stream and returns the device status word of the
    last call that used `workspace` (0 = ok); raises RelPosError on a timeout."""
    st = ctypes.c_int32()
    _check(lib().relpos_check_workspace(workspace.data_ptr(), _stream(workspace.device), ctypes.byref(st)),
           "relpos_check_workspace")
    return st.value


def sum_partials(partials: torch.Tensor, out: Optional[torch.Tensor] = None) -> torch.Tensor:
    """relpos_sum_partials: partials [world, n] fp32 CUDA (contiguous) -> [n], the
    rows added in ascending order.  out may be partials[0] or a separate [n] buffer."""
    if partials.device.type != "cuda" or partials.dtype != torch.float32 or partials.dim() != 2 \
            or not partials.is_contiguous():
        raise ValueError("partials must be a contiguous [world, n] float32 CUDA tensor")
    world, n = partials.shape
    if out is None:
        out = torch.empty(n, device=partials.device, dtype=torch.float32)
    if out.device != partials.device or out.dtype != torch.float32 or out.numel() != n or not out.is_contiguous():
        raise ValueError("out must be a contiguous float32 tensor of n entries on the partials' device")
    _check(lib().relpos_sum_partials(partials.data_ptr(), world, n, out.data_ptr(), _stream(partials.device)),
           "relpos_sum_partials")
    return out
