"""Seeded synthetic inputs for one relative-position attention layer.

The five named workloads follow the layer benchmark of "Fast and Exact
Relative-Position Attention via Structure-Aware Kernels" (arXiv 2611.01182,
experimental setup: 12 heads, head dim 64, FP16, bidirectional, the
per-mechanism maps Shaw clip / Transformer-XL identity / DeBERTa log buckets /
T5 32 buckets to distance 128).  The pages benchmark shapes only, with no
dataset, so every tensor here is drawn from a seeded generator.

Recipe (one torch.Generator on the CPU, seed 0 unless given, every draw in
float32 and then rounded to nearest-even into the compute dtype):
  Q, K, V, dO ~ N(0, 1) in that order;
  aQ, aK ~ N(0, table_std) when the term is present (shape [R, d] shared or
  [H, R, d] per head);  b ~ N(0, b_std) [H, R] float32 when present;
  Transformer-XL: W_r ~ N(0, 0.02) [H, H*d, d], u, v ~ N(0, 0.02) [H, d];
  key padding: U_b ~ U[0, 1) per batch element, key_len[b] = N - floor(U_b*0.1*N).
Transformer-XL inputs are then rewritten into the unified score form
(Q + u as the query, aQ_h = R_sin W_r^h, b_h = (v - u) . aQ_h), which is a
re-parameterisation of the inputs, not part of the attention arithmetic.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import torch

MAP_KINDS = ("truncated", "identity", "t5", "log", "log_rev")


def table_rows(map_kind: str, N: int, clip: int = 0, num_buckets: int = 0) -> int:
    """Number of rows R of a relation table for the given map (a shape rule)."""
    if map_kind == "truncated":
        return 2 * clip + 1
    if map_kind == "identity":
        return 2 * N - 1
    if map_kind == "t5":
        return num_buckets
    if map_kind in ("log", "log_rev"):
        return 2 * num_buckets
    raise ValueError(map_kind)


@dataclass
class Workload:
    name: str
    B: int
    H: int
    N: int
    d: int
    map_kind: str
    clip: int = 0
    num_buckets: int = 0
    max_distance: int = 0
    bidirectional: int = 1
    terms: tuple = ()
    per_head_tables: bool = False
    tau: float = 0.125
    causal: bool = False
    key_padding: bool = False
    dtype: torch.dtype = torch.float16
    table_std: float = 0.02
    b_std: float = 0.5
    txl: bool = False
    seed: int = 0
    # filled by make_workload
    R: int = 0
    q: Optional[torch.Tensor] = None
    k: Optional[torch.Tensor] = None
    v: Optional[torch.Tensor] = None
    do: Optional[torch.Tensor] = None
    aq: Optional[torch.Tensor] = None
    ak: Optional[torch.Tensor] = None
    b: Optional[torch.Tensor] = None
    key_len: Optional[torch.Tensor] = None
    extra: dict = field(default_factory=dict)

    @property
    def dtype_name(self) -> str:
        return {torch.float16: "f16", torch.bfloat16: "bf16"}[self.dtype]

    def describe(self) -> dict:
        return {
            "workload": self.name, "B": self.B, "H": self.H, "N": self.N, "d": self.d,
            "map": self.map_kind, "clip": self.clip, "num_buckets": self.num_buckets,
            "max_distance": self.max_distance, "terms": list(self.terms),
            "per_head_tables": self.per_head_tables, "tau": self.tau,
            "causal": self.causal, "key_padding": self.key_padding,
            "dtype": self.dtype_name, "R": self.R,
        }


# The five layer workloads (shape, map, terms, distributions, tau, mask, dtype).
CONFIGS = {
    "shaw_clip16_n256": dict(
        B=1, H=2, N=256, d=64, map_kind="truncated", clip=16, terms=("aQ",),
        tau=1 / 8, dtype=torch.float16),
    "deberta_log256_n2048": dict(
        B=2, H=12, N=2048, d=64, map_kind="log", num_buckets=256, max_distance=512,
        terms=("aQ", "aK"), per_head_tables=True, tau=1 / math.sqrt(3 * 64),
        key_padding=True, dtype=torch.float16),
    "t5_bucket32_n8192": dict(
        B=1, H=12, N=8192, d=64, map_kind="t5", num_buckets=32, max_distance=128,
        bidirectional=1, terms=("b",), tau=1.0, b_std=0.5, dtype=torch.float16),
    "shaw_clip64_n8192": dict(
        B=1, H=12, N=8192, d=64, map_kind="truncated", clip=64, terms=("aQ", "aK"),
        tau=1 / 8, dtype=torch.float16),
    "txl_identity_causal_n16384": dict(
        B=1, H=8, N=16384, d=64, map_kind="identity", terms=("aQ", "b"),
        per_head_tables=True, tau=1 / 8, causal=True, txl=True, dtype=torch.bfloat16),
}


# The pages' sequence-length sweep: the four mechanisms at a fixed budget of
# 16384 tokens per batch (B = 16384 / N) for N = 128 ... 8192, 12 heads,
# head dim 64, fp16, bidirectional (no mask).
SWEEP_TOKENS = 16384
SWEEP_LENGTHS = (128, 256, 512, 1024, 2048, 4096, 8192)
SWEEP_MECHANISMS = {
    "shaw_clip256": dict(map_kind="truncated", clip=256, terms=("aQ", "aK"), tau=1 / 8),
    "txl_identity": dict(map_kind="identity", terms=("aQ", "b"), per_head_tables=True, tau=1 / 8, txl=True),
    "deberta_log256": dict(map_kind="log", num_buckets=256, max_distance=512, terms=("aQ", "aK"),
                           per_head_tables=True, tau=1 / math.sqrt(3 * 64)),
    "t5_bucket32": dict(map_kind="t5", num_buckets=32, max_distance=128, bidirectional=1, terms=("b",), tau=1.0,
                        b_std=0.5),
}


def sweep_workload(mechanism: str, N: int, seed: int = 0, tokens: int = SWEEP_TOKENS, H: int = 12,
                   **overrides) -> "Workload":
    """One point of the sequence-length sweep: `mechanism` at length N with
    B = tokens / N (rounded down, at least 1)."""
    spec = dict(SWEEP_MECHANISMS[mechanism])
    spec.update(name=f"{mechanism}_n{N}", B=max(1, tokens // N), H=H, N=N, d=64, dtype=torch.float16)
    spec.update(overrides)
    return make_workload(spec, seed=seed)


def _normal(gen, shape, std):
    return torch.randn(shape, generator=gen, dtype=torch.float32) * std


def _sinusoid(N: int, dim: int) -> torch.Tensor:
    """Sinusoidal relative-position embeddings for offsets -(N-1)..(N-1), row r <-> offset r-(N-1)."""
    off = torch.arange(-(N - 1), N, dtype=torch.float64)
    m = torch.arange(dim // 2, dtype=torch.float64)
    omega = torch.pow(10000.0, -2.0 * m / dim)
    ang = off[:, None] * omega[None, :]
    return torch.cat([torch.sin(ang), torch.cos(ang)], dim=1)


def make_workload(name_or_spec, seed: int = 0, **overrides) -> Workload:
    """Build a workload by config name (or a dict spec) with seeded tensors on the CPU."""
    if isinstance(name_or_spec, str):
        spec = dict(CONFIGS[name_or_spec])
        name = name_or_spec
    else:
        spec = dict(name_or_spec)
        name = spec.pop("name", "custom")
    spec.update(overrides)
    w = Workload(name=name, seed=seed, **spec)
    w.R = table_rows(w.map_kind, w.N, w.clip, w.num_buckets)
    gen = torch.Generator().manual_seed(seed)
    shape = (w.B, w.H, w.N, w.d)
    q = _normal(gen, shape, 1.0)
    k = _normal(gen, shape, 1.0)
    v = _normal(gen, shape, 1.0)
    do = _normal(gen, shape, 1.0)
    tshape = (w.H, w.R, w.d) if w.per_head_tables else (w.R, w.d)
    if w.txl:
        # Transformer-XL: relation rows are sinusoids projected per head; u/v global biases.
        wr = _normal(gen, (w.H, w.H * w.d, w.d), 0.02)
        u = _normal(gen, (w.H, w.d), 0.02)
        vv = _normal(gen, (w.H, w.d), 0.02)
        rsin = _sinusoid(w.N, w.H * w.d)                                  # [R, H*d] f64
        aq32 = torch.einsum("rc,hcd->hrd", rsin, wr.double())             # [H, R, d]
        aq = aq32.to(w.dtype)
        b = torch.einsum("hd,hrd->hr", (vv - u).double(), aq32).float()   # [H, R]
        q = q + u[None, :, None, :]
        w.extra.update(w_r=wr, u=u, v=vv)
        w.aq, w.ak, w.b = aq, None, b
    else:
        w.aq = _normal(gen, tshape, w.table_std).to(w.dtype) if "aQ" in w.terms else None
        w.ak = _normal(gen, tshape, w.table_std).to(w.dtype) if "aK" in w.terms else None
        w.b = _normal(gen, (w.H, w.R), w.b_std) if "b" in w.terms else None
    if w.key_padding:
        ub = torch.rand((w.B,), generator=gen, dtype=torch.float32)
        w.key_len = (w.N - torch.floor(ub * 0.1 * w.N)).to(torch.int32)
    w.q, w.k, w.v, w.do = (t.to(w.dtype) for t in (q, k, v, do))
    return w


def small_workload(map_kind="truncated", B=1, H=2, N=200, d=64, clip=16, num_buckets=32,
                   max_distance=128, bidirectional=1, terms=("aQ", "aK", "b"),
                   per_head_tables=False, tau=0.125, causal=False, key_padding=False,
                   dtype=torch.float16, seed=0, table_std=0.02, b_std=0.5,
                   key_len=None) -> Workload:
    """A small custom workload for parity tests (same recipe, chosen shape)."""
    spec = dict(name=f"{map_kind}_B{B}H{H}N{N}d{d}", B=B, H=H, N=N, d=d, map_kind=map_kind,
                clip=clip, num_buckets=num_buckets, max_distance=max_distance,
                bidirectional=bidirectional, terms=tuple(terms),
                per_head_tables=per_head_tables, tau=tau, causal=causal,
                key_padding=key_padding, dtype=dtype, table_std=table_std, b_std=b_std)
    w = make_workload(spec, seed=seed)
    if key_len is not None:
        w.key_len = torch.as_tensor(key_len, dtype=torch.int32)
        w.key_padding = True
    return w
