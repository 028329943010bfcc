"""Model-level adapters over `relpos_attention`: Transformer-XL and DeBERTa.

Transformer-XL's relative attention written in the unified score of the paper
digest ("Fast and Exact Relative-Position Attention via Structure-Aware
Kernels", Eq. (1); the Transformer-XL workload of its experimental setup): for
head h,

    score_ij = tau [ (q_i + u_h) . k_j  +  (q_i + v_h) . W_r^h R_(j - i) ]

with R the fixed sinusoid table over offsets and W_r^h the layer's relation
projection.  In the unified form this is

    q' = q + u,   aQ_h = R W_r^h (identity map, one row per offset),
    b_h[r] = (v_h - u_h) . aQ_h[r],

so the kernel sees q'.k + q'.aQ + b.  The re-parameterisation is plain PyTorch,
so autograd carries the kernel's gradients (dq, daQ, db) on to u, v and W_r.
Offsets follow the library's convention delta = j - i (Transformer-XL writes
R_(i - j): the same table with its rows reversed).
"""
from __future__ import annotations

import math

import torch

from . import RelPosMap, relpos_attention


def sinusoid_table(N: int, dim: int, device=None) -> torch.Tensor:
    """[2N - 1, dim] float32: row r is offset r - (N - 1), columns
    [sin(delta w_m) | cos(delta w_m)] with w_m = 10000^(-2m / dim)."""
    off = torch.arange(-(N - 1), N, dtype=torch.float64, device=device)
    m = torch.arange(dim // 2, dtype=torch.float64, device=device)
    omega = torch.pow(10000.0, -2.0 * m / dim)
    ang = off[:, None] * omega[None, :]
    return torch.cat([torch.sin(ang), torch.cos(ang)], dim=1).float()


class TransformerXLRelPos(torch.nn.Module):
    """One Transformer-XL relative attention layer over given q, k, v.

    Parameters: W_r [H, d_model, d_head] (relation projection per head), u, v
    [H, d_head] (the content and position biases).  forward(q, k, v) with
    q, k, v [B, H, N, d_head] fp16/bf16 on the GPU returns O [B, H, N, d_head].
    """

    def __init__(self, n_heads: int, d_head: int = 64, d_model: int | None = None, causal: bool = True,
                 tau: float | None = None, init_std: float = 0.02, projection: str = "retained"):
        super().__init__()
        self.n_heads, self.d_head = n_heads, d_head
        self.d_model = d_model or n_heads * d_head
        self.causal = causal
        # "recompute": the kernel projects q'.aQ inside every tile, so the
        # forward never stores the quadratic identity-map projection
        self.projection = projection
        self.tau = tau if tau is not None else 1.0 / math.sqrt(d_head)
        self.W_r = torch.nn.Parameter(torch.randn(n_heads, self.d_model, d_head) * init_std)
        self.u = torch.nn.Parameter(torch.randn(n_heads, d_head) * init_std)
        self.v = torch.nn.Parameter(torch.randn(n_heads, d_head) * init_std)

    def unified_inputs(self, q: torch.Tensor):
        """q' = q + u, aQ [H, 2N - 1, d] (in q's dtype) and b [H, 2N - 1] fp32."""
        N = q.shape[2]
        R = sinusoid_table(N, self.d_model, device=q.device)
        aq32 = torch.einsum("rc,hcd->hrd", R, self.W_r.float())
        b = torch.einsum("hd,hrd->hr", (self.v - self.u).float(), aq32)
        qp = q + self.u[None, :, None, :].to(q.dtype)
        return qp, aq32.to(q.dtype).contiguous(), b.contiguous()

    def forward(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor) -> torch.Tensor:
        qp, aq, b = self.unified_inputs(q)
        return relpos_attention(qp, k, v, aq, None, b, tau=self.tau, map=RelPosMap("identity"), causal=self.causal,
                                projection=self.projection)


class DebertaRelPos(torch.nn.Module):
    """DeBERTa's disentangled attention over given content q, k, v.

    score_ij = tau [ q_i . k_j  +  q_i . (E W_kr)[row(i - j)]  +  k_j . (E W_qr)[row(i - j)] ]

    with E the relative-position embeddings [2 span, d_model], W_kr / W_qr the
    per-head position-key and position-query projections, tau = 1/sqrt(3 d),
    and row(x) the DeBERTa log-bucket row of the query-minus-key position x
    (content-to-position and position-to-content both land on it).  In the
    unified score of the paper digest (Eq. (1)) this is aQ = E W_kr,
    aK = E W_qr with the map 'log_rev' (the log row of -delta, delta = j - i),
    one table pair per head.  Gradients reach E, W_kr and W_qr through
    PyTorch's autograd around the kernel's daQ / daK.  forward(q, k, v,
    key_len=None) with q, k, v [B, H, N, d_head] fp16/bf16 on the GPU returns
    O [B, H, N, d_head]; key_len [B] masks padded keys.
    """

    def __init__(self, n_heads: int, d_head: int = 64, d_model: int | None = None, span: int = 256,
                 max_position: int = 512, tau: float | None = None, init_std: float = 0.02):
        super().__init__()
        self.n_heads, self.d_head = n_heads, d_head
        self.d_model = d_model or n_heads * d_head
        self.span, self.max_position = span, max_position
        self.tau = tau if tau is not None else 1.0 / math.sqrt(3 * d_head)
        self.rel_embeddings = torch.nn.Parameter(torch.randn(2 * span, self.d_model) * init_std)
        self.W_kr = torch.nn.Parameter(torch.randn(n_heads, self.d_model, d_head) * init_std)
        self.W_qr = torch.nn.Parameter(torch.randn(n_heads, self.d_model, d_head) * init_std)

    def rel_map(self) -> RelPosMap:
        return RelPosMap("log_rev", num_buckets=self.span, max_distance=self.max_position)

    def unified_inputs(self, dtype):
        """aQ = E W_kr and aK = E W_qr, [H, 2 span, d] each, in the kernel's dtype."""
        ct = torch.promote_types(self.rel_embeddings.dtype, torch.float32)   # at least fp32 for the products
        E = self.rel_embeddings.to(ct)
        aq = torch.einsum("rc,hcd->hrd", E, self.W_kr.to(ct)).to(dtype).contiguous()
        ak = torch.einsum("rc,hcd->hrd", E, self.W_qr.to(ct)).to(dtype).contiguous()
        return aq, ak

    def forward(self, q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, key_len=None) -> torch.Tensor:
        aq, ak = self.unified_inputs(q.dtype)
        return relpos_attention(q, k, v, aq, ak, None, tau=self.tau, map=self.rel_map(), key_len=key_len)
