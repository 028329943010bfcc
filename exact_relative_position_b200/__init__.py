"""Exact relative-position attention for B200 (sm_100a).

    S_ij = tau (q_i.k_j + q_i.aQ_phi(i,j) + k_j.aK_phi(i,j) + b_phi(i,j)) + M_ij

Shaw (truncated), Transformer-XL (identity), DeBERTa (log buckets) and T5
(buckets) relative attention, forward and backward, computed by the CUDA
library behind the C ABI in include/relpos_attn.h.  PyTorch supplies device
memory and streams only.
"""
from ._binding import (  # noqa: F401
    RelPosError, RelPosMap, check_noalloc, check_workspace, debug_phi, debug_phi_device, debug_projection,
    debug_tile_plan, debug_tile_plan_device, expanded_bounds, kernel_launches, lib, profile_start, profile_stop,
    relpos_attn_bwd, relpos_attn_fwd, set_wait_limit_ns, sum_partials, table_rows, workspace_size,
)

import torch


class RelPosAttention(torch.autograd.Function):
    """Autograd wrapper: O = attention(q, k, v, aq, ak, b) through the CUDA library."""

    @staticmethod
    def forward(ctx, q, k, v, aq, ak, b, tau, rmap, causal, key_len, dropout=(0.0, 0, 0), projection="retained",
                varlen=(None, None)):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        # one workspace for both passes: the backward reads the forward's
        # tables and projections from it instead of recomputing them
        kl = None if key_len is None else key_len.to(device=q.device, dtype=torch.int32)
        cu, max_len = varlen
        fws, bws = workspace_size(q, aq, ak, b, tau, rmap, causal=causal, key_len=kl, projection=projection,
                                  cu_seqlens=cu, max_seqlen=max_len)
        ws = torch.empty(max(fws, bws, 256), device=q.device, dtype=torch.uint8)
        dp, dseed, doff = dropout
        o, lse = relpos_attn_fwd(q, k, v, aq, ak, b, tau=tau, map=rmap, causal=causal, key_len=key_len, workspace=ws,
                                 dropout_p=dp, dropout_seed=dseed, dropout_offset=doff, projection=projection,
                                 cu_seqlens=cu, max_seqlen=max_len)
        ctx.save_for_backward(q, k, v, o, lse, aq, ak, b, key_len)
        ctx.cfg = (tau, rmap, causal, dropout, projection, varlen)
        ctx.ws = ws
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, o, lse, aq, ak, b, key_len = ctx.saved_tensors
        tau, rmap, causal, (dp, dseed, doff), projection, (cu, max_len) = ctx.cfg
        dq, dk, dv, daq, dak, db = relpos_attn_bwd(do.contiguous(), q, k, v, o, lse, aq, ak, b, tau=tau, map=rmap,
                                                   causal=causal, key_len=key_len, workspace=ctx.ws,
                                                   reuse_forward=True, dropout_p=dp, dropout_seed=dseed,
                                                   dropout_offset=doff, projection=projection, cu_seqlens=cu,
                                                   max_seqlen=max_len)
        ctx.ws = None
        cast = lambda g, t: None if g is None else g.to(t.dtype)
        return dq, dk, dv, cast(daq, aq), cast(dak, ak), db, None, None, None, None, None, None, None


def relpos_attention(q, k, v, aq=None, ak=None, b=None, *, tau, map, causal=False, key_len=None,
                     dropout_p=0.0, dropout_seed=0, dropout_offset=0, projection="retained",
                     cu_seqlens=None, max_seqlen=None):
    """Differentiable exact relative-position attention (CUDA only); optional
    attention dropout with the Philox mask of (seed, offset) at dropout_p rounded
    up to a multiple of 1/256; projection
    "recompute" keeps the forward's memory linear (q.aQ projected per tile);
    a packed variable-length batch passes q, k, v as [T, H, d] with cu_seqlens
    (int32 CUDA [B + 1]) and max_seqlen."""
    return RelPosAttention.apply(q, k, v, aq, ak, b, tau, map, causal, key_len,
                                 (float(dropout_p), int(dropout_seed), int(dropout_offset)), projection,
                                 (cu_seqlens, max_seqlen))
