"""The data-parallel exchange of the layer: summing shared-table gradients.

With the batch split over ranks, every (batch, head) slice stays on one rank,
so the forward and the gradients dQ, dK, dV and those of per-head tables need
no communication.  A table shared across the batch is different: its gradient
is the sum over every cell that reads it (paper digest "Fast and Exact
Relative-Position Attention via Structure-Aware Kernels", Eq. (4)), and each
rank's backward holds only the part from its own batch elements.

`reduce_table_grads` completes those sums with one all-gather of the partials
(NCCL over NVLink on GPUs) and the library's ascending-rank sum
(`relpos_sum_partials`), so every rank ends with the same bits whatever the
collective's internal order.
"""
from __future__ import annotations

from typing import Callable, Optional, Sequence

import torch
import torch.distributed as dist

from ._binding import sum_partials as _library_sum


def reduce_table_grads(grads: Sequence[Optional[torch.Tensor]], group=None,
                       sum_partials: Optional[Callable[[torch.Tensor], torch.Tensor]] = None):
    """Replace each tensor of `grads` (None entries are skipped) by its sum over
    the ranks of `group`, added in ascending rank order; returns `grads`.

    The tensors are fp32 and alike on every rank (same shapes, same order,
    e.g. (daq, dak, db) of relpos_attn_bwd with shared tables).  They travel as
    one flat buffer: one all-gather per call.  `sum_partials` maps the gathered
    [world, n] buffer to the [n] sum; the default is the library's CUDA kernel,
    which requires CUDA tensors.
    """
    ts = [t for t in grads if t is not None]
    if not ts:
        return grads
    if any(t.dtype != torch.float32 for t in ts):
        raise ValueError("table gradients are float32")
    world = dist.get_world_size(group)
    flat = torch.cat([t.reshape(-1) for t in ts])
    gathered = torch.empty(world, flat.numel(), dtype=torch.float32, device=flat.device)
    dist.all_gather(list(gathered.unbind(0)), flat, group=group)
    total = (sum_partials or _library_sum)(gathered)
    off = 0
    for t in ts:
        n = t.numel()
        t.copy_(total[off:off + n].view_as(t))
        off += n
    return grads
