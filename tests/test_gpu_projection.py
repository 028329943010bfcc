"""The grouped projections Z^Q = Q aQ_exp^T and Z^K = K aK_exp^T as the library
stores them ([digest] Eq. (2)/(3), "grouped reachable range"), read back
through relpos_debug_projection and compared with the oracle's definition
column by column: every stored column of every 128-row group, and that each
group stores every offset its rows can reach (so a wrong column in a part of
a group that no tile happens to read would still be caught).
"""
import numpy as np
import pytest
import torch

import oracle as orc
from synth import small_workload
from relpos_harness import lmap, omap, to_dev
import exact_relative_position_b200 as rp

pytestmark = pytest.mark.gpu

CASES = {
    # identity map past N = 512: R_exp = 2N - 1 > N + 127, so each group stores its own reach
    "identity_grouped": dict(map_kind="identity", N=520, B=1, H=2, terms=("aQ", "aK")),
    "identity_grouped_causal": dict(map_kind="identity", N=520, B=2, H=1, terms=("aQ", "aK"), causal=True),
    "identity_ragged_bf16": dict(map_kind="identity", N=777, B=1, H=1, terms=("aQ", "aK"), dtype=torch.bfloat16,
                                 per_head_tables=True),
    "truncated_per_head": dict(map_kind="truncated", clip=16, N=300, B=2, H=3, terms=("aQ", "aK"),
                               per_head_tables=True),
    # bucketed maps: the expanded table copies each bucket row once per offset it covers
    "log_buckets": dict(map_kind="log", num_buckets=32, max_distance=128, N=600, B=1, H=2, terms=("aQ", "aK")),
    "t5_query_side": dict(map_kind="t5", num_buckets=32, max_distance=128, bidirectional=1, N=400, B=1, H=2,
                          terms=("aQ", "b")),
}


def _floats(ws, off, n):
    return ws[off:off + 4 * n].view(torch.float32).cpu().double().numpy()


@pytest.mark.parametrize("case", sorted(CASES))
def test_projection_every_stored_column(case):
    w = small_workload(**CASES[case])
    dev = to_dev(w)
    N, B, H = w.N, w.B, w.H
    lay, ws, (gq, gq_base), (gk, gk_base) = rp.debug_projection(
        dev["q"], dev["k"], dev["aq"], dev["ak"], dev["b"], tau=w.tau, map=lmap(w), causal=w.causal,
        key_len=dev["key_len"])
    m = omap(w)
    elo, ehi = orc.expanded_bounds(m, N)
    assert (lay.E_lo, lay.E_hi, lay.R_exp, lay.nT) == (elo, ehi, ehi - elo + 1, (N + 127) // 128)
    table_row = orc.phi_of_delta(m, np.arange(elo, ehi + 1), N)      # table row of each expanded column
    nT = lay.nT
    for side, X, A, off, head, gi, gb in (("q", w.q, w.aq, lay.zq_offset, lay.zq_head, gq, gq_base),
                                          ("k", w.k, w.ak, lay.zk_offset, lay.zk_head, gk, gk_base)):
        if A is None:
            assert off == -1
            continue
        Z = _floats(ws, off, B * H * head).reshape(B * H, head)
        X64, A64 = X.double().numpy(), A.double().numpy()
        for bh in range(B * H):
            b_, h = divmod(bh, H)
            A_exp = (A64[h] if A64.ndim == 3 else A64)[table_row]      # [R_exp, d]
            for g in range(nT):
                e0, W, S, _ = (int(x) for x in gi[g])
                base = int(gb[g])
                r0, n = 128 * g, min(128, N - 128 * g)
                # reach: query i sees offsets [-i, N-1-i], key j sees [j-(N-1), j]; causal keeps <= 0
                lo, hi = (-(r0 + n - 1), N - 1 - r0) if side == "q" else (r0 - (N - 1), r0 + n - 1)
                if w.causal:
                    hi = min(hi, 0)
                lo_e, hi_e = min(max(lo, elo), ehi) - elo, min(max(hi, elo), ehi) - elo
                assert e0 <= lo_e and hi_e < e0 + W <= lay.R_exp, (case, side, g, e0, W, lo_e, hi_e)
                assert W <= min(lay.R_exp, N + 127) and S >= W and S % 4 == 0
                got = Z[bh, base:base + n * S].reshape(n, S)[:, :W]
                xs = X64[b_, h, r0:r0 + n]
                ref = xs @ A_exp[e0:e0 + W].T
                # fp16/bf16 products are exact in fp32; 64-term fp32 sums stay within 1e-5 of sum |terms|
                bound = 1e-5 * (np.abs(xs) @ np.abs(A_exp[e0:e0 + W]).T) + 1e-30
                bad = np.abs(got - ref) > bound
                assert not bad.any(), (case, side, bh, g, np.argwhere(bad)[:5])
