"""Packed variable-length batches: sequences of different lengths stored back
to back (token-major [T, H, d], cu_seqlens [B + 1]), each attending only to
its own keys.

Reference: the same sequences padded to the longest one, with the padded
keys masked (key_len = the lengths) and the upstream gradient zero on the
padded query rows, so that those rows add nothing to dK, dV or the table
gradients; the fp64 oracle of that padded batch, restricted to the real rows,
is the packed batch's answer.  Outputs, every gradient and the table
gradients are compared element by element, for every map, both masks, both
dtypes, the recompute projection, empty and one-token sequences.
"""
import numpy as np
import pytest
import torch

from synth import small_workload
from relpos_harness import check_backward, check_forward, lmap, run_oracle
import exact_relative_position_b200 as rp

pytestmark = pytest.mark.gpu


def _pack(x, lens):
    """[B, H, N, d] -> token-major [T, H, d] of the real rows."""
    return torch.cat([x[b, :, :n].transpose(0, 1) for b, n in enumerate(lens)], dim=0).contiguous()


def _unpack(x, lens, N):
    """[T, H, d] (or [H, T] for the LSE) -> [B, H, N, ...] with zeros on padded rows."""
    lse = x.dim() == 2
    H = x.shape[0] if lse else x.shape[1]
    out = torch.zeros((len(lens), H, N) + (() if lse else (x.shape[2],)), dtype=x.dtype, device=x.device)
    r = 0
    for b, n in enumerate(lens):
        out[b, :, :n] = x[:, r:r + n] if lse else x[r:r + n].transpose(0, 1)
        r += n
    return out


CASES = [
    dict(map_kind="truncated", clip=16, lens=[300, 1, 129, 517], terms=("aQ", "aK", "b")),
    dict(map_kind="identity", lens=[517, 200, 0, 64], terms=("aQ", "b"), causal=True, per_head_tables=True),
    dict(map_kind="log", num_buckets=32, max_distance=128, lens=[255, 384, 2], terms=("aQ", "aK"),
         dtype=torch.bfloat16),
    dict(map_kind="t5", num_buckets=32, max_distance=128, lens=[128, 640], terms=("b",), causal=True),
    dict(map_kind="identity", lens=[333, 129], terms=("aQ", "b"), projection="recompute"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c['map_kind']}-{'-'.join(map(str, c['lens']))}"
                                                     f"{'-rc' if c.get('projection') else ''}")
def test_packed_batch_matches_padded_oracle(case):
    case = dict(case)
    lens = case.pop("lens")
    projection = case.pop("projection", "retained")
    N = max(lens)
    w = small_workload(N=N, B=len(lens), H=2, key_len=lens, **case)
    for b, n in enumerate(lens):          # padded query rows carry no upstream gradient
        w.do[b, :, n:] = 0
    out_f32 = w.dtype == torch.bfloat16
    cu = torch.tensor(np.concatenate([[0], np.cumsum(lens)]), dtype=torch.int32, device="cuda")
    d = lambda t: None if t is None else t.to("cuda").contiguous()
    q, k, v, do = (_pack(d(getattr(w, n)), lens) for n in ("q", "k", "v", "do"))
    aq, ak, b = d(w.aq), d(w.ak), d(w.b)
    kw = dict(tau=w.tau, map=lmap(w), causal=w.causal, cu_seqlens=cu, max_seqlen=N, projection=projection)
    o, lse = rp.relpos_attn_fwd(q, k, v, aq, ak, b, out_f32=out_f32, **kw)
    dq, dk, dv, daq, dak, db = rp.relpos_attn_bwd(do, q, k, v, o, lse, aq, ak, b, **kw)
    torch.cuda.synchronize()
    f64 = lambda t: None if t is None else t.double().cpu().numpy()
    got = dict(o=f64(_unpack(o, lens, N)), lse=f64(_unpack(lse, lens, N)), dq=f64(_unpack(dq, lens, N)),
               dk=f64(_unpack(dk, lens, N)), dv=f64(_unpack(dv, lens, N)), daq=f64(daq), dak=f64(dak), db=f64(db))
    want = run_oracle(w)
    # compare the real rows only: padded rows are not part of a packed batch
    rows = np.zeros((len(lens), N), bool)
    for bi, n in enumerate(lens):
        rows[bi, :n] = True
    for name in ("o", "dq", "dk", "dv"):
        got[name] = np.where(rows[:, None, :, None], got[name], 0.0)
        want[name] = np.where(rows[:, None, :, None], want[name], 0.0)
    got["lse"] = np.where(rows[:, None, :], got["lse"], 0.0)
    want["lse"] = np.where(rows[:, None, :], want["lse"], 0.0)
    check_forward(got, want, str(lens))
    check_backward(got, want, str(lens))
