"""Plain fp64 CPU oracle for exact relative-position attention.

TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke check and the
benchmark's CPU-baseline arm, never by the library.  It is deliberately
slow and literal: it materialises the full N x N score, probability and
score-gradient matrices of one (batch, head) slice and applies the
definitions directly, with NumPy matmuls as the only library primitive.

Source of every definition: the digest page of "Fast and Exact
Relative-Position Attention via Structure-Aware Kernels" (arXiv 2611.01182),
cited below as [digest] with its section names:
  * score formula, Eq. (1):  S_ij = tau (q_i.k_j + q_i.aQ_phi + k_j.aK_phi + b_phi) + M_ij
  * projections, Eq. (2)/(3): Z^Q_ir = q_i.aQ_r, Z^K_jr = k_j.aK_r
  * relation gradients, Eq. (4): dZ^Q_ir = tau sum_{j: phi(i,j)=r} dS_ij (key side symmetric)
  * "constant tiles and the saturated region": two comparisons of a tile's
    min/max offset against the saturation bounds; bucketed maps expanded to
    a truncated map by copying each bucket row once per offset it covers.
  * experimental setup: Shaw truncated, Transformer-XL identity, DeBERTa
    log buckets, T5 32 bidirectional buckets to distance 128.
The pages leave open the offset sign, the bucket formulas, the mask forms
and the tile-class rule's exact bounds; the readings taken are:
  * offset delta = j - i (key position minus query position);
  * truncated: phi = clamp(delta, -c, c) + c;  identity: phi = delta + N - 1;
  * T5 buckets and DeBERTa log buckets as defined in t5_bucket/log_bucket,
    evaluated in fp64 with a 1e-9 guard so that exact integer crossings of
    the real-valued formula round the way exact arithmetic rounds them;
  * M_ij = -inf where masked (causal: j > i; key padding: j >= key_len[b]);
  * a query row with every key masked has O = 0 and LSE = -inf.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

GUARD = 1e-9

# Tile classes of the tile plan.
MASKED, CONST_LO, BAND, CONST_HI = 0, 1, 2, 3


@dataclass(frozen=True)
class MapDesc:
    """Offset map phi: 'truncated' (clip), 'identity', 't5' (num_buckets,
    max_distance, bidirectional), 'log' (DeBERTa log buckets: num_buckets =
    bucket span, max_distance = max position) or 'log_rev' (the 'log' row of
    the reversed offset -delta = i - j, the query-minus-key position by which
    DeBERTa's content-to-position and position-to-content terms both index
    their relation rows)."""
    kind: str
    clip: int = 0
    num_buckets: int = 0
    max_distance: int = 0
    bidirectional: int = 1


# ----------------------------------------------------------------------------
# Offset maps phi  ([digest] experimental setup; readings in the header)
# ----------------------------------------------------------------------------

def phi_truncated(delta, clip):
    """Truncated map: offsets beyond +-clip saturate to the first/last row."""
    delta = np.asarray(delta, dtype=np.int64)
    return np.clip(delta, -clip, clip) + clip


def phi_identity(delta, N):
    """Identity map: one row per offset, 2N-1 rows."""
    return np.asarray(delta, dtype=np.int64) + (N - 1)


def t5_bucket(delta, num_buckets=32, max_distance=128, bidirectional=1):
    """T5 relative-attention buckets.

    Bidirectional: half the buckets for delta <= 0, the other half (offset by
    num_buckets/2) for delta > 0.  Within a half of size h: magnitudes below
    h/2 get their own bucket; larger magnitudes n get
    h/2 + floor(ln(n/(h/2)) / ln(max_distance/(h/2)) * (h - h/2)), capped at h-1.
    Unidirectional: only delta <= 0 is distinguished (n = max(-delta, 0)).
    """
    delta = np.asarray(delta, dtype=np.int64)
    h = num_buckets
    if bidirectional:
        h = num_buckets // 2
        base = np.where(delta > 0, h, 0)
        n = np.abs(delta)
    else:
        base = np.zeros_like(delta)
        n = np.maximum(-delta, 0)
    exact = h // 2
    nf = np.maximum(n, 1).astype(np.float64)
    x = np.log(nf / exact) / np.log(max_distance / exact) * (h - exact)
    large = exact + np.floor(x + GUARD).astype(np.int64)
    large = np.minimum(large, h - 1)
    return base + np.where(n < exact, n, large)


def log_bucket(delta, num_buckets=256, max_distance=512):
    """DeBERTa log-bucketed relative positions, as a table row in [0, 2*num_buckets).

    mid = num_buckets/2.  |delta| <= mid keeps delta; beyond it the position
    becomes sign(delta) * (mid + ceil(ln(|delta|/mid) / ln((max_distance-1)/mid) * (mid-1))).
    The row is that position + num_buckets, clamped to the table.
    """
    delta = np.asarray(delta, dtype=np.int64)
    mid = num_buckets // 2
    n = np.abs(delta)
    nf = np.maximum(n, 1).astype(np.float64)
    x = np.log(nf / mid) / np.log((max_distance - 1) / mid) * (mid - 1)
    logpos = mid + np.ceil(x - GUARD).astype(np.int64)
    pos = np.where(n <= mid, delta, np.sign(delta) * logpos)
    return np.clip(pos + num_buckets, 0, 2 * num_buckets - 1)


def table_rows(m: MapDesc, N: int) -> int:
    if m.kind == "truncated":
        return 2 * m.clip + 1
    if m.kind == "identity":
        return 2 * N - 1
    if m.kind == "t5":
        return m.num_buckets
    if m.kind in ("log", "log_rev"):
        return 2 * m.num_buckets
    raise ValueError(m.kind)


def phi_of_delta(m: MapDesc, delta, N: int):
    if m.kind == "truncated":
        return phi_truncated(delta, m.clip)
    if m.kind == "identity":
        return phi_identity(delta, N)
    if m.kind == "t5":
        return t5_bucket(delta, m.num_buckets, m.max_distance, m.bidirectional)
    if m.kind == "log":
        return log_bucket(delta, m.num_buckets, m.max_distance)
    if m.kind == "log_rev":
        return log_bucket(-np.asarray(delta, dtype=np.int64), m.num_buckets, m.max_distance)
    raise ValueError(m.kind)


def phi_matrix(m: MapDesc, N: int, rows=None):
    """phi(i, j) for every cell (rows = query positions; all keys), brute force per cell."""
    i = np.arange(N, dtype=np.int64) if rows is None else np.asarray(rows, dtype=np.int64)
    j = np.arange(N, dtype=np.int64)
    return phi_of_delta(m, j[None, :] - i[:, None], N)


def allowed_matrix(N: int, causal: bool, key_len_b: Optional[int], rows=None):
    """True where the additive mask M_ij is 0 (kept), False where it is -inf."""
    i = np.arange(N) if rows is None else np.asarray(rows)
    j = np.arange(N)
    ok = np.ones((len(i), N), dtype=bool)
    if causal:
        ok &= j[None, :] <= i[:, None]
    if key_len_b is not None:
        ok &= j[None, :] < int(key_len_b)
    return ok


# ----------------------------------------------------------------------------
# Expanded (bucket -> truncated) form and the tile plan
# ([digest] "constant tiles and the saturated region")
# ----------------------------------------------------------------------------

def expanded_bounds(m: MapDesc, N: int):
    """Saturation bounds (E_lo, E_hi) over the reachable offsets 1-N .. N-1.

    E_lo is the last offset of the leading run of offsets that share one row
    (every offset <= E_lo maps to that row); E_hi the first offset of the
    trailing run.  The expanded truncated map has one row per offset in
    [E_lo, E_hi]: row(delta) = clamp(delta, E_lo, E_hi) - E_lo.
    """
    deltas = np.arange(1 - N, N, dtype=np.int64)
    p = phi_of_delta(m, deltas, N)
    lo = 0
    while lo + 1 < len(p) and p[lo + 1] == p[0]:
        lo += 1
    hi = len(p) - 1
    while hi - 1 >= 0 and p[hi - 1] == p[-1]:
        hi -= 1
    if hi < lo:            # a single row covers every offset
        hi = lo
    return int(deltas[lo]), int(deltas[hi])


def tile_plan_brute(m: MapDesc, N: int, T: int, causal: bool, key_len=None, B: int = 1):
    """Tile classes by inspecting every cell of every tile.

    A tile is MASKED when none of its in-range cells is kept, CONST_LO/CONST_HI
    when every kept cell maps to the low/high saturated row, BAND otherwise.
    Returns int32 [B, nQ, nK]."""
    nT = (N + T - 1) // T
    elo, ehi = expanded_bounds(m, N)
    row_lo = phi_of_delta(m, np.array([elo]), N)[0]
    row_hi = phi_of_delta(m, np.array([ehi]), N)[0]
    phi = phi_matrix(m, N)
    out = np.zeros((B, nT, nT), dtype=np.int32)
    for b in range(B):
        kl = None if key_len is None else int(key_len[b])
        ok = allowed_matrix(N, causal, kl)
        for qi in range(nT):
            for kj in range(nT):
                sl = (slice(qi * T, min(qi * T + T, N)), slice(kj * T, min(kj * T + T, N)))
                cells = phi[sl][ok[sl]]
                # padding keys beyond key_len are masked; causal cells stay "in range"
                # for classification (the tile is still visited), so classify on
                # the key-valid cells irrespective of causality
                kv = np.ones_like(ok[sl])
                if kl is not None:
                    kv &= (np.arange(kj * T, min(kj * T + T, N)) < kl)[None, :]
                cls_cells = phi[sl][kv]
                if cells.size == 0:
                    out[b, qi, kj] = MASKED
                elif np.all(cls_cells == row_lo):
                    out[b, qi, kj] = CONST_LO
                elif np.all(cls_cells == row_hi):
                    out[b, qi, kj] = CONST_HI
                else:
                    out[b, qi, kj] = BAND
    return out


def tile_plan_rule(m: MapDesc, N: int, T: int, causal: bool, key_len=None, B: int = 1):
    """Tile classes by the two comparisons of the tile's offset range
    [j_min - i_max, j_max - i_min] (keys clipped to the valid length) against
    (E_lo, E_hi).  Returns (classes int32 [B,nQ,nK], segments int32 [B,nQ,4])
    with segments = (end of CONST_LO run, end of BAND run, end of live tiles, nK)."""
    nT = (N + T - 1) // T
    elo, ehi = expanded_bounds(m, N)
    cls = np.zeros((B, nT, nT), dtype=np.int32)
    seg = np.zeros((B, nT, 4), dtype=np.int32)
    for b in range(B):
        nkv = N if key_len is None else int(key_len[b])
        for qi in range(nT):
            i0, i1 = qi * T, min(qi * T + T, N) - 1
            for kj in range(nT):
                j0, j1 = kj * T, min(kj * T + T, N) - 1
                j1v = min(j1, nkv - 1)
                if j0 >= nkv or (causal and j0 > i1):
                    c = MASKED
                elif j1v - i0 <= elo:
                    c = CONST_LO
                elif j0 - i1 >= ehi:
                    c = CONST_HI
                else:
                    c = BAND
                cls[b, qi, kj] = c
            row = cls[b, qi]
            live = int(np.sum(row != MASKED))
            seg[b, qi] = (int(np.sum(row == CONST_LO)),
                          int(np.sum(row == CONST_LO) + np.sum(row == BAND)),
                          live, nT)
    return cls, seg


# ----------------------------------------------------------------------------
# Forward and backward of one (batch, head) slice  ([digest] Eq. (1)-(4))
# ----------------------------------------------------------------------------

def _f64(x):
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().cpu().float().numpy()
    return np.asarray(x, dtype=np.float64)


# ----------------------------------------------------------------------------
# Attention dropout (the scope table's next row f3; not on the pages, the
# standard attention-dropout semantics): O = (P o M / (1 - p')) V with P the
# softmax of S (so LSE is that of S), M_ij in {0, 1}, and p' the rate p
# rounded up to a multiple of 2^-8 (the mask compares 8-bit uniforms).  The
# mask is drawn by the counter-based generator Philox4x32-10 (Salmon, Moraes,
# Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC 2011),
# restated here from that definition: ten rounds of
#     (hi0, lo0) = M0 * x0,  (hi1, lo1) = M1 * x2   (32 x 32 -> 64-bit products)
#     x = (hi1 ^ x1 ^ k0, lo1, hi0 ^ x3 ^ k1, lo0)
# with the key bumped by (W0, W1) before every round after the first.  The
# cell layout (which output byte serves which cell) is in dropout_keep.
# ----------------------------------------------------------------------------

PHILOX_M0, PHILOX_M1 = 0xD2511F53, 0xCD9E8D57
PHILOX_W0, PHILOX_W1 = 0x9E3779B9, 0xBB67AE85


def philox4x32_10(ctr, key):
    """ctr: 4 arrays (or ints) of uint32, key: 2 of them (broadcast together).
    Returns the 4 output words as uint64 arrays holding 32-bit values."""
    mask = np.uint64(0xFFFFFFFF)
    x = [np.asarray(c, dtype=np.uint64) & mask for c in ctr]
    k0, k1 = (np.asarray(c, dtype=np.uint64) & mask for c in key)
    for r in range(10):
        if r > 0:
            k0 = (k0 + np.uint64(PHILOX_W0)) & mask
            k1 = (k1 + np.uint64(PHILOX_W1)) & mask
        p0 = np.uint64(PHILOX_M0) * x[0]
        p1 = np.uint64(PHILOX_M1) * x[2]
        hi0, lo0 = p0 >> np.uint64(32), p0 & mask
        hi1, lo1 = p1 >> np.uint64(32), p1 & mask
        x = [hi1 ^ x[1] ^ k0, lo1, hi0 ^ x[3] ^ k1, lo0]
    return x


def dropout_rate(p):
    """The rate the mask realises: p rounded up to a multiple of 2^-8 (a cell is
    dropped when its 8-bit uniform u has u 2^-8 < p, i.e. u < ceil(256 p))."""
    return np.ceil(np.float64(p) * 256.0) / 256.0


def dropout_keep(bh, rows, N, p, seed, offset):
    """Kept cells [len(rows), N] (bool) of slice bh = b * H + h.

    One Philox4x32-10 call serves a block of 4 query rows x 4 keys: counter
    (j >> 2, i >> 2, bh, offset), key (low, high 32 bits of seed).  Query row
    i & 3 of the block reads output word i & 3, key j & 3 its byte j & 3 (least
    significant byte first), as a uniform u in [0, 256); the cell is kept when
    u 2^-8 >= p."""
    i = np.asarray(rows, dtype=np.uint64)[:, None]
    j = np.arange(N, dtype=np.uint64)[None, :]
    w = philox4x32_10((j >> np.uint64(2), i >> np.uint64(2), np.uint64(bh), np.uint64(offset & 0xFFFFFFFF)),
                      (np.uint64(seed & 0xFFFFFFFF), np.uint64((seed >> 32) & 0xFFFFFFFF)))
    word = np.choose((i & np.uint64(3)).astype(np.int64) + np.zeros(w[0].shape, dtype=np.int64), w)
    u8 = (word >> (np.uint64(8) * (j & np.uint64(3)))) & np.uint64(0xFF)
    return u8.astype(np.float64) * 2.0 ** -8 >= p


def head_scores(q, k, aq, ak, bvec, tau, phi, allowed):
    """S for query rows q [n, d] against all keys k [N, d] (Eq. (1) via Eq. (2)/(3)).

    phi [n, N] row indices, allowed [n, N] mask.  Returns S with -inf where masked."""
    N = k.shape[0]
    S = q @ k.T
    if aq is not None:
        ZQ = q @ aq.T                                   # Z^Q_ir = q_i . aQ_r
        S = S + np.take_along_axis(ZQ, phi, axis=1)     # Z^Q_{i, phi(i,j)}
    if ak is not None:
        ZK = k @ ak.T                                   # Z^K_jr = k_j . aK_r
        S = S + ZK[np.arange(N)[None, :], phi]          # Z^K_{j, phi(i,j)}
    if bvec is not None:
        S = S + bvec[phi]                               # b_{phi(i,j)}
    S = tau * S
    return np.where(allowed, S, -np.inf)


def head_softmax(S):
    """Row softmax with logsumexp; rows with every entry masked give P = 0, LSE = -inf."""
    m = S.max(axis=1, keepdims=True)
    dead = ~np.isfinite(m[:, 0])
    m_safe = np.where(np.isfinite(m), m, 0.0)
    E = np.exp(S - m_safe)
    l = E.sum(axis=1, keepdims=True)
    P = np.where(l > 0, E / np.where(l > 0, l, 1.0), 0.0)
    lse = np.where(dead, -np.inf, m_safe[:, 0] + np.log(np.where(l[:, 0] > 0, l[:, 0], 1.0)))
    return P, lse


def head_forward(q, k, v, aq, ak, bvec, tau, phi, allowed, keep=None, p=0.0):
    """O, LSE, P of one slice; with `keep` (bool [n, N]) O uses P o keep / (1 - p)
    (p: the realised rate, dropout_rate of the requested one)."""
    S = head_scores(q, k, aq, ak, bvec, tau, phi, allowed)
    P, lse = head_softmax(S)
    Pv = P if keep is None else np.where(keep, P / (1.0 - p), 0.0)
    return Pv @ v, lse, P


def head_backward(q, k, v, do, aq, ak, bvec, tau, phi, allowed, R, keep=None, p=0.0):
    """Gradients of one full (b, h) slice for the upstream gradient dO.

    Returns dict: dq, dk, dv, dzq [N,R], dzk [N,R], daq [R,d], dak [R,d], db [R],
    plus o, lse.  With dropout (`keep`), O = (P o M s) V, s = 1 / (1 - p) (p the realised rate):
    dV = (P o M s)^T dO, dS = P o (M s o dO V^T - D), D_i = sum_c dO_ic O_ic."""
    N, d = q.shape
    O, lse, P = head_forward(q, k, v, aq, ak, bvec, tau, phi, allowed, keep, p)
    Ms = None if keep is None else np.where(keep, 1.0 / (1.0 - p), 0.0)
    dV = (P if Ms is None else P * Ms).T @ do
    dP = do @ v.T
    if Ms is not None:
        dP = dP * Ms
    D = np.sum(do * O, axis=1, keepdims=True)
    dS = P * (dP - D)                                   # gradient w.r.t. S (incl. tau)
    rows = np.repeat(np.arange(N), N)
    cols = np.tile(np.arange(N), N)
    flat_phi = phi.reshape(-1)
    # Eq. (4): dZ^Q_ir = tau sum_{j: phi(i,j)=r} dS_ij ; dZ^K_jr = tau sum_{i: phi(i,j)=r} dS_ij
    dzq = tau * np.bincount(rows * R + flat_phi, weights=dS.reshape(-1), minlength=N * R).reshape(N, R)
    dzk = tau * np.bincount(cols * R + flat_phi, weights=dS.reshape(-1), minlength=N * R).reshape(N, R)
    dq = tau * (dS @ k)
    dk = tau * (dS.T @ q)
    out = dict(dv=dV, o=O, lse=lse, dzq=dzq, dzk=dzk)
    if aq is not None:
        dq = dq + dzq @ aq
        out["daq"] = dzq.T @ q
    if ak is not None:
        dk = dk + dzk @ ak
        out["dak"] = dzk.T @ k
    if bvec is not None:
        out["db"] = tau * np.bincount(flat_phi, weights=dS.reshape(-1), minlength=R)
    out["dq"] = dq
    out["dk"] = dk
    return out


# ----------------------------------------------------------------------------
# Whole-layer wrappers over [B, H, N, d]
# ----------------------------------------------------------------------------

def _table(t, h):
    if t is None:
        return None
    return t[h] if t.ndim == 3 else t


def forward(q, k, v, aq, ak, b, tau, m: MapDesc, causal=False, key_len=None, rows=None,
            dropout_p=0.0, dropout_seed=0, dropout_offset=0):
    """O [B,H,n,d] and LSE [B,H,n] for the query rows `rows` (default all).

    q, k, v: [B,H,N,d]; aq, ak: [R,d] (shared) or [H,R,d] (per head) or None;
    b: [H,R] or None; key_len: [B] or None; dropout as in dropout_keep."""
    q, k, v, aq, ak, b = (_f64(x) for x in (q, k, v, aq, ak, b))
    B, H, N, d = q.shape
    rows = np.arange(N) if rows is None else np.asarray(rows)
    kl = None if key_len is None else np.asarray(key_len).reshape(-1)
    phi = phi_matrix(m, N, rows)
    O = np.zeros((B, H, len(rows), d))
    L = np.zeros((B, H, len(rows)))
    for bi in range(B):
        allowed = allowed_matrix(N, causal, None if kl is None else kl[bi], rows)
        for h in range(H):
            keep = None if dropout_p == 0 else dropout_keep(bi * H + h, rows, N, dropout_p, dropout_seed,
                                                             dropout_offset)
            o, lse, _ = head_forward(q[bi, h, rows], k[bi, h], v[bi, h], _table(aq, h),
                                     _table(ak, h), None if b is None else b[h], tau, phi, allowed, keep,
                                     dropout_rate(dropout_p))
            O[bi, h], L[bi, h] = o, lse
    return O, L


def backward(q, k, v, do, aq, ak, b, tau, m: MapDesc, causal=False, key_len=None,
             dropout_p=0.0, dropout_seed=0, dropout_offset=0):
    """All outputs and gradients of the layer for upstream gradient dO.

    Shared tables ([R,d]) get gradients summed over batch then heads in
    ascending order; per-head tables ([H,R,d]) summed over batch only;
    db [H,R] summed over batch."""
    q, k, v, do, aq, ak, b = (_f64(x) for x in (q, k, v, do, aq, ak, b))
    B, H, N, d = q.shape
    R = table_rows(m, N)
    kl = None if key_len is None else np.asarray(key_len).reshape(-1)
    phi = phi_matrix(m, N)
    res = {n: np.zeros((B, H, N, d)) for n in ("o", "dq", "dk", "dv")}
    res["lse"] = np.zeros((B, H, N))
    daq = None if aq is None else np.zeros(aq.shape)
    dak = None if ak is None else np.zeros(ak.shape)
    db = None if b is None else np.zeros(b.shape)
    for h in range(H):
        for bi in range(B):
            allowed = allowed_matrix(N, causal, None if kl is None else kl[bi])
            keep = None if dropout_p == 0 else dropout_keep(bi * H + h, np.arange(N), N, dropout_p, dropout_seed,
                                                             dropout_offset)
            g = head_backward(q[bi, h], k[bi, h], v[bi, h], do[bi, h], _table(aq, h),
                              _table(ak, h), None if b is None else b[h], tau, phi, allowed, R, keep,
                              dropout_rate(dropout_p))
            for n in ("o", "dq", "dk", "dv", "lse"):
                res[n][bi, h] = g[n]
            if aq is not None:
                if aq.ndim == 3:
                    daq[h] += g["daq"]
                else:
                    daq += g["daq"]
            if ak is not None:
                if ak.ndim == 3:
                    dak[h] += g["dak"]
                else:
                    dak += g["dak"]
            if b is not None:
                db[h] += g["db"]
    res["daq"], res["dak"], res["db"] = daq, dak, db
    return res


# ----------------------------------------------------------------------------
# Sampled evaluation for sequence lengths where whole N x N matrices per head
# are too large to keep: the definitions above applied to chosen query rows
# (dQ) and chosen key columns (dK, dV).  Every query row of the forward is
# independent, so O and LSE of all rows are produced row-chunk by row-chunk.
# ----------------------------------------------------------------------------

def head_forward_all_rows(q, k, v, aq, ak, bvec, tau, m: MapDesc, causal, key_len_b, chunk=1024):
    N = q.shape[0]
    O = np.zeros_like(q)
    L = np.zeros(N)
    for r0 in range(0, N, chunk):
        rows = np.arange(r0, min(N, r0 + chunk))
        phi = phi_matrix(m, N, rows)
        allowed = allowed_matrix(N, causal, key_len_b, rows)
        o, lse, _ = head_forward(q[rows], k, v, aq, ak, bvec, tau, phi, allowed)
        O[rows], L[rows] = o, lse
    return O, L


def head_grads_sampled(q, k, v, do, aq, ak, bvec, tau, m: MapDesc, causal, key_len_b, qrows, kcols, chunk=1024):
    """dQ at query rows `qrows` and dK, dV at key columns `kcols` of one (b, h) slice,
    plus O and LSE of every row.  Same formulas as head_backward."""
    N = q.shape[0]
    O, L = head_forward_all_rows(q, k, v, aq, ak, bvec, tau, m, causal, key_len_b, chunk)
    D = np.sum(do * O, axis=1)
    R = table_rows(m, N)
    # query rows
    qrows = np.asarray(qrows)
    phi = phi_matrix(m, N, qrows)
    allowed = allowed_matrix(N, causal, key_len_b, qrows)
    S = head_scores(q[qrows], k, aq, ak, bvec, tau, phi, allowed)
    Lr = L[qrows][:, None]
    P = np.where(np.isfinite(Lr), np.exp(S - np.where(np.isfinite(Lr), Lr, 0.0)), 0.0)
    dS = P * (do[qrows] @ v.T - D[qrows][:, None])
    dq = tau * (dS @ k)
    if aq is not None:
        dzq = np.zeros((len(qrows), R))
        for a in range(len(qrows)):
            dzq[a] = tau * np.bincount(phi[a], weights=dS[a], minlength=R)
        dq = dq + dzq @ aq
    # key columns: scores of every query row against the chosen keys
    kcols = np.asarray(kcols)
    dk = np.zeros((len(kcols), q.shape[1]))
    dv = np.zeros_like(dk)
    dzk = np.zeros((len(kcols), R))
    for r0 in range(0, N, chunk):
        rows = np.arange(r0, min(N, r0 + chunk))
        i = rows[:, None]
        j = kcols[None, :]
        phi_c = phi_of_delta(m, j - i, N)
        ok = allowed_matrix(N, causal, key_len_b, rows)[:, kcols]
        Sc = q[rows] @ k[kcols].T
        if aq is not None:
            ZQ = q[rows] @ aq.T
            Sc = Sc + np.take_along_axis(ZQ, phi_c, axis=1)
        if ak is not None:
            ZK = k[kcols] @ ak.T
            Sc = Sc + ZK[np.arange(len(kcols))[None, :], phi_c]
        if bvec is not None:
            Sc = Sc + bvec[phi_c]
        Sc = np.where(ok, tau * Sc, -np.inf)
        Lc = L[rows][:, None]
        Pc = np.where(np.isfinite(Lc), np.exp(Sc - np.where(np.isfinite(Lc), Lc, 0.0)), 0.0)
        dSc = Pc * (do[rows] @ v[kcols].T - D[rows][:, None])
        dv += Pc.T @ do[rows]
        dk += tau * (dSc.T @ q[rows])
        for c in range(len(kcols)):
            dzk[c] += tau * np.bincount(phi_c[:, c], weights=dSc[:, c], minlength=R)
    if ak is not None:
        dk = dk + dzk @ ak
    return dict(o=O, lse=L, dq=dq, dk=dk, dv=dv)


def head_block_step(q, k, v, do, aq, ak, bvec, tau, m: MapDesc, causal, key_len_b, rows):
    """Forward and backward restricted to the query rows `rows` of one (b, h) slice.

    Returns the block's outputs (o, lse, dq for those rows) and its additive
    contributions to the sums over query rows (dv, dk, daq, dak, db).  Summed
    over a partition of the rows these contributions give head_backward's
    dV, dK and table gradients; this is the unit of work the CPU baseline
    times."""
    N = k.shape[0]
    rows = np.asarray(rows)
    R = table_rows(m, N)
    phi = phi_matrix(m, N, rows)
    allowed = allowed_matrix(N, causal, key_len_b, rows)
    O, lse, P = head_forward(q[rows], k, v, aq, ak, bvec, tau, phi, allowed)
    D = np.sum(do[rows] * O, axis=1, keepdims=True)
    dS = P * (do[rows] @ v.T - D)
    n = len(rows)
    ri = np.repeat(np.arange(n), N)
    cj = np.tile(np.arange(N), n)
    fp = phi.reshape(-1)
    out = dict(o=O, lse=lse, dv=P.T @ do[rows], dq=tau * (dS @ k), dk=tau * (dS.T @ q[rows]))
    # each relation gradient only when its term is present (the key-side one is
    # N x R per block: 4 GB for the identity map at N = 16384)
    if aq is not None:
        dzq = tau * np.bincount(ri * R + fp, weights=dS.reshape(-1), minlength=n * R).reshape(n, R)
        out["dq"] = out["dq"] + dzq @ aq
        out["daq"] = dzq.T @ q[rows]
    if ak is not None:
        dzk = tau * np.bincount(cj * R + fp, weights=dS.reshape(-1), minlength=N * R).reshape(N, R)
        out["dak"] = dzk.T @ k
        out["dk_rel"] = dzk @ ak
    if bvec is not None:
        out["db"] = tau * np.bincount(fp, weights=dS.reshape(-1), minlength=R)
    return out


def head_table_grads(q, k, v, do, aq, ak, bvec, tau, m: MapDesc, causal, key_len_b, block=512):
    """Table gradients daq, dak, db of one (b, h) slice (those whose term is
    present), as the sum of head_block_step's contributions over consecutive
    blocks of query rows: the Eq. (4) sums taken over all query rows without
    holding an N x N matrix."""
    N = q.shape[0]
    acc = {}
    for r0 in range(0, N, block):
        part = head_block_step(q, k, v, do, aq, ak, bvec, tau, m, causal, key_len_b,
                               np.arange(r0, min(N, r0 + block)))
        for name in ("daq", "dak", "db"):
            if name in part:
                acc[name] = part[name] if name not in acc else acc[name] + part[name]
    return acc
