"""Pins of the fp64 oracle to facts outside itself (CPU only).

Each test fixes the oracle against a closed form, an invariant of the
mathematics, a library routine (torch scaled-dot-product attention in fp64),
brute-force evaluation at high precision, or central finite differences,
chosen so that a dropped term, a flipped offset sign or a transposed operand
anywhere in the oracle fails one of them.  Definitions follow the digest page
of "Fast and Exact Relative-Position Attention via Structure-Aware Kernels"
(Eq. (1)-(4); "constant tiles and the saturated region").
"""
import decimal
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------
# Offset maps
# --------------------------------------------------------------------------

def _dec_ln(x, prec=60):
    with decimal.localcontext() as c:
        c.prec = prec
        return decimal.Decimal(x).ln()


def _t5_decimal(delta, nb, md, bidir):
    """T5 bucket with the logarithm evaluated in 60-digit decimal arithmetic."""
    h = nb // 2 if bidir else nb
    base = h if (bidir and delta > 0) else 0
    n = abs(delta) if bidir else max(-delta, 0)
    exact = h // 2
    if n < exact:
        return base + n
    with decimal.localcontext() as c:
        c.prec = 60
        x = _dec_ln(decimal.Decimal(n) / exact) / _dec_ln(decimal.Decimal(md) / exact) * (h - exact)
        t = int(x.to_integral_value(rounding=decimal.ROUND_FLOOR))
    return base + min(exact + t, h - 1)


def _log_decimal(delta, nb, md):
    """DeBERTa log bucket row with 60-digit decimal logarithms."""
    mid = nb // 2
    n = abs(delta)
    if n <= mid:
        pos = delta
    else:
        with decimal.localcontext() as c:
            c.prec = 60
            x = _dec_ln(decimal.Decimal(n) / mid) / _dec_ln(decimal.Decimal(md - 1) / mid) * (mid - 1)
            t = int(x.to_integral_value(rounding=decimal.ROUND_CEILING))
        pos = int(math.copysign(mid + t, delta))
    return min(max(pos + nb, 0), 2 * nb - 1)


@pytest.mark.parametrize("nb,md,bidir", [(32, 128, 1), (32, 128, 0), (64, 256, 1), (16, 64, 1)])
def test_t5_bucket_matches_high_precision(nb, md, bidir):
    deltas = np.arange(-3000, 3001)
    got = orc.t5_bucket(deltas, nb, md, bidir)
    want = np.array([_t5_decimal(int(x), nb, md, bidir) for x in deltas])
    assert np.array_equal(got, want)


def test_t5_bucket_integer_form_standard_constants():
    # For 32 bidirectional buckets / distance 128: large bucket = 8 + floor(2 log2(n/8)),
    # i.e. the largest t with 64 * 2^t <= n^2 (exact integer arithmetic).
    for delta in range(-20000, 20001, 7):
        n = abs(delta)
        base = 16 if delta > 0 else 0
        if n < 8:
            want = base + n
        else:
            t = 0
            while 64 * 2 ** (t + 1) <= n * n:
                t += 1
            want = base + min(8 + t, 15)
        assert orc.t5_bucket(delta) == want, delta


def test_t5_closed_form_values():
    # hand-derived values of the bidirectional 32/128 map
    cases = {0: 0, -1: 1, -7: 7, -8: 8, -11: 8, -12: 9, -16: 10, -90: 14, -91: 15,
             -10 ** 6: 15, 1: 17, 7: 23, 8: 24, 91: 31, 10 ** 6: 31}
    for d, want in cases.items():
        assert orc.t5_bucket(d) == want, d


@pytest.mark.parametrize("nb,md", [(256, 512), (128, 256), (64, 512)])
def test_log_bucket_matches_high_precision(nb, md):
    deltas = np.arange(-4000, 4001)
    got = orc.log_bucket(deltas, nb, md)
    want = np.array([_log_decimal(int(x), nb, md) for x in deltas])
    assert np.array_equal(got, want)


def test_log_bucket_saturation_and_coverage():
    d = np.arange(-3000, 3001)
    rows = orc.log_bucket(d, 256, 512)
    assert np.all(np.diff(rows) >= 0)                   # monotone in the offset
    assert set(rows.tolist()) == set(range(512))        # every row is reached
    # closed forms: row 0 iff delta <= -512 (ceil(127 ln(n/128)/ln(511/128)) >= 128 iff n >= 512);
    # row 511 iff delta >= 506 (127 ln(n/128)/ln(511/128) > 126 iff n > 128 (511/128)^(126/127) = 505.4)
    assert rows[d == -512][0] == 0 and rows[d == -511][0] == 1
    assert rows[d == 506][0] == 511 and rows[d == 505][0] == 510
    assert orc.expanded_bounds(orc.MapDesc("log", num_buckets=256, max_distance=512), 2048) == (-512, 506)


@pytest.mark.parametrize("nb,md", [(256, 512), (64, 512)])
def test_log_rev_map_matches_high_precision(nb, md):
    """'log_rev' is the DeBERTa bucket row of the query-minus-key position
    i - j = -delta: the decimal evaluation of the log formula at -delta."""
    deltas = np.arange(-4000, 4001)
    got = orc.phi_of_delta(orc.MapDesc("log_rev", num_buckets=nb, max_distance=md), deltas, 5000)
    want = np.array([_log_decimal(-int(x), nb, md) for x in deltas])
    assert np.array_equal(got, want)


def test_log_rev_saturation_closed_forms():
    m = orc.MapDesc("log_rev", num_buckets=256, max_distance=512)
    d = np.arange(-3000, 3001)
    rows = orc.phi_of_delta(m, d, 3001)
    assert np.all(np.diff(rows) <= 0)                   # monotone, decreasing in delta = j - i
    # mirror of the 'log' map's closed forms: row 511 iff delta <= -506, row 0 iff delta >= 512
    assert rows[d == -506][0] == 511 and rows[d == -505][0] == 510
    assert rows[d == 512][0] == 0 and rows[d == 511][0] == 1
    assert orc.expanded_bounds(m, 2048) == (-506, 512)
    assert orc.table_rows(m, 2048) == 512


def test_deberta_disentangled_score_is_unified_with_log_rev():
    """DeBERTa's disentangled score, built the way its attention forms it --
    c2p gathers q_i . K^r at the bucket row of the relative position i - j;
    p2c gathers k . Q^r key-major at the row of the negated relative position
    and is then transposed -- equals Eq. (1) with aQ = K^r, aK = Q^r and the
    one map 'log_rev' (both terms land on the row of i - j)."""
    N, d, nb, md = 37, 4, 8, 24
    rng = np.random.default_rng(11)
    q, k = rng.standard_normal((N, d)), rng.standard_normal((N, d))
    Kr, Qr = rng.standard_normal((2 * nb, d)), rng.standard_normal((2 * nb, d))
    tau = 1.0 / math.sqrt(3 * d)
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    rel = i - j                                          # relative position, query minus key
    c2p_idx = orc.log_bucket(rel, nb, md)                # [query, key]
    c2p = np.take_along_axis(q @ Kr.T, c2p_idx, axis=1)
    p2c_idx = orc.log_bucket(-rel, nb, md)               # the negated relative position matrix
    g = np.take_along_axis(k @ Qr.T, p2c_idx, axis=1)    # rows of the key-major product
    p2c = g.T
    want = tau * (q @ k.T + c2p + p2c)
    phi = orc.phi_matrix(orc.MapDesc("log_rev", num_buckets=nb, max_distance=md), N)
    got = orc.head_scores(q, k, Kr, Qr, None, tau, phi, np.ones((N, N), bool))
    np.testing.assert_allclose(got, want, rtol=1e-13, atol=1e-13)


def test_truncated_identity_closed_forms():
    d = np.arange(-50, 51)
    assert np.array_equal(orc.phi_truncated(d, 16), np.minimum(np.maximum(d, -16), 16) + 16)
    assert np.array_equal(orc.phi_identity(d, 51), d + 50)
    assert orc.table_rows(orc.MapDesc("truncated", clip=16), 256) == 33
    assert orc.table_rows(orc.MapDesc("truncated", clip=64), 8192) == 129
    assert orc.table_rows(orc.MapDesc("identity"), 16384) == 32767


def test_phi_matrix_sign_convention():
    # phi(i, j) depends on the key position minus the query position, cell by cell
    m = orc.MapDesc("identity")
    N = 9
    P = orc.phi_matrix(m, N)
    for i in range(N):
        for j in range(N):
            assert P[i, j] == (j - i) + N - 1


def test_expanded_bounds_cases():
    t5 = orc.MapDesc("t5", num_buckets=32, max_distance=128, bidirectional=1)
    assert orc.expanded_bounds(t5, 8192) == (-91, 91)
    assert orc.expanded_bounds(orc.MapDesc("truncated", clip=16), 256) == (-16, 16)
    assert orc.expanded_bounds(orc.MapDesc("truncated", clip=64), 8192) == (-64, 64)
    assert orc.expanded_bounds(orc.MapDesc("identity"), 100) == (-99, 99)
    # clip beyond the sequence: nothing saturates
    assert orc.expanded_bounds(orc.MapDesc("truncated", clip=500), 100) == (-99, 99)
    # short sequence for T5: offsets 46..49 already share bucket 13 (8 + floor(2 log2(n/8))
    # is 13 for 45.3 <= n < 64), so the leading/trailing runs start at +-46
    assert orc.expanded_bounds(t5, 50) == (-46, 46)


def test_golden_pages_facts():
    """Facts the digest page states (tests/golden/pages_facts.json, each entry cited)."""
    with open(os.path.join(GOLDEN, "pages_facts.json")) as f:
        g = json.load(f)
    for case in g["maps"]:
        m = orc.MapDesc(**case["map"])
        assert orc.table_rows(m, case["N"]) == case["rows"], case["cite"]
        rows = orc.phi_of_delta(m, np.arange(1 - case["N"], case["N"]), case["N"])
        assert len(set(rows.tolist())) == case["distinct_rows_reached"], case["cite"]
    ov = g["group_overhead"]
    assert abs((ov["G"] - 1) / ov["N"] - ov["fraction"]) < ov["abs_tol"], ov["cite"]


# --------------------------------------------------------------------------
# Forward pins
# --------------------------------------------------------------------------

def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _sdpa(q, k, v, mask, tau):
    t = lambda x: torch.from_numpy(np.ascontiguousarray(x))
    out = torch.nn.functional.scaled_dot_product_attention(
        t(q)[None], t(k)[None], t(v)[None], attn_mask=None if mask is None else t(mask)[None], scale=tau)
    return out[0].numpy()


@pytest.mark.parametrize("causal", [False, True])
def test_no_relation_terms_is_softmax_attention(causal):
    B, H, N, d = 1, 2, 37, 8
    q, k, v = (_rand((B, H, N, d), s) for s in range(3))
    m = orc.MapDesc("truncated", clip=4)
    O, L = orc.forward(q, k, v, None, None, None, 0.3, m, causal=causal)
    for h in range(H):
        mask = None
        if causal:
            mask = np.where(np.tril(np.ones((N, N), bool)), 0.0, -np.inf)
        ref = _sdpa(q[0, h], k[0, h], v[0, h], mask, 0.3)
        np.testing.assert_allclose(O[0, h], ref, rtol=1e-12, atol=1e-12)
        # LSE against its definition, log of the summed exponentials (textbook form)
        S = 0.3 * q[0, h] @ k[0, h].T
        if causal:
            S = np.where(np.tril(np.ones((N, N), bool)), S, -np.inf)
        np.testing.assert_allclose(L[0, h], np.log(np.exp(S).sum(1)), rtol=1e-12)


@pytest.mark.parametrize("kind", ["truncated", "identity", "t5", "log"])
def test_relation_terms_cell_by_cell(kind):
    """Eq. (1) evaluated per cell with vector dot products, fed to SDPA as a float mask."""
    N, d, H = 23, 4, 2
    m = {"truncated": orc.MapDesc("truncated", clip=5), "identity": orc.MapDesc("identity"),
         "t5": orc.MapDesc("t5", num_buckets=8, max_distance=16, bidirectional=1),
         "log": orc.MapDesc("log", num_buckets=8, max_distance=16)}[kind]
    R = orc.table_rows(m, N)
    q, k, v = (_rand((1, H, N, d), s) for s in range(3))
    aq, ak = _rand((H, R, d), 5, 0.5), _rand((H, R, d), 6, 0.5)
    b = _rand((H, R), 7)
    tau = 0.41
    O, _ = orc.forward(q, k, v, aq, ak, b, tau, m, causal=True)
    for h in range(H):
        mask = np.full((N, N), -np.inf)
        for i in range(N):
            for j in range(i + 1):
                r = int(orc.phi_of_delta(m, np.array([j - i]), N)[0])
                mask[i, j] = tau * (np.dot(q[0, h, i], aq[h, r]) + np.dot(k[0, h, j], ak[h, r]) + b[h, r])
        ref = _sdpa(q[0, h], k[0, h], v[0, h], mask, tau)
        np.testing.assert_allclose(O[0, h], ref, rtol=1e-11, atol=1e-12)


def test_bias_shift_invariance():
    B, H, N, d = 2, 2, 19, 4
    m = orc.MapDesc("t5", num_buckets=8, max_distance=16)
    R = orc.table_rows(m, N)
    q, k, v, do = (_rand((B, H, N, d), s) for s in range(4))
    b = _rand((H, R), 9)
    tau = 0.7
    r0 = orc.backward(q, k, v, do, None, None, b, tau, m)
    r1 = orc.backward(q, k, v, do, None, None, b + 3.25, tau, m)
    for n in ("o", "dq", "dk", "dv", "db"):
        np.testing.assert_allclose(r1[n], r0[n], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(r1["lse"], r0["lse"] + tau * 3.25, rtol=1e-12)


def test_constant_aq_rows_shift_rows_only():
    B, H, N, d = 1, 2, 17, 4
    m = orc.MapDesc("truncated", clip=3)
    R = orc.table_rows(m, N)
    q, k, v = (_rand((B, H, N, d), s) for s in range(3))
    w = _rand((d,), 11)
    aq = np.tile(w, (R, 1))
    tau = 0.5
    O1, L1 = orc.forward(q, k, v, aq, None, None, tau, m)
    O0, L0 = orc.forward(q, k, v, None, None, None, tau, m)
    np.testing.assert_allclose(O1, O0, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(L1, L0 + tau * (q @ w), rtol=1e-11, atol=1e-12)


def test_constant_ak_rows_equal_query_shift():
    N, d = 21, 4
    m = orc.MapDesc("log", num_buckets=8, max_distance=16)
    R = orc.table_rows(m, N)
    q, k, v = (_rand((1, 1, N, d), s) for s in range(3))
    w = _rand((d,), 12)
    ak = np.tile(w, (R, 1))
    O, _ = orc.forward(q, k, v, None, ak, None, 0.6, m)
    ref = _sdpa(q[0, 0] + w, k[0, 0], v[0, 0], None, 0.6)
    np.testing.assert_allclose(O[0, 0], ref, rtol=1e-11, atol=1e-12)


def test_fully_masked_row():
    q, k, v = (_rand((1, 1, 8, 4), s) for s in range(3))
    O, L = orc.forward(q, k, v, None, None, None, 1.0, orc.MapDesc("truncated", clip=2), key_len=[0])
    assert np.all(O == 0) and np.all(L == -np.inf)


def test_truncated_wide_clip_equals_identity_shifted():
    N, d, c = 13, 4, 20
    q, k, v, do = (_rand((1, 1, N, d), s) for s in range(4))
    aid = _rand((2 * N - 1, d), 20)
    atr = np.zeros((2 * c + 1, d))
    shift = c - (N - 1)
    atr[shift:shift + 2 * N - 1] = aid
    r_id = orc.backward(q, k, v, do, aid, aid, None, 0.5, orc.MapDesc("identity"))
    r_tr = orc.backward(q, k, v, do, atr, atr, None, 0.5, orc.MapDesc("truncated", clip=c))
    np.testing.assert_allclose(r_tr["o"], r_id["o"], rtol=1e-12)
    np.testing.assert_allclose(r_tr["daq"][shift:shift + 2 * N - 1], r_id["daq"], rtol=1e-10, atol=1e-12)
    assert np.all(r_tr["daq"][:shift] == 0)


@pytest.mark.parametrize("kind", ["t5", "log"])
def test_bucketed_equals_expanded_truncated(kind):
    """A bucketed map equals its expanded truncated form with copied rows, and the
    expanded run's table gradients, summed back into their buckets, equal the bucketed ones."""
    N, d, H = 40, 4, 2
    m = (orc.MapDesc("t5", num_buckets=8, max_distance=16) if kind == "t5"
         else orc.MapDesc("log", num_buckets=8, max_distance=16))
    R = orc.table_rows(m, N)
    q, k, v, do = (_rand((1, H, N, d), s) for s in range(4))
    aq, ak, b = _rand((R, d), 21, 0.5), _rand((R, d), 22, 0.5), _rand((H, R), 23)
    tau = 0.35
    r_b = orc.backward(q, k, v, do, aq, ak, b, tau, m)
    elo, ehi = orc.expanded_bounds(m, N)
    rowmap = orc.phi_of_delta(m, np.arange(elo, ehi + 1), N)          # expanded row -> bucket
    i = np.arange(N)
    phi_e = np.clip(i[None, :] - i[:, None], elo, ehi) - elo           # expanded truncated map
    aq_e, ak_e, b_e = aq[rowmap], ak[rowmap], b[:, rowmap]
    Re = ehi - elo + 1
    allowed = np.ones((N, N), bool)
    for h in range(H):
        g = orc.head_backward(q[0, h], k[0, h], v[0, h], do[0, h], aq_e, ak_e, b_e[h], tau, phi_e, allowed, Re)
        np.testing.assert_allclose(g["o"], r_b["o"][0, h], rtol=1e-12, atol=1e-13)
        np.testing.assert_allclose(g["dq"], r_b["dq"][0, h], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(g["dk"], r_b["dk"][0, h], rtol=1e-10, atol=1e-12)
        fold_db = np.zeros(R)
        np.add.at(fold_db, rowmap, g["db"])
        np.testing.assert_allclose(fold_db, r_b["db"][h], rtol=1e-10, atol=1e-12)
    # shared-table gradient: fold then sum heads
    fold = np.zeros((R, d))
    for h in range(H):
        g = orc.head_backward(q[0, h], k[0, h], v[0, h], do[0, h], aq_e, ak_e, b_e[h], tau, phi_e, allowed, Re)
        np.add.at(fold, rowmap, g["daq"])
    np.testing.assert_allclose(fold, r_b["daq"], rtol=1e-10, atol=1e-12)


# --------------------------------------------------------------------------
# Gradient pins
# --------------------------------------------------------------------------

def test_gradient_row_sum_invariants():
    B, H, N, d = 1, 2, 30, 4
    m = orc.MapDesc("t5", num_buckets=8, max_distance=16)
    R = orc.table_rows(m, N)
    q, k, v, do = (_rand((B, H, N, d), s) for s in range(4))
    aq, b = _rand((R, d), 31), _rand((H, R), 32)
    phi = orc.phi_matrix(m, N)
    for h in range(H):
        g = orc.head_backward(q[0, h], k[0, h], v[0, h], do[0, h], aq, None, b[h], 0.5, phi,
                              np.ones((N, N), bool), R)
        # sum_j dS_ij = 0 for every row => sum_r dZ^Q_ir = 0 and sum_r db_r = 0
        assert np.max(np.abs(g["dzq"].sum(1))) < 1e-12 * np.abs(g["dzq"]).max() * N
        assert abs(g["db"].sum()) < 1e-12 * np.abs(g["db"]).max() * R


def _fd_case(kind, causal, key_len, shared):
    N, d, H, B = 9, 3, 2, 2
    m = {"truncated": orc.MapDesc("truncated", clip=2), "identity": orc.MapDesc("identity"),
         "t5": orc.MapDesc("t5", num_buckets=8, max_distance=8), "log": orc.MapDesc("log", num_buckets=6, max_distance=8)}[kind]
    R = orc.table_rows(m, N)
    rng = np.random.default_rng(7)
    x = dict(q=rng.standard_normal((B, H, N, d)), k=rng.standard_normal((B, H, N, d)),
             v=rng.standard_normal((B, H, N, d)),
             aq=rng.standard_normal((R, d) if shared else (H, R, d)) * 0.5,
             ak=rng.standard_normal((R, d) if shared else (H, R, d)) * 0.5,
             b=rng.standard_normal((H, R)))
    do = rng.standard_normal((B, H, N, d))
    return m, x, do, 0.45


@pytest.mark.parametrize("kind,causal,key_len,shared", [
    ("truncated", False, None, True), ("identity", True, None, False),
    ("t5", False, [9, 6], True), ("log", True, [7, 9], False)])
def test_gradients_central_differences(kind, causal, key_len, shared):
    m, x, do, tau = _fd_case(kind, causal, key_len, shared)

    def loss(xx):
        O, _ = orc.forward(xx["q"], xx["k"], xx["v"], xx["aq"], xx["ak"], xx["b"], tau, m,
                           causal=causal, key_len=key_len)
        return float(np.sum(O * do))

    g = orc.backward(x["q"], x["k"], x["v"], do, x["aq"], x["ak"], x["b"], tau, m,
                     causal=causal, key_len=key_len)
    names = {"q": "dq", "k": "dk", "v": "dv", "aq": "daq", "ak": "dak", "b": "db"}
    eps = 1e-6
    rng = np.random.default_rng(3)
    for n, gn in names.items():
        flat = x[n].reshape(-1)
        idx = rng.choice(flat.size, size=min(flat.size, 40), replace=False)
        for t in idx:
            xp = {kk: vv.copy() for kk, vv in x.items()}
            xm = {kk: vv.copy() for kk, vv in x.items()}
            xp[n].reshape(-1)[t] += eps
            xm[n].reshape(-1)[t] -= eps
            fd = (loss(xp) - loss(xm)) / (2 * eps)
            an = g[gn].reshape(-1)[t]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (n, t, fd, an)


# --------------------------------------------------------------------------
# Tile plan pins
# --------------------------------------------------------------------------

@pytest.mark.parametrize("kind,N,T,causal,key_len", [
    ("truncated", 300, 32, False, None), ("truncated", 257, 64, False, [257, 100]),
    ("t5", 400, 32, False, None), ("log", 700, 64, False, [650, 700]),
    ("identity", 200, 32, True, None), ("t5", 130, 32, True, [100, 130]),
    ("truncated", 64, 64, False, None)])
def test_tile_plan_rule_matches_brute_force(kind, N, T, causal, key_len):
    m = {"truncated": orc.MapDesc("truncated", clip=16), "identity": orc.MapDesc("identity"),
         "t5": orc.MapDesc("t5", num_buckets=32, max_distance=128),
         "log": orc.MapDesc("log", num_buckets=64, max_distance=128)}[kind]
    B = 1 if key_len is None else len(key_len)
    brute = orc.tile_plan_brute(m, N, T, causal, key_len, B)
    rule, seg = orc.tile_plan_rule(m, N, T, causal, key_len, B)
    assert np.array_equal(brute, rule)
    # segments: CONST_LO run, then BAND, then CONST_HI, then MASKED tail
    for b in range(B):
        for qi in range(rule.shape[1]):
            a, bb, c, nk = seg[b, qi]
            row = rule[b, qi]
            assert np.all(row[:a] == orc.CONST_LO) and np.all(row[a:bb] == orc.BAND)
            assert np.all(row[bb:c] == orc.CONST_HI) and np.all(row[c:] == orc.MASKED)
            assert nk == rule.shape[2]


def test_group_reach_overhead_matches_pages():
    # G consecutive queries reach N + G - 1 contiguous offsets; the extra (G-1)/N at
    # N = 8192, G = 128 is the "about 1.6%" the digest quotes.
    N, G = 8192, 128
    i0 = 4096
    reach = set()
    for i in range(i0, i0 + G):
        reach.update(range(-i, N - i))
    assert len(reach) == N + G - 1
    assert abs((G - 1) / N - 0.016) < 0.001


@pytest.mark.parametrize("kind,causal,kl", [("truncated", False, None), ("identity", True, None), ("log", False, 21)])
def test_sampled_grads_equal_full_backward(kind, causal, kl):
    """The sampled evaluation used at large N equals the full-matrix backward."""
    N, d = 29, 4
    m = {"truncated": orc.MapDesc("truncated", clip=3), "identity": orc.MapDesc("identity"),
         "log": orc.MapDesc("log", num_buckets=8, max_distance=16)}[kind]
    R = orc.table_rows(m, N)
    q, k, v, do = (_rand((N, d), s) for s in range(4))
    aq, ak, b = _rand((R, d), 5, 0.5), _rand((R, d), 6, 0.5), _rand((R,), 7)
    phi = orc.phi_matrix(m, N)
    allowed = orc.allowed_matrix(N, causal, kl)
    full = orc.head_backward(q, k, v, do, aq, ak, b, 0.4, phi, allowed, R)
    rows, cols = np.array([0, 5, 28]), np.array([1, 13, 28])
    smp = orc.head_grads_sampled(q, k, v, do, aq, ak, b, 0.4, m, causal, kl, rows, cols, chunk=7)
    np.testing.assert_allclose(smp["o"], full["o"], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(smp["lse"], full["lse"], rtol=1e-12)
    np.testing.assert_allclose(smp["dq"], full["dq"][rows], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(smp["dk"], full["dk"][cols], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(smp["dv"], full["dv"][cols], rtol=1e-10, atol=1e-12)


def test_row_blocks_sum_to_full_backward():
    """The CPU-baseline unit of work (a block of query rows) sums to the full backward."""
    N, d = 31, 4
    m = orc.MapDesc("truncated", clip=4)
    R = orc.table_rows(m, N)
    q, k, v, do = (_rand((N, d), s) for s in range(4))
    aq, ak, b = _rand((R, d), 5, 0.5), _rand((R, d), 6, 0.5), _rand((R,), 7)
    phi = orc.phi_matrix(m, N)
    full = orc.head_backward(q, k, v, do, aq, ak, b, 0.3, phi, np.ones((N, N), bool), R)
    acc = {n: 0.0 for n in ("dv", "dk", "daq", "dak", "db", "dk_rel")}
    for r0 in range(0, N, 8):
        rows = np.arange(r0, min(N, r0 + 8))
        blk = orc.head_block_step(q, k, v, do, aq, ak, b, 0.3, m, False, None, rows)
        np.testing.assert_allclose(blk["dq"], full["dq"][rows], rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(blk["o"], full["o"][rows], rtol=1e-12, atol=1e-13)
        for n in acc:
            acc[n] = acc[n] + blk[n]
    np.testing.assert_allclose(acc["dv"], full["dv"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(acc["dk"] + acc["dk_rel"], full["dk"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(acc["daq"], full["daq"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(acc["dak"], full["dak"], rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(acc["db"], full["db"], rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("kind,terms,causal,kl", [
    ("identity", ("aq", "b"), True, None), ("truncated", ("aq", "ak"), False, 23),
    ("t5", ("b",), False, None), ("log", ("aq", "ak", "b"), True, 17)])
def test_row_block_table_grads_equal_full_backward(kind, terms, causal, kl):
    """The row-block sums behind the config-size table-gradient checks equal the
    full-matrix backward (itself pinned by central differences), for every term
    subset, with causal and key-padding masks."""
    N, d = 29, 4
    kw = {"truncated": dict(clip=5), "identity": {}, "t5": dict(num_buckets=8, max_distance=20, bidirectional=1),
          "log": dict(num_buckets=8, max_distance=24)}[kind]
    m = orc.MapDesc(kind, **kw)
    R = orc.table_rows(m, N)
    q, k, v, do = (_rand((N, d), s) for s in range(4))
    aq = _rand((R, d), 5, 0.5) if "aq" in terms else None
    ak = _rand((R, d), 6, 0.5) if "ak" in terms else None
    b = _rand((R,), 7) if "b" in terms else None
    phi = orc.phi_matrix(m, N)
    full = orc.head_backward(q, k, v, do, aq, ak, b, 0.3, phi, orc.allowed_matrix(N, causal, kl), R)
    got = orc.head_table_grads(q, k, v, do, aq, ak, b, 0.3, m, causal, kl, block=6)
    assert set(got) == {n for n, t in (("daq", aq), ("dak", ak), ("db", b)) if t is not None}
    for n in got:
        np.testing.assert_allclose(got[n], full[n], rtol=1e-10, atol=1e-12)
