"""Pins of the oracle's attention dropout (scope-table next row f3).

The Philox4x32-10 generator against its published known-answer vectors
(tests/golden/philox4x32_10_kat.json); the keep rate and its rounding to
multiples of 2^-8; sixteen distinct uniforms per call; the p = 0 case against
the dropout-free oracle; and the dropout backward against central finite
differences of sum(dO o O) with the mask held fixed (the mask depends only on
(seed, offset, b, h, i, j), never on the inputs)."""
import json
import os

import numpy as np
import pytest

import oracle as orc

HERE = os.path.dirname(os.path.abspath(__file__))


def test_philox_known_answer_vectors():
    with open(os.path.join(HERE, "golden", "philox4x32_10_kat.json")) as f:
        kat = json.load(f)
    for v in kat["vectors"]:
        ctr = [int(x, 16) for x in v["ctr"]]
        key = [int(x, 16) for x in v["key"]]
        out = orc.philox4x32_10(ctr, key)
        assert [int(o) for o in out] == [int(x, 16) for x in v["out"]]


def test_philox_vectorised_matches_scalar():
    rng = np.random.default_rng(0)
    ctr = rng.integers(0, 2 ** 32, size=(4, 50), dtype=np.uint64)
    key = rng.integers(0, 2 ** 32, size=(2, 50), dtype=np.uint64)
    vec = orc.philox4x32_10(list(ctr), list(key))
    for t in range(50):
        sc = orc.philox4x32_10([int(c[t]) for c in ctr], [int(k[t]) for k in key])
        assert [int(w[t]) for w in vec] == [int(x) for x in sc]


@pytest.mark.parametrize("p", [0.1, 0.5, 0.9])
def test_keep_rate(p):
    keep = orc.dropout_keep(5, np.arange(512), 512, p, seed=0x1234_5678_9ABC_DEF0, offset=77)
    n = keep.size
    q = orc.dropout_rate(p)
    assert q >= p and q - p < 2.0 ** -8
    sd = np.sqrt(q * (1 - q) / n)
    assert abs(keep.mean() - (1 - q)) < 6 * sd


def test_rate_is_rounded_up_to_eighth_bit_steps():
    """A rate between two multiples of 2^-8 masks exactly like the next one up;
    the cells a step of 2^-8 adds are those whose uniform equals the step's
    numerator, about 1 / 256 of them, and the masks are nested."""
    kw = dict(seed=0x0F0F_1234, offset=11)
    for p in (0.1, 0.3, 0.77):
        q = np.ceil(256 * p) / 256
        assert orc.dropout_rate(p) == q
        assert np.array_equal(orc.dropout_keep(1, np.arange(256), 256, p, **kw),
                              orc.dropout_keep(1, np.arange(256), 256, q, **kw))
    lo = orc.dropout_keep(1, np.arange(256), 256, 26 / 256, **kw)
    hi = orc.dropout_keep(1, np.arange(256), 256, 27 / 256, **kw)
    assert np.all(lo >= hi)                          # dropped at 26/256 => dropped at 27/256
    frac = np.mean(lo & ~hi)
    assert abs(frac - 1 / 256) < 6 * np.sqrt(1 / 256 / lo.size)
    assert orc.dropout_rate(0.0) == 0.0 and orc.dropout_rate(1.0) == 1.0
    assert orc.dropout_rate(2.0 ** -12) == 2.0 ** -8


def test_block_cells_use_distinct_uniforms():
    """Each Philox call serves 4 x 4 cells with sixteen distinct 8-bit uniforms:
    every pair of cell positions within a block agrees about half the time at
    p = 0.5 (two cells reading the same byte would always agree), and so do
    cells of neighbouring blocks along both axes."""
    keep = orc.dropout_keep(2, np.arange(512), 512, 0.5, seed=0xDEADBEEF, offset=3)
    blocks = keep.reshape(128, 4, 128, 4).transpose(0, 2, 1, 3).reshape(-1, 16)   # [block, 4 (i & 3) + (j & 3)]
    n = blocks.shape[0]
    for a in range(16):
        for b in range(a + 1, 16):
            agree = np.mean(blocks[:, a] == blocks[:, b])
            assert abs(agree - 0.5) < 6 * 0.5 / np.sqrt(n), (a, b, agree)
    agree_next = np.mean(keep[:, 3::4][:, :-1] == keep[:, 4::4])   # last key of a block vs first of the next
    assert abs(agree_next - 0.5) < 6 * 0.5 / np.sqrt(keep[:, 4::4].size)
    agree_down = np.mean(keep[3::4][:-1] == keep[4::4])             # last row of a block vs first of the next
    assert abs(agree_down - 0.5) < 6 * 0.5 / np.sqrt(keep[4::4].size)


def test_mask_is_the_published_generator_bytes():
    """Cell (i, j) of slice bh is byte j & 3 of word i & 3 of the generator's
    output for counter (j >> 2, i >> 2, bh, offset), computed here for single
    cells with the scalar generator (a transposed word / byte choice or a
    wrong counter component fails it)."""
    seed, off, bh = 0x0123_4567_89AB_CDEF, 9, 6
    keep = orc.dropout_keep(bh, np.arange(24), 24, 0.5, seed, off)
    for (i, j) in [(0, 0), (1, 2), (2, 1), (3, 3), (5, 9), (7, 4), (13, 22), (22, 13), (23, 23)]:
        w = orc.philox4x32_10([j >> 2, i >> 2, bh, off], [seed & 0xFFFFFFFF, seed >> 32])
        u = (int(w[i & 3]) >> (8 * (j & 3))) & 0xFF
        assert keep[i, j] == (u >= 128), (i, j)


def test_mask_rows_are_independent_of_the_row_subset():
    full = orc.dropout_keep(3, np.arange(40), 40, 0.3, seed=9, offset=4)
    rows = np.array([0, 7, 8, 33])
    assert np.array_equal(orc.dropout_keep(3, rows, 40, 0.3, seed=9, offset=4), full[rows])
    # another slice, seed or offset gives another mask
    assert not np.array_equal(orc.dropout_keep(4, np.arange(40), 40, 0.3, 9, 4), full)
    assert not np.array_equal(orc.dropout_keep(3, np.arange(40), 40, 0.3, 10, 4), full)
    assert not np.array_equal(orc.dropout_keep(3, np.arange(40), 40, 0.3, 9, 5), full)


def _case():
    N, d, H, B = 9, 3, 2, 2
    m = orc.MapDesc("truncated", clip=2)
    R = orc.table_rows(m, N)
    rng = np.random.default_rng(7)
    x = dict(q=rng.standard_normal((B, H, N, d)), k=rng.standard_normal((B, H, N, d)),
             v=rng.standard_normal((B, H, N, d)), aq=rng.standard_normal((R, d)) * 0.5,
             ak=rng.standard_normal((R, d)) * 0.5, b=rng.standard_normal((H, R)))
    return m, x, rng.standard_normal((B, H, N, d)), 0.45


def test_zero_rate_equals_no_dropout():
    m, x, do, tau = _case()
    a = orc.backward(x["q"], x["k"], x["v"], do, x["aq"], x["ak"], x["b"], tau, m, causal=True)
    b = orc.backward(x["q"], x["k"], x["v"], do, x["aq"], x["ak"], x["b"], tau, m, causal=True,
                     dropout_p=0.0, dropout_seed=5, dropout_offset=1)
    for n in ("o", "lse", "dq", "dk", "dv", "daq", "dak", "db"):
        assert np.array_equal(a[n], b[n])


@pytest.mark.parametrize("p,causal", [(0.3, False), (0.6, True)])
def test_dropout_gradients_central_differences(p, causal):
    m, x, do, tau = _case()
    kw = dict(causal=causal, dropout_p=p, dropout_seed=0xABCDEF0123, dropout_offset=3)

    def loss(xx):
        O, _ = orc.forward(xx["q"], xx["k"], xx["v"], xx["aq"], xx["ak"], xx["b"], tau, m, **kw)
        return float(np.sum(O * do))

    g = orc.backward(x["q"], x["k"], x["v"], do, x["aq"], x["ak"], x["b"], tau, m, **kw)
    # the forward inside backward() agrees with forward()
    O, L = orc.forward(x["q"], x["k"], x["v"], x["aq"], x["ak"], x["b"], tau, m, **kw)
    assert np.allclose(g["o"], O, rtol=0, atol=1e-13) and np.allclose(g["lse"], L, rtol=0, atol=1e-13)
    names = {"q": "dq", "k": "dk", "v": "dv", "aq": "daq", "ak": "dak", "b": "db"}
    eps = 1e-6
    rng = np.random.default_rng(3)
    for n, gn in names.items():
        flat = x[n].reshape(-1)
        for t in rng.choice(flat.size, size=min(flat.size, 30), replace=False):
            xp = {kk: vv.copy() for kk, vv in x.items()}
            xm = {kk: vv.copy() for kk, vv in x.items()}
            xp[n].reshape(-1)[t] += eps
            xm[n].reshape(-1)[t] -= eps
            fd = (loss(xp) - loss(xm)) / (2 * eps)
            an = g[gn].reshape(-1)[t]
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), (n, t, fd, an)
