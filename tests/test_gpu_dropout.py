"""Attention dropout on the GPU against the oracle (scope-table next row f3):
the kernels draw the Philox4x32-10 mask of (seed, offset, b*H + h, i, j)
themselves, so outputs and every gradient must match the oracle's dropout
forward / backward, which draws the same mask from its own implementation of
the generator.  Also: identical results for identical (seed, offset), other
results for another offset, and the dropout rate of zero equal to no dropout."""
import numpy as np
import pytest

from synth import small_workload
from relpos_harness import check_backward, check_forward, run_library, run_oracle

pytestmark = pytest.mark.gpu

CASES = [
    dict(map_kind="truncated", clip=16, terms=("aQ", "aK"), N=200),
    dict(map_kind="t5", terms=("b",), N=300, causal=True, tau=1.0),
    dict(map_kind="log", num_buckets=32, max_distance=64, terms=("aQ", "aK"), per_head_tables=True, N=257,
         key_len=[257, 180]),
    dict(map_kind="identity", terms=("aQ", "b"), per_head_tables=True, N=150, causal=True),
    dict(map_kind="truncated", clip=8, terms=("aQ", "aK", "b"), N=129, dtype="bf16"),
]


def _wl(c):
    import torch
    c = dict(c)
    dt = torch.bfloat16 if c.pop("dtype", "fp16") == "bf16" else torch.float16
    kl = c.pop("key_len", None)
    B = 2 if kl is not None else 1
    tau = c.pop("tau", 0.125 if dt == torch.bfloat16 else 0.2)
    return small_workload(B=B, H=2, dtype=dt, key_len=kl, tau=tau, **c)


@pytest.mark.parametrize("case", range(len(CASES)))
@pytest.mark.parametrize("p", [0.125, 0.5])
def test_dropout_matches_oracle(case, p):
    w = _wl(CASES[case])
    drop = (p, 0x1F2E3D4C5B6A7988 + case, 11 * case + 3)
    bf16 = str(w.dtype).endswith("bfloat16")
    got = run_library(w, out_f32=bf16, dropout=drop)
    want = run_oracle(w, dropout=drop)
    check_forward(got, want, f"case {case} p {p}")
    check_backward(got, want, f"case {case} p {p}")


@pytest.mark.parametrize("case", [0, 4])
def test_dropout_rate_between_eighth_bit_steps(case):
    """p = 0.1 is not a multiple of 1/256: both sides mask at ceil(25.6) = 26 /
    256 and scale the kept cells by 256 / 230."""
    w = _wl(CASES[case])
    drop = (0.1, 0x0BAD_F00D + case, 17)
    bf16 = str(w.dtype).endswith("bfloat16")
    got = run_library(w, out_f32=bf16, dropout=drop)
    want = run_oracle(w, dropout=drop)
    check_forward(got, want, f"case {case} p 0.1")
    check_backward(got, want, f"case {case} p 0.1")


def test_dropout_is_deterministic_and_keyed():
    w = _wl(CASES[0])
    a = run_library(w, dropout=(0.25, 99, 5))
    b = run_library(w, dropout=(0.25, 99, 5))
    c = run_library(w, dropout=(0.25, 99, 6))
    for n in a:
        if a[n] is not None:
            assert np.array_equal(a[n], b[n]), n
    assert not np.array_equal(a["o"], c["o"])


def test_zero_rate_is_no_dropout():
    w = _wl(CASES[1])
    a = run_library(w)
    b = run_library(w, dropout=(0.0, 1234, 7))
    for n in a:
        if a[n] is not None:
            assert np.array_equal(a[n], b[n]), n
