"""Parity of the four mechanisms of the sequence-length sweep (Shaw clip 256,
Transformer-XL identity, DeBERTa 256 buckets / 512, T5 32 buckets / 128; fp16,
bidirectional) against the full fp64 oracle, at a full-tile length and a
ragged one, with fewer batch elements and heads than the 16K-token budget so
that the oracle stays fast."""
import pytest

from synth import SWEEP_MECHANISMS, sweep_workload
from relpos_harness import check_backward, check_forward, run_library, run_oracle

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("mech", sorted(SWEEP_MECHANISMS))
@pytest.mark.parametrize("N", [128, 300])
def test_sweep_mechanism_parity(mech, N):
    w = sweep_workload(mech, N, B=2, H=2)
    got, want = run_library(w), run_oracle(w)
    check_forward(got, want, w.name)
    check_backward(got, want, w.name)
