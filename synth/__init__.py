"""Seeded synthetic workloads for relative-position attention.

This package only draws random numbers and shapes them into the inputs of
one attention layer.  It holds none of the attention arithmetic: both the
CUDA library's tests/benchmarks and the CPU oracle consume what it returns.
"""
from .workloads import (CONFIGS, SWEEP_LENGTHS, SWEEP_MECHANISMS, SWEEP_TOKENS, Workload, make_workload,  # noqa: F401
                        small_workload, sweep_workload)
