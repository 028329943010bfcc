"""CPU fp64 oracle for exact relative-position attention.

TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the benchmark's
CPU-baseline arm may import this package; the library never does, and the
library's CUDA path shares no code with it.
"""
from .relpos import *  # noqa: F401,F403
