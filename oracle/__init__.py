"""CPU oracle for the PackKV packed cache (test infrastructure only).

Only the tests, the smoke check and the benchmark's CPU-baseline leg import
this package; the CUDA library never does.
"""
from .packkv_oracle import *  # noqa: F401,F403
