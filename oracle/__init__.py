"""fp64 CPU oracle for shifted sparse attention (test infrastructure only).

Only the test suite, the package smoke check and the benchmark's CPU-baseline
leg import this package.  It shares no code with the CUDA path.
"""
from .s2_ref import *  # noqa: F401,F403
