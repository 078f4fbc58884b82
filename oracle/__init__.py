"""fp64 CPU oracle for HiLS-Attention (test infrastructure only).

Only the tests, the smoke check and the benchmark's CPU-baseline leg import
this package; the CUDA library never does.
"""
from . import hils_oracle  # noqa: F401
