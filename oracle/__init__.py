"""fp64 CPU oracle (test infrastructure only).

Only the tests, the package smoke check and the benchmark's CPU-baseline / reference leg
may import this package. The CUDA path never imports it and shares no code with it.
"""
from . import dkv_oracle  # noqa: F401
