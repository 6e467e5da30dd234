"""fp64 CPU oracle (test infrastructure only: imported by tests, the smoke check
and the benchmark's CPU baseline, never by the CUDA path)."""
from . import moe_oracle  # noqa: F401
