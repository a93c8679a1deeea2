"""fp64 CPU oracle for the VSA / dense attention path (test infrastructure only).

Only the tests, the package's smoke check and the benchmark's CPU-baseline
leg use this package; the CUDA product path never imports it.
"""
from . import vsa_oracle  # noqa: F401
