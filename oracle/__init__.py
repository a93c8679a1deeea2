"""fp64 CPU oracles for the VSA / dense attention path and its pre-attention pass (test infrastructure only).

Only the tests, the package's smoke check and the benchmark's CPU-baseline
leg use this package; the CUDA product path never imports it.
"""
from . import prenorm_oracle, vsa_oracle  # noqa: F401
