"""CPU oracle (float64) for decode-time MLA.  TEST INFRASTRUCTURE ONLY: the
test suite, the smoke check and the benchmark's CPU-baseline leg are its only
callers; the CUDA library neither imports nor links it."""

from . import mla_oracle  # noqa: F401
