"""fp64 CPU oracle of the Swimba layer.  TEST INFRASTRUCTURE ONLY: imported by the tests, the smoke
check and the benchmark's CPU-baseline leg, never by the library's own code path."""
from . import swimba_oracle  # noqa: F401
