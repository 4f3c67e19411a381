"""CPU oracle for the Medusa decode-verify step.

TEST INFRASTRUCTURE: imported only by the test suite, the package smoke check
and the benchmark's CPU-baseline leg.  The product path never imports it.
"""
from . import medusa_oracle  # noqa: F401
