"""CPU oracle for the SharQ hot path -- test infrastructure only.

Only the test-suite, the smoke check and the benchmark's CPU-baseline leg may
import this package.  It never imports the CUDA package and shares no code
with it.
"""
from .oracle import *  # noqa: F401,F403
