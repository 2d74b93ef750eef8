"""Float64 CPU oracle for the ReHyAt hybrid attention forward.

Test infrastructure: only the tests, the smoke check and the benchmark's CPU-baseline leg use it.
"""
from .rehyat_oracle import *  # noqa: F401,F403
