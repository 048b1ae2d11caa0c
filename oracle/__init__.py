"""FP64 CPU oracle for the DSA hot path (test infrastructure only).

Only the tests, the package smoke check and the benchmark's CPU-baseline /
reference arm import this package.  It shares no code with the CUDA path.
"""
from .dsa_oracle import *  # noqa: F401,F403
