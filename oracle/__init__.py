"""fp64 CPU oracle for the block-sparse FlashAttention forward.

Test infrastructure: only the tests, the smoke check and the benchmark's
CPU-baseline leg import this package.  It shares no code with the CUDA path.
"""
from .sbfa_oracle import *  # noqa: F401,F403
