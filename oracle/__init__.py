"""CPU oracle of the quantised MoE layer (test infrastructure only).

Only the test suite, the smoke check and the benchmark's CPU-baseline leg may
import this package.  The product library never does; it fails loudly when
its CUDA extension is missing instead of falling back to anything here.
"""
from .moe_oracle import *  # noqa: F401,F403
