"""CPU oracle for the MoE layer forward -- TEST INFRASTRUCTURE ONLY.

This package is a plain, slow restatement of what the MoE layer computes, in
numpy and fp64, written from the pages' definitions.  It exists to check the
CUDA library.  Only the test-suite, the package smoke entry point's self-check
and the benchmark's CPU-baseline leg may import or call it; the library itself
never does, and it shares no code, tables or helpers with the CUDA sources.

Parity status per function is stated in ``oracle.moe_oracle``'s header.
"""
from .moe_oracle import *  # noqa: F401,F403
