"""CPU oracle for the sparse MoE FFN layer forward (TEST INFRASTRUCTURE).

A plain, slow fp64 restatement of what the layer computes, written from the
reference pages' definitions.  Only the test suite, the smoke check and the
benchmark's CPU-baseline leg may import it; the product library never does,
and the two share no code.
"""
from .moe_oracle import *  # noqa: F401,F403
