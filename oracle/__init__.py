"""CPU oracle for the sparse MoE layer forward (test infrastructure only).

Only the tests, the smoke check and the benchmark's CPU-baseline leg may
import this package; the product path never does.  See ``moe_oracle``.
"""
from .moe_oracle import *  # noqa: F401,F403
