"""CPU oracle for the FP8 block-scaled biased MoE layer (test infrastructure only).

Only tests/, __graft_entry__.smoke() and bench.py's CPU-baseline leg may import
this package. The CUDA library never uses it.
"""
from .fp8moe_oracle import *  # noqa: F401,F403
