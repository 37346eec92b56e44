"""CPU oracle of the FP8 MoE layer forward (test infrastructure: tests, smoke check and the
benchmark's CPU-baseline leg only)."""
from .moe_oracle import *  # noqa: F401,F403
