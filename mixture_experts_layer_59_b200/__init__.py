"""B200-native (sm_100a) token-choice MoE expert layer, forward and backward.

The compute lives in ``libmoe_b200.so`` (hand-written CUDA); ``binding``
exposes its C entry points to Python, ``layer`` strings them into one step,
and ``synth`` draws the seeded synthetic workloads.  Importing this package
does not load the library; the first binding call does, and raises if the
library has not been built.
"""
from .binding import (MOE_BF16, MOE_F32, MOE_ROUND_NEAREST, MOE_ROUND_NONE, MoEError,  # noqa: F401
                      moe_check_status, moe_combine, moe_expert_ffn_fwd, moe_layer_bwd,
                      moe_permute, moe_route, moe_row_capacity)

__all__ = ["moe_route", "moe_permute", "moe_expert_ffn_fwd", "moe_combine", "moe_layer_bwd",
           "moe_check_status", "moe_row_capacity", "MoEError"]
