"""B200-native (sm_100a) forward pass of a DeepSeek-V3/R1 Mixture-of-Experts block.

The block runs in four C-ABI CUDA libraries (moe_router, moe_dispatch,
moe_experts, moe_combine; headers in include/); this package is their thin
Python binding plus the seeded input generator.
"""
from .moe import (BlockParams, BlockShape, MoEBlock, combine, dispatch_build,  # noqa: F401
                  expert_weights_struct, experts_forward, router_forward, selftest_wait)
