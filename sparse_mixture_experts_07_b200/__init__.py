"""B200-native dropless sparse Mixture-of-Experts feed-forward block.

The kernels live in libmoe.so (CUDA for sm_100a, C ABI in include/moe.h);
`moe` is its ctypes binding and `inputs` the seeded synthetic workloads.
"""
from . import inputs  # noqa: F401
from .moe import (MOE_BF16, MOE_F32, MoEError, MoELayer, Shape, alloc_workspace,  # noqa: F401
                  combine, forward, forward_mxfp4, load_library, permute, route, router_split,
                  workspace_size)
