"""B200-native dropless sparse Mixture-of-Experts feed-forward block.

The kernels live in libmoe.so (CUDA for sm_100a, C ABI in include/moe.h);
`moe` is its ctypes binding and `inputs` the seeded synthetic workloads.
"""
from . import inputs  # noqa: F401
from .moe import (MOE_BF16, MOE_F32, MoEError, MoEGraph, MoELayer, Shape,  # noqa: F401
                  alloc_workspace, backward, backward_workspace_size, cast_f32, combine,
                  combine_experts, forward, forward_experts, forward_mxfp4,
                  forward_mxfp4_prepared, forward_train, mxfp4_prepare,
                  load_library, permute, route, route_noaux_tc, route_permute, router_split,
                  shared_merge, train_state_size, workspace_size)
from .expert_parallel import MoELayerEP, allreduce_partial, expert_range  # noqa: F401
