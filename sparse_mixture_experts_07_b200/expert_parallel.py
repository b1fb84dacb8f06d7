"""Expert parallelism for the MoE block: one process per GPU, the routed
experts split across the ranks of a torch.distributed process group.

"Mixture of Experts in Transformers", section "expert parallelism":
GroupedGemmParallel gives each of N ranks E/N of the experts (a slice of dim 0
of the packed gate_up_proj and down_proj); RouterParallel maps the router's
global expert indices to the rank's local ones and masks the other ranks'
experts; an all-reduce sums the ranks' partial outputs.

Here every rank routes and plans all T tokens over all E experts (the router
weight is replicated, and moe_route / moe_permute are deterministic, so every
rank gets the same plan), runs the expert FFNs of its own contiguous range of
experts (moe_forward_experts), combines the slots of its experts into a
float32 partial (moe_combine_experts), and the partials are summed by an
all-reduce over the process group (NCCL over NVLink between GPUs) before one
rounding to the block's dtype (moe_cast_f32).  Rank 0 also runs the shared
experts.  Every compute step runs in libmoe.so; this module only splits the
work and calls the collective.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch

from . import moe


def expert_range(E: int, world: int, rank: int) -> Tuple[int, int]:
    """Contiguous experts [begin, end) of `rank`: E // world each, the first
    E % world ranks one more (GroupedGemmParallel's split of dim 0)."""
    if world <= 0 or not 0 <= rank < world or E < 0:
        raise ValueError(f"bad partition: E={E}, world={world}, rank={rank}")
    base, extra = divmod(E, world)
    begin = rank * base + min(rank, extra)
    return begin, begin + base + (1 if rank < extra else 0)


def allreduce_partial(y_partial: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the ranks' float32 partial outputs in place (the pages' all-reduce)."""
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(y_partial, op=dist.ReduceOp.SUM, group=group)
    return y_partial


class MoELayerEP:
    """One rank's share of the block under expert parallelism.

    Holds the replicated router and the weights of this rank's experts
    (`gate_up_local` [e_end - e_begin, 2I, H], `down_local` [e_end - e_begin,
    H, I]); rank 0 also holds the shared experts.  `__call__(x)` takes the same
    x [T, H] on every rank and returns the full block output y [T, H] on every
    rank."""

    def __init__(self, shape: moe.Shape, rank: int, world: int, w_router, router_bias,
                 gate_up_local, down_local, sh_gate_up=None, sh_down=None, group=None):
        self.shape, self.rank, self.world, self.group = shape, rank, world, group
        self.e_begin, self.e_end = expert_range(shape.E, world, rank)
        n_local = self.e_end - self.e_begin
        if gate_up_local is not None and gate_up_local.shape[0] != n_local:
            raise ValueError(f"rank {rank} holds experts [{self.e_begin}, {self.e_end}) but "
                             f"gate_up_local has {gate_up_local.shape[0]}")
        self.with_shared = rank == 0 and shape.n_shared > 0
        self.w_router, self.router_bias = w_router, router_bias
        self.w_split = moe.router_split(shape, w_router)
        self.gate_up, self.down = gate_up_local, down_local
        self.sh_gate_up = sh_gate_up if self.with_shared else None
        self.sh_down = sh_down if self.with_shared else None
        dev = w_router.device
        self.workspace = moe.alloc_workspace(shape, dev)
        self.err_flag = torch.zeros(1, dtype=torch.int32, device=dev)
        T, k, E, H = shape.T, shape.k, shape.E, shape.H
        self.buf = {
            "topk_idx": torch.empty(T, k, dtype=torch.int32, device=dev),
            "topk_w": torch.empty(T, k, dtype=torch.float32, device=dev),
            "counts": torch.empty(E, dtype=torch.int32, device=dev),
            "offsets": torch.empty(E + 1, dtype=torch.int32, device=dev),
            "perm": torch.empty(T * k, dtype=torch.int32, device=dev),
            "inv": torch.empty(T * k, dtype=torch.int32, device=dev),
            "y_slots": torch.empty(shape.slot_rows, H, dtype=shape.torch_dtype, device=dev),
            "y_partial": torch.empty(T, H, dtype=torch.float32, device=dev),
            "y": torch.empty(T, H, dtype=shape.torch_dtype, device=dev),
        }

    def partial(self, x, stream=None) -> torch.Tensor:
        """This rank's float32 partial output (before the all-reduce)."""
        s, b = self.shape, self.buf
        idx, w, _ = moe.route(s, x, self.w_router, self.router_bias, out=b, stream=stream,
                              err_flag=self.err_flag, w_split=self.w_split)
        moe.permute(s, idx, self.workspace, self.err_flag, out=b, stream=stream)
        moe.forward_experts(s, self.e_begin, self.e_end, x, b["offsets"], b["perm"], w,
                            self.gate_up, self.down, self.sh_gate_up, self.sh_down,
                            self.workspace, self.err_flag, b["y_slots"], stream=stream)
        return moe.combine_experts(s, self.e_begin, self.e_end, self.with_shared, b["y_slots"],
                                   b["inv"], idx, y_partial=b["y_partial"], stream=stream)

    def __call__(self, x, stream=None, y: Optional[torch.Tensor] = None) -> torch.Tensor:
        part = self.partial(x, stream=stream)
        if stream is not None:
            with torch.cuda.stream(stream):
                allreduce_partial(part, self.group)
        else:
            allreduce_partial(part, self.group)
        return moe.cast_f32(self.shape, part, y=self.buf["y"] if y is None else y, stream=stream)

    def device_error(self) -> int:
        return int(self.err_flag.item())
