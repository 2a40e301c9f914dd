"""Expert parallelism over ranks: the layer's experts split into contiguous shards, one per
rank, and the shards' partial outputs summed.

TokenSpeed SiTU package description, "Supported contract": every rank routes with the
global expert ids, the layer filters them to its contiguous shard of local experts (local
expert offset = rank x experts per rank) and produces a partial output, and the caller
all-reduces the partial outputs over the expert-parallel group.  On one rank the filtering
and the float32 partial output are moe_mx_forward_routed (CUDA); this module adds the
shard bookkeeping and the sum over ranks (torch.distributed; NCCL on GPUs).  The result
is the float32 sum; rounding it to bf16, if wanted, is the caller's.
"""
from __future__ import annotations

import torch

from . import moe_mx


def shard_range(num_experts: int, world: int, rank: int) -> tuple[int, int]:
    """(local expert offset, local expert count) of `rank`: contiguous, equal shards."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError(f"rank {rank} outside a group of {world}")
    if num_experts % world:
        raise ValueError(f"{num_experts} experts do not split evenly over {world} ranks")
    n = num_experts // world
    return rank * n, n


def reduce_partials(partial: torch.Tensor, group=None) -> torch.Tensor:
    """Sum the ranks' float32 partial outputs [T, H] in place over `group`; returns it."""
    import torch.distributed as dist
    if partial.dtype != torch.float32:
        raise TypeError("partial outputs are summed in float32")
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(partial, op=dist.ReduceOp.SUM, group=group)
    return partial


def ep_forward(layer: moe_mx.MoeMxLayer, x, topk_ids, topk_w, w1, w1_scale, w2, w2_scale, num_experts: int,
               rank: int, world: int, group=None, act_dtype: int = moe_mx.MOE_MX_ACT_BF16) -> torch.Tensor:
    """One expert-parallel forward: `layer` holds this rank's shard (layer.E local experts, their
    weights in w1..w2_scale); topk_ids are global ids over num_experts.  Returns the float32 sum
    of all ranks' partial outputs."""
    offset, n = shard_range(num_experts, world, rank)
    if layer.E != n:
        raise ValueError(f"layer holds {layer.E} experts, rank {rank}'s shard has {n}")
    partial = layer.forward_routed(x, topk_ids, topk_w, w1, w1_scale, w2, w2_scale, offset, act_dtype,
                                   moe_mx.MOE_MX_OUT_F32)
    return reduce_partials(partial, group)
