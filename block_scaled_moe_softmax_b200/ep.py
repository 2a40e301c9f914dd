"""Expert and tensor parallelism over ranks: the layer's experts split into contiguous shards
(or every expert's intermediate dimension split into slices), one per rank, and the ranks'
partial outputs summed.

TokenSpeed SiTU package description, "Supported contract": every rank routes with the
global expert ids, the layer filters them to its contiguous shard of local experts (local
expert offset = rank x experts per rank) and produces a partial output, and the caller
all-reduces the partial outputs over the expert-parallel group.  On one rank the routing,
the filtering and the float32 partial output are CUDA: moe_mx_forward_shard from the whole
layer's router logits (every rank routes all tokens; ep_forward_logits), or
moe_mx_forward_routed from precomputed global ids (ep_forward).  This module adds the shard
bookkeeping and the sum over ranks (torch.distributed; NCCL on GPUs).  The result is the
float32 sum; rounding it to bf16, if wanted, is the caller's.

Tensor parallelism (the same page's TP8 configuration: all experts on every rank, each with
a slice of the intermediate dimension) needs no kernel of its own: SwiGLU acts element by
element along the intermediate index, so a rank holding gate/up rows and W2 columns of one
slice computes that slice's share of every expert's output, and the shares add up.
tp_shard_weights cuts a rank's slice out of the full weights; the rank then runs
moe_mx_forward_routed on all experts (offset 0) with inter = I / world and a float32 output,
and reduce_partials sums the ranks' outputs.
"""
from __future__ import annotations

import numpy as np
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


def ep_forward_logits(layer, x, router_logits, w1, w1_scale, w2, w2_scale, top_k: int, num_experts: int,
                      rank: int, world: int, group=None, act_dtype: int = moe_mx.MOE_MX_ACT_BF16,
                      partial_fn=None) -> torch.Tensor:
    """One expert-parallel forward routed from the whole layer's logits [T, num_experts]: this rank
    routes every token over all experts, runs the pairs of its contiguous shard
    (moe_mx_forward_shard: float32 partial output) and the partials are summed over the group.
    `layer` holds this rank's shard (its E local experts' weights in w1..w2_scale).
    partial_fn(offset, n) may replace the rank's partial computation (it must return the float32
    partial [T, H] of the shard [offset, offset + n)); by default the layer computes it.
    Returns the float32 sum of all ranks' partial outputs."""
    offset, n = shard_range(num_experts, world, rank)
    if partial_fn is None:
        if layer.E != n:
            raise ValueError(f"layer holds {layer.E} experts, rank {rank}'s shard has {n}")
        partial = layer.forward_shard(x, router_logits, w1, w1_scale, w2, w2_scale, top_k, offset, act_dtype,
                                      moe_mx.MOE_MX_OUT_F32)
    else:
        partial = partial_fn(offset, n)
    return reduce_partials(partial, group)


def tp_shard_weights(w1, w1_scale, w2, w2_scale, rank: int, world: int):
    """Rank `rank`'s slice of the intermediate dimension of every expert: w1 [E, 2I, H/2] and its
    scales keep gate rows and up rows [rank * I/world, (rank + 1) * I/world) (gate rows first,
    as the layer expects); w2 [E, H, I/2] and its scales keep the matching columns.  I / world
    must be a multiple of 128 (the layer's smallest intermediate tile).  Works on numpy arrays and
    torch tensors alike; returns contiguous copies."""
    E, two_i = w1.shape[0], w1.shape[1]
    I = two_i // 2
    if I % world or (I // world) % 128:
        raise ValueError(f"intermediate size {I} does not split into {world} slices of a multiple of 128")
    n = I // world
    lo = rank * n

    def rows(a):  # gate rows then up rows of the slice
        g, u = a[:, lo:lo + n], a[:, I + lo:I + lo + n]
        if isinstance(a, torch.Tensor):
            return torch.cat([g, u], dim=1).contiguous()
        return np.ascontiguousarray(np.concatenate([g, u], axis=1))

    def cols(a, per):  # columns of the slice along the last dim, `per` elements per stored byte
        c = a[:, :, lo // per:(lo + n) // per]
        return c.contiguous() if isinstance(c, torch.Tensor) else np.ascontiguousarray(c)

    return rows(w1), rows(w1_scale), cols(w2, 2), cols(w2_scale, 32)

