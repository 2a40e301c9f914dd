"""Seeded synthetic workloads for the fused MXFP4 routed-MoE layer.

This module only draws random inputs; it holds none of the layer's arithmetic
(no quantisation, no softmax, no matmul).  The tests, the smoke check and the
bench share it, so that the CUDA path and the CPU oracle see the same inputs.

Recipe (per workload, seed 0, fixed draw order x, logits, bias, w1, w2; each
tensor and each expert has its own generator so sizes do not shift streams):
  x      ~ N(0, 1) drawn in float32, rounded to bf16 (RNE)        [T, H]
  logits ~ N(0, 1) float32, plus a per-expert bias folded in      [T, E]
           'normal': b_e ~ N(0, 0.5)              (mildly uneven loads)
           'zipf'  : b_e = 2*ln(1/(rank_e + 1)),  rank = seeded permutation
  w1     ~ N(0, 0.02) float32 per expert                          [E, 2I, H]
           rows [0, I) are the gate projection, rows [I, 2I) the up projection
  w2     ~ N(0, 0.02) float32 per expert                          [E, H, I]
Workloads with the routing given (precomputed top-k) draw it instead of logits:
  ids    k distinct global experts per token, uniform over the E_global
         experts (the first k of a seeded random ordering)        [T, k]
  w      U(0.1, 1) per slot, divided by the token's sum           [T, k]
         (the weights a router would hand over: positive, summing to 1)
Such a workload runs one contiguous shard of E local experts, global ids
[local_offset, local_offset + E); its weights are drawn per local expert.
A workload with a shared expert draws its `shared` chunks like experts
E..E+shared-1 (the same per-expert N(0, 0.02) generators).
The float32 weights are then quantised to MXFP4 along the reduction dim by the
caller (the oracle's quantiser in tests, the library's quantiser in the bench;
the two are checked bit-exact against each other).

Weights are drawn on the device the caller names with torch's Philox-based
generator; x and logits are always drawn on the CPU.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int
    H: int
    I: int
    E: int
    top_k: int
    act: str = "bf16"          # "bf16" (w4a16) or "mxfp8" (w4a8)
    bias: str = "none"         # "none" | "normal" | "zipf"
    seed: int = 0
    description: str = ""
    routing: str = "logits"    # "logits" (router) or "given" (precomputed top-k, global ids)
    experts_global: int = 0    # given routing: experts of the whole layer (0: E)
    local_offset: int = 0      # given routing: global id of local expert 0
    shared: int = 0            # shared-expert chunks of I, held as weight slots E..E+shared-1

    @property
    def slots(self) -> int:
        """Expert weight slots: the routed experts, then the shared expert's chunks."""
        return self.E + self.shared

    @property
    def pairs(self) -> int:
        return self.T * self.top_k

    def with_tokens(self, T: int) -> "Workload":
        return dataclasses.replace(self, T=T, name=f"{self.name}[T={T}]")


WORKLOADS = {
    "tiny": Workload("tiny", 16, 256, 128, 8, 2, "bf16", "none", 0,
                     "tiny MoE, w4a16: T=16 H=256 I=128 E=8 top-2"),
    "decode": Workload("decode", 16, 7168, 2048, 384, 8, "bf16", "none", 0,
                       "decode-shaped, w4a16: T=16 H=7168 I=2048 E=384 top-8"),
    "batched_decode": Workload("batched_decode", 256, 7168, 2048, 384, 8, "bf16", "normal", 0,
                               "batched decode, w4a16: T=256, logits + N(0,0.5) expert bias"),
    "prefill": Workload("prefill", 8192, 7168, 2048, 384, 8, "bf16", "zipf", 0,
                        "prefill, w4a16: T=8192, Zipf-like expert bias"),
    # the decode shape at 1 and 4 tokens (the small-batch end of decode)
    "decode_t1": Workload("decode_t1", 1, 7168, 2048, 384, 8, "bf16", "none", 0,
                          "decode-shaped, w4a16, a single token"),
    "decode_t4": Workload("decode_t4", 4, 7168, 2048, 384, 8, "bf16", "none", 0,
                          "decode-shaped, w4a16, 4 tokens"),
    # the decode routing (16 tokens, 384 experts, top-8) with small expert matrices: a profiling case
    # for the routing and grouping kernel
    "route_e384": Workload("route_e384", 16, 256, 128, 384, 8, "bf16", "none", 0,
                           "decode routing shape with small experts (profiling case)"),
    "decode_t2": Workload("decode_t2", 2, 7168, 2048, 384, 8, "bf16", "none", 0,
                          "decode-shaped, w4a16, 2 tokens"),
    # one decode token over 64 experts: a capture-sized case (about 1.5 GB of weights) with the GEMM
    # work of the single-token decode (8 experts hit), for profiling
    "decode_t1_e64": Workload("decode_t1_e64", 1, 7168, 2048, 64, 8, "bf16", "none", 0,
                              "decode-shaped, w4a16, a single token, 64 experts (profiling case)"),
    # the decode shape with 64 experts: a capture-sized case (about 1.5 GB of weights) for profiling
    "decode_e64": Workload("decode_e64", 16, 7168, 2048, 64, 8, "bf16", "none", 0,
                           "decode-shaped, w4a16, 64 experts (profiling case)"),
    # the batched-decode routing mix (about 8 pairs per hit expert, some experts over 16 rows) with
    # 64 experts and 64 tokens: a capture-sized case (about 1.5 GB of weights) for profiling
    "batched_decode_e64": Workload("batched_decode_e64", 64, 7168, 2048, 64, 8, "bf16", "normal", 0,
                                   "batched-decode-shaped, w4a16, 64 tokens, 64 experts (profiling case)"),
    # a prefill shape with 64 experts and 2048 tokens: a capture-sized case for profiling
    "prefill_e64": Workload("prefill_e64", 2048, 7168, 2048, 64, 8, "bf16", "none", 0,
                            "prefill-shaped, w4a16, 64 experts, 2048 tokens (profiling case)"),
    "prefill_w4a8": Workload("prefill_w4a8", 16384, 4096, 1536, 128, 8, "mxfp8", "none", 0,
                             "prefill, w4a8: T=16384 H=4096 I=1536 E=128 top-8"),
    # the w4a8 prefill shape with 4096 tokens: a capture-sized case (about 2.5 GB on the device)
    "prefill_w4a8_t4k": Workload("prefill_w4a8_t4k", 4096, 4096, 1536, 128, 8, "mxfp8", "none", 0,
                                 "prefill-shaped, w4a8, 4096 tokens (profiling case)"),
    # the decode shape with a shared expert of intermediate size I added to every token
    "decode_shared": Workload("decode_shared", 16, 7168, 2048, 384, 8, "bf16", "none", 0,
                              "decode-shaped, w4a16, plus one shared expert (I = 2048)", shared=1),
    # the hidden size, expert count and top-k of the TokenSpeed SiTU bundle's supported contract, with the
    # routing given as precomputed top-k: TP8 (all 896 experts, intermediate shard 384) and the
    # first EP8 shard (112 local experts of 896, intermediate 3072); 128 tokens
    "situ_tp8": Workload("situ_tp8", 128, 3584, 384, 896, 16, "bf16", "none", 0,
                         "routed MoE, TP8 shard: T=128 H=3584 I=384 E=896 top-16, precomputed top-k",
                         "given", 896, 0),
    "situ_ep8": Workload("situ_ep8", 128, 3584, 3072, 112, 16, "bf16", "none", 0,
                         "routed MoE, EP8 shard 0: T=128 H=3584 I=3072, 112 of 896 experts, top-16, precomputed top-k",
                         "given", 896, 0),
}

_STREAM = {"x": 1, "logits": 2, "bias": 3, "w1": 4, "w2": 5, "topk": 6}


def _gen(wl: Workload, stream: str, index: int = 0, device: str = "cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed((wl.seed * 1_000_003 + _STREAM[stream] * 100_003 + index) & 0x7FFF_FFFF_FFFF_FFFF)
    return g


def draw_x(wl: Workload) -> torch.Tensor:
    """bf16 [T, H] on the CPU."""
    g = _gen(wl, "x")
    return torch.randn(wl.T, wl.H, generator=g, dtype=torch.float32).to(torch.bfloat16)


def draw_bias(wl: Workload) -> torch.Tensor:
    """float32 [E] per-expert logit bias (zeros for 'none')."""
    g = _gen(wl, "bias")
    if wl.bias == "none":
        return torch.zeros(wl.E, dtype=torch.float32)
    if wl.bias == "normal":
        return torch.randn(wl.E, generator=g, dtype=torch.float32) * 0.5
    if wl.bias == "zipf":
        rank = torch.randperm(wl.E, generator=g)
        return torch.tensor([2.0 * math.log(1.0 / (int(r) + 1)) for r in rank], dtype=torch.float32)
    raise ValueError(f"unknown bias kind {wl.bias!r}")


def draw_logits(wl: Workload) -> torch.Tensor:
    """float32 [T, E] on the CPU, the expert bias already folded in."""
    g = _gen(wl, "logits")
    base = torch.randn(wl.T, wl.E, generator=g, dtype=torch.float32)
    return (base + draw_bias(wl)[None, :]).contiguous()


def draw_topk(wl: Workload):
    """Given routing: (global ids int32 [T, k], weights float32 [T, k]) on the CPU."""
    g = _gen(wl, "topk")
    eg = wl.experts_global or wl.E
    keys = torch.rand(wl.T, eg, generator=g)
    ids = torch.argsort(keys, dim=1)[:, : wl.top_k].to(torch.int32).contiguous()
    u = torch.rand(wl.T, wl.top_k, generator=g) * 0.9 + 0.1
    return ids, (u / u.sum(dim=1, keepdim=True)).to(torch.float32).contiguous()


def draw_w1_expert(wl: Workload, e: int, device: str = "cpu") -> torch.Tensor:
    """float32 [2I, H] for expert e (gate rows then up rows)."""
    g = _gen(wl, "w1", e, device)
    return torch.randn(2 * wl.I, wl.H, generator=g, dtype=torch.float32, device=device) * 0.02


def draw_w2_expert(wl: Workload, e: int, device: str = "cpu") -> torch.Tensor:
    """float32 [H, I] for expert e."""
    g = _gen(wl, "w2", e, device)
    return torch.randn(wl.H, wl.I, generator=g, dtype=torch.float32, device=device) * 0.02


def bf16_bits(t: torch.Tensor):
    """The uint16 bit patterns (numpy) of a bf16 tensor."""
    import numpy as np
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
