#!/usr/bin/env python
"""Benchmark of the fused MXFP4 routed-MoE layer on B200; prints ONE JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--parallel replicas|ep] [--no-cpu-baseline]
                    (K defaults to 1000, or 200 for the reference arm)

Default run: the decode-shaped layer is the headline (w4a16, T=16 tokens,
H=7168, I=2048, E=384 experts, top-8), and all five configurations of the layer
are measured in the same run under "per_config": tiny (T=16, H=256, I=128,
E=8, top-2), decode, batched decode (T=256, logits + a N(0, 0.5) expert bias),
prefill (T=8192, Zipf-like expert bias) and prefill w4a8 (T=16384, H=4096,
I=1536, E=128), and the small-batch decode shapes (1 and 4 tokens).  --workload NAME measures one workload alone (also the
small-batch decode shapes decode_t1 / decode_t4, the shared-expert decode, and
shards of the 896-expert, top-16 layer with the routing given as precomputed
top-k: situ_tp8, situ_ep8).  Inputs are synthetic and seeded (bf16 x ~ N(0,1),
float32 logits ~ N(0,1) plus the workload's bias, weights N(0, 0.02) quantised
to MXFP4 on the GPU by the library's quantiser).  One step = one whole forward
(routing, grouping, FC1 + SwiGLU, FC2, combine) through the C ABI, inputs
resident in HBM.  The decode weights (8.98 GB) are far larger than L2, and L2 is
additionally flushed (512 MiB write) before every timed step; each step is
timed with CUDA events on the launching stream.

--impl ours (default): the CUDA path.  Reported per workload: tokens/s, the same
metric end to end with host buffers (e2e: pinned H2D of x and the routing
input, forward, D2H of the output, all inside the timed step), the roofline of
the dominant kernel (the FC1 grouped GEMM) and of the whole step, the per-stage
times, the clocks sampled during the timed region and the library's own count
of kernel launches in it.  The headline also carries the CPU oracle timed on a
bounded sample on all host cores (cpu_baseline).  FC1's bound is whichever of
its two costs is larger at the measured peaks: bytes (FP4 codes + E8M0 scales of
the hit experts' W1 + activation rows read + h rows written) against the HBM
copy bandwidth -- the decode shapes -- or FLOPs (2 * pairs * 2I * H) against the
sustained bf16 GEMM rate (x2 for w4a8's MXFP8 operands) -- the prefill shapes;
achieved = that work / FC1's mean CUDA-event duration.  The timed steps carry no
events between kernels (each kernel after the router may launch while the one
before it still runs); FC1's own duration comes from a second pass of the same
steps (at most 300) with events between the kernels, which the library then
launches one after another.

--impl reference: the CPU oracle (the only reference this path has), timed on
the host cores on a bounded sample of the same workload per step.

Multi-GPU (torchrun, one process per GPU).  --parallel replicas (default):
every rank runs an independent replica of the workload, timed between
barriers; value = tokens of all ranks / max-over-ranks time ("scaling": weak).
--parallel ep: expert parallelism -- each rank holds a contiguous shard of the
experts, routes all tokens of the one batch and runs the pairs of its shard
(moe_mx_forward_shard, float32 partial output), and the partials are summed
over the ranks by an NCCL all-reduce inside the step; value = the batch's
tokens / max-over-ranks time ("scaling": strong).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from block_scaled_moe_softmax_b200 import moe_mx, workloads  # noqa: E402

METRIC = "MoE layer tokens/s; % of HBM roofline (decode) / MMA peak (prefill)"
FLUSH_BYTES = 512 << 20
def log(*a):
    print(*a, file=sys.stderr, flush=True)


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return (d.get("hbm_gbs", 6650.0), d.get("bf16_tflops", 1590.0),
                d.get("bf16_tflops_sustained", d.get("bf16_tflops", 1400.0)), "measured")
    return 6650.0, 1590.0, 1400.0, "fallback"


def workload_desc(wl):
    if wl.routing == "given":
        route = (f"precomputed top-k over {wl.experts_global or wl.E} experts, local shard "
                 f"[{wl.local_offset}, {wl.local_offset + wl.E})")
    else:
        route = f"logit bias {wl.bias}"
    if wl.shared:
        route += f", plus a shared expert of intermediate {wl.shared * wl.I}"
    return (f"{wl.name}: T={wl.T} H={wl.H} I={wl.I} E={wl.E} top-{wl.top_k} "
            f"{'w4a8' if wl.act == 'mxfp8' else 'w4a16'}, {route}")


# ------------------------------------------------------------------ inputs
def make_gpu_weights(wl, dev, experts=None):
    """Draw float32 weights per expert (and shared-expert chunk) on the GPU and quantise them with
    the library's MX quantiser; `experts` (a range of global ids) keeps only those slots."""
    experts = range(wl.slots) if experts is None else experts
    E, H, I = len(experts), wl.H, wl.I
    w1 = torch.empty(E, 2 * I, H // 2, dtype=torch.uint8, device=dev)
    w1s = torch.empty(E, 2 * I, H // 32, dtype=torch.uint8, device=dev)
    w2 = torch.empty(E, H, I // 2, dtype=torch.uint8, device=dev)
    w2s = torch.empty(E, H, I // 32, dtype=torch.uint8, device=dev)
    for i, e in enumerate(experts):
        f1 = workloads.draw_w1_expert(wl, e, device=str(dev))
        moe_mx.moe_mx_quantize(f1, 2 * I, H, moe_mx.MOE_MX_FMT_MXFP4, w1[i], w1s[i])
        f2 = workloads.draw_w2_expert(wl, e, device=str(dev))
        moe_mx.moe_mx_quantize(f2, H, I, moe_mx.MOE_MX_FMT_MXFP4, w2[i], w2s[i])
    torch.cuda.synchronize(dev)
    return w1, w1s, w2, w2s


def oracle_weights_for(wl, experts, dev):
    """Oracle-quantised weights (host, numpy) for the given experts; other experts stay zero."""
    import oracle
    E, H, I = wl.slots, wl.H, wl.I
    w1 = np.zeros((E, 2 * I, H // 2), np.uint8)
    w1s = np.zeros((E, 2 * I, H // 32), np.uint8)
    w2 = np.zeros((E, H, I // 2), np.uint8)
    w2s = np.zeros((E, H, I // 32), np.uint8)
    for e in experts:
        w1[e], w1s[e] = oracle.mx_quantize(workloads.draw_w1_expert(wl, e, device=dev).cpu().numpy(),
                                           oracle.FMT_E2M1)
        w2[e], w2s[e] = oracle.mx_quantize(workloads.draw_w2_expert(wl, e, device=dev).cpu().numpy(),
                                           oracle.FMT_E2M1)
    return w1, w1s, w2, w2s


# ------------------------------------------------------------------ clocks
class ClockSampler:
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, dev_index):
        try:
            props = torch.cuda.get_device_properties(dev_index)
            self.bus = f"{props.pci_domain_id:08X}:{props.pci_bus_id:02X}:{props.pci_device_id:02X}.0"
        except (AttributeError, RuntimeError):
            self.bus = str(dev_index)
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self.bus, f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        time.sleep(0.2)
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                smax = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------------ distributed plumbing
def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, world):
    if world == 1:
        return v
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([v], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ CPU oracle timing
def reference_pairs(wl, sample_tokens):
    """The (token, slot) pairs of the sampled tokens that the layer evaluates -- the routed slots
    (the oracle's router, or the given routing restricted to the local shard) and the shared
    expert's slots -- as (token, local expert, weight); and the pairs per token of the whole
    workload, to convert pairs/s to tokens/s."""
    import oracle
    if wl.routing == "given":
        ids, w = (a.numpy() for a in workloads.draw_topk(wl))
        loc = ids - wl.local_offset
        inside = (loc >= 0) & (loc < wl.E)
        per_token = float(inside.sum()) / wl.T
    else:
        ids, w = oracle.route(workloads.draw_logits(wl).numpy()[sample_tokens], wl.top_k)
        loc, inside = ids, np.ones(ids.shape, bool)
        per_token = float(wl.top_k)
    pairs = []
    for i, t in enumerate(sample_tokens):
        row = t if wl.routing == "given" else i
        pairs += [(t, int(loc[row, j]), float(w[row, j])) for j in range(wl.top_k) if inside[row, j]]
        pairs += [(t, wl.E + c, 1.0) for c in range(wl.shared)]
    return pairs, per_token + wl.shared


class PairSampler:
    """The oracle on (token, slot) pairs of a workload: one pair = one token's FC1, SwiGLU and FC2
    through one expert, weighted -- the unit of the layer's work (a decode token is k of them).
    The pairs are those of the given sample tokens (their routing taken once, here, outside any
    timed region); batches of up to `threads` pairs run concurrently, one thread each, through the
    oracle's routed form with one slot per evaluated row."""

    def __init__(self, wl, sample_tokens, threads):
        self.wl, self.threads = wl, threads
        self.pairs, self.per_token = reference_pairs(wl, sample_tokens)
        self.experts = sorted({e for _, e, _ in self.pairs})
        dev = "cuda" if torch.cuda.is_available() else "cpu"
        self.wq = oracle_weights_for(wl, [e for e in self.experts if e < wl.E] + list(range(wl.E, wl.slots)), dev)
        self.xb = workloads.bf16_bits(workloads.draw_x(wl))
        self.act = 1 if wl.act == "mxfp8" else 0
        self.done = 0

    def run(self, n):
        """Evaluate the next n pairs (cycling); returns the wall seconds of the oracle calls."""
        import oracle
        wall = 0.0
        end = self.done + n
        while self.done < end:
            batch = min(self.threads, end - self.done)
            sel = [self.pairs[(self.done + i) % len(self.pairs)] for i in range(batch)]
            xs = np.ascontiguousarray(self.xb[[t for t, _, _ in sel]])
            ids = np.array([[e] for _, e, _ in sel], np.int32)
            ws = np.array([[w] for _, _, w in sel], np.float32)
            t0 = time.perf_counter()
            oracle.moe_forward_routed(xs, ids, ws, 0, *self.wq, self.act, nthreads=batch)
            wall += time.perf_counter() - t0
            self.done += batch
        return wall


def cpu_baseline(wl, cores, min_wall=3.0):
    """The oracle on a bounded sample of the workload, on all the host's cores: batches of one
    (token, slot) pair per core, one thread each, until at least min_wall seconds of oracle time;
    tokens/s = pairs/s / pairs per token."""
    n_tok = min(wl.T, max(1, -(-cores // max(1, wl.top_k))))
    ps = PairSampler(wl, list(range(n_tok)), cores)
    wall, pairs = 0.0, 0
    while wall < min_wall:
        wall += ps.run(cores)
        pairs += cores
    return {"value": pairs / wall / ps.per_token, "unit": "tokens/s", "cores": cores, "threads": cores,
            "kind": "oracle",
            "sample": f"{pairs} (token, slot) pairs of the {wl.name} workload (the {len(ps.pairs)} pairs of tokens "
                      f"0..{n_tok - 1} cycled, {len(ps.experts)} experts), {cores} at a time, one thread per core "
                      f"on {cores} cores, {wall:.1f} s of oracle wall time; {ps.per_token:g} pairs per token"}


def run_reference(args, wl):
    """The oracle as the reference arm.  One step = one (token, slot) pair of the workload (see
    PairSampler), small enough that K steps take a few minutes.  The pairs come from the first
    `cores` tokens and run up to `cores` at a time, one thread each.
    tokens/s = pairs/s / pairs per token."""
    cores = len(os.sched_getaffinity(0))
    sample = list(range(min(wl.T, cores)))
    ps = PairSampler(wl, sample, cores)
    ps.run(args.warmup)
    total = ps.run(args.steps)
    value = args.steps / total / ps.per_token
    used = min(cores, args.steps)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": 0,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1000 * total / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic",
        "config": {"workload": workload_desc(wl), "pairs_per_step": 1, "pairs_per_token": ps.per_token},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": used, "threads": used, "kind": "oracle",
                         "sample": f"one (token, slot) pair of {wl.name} per step: the {len(ps.pairs)} pairs of "
                                   f"tokens 0..{len(sample) - 1} cycled ({len(ps.experts)} experts), up to {cores} "
                                   f"steps concurrently on {cores} cores; {ps.per_token:g} pairs per token"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ the CUDA path
def fc1_algorithmic_flops(wl, counts):
    """2 * pairs * 2I * H: the multiply-adds of the gate and up projections of every routed pair."""
    return 2.0 * int(counts.sum()) * 2 * wl.I * wl.H


def fc1_algorithmic_bytes(wl, counts):
    hit = int((counts > 0).sum())
    P = int(counts.sum())
    w = hit * (2 * wl.I * wl.H // 2 + 2 * wl.I * wl.H // 32)
    return w + P * wl.H * 2 + P * wl.I * 2, hit


def fc2_algorithmic_bytes(wl, counts):
    """FC2's bytes: the hit experts' W2 codes and scales, h rows read (bf16-equivalent) and the
    float32 Y rows written."""
    hit = int((counts > 0).sum())
    P = int(counts.sum())
    return hit * (wl.I * wl.H // 2 + wl.I * wl.H // 32) + P * wl.I * 2 + P * wl.H * 4


def one_launch_gemms(stage):
    """True when the forward ran FC1 and FC2 as one launch (two phases): its FC1 stage then
    holds both GEMMs, and the FC2 stage no kernel, only the gap between two events (a few
    microseconds), while a separate FC2 launch takes a large share of FC1's time."""
    return stage["fc2"] < 0.2 * stage["fc1"]


def layer_weight_bytes(wl, hit):
    return hit * (3 * wl.I * wl.H // 2 + 3 * wl.I * wl.H // 32)


# the sources the FC GEMM kernel is built from (the kernel the traffic record describes)
FC_GEMM_SOURCES = ("fc_gemm.cu", "kernels.cuh", "ptx.cuh")


def _code_only(text: str) -> str:
    """C/CUDA source with its comments removed and whitespace collapsed: what the compiler sees
    of it, so that an edit of a comment does not count as a change of the kernel."""
    import re
    text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
    text = re.sub(r"//[^\n]*", " ", text)
    return " ".join(text.split())


def kernel_source_sha(read=None):
    """sha256 (first 16 hex digits) over the FC GEMM kernel's CUDA sources, in name order, code
    only (comments and whitespace stripped).  read(name) returns a source's text (default: the
    working tree)."""
    csrc = os.path.join(ROOT, "block_scaled_moe_softmax_b200", "csrc")
    if read is None:
        def read(name):
            with open(os.path.join(csrc, name)) as f:
                return f.read()
    h = hashlib.sha256()
    for name in sorted(FC_GEMM_SOURCES):
        h.update(name.encode() + b"\0" + _code_only(read(name)).encode())
    return h.hexdigest()[:16]


def traffic_record(wl, fc1_bytes):
    """DRAM bytes of one FC1 launch from the committed ncu capture, if the kernel source is unchanged.

    A capture of the workload itself is used as is.  A capture of a smaller case of the
    same weight-streaming regime (listed under "scales_to") is scaled by the ratio of
    algorithmic bytes, since there the traffic grows with the experts hit.  Otherwise None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    if rec.get("kernel_sha") != kernel_source_sha():
        return None
    for cap in rec.get("fc1_captures", []):
        dram = cap["dram_bytes_read"] + cap["dram_bytes_write"]
        if cap["workload"] == wl.name:
            return dram
        if wl.name in cap.get("scales_to", []):
            return dram * fc1_bytes / cap["algorithmic_bytes"]
    return None


class WeightCache:
    """One resident weight set at a time: the decode, batched-decode and prefill workloads share
    theirs (same H, I, E, seed), so the default run draws and quantises it once."""

    def __init__(self, dev, experts_of=None):
        self.dev, self.key, self.w = dev, None, None
        self.experts_of = experts_of  # workload -> the range of experts this rank holds (None: all)

    def get(self, wl):
        experts = self.experts_of(wl) if self.experts_of else None
        key = (wl.H, wl.I, wl.E, wl.shared, wl.seed, None if experts is None else (experts.start, experts.stop))
        if key != self.key:
            self.w = None
            torch.cuda.empty_cache()
            log(f"generating weights for {workload_desc(wl)}")
            self.w = make_gpu_weights(wl, self.dev, experts)
            self.key = key
        return self.w


def measure(args, wl, weights, world, rank, with_e2e=True):
    """Time one workload: K steps device-resident (the value), then the same steps with events
    between the kernels (each kernel's own duration), then K steps end to end from pinned host
    buffers.  Returns the workload's record (rank 0's view of the max-over-ranks times).
    With --parallel ep each rank holds a contiguous shard of the experts; a step is every rank's
    forward over its shard routed from all tokens' logits (moe_mx_forward_shard, float32 partial
    output) and the sum of the partials over the ranks (NCCL all-reduce)."""
    dev = torch.device("cuda", torch.cuda.current_device())
    hbm_peak, bf16_peak, bf16_sustained, peak_src = measured_peaks()
    act = moe_mx.MOE_MX_ACT_MXFP8 if wl.act == "mxfp8" else moe_mx.MOE_MX_ACT_BF16
    w1, w1s_rm, w2, w2s_rm = weights
    x = workloads.draw_x(wl).to(dev)
    given = wl.routing == "given"
    ep_mode = args.parallel == "ep"
    if ep_mode and (given or wl.shared):
        raise SystemExit(f"--parallel ep runs the logits form without a shared expert; {wl.name} is not one")
    # the routing input: router logits, or the given top-k (global ids and weights)
    route_host = workloads.draw_topk(wl) if given else (workloads.draw_logits(wl),)
    route_in = tuple(a.to(dev) for a in route_host)
    E_local, offset = wl.E, 0
    if ep_mode:
        from block_scaled_moe_softmax_b200 import ep
        offset, E_local = ep.shard_range(wl.E, world, rank)
    out = torch.empty(wl.T, wl.H, dtype=torch.float32 if ep_mode else torch.bfloat16, device=dev)
    layer = moe_mx.MoeMxLayer(wl.H, wl.I, E_local, wl.T, wl.top_k, device=dev.index, num_shared=wl.shared)
    # weight preparation, once, like the quantisation: the E8M0 scales in the tiled layout
    w1s, w2s = layer.prepare_scales(w1s_rm, w2s_rm)
    torch.cuda.synchronize()
    flush = torch.empty(FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream()

    def forward(xin, rin):
        if ep_mode:
            moe_mx.moe_mx_forward_shard(layer.handle, xin, rin[0], wl.T, wl.E, offset, w1, w1s, w2, w2s, wl.top_k,
                                        act, out, moe_mx.MOE_MX_OUT_F32, stream)
            ep.reduce_partials(out)
        elif given:
            moe_mx.moe_mx_forward_routed(layer.handle, xin, rin[0], rin[1], wl.T, wl.top_k, wl.local_offset, w1, w1s,
                                         w2, w2s, act, out, moe_mx.MOE_MX_OUT_BF16, stream)
        else:
            moe_mx.moe_mx_forward(layer.handle, xin, rin[0], wl.T, w1, w1s, w2, w2s, wl.top_k, act, out, stream)

    for _ in range(args.warmup):
        flush.zero_()
        forward(x, route_in)
    torch.cuda.synchronize()
    status = layer.sync_status()
    assert status == moe_mx.MOE_MX_OK, moe_mx.moe_mx_last_error()
    _, _, counts, _, _ = layer.routing(wl.T, wl.top_k)
    counts = counts.cpu().numpy()
    fc1_bytes, hit = fc1_algorithmic_bytes(wl, counts)
    fc1_flops = fc1_algorithmic_flops(wl, counts)

    # ---------------- timed region (device-resident inputs)
    sampler = ClockSampler(dev.index) if rank == 0 else None
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    if sampler:
        sampler.start()
    launches0 = moe_mx.moe_mx_launch_count(layer.handle)
    for i in range(args.steps):
        flush.zero_()
        evs[i][0].record(stream)
        forward(x, route_in)
        evs[i][1].record(stream)
    launches = moe_mx.moe_mx_launch_count(layer.handle) - launches0
    torch.cuda.synchronize()
    barrier(world)
    clocks = sampler.stop() if sampler else None
    step_ms = [a.elapsed_time(b) for a, b in evs]
    assert layer.sync_status() == moe_mx.MOE_MX_OK, moe_mx.moe_mx_last_error()
    ms_all = max_over_ranks(statistics.mean(step_ms), world)
    # replicas: every rank its own batch; expert parallelism: one batch over all ranks
    batch_tokens = wl.T if ep_mode else world * wl.T
    value = batch_tokens / (ms_all / 1000.0)

    # ---------------- per-kernel times: the same steps with CUDA events between the kernels.
    # (In the timed steps above each kernel may launch while the one before it still runs, and
    # the FC GEMMs start streaming weights early; with events between them the library
    # launches them one after another, so each kernel's own duration is measured here.)
    stage_steps = min(args.steps, 300)
    moe_mx.moe_mx_set_stage_timing(layer.handle, True)
    for i in range(stage_steps):
        flush.zero_()
        forward(x, route_in)
    stage = moe_mx.moe_mx_get_stage_times(layer.handle)
    moe_mx.moe_mx_set_stage_timing(layer.handle, False)
    assert layer.sync_status() == moe_mx.MOE_MX_OK, moe_mx.moe_mx_last_error()

    # ---------------- end to end through the public API with host buffers
    e2e = None
    if with_e2e:
        x_h = workloads.draw_x(wl).pin_memory()
        r_h = tuple(a.pin_memory() for a in route_host)
        o_h = torch.empty(wl.T, wl.H, dtype=out.dtype).pin_memory()
        x_d = torch.empty_like(x)
        r_d = tuple(torch.empty_like(a) for a in route_in)
        e2e_steps = max(3, min(args.steps, 200))
        e2e_evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(e2e_steps)]
        barrier(world)
        torch.cuda.synchronize()
        for i in range(e2e_steps):
            flush.zero_()
            e2e_evs[i][0].record(stream)
            x_d.copy_(x_h, non_blocking=True)
            for dst, src in zip(r_d, r_h):
                dst.copy_(src, non_blocking=True)
            forward(x_d, r_d)
            o_h.copy_(out, non_blocking=True)
            e2e_evs[i][1].record(stream)
        torch.cuda.synchronize()
        barrier(world)
        e2e_ms = max_over_ranks(statistics.mean(a.elapsed_time(b) for a, b in e2e_evs), world)
        assert torch.equal(o_h, out.cpu()) if ep_mode else torch.equal(o_h.view(torch.int16),
                                                                       out.cpu().view(torch.int16))
        e2e = {"value": batch_tokens / (e2e_ms / 1000.0), "unit": "tokens/s",
               "h2d_bytes_per_step": wl.T * wl.H * 2 + sum(a.numel() * a.element_size() for a in route_host),
               "d2h_bytes_per_step": wl.T * wl.H * out.element_size()}

    fc1_ms = stage["fc1"]
    kernel_name = "fc_gemm_kernel (FC1 + SwiGLU)"
    if one_launch_gemms(stage):
        # at the smallest batches the library runs FC1 and FC2 as one launch (two phases): the
        # roofline kernel is that launch, with both GEMMs' work
        kernel_name = "fc_gemm_kernel (FC1 + SwiGLU, then FC2, one launch)"
        fc1_bytes += fc2_algorithmic_bytes(wl, counts)
        fc1_flops *= 1.5
    layer_bytes = layer_weight_bytes(wl, hit)
    # FC1 is bound by whichever of its weight stream and its MMA work takes longer at the
    # measured peaks.  The tensor peak is the bf16 one (the w4a16 path's two-term MXFP8
    # expansion costs what one bf16 MMA costs); w4a8's single MXFP8 term runs at twice it.
    # The sustained figure applies: the kernel is timed inside seconds of back-to-back steps.
    mma_peak = bf16_sustained * (2.0 if wl.act == "mxfp8" else 1.0)
    traffic = traffic_record(wl, fc1_bytes)
    if fc1_flops / (mma_peak * 1e12) > fc1_bytes / (hbm_peak * 1e9):
        achieved = fc1_flops / (fc1_ms / 1000.0) / 1e12
        roofline = {"bound": "tensor", "kernel": kernel_name, "achieved": achieved,
                    "peak": mma_peak, "unit": "TFLOP/s", "frac": achieved / mma_peak, "traffic": traffic,
                    "peak_source": f"{peak_src} sustained cuBLAS bf16 GEMM"
                                   + (" x 2 (MXFP8 / bf16 nominal ratio)" if wl.act == "mxfp8" else ""),
                    "algorithmic_flops_per_launch": fc1_flops, "algorithmic_bytes_per_launch": fc1_bytes}
    else:
        achieved = fc1_bytes / (fc1_ms / 1000.0) / 1e9
        roofline = {"bound": "hbm", "kernel": kernel_name, "achieved": achieved,
                    "peak": hbm_peak, "unit": "GB/s", "frac": achieved / hbm_peak, "traffic": traffic,
                    "peak_source": f"{peak_src} HBM copy bandwidth",
                    "algorithmic_bytes_per_launch": fc1_bytes}
    # the whole step against the same bound: weight bytes of the hit experts (FC1 + FC2), or
    # the MMA work of both GEMMs (2 * pairs * 3I * H)
    if roofline["bound"] == "tensor":
        layer_flops = 6.0 * int(counts.sum()) * wl.I * wl.H
        layer_roofline = {"bound": "tensor", "flops": layer_flops,
                          "achieved_tflops": layer_flops / (ms_all / 1000.0) / 1e12,
                          "frac": layer_flops / (ms_all / 1000.0) / 1e12 / mma_peak}
    else:
        layer_roofline = {"bound": "hbm", "weight_bytes": layer_bytes,
                          "achieved_gbs": layer_bytes / (ms_all / 1000.0) / 1e9,
                          "frac": layer_bytes / (ms_all / 1000.0) / 1e9 / hbm_peak}
    rec = {"workload": workload_desc(wl), "ms_per_step": ms_all, "tokens_per_s": value, "hit_experts": hit,
           "gpu_launches": launches, "roofline": roofline, "layer_roofline": layer_roofline, "stage_ms": stage,
           "stage_ms_steps": stage_steps, "clocks": clocks, "e2e": e2e,
           "weight_bytes_resident": (w1.numel() + w1s.numel() + w2.numel() + w2s.numel())}
    layer.close()
    return rec


# the five configurations of the layer, measured by the default run (the first is the headline)
DEFAULT_SET = ("decode", "tiny", "batched_decode", "prefill", "prefill_w4a8", "decode_t1", "decode_t4")


def run_ours(args):
    world, rank, local = dist_setup(args.gpus)
    dev = torch.device("cuda", torch.cuda.current_device())
    names = [args.workload] if args.workload else list(DEFAULT_SET)
    experts_of = None
    if args.parallel == "ep":
        from block_scaled_moe_softmax_b200 import ep

        def experts_of(wl):
            off, n = ep.shard_range(wl.E, world, rank)
            return range(off, off + n)
    cache = WeightCache(dev, experts_of)
    recs = {}
    for name in names:
        wl = workloads.WORKLOADS[name]
        recs[name] = measure(args, wl, cache.get(wl), world, rank)
    head_name = names[0]
    wl = workloads.WORKLOADS[head_name]
    head = recs[head_name]
    line = {
        "metric": METRIC, "value": head["tokens_per_s"], "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": head["ms_per_step"], "higher_is_better": True,
        "scaling": "strong" if args.parallel == "ep" else "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic",
        "config": {"workload": head["workload"], "T": wl.T, "H": wl.H, "I": wl.I, "E": wl.E, "top_k": wl.top_k,
                   "act": wl.act, "hit_experts": head["hit_experts"],
                   "global_batch": wl.T if args.parallel == "ep" else wl.T * world,
                   "parallelism": f"ep{world}" if args.parallel == "ep" else f"replicas{world}",
                   "l2": f"weights {head['weight_bytes_resident'] / 1e9:.2f} GB, a 512 MiB L2 flush before every "
                         "timed step",
                   "weight_scales": "tiled layout (moe_mx_prepare_scales, once before timing)"},
        "e2e": head["e2e"],
        "gpu_launches": head["gpu_launches"],
        "roofline": head["roofline"],
        "layer_roofline": head["layer_roofline"],
        "stage_ms": head["stage_ms"],
        "stage_ms_steps": head["stage_ms_steps"],
        "clocks": head["clocks"],
    }
    if len(recs) > 1:
        line["per_config"] = {n: {k: v for k, v in r.items() if k != "weight_bytes_resident"}
                              for n, r in recs.items()}
    if rank == 0 and not args.no_cpu_baseline:
        cores = len(os.sched_getaffinity(0))
        line["cpu_baseline"] = cpu_baseline(wl, cores)
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default 1000; 200 for --impl reference, whose step is a CPU pair-evaluation)")
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=sorted(workloads.WORKLOADS), default=None,
                    help="one workload only (default: decode as the headline, plus the other four "
                         "configurations in per_config)")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--parallel", choices=["replicas", "ep"], default="replicas",
                    help="replicas: an independent batch per GPU (default); ep: one batch, the experts split "
                         "into contiguous shards over the GPUs, partial outputs all-reduced (NCCL)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    wl = workloads.WORKLOADS[args.workload or DEFAULT_SET[0]]
    if args.steps is None:
        args.steps = 200 if args.impl == "reference" else 1000
    if args.impl == "reference":
        if int(os.environ.get("RANK", "0")) != 0:
            return
        run_reference(args, wl)
        return
    from block_scaled_moe_softmax_b200 import build as lib_build
    lib_build.build()
    run_ours(args)


if __name__ == "__main__":
    main()
