"""Host logic of the multi-process paths on CPU: gloo ranks.

bench.py runs one independent replica of the layer per GPU; its only
cross-rank steps are a barrier around the timed region and a max over ranks of
the measured time.  These run here with the gloo backend (world size 2), and the
reference arm's non-zero ranks must exit without work.

Expert parallelism (block_scaled_moe_softmax_b200.ep): each rank's partial output
over its contiguous expert shard, summed over the ranks, must equal the whole
layer.  Here the partial outputs come from the oracle (no GPU), the sum from
ep.reduce_partials over gloo ranks (world sizes 2 and 4).
"""
import os
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _rank_main(rank, world, port, results):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        bench.barrier(world)
        t = bench.max_over_ranks(1.0 + rank * 0.5, world)  # rank 0: 1.0 ms, rank 1: 1.5 ms
        results[rank] = t
        bench.barrier(world)
    finally:
        dist.destroy_process_group()


def _free_port():
    import socket
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_max_over_ranks_two_gloo_ranks():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, results)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    assert dict(results) == {0: 1.5, 1: 1.5}


def test_reference_arm_nonzero_rank_exits_without_work():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert r.stdout.strip() == ""


@pytest.mark.parametrize("world", [1])
def test_max_over_ranks_single_rank_is_identity(world):
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(3.25, world) == 3.25


def _ep_rank_main(rank, world, port, results):
    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from block_scaled_moe_softmax_b200 import ep, workloads
    from tests import helpers
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = workloads.Workload("ep", 12, 64, 32, 8, 4, seed=5, routing="given", experts_global=8)
        x = workloads.draw_x(wl)
        ids, w = (a.numpy() for a in workloads.draw_topk(wl))
        wq = helpers.quantize_weights_cpu(wl)
        off, n = ep.shard_range(wl.E, world, rank)
        shard = {k: np.ascontiguousarray(v[off:off + n]) for k, v in wq.items()}
        _, part, _ = oracle.moe_forward_routed(workloads.bf16_bits(x), ids, w, off, shard["w1"], shard["w1s"],
                                               shard["w2"], shard["w2s"])
        total = ep.reduce_partials(torch.from_numpy(part).to(torch.float32))
        _, full, _ = oracle.moe_forward_routed(workloads.bf16_bits(x), ids, w, 0, wq["w1"], wq["w1s"], wq["w2"],
                                               wq["w2s"])
        results[rank] = (float(np.abs(total.double().numpy() - full).max()), float(np.abs(full).max()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_expert_parallel_partials_sum_to_the_layer(world):
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_ep_rank_main, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    for r in range(world):
        err, scale = results[r]
        assert err <= 1e-6 * scale  # float32 rounding of the shards' sums only


def _ep_logits_rank_main(rank, world, port, results):
    """The logits-form chain (ep.ep_forward_logits) on one gloo rank, with the oracle standing in
    for the rank's CUDA partial: every rank routes all tokens over all experts (the oracle's
    router) and evaluates the pairs of its shard (the oracle's routed form at its offset)."""
    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from block_scaled_moe_softmax_b200 import ep, workloads
    from tests import helpers
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = workloads.Workload("ep_logits", 12, 64, 32, 8, 4, seed=9)
        x = workloads.draw_x(wl)
        logits = workloads.draw_logits(wl).numpy()
        wq = helpers.quantize_weights_cpu(wl)
        xb = workloads.bf16_bits(x)

        def partial(offset, n):
            ids, w = oracle.route(logits, wl.top_k)
            shard = {k: np.ascontiguousarray(v[offset:offset + n]) for k, v in wq.items()}
            _, part, _ = oracle.moe_forward_routed(xb, ids, w, offset, shard["w1"], shard["w1s"], shard["w2"],
                                                   shard["w2s"])
            return torch.from_numpy(part).to(torch.float32)

        total = ep.ep_forward_logits(None, None, None, None, None, None, None, wl.top_k, wl.E, rank, world,
                                     partial_fn=partial)
        _, _, _, full = oracle.moe_forward(xb, logits, wq["w1"], wq["w1s"], wq["w2"], wq["w2s"], wl.top_k,
                                           exact=True)
        results[rank] = (float(np.abs(total.double().numpy() - full).max()), float(np.abs(full).max()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
def test_expert_parallel_logits_chain_sums_to_the_layer(world):
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_ep_logits_rank_main, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    for r in range(world):
        err, scale = results[r]
        assert err <= 1e-6 * scale  # float32 rounding of the shards' sums only


def test_shard_range():
    sys.path.insert(0, ROOT)
    from block_scaled_moe_softmax_b200 import ep
    assert ep.shard_range(896, 8, 3) == (336, 112)
    assert ep.shard_range(8, 1, 0) == (0, 8)
    with pytest.raises(ValueError):
        ep.shard_range(10, 4, 0)
    with pytest.raises(ValueError):
        ep.shard_range(8, 2, 2)


def _tp_rank_main(rank, world, port, results):
    import numpy as np
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import oracle
    from block_scaled_moe_softmax_b200 import ep, workloads
    from tests import helpers
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        wl = workloads.Workload("tp", 10, 64, 256, 4, 2, seed=6, routing="given", experts_global=4)
        x = workloads.draw_x(wl)
        ids, w = (a.numpy() for a in workloads.draw_topk(wl))
        wq = helpers.quantize_weights_cpu(wl)
        s1, s1s, s2, s2s = ep.tp_shard_weights(wq["w1"], wq["w1s"], wq["w2"], wq["w2s"], rank, world)
        _, part, _ = oracle.moe_forward_routed(workloads.bf16_bits(x), ids, w, 0, s1, s1s, s2, s2s)
        total = ep.reduce_partials(torch.from_numpy(part).to(torch.float32))
        _, full, _ = oracle.moe_forward_routed(workloads.bf16_bits(x), ids, w, 0, wq["w1"], wq["w1s"], wq["w2"],
                                               wq["w2s"])
        results[rank] = (float(np.abs(total.double().numpy() - full).max()), float(np.abs(full).max()))
    finally:
        dist.destroy_process_group()


def test_tensor_parallel_slices_sum_to_the_layer():
    """Two ranks, each with half of every expert's intermediate dimension (gate/up rows and W2
    columns of one slice): their partial outputs (oracle) summed over gloo equal the layer, as
    SwiGLU acts element by element along the intermediate index."""
    world = 2
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    results = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_tp_rank_main, args=(r, world, port, results)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=300)
        assert p.exitcode == 0
    for r in range(world):
        err, scale = results[r]
        assert err <= 1e-6 * scale


def test_tp_shard_weights_rejects_uneven_slices():
    sys.path.insert(0, ROOT)
    import numpy as np
    from block_scaled_moe_softmax_b200 import ep
    w1 = np.zeros((2, 2 * 256, 32), np.uint8)
    with pytest.raises(ValueError):
        ep.tp_shard_weights(w1, w1, np.zeros((2, 64, 128), np.uint8), np.zeros((2, 64, 8), np.uint8), 0, 4)

