"""GPU parity of moe_mx_forward_routed (routing given as precomputed top-k with global expert
ids, one contiguous local expert shard, partial outputs) against the CPU oracle.

Checked through the C ABI, on seeded inputs (workloads.draw_topk):
  * the local ids (-1 outside the shard), the weights as given, the per-expert counts,
    the padded offsets and the grouped permutation of the local pairs: bit-exact;
  * each shard's float32 partial output and the bf16 output of the whole layer: within the
    layer's tolerance of the oracle (relative Frobenius <= 5e-3, max err <= 2e-2 RMS);
  * the float32 partial outputs of a partition of the experts add up to the whole layer;
  * edge cases: every id foreign to the shard (exact zeros), repeated ids within a token,
    top-k larger than the shard, both activation modes, both routing kernel paths (a single
    CTA up to 64 tokens, chunked beyond);
  * the shapes of the TokenSpeed SiTU bundle's supported contract (hidden 3584, 896 experts,
    top-16): the TP8 shard (all experts, intermediate 384) and the first EP8 shard (112
    experts, intermediate 3072), with routing bit-exact for every token and the outputs of
    sampled tokens against the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from block_scaled_moe_softmax_b200 import moe_mx, workloads
from tests import helpers

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _dev(wq):
    return {n: torch.from_numpy(v).cuda() for n, v in wq.items()}


def _check_grouping(layer, T, k, E, ids_glob, w_glob, offset):
    """Local ids, weights, counts, padded offsets and permutation against plain numpy."""
    ids_g, w_g, counts_g, pad_g, sp_g = [a.cpu().numpy() for a in layer.routing(T, k)]
    loc = np.where((ids_glob >= offset) & (ids_glob < offset + E), ids_glob - offset, -1).astype(np.int32)
    assert np.array_equal(ids_g, loc), "local expert ids differ"
    assert np.array_equal(w_g.view(np.uint32), w_glob.view(np.uint32)), "weights must be passed through bit for bit"
    flat = loc.reshape(-1)
    counts = np.bincount(flat[flat >= 0], minlength=E).astype(np.int32)
    assert np.array_equal(counts_g, counts), "per-expert counts differ"
    pad = np.concatenate([[0], np.cumsum((counts + 127) // 128 * 128)]).astype(np.int32)
    assert np.array_equal(pad_g, pad), "padded offsets differ"
    order = np.argsort(np.where(flat >= 0, flat, E), kind="stable")  # local pairs by expert, stable
    start = 0
    for e in range(E):
        seg = sp_g[pad[e]:pad[e + 1]]
        assert np.array_equal(seg[:counts[e]], order[start:start + counts[e]]), f"permutation differs at {e}"
        assert np.all(seg[counts[e]:] == -1)
        start += counts[e]


def _setup(T, E, k, H=256, I=128, seed=0):
    wl = workloads.Workload("routed", T, H, I, E, k, seed=seed, routing="given", experts_global=E)
    x = workloads.draw_x(wl)
    ids, w = workloads.draw_topk(wl)
    wq = helpers.quantize_weights_cpu(wl)
    return wl, x, ids.numpy(), w.numpy(), wq


def _gpu(wl, x, ids, w, wq, offset, E_local, act, out_dtype, lo=0):
    layer = moe_mx.MoeMxLayer(wl.H, wl.I, E_local, wl.T, ids.shape[1])
    shard = {n: np.ascontiguousarray(v[lo:lo + E_local]) for n, v in wq.items()}
    d = _dev(shard)
    out = layer.forward_routed(x.cuda(), torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(), d["w1"],
                               d["w1s"], d["w2"], d["w2s"], offset, act, out_dtype)
    assert layer.sync_status() == moe_mx.MOE_MX_OK, moe_mx.moe_mx_last_error()
    return layer, out, shard


@pytest.mark.parametrize("T", [12, 200])
@pytest.mark.parametrize("act", [0, 1], ids=["w4a16", "w4a8"])
def test_shards_match_oracle_and_add_up(T, act):
    E, k = 8, 4
    wl, x, ids, w, wq = _setup(T, E, k)
    ids = ids.copy()
    ids[0, 1] = ids[0, 0]      # a repeated expert within one token
    ids[1, 2] = -1             # no expert
    ids[2, 3] = 1000           # an id beyond the layer
    xb = workloads.bf16_bits(x)
    total = torch.zeros(T, wl.H, dtype=torch.float64)
    for lo, hi in ((0, 3), (3, 5), (5, 8)):
        layer, part, shard = _gpu(wl, x, ids, w, wq, lo, hi - lo, act, moe_mx.MOE_MX_OUT_F32, lo)
        _check_grouping(layer, T, k, hi - lo, ids, w, lo)
        _, ref, _ = oracle.moe_forward_routed(xb, ids, w, lo, shard["w1"], shard["w1s"], shard["w2"], shard["w2s"],
                                              act)
        got = part.double().cpu()
        assert helpers.rel_frobenius(got.numpy(), ref) <= helpers.TOL_REL_FRO
        assert helpers.max_abs_over_rms(got.numpy(), ref) <= helpers.TOL_MAX_OVER_RMS
        total += got
        layer.close()
    _, ref_all, _ = oracle.moe_forward_routed(xb, ids, w, 0, wq["w1"], wq["w1s"], wq["w2"], wq["w2s"], act)
    assert helpers.rel_frobenius(total.numpy(), ref_all) <= helpers.TOL_REL_FRO
    assert helpers.max_abs_over_rms(total.numpy(), ref_all) <= helpers.TOL_MAX_OVER_RMS
    # the whole layer in one call, bf16 output
    layer, out, _ = _gpu(wl, x, ids, w, wq, 0, E, act, moe_mx.MOE_MX_OUT_BF16)
    helpers.check_output(out, ref_all, f"routed T={T} act={act}")
    layer.close()


def test_top_k_beyond_shard_and_foreign_routing():
    wl, x, ids, w, wq = _setup(40, 8, 6)
    layer, part, shard = _gpu(wl, x, ids, w, wq, 6, 2, 0, moe_mx.MOE_MX_OUT_F32, 6)
    _check_grouping(layer, 40, 6, 2, ids, w, 6)
    _, ref, _ = oracle.moe_forward_routed(workloads.bf16_bits(x), ids, w, 6, shard["w1"], shard["w1s"],
                                          shard["w2"], shard["w2s"], 0)
    assert helpers.rel_frobenius(part.double().cpu().numpy(), ref) <= helpers.TOL_REL_FRO
    # every id outside the shard: nothing grouped, exact zeros written over the output
    out = torch.full((40, wl.H), 7.0, dtype=torch.float32, device="cuda")
    d = _dev(shard)
    layer.forward_routed(x.cuda(), torch.from_numpy(ids + 100).cuda(), torch.from_numpy(w).cuda(), d["w1"], d["w1s"],
                         d["w2"], d["w2s"], 6, 0, moe_mx.MOE_MX_OUT_F32, out=out)
    assert layer.sync_status() == moe_mx.MOE_MX_OK, moe_mx.moe_mx_last_error()
    assert torch.count_nonzero(out).item() == 0
    layer.close()


@pytest.mark.parametrize("T", [12, 200])
@pytest.mark.parametrize("act", [0, 1], ids=["w4a16", "w4a8"])
def test_logits_shards_match_oracle_and_add_up(T, act):
    """moe_mx_forward_shard: the whole layer's router on every token, the pairs of one contiguous
    shard kept.  Local ids (-1 outside the shard) bit-exact and the whole layer's weights within
    2e-6 of the oracle's router; counts and the grouping of the local pairs bit-exact; each shard's
    float32 partial within the tolerance of the oracle's routed form at the shard's offset; the
    partials of a partition adding up to the oracle's layer; and the shard [0, E) giving the bits
    of moe_mx_forward."""
    E, k = 8, 4
    wl = workloads.Workload("shard", T, 256, 128, E, k, "bf16", "normal", 4)
    x, logits = workloads.draw_x(wl), workloads.draw_logits(wl)
    wq = helpers.quantize_weights_cpu(wl)
    xb = workloads.bf16_bits(x)
    ids_o, w_o = oracle.route(logits.numpy(), k)
    total = torch.zeros(T, wl.H, dtype=torch.float64)
    for lo, hi in ((0, 3), (3, 5), (5, 8)):
        layer = moe_mx.MoeMxLayer(wl.H, wl.I, hi - lo, T, k)
        d = _dev({n: np.ascontiguousarray(v[lo:hi]) for n, v in wq.items()})
        part = layer.forward_shard(x.cuda(), logits.cuda(), d["w1"], d["w1s"], d["w2"], d["w2s"], k, lo, act)
        assert layer.sync_status() == moe_mx.MOE_MX_OK, moe_mx.moe_mx_last_error()
        ids_g, w_g = [a.cpu().numpy() for a in layer.routing(T, k)[:2]]
        np.testing.assert_allclose(w_g, w_o, rtol=2e-6, atol=0)
        _check_grouping(layer, T, k, hi - lo, ids_o, w_g, lo)
        shard = {n: np.ascontiguousarray(v[lo:hi]) for n, v in wq.items()}
        _, ref, _ = oracle.moe_forward_routed(xb, ids_o, w_o, lo, shard["w1"], shard["w1s"], shard["w2"],
                                              shard["w2s"], act)
        got = part.double().cpu()
        assert helpers.rel_frobenius(got.numpy(), ref) <= helpers.TOL_REL_FRO
        assert helpers.max_abs_over_rms(got.numpy(), ref) <= helpers.TOL_MAX_OVER_RMS
        total += got
        layer.close()
    inp = dict(xb=xb, logits=logits, **wq)
    ref_all, _, _ = helpers.oracle_forward(inp, k, act)
    assert helpers.rel_frobenius(total.numpy(), ref_all) <= helpers.TOL_REL_FRO
    assert helpers.max_abs_over_rms(total.numpy(), ref_all) <= helpers.TOL_MAX_OVER_RMS
    # the shard of all experts, bf16 output: the bits of moe_mx_forward
    layer = moe_mx.MoeMxLayer(wl.H, wl.I, E, T, k)
    d = _dev(wq)
    full = layer.forward(x.cuda(), logits.cuda(), d["w1"], d["w1s"], d["w2"], d["w2s"], k, act)
    sh = layer.forward_shard(x.cuda(), logits.cuda(), d["w1"], d["w1s"], d["w2"], d["w2s"], k, 0, act,
                             moe_mx.MOE_MX_OUT_BF16)
    assert layer.sync_status() == moe_mx.MOE_MX_OK, moe_mx.moe_mx_last_error()
    assert torch.equal(full.view(torch.int16), sh.view(torch.int16))
    layer.close()


def test_shard_form_rejects_bad_shards():
    layer = moe_mx.MoeMxLayer(256, 128, 4, 8, 2)
    x = torch.zeros(8, 256, dtype=torch.bfloat16, device="cuda")
    lg = torch.zeros(8, 8, dtype=torch.float32, device="cuda")
    w1 = torch.zeros(4, 256, 128, dtype=torch.uint8, device="cuda")
    w1s = torch.full((4, 256, 8), 127, dtype=torch.uint8, device="cuda")
    w2 = torch.zeros(4, 256, 64, dtype=torch.uint8, device="cuda")
    w2s = torch.full((4, 256, 4), 127, dtype=torch.uint8, device="cuda")
    out = torch.empty(8, 256, dtype=torch.float32, device="cuda")
    for E_g, off in ((8, 5), (8, -1), (3, 0), (2000, 0)):   # shard beyond the layer, negative, too small, too many
        with pytest.raises(moe_mx.MoeMxError) as ei:
            moe_mx.moe_mx_forward_shard(layer.handle, x, lg, 8, E_g, off, w1, w1s, w2, w2s, 2, 0, out)
        assert ei.value.code == moe_mx.MOE_MX_ERR_INVALID_ARG
    layer.close()


def _tokens(ids, E_local, offset, T, n_random=6):
    loc = (ids >= offset) & (ids < offset + E_local)
    n_local = loc.sum(axis=1)
    toks = {0, T - 1, int(np.argmax(n_local)), int(np.argmin(n_local))}
    rng = np.random.default_rng(77)
    toks.update(int(t) for t in rng.choice(T, size=n_random, replace=False))
    return sorted(toks)


@pytest.mark.slow
@pytest.mark.parametrize("name", ["situ_tp8", "situ_ep8"])
def test_page_contract_shapes(name):
    wl = workloads.WORKLOADS[name]
    E, H, I = wl.E, wl.H, wl.I
    host = dict(w1=np.empty((E, 2 * I, H // 2), np.uint8), w1s=np.empty((E, 2 * I, H // 32), np.uint8),
                w2=np.empty((E, H, I // 2), np.uint8), w2s=np.empty((E, H, I // 32), np.uint8))
    for e in range(E):
        host["w1"][e], host["w1s"][e] = oracle.mx_quantize(workloads.draw_w1_expert(wl, e, "cuda").cpu().numpy(),
                                                           oracle.FMT_E2M1)
        host["w2"][e], host["w2s"][e] = oracle.mx_quantize(workloads.draw_w2_expert(wl, e, "cuda").cpu().numpy(),
                                                           oracle.FMT_E2M1)
    x = workloads.draw_x(wl)
    ids, w = (a.numpy() for a in workloads.draw_topk(wl))
    layer, out, _ = _gpu(wl, x, ids, w, host, wl.local_offset, E, 0, moe_mx.MOE_MX_OUT_F32)
    _check_grouping(layer, wl.T, wl.top_k, E, ids, w, wl.local_offset)
    toks = _tokens(ids, E, wl.local_offset, wl.T)
    _, ref, _ = oracle.moe_forward_routed(workloads.bf16_bits(x), ids, w, wl.local_offset, host["w1"], host["w1s"],
                                          host["w2"], host["w2s"], 0, tokens=toks)
    got = out[toks].double().cpu().numpy()
    assert helpers.rel_frobenius(got, ref) <= helpers.TOL_REL_FRO, name
    assert helpers.max_abs_over_rms(got, ref) <= helpers.TOL_MAX_OVER_RMS, name
    layer.close()


def test_expert_parallel_forward_two_shards_on_one_gpu():
    """ep.ep_forward per rank of a 2-way expert split (run one after another on one GPU, with no
    process group, so each returns its own partial output): their sum is the whole layer."""
    from block_scaled_moe_softmax_b200 import ep
    wl, x, ids, w, wq = _setup(40, 8, 4)
    total = torch.zeros(40, wl.H, dtype=torch.float64)
    for rank in range(2):
        off, n = ep.shard_range(wl.E, 2, rank)
        layer = moe_mx.MoeMxLayer(wl.H, wl.I, n, wl.T, 4)
        d = _dev({k: np.ascontiguousarray(v[off:off + n]) for k, v in wq.items()})
        part = ep.ep_forward(layer, x.cuda(), torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(), d["w1"],
                             d["w1s"], d["w2"], d["w2s"], wl.E, rank, 2)
        assert layer.sync_status() == moe_mx.MOE_MX_OK, moe_mx.moe_mx_last_error()
        total += part.double().cpu()
        layer.close()
    _, ref, _ = oracle.moe_forward_routed(workloads.bf16_bits(x), ids, w, 0, wq["w1"], wq["w1s"], wq["w2"], wq["w2s"])
    assert helpers.rel_frobenius(total.numpy(), ref) <= helpers.TOL_REL_FRO
    assert helpers.max_abs_over_rms(total.numpy(), ref) <= helpers.TOL_MAX_OVER_RMS


def test_tensor_parallel_slices_on_one_gpu():
    """ep.tp_shard_weights: two ranks' slices of every expert's intermediate dimension, each run
    through moe_mx_forward_routed with a float32 output (one after another on one GPU); their sum
    is the whole layer."""
    from block_scaled_moe_softmax_b200 import ep
    wl, x, ids, w, wq = _setup(24, 4, 2, H=256, I=256)
    total = torch.zeros(24, wl.H, dtype=torch.float64)
    for rank in range(2):
        s1, s1s, s2, s2s = ep.tp_shard_weights(*(torch.from_numpy(wq[n]).cuda() for n in ("w1", "w1s", "w2", "w2s")),
                                               rank, 2)
        layer = moe_mx.MoeMxLayer(wl.H, wl.I // 2, wl.E, wl.T, 2)
        part = layer.forward_routed(x.cuda(), torch.from_numpy(ids).cuda(), torch.from_numpy(w).cuda(), s1, s1s, s2,
                                    s2s, 0, 0, moe_mx.MOE_MX_OUT_F32)
        assert layer.sync_status() == moe_mx.MOE_MX_OK, moe_mx.moe_mx_last_error()
        total += part.double().cpu()
        layer.close()
    _, ref, _ = oracle.moe_forward_routed(workloads.bf16_bits(x), ids, w, 0, wq["w1"], wq["w1s"], wq["w2"], wq["w2s"])
    assert helpers.rel_frobenius(total.numpy(), ref) <= helpers.TOL_REL_FRO
    assert helpers.max_abs_over_rms(total.numpy(), ref) <= helpers.TOL_MAX_OVER_RMS
