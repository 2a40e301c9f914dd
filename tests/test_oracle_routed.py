"""Pins for the oracle's layer with the routing given (precomputed top-k, global ids, a local
expert shard), CPU only.

What the routed form computes (tokenspeed-situ package description, "Supported contract"):
the caller hands over each token's k global expert ids and weights; only the experts of
the local contiguous shard contribute, and the shards' partial outputs add up to the
whole layer.  The pins tie it to things other than its own code:
  * brute-force dense evaluation: every expert applied to every token (torch float64
    matmuls on weights decoded by ml_dtypes), weighted by a [T, E] matrix built from the
    given ids -- repeated ids add their weights, ids outside the shard add nothing;
  * the sum over a partition of the experts into shards equals the unsharded result;
  * an all-foreign routing gives exact zeros; the logits form's own routing, handed
    over as given ids, reproduces the logits form exactly.
"""
import numpy as np
import pytest
import torch

import oracle
from block_scaled_moe_softmax_b200 import workloads
from tests import helpers


def _silu(g):
    return g / (1.0 + np.exp(-g))


def _bf16(a):
    return torch.from_numpy(np.asarray(a, np.float64)).to(torch.bfloat16).to(torch.float64).numpy()


def _dense(xf, ids, w, offset, wq, act_mode=0):
    """Every local expert on every token, weighted by the given routing."""
    T = xf.shape[0]
    W1 = helpers.dequant_mxfp4_lib(wq["w1"], wq["w1s"])
    W2 = helpers.dequant_mxfp4_lib(wq["w2"], wq["w2s"])
    E, I = W1.shape[0], W1.shape[1] // 2
    gw = np.zeros((T, E))
    for t in range(T):
        for j in range(ids.shape[1]):
            e = int(ids[t, j]) - offset
            if 0 <= e < E:
                gw[t, e] += float(w[t, j])
    a = xf
    if act_mode == 1:
        c, s = oracle.mx_quantize(xf.astype(np.float32), oracle.FMT_E4M3)
        a = helpers.dequant_mxfp8_lib(c, s)
    out = np.zeros((T, W2.shape[1]))
    for e in range(E):
        gu = (torch.from_numpy(a) @ torch.from_numpy(W1[e]).T).numpy()
        h = _silu(gu[:, :I]) * gu[:, I:]
        if act_mode == 1:
            c, s = oracle.mx_quantize(h.astype(np.float32), oracle.FMT_E4M3)
            h = helpers.dequant_mxfp8_lib(c, s)
        else:
            h = _bf16(h)
        out += gw[:, e:e + 1] * (torch.from_numpy(h) @ torch.from_numpy(W2[e]).T).numpy()
    return out


def _setup(E=8, T=12, k=4, H=64, I=32, seed=3):
    wl = workloads.Workload("routed", T, H, I, E, k, routing="given", experts_global=E)
    x = workloads.draw_x(wl)
    wq = helpers.quantize_weights_cpu(wl)
    ids, w = workloads.draw_topk(wl)
    return wl, workloads.bf16_bits(x), x.to(torch.float64).numpy(), ids.numpy(), w.numpy(), wq


def _routed(xb, ids, w, offset, wq, act_mode=0, tokens=None):
    return oracle.moe_forward_routed(xb, ids, w, offset, wq["w1"], wq["w1s"], wq["w2"], wq["w2s"], act_mode,
                                     tokens=tokens)


@pytest.mark.parametrize("act_mode", [0, 1])
def test_brute_force_dense_with_given_routing(act_mode):
    wl, xb, xf, ids, w, wq = _setup()
    ids = ids.copy()
    ids[0, 1] = ids[0, 0]        # a repeated expert: its weights add
    ids[1, 2] = -1               # no expert
    ids[2, 3] = 1000             # an id beyond the layer
    _, exact, loc = _routed(xb, ids, w, 0, wq, act_mode)
    ref = _dense(xf, ids, w, 0, wq, act_mode)
    assert helpers.rel_frobenius(exact, ref) < 5e-3
    assert helpers.max_abs_over_rms(exact, ref) < 2e-2
    assert loc[1, 2] == -1 and loc[2, 3] == -1 and loc[0, 1] == loc[0, 0]


def test_shard_partial_outputs_add_up():
    wl, xb, xf, ids, w, wq = _setup(E=8, k=6)
    _, full, _ = _routed(xb, ids, w, 0, wq)
    total = np.zeros_like(full)
    for a, b in ((0, 3), (3, 5), (5, 8)):
        shard = {n: np.ascontiguousarray(v[a:b]) for n, v in wq.items()}
        _, part, loc = _routed(xb, ids, w, a, shard)
        # the shard's local ids are the global ones minus the offset, -1 elsewhere
        exp_loc = np.where((ids >= a) & (ids < b), ids - a, -1)
        assert np.array_equal(loc, exp_loc)
        # and the partial output is the dense evaluation restricted to the shard
        ref = _dense(xf, ids, w, a, shard)
        assert helpers.rel_frobenius(part, ref) < 5e-3 or np.abs(ref).max() == 0
        total += part
    np.testing.assert_allclose(total, full, rtol=1e-12, atol=1e-12 * np.abs(full).max())


def test_top_k_beyond_the_shard_size():
    # k = 6 slots over a shard of 2 experts: accepted, only local slots count
    wl, xb, xf, ids, w, wq = _setup(E=8, k=6)
    shard = {n: np.ascontiguousarray(v[6:8]) for n, v in wq.items()}
    _, part, _ = _routed(xb, ids, w, 6, shard)
    ref = _dense(xf, ids, w, 6, shard)
    assert helpers.rel_frobenius(part, ref) < 5e-3


def test_foreign_routing_gives_zero():
    wl, xb, xf, ids, w, wq = _setup()
    out, exact, loc = _routed(xb, ids + 100, w, 0, wq)
    assert np.all(exact == 0.0) and np.all(out == 0) and np.all(loc == -1)


def test_logits_routing_handed_over_reproduces_the_logits_form():
    wl = workloads.WORKLOADS["tiny"]
    x = workloads.draw_x(wl)
    xb = workloads.bf16_bits(x)
    logits = workloads.draw_logits(wl).numpy()
    wq = helpers.quantize_weights_cpu(wl)
    out_l, ids, w, exact_l = oracle.moe_forward(xb, logits, wq["w1"], wq["w1s"], wq["w2"], wq["w2s"], wl.top_k, 0,
                                                exact=True)
    out_r, exact_r, loc = _routed(xb, ids, w, 0, wq)
    assert np.array_equal(loc, ids)
    assert np.array_equal(exact_r, exact_l) and np.array_equal(out_r, out_l)
