"""Pins for the oracle's shared expert (CPU only).

The shared expert (mxfp6-sm120 package description, routed-MoE path: "shared-expert
combine and routed/shared reduction") is a SwiGLU MLP of intermediate size S*I that
every token passes through, its output added to the routed sum with weight 1.  The
oracle holds it as S chunks of I in expert slots E..E+S-1.  The pins check it against
a dense evaluation of the whole shared MLP from its unchunked weights (torch float64
matmuls on weights decoded by ml_dtypes), which fixes the chunk layout (gate rows,
then up rows of each chunk; W2 column blocks) and the weight of 1, and check that the
routed part is unchanged by adding it.
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


def _shared_setup(S, I=32, H=64, E=4, T=10, k=2, seed=11):
    wl = workloads.Workload("shared", T, H, I, E, k, seed=seed)
    x = workloads.draw_x(wl)
    logits = workloads.draw_logits(wl).numpy()
    routed = helpers.quantize_weights_cpu(wl)
    g = torch.Generator().manual_seed(seed + 1)
    Is = S * I
    w1s_f = (torch.randn(2 * Is, H, generator=g) * 0.02).numpy()   # gate rows [0, Is), up rows [Is, 2Is)
    w2s_f = (torch.randn(H, Is, generator=g) * 0.02).numpy()
    c1, s1 = oracle.mx_quantize(w1s_f, oracle.FMT_E2M1)            # quantised along H, row by row
    c2, s2 = oracle.mx_quantize(w2s_f, oracle.FMT_E2M1)            # quantised along Is in 32-blocks
    # chunk c: gate rows c*I.., then up rows Is + c*I..; W2 columns c*I.. (codes: two per byte)
    ch = {n: [] for n in ("w1", "w1s", "w2", "w2s")}
    for c in range(S):
        rows = np.r_[c * I:(c + 1) * I, Is + c * I:Is + (c + 1) * I]
        ch["w1"].append(c1[rows])
        ch["w1s"].append(s1[rows])
        ch["w2"].append(c2[:, c * I // 2:(c + 1) * I // 2])
        ch["w2s"].append(s2[:, c * I // 32:(c + 1) * I // 32])
    full = {n: np.ascontiguousarray(np.concatenate([routed[n], np.stack(ch[n])])) for n in ch}
    dense = dict(W1=helpers.dequant_mxfp4_lib(c1, s1), W2=helpers.dequant_mxfp4_lib(c2, s2), Is=Is)
    return wl, x, logits, routed, full, dense


def _dense_shared(xf, dense, act_mode):
    a = xf
    if act_mode == 1:
        c, s = oracle.mx_quantize(xf.astype(np.float32), oracle.FMT_E4M3)
        a = helpers.dequant_mxfp8_lib(c, s)
    Is = dense["Is"]
    gu = (torch.from_numpy(a) @ torch.from_numpy(dense["W1"]).T).numpy()
    h = _silu(gu[:, :Is]) * gu[:, Is:]
    if act_mode == 1:
        c, s = oracle.mx_quantize(h.astype(np.float32), oracle.FMT_E4M3)
        h = helpers.dequant_mxfp8_lib(c, s)
    else:
        h = _bf16(h)
    return (torch.from_numpy(h) @ torch.from_numpy(dense["W2"]).T).numpy()


@pytest.mark.parametrize("S", [1, 3])
@pytest.mark.parametrize("act_mode", [0, 1])
def test_shared_expert_is_the_dense_mlp_added_with_weight_one(S, act_mode):
    wl, x, logits, routed, full, dense = _shared_setup(S)
    xb = workloads.bf16_bits(x)
    _, ids, w, with_shared = oracle.moe_forward(xb, logits, full["w1"], full["w1s"], full["w2"], full["w2s"],
                                                wl.top_k, act_mode, exact=True, num_shared=S)
    _, ids_r, w_r, routed_only = oracle.moe_forward(xb, logits, routed["w1"], routed["w1s"], routed["w2"],
                                                    routed["w2s"], wl.top_k, act_mode, exact=True)
    # routed slots unchanged, then the shared slots: experts E.., weight 1
    assert np.array_equal(ids[:, :wl.top_k], ids_r) and np.array_equal(w[:, :wl.top_k], w_r)
    assert np.all(ids[:, wl.top_k:] == np.arange(wl.E, wl.E + S)) and np.all(w[:, wl.top_k:] == 1.0)
    ref = _dense_shared(x.to(torch.float64).numpy(), dense, act_mode)
    got = with_shared - routed_only
    assert helpers.rel_frobenius(got, ref) < 1e-5
    # a plausible mistake is visible: the shared output at half weight, or a chunk missing
    assert helpers.rel_frobenius(0.5 * got, ref) > 0.1


def test_relabelling_routed_experts_leaves_the_layer_unchanged():
    # the shared slots stay at E.. whatever the routed experts' labels
    S = 2
    wl, x, logits, routed, full, dense = _shared_setup(S)
    xb = workloads.bf16_bits(x)
    perm = np.random.default_rng(5).permutation(wl.E)
    inv = np.argsort(perm)
    full2 = {n: np.ascontiguousarray(np.concatenate([v[:wl.E][inv], v[wl.E:]])) for n, v in full.items()}
    a = oracle.moe_forward(xb, logits, full["w1"], full["w1s"], full["w2"], full["w2s"], wl.top_k, 0, num_shared=S)
    b = oracle.moe_forward(xb, np.ascontiguousarray(logits[:, inv]), full2["w1"], full2["w1s"], full2["w2"],
                           full2["w2s"], wl.top_k, 0, num_shared=S)
    assert np.array_equal(a[0], b[0])
