"""Pins for the oracle's layer evaluation (FC1 -> SwiGLU -> FC2 -> combine), CPU only.

The oracle is checked against code paths that do not share its structure:
  * E = 1, k = 1 reduces the layer to a dense SwiGLU MLP, evaluated here with
    torch.matmul in float64 on weights decoded by ml_dtypes (textbook case);
  * brute-force dense evaluation of ALL experts per token with a 0/1 top-k mask
    (no grouping, no per-token expert loop), on the tiny workload;
  * closed forms: identical experts make the output independent of routing
    (the weights sum to 1); relabelling experts leaves the output unchanged;
  * w4a8: MXFP8 activation quantisation applied through ml_dtypes decoding.
Tolerances are far below the size of a plausible mistake (a wrong gate/up
half, a transposed operand, a dropped weight or term) -- each of those is an
O(1) relative error.
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
    # float64 -> bf16 value (torch rounds through float32; fine for these tolerances)
    return torch.from_numpy(np.asarray(a, np.float64)).to(torch.bfloat16).to(torch.float64).numpy()


def _reference_layer(x, logits, wq, k, act_mode=0):
    """Dense reference: every expert for every token, masked by the top-k selection."""
    T, H = x.shape
    E = logits.shape[1]
    W1 = helpers.dequant_mxfp4_lib(wq["w1"], wq["w1s"])  # [E, 2I, H]
    W2 = helpers.dequant_mxfp4_lib(wq["w2"], wq["w2s"])  # [E, H, I]
    I = W1.shape[1] // 2
    a = x.astype(np.float64)
    if act_mode == 1:
        c, s = oracle.mx_quantize(x.astype(np.float32), oracle.FMT_E4M3)
        a = helpers.dequant_mxfp8_lib(c, s)
    # selection mask from torch.topk (tie-free logits) and the renormalised softmax
    lt = torch.from_numpy(logits.astype(np.float64))
    probs = torch.softmax(lt, dim=1)
    _, top = torch.topk(lt, k, dim=1)
    mask = torch.zeros_like(probs).scatter_(1, top, 1.0)
    gate_w = (probs * mask / (probs * mask).sum(dim=1, keepdim=True)).numpy()  # [T, E]
    out = np.zeros((T, H))
    for e in range(E):
        gu = torch.from_numpy(a) @ torch.from_numpy(W1[e]).T  # [T, 2I]
        gu = gu.numpy()
        h = _silu(gu[:, :I]) * gu[:, I:]
        if act_mode == 1:
            c, s = oracle.mx_quantize(h.astype(np.float32), oracle.FMT_E4M3)
            h = helpers.dequant_mxfp8_lib(c, s)
        else:
            h = _bf16(h)
        y = (torch.from_numpy(h) @ torch.from_numpy(W2[e]).T).numpy()  # [T, H]
        out += gate_w[:, e:e + 1] * y
    return out


def _inputs(wl):
    x = workloads.draw_x(wl)
    xb = workloads.bf16_bits(x)
    xf = x.to(torch.float64).numpy()
    logits = workloads.draw_logits(wl).numpy()
    wq = helpers.quantize_weights_cpu(wl)
    return xb, xf, logits, wq


def _oracle_out(xb, logits, wq, k, act_mode=0, tokens=None):
    out, ids, w = oracle.moe_forward(xb, logits, wq["w1"], wq["w1s"], wq["w2"], wq["w2s"], k,
                                     act_mode, tokens=tokens)
    return oracle.bf16_bits_to_f64(out), ids, w


def test_dense_mlp_special_case():
    wl = workloads.Workload("mlp", 8, 64, 32, 1, 1)
    xb, xf, logits, wq = _inputs(wl)
    got, ids, w = _oracle_out(xb, logits, wq, 1)
    assert np.all(ids == 0) and np.all(w == 1.0)
    W1 = helpers.dequant_mxfp4_lib(wq["w1"][0], wq["w1s"][0])
    W2 = helpers.dequant_mxfp4_lib(wq["w2"][0], wq["w2s"][0])
    g = xf @ W1[:32].T
    u = xf @ W1[32:].T
    ref = _bf16(_silu(g) * u) @ W2.T
    assert helpers.rel_frobenius(got, ref) < 4e-3
    assert np.max(np.abs(got - ref)) <= np.max(np.abs(ref)) * 2 ** -7
    # swapping the gate and up halves must be visible (pin against a transposed/misordered FC1)
    ref_swapped = _bf16(_silu(u) * g) @ W2.T
    assert helpers.rel_frobenius(got, ref_swapped) > 0.1


@pytest.mark.parametrize("act_mode", [0, 1])
def test_brute_force_dense_tiny(act_mode):
    wl = workloads.WORKLOADS["tiny"]
    xb, xf, logits, wq = _inputs(wl)
    got, ids, w = _oracle_out(xb, logits, wq, wl.top_k, act_mode)
    ref = _reference_layer(xf, logits, wq, wl.top_k, act_mode)
    assert helpers.rel_frobenius(got, ref) < 5e-3
    assert helpers.max_abs_over_rms(got, ref) < 2e-2


def test_identical_experts_make_routing_irrelevant():
    wl = workloads.Workload("same", 12, 64, 32, 6, 3)
    x = workloads.draw_x(wl)
    xb = workloads.bf16_bits(x)
    f1 = workloads.draw_w1_expert(wl, 0).numpy()
    f2 = workloads.draw_w2_expert(wl, 0).numpy()
    wq = helpers.quantize_weights_cpu(wl, fp32_override=([f1] * wl.E, [f2] * wl.E))
    logits = workloads.draw_logits(wl).numpy()
    got, _, _ = _oracle_out(xb, logits, wq, wl.top_k)
    one = {k: v[:1].copy() for k, v in wq.items()}
    single, _, _ = _oracle_out(xb, np.zeros((wl.T, 1), np.float32), one, 1)
    # sum_j w_j y == y up to the final rounding (weights sum to 1 within 1e-7)
    np.testing.assert_allclose(got, single, rtol=2 ** -7, atol=0)


def test_relabelling_experts_is_invisible():
    wl = workloads.WORKLOADS["tiny"]
    xb, xf, logits, wq = _inputs(wl)
    got, ids, _ = _oracle_out(xb, logits, wq, wl.top_k)
    perm = np.random.default_rng(9).permutation(wl.E)  # new expert perm[e] = old expert e
    inv = np.argsort(perm)
    wq2 = {k: np.ascontiguousarray(v[inv]) for k, v in wq.items()}
    logits2 = np.ascontiguousarray(logits[:, inv])
    got2, ids2, _ = _oracle_out(xb, logits2, wq2, wl.top_k)
    assert np.array_equal(perm[ids], ids2)
    assert np.array_equal(got, got2)


def test_token_subset_matches_full_run():
    wl = workloads.WORKLOADS["tiny"]
    xb, xf, logits, wq = _inputs(wl)
    full, ids, w = _oracle_out(xb, logits, wq, wl.top_k)
    sel = [13, 2, 2, 7]
    part, ids_p, w_p = _oracle_out(xb, logits, wq, wl.top_k, tokens=sel)
    assert np.array_equal(part, full[sel])
    assert np.array_equal(ids_p, ids[sel]) and np.array_equal(w_p, w[sel])


def test_w4a8_on_grid_inputs():
    # With x already on the MXFP8 grid the activation quantisation is the identity, so
    # the two modes differ only through the rounding of h (bf16 vs MXFP8), and the
    # w4a8 result matches the dense reference that applies the MXFP8 steps itself.
    wl = workloads.Workload("grid", 4, 64, 32, 1, 1)
    x = workloads.draw_x(wl).to(torch.float32).numpy()
    c, s = oracle.mx_quantize(x, oracle.FMT_E4M3)
    xg = helpers.dequant_mxfp8_lib(c, s)                    # on the MXFP8 grid, exact in bf16
    xb = workloads.bf16_bits(torch.from_numpy(xg).to(torch.bfloat16))
    c2, s2 = oracle.mx_quantize(xg.astype(np.float32), oracle.FMT_E4M3)
    assert np.array_equal(c, c2) and np.array_equal(s, s2)  # quantising grid values is exact
    wq = helpers.quantize_weights_cpu(wl)
    logits = np.zeros((wl.T, 1), np.float32)
    a16, _, _ = _oracle_out(xb, logits, wq, 1, 0)
    a8, _, _ = _oracle_out(xb, logits, wq, 1, 1)
    # differ only through h's rounding (bf16 vs MXFP8): both ~2^-9 / 2^-4 relative per element
    assert helpers.rel_frobenius(a8, a16) < 0.05
    ref8 = _reference_layer(xg, logits, wq, 1, 1)
    assert helpers.rel_frobenius(a8, ref8) < 5e-3


def test_exact_output_rounds_to_the_bf16_output():
    wl = workloads.WORKLOADS["tiny"]
    xb, xf, logits, wq = _inputs(wl)
    out, _, _, exact = oracle.moe_forward(xb, logits, wq["w1"], wq["w1s"], wq["w2"], wq["w2s"], wl.top_k, 0,
                                          exact=True)
    rounded = np.array([oracle.round_bf16(v) for v in exact.reshape(-1)]).reshape(exact.shape)
    assert np.array_equal(rounded, oracle.bf16_bits_to_f64(out))
