"""Shared test helpers: seeded inputs quantised by the oracle, reference dequant, metrics.

Expected values in the tests come only from the oracle (or from independent
libraries); nothing here calls the CUDA library.
"""
import ml_dtypes
import numpy as np
import torch

import oracle
from block_scaled_moe_softmax_b200 import workloads


def quantize_weights_cpu(wl, experts=None, fp32_override=None):
    """MXFP4 weights for workload wl, drawn on the CPU and quantised by the oracle.

    Returns dict with w1, w1s, w2, w2s (numpy uint8, the C-ABI layouts).
    fp32_override: optional (w1_f32 [E,2I,H], w2_f32 [E,H,I]) numpy arrays to quantise instead.
    """
    E, H, I = wl.slots, wl.H, wl.I  # routed experts, then the shared expert's chunks
    w1 = np.zeros((E, 2 * I, H // 2), np.uint8)
    w1s = np.zeros((E, 2 * I, H // 32), np.uint8)
    w2 = np.zeros((E, H, I // 2), np.uint8)
    w2s = np.zeros((E, H, I // 32), np.uint8)
    for e in range(E) if experts is None else experts:
        if fp32_override is not None:
            f1, f2 = fp32_override[0][e], fp32_override[1][e]
        else:
            f1 = workloads.draw_w1_expert(wl, e).numpy()
            f2 = workloads.draw_w2_expert(wl, e).numpy()
        w1[e], w1s[e] = oracle.mx_quantize(f1, oracle.FMT_E2M1)
        w2[e], w2s[e] = oracle.mx_quantize(f2, oracle.FMT_E2M1)
    return dict(w1=w1, w1s=w1s, w2=w2, w2s=w2s)


def dequant_mxfp4_lib(codes, scales):
    """MXFP4 -> float64 through ml_dtypes (independent of the oracle's tables)."""
    lo = (codes & 0xF).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    hi = (codes >> 4).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    vals = np.stack([lo, hi], axis=-1).reshape(codes.shape[:-1] + (codes.shape[-1] * 2,))
    s = scales.view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    return vals * np.repeat(s, 32, axis=-1)


def dequant_mxfp8_lib(codes, scales):
    vals = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    s = scales.view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    return vals * np.repeat(s, 32, axis=-1)


def rel_frobenius(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))


def max_abs_over_rms(got, ref):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    rms = float(np.sqrt(np.mean(ref * ref)))
    return float(np.max(np.abs(got - ref)) / max(rms, 1e-300))


# The layer's stated output tolerance (relative Frobenius error and max error in
# units of the reference RMS), used by every GPU-vs-oracle output comparison.
TOL_REL_FRO = 5e-3
TOL_MAX_OVER_RMS = 2e-2


# ---------------------------------------------------------------- GPU-side helpers
def host_inputs(wl, weights=None):
    """Seeded inputs for workload wl on the host (weights quantised by the oracle on the CPU)."""
    x = workloads.draw_x(wl)
    logits = workloads.draw_logits(wl)
    wq = weights if weights is not None else quantize_weights_cpu(wl)
    return dict(x=x, xb=workloads.bf16_bits(x), logits=logits, **wq)


def to_device(inp, device="cuda"):
    out = {"x": inp["x"].to(device), "logits": inp["logits"].to(device)}
    for k in ("w1", "w1s", "w2", "w2s"):
        out[k] = torch.from_numpy(inp[k]).to(device)
    return out


def oracle_forward(inp, top_k, act_mode, tokens=None):
    """The oracle's output for GPU comparisons: the exact (float64) combined value before
    the final bf16 rounding -- a bf16 result is measured against the value it rounds, not
    against a second, independent rounding of it -- plus the ids and weights."""
    _, ids, w, exact = oracle.moe_forward(inp["xb"], inp["logits"].numpy(), inp["w1"], inp["w1s"], inp["w2"],
                                          inp["w2s"], top_k, act_mode, tokens=tokens, exact=True,
                                          num_shared=inp["w1"].shape[0] - inp["logits"].shape[1])
    return exact, ids, w


def check_output(got_bf16, ref_f64, tag=""):
    got = got_bf16.float().cpu().double().numpy()
    rf = rel_frobenius(got, ref_f64)
    mx = max_abs_over_rms(got, ref_f64)
    assert np.all(np.isfinite(got)), f"{tag}: non-finite outputs"
    assert rf <= TOL_REL_FRO, f"{tag}: relative Frobenius error {rf:.3e} > {TOL_REL_FRO}"
    assert mx <= TOL_MAX_OVER_RMS, f"{tag}: max|gpu-ref|/RMS(ref) {mx:.3e} > {TOL_MAX_OVER_RMS}"
    return rf, mx


def check_output_rows(got_bf16, ref_f64, tag=""):
    """The layer's tolerance applied to each token row against that row's own RMS.  For inputs
    whose tokens differ in scale by orders of magnitude (outlier channels), the final bf16
    rounding alone (2^-9 of each element) of the largest rows exceeds 2e-2 of the whole output's
    RMS -- the oracle's own correctly rounded output does too -- so such cases are held to the
    bound row by row, where the rounding is within it."""
    got = got_bf16.float().cpu().double().numpy()
    ref = np.asarray(ref_f64, np.float64)
    assert np.all(np.isfinite(got)), f"{tag}: non-finite outputs"
    worst_rf, worst_mx = 0.0, 0.0
    for t in range(ref.shape[0]):
        if not np.any(ref[t]):
            assert not np.any(got[t]), f"{tag}: row {t} should be zero"
            continue
        rf, mx = rel_frobenius(got[t], ref[t]), max_abs_over_rms(got[t], ref[t])
        assert rf <= TOL_REL_FRO, f"{tag}: row {t} relative Frobenius error {rf:.3e} > {TOL_REL_FRO}"
        assert mx <= TOL_MAX_OVER_RMS, f"{tag}: row {t} max|gpu-ref|/RMS(row) {mx:.3e} > {TOL_MAX_OVER_RMS}"
        worst_rf, worst_mx = max(worst_rf, rf), max(worst_mx, mx)
    return worst_rf, worst_mx


def check_routing(layer, T, k, E, logits_np):
    """Bit-exact ids/counts/offsets/permutation against the oracle; weights within 2e-6 relative."""
    ids_g, w_g, counts_g, pad_g, sp_g = [a.cpu().numpy() for a in layer.routing(T, k)]
    ids_o, w_o = oracle.route(logits_np, k)
    assert np.array_equal(ids_g, ids_o), "top-k expert ids differ from the oracle"
    np.testing.assert_allclose(w_g, w_o, rtol=2e-6, atol=0)
    counts_o, offs_o, sp_o = oracle.group(ids_o, E)
    assert np.array_equal(counts_g, counts_o), "per-expert counts differ"
    bm = 128
    padded = (counts_o + bm - 1) // bm * bm
    pad_o = np.concatenate([[0], np.cumsum(padded)]).astype(np.int32)
    assert np.array_equal(pad_g, pad_o), "padded segment offsets differ"
    for e in range(E):
        seg = sp_g[pad_o[e]:pad_o[e + 1]]
        assert np.array_equal(seg[:counts_o[e]], sp_o[offs_o[e]:offs_o[e + 1]]), f"permutation differs at expert {e}"
        assert np.all(seg[counts_o[e]:] == -1), f"padding rows of expert {e} are not marked -1"
    return ids_o


# ---------------------------------------------------------------- the activation operand format
def atoms_to_rowmajor(atoms, rows, K):
    """E8M0 scale bytes from the scale-atom layout the library documents (moe_mx.h,
    MOE_MX_INTER_ASF): for row r, 32-element block b and term t, the byte at
    ((r/128)*(K/128) + b/4)*1024 + t*512 + (r%32)*16 + ((r%128)/32)*4 + b%4.
    Returns uint8 [2, rows, K/32]."""
    atoms = np.asarray(atoms, np.uint8).reshape(-1)
    r = np.arange(rows)[:, None]
    b = np.arange(K // 32)[None, :]
    out = np.empty((2, rows, K // 32), np.uint8)
    for t in range(2):
        idx = ((r // 128) * (K // 128) + b // 4) * 1024 + t * 512 + (r % 32) * 16 + ((r % 128) // 32) * 4 + b % 4
        out[t] = atoms[idx]
    return out


def check_two_term_split(codes2, scales2, ref, tag=""):
    """The w4a16 operand: two E4M3 term planes (decoded with ml_dtypes) must add up to the bf16
    values `ref` exactly wherever |ref| >= 2^-13 * the block's max |ref|, and within 2^-20 of the
    block max elsewhere (the mathematics of the split: term 0 keeps each element's top 4
    significant bits at block exponent floor(log2 amax) - 7, term 1 the remainder).
    codes2 uint8 [2, n, K], scales2 uint8 [2, n, K/32], ref float64 [n, K] (finite)."""
    ref = np.asarray(ref, np.float64)
    got = dequant_mxfp8_lib(codes2[0], scales2[0]) + dequant_mxfp8_lib(codes2[1], scales2[1])
    n, K = ref.shape
    amax = np.repeat(np.abs(ref).reshape(n, K // 32, 32).max(axis=2), 32, axis=1)
    big = np.abs(ref) >= amax * 2.0 ** -13
    bad = big & (got != ref)
    assert not bad.any(), f"{tag}: {int(bad.sum())} elements >= 2^-13 amax not exact, e.g. " \
                          f"{ref[bad][:4]} -> {got[bad][:4]}"
    err = np.abs(got - ref)
    over = ~big & (err >= amax * 2.0 ** -20)
    assert not over.any(), f"{tag}: {int(over.sum())} small elements err by >= 2^-20 amax"
    return got


def bf16_round(v):
    """float32 -> nearest bf16 (ties to even) through ml_dtypes, as float64."""
    return np.asarray(v, np.float32).astype(ml_dtypes.bfloat16).astype(np.float64)
