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
    E, H, I = wl.E, wl.H, wl.I
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
