"""Pins for the oracle's MX codecs and quantiser (CPU only).

Each test ties the oracle to something other than itself: the hand-derived
golden cases in tests/golden/mx_quant_cases.txt, the bit-field definitions of
the OCP MX v1.0 formats, and independent library routines (ml_dtypes'
float4_e2m1fn / float8_e4m3fn / float8_e8m0fnu, torch's float8_e4m3fn).
"""
import os

import ml_dtypes
import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "mx_quant_cases.txt")


def _golden_cases():
    cases = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            fmt, scale, vals, codes = [p.strip() for p in line.split("|")]
            cases.append((fmt, int(scale), [float(v) for v in vals.split(",")],
                          [int(c) for c in codes.split(",")]))
    return cases


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: f"{c[0]}-{c[1]}")
def test_quantise_golden(case):
    fmt_name, scale, vals, codes = case
    fmt = oracle.FMT_E2M1 if fmt_name == "e2m1" else oracle.FMT_E4M3
    v = np.array([vals], dtype=np.float32)
    assert len(vals) == 32 and len(codes) == 32
    c, s = oracle.mx_quantize(v, fmt)
    assert int(s[0, 0]) == scale
    if fmt == oracle.FMT_E2M1:
        got = [int(c[0, i // 2] >> (4 * (i & 1))) & 0xF for i in range(32)]
    else:
        got = [int(x) for x in c[0]]
    assert got == codes


def test_e2m1_decode_against_bitfields_and_ml_dtypes():
    lib_vals = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    for code in range(16):
        s, e, m = code >> 3, (code >> 1) & 3, code & 1
        # OCP MX E2M1: bias 1; e == 0 is subnormal (m * 2^-1)
        mag = m * 0.5 if e == 0 else 2.0 ** (e - 1) * (1 + m / 2)
        want = -mag if s else mag
        got = oracle.e2m1_decode(code)
        assert got == want == lib_vals[code]
        assert np.signbit(got) == bool(s)


def test_e4m3_decode_exhaustive_against_libraries():
    codes = np.arange(256, dtype=np.uint8)
    via_torch = torch.from_numpy(codes.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    via_ml = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    for c in range(256):
        got = oracle.e4m3_decode(c)
        if (c & 0x7F) == 0x7F:
            assert np.isnan(got) and np.isnan(via_torch[c]) and np.isnan(via_ml[c])
        else:
            assert got == via_torch[c] == via_ml[c], c
    assert oracle.e4m3_decode(0x7E) == 448.0
    assert oracle.e4m3_decode(0x01) == 2.0 ** -9


def test_e8m0_decode_all_bytes():
    lib = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e8m0fnu).astype(np.float64)
    for b in range(255):
        assert oracle.e8m0_decode(b) == 2.0 ** (b - 127) == lib[b]
    assert np.isnan(oracle.e8m0_decode(255)) and np.isnan(lib[255])


def _random_blocks(rng, n, scale_range=(-12, 12)):
    # blocks with widely varying magnitudes, some exact grid ties mixed in
    mags = 2.0 ** rng.uniform(*scale_range, size=(n, 1))
    v = rng.standard_normal((n, 32)) * mags
    return v.astype(np.float32)


def _scale_rule(v, emax):
    amax = np.abs(v).max(axis=1).astype(np.float64)
    out = np.zeros(len(v), dtype=np.int64)
    nz = amax > 0
    # floor(log2(amax)) for amax in [2^m, 2^(m+1)) is m; frexp gives the exponent exactly
    m = np.frexp(amax[nz])[1] - 1
    out[nz] = np.clip(m - emax, -127, 127) + 127
    return out


@pytest.mark.parametrize("fmt", [oracle.FMT_E2M1, oracle.FMT_E4M3])
def test_scale_rule_binade(fmt):
    rng = np.random.default_rng(1)
    v = _random_blocks(rng, 2000)
    _, s = oracle.mx_quantize(v, fmt)
    emax = 2 if fmt == oracle.FMT_E2M1 else 8
    want = _scale_rule(v, emax)
    assert np.array_equal(s[:, 0].astype(np.int64), want)
    # and the defining property: 2^(byte-127+emax) <= amax < 2^(byte-127+emax+1)
    amax = np.abs(v).max(axis=1).astype(np.float64)
    lo = 2.0 ** (s[:, 0].astype(np.float64) - 127 + emax)
    assert np.all(lo <= amax) and np.all(amax < 2 * lo)


def test_e2m1_rounding_matches_ml_dtypes():
    rng = np.random.default_rng(2)
    v = _random_blocks(rng, 3000)
    # plant exact ties of the E2M1 grid (relative to the block scale)
    v[:, 1] = v[:, 0] * 0  # zeros
    codes, s = oracle.mx_quantize(v, oracle.FMT_E2M1)
    scale = 2.0 ** (s.astype(np.float64) - 127)
    t = (v.astype(np.float64) / np.repeat(scale, 32, axis=1)).astype(np.float32)
    lib = t.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    got = np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(v.shape)
    assert np.array_equal(got, lib)


def test_e2m1_ties_against_ml_dtypes():
    # every half-way point of the grid, both signs, with the block amax pinned to 6
    ties = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0], dtype=np.float32)
    blk = np.zeros((2, 32), dtype=np.float32)
    blk[0, :7] = ties
    blk[0, 7] = 6.0
    blk[1, :7] = -ties
    blk[1, 7] = -6.0
    codes, s = oracle.mx_quantize(blk, oracle.FMT_E2M1)
    assert list(s[:, 0]) == [127, 127]
    got = np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(2, 32)
    lib = blk.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    assert np.array_equal(got, lib)


def test_e4m3_rounding_matches_libraries():
    rng = np.random.default_rng(3)
    v = _random_blocks(rng, 3000)
    codes, s = oracle.mx_quantize(v, oracle.FMT_E4M3)
    scale = 2.0 ** (s.astype(np.float64) - 127)
    t = v.astype(np.float64) / np.repeat(scale, 32, axis=1)
    t = np.clip(t, -448.0, 448.0).astype(np.float32)  # the libraries do not saturate
    lib_ml = t.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    lib_torch = torch.from_numpy(t).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(codes, lib_ml)
    assert np.array_equal(codes, lib_torch)


@pytest.mark.parametrize("fmt", [oracle.FMT_E2M1, oracle.FMT_E4M3])
def test_round_trip_is_identity_on_codes(fmt):
    # every code appears in a block whose amax code is the format maximum:
    # quantising the dequantised values must give back the same codes and scale
    ncode = 16 if fmt == oracle.FMT_E2M1 else 256
    valid = [c for c in range(ncode) if fmt == oracle.FMT_E2M1 or (c & 0x7F) != 0x7F]
    maxcode = 7 if fmt == oracle.FMT_E2M1 else 0x7E
    for scale_byte in (100, 120, 127, 131):
        for start in range(0, len(valid), 31):
            chunk = valid[start:start + 31]
            blk_codes = np.array(chunk + [maxcode] * (32 - len(chunk)), dtype=np.uint8)
            if fmt == oracle.FMT_E2M1:
                packed = (blk_codes[0::2] | (blk_codes[1::2] << 4)).astype(np.uint8)[None]
            else:
                packed = blk_codes[None]
            sc = np.array([[scale_byte]], dtype=np.uint8)
            vals = oracle.mx_dequantize(packed, sc, fmt).astype(np.float32)
            c2, s2 = oracle.mx_quantize(vals, fmt)
            assert int(s2[0, 0]) == scale_byte
            assert np.array_equal(c2, packed)


def test_quantisation_error_bound():
    # |v - dequant(q)| <= half a grid step at v's magnitude, except above the largest
    # magnitude 6 where saturation costs t - 6; measured relative to the block scale
    rng = np.random.default_rng(4)
    v = _random_blocks(rng, 500)
    codes, s = oracle.mx_quantize(v, oracle.FMT_E2M1)
    dq = oracle.mx_dequantize(codes, s, oracle.FMT_E2M1)
    scale = np.repeat(2.0 ** (s.astype(np.float64) - 127), 32, axis=1)
    t = np.abs(v.astype(np.float64)) / scale
    step = np.where(t < 2, 0.5, np.where(t < 4, 1.0, 2.0))
    bound = np.maximum(step / 2, t - 6.0)
    assert np.all(np.abs(v - dq) / scale <= bound + 1e-12)
    assert np.any(t > 7.0)  # the saturating branch is exercised


def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(5)
    vals = (rng.standard_normal(20000) * 2.0 ** rng.uniform(-40, 40, 20000)).astype(np.float32)
    # plus exact ties: bf16 value + half ulp
    base = torch.from_numpy(vals[:2000]).to(torch.bfloat16).to(torch.float32).numpy()
    half_ulp = 2.0 ** (np.frexp(base.astype(np.float64))[1] - 9)
    ties = (base.astype(np.float64) + np.sign(base) * half_ulp).astype(np.float32)
    allv = np.concatenate([vals, ties, np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8], np.float32)])
    want = torch.from_numpy(allv).to(torch.bfloat16).to(torch.float64).numpy()
    got = np.array([oracle.round_bf16(float(x)) for x in allv])
    assert np.array_equal(got, want)
    # the two hand-checked ties: 1 + 2^-8 -> 1 (even), 1 + 3*2^-8 -> 1 + 2^-6
    assert oracle.round_bf16(1.0 + 2 ** -8) == 1.0
    assert oracle.round_bf16(1.0 + 3 * 2 ** -8) == 1.0 + 2 ** -6


def test_quantise_rejects_bad_shapes():
    with pytest.raises(ValueError):
        oracle.mx_quantize(np.zeros((2, 48), np.float32), oracle.FMT_E2M1)
