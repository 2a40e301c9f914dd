"""The forward's activation encoders, run on caller data through moe_mx_debug_encode_act.

These are the device functions the forward itself runs (the gather on x, FC1's
epilogue on h, in both of its forms: one thread or one warp per 32-element
block).  w4a8: the codes and E8M0 bytes must equal the oracle's OCP MXFP8
quantiser bit for bit.  w4a16: the two E4M3 term planes must add up to the
bf16-rounded input exactly for every element of at least 2^-13 of its block's
maximum, and within 2^-20 of the maximum below that (the arithmetic of the
split).  Both: a block holding a NaN or an infinity gets the E8M0 NaN byte 0xFF
and zero codes (the oracle's rule for such a block).  Inputs mix magnitudes over
many binades, outlier channels (one element 2^10 .. 2^20 above the rest of its
block), +-0, float32 and bf16 subnormals, exact rounding ties of both terms,
saturation and non-finite blocks.
"""
import numpy as np
import pytest
import torch

import oracle
from block_scaled_moe_softmax_b200 import moe_mx
from tests import helpers

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


K = 256


def _inputs(seed=5):
    rng = np.random.default_rng(seed)
    n = 300  # not a multiple of 128: a ragged last atom row
    mags = 2.0 ** rng.uniform(-40, 40, size=(n, K // 32, 1))
    v = (rng.standard_normal((n, K // 32, 32)) * mags).astype(np.float32)
    # outlier channels: one element 2^10 .. 2^20 above the rest of its block
    for r in range(10, 40):
        b = r % (K // 32)
        v[r, b, :] = rng.standard_normal(32).astype(np.float32)
        v[r, b, r % 32] = np.float32(2.0 ** (10 + (r % 11)) * (1 if r % 2 else -1))
    v[40] = 0.0
    v[41] = -0.0
    v[42, 0, :8] = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0]            # E2M1-grid ties (any scale)
    v[42, 1, :8] = [1.0625, 1.1875, 17.0, 19.0, 448.0, 464.0, 304.0, 240.0]  # E4M3 ties at amax 448
    v[43, 0, :4] = [1e-40, -3e-39, 1.4e-45, 2.0 ** -126]                    # float32 subnormals
    v[43, 1, :3] = [9.2e-41, -9.2e-41, 1.0e-39]                            # bf16 subnormals
    v[44, 0, 5] = np.nan                                                   # non-finite blocks
    v[44, 2, 0] = np.inf
    v[44, 3, 31] = -np.inf
    v[45, :, :] = np.float32(3.4e38)                                      # rounds to bf16 infinity
    v[46, 0, :] = np.float32(2.0 ** 127) * np.linspace(-1, 1, 32, dtype=np.float32)
    return v.reshape(n, K)


def _encode(v, act, method):
    n = v.shape[0]
    src = torch.from_numpy(v).cuda()
    codes = torch.full((2, n, K), 0x5A, dtype=torch.uint8, device="cuda")
    atoms = torch.full(((n + 127) // 128 * (K // 128) * 1024,), 0x5A, dtype=torch.uint8, device="cuda")
    moe_mx.moe_mx_debug_encode_act(src, n, K, act, method, codes, atoms)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), helpers.atoms_to_rowmajor(atoms.cpu().numpy(), n, K)


def _finite_blocks(v):
    return np.isfinite(v.reshape(v.shape[0], K // 32, 32)).all(axis=2)


@pytest.mark.parametrize("method", [0, 1], ids=["thread_per_block", "warp_per_block"])
def test_mxfp8_encoder_matches_oracle_quantiser(method):
    v = _inputs()
    codes, scales = _encode(v, moe_mx.MOE_MX_ACT_MXFP8, method)
    codes_o, scales_o = oracle.mx_quantize(v, oracle.FMT_E4M3)
    assert np.array_equal(scales[0], scales_o)
    assert np.array_equal(codes[0], codes_o)


@pytest.mark.parametrize("method", [0, 1], ids=["thread_per_block", "warp_per_block"])
def test_two_term_split_is_exact(method):
    v = _inputs()
    codes, scales = _encode(v, moe_mx.MOE_MX_ACT_BF16, method)
    ref = helpers.bf16_round(v)
    fin = np.isfinite(ref.reshape(-1, K // 32, 32)).all(axis=2)
    rows = np.nonzero(fin.all(axis=1))[0]
    helpers.check_two_term_split(codes[:, rows], scales[:, rows], ref[rows], "split")
    # blocks that are not finite after the bf16 rounding: 0xFF in both terms, zero codes
    bad = ~fin
    assert bad.sum() >= 4
    for t in range(2):
        assert np.all(scales[t][bad] == 0xFF)
        assert np.all(codes[t].reshape(-1, K // 32, 32)[bad] == 0)


@pytest.mark.parametrize("act", [moe_mx.MOE_MX_ACT_BF16, moe_mx.MOE_MX_ACT_MXFP8], ids=["w4a16", "w4a8"])
def test_both_encoder_forms_agree(act):
    v = _inputs(seed=9)
    c0, s0 = _encode(v, act, 0)
    c1, s1 = _encode(v, act, 1)
    planes = 2 if act == moe_mx.MOE_MX_ACT_BF16 else 1
    assert np.array_equal(c0[:planes], c1[:planes])
    assert np.array_equal(s0[:planes], s1[:planes])


def test_bf16_inputs_encode_without_rounding():
    """The gather hands the encoder bf16 values: the w4a16 split of bf16-valued input reproduces
    it exactly wherever the split is exact (no second rounding)."""
    rng = np.random.default_rng(3)
    v = helpers.bf16_round(rng.standard_normal((128, K)).astype(np.float32) * 3.0).astype(np.float32)
    codes, scales = _encode(v, moe_mx.MOE_MX_ACT_BF16, 0)
    helpers.check_two_term_split(codes, scales, v.astype(np.float64), "bf16 input")


def test_encoder_rejects_bad_arguments():
    src = torch.zeros(4, 200, dtype=torch.float32, device="cuda")
    codes = torch.zeros(2, 4, 256, dtype=torch.uint8, device="cuda")
    atoms = torch.zeros(2048, dtype=torch.uint8, device="cuda")
    for args in ((src, 4, 200, 0, 0), (src, 4, 256, 3, 0), (src, 4, 256, 0, 2), (src.cpu(), 4, 256, 0, 0)):
        with pytest.raises(moe_mx.MoeMxError) as ei:
            moe_mx.moe_mx_debug_encode_act(*args, codes, atoms)
        assert ei.value.code == moe_mx.MOE_MX_ERR_INVALID_ARG
