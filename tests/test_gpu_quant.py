"""GPU MX quantiser (moe_mx_quantize) against the oracle's quantiser: bit-exact.

Its MXFP8 path runs mx_encode32, the encoder of the forward's gather; the
forward's own encoders (the gather and FC1's epilogue, on caller data and
inside a forward) are pinned in tests/test_gpu_encoders.py and
tests/test_gpu_intermediates.py.  Inputs mix magnitudes over many binades,
all-zero blocks, exact rounding ties, saturation, negative zeros, subnormals
and non-finite blocks (scale byte 0xFF, zero codes).
"""
import numpy as np
import pytest
import torch

import oracle
from block_scaled_moe_softmax_b200 import moe_mx

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _inputs():
    rng = np.random.default_rng(123)
    n = 4096
    mags = 2.0 ** rng.uniform(-30, 30, size=(n, 1))
    v = (rng.standard_normal((n, 32)) * mags).astype(np.float32)
    v[0] = 0.0
    v[1] = -0.0
    # ties of the E2M1 grid at scale 2^0 (amax 6) and of E4M3 at scale 2^0 (amax 448)
    v[2, :8] = [0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 6.0]
    v[3, :8] = -v[2, :8]
    v[4, :4] = [448.0, 464.0, 304.0, 2.0 ** -10]
    v[5, :3] = [7.9, 7.0, 6.5]                       # saturation above 6
    v[6, :2] = [1e-40, -3e-39]                       # float32 subnormals
    v[7] = np.float32(1e-45)
    v[8, 3] = np.nan                                 # non-finite blocks
    v[9, 0] = np.inf
    v[10, 31] = -np.inf
    return v.reshape(64, 2048)


@pytest.mark.parametrize("fmt", [moe_mx.MOE_MX_FMT_MXFP4, moe_mx.MOE_MX_FMT_MXFP8], ids=["mxfp4", "mxfp8"])
def test_gpu_quantiser_bit_exact(fmt):
    v = _inputs()
    codes_o, scales_o = oracle.mx_quantize(v, fmt)
    codes_g, scales_g = moe_mx.quantize_mx(torch.from_numpy(v).cuda(), fmt)
    torch.cuda.synchronize()
    assert np.array_equal(scales_g.cpu().numpy(), scales_o)
    assert np.array_equal(codes_g.cpu().numpy(), codes_o)


def test_gpu_quantiser_on_weight_distribution():
    from block_scaled_moe_softmax_b200 import workloads
    wl = workloads.WORKLOADS["decode"]
    f = workloads.draw_w1_expert(wl, 3, device="cuda")
    codes_g, scales_g = moe_mx.quantize_mx(f)
    codes_o, scales_o = oracle.mx_quantize(f.cpu().numpy(), oracle.FMT_E2M1)
    assert np.array_equal(scales_g.cpu().numpy(), scales_o)
    assert np.array_equal(codes_g.cpu().numpy(), codes_o)
