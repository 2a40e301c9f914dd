"""The forward on special values, against the oracle.

* Weight scale bytes at the ends of the E8M0 range: 0 and 1 (2^-127, 2^-126)
  in random blocks of W1 and W2, and 253, 254 (2^126, 2^127) in a few W2 rows,
  all within the layer's tolerance of the oracle (contributions below float32's
  normal range may be flushed to zero; they are far below the tolerance).
* The E8M0 NaN byte 0xFF in one W2 block: exactly the outputs that block
  reaches are NaN, as in the oracle; the others meet the tolerance.
* A NaN or an infinity in a token's activations: that token's outputs are NaN
  (its block is encoded with the NaN scale byte, as the oracle's MXFP8 rule
  does; the oracle's bf16 evaluation is NaN as well), the other tokens meet the
  tolerance.
"""
import numpy as np
import pytest
import torch

from block_scaled_moe_softmax_b200 import moe_mx, workloads
from tests import helpers

pytestmark = pytest.mark.gpu

WL = workloads.WORKLOADS["tiny"]


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _run(inp, act):
    d = helpers.to_device(inp)
    layer = moe_mx.MoeMxLayer(WL.H, WL.I, WL.E, WL.T, WL.top_k)
    out = layer.forward(d["x"], d["logits"], d["w1"], d["w1s"], d["w2"], d["w2s"], WL.top_k, act)
    assert layer.sync_status() == moe_mx.MOE_MX_OK, moe_mx.moe_mx_last_error()
    layer.close()
    ref, ids, _ = helpers.oracle_forward(inp, WL.top_k, act)
    return out.float().cpu().double().numpy(), ref, ids


def _compare_with_nans(got, ref, tag):
    nan_ref = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan_ref), \
        f"{tag}: NaN outputs differ ({int(np.isnan(got).sum())} GPU vs {int(nan_ref.sum())} oracle)"
    fin = ~nan_ref
    assert helpers.rel_frobenius(got[fin], ref[fin]) <= helpers.TOL_REL_FRO, tag
    assert helpers.max_abs_over_rms(got[fin], ref[fin]) <= helpers.TOL_MAX_OVER_RMS, tag
    return int(nan_ref.sum())


@pytest.mark.parametrize("act", [0, 1], ids=["w4a16", "w4a8"])
def test_smallest_scale_bytes(act):
    inp = helpers.host_inputs(WL)
    rng = np.random.default_rng(5)
    for name in ("w1s", "w2s"):
        s = inp[name].copy()
        mask = rng.random(s.shape) < 0.2
        s[mask] = rng.choice(np.array([0, 1], np.uint8), size=int(mask.sum()))
        inp[name] = s
    got, ref, _ = _run(inp, act)
    helpers.check_output(torch.from_numpy(got), ref, "scale bytes 0 and 1")


@pytest.mark.parametrize("act", [0, 1], ids=["w4a16", "w4a8"])
def test_largest_finite_scale_bytes(act):
    inp = helpers.host_inputs(WL)
    _, ids, _ = helpers.oracle_forward(inp, WL.top_k, act)
    e = int(ids[0, 0])                      # an expert that token 0 uses
    w2, w2s = inp["w2"].copy(), inp["w2s"].copy()
    rows = np.arange(0, 16)
    w2[e, rows, :16] = np.where(rows[:, None] % 2 == 0, 0x11, 0x99).astype(np.uint8)  # +-0.5 codes, block 0
    w2s[e, rows, 0] = np.where(rows % 2 == 0, 253, 254).astype(np.uint8)
    inp["w2"], inp["w2s"] = w2, w2s
    got, ref, _ = _run(inp, act)
    assert np.abs(ref).max() > 1e30, "the case needs outputs near the top of the float32 range"
    assert np.all(np.isfinite(got))
    helpers.check_output(torch.from_numpy(got), ref, "scale bytes 253 and 254")


@pytest.mark.parametrize("act", [0, 1], ids=["w4a16", "w4a8"])
def test_nan_scale_byte(act):
    inp = helpers.host_inputs(WL)
    _, ids, _ = helpers.oracle_forward(inp, WL.top_k, act)
    e = int(ids[0, 0])
    w2s = inp["w2s"].copy()
    w2s[e, 5, 1] = 0xFF                    # output column 5 of every token routed to expert e
    inp["w2s"] = w2s
    got, ref, _ = _run(inp, act)
    n = _compare_with_nans(got, ref, "scale byte 0xFF")
    assert n >= 1 and np.isnan(ref[:, 5]).sum() == n


@pytest.mark.parametrize("act", [0, 1], ids=["w4a16", "w4a8"])
def test_non_finite_activations(act):
    inp = helpers.host_inputs(WL)
    x = inp["x"].float().clone()
    x[2, 7] = float("nan")
    x[9, 200] = float("inf")
    x[11, 0] = float("-inf")
    inp["x"] = x.to(torch.bfloat16)
    inp["xb"] = workloads.bf16_bits(inp["x"])
    got, ref, _ = _run(inp, act)
    _compare_with_nans(got, ref, "non-finite x")
    assert np.isnan(ref[[2, 9, 11]]).all()
