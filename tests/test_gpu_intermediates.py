"""Stage-by-stage checks of the forward through moe_mx_get_intermediate.

(a) w4a8: every grouped row of FC1's activation operand (codes and E8M0 bytes)
    equals the oracle's OCP MXFP8 quantisation of that row's token, bit for bit.
(b) w4a16: the operand's two E4M3 term planes add up to the token's bf16 row
    exactly wherever the split is exact (elements of at least 2^-13 of their
    block's maximum) and within 2^-20 of the maximum elsewhere, on rows with
    outlier channels, +-0, bf16 subnormals and exact ties.
(c)/(d) Exact special cases, in the spirit of the mxfp6-sm120 package
    description ("Performance", dense GEMM and MoE layer: outputs exact against a
    decoded FP32 matmul reference): power-of-two activations, power-of-two
    scales and small E2M1 codes, chosen so that every FC1 sum is exact in
    float32 and every gate value g is at least 17, where 1 + exp(-g) rounds to 1
    in float32 and SwiGLU's h = silu(g) * u is exactly g * u.
    (i)  x varies along K and W1's block scales vary: FC1's h operand equals the
         bf16 rounding (w4a16) or the oracle's MXFP8 quantisation (w4a8) of the
         exact g * u, bit for bit -- the MMAs, the K order, the SwiGLU epilogue
         and its encoder, with the GPU's own float32 h known exactly;
    (ii) x constant per token, every scale 2^0: h takes few significant bits.
    In both, FC2's float32 rows Y must equal the decoded float64 matmul of W2
    with the GPU's own h operand exactly, and the output must meet the tolerance
    against the exact weighted sum of those rows.  (The oracle's SwiGLU runs in
    double, where 1 + exp(-g) is not 1: its h sits a hair below g * u and lands
    on the other side of a rounding tie now and then, so the output is compared
    with the oracle only where h needs no rounding: case (ii), w4a16.)
    Every kernel variant (activation tiles of 16, 32, 64 or 128 rows, the wide
    two-tile variant, both orientations) and both activation modes.
"""
import ml_dtypes
import numpy as np
import pytest
import torch

import oracle
from block_scaled_moe_softmax_b200 import moe_mx, workloads
from tests import helpers
from tests.test_gpu_forward import VARIANTS

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _set_variant(monkeypatch, variant):
    tile_rows, swap_rows, wide = VARIANTS[variant]
    for name, val in (("MOE_MX_TILE_ROWS", tile_rows), ("MOE_MX_SWAP_ROWS", swap_rows), ("MOE_MX_WIDE", wide)):
        if val is not None:
            monkeypatch.setenv(name, str(val))


def _grouped_rows(layer, T, k, E):
    """(grouped row, token, expert, slot) of every real pair of the last forward."""
    ids, _, counts, pad, sp = [a.cpu().numpy() for a in layer.routing(T, k)]
    rows = []
    for e in range(E):
        for r in range(pad[e], pad[e] + counts[e]):
            p = int(sp[r])
            rows.append((r, p // k, int(ids[p // k, p % k]), p % k))
    return np.array(rows, dtype=np.int64).reshape(-1, 4)


def _forward(wl, x_bf16, logits, w, act):
    layer = moe_mx.MoeMxLayer(wl.H, wl.I, wl.E, wl.T, wl.top_k)
    out = layer.forward(x_bf16.cuda(), logits.cuda(), *(torch.from_numpy(w[n]).cuda() for n in
                                                          ("w1", "w1s", "w2", "w2s")), wl.top_k, act)
    assert layer.sync_status() == moe_mx.MOE_MX_OK, moe_mx.moe_mx_last_error()
    inter = {n: t.cpu().numpy() for n, t in layer.intermediates(wl.T, wl.top_k).items()}
    grows = _grouped_rows(layer, wl.T, wl.top_k, wl.E)
    return layer, out, inter, grows


def _operand(inter, name, rows_total, K):
    codes = inter[name[0] + "q"]
    scales = helpers.atoms_to_rowmajor(inter[name[0] + "sf"], rows_total, K)
    return codes, scales


# ---------------------------------------------------------------- (a), (b) random activations
SHAPES = {
    "tiny": workloads.WORKLOADS["tiny"],
    "multi": workloads.Workload("multi", 200, 512, 256, 16, 4, "bf16", "normal", 3),
}


def _crafted_x(wl):
    """x of the workload with special rows: outlier channels, +-0, bf16 subnormals, ties."""
    x = workloads.draw_x(wl).float().numpy()
    rng = np.random.default_rng(17)
    for t in range(0, min(wl.T, 12)):
        b = t % (wl.H // 32)
        x[t, 32 * b + (t * 7) % 32] = (2.0 ** (10 + t % 11)) * (1 if t % 2 else -1)
    if wl.T > 13:
        x[12, :32] = 0.0
        x[12, 32:64] = -0.0
        x[13, :8] = [9.2e-41, -9.2e-41, 1.0e-39, 2.0 ** -126, 1.0625, 1.1875, 17.0, 19.0]
    return torch.from_numpy(x).to(torch.bfloat16)


@pytest.mark.parametrize("name", list(SHAPES))
@pytest.mark.parametrize("variant", ["auto", "t128_wide", "t128_weights_on_M", "t16"])
def test_w4a8_activation_operand_bit_exact(name, variant, monkeypatch):
    _set_variant(monkeypatch, variant)
    wl = SHAPES[name]
    inp = helpers.host_inputs(wl)
    layer, out, inter, grows = _forward(wl, inp["x"], inp["logits"], inp, moe_mx.MOE_MX_ACT_MXFP8)
    rows_total = inter["aq"].shape[1]
    codes, scales = _operand(inter, "aq", rows_total, wl.H)
    q_o, s_o = oracle.mx_quantize(inp["x"].float().numpy(), oracle.FMT_E4M3)
    r, t = grows[:, 0], grows[:, 1]
    assert np.array_equal(codes[0][r], q_o[t])
    assert np.array_equal(scales[0][r], s_o[t])
    layer.close()


@pytest.mark.parametrize("name", list(SHAPES))
@pytest.mark.parametrize("variant", ["auto", "t128_wide", "t16"])
def test_w4a16_activation_operand_is_exact_split(name, variant, monkeypatch):
    _set_variant(monkeypatch, variant)
    wl = SHAPES[name]
    inp = helpers.host_inputs(wl)
    x = _crafted_x(wl)
    layer, out, inter, grows = _forward(wl, x, inp["logits"], inp, moe_mx.MOE_MX_ACT_BF16)
    rows_total = inter["aq"].shape[1]
    codes, scales = _operand(inter, "aq", rows_total, wl.H)
    r, t = grows[:, 0], grows[:, 1]
    helpers.check_two_term_split(codes[:, r], scales[:, r], x.float().numpy().astype(np.float64)[t], name)
    # and the layer's output still meets the tolerance against the oracle on this input (row by
    # row: the outlier tokens' outputs are up to 10^6 times the others')
    inp2 = dict(inp, x=x, xb=workloads.bf16_bits(x))
    ref, _, _ = helpers.oracle_forward(inp2, wl.top_k, 0)
    helpers.check_output_rows(out, ref, f"{name} crafted x")
    layer.close()


# ---------------------------------------------------------------- (c), (d) exact special cases
EXACT = workloads.Workload("exact", 200, 512, 256, 16, 4, "bf16", "normal", 21)
E2M1_ONE, E2M1_HALF, E2M1_MHALF, E2M1_MONE = 0x2, 0x1, 0x9, 0xA


def _pack(codes):
    """E2M1 codes [..., K] -> bytes [..., K/2], element 2i in the low nibble."""
    return (codes[..., 0::2] | (codes[..., 1::2] << 4)).astype(np.uint8)


def _exact_weights(case, rng):
    E, H, I = EXACT.E, EXACT.H, EXACT.I
    w1c = np.zeros((E, 2 * I, H), np.uint8)
    lo, hi = (34, 48) if case == "fc1" else (17, 24)
    for e in range(E):
        for i in range(I):
            n = rng.integers(lo, hi + 1)
            w1c[e, i, rng.choice(H, n, replace=False)] = E2M1_ONE                   # gate: n ones
            pos = rng.choice(H, 3, replace=False)
            w1c[e, I + i, pos] = rng.choice([E2M1_HALF, E2M1_ONE, E2M1_MHALF, E2M1_MONE], 3)  # up
    if case == "fc1":
        w1s = rng.choice(np.array([126, 127, 128], np.uint8), size=(E, 2 * I, H // 32))
    else:
        w1s = np.full((E, 2 * I, H // 32), 127, np.uint8)
    w2c = rng.integers(0, 16, size=(E, H, I)).astype(np.uint8)
    w2s = np.full((E, H, I // 32), 127, np.uint8)
    return dict(w1=_pack(w1c), w1s=w1s, w2=_pack(w2c), w2s=w2s)


def _exact_x(case, rng):
    T, H = EXACT.T, EXACT.H
    c = rng.choice([1.0, 2.0], size=(T, 1))
    m = rng.choice([1.0, 2.0], size=(T, H)) if case == "fc1" else np.ones((T, H))
    return torch.from_numpy((c * m).astype(np.float32)).to(torch.bfloat16)


def _per_expert_matmul(a, w, experts):
    """Row i of the result = a[i] @ w[experts[i]].T, float64 (a library matmul per expert)."""
    out = np.zeros((a.shape[0], w.shape[1]), np.float64)
    for ex in np.unique(experts):
        idx = experts == ex
        out[idx] = a[idx] @ w[ex].T
    return out


@pytest.mark.parametrize("case", ["fc1", "fc1_fc2"])
@pytest.mark.parametrize("act", [0, 1], ids=["w4a16", "w4a8"])
@pytest.mark.parametrize("variant", list(VARIANTS))
def test_exact_special_case(case, act, variant, monkeypatch):
    _set_variant(monkeypatch, variant)
    rng = np.random.default_rng(100 + (case == "fc1_fc2"))
    wl = EXACT
    w = _exact_weights(case, rng)
    x = _exact_x(case, rng)
    logits = workloads.draw_logits(wl)
    layer, out, inter, grows = _forward(wl, x, logits, w, act)
    r, t, e, j = grows[:, 0], grows[:, 1], grows[:, 2], grows[:, 3]
    rows_total = inter["aq"].shape[1]
    xf = x.float().numpy().astype(np.float64)
    # FC1's operand: x is exactly representable (w4a16: term 0 alone; w4a8: one code per value)
    acodes, ascales = _operand(inter, "aq", rows_total, wl.H)
    a_dec = helpers.dequant_mxfp8_lib(acodes[0][r], ascales[0][r])
    if act == 0:
        a_dec = a_dec + helpers.dequant_mxfp8_lib(acodes[1][r], ascales[1][r])
    assert np.array_equal(a_dec, xf[t])
    # exact g and u by a float64 matmul of the decoded weights (ml_dtypes), then h = g * u
    w1d = helpers.dequant_mxfp4_lib(w["w1"], w["w1s"])                 # [E, 2I, H]
    gu = _per_expert_matmul(xf[t], w1d, e)                             # [rows, 2I]
    g, u = gu[:, :wl.I], gu[:, wl.I:]
    assert g.min() >= 17.0, "the case needs every gate value >= 17"
    h = (g * u).astype(np.float32)
    assert np.array_equal(h.astype(np.float64), g * u), "g * u must be exact in float32"
    hcodes, hscales = _operand(inter, "hq", rows_total, wl.I)
    if act == 0:
        h_dec = helpers.dequant_mxfp8_lib(hcodes[0][r], hscales[0][r]) + \
            helpers.dequant_mxfp8_lib(hcodes[1][r], hscales[1][r])
        assert np.array_equal(h_dec, helpers.bf16_round(h)), "h operand != bf16(g * u)"
    else:
        q_o, s_o = oracle.mx_quantize(h, oracle.FMT_E4M3)
        assert np.array_equal(hscales[0][r], s_o), "h scale bytes != the oracle's MXFP8 quantisation of g * u"
        assert np.array_equal(hcodes[0][r], q_o), "h codes != the oracle's MXFP8 quantisation of g * u"
        h_dec = helpers.dequant_mxfp8_lib(q_o, s_o)
    # FC2's float32 rows equal the float64 matmul of W2 with the GPU's own h operand (the sums
    # are exact in float32 by construction)
    w2d = helpers.dequant_mxfp4_lib(w["w2"], w["w2s"])                 # [E, H, I]
    y_ref = _per_expert_matmul(h_dec, w2d, e)
    y = inter["y"][r].astype(np.float64)
    assert np.array_equal(y, y_ref), f"FC2 rows differ from the exact matmul: max |d| = {np.abs(y - y_ref).max()}"
    # the combine of those rows, within the tolerance of the exact weighted sum
    w_g = layer.routing(wl.T, wl.top_k)[1].cpu().numpy().astype(np.float64)
    exact_out = np.zeros((wl.T, wl.H))
    np.add.at(exact_out, t, w_g[t, j][:, None] * y_ref)
    helpers.check_output(out, exact_out, f"exact {case} combine")
    if act == 0 and case == "fc1_fc2":
        # here h needs no rounding, so the oracle (whose SwiGLU in double makes h = g * u * (1 - ~e^-g),
        # on the other side of a rounding tie now and then) meets the same values: compare with it too
        inp = dict(xb=workloads.bf16_bits(x), logits=logits, **w)
        ref, _, _ = helpers.oracle_forward(inp, wl.top_k, act)
        helpers.check_output(out, ref, f"exact {case}")
    layer.close()


def test_get_intermediate_rejects_bad_arguments():
    wl = SHAPES["tiny"]
    layer = moe_mx.MoeMxLayer(wl.H, wl.I, wl.E, wl.T, wl.top_k)
    dst = torch.empty(16, dtype=torch.uint8, device="cuda")
    # before any forward there is nothing to copy
    moe_mx.moe_mx_get_intermediate(layer.handle, moe_mx.MOE_MX_INTER_Y, dst)
    with pytest.raises(moe_mx.MoeMxError) as ei:
        moe_mx.moe_mx_get_intermediate(layer.handle, 9, dst)
    assert ei.value.code == moe_mx.MOE_MX_ERR_INVALID_ARG
    layer.close()
