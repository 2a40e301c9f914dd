"""GPU parity of the shared expert (moe_mx_create_ex with num_shared > 0) against the oracle.

The shared expert -- a SwiGLU MLP of intermediate size S*I added to every token with
weight 1 in the combine (mxfp6-sm120 package description, routed-MoE path: "shared-expert
combine and routed/shared reduction") -- is held as S extra expert slots of the weights.
Checked through the C ABI: each token's slots (its routed top-k, then the shared chunks
with weight 1), the counts and the grouped permutation over all expert slots bit-exact
against the oracle; outputs within the layer's tolerance (relative Frobenius <= 5e-3,
max err <= 2e-2 RMS) of the oracle's exact output; both activation modes, both routing
kernel paths; and the full decode shape with one shared expert, routing bit-exact for
every token and sampled outputs against the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from block_scaled_moe_softmax_b200 import moe_mx, workloads
from tests import helpers

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _check_routing(layer, T, k, wl, logits_np):
    ids_g, w_g, counts_g, pad_g, sp_g = [a.cpu().numpy() for a in layer.routing(T, k)]
    ids_r, w_r = oracle.route(logits_np, k)
    S = wl.shared
    assert np.array_equal(ids_g[:, :k], ids_r)
    np.testing.assert_allclose(w_g[:, :k], w_r, rtol=2e-6, atol=0)
    assert np.all(ids_g[:, k:] == np.arange(wl.E, wl.E + S)) and np.all(w_g[:, k:] == 1.0)
    counts_o, offs_o, sp_o = oracle.group(ids_g, wl.slots)  # the oracle's stable grouping of all slots
    assert np.array_equal(counts_g, counts_o)
    pad_o = np.concatenate([[0], np.cumsum((counts_o + 127) // 128 * 128)]).astype(np.int32)
    assert np.array_equal(pad_g, pad_o)
    for e in range(wl.slots):
        seg = sp_g[pad_o[e]:pad_o[e + 1]]
        assert np.array_equal(seg[:counts_o[e]], sp_o[offs_o[e]:offs_o[e + 1]])
        assert np.all(seg[counts_o[e]:] == -1)


@pytest.mark.parametrize("T", [1, 12, 200])
@pytest.mark.parametrize("S", [1, 2])
@pytest.mark.parametrize("act", [0, 1], ids=["w4a16", "w4a8"])
def test_shared_expert_matches_oracle(T, S, act):
    wl = workloads.Workload("shared", T, 256, 128, 8, 2, "bf16", "normal", 4, shared=S)
    inp = helpers.host_inputs(wl)
    d = helpers.to_device(inp)
    layer = moe_mx.MoeMxLayer(wl.H, wl.I, wl.E, wl.T, wl.top_k, num_shared=S)
    out = layer.forward(d["x"], d["logits"], d["w1"], d["w1s"], d["w2"], d["w2s"], wl.top_k, act)
    assert layer.sync_status() == moe_mx.MOE_MX_OK, moe_mx.moe_mx_last_error()
    _check_routing(layer, T, wl.top_k, wl, inp["logits"].numpy())
    ref, ids_o, _ = helpers.oracle_forward(inp, wl.top_k, act)
    assert ids_o.shape == (T, wl.top_k + S)
    helpers.check_output(out, ref, f"shared T={T} S={S} act={act}")
    layer.close()


def test_routed_form_rejects_a_shared_expert():
    layer = moe_mx.MoeMxLayer(256, 128, 8, 4, 2, num_shared=1)
    z = torch.zeros(4, 256, dtype=torch.bfloat16, device="cuda")
    ids = torch.zeros(4, 2, dtype=torch.int32, device="cuda")
    w = torch.zeros(4, 2, dtype=torch.float32, device="cuda")
    wt = torch.zeros(9 * 256 * 128, dtype=torch.uint8, device="cuda")
    with pytest.raises(moe_mx.MoeMxError) as e:
        layer.forward_routed(z, ids, w, wt, wt, wt, wt)
    assert e.value.code == moe_mx.MOE_MX_ERR_UNSUPPORTED
    layer.close()


@pytest.mark.slow
def test_decode_with_shared_expert_full_size():
    wl = workloads.WORKLOADS["decode_shared"]
    E, H, I = wl.slots, wl.H, wl.I
    dev = {n: torch.empty(shape, dtype=torch.uint8, device="cuda") for n, shape in
           (("w1", (E, 2 * I, H // 2)), ("w1s", (E, 2 * I, H // 32)), ("w2", (E, H, I // 2)), ("w2s", (E, H, I // 32)))}
    for e in range(E):  # the library's quantiser (bit-exact with the oracle's: test_gpu_fullsize, test_gpu_quant)
        moe_mx.moe_mx_quantize(workloads.draw_w1_expert(wl, e, "cuda"), 2 * I, H, moe_mx.MOE_MX_FMT_MXFP4,
                               dev["w1"][e], dev["w1s"][e])
        moe_mx.moe_mx_quantize(workloads.draw_w2_expert(wl, e, "cuda"), H, I, moe_mx.MOE_MX_FMT_MXFP4,
                               dev["w2"][e], dev["w2s"][e])
    x = workloads.draw_x(wl)
    logits = workloads.draw_logits(wl)
    layer = moe_mx.MoeMxLayer(wl.H, wl.I, wl.E, wl.T, wl.top_k, num_shared=wl.shared)
    out = layer.forward(x.cuda(), logits.cuda(), dev["w1"], dev["w1s"], dev["w2"], dev["w2s"], wl.top_k, 0)
    assert layer.sync_status() == moe_mx.MOE_MX_OK, moe_mx.moe_mx_last_error()
    _check_routing(layer, wl.T, wl.top_k, wl, logits.numpy())
    host = {n: v.cpu().numpy() for n, v in dev.items()}
    toks = [0, 5, wl.T - 1]
    inp = dict(xb=workloads.bf16_bits(x), logits=logits, **host)
    ref, _, _ = helpers.oracle_forward(inp, wl.top_k, 0, tokens=toks)
    helpers.check_output(out[toks], ref, "decode + shared expert, sampled tokens")
    layer.close()
