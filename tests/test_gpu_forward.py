"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Inputs are the seeded synthetic workloads; weights are quantised by the
oracle's quantiser.  Routing ids, counts, offsets and the permutation must match
bit-exactly; outputs must meet the layer's tolerance (relative Frobenius error
<= 5e-3 and max |gpu - ref| <= 2e-2 * RMS(ref)).  Shapes here span several
GEMM tiles, ragged row blocks and both MMA orientations (tokens on M, or
weight rows on M with the tokens on N), forced through MOE_MX_SWAP_ROWS.
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


SHAPES = {
    "tiny": workloads.WORKLOADS["tiny"],
    # several n-tiles, K-stages and row blocks; T*k/E ~ 50 rows per expert with a ragged spread
    "multi": workloads.Workload("multi", 200, 512, 256, 16, 4, "bf16", "normal", 3),
    # one expert over many row blocks (ragged tail of 37 rows)
    "single_expert": workloads.Workload("single_expert", 421, 256, 256, 1, 1, "bf16", "none", 5),
}


def _run(wl, act_mode, monkeypatch, swap_rows=None, inp=None):
    if swap_rows is not None:
        monkeypatch.setenv("MOE_MX_SWAP_ROWS", str(swap_rows))
    inp = inp or helpers.host_inputs(wl)
    d = helpers.to_device(inp)
    layer = moe_mx.MoeMxLayer(wl.H, wl.I, wl.E, max(wl.T, 1), wl.top_k)
    out = layer.forward(d["x"], d["logits"], d["w1"], d["w1s"], d["w2"], d["w2s"], wl.top_k, act_mode)
    assert layer.sync_status() == moe_mx.MOE_MX_OK, moe_mx.moe_mx_last_error()
    return layer, inp, out


@pytest.mark.parametrize("name", list(SHAPES))
@pytest.mark.parametrize("act_mode", [0, 1], ids=["w4a16", "w4a8"])
@pytest.mark.parametrize("swap_rows", [0, 128, 64], ids=["tokens_on_M", "weights_on_M", "mixed"])
def test_forward_matches_oracle(name, act_mode, swap_rows, monkeypatch):
    wl = SHAPES[name]
    layer, inp, out = _run(wl, act_mode, monkeypatch, swap_rows)
    helpers.check_routing(layer, wl.T, wl.top_k, wl.E, inp["logits"].numpy())
    ref, _, _ = helpers.oracle_forward(inp, wl.top_k, act_mode)
    helpers.check_output(out, ref, f"{name}/{act_mode}/{swap_rows}")
    layer.close()


def test_forward_is_deterministic(monkeypatch):
    wl = SHAPES["multi"]
    layer, inp, out1 = _run(wl, 0, monkeypatch)
    d = helpers.to_device(inp)
    out2 = layer.forward(d["x"], d["logits"], d["w1"], d["w1s"], d["w2"], d["w2s"], wl.top_k, 0)
    torch.cuda.synchronize()
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    layer.close()


@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (3, 4, 4), (16, 8, 1), (130, 2, 2)])
def test_edge_shapes(T, E, k, monkeypatch):
    wl = workloads.Workload(f"edge{T}_{E}_{k}", T, 256, 128, E, k, "bf16", "none", 7)
    layer, inp, out = _run(wl, 0, monkeypatch)
    helpers.check_routing(layer, T, k, E, inp["logits"].numpy())
    ref, _, _ = helpers.oracle_forward(inp, k, 0)
    helpers.check_output(out, ref, wl.name)
    layer.close()


def test_zero_tokens_is_a_noop():
    wl = SHAPES["tiny"]
    inp = helpers.host_inputs(wl)
    d = helpers.to_device(inp)
    layer = moe_mx.MoeMxLayer(wl.H, wl.I, wl.E, wl.T, wl.top_k)
    out = torch.full((wl.T, wl.H), 7.0, dtype=torch.bfloat16, device="cuda")
    moe_mx.moe_mx_forward(layer.handle, d["x"], d["logits"], 0, d["w1"], d["w1s"], d["w2"], d["w2s"], wl.top_k, 0,
                          out)
    assert layer.sync_status() == moe_mx.MOE_MX_OK
    assert torch.all(out == 7.0)
    layer.close()


def test_tied_logits_route_to_lowest_index(monkeypatch):
    wl = workloads.Workload("ties", 64, 256, 128, 16, 4, "bf16", "none", 11)
    inp = helpers.host_inputs(wl)
    g = torch.Generator().manual_seed(3)
    inp["logits"] = (torch.randint(-2, 2, (wl.T, wl.E), generator=g).float() * 0.5).contiguous()
    layer, inp, out = _run(wl, 0, monkeypatch, inp=inp)
    helpers.check_routing(layer, wl.T, wl.top_k, wl.E, inp["logits"].numpy())
    ref, _, _ = helpers.oracle_forward(inp, wl.top_k, 0)
    helpers.check_output(out, ref, "ties")
    layer.close()


def test_invalid_arguments_are_rejected_before_launch():
    wl = SHAPES["tiny"]
    inp = helpers.host_inputs(wl)
    d = helpers.to_device(inp)
    layer = moe_mx.MoeMxLayer(wl.H, wl.I, wl.E, wl.T, wl.top_k)
    out = torch.empty(wl.T, wl.H, dtype=torch.bfloat16, device="cuda")
    args = [d["x"], d["logits"], wl.T, d["w1"], d["w1s"], d["w2"], d["w2s"], wl.top_k, 0, out]
    bad = [
        (2, wl.T + 1, "num_tokens"),
        (7, wl.E + 1, "top_k"),
        (8, 5, "act_dtype"),
        (0, inp["x"], "device pointer"),            # host tensor
        (9, d["x"], "alias"),                       # out aliases x
        (3, d["w1"][0, 0, 1:], "aligned"),          # misaligned pointer
    ]
    for pos, val, msg in bad:
        a = list(args)
        a[pos] = val
        with pytest.raises(moe_mx.MoeMxError) as ei:
            moe_mx.moe_mx_forward(layer.handle, *a)
        assert ei.value.code == moe_mx.MOE_MX_ERR_INVALID_ARG
        assert msg in str(ei.value)
    assert layer.sync_status() == moe_mx.MOE_MX_OK
    layer.close()


def test_watchdog_reports_timeout_and_context_survives(monkeypatch):
    wl = SHAPES["tiny"]
    layer = moe_mx.MoeMxLayer(wl.H, wl.I, wl.E, wl.T, wl.top_k)
    moe_mx.moe_mx_debug_watchdog(layer.handle, 2000)  # 2 ms wait on a flag nothing sets
    assert layer.sync_status() == moe_mx.MOE_MX_ERR_TIMEOUT
    assert layer.sync_status() == moe_mx.MOE_MX_OK    # the word was cleared
    layer.close()
    # the context is still usable: a full forward afterwards is correct
    layer2, inp, out = _run(wl, 0, monkeypatch)
    ref, _, _ = helpers.oracle_forward(inp, wl.top_k, 0)
    helpers.check_output(out, ref, "after watchdog")
    layer2.close()
