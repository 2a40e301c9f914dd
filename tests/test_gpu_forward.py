"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Inputs are the seeded synthetic workloads; weights are quantised by the
oracle's quantiser.  Routing ids, counts, offsets and the permutation must match
bit-exactly; outputs must meet the layer's tolerance (relative Frobenius error
<= 5e-3 and max |gpu - ref| <= 2e-2 * RMS(ref)).  Shapes here span several
GEMM tiles, ragged row blocks, every kernel variant (activation tiles of 16,
32, 64 or 128 rows per term, forced through MOE_MX_TILE_ROWS: below 128 the
expert segments are split into work blocks of that many rows) and both MMA
orientations of the 128-row variant (tokens on M, or weight rows on M with the
tokens on N), forced through MOE_MX_SWAP_ROWS.
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


def _run(wl, act_mode, monkeypatch, swap_rows=None, inp=None, tile_rows=None, wide=None):
    if swap_rows is not None:
        monkeypatch.setenv("MOE_MX_SWAP_ROWS", str(swap_rows))
    if tile_rows is not None:
        monkeypatch.setenv("MOE_MX_TILE_ROWS", str(tile_rows))
    if wide is not None:
        monkeypatch.setenv("MOE_MX_WIDE", str(wide))
    inp = inp or helpers.host_inputs(wl)
    d = helpers.to_device(inp)
    layer = moe_mx.MoeMxLayer(wl.H, wl.I, wl.E, max(wl.T, 1), wl.top_k)
    out = layer.forward(d["x"], d["logits"], d["w1"], d["w1s"], d["w2"], d["w2s"], wl.top_k, act_mode)
    assert layer.sync_status() == moe_mx.MOE_MX_OK, moe_mx.moe_mx_last_error()
    return layer, inp, out


# (tile rows, swap rows, wide): the 128-row blocks on the wide two-tile variant (tokens always on
# M, whatever the swap setting) and on the one-tile variant in both orientations and mixed, each
# smaller variant (always tokens on N), and the automatic choice by token count
VARIANTS = {
    "t128_wide": (128, 0, None), "t128_wide_swaprows": (128, 128, None),
    "t128_tokens_on_M": (128, 0, 0), "t128_weights_on_M": (128, 128, 0), "t128_mixed": (128, 64, 0),
    "t64": (64, None, None), "t32": (32, None, None), "t16": (16, None, None), "auto": (None, None, None),
}


@pytest.mark.parametrize("name", list(SHAPES))
@pytest.mark.parametrize("act_mode", [0, 1], ids=["w4a16", "w4a8"])
@pytest.mark.parametrize("variant", list(VARIANTS))
def test_forward_matches_oracle(name, act_mode, variant, monkeypatch):
    wl = SHAPES[name]
    tile_rows, swap_rows, wide = VARIANTS[variant]
    layer, inp, out = _run(wl, act_mode, monkeypatch, swap_rows, tile_rows=tile_rows, wide=wide)
    helpers.check_routing(layer, wl.T, wl.top_k, wl.E, inp["logits"].numpy())
    ref, _, _ = helpers.oracle_forward(inp, wl.top_k, act_mode)
    helpers.check_output(out, ref, f"{name}/{act_mode}/{variant}")
    layer.close()


@pytest.mark.parametrize("name", ["multi", "single_expert"])
@pytest.mark.parametrize("act_mode", [0, 1], ids=["w4a16", "w4a8"])
@pytest.mark.parametrize("variant", list(VARIANTS))
def test_tiled_scales_match_row_major(name, act_mode, variant, monkeypatch):
    """The tiled weight-scale layout (moe_mx_prepare_scales) gives bit-identical outputs."""
    wl = SHAPES[name]
    tile_rows, swap_rows, wide = VARIANTS[variant]
    layer, inp, out_rm = _run(wl, act_mode, monkeypatch, swap_rows, tile_rows=tile_rows, wide=wide)
    d = helpers.to_device(inp)
    t1, t2 = layer.prepare_scales(d["w1s"], d["w2s"])
    out_t = layer.forward(d["x"], d["logits"], d["w1"], t1, d["w2"], t2, wl.top_k, act_mode)
    assert layer.sync_status() == moe_mx.MOE_MX_OK, moe_mx.moe_mx_last_error()
    assert torch.equal(out_t.view(torch.int16), out_rm.view(torch.int16))
    layer.close()


def test_prepare_scales_rejects_bad_arguments():
    wl = SHAPES["tiny"]
    layer = moe_mx.MoeMxLayer(wl.H, wl.I, wl.E, wl.T, wl.top_k)
    src = torch.zeros(wl.E, 2 * wl.I, wl.H // 32, dtype=torch.uint8, device="cuda")
    with pytest.raises(moe_mx.MoeMxError):
        moe_mx.moe_mx_prepare_scales(layer.handle, 7, src, torch.empty_like(src))
    with pytest.raises(moe_mx.MoeMxError):
        moe_mx.moe_mx_prepare_scales(layer.handle, moe_mx.MOE_MX_W1, src, src)  # overlapping
    with pytest.raises(moe_mx.MoeMxError):
        moe_mx.moe_mx_set_scale_layout(layer.handle, 5)
    layer.close()


def test_forward_is_deterministic(monkeypatch):
    wl = SHAPES["multi"]
    layer, inp, out1 = _run(wl, 0, monkeypatch)
    d = helpers.to_device(inp)
    out2 = layer.forward(d["x"], d["logits"], d["w1"], d["w1s"], d["w2"], d["w2s"], wl.top_k, 0)
    torch.cuda.synchronize()
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    layer.close()


# ... including expert counts that take each top-k width (8, 16 and 32 candidates per lane) on
# both routing paths (one CTA up to 256 tokens, three kernels beyond)
@pytest.mark.parametrize("T,E,k", [(1, 8, 2), (3, 4, 4), (16, 8, 1), (130, 2, 2), (20, 1000, 4), (300, 600, 8),
                                   (257, 300, 6), (40, 384, 8), (1, 384, 8), (2, 384, 8), (4, 384, 8), (8, 384, 8)])
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


@pytest.mark.parametrize("name", ["tiny", "multi"])
@pytest.mark.parametrize("act_mode", [0, 1], ids=["w4a16", "w4a8"])
def test_dependent_launch_gives_same_bits(name, act_mode, monkeypatch):
    """Kernels launched as programmatic dependents (the default) and one after another
    (MOE_MX_PDL=0) give bit-identical routing and outputs."""
    wl = SHAPES[name]
    inp = helpers.host_inputs(wl)
    outs = []
    for pdl in ("1", "0"):
        monkeypatch.setenv("MOE_MX_PDL", pdl)
        layer, _, out = _run(wl, act_mode, monkeypatch, inp=inp)
        outs.append((out.clone(), [a.clone() for a in layer.routing(wl.T, wl.top_k)]))
        layer.close()
    assert torch.equal(outs[0][0].view(torch.int16), outs[1][0].view(torch.int16))
    for a, b in zip(outs[0][1], outs[1][1]):
        assert torch.equal(a, b)



# up to 16 tokens the activation scales also go through the N layout (one bulk copy per GEMM stage)
N_LAYOUT_SHAPES = {
    "tiny": workloads.WORKLOADS["tiny"],
    "t16_e64": workloads.Workload("t16_e64", 16, 512, 256, 64, 8, "bf16", "none", 7),
    "t4_e64": workloads.Workload("t4_e64", 4, 512, 256, 64, 8, "bf16", "none", 8),
    "t1_e64": workloads.Workload("t1_e64", 1, 512, 256, 64, 8, "bf16", "none", 9),  # one launch, two phases
}


@pytest.mark.parametrize("name", list(N_LAYOUT_SHAPES))
@pytest.mark.parametrize("act_mode", [0, 1], ids=["w4a16", "w4a8"])
def test_n_layout_scales_give_same_bits(name, act_mode, monkeypatch):
    """The activation scales taken from the N layout (the default up to 16 tokens) and through
    4-byte copies from the row-block atoms (MOE_MX_SCALES_N=0) give bit-identical outputs."""
    wl = N_LAYOUT_SHAPES[name]
    inp = helpers.host_inputs(wl)
    outs = []
    for sn in ("1", "0"):
        monkeypatch.setenv("MOE_MX_SCALES_N", sn)
        layer, _, out = _run(wl, act_mode, monkeypatch, inp=inp)
        outs.append(out.clone())
        layer.close()
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))
    ref, _, _ = helpers.oracle_forward(inp, wl.top_k, act_mode)
    helpers.check_output(outs[0], ref, f"{name} N-layout scales")


def test_router_matches_hand_derived_cases():
    """The router on the hand-derived cases of tests/golden/routing_cases.txt (ties, -0 / +0, NaN
    and -inf logits, k = E), each padded to 8 experts with -inf logits and run as one token of a
    batch: ids as written, weights within 2e-6."""
    from tests.test_oracle_routing import _golden_routing_cases
    cases = _golden_routing_cases()
    E, T = 8, len(cases)
    k = max(c[0] for c in cases)
    layer = moe_mx.MoeMxLayer(256, 128, E, T, k)
    x = torch.zeros(T, 256, dtype=torch.bfloat16, device="cuda")
    w1 = torch.zeros(E, 256, 128, dtype=torch.uint8, device="cuda")
    w1s = torch.full((E, 256, 8), 127, dtype=torch.uint8, device="cuda")
    w2 = torch.zeros(E, 256, 64, dtype=torch.uint8, device="cuda")
    w2s = torch.full((E, 256, 4), 127, dtype=torch.uint8, device="cuda")
    for kk in sorted({c[0] for c in cases}):
        rows = [i for i, c in enumerate(cases) if c[0] == kk]
        lg = torch.full((len(rows), E), float("-inf"), dtype=torch.float32)
        for r, i in enumerate(rows):
            lg[r, :len(cases[i][1])] = torch.tensor(cases[i][1], dtype=torch.float32)
        layer.forward(x[:len(rows)], lg.cuda(), w1, w1s, w2, w2s, kk)
        assert layer.sync_status() == moe_mx.MOE_MX_OK, moe_mx.moe_mx_last_error()
        ids, w = [a.cpu().numpy() for a in layer.routing(len(rows), kk)[:2]]
        for r, i in enumerate(rows):
            assert ids[r].tolist() == cases[i][2], (cases[i], ids[r])
            np.testing.assert_allclose(w[r], cases[i][3], rtol=2e-6, atol=1e-7)
    layer.close()


@pytest.mark.parametrize("name", ["tiny", "multi"])
@pytest.mark.parametrize("act_mode", [0, 1], ids=["w4a16", "w4a8"])
@pytest.mark.parametrize("variant", ["auto", "t16", "t32", "t64"])
def test_fused_combine_gives_same_bits(name, act_mode, variant, monkeypatch):
    """Up to 512 tokens (every FC2 unit with its tokens on N) the combine may run in FC2's epilogue
    (MOE_MX_FUSE_COMBINE=1; off by default, it measured slower); it must give exactly the bits of
    the separate combine kernel, on two forwards in a row (its per-token counters must be back at
    zero after each)."""
    wl = SHAPES[name]
    tile_rows = VARIANTS[variant][0]
    inp = helpers.host_inputs(wl)
    outs = []
    for fuse in ("1", "0"):
        monkeypatch.setenv("MOE_MX_FUSE_COMBINE", fuse)
        layer, _, out = _run(wl, act_mode, monkeypatch, inp=inp, tile_rows=tile_rows)
        d = helpers.to_device(inp)
        out2 = layer.forward(d["x"], d["logits"], d["w1"], d["w1s"], d["w2"], d["w2s"], wl.top_k, act_mode)
        assert layer.sync_status() == moe_mx.MOE_MX_OK, moe_mx.moe_mx_last_error()
        assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
        outs.append(out)
        layer.close()
    assert torch.equal(outs[0].view(torch.int16), outs[1].view(torch.int16))


@pytest.mark.parametrize("T,E,k", [(1, 16, 4), (3, 384, 8), (16, 40, 8), (16, 8, 2)])
@pytest.mark.parametrize("act_mode", [0, 1], ids=["w4a16", "w4a8"])
def test_two_phase_launch_matches_oracle(T, E, k, act_mode, monkeypatch):
    """FC1 and FC2 as one launch (FC2's units wait for their row block's FC1 units; by default up to
    2 tokens, here forced up to 16) and as two launches (MOE_MX_TWO_PHASE=0).  Both meet the oracle's tolerance, the
    routing is bit-exact, and two forwards in a row give the same bits (the per-row-block counts
    start from zero every forward).  I = 128 makes FC2 a single K stage per unit."""
    for I in (256, 128):
        wl = workloads.Workload(f"two_phase{T}_{E}_{k}_{I}", T, 512, I, E, k, "bf16", "normal", 13)
        inp = helpers.host_inputs(wl)
        ref, _, _ = helpers.oracle_forward(inp, k, act_mode)
        monkeypatch.setenv("MOE_MX_TWO_PHASE_TOKENS", "16")   # every T here through the one launch
        for two in ("1", "0"):
            monkeypatch.setenv("MOE_MX_TWO_PHASE", two)
            layer, _, out = _run(wl, act_mode, monkeypatch, inp=inp)
            helpers.check_routing(layer, T, k, E, inp["logits"].numpy())
            helpers.check_output(out, ref, f"{wl.name} two_phase={two}")
            d = helpers.to_device(inp)
            out2 = layer.forward(d["x"], d["logits"], d["w1"], d["w1s"], d["w2"], d["w2s"], k, act_mode)
            assert layer.sync_status() == moe_mx.MOE_MX_OK, moe_mx.moe_mx_last_error()
            assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
            layer.close()
