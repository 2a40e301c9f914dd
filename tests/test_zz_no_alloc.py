"""moe_mx_route_group_noalloc: routing + grouping with no handle and no allocation.

Its results must equal the oracle's routing and grouping (expert ids, counts,
padded offsets and the grouped permutation bit for bit, weights within the
routing tolerance used everywhere, rtol 2e-6) and those of the existing path
(moe_mx_forward followed by moe_mx_get_routing on a handle) for the same
logits.  The cases cover both routing kernel paths: up to 64 tokens one CTA
routes and groups (T = 1, 16, 64), beyond that three kernels do (T = 77, 300).
Calls follow one another with different token counts, expert counts and
logits, so that the shared static scratch is seen to carry nothing from one
call into the next.  The file is collected last so that it also runs after
every other test in one process.
"""
import numpy as np
import pytest
import torch

import oracle
from block_scaled_moe_softmax_b200 import moe_mx

pytestmark = pytest.mark.gpu

H, I, K = 128, 128, 8
BM = 128


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _logits(T, E, seed):
    g = torch.Generator().manual_seed(seed)
    lg = torch.randn(T, E, generator=g, dtype=torch.float32)
    lo, hi = (5, 9) if E > 9 else (1, 6)
    lg[::7, lo] = lg[::7, hi]        # exact ties: the lower index must win
    if T > 3:
        lg[3, :] = 0.0               # a row of all-equal logits
    return lg


def _weights(E):
    g = torch.Generator(device="cuda").manual_seed(7)
    w1f = torch.randn(E, 2 * I, H, generator=g, device="cuda") * 0.02
    w2f = torch.randn(E, H, I, generator=g, device="cuda") * 0.02
    w1, w1s = moe_mx.quantize_mx(w1f, moe_mx.MOE_MX_FMT_MXFP4)
    w2, w2s = moe_mx.quantize_mx(w2f, moe_mx.MOE_MX_FMT_MXFP4)
    return w1, w1s, w2, w2s


def _via_handle(layer, weights, logits):
    T = logits.shape[0]
    x = torch.randn(T, H, dtype=torch.float32).to(torch.bfloat16).cuda()
    layer.forward(x, logits.cuda(), *weights, K)
    assert layer.sync_status() == moe_mx.MOE_MX_OK, moe_mx.moe_mx_last_error()
    return [a.cpu().numpy() for a in layer.routing(T, K)]


def _rows(T, E):
    P = T * K
    return (P + min(P, E) * (BM - 1) + BM - 1) // BM * BM


def _via_noalloc(logits):
    T, E = logits.shape
    lg = logits.cuda()
    # caller buffers filled with a pattern, so a value the call fails to write shows
    ids = torch.full((T, K), 0x7B7B7B7B, dtype=torch.int32, device="cuda")
    w = torch.full((T, K), -3.0, dtype=torch.float32, device="cuda")
    counts = torch.full((E,), 0x7B7B7B7B, dtype=torch.int32, device="cuda")
    pad = torch.full((E + 1,), 0x7B7B7B7B, dtype=torch.int32, device="cuda")
    sp = torch.full((_rows(T, E),), 0x7B7B7B7B, dtype=torch.int32, device="cuda")
    pos = torch.full((T * K,), 0x7B7B7B7B, dtype=torch.int32, device="cuda")
    moe_mx.moe_mx_route_group_noalloc(lg, T, E, K, ids, w, counts, pad, sp, pos)
    torch.cuda.synchronize()
    return [a.cpu().numpy() for a in (ids, w, counts, pad, sp, pos)]


def _check_against_oracle(got, logits):
    T, E = logits.shape
    ids_g, w_g, counts_g, pad_g, sp_g, pos_g = got
    ids_o, w_o = oracle.route(logits.numpy(), K)
    assert np.array_equal(ids_g, ids_o)
    np.testing.assert_allclose(w_g, w_o, rtol=2e-6, atol=0)
    counts_o, offs_o, sp_o = oracle.group(ids_o, E)
    assert np.array_equal(counts_g, counts_o)
    pad_o = np.concatenate([[0], np.cumsum((counts_o + BM - 1) // BM * BM)]).astype(np.int32)
    assert np.array_equal(pad_g, pad_o)
    for e in range(E):
        seg = sp_g[pad_o[e]:pad_o[e + 1]]
        assert np.array_equal(seg[:counts_o[e]], sp_o[offs_o[e]:offs_o[e + 1]]), f"permutation differs at {e}"
        assert np.all(seg[counts_o[e]:] == -1), f"padding rows of expert {e} are not marked -1"
    # pos_of_pair is the inverse of the permutation on the pairs
    assert np.array_equal(sp_g[pos_g], np.arange(T * K, dtype=np.int32))


def _check_against_handle(ref, got):
    ids_r, w_r, counts_r, pad_r, sp_r = ref
    ids_g, w_g, counts_g, pad_g, sp_g, pos_g = got
    assert np.array_equal(ids_g, ids_r)
    assert np.array_equal(w_g.view(np.int32), w_r.view(np.int32))   # the same kernels: the same bits
    assert np.array_equal(counts_g, counts_r)
    assert np.array_equal(pad_g, pad_r)
    n = int(pad_r[-1])
    assert np.array_equal(sp_g[:n], sp_r[:n])


@pytest.mark.parametrize("E", [384, 8])
def test_noalloc_routing_matches_oracle_and_forward_calls_in_a_row(E):
    weights = _weights(E)
    layer = moe_mx.MoeMxLayer(H, I, E, 300, K)
    try:
        # one CTA up to 64 tokens (T = 1, 16, 64), three kernels beyond (T = 300, 77): large and
        # small calls alternate over the same scratch
        for T, seed in ((300, 11), (16, 12), (1, 13), (77, 14), (64, 15)):
            logits = _logits(T, E, seed)
            got = _via_noalloc(logits)
            _check_against_oracle(got, logits)
            _check_against_handle(_via_handle(layer, weights, logits), got)
    finally:
        layer.close()


def test_noalloc_rejects_shapes_beyond_its_scratch():
    small = torch.zeros(64, dtype=torch.int32, device="cuda")
    smallf = torch.zeros(64, dtype=torch.float32, device="cuda")
    with pytest.raises(moe_mx.MoeMxError) as ei:
        # 65536 tokens x 1024 experts needs 4 MiB of histograms: rejected on the host, nothing launched
        moe_mx.moe_mx_route_group_noalloc(smallf, 65536, 1024, 8, small, smallf, small, small, small, small)
    assert ei.value.code == moe_mx.MOE_MX_ERR_UNSUPPORTED
    assert "scratch" in str(ei.value)
    # zero tokens is a no-op
    moe_mx.moe_mx_route_group_noalloc(smallf, 0, 384, K, small, smallf, small, small, small, small)
