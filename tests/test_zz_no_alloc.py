"""moe_mx_route_group_noalloc: routing + grouping with no handle and no allocation.

Its results must equal those of the existing path (moe_mx_forward followed by
moe_mx_get_routing on a handle) for the same logits: expert ids, counts, padded
offsets and the grouped permutation bit for bit, weights within the routing
tolerance used everywhere (rtol 2e-6).  Two calls in a row with different
token counts and logits check that the shared static scratch carries nothing
from one call into the next.  The file is collected last so that it also runs
after every other test in one process.
"""
import numpy as np
import pytest
import torch

from block_scaled_moe_softmax_b200 import moe_mx

pytestmark = pytest.mark.gpu

H, I, E, K = 128, 128, 384, 8


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _logits(T, seed):
    g = torch.Generator().manual_seed(seed)
    lg = torch.randn(T, E, generator=g, dtype=torch.float32)
    lg[::7, 5] = lg[::7, 9]          # exact ties: the lower index must win
    lg[3, :] = 0.0                    # a row of all-equal logits
    return lg


def _weights():
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


def _via_noalloc(logits, rows):
    T = logits.shape[0]
    lg = logits.cuda()
    # caller buffers filled with a pattern, so a value the call fails to write shows
    ids = torch.full((T, K), 0x7B7B7B7B, dtype=torch.int32, device="cuda")
    w = torch.full((T, K), -3.0, dtype=torch.float32, device="cuda")
    counts = torch.full((E,), 0x7B7B7B7B, dtype=torch.int32, device="cuda")
    pad = torch.full((E + 1,), 0x7B7B7B7B, dtype=torch.int32, device="cuda")
    sp = torch.full((rows,), 0x7B7B7B7B, dtype=torch.int32, device="cuda")
    pos = torch.full((T * K,), 0x7B7B7B7B, dtype=torch.int32, device="cuda")
    moe_mx.moe_mx_route_group_noalloc(lg, T, E, K, ids, w, counts, pad, sp, pos)
    torch.cuda.synchronize()
    return [a.cpu().numpy() for a in (ids, w, counts, pad, sp, pos)]


def _compare(ref, got, T):
    ids_r, w_r, counts_r, pad_r, sp_r = ref
    ids_g, w_g, counts_g, pad_g, sp_g, pos_g = got
    assert np.array_equal(ids_g, ids_r)
    np.testing.assert_allclose(w_g, w_r, rtol=2e-6, atol=0)
    assert np.array_equal(counts_g, counts_r)
    assert np.array_equal(pad_g, pad_r)
    n = int(pad_r[E])
    assert np.array_equal(sp_g[:n], sp_r[:n])
    # pos_of_pair is the inverse of the permutation on the pairs
    assert np.array_equal(sp_g[pos_g], np.arange(T * K, dtype=np.int32))


def test_noalloc_routing_matches_forward_two_calls_in_a_row():
    weights = _weights()
    layer = moe_mx.MoeMxLayer(H, I, E, 300, K)
    try:
        for T, seed in ((300, 11), (77, 12)):   # a large call, then a smaller one over the same scratch
            logits = _logits(T, seed)
            ref = _via_handle(layer, weights, logits)
            rows = moe_mx.moe_mx_max_grouped_rows(layer.handle, T, K)
            got = _via_noalloc(logits, rows)
            _compare(ref, got, T)
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
    moe_mx.moe_mx_route_group_noalloc(smallf, 0, E, K, small, smallf, small, small, small, small)
