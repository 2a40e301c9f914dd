"""GPU parity at the full workload sizes (the shapes and launch configuration bench.py times).

For each workload: the whole forward runs on the GPU for all T tokens; routing
ids, per-expert counts, padded offsets and the permutation are compared with
the oracle for EVERY token (bit-exact); the output is compared with the oracle's
per-token evaluation on a sample of tokens (the oracle is too slow for all of
them): the first and last tokens, tokens routed to the most- and least-loaded
experts, seeded random ones, and tokens covering the last, partial work block
of every expert segment whose rows are not a whole number of work blocks.  Tolerance as everywhere: relative Frobenius
error <= 5e-3 and max |gpu - ref| <= 2e-2 * RMS(ref) over the sampled rows.

Weights are drawn per expert on the GPU (float32, N(0, 0.02)), copied to the
host and quantised by the ORACLE's quantiser; the library's GPU quantiser is
run on the same float32 tensors and must agree bit-exactly (a full-size pin of
moe_mx_quantize).  The decode, batched-decode and prefill workloads share one
weight set (same H, I, E and seed).  Each workload is also run with the weight
scales in the tiled layout (moe_mx_prepare_scales) and must give the same bits.
"""
import numpy as np
import pytest
import torch

import oracle
from block_scaled_moe_softmax_b200 import moe_mx, workloads
from tests import helpers

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

_WEIGHT_CACHE = {}


@pytest.fixture(autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def _weights(wl):
    key = (wl.H, wl.I, wl.E, wl.seed)
    if key in _WEIGHT_CACHE:
        return _WEIGHT_CACHE[key]
    _WEIGHT_CACHE.clear()
    torch.cuda.empty_cache()
    E, H, I = wl.E, wl.H, wl.I
    host = dict(w1=np.empty((E, 2 * I, H // 2), np.uint8), w1s=np.empty((E, 2 * I, H // 32), np.uint8),
                w2=np.empty((E, H, I // 2), np.uint8), w2s=np.empty((E, H, I // 32), np.uint8))
    dev = {k: torch.empty(v.shape, dtype=torch.uint8, device="cuda") for k, v in host.items()}
    mismatched = 0
    for e in range(E):
        for name, draw, K in (("w1", workloads.draw_w1_expert, H), ("w2", workloads.draw_w2_expert, I)):
            f = draw(wl, e, device="cuda")
            c, s = oracle.mx_quantize(f.cpu().numpy(), oracle.FMT_E2M1)
            host[name][e], host[name + "s"][e] = c, s
            gc, gs = moe_mx.quantize_mx(f, moe_mx.MOE_MX_FMT_MXFP4)
            dev[name][e].copy_(torch.from_numpy(c))
            dev[name + "s"][e].copy_(torch.from_numpy(s))
            mismatched += int((gc.cpu().numpy() != c).sum()) + int((gs.cpu().numpy() != s).sum())
    torch.cuda.synchronize()
    _WEIGHT_CACHE[key] = (host, dev, mismatched)
    return _WEIGHT_CACHE[key]


def _work_block_rows(T):
    """Rows per GEMM work block the library picks for T tokens (16 up to 256 tokens, 32 up to 512,
    then whole 128-row segments)."""
    return 16 if T <= 256 else 32 if T <= 512 else 128


def _sample_tokens(ids, wl, n_random=8):
    """First and last tokens, tokens of the most and least loaded experts, seeded random ones, and
    a cover of every ragged segment tail: for each expert whose row count is not a multiple of the
    work-block rows, at least one token whose row lies in that segment's last, partial work block
    (chosen greedily, the token covering most uncovered tails first)."""
    T = wl.T
    counts = np.bincount(ids.reshape(-1), minlength=wl.E)
    hit = np.nonzero(counts)[0]
    big = hit[np.argmax(counts[hit])]
    small = hit[np.argmin(counts[hit])]
    toks = {0, T - 1}
    toks.add(int(np.nonzero((ids == big).any(axis=1))[0][0]))
    toks.add(int(np.nonzero((ids == small).any(axis=1))[0][-1]))
    rng = np.random.default_rng(1234)
    toks.update(int(t) for t in rng.choice(T, size=min(n_random, T), replace=False))
    split = _work_block_rows(T)
    tails = {}  # ragged expert -> tokens whose rows sit in its last, partial work block
    for e in hit:
        if counts[e] % split == 0:
            continue
        members = np.nonzero((ids == e).any(axis=1))[0]   # ascending token = ascending grouped row
        tails[int(e)] = set(int(t) for t in members[(counts[e] // split) * split:])
    uncovered = {e for e, ts in tails.items() if not (ts & toks)}
    while uncovered:
        score = {}
        for e in uncovered:
            for t in tails[e]:
                score[t] = score.get(t, 0) + 1
        best = max(sorted(score), key=lambda t: score[t])
        toks.add(best)
        uncovered = {e for e in uncovered if best not in tails[e]}
    return sorted(toks)


@pytest.mark.parametrize("name", ["decode", "batched_decode", "prefill", "prefill_w4a8"])
def test_full_size_forward(name):
    wl = workloads.WORKLOADS[name]
    host, dev, mismatched = _weights(wl)
    assert mismatched == 0, "GPU MX quantiser disagrees with the oracle's at full size"
    x = workloads.draw_x(wl)
    logits = workloads.draw_logits(wl)
    act = moe_mx.MOE_MX_ACT_MXFP8 if wl.act == "mxfp8" else moe_mx.MOE_MX_ACT_BF16
    layer = moe_mx.MoeMxLayer(wl.H, wl.I, wl.E, wl.T, wl.top_k)
    out = layer.forward(x.cuda(), logits.cuda(), dev["w1"], dev["w1s"], dev["w2"], dev["w2s"], wl.top_k, act)
    assert layer.sync_status() == moe_mx.MOE_MX_OK, moe_mx.moe_mx_last_error()
    ids = helpers.check_routing(layer, wl.T, wl.top_k, wl.E, logits.numpy())
    toks = _sample_tokens(ids, wl)
    inp = dict(xb=workloads.bf16_bits(x), logits=logits, **host)
    ref, ids_o, _ = helpers.oracle_forward(inp, wl.top_k, act, tokens=toks)
    assert np.array_equal(ids_o, ids[toks])
    helpers.check_output(out[toks], ref, f"{name} sampled tokens {toks}")
    # the tiled weight-scale layout (the one bench.py times) gives the same bits for all tokens
    t1, t2 = layer.prepare_scales(dev["w1s"], dev["w2s"])
    out_t = layer.forward(x.cuda(), logits.cuda(), dev["w1"], t1, dev["w2"], t2, wl.top_k, act)
    assert layer.sync_status() == moe_mx.MOE_MX_OK, moe_mx.moe_mx_last_error()
    assert torch.equal(out_t.view(torch.int16), out.view(torch.int16))
    layer.close()
