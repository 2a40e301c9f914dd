"""Pins for the oracle's top-k softmax routing and expert grouping (CPU only).

Routing follows "softmax, then top-k with the lowest expert index winning
ties, weights renormalised to sum to 1" (TokenSpeed-kernel README, "Public
API" -- moe_route; fusedtok package description, "Operators" and "API
stability").  The pins: library routines (torch.topk / torch.softmax on
tie-free rows, numpy's stable argsort), invariants, brute force on ties and
the k = E special case.
"""
import os

import numpy as np
import pytest
import torch

import oracle
from block_scaled_moe_softmax_b200 import workloads


@pytest.mark.parametrize("E,k", [(8, 2), (64, 8), (384, 8), (128, 8), (896, 16), (5, 5)])
def test_route_matches_torch_on_tie_free_rows(E, k):
    g = torch.Generator().manual_seed(E * 31 + k)
    logits = torch.randn(64, E, generator=g, dtype=torch.float32)
    ids, w = oracle.route(logits.numpy(), k)
    tv, ti = torch.topk(logits.double(), k, dim=1, largest=True, sorted=True)
    assert np.array_equal(ids, ti.numpy().astype(np.int32))
    probs = torch.softmax(logits.double(), dim=1)
    sel = torch.gather(probs, 1, ti)
    want = (sel / sel.sum(dim=1, keepdim=True)).numpy()
    np.testing.assert_allclose(w, want, rtol=1e-6, atol=0)
    # softmax over the selected logits only is the same thing
    want2 = torch.softmax(tv, dim=1).numpy()
    np.testing.assert_allclose(w, want2, rtol=1e-6, atol=0)


def test_route_invariants_on_workloads():
    for name in ("tiny", "decode", "batched_decode"):
        wl = workloads.WORKLOADS[name]
        logits = workloads.draw_logits(wl).numpy()
        ids, w = oracle.route(logits, wl.top_k)
        for t in range(wl.T):
            assert len(set(ids[t].tolist())) == wl.top_k
            assert np.all((ids[t] >= 0) & (ids[t] < wl.E))
            lt = logits[t, ids[t]]
            assert np.all(lt[:-1] >= lt[1:])            # descending logit
            assert np.all(w[t][:-1] >= w[t][1:])        # weights non-increasing
            assert abs(float(w[t].astype(np.float64).sum()) - 1.0) < 1e-6
            # nothing outside the selection beats the k-th selected logit
            rest = np.delete(logits[t], ids[t])
            assert rest.size == 0 or rest.max() <= lt[-1]


def test_route_ties_lowest_index_wins_brute_force():
    rng = np.random.default_rng(7)
    for _ in range(200):
        E = int(rng.integers(2, 40))
        k = int(rng.integers(1, E + 1))
        # few distinct values -> many ties
        logits = rng.integers(-3, 3, size=E).astype(np.float32) * 0.5
        ids, w = oracle.route(logits[None], k)
        order = sorted(range(E), key=lambda e: (-float(logits[e]), e))  # brute-force key sort
        assert ids[0].tolist() == order[:k]
        # equal logits get equal weights
        for a in range(k):
            for b in range(k):
                if logits[ids[0, a]] == logits[ids[0, b]]:
                    assert w[0, a] == w[0, b]


def test_route_k_equals_E_is_full_softmax():
    g = torch.Generator().manual_seed(11)
    logits = torch.randn(16, 12, generator=g)
    ids, w = oracle.route(logits.numpy(), 12)
    full = torch.softmax(logits.double(), dim=1).numpy()
    for t in range(16):
        np.testing.assert_allclose(w[t], full[t, ids[t]], rtol=1e-6)
        assert sorted(ids[t].tolist()) == list(range(12))


def test_route_uniform_logits():
    logits = np.zeros((3, 10), np.float32)
    ids, w = oracle.route(logits, 4)
    assert ids.tolist() == [[0, 1, 2, 3]] * 3
    assert np.all(w == np.float32(0.25))


def test_group_matches_stable_argsort():
    for name in ("tiny", "decode", "batched_decode"):
        wl = workloads.WORKLOADS[name]
        ids, _ = oracle.route(workloads.draw_logits(wl).numpy(), wl.top_k)
        counts, offsets, sorted_pair = oracle.group(ids, wl.E)
        flat = ids.reshape(-1)
        assert np.array_equal(counts, np.bincount(flat, minlength=wl.E))
        assert offsets[0] == 0 and np.array_equal(np.diff(offsets), counts)
        assert np.array_equal(sorted_pair, np.argsort(flat, kind="stable").astype(np.int32))
        assert counts.sum() == wl.T * wl.top_k
        # a bijection of [0, P)
        assert np.array_equal(np.sort(sorted_pair), np.arange(wl.T * wl.top_k))
        # within an expert segment: ascending token
        for e in range(wl.E):
            seg = sorted_pair[offsets[e]:offsets[e + 1]]
            assert np.all(np.diff(seg // wl.top_k) > 0)
            assert np.all(flat[seg] == e)


def test_group_degenerate():
    ids = np.zeros((0, 2), np.int32)
    counts, offsets, sp = oracle.group(ids, 4)
    assert counts.tolist() == [0, 0, 0, 0] and offsets.tolist() == [0] * 5 and sp.size == 0


def _golden_routing_cases():
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "routing_cases.txt")
    cases = []
    for line in open(path):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k, lg, ids, w = (f.strip() for f in line.split("|"))
        cases.append((int(k), [float(v) for v in lg.split(",")], [int(v) for v in ids.split(",")],
                      [float(v) for v in w.split(",")]))
    return cases


@pytest.mark.parametrize("k,logits,ids,w", _golden_routing_cases())
def test_route_hand_derived_cases(k, logits, ids, w):
    got_ids, got_w = oracle.route(np.array([logits], np.float32), k)
    assert got_ids[0].tolist() == ids
    np.testing.assert_allclose(got_w[0], w, rtol=2e-7, atol=1e-9)
