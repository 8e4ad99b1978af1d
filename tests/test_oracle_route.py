"""Pins for the oracle's router, top-k, gates and bucketing (CPU only)."""
import itertools

import numpy as np
import torch

from oracle import route


def test_router_logits_exact_integers():
    # small integers: every product and sum is exact in any precision
    x = torch.tensor([[1, 2, 0, -1], [3, -2, 1, 1]], dtype=torch.bfloat16)
    w = torch.tensor([[1, 0, 0, 0], [0, 1, 1, 0], [2, -1, 0, 4]], dtype=torch.bfloat16)
    b = np.array([0.5, 0.0, -1.0], np.float32)
    lg = route.router_logits(x, w, b)
    assert lg.tolist() == [[1.5, 2.0, -5.0], [3.5, -1.0, 11.0]]
    assert route.router_logits(x, w).tolist() == [[1.0, 2.0, -4.0], [3.0, -1.0, 12.0]]


def test_topk_brute_force_subsets():
    """The chosen set is the unique k-subset with the largest logit sum, and
    the slots list it largest first."""
    rng = np.random.default_rng(7)
    for E, k in [(6, 1), (6, 2), (6, 3), (8, 8), (5, 4)]:
        lg = rng.standard_normal((40, E))
        ok = route.topk_margin_ok(lg, k)
        ids = route.topk_select(lg, k)
        for t in np.flatnonzero(ok):
            best = max(itertools.combinations(range(E), k), key=lambda c: lg[t, list(c)].sum())
            assert sorted(ids[t].tolist()) == sorted(best)
            assert all(lg[t, ids[t, j]] > lg[t, ids[t, j + 1]] for j in range(k - 1))
            assert len(set(ids[t].tolist())) == k


def test_topk_ties_lower_index():
    lg = np.array([[1.0, 3.0, 3.0, 0.0, 3.0]])
    assert route.topk_select(lg, 2).tolist() == [[1, 2]]
    assert route.topk_select(lg, 4).tolist() == [[1, 2, 4, 0]]


def test_gates_closed_forms():
    lg = np.array([[0.0, -1.0], [2.0, 5.0]])
    ids = route.topk_select(lg, 1)
    g = route.gate_values(lg, ids)
    assert g[0, 0] == 0.5                              # sigmoid(0)
    assert abs(g[1, 0] - 1 / (1 + np.exp(-5.0))) < 1e-15
    # k = 2 softmax: gate of the larger = sigmoid(difference)
    ids2 = route.topk_select(lg, 2)
    g2 = route.gate_values(lg, ids2)
    assert abs(g2[1, 0] - 1 / (1 + np.exp(-3.0))) < 1e-15
    assert abs(g2[0, 0] - 1 / (1 + np.exp(-1.0))) < 1e-15


def test_softmax_gates_sum_to_one():
    rng = np.random.default_rng(8)
    lg = rng.standard_normal((100, 128)) * 3
    ids = route.topk_select(lg, 8)
    g = route.gate_values(lg, ids)
    assert np.allclose(g.sum(axis=1), 1.0, atol=1e-12, rtol=0)
    assert (np.diff(g, axis=1) <= 0).all()              # ordered like the logits


def test_bucket_brute_force():
    rng = np.random.default_rng(9)
    for T, E, k in [(1, 4, 1), (37, 5, 2), (64, 16, 1), (50, 8, 8)]:
        lg = rng.standard_normal((T, E))
        ids = route.topk_select(lg, k)
        counts, offsets, perm, inv = route.bucket(ids, E)
        assert counts.sum() == T * k and offsets[0] == 0 and offsets[-1] == T * k
        assert sorted(perm.tolist()) == list(range(T * k))
        for e in range(E):
            seg = perm[offsets[e]:offsets[e + 1]].tolist()
            want = [s for s in range(T * k) if ids.reshape(-1)[s] == e]   # ascending slots
            assert seg == want and counts[e] == len(want)
        assert (perm[inv] == np.arange(T * k)).all()


def test_bucket_empty_experts_and_all_on_one():
    ids = np.zeros((10, 1), np.int32)
    counts, offsets, perm, _ = route.bucket(ids, 4)
    assert counts.tolist() == [10, 0, 0, 0] and offsets.tolist() == [0, 10, 10, 10, 10]
    assert perm.tolist() == list(range(10))


def test_margin_filter():
    lg = np.array([[1.0, 1.0005, -2.0], [1.0, 1.1, 1.2], [0.0, 5.0, 5.0005]])
    assert route.topk_margin_ok(lg, 1).tolist() == [False, True, False]
    # k = 1 compares only the two largest: row 0's top two are 1.0005 and 1.0
    lg2 = np.array([[3.0, 1.0, 1.0]])
    assert route.topk_margin_ok(lg2, 1).tolist() == [True]
    assert route.topk_margin_ok(lg2, 2).tolist() == [False]
