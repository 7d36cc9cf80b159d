"""Pins for the oracle's top-k selection: brute-force sort, invariants, special cases."""
import json
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example.json")


def _brute(scores, m):
    order = sorted(range(len(scores)), key=lambda i: (-float(scores[i]), i))
    return sorted(order[:m])


@pytest.mark.parametrize("levels", [None, 3, 16])
def test_matches_brute_force_sort(levels):
    rs = np.random.default_rng(1 if levels is None else levels)
    for _ in range(50):
        n = int(rs.integers(1, 300))
        s = rs.normal(size=n).astype(np.float32)
        if levels:
            s = np.round(s * levels / 4).astype(np.float32)
        m = int(rs.integers(1, 80))
        assert list(oracle.topk_indices(s, m)) == _brute(s, m)


def test_invariants():
    rs = np.random.default_rng(7)
    L, k = 500, 64
    scores = np.full((L, L), -np.inf, np.float32)
    for t in range(L):
        scores[t, : t + 1] = np.round(rs.normal(size=t + 1) * 4).astype(np.float32)
    idx = oracle.topk_rows(scores, np.arange(1, L + 1), k)
    for t in range(L):
        sel = idx[t][idx[t] >= 0]
        assert len(sel) == min(k, t + 1)
        assert np.all(idx[t][len(sel):] == -1)
        assert np.all(np.diff(sel) > 0) and sel.min() >= 0 and sel.max() <= t
        rest = np.setdiff1d(np.arange(t + 1), sel)
        if len(rest):
            lo, hi = scores[t, sel].min(), scores[t, rest].max()
            assert lo >= hi
            if lo == hi:   # ties at the boundary: every selected tie precedes every dropped tie
                assert sel[scores[t, sel] == lo].max() < rest[scores[t, rest] == hi].min()


def test_special_cases():
    s = np.array([0.5, 3.0, -1.0, 3.0, 2.0], np.float32)
    assert list(oracle.topk_indices(s, 1)) == [int(np.argmax(s))] == [1]
    assert list(oracle.topk_indices(np.full(100, 7.0, np.float32), 10)) == list(range(10))
    assert list(oracle.topk_indices(np.array([-0.0, 0.0, -0.0], np.float32), 1)) == [0]
    assert list(oracle.topk_indices(np.array([0.0, -0.0, 1.0], np.float32), 2)) == [0, 2]
    assert list(oracle.topk_indices(s, 99)) == [0, 1, 2, 3, 4]
    with pytest.raises(ValueError):
        oracle.topk_indices(np.array([1.0, np.nan], np.float32), 1)


def test_hand_worked_example():
    g = json.load(open(GOLDEN))["indexer"]
    S = np.array([[float(x) for x in row] for row in g["expected_scores"]], np.float32)
    assert oracle.topk_rows(S, np.array([1, 2, 3]), 2).tolist() == g["expected_topk_k2"]
    assert oracle.topk_rows(S, np.array([1, 2, 3]), 1).tolist() == g["expected_topk_k1"]


def test_order_key_is_monotone():
    rs = np.random.default_rng(2)
    s = np.concatenate([rs.normal(size=1000) * 1e3, [0.0, -0.0, np.inf, -np.inf, 1e-45, -1e-45]]).astype(np.float32)
    keys = oracle.order_key_f32(s)
    for a in range(0, len(s), 7):
        for b in range(0, len(s), 11):
            assert (keys[a] < keys[b]) == (s[a] < s[b])
            assert (keys[a] == keys[b]) == (s[a] == s[b])


def test_pin_catches_planted_mistake():
    # a selection that breaks ties toward the higher index must disagree with the brute force
    s = np.array([1.0, 2.0, 2.0, 0.0], np.float32)
    wrong = sorted(sorted(range(4), key=lambda i: (-s[i], -i))[:1])
    assert wrong != _brute(s, 1) == list(oracle.topk_indices(s, 1))
