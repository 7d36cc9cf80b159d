"""Pins for the oracle's lightning indexer (the score I[t,s] = sum_j w[t,j] ReLU(q_I[t,j].k_I[s])).

Each pin is independent of the oracle's own code: exact rational brute force, a library matmul
on the single-head special case, a hand-worked example, and invariants.  The mutation tests at
the end plant plausible mistakes in copies of the oracle and check the pins catch them.
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example.json")


def _random_case(rs, L=6, H_I=3, d_I=5):
    # finite e4m3 codes only (exclude the NaN codes 0x7F / 0xFF)
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    q8 = rs.choice(codes, size=(L, H_I, d_I)).astype(np.uint8)
    k8 = rs.choice(codes, size=(L, d_I)).astype(np.uint8)
    q_scale = rs.uniform(0.01, 2.0, size=L).astype(np.float32).astype(np.float64)
    k_scale = rs.uniform(0.01, 2.0, size=L).astype(np.float32).astype(np.float64)
    w = rs.normal(size=(L, H_I)).astype(np.float32).astype(np.float64)
    return q8, q_scale, w, k8, k_scale


def _e4m3_fraction(code):
    """Exact rational value of an e4m3 code, from the bit fields (independent of the table)."""
    s = -1 if code & 0x80 else 1
    e = (code >> 3) & 0xF
    m = code & 7
    if e == 0:
        return s * Fraction(m, 8) * Fraction(1, 64)
    return s * (1 + Fraction(m, 8)) * (Fraction(2) ** (e - 7))


def _brute_force(q8, q_scale, w, k8, k_scale):
    """Exact rational scores; q_scale [L] (one per token) or [L, H_I] (one per token and head)."""
    L, H_I, d_I = q8.shape
    out = np.full((L, L), -np.inf)
    for t in range(L):
        for s in range(t + 1):
            total = Fraction(0)
            for j in range(H_I):
                qs = Fraction(q_scale[t, j]) if q_scale.ndim == 2 else Fraction(q_scale[t])
                dot = Fraction(0)
                for d in range(d_I):
                    dot += _e4m3_fraction(int(q8[t, j, d])) * qs * \
                        _e4m3_fraction(int(k8[s, d])) * Fraction(k_scale[s])
                total += Fraction(w[t, j]) * max(dot, Fraction(0))
            out[t, s] = float(total)
    return out


def _close(a, b, rtol=1e-12):
    fa, fb = np.isfinite(a), np.isfinite(b)
    if not np.array_equal(fa, fb) or not np.array_equal(a[~fa], b[~fb]):
        return False
    scale = np.maximum(np.abs(b[fb]), 1e-300)
    return bool(np.all(np.abs(a[fa] - b[fb]) <= rtol * scale + 1e-300))


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_matches_exact_rational_brute_force(seed):
    args = _random_case(np.random.default_rng(seed))
    assert _close(oracle.indexer_scores(*args), _brute_force(*args))


def _per_head_case(rs, L=6, H_I=3, d_I=5):
    q8, _, w, k8, k_scale = _random_case(rs, L, H_I, d_I)
    # scales spread over four decades so that a head paired with the wrong scale shows
    q_scale = (10.0 ** rs.uniform(-2, 2, size=(L, H_I))).astype(np.float32).astype(np.float64)
    return q8, q_scale, w, k8, k_scale


@pytest.mark.parametrize("seed", [3, 4])
def test_per_head_scales_match_exact_rational_brute_force(seed):
    args = _per_head_case(np.random.default_rng(seed))
    assert _close(oracle.indexer_scores(*args), _brute_force(*args))


def test_per_head_scales_equal_to_the_token_scale_give_the_per_token_scores():
    q8, q_scale, w, k8, k_scale = _random_case(np.random.default_rng(8), L=9, H_I=4, d_I=6)
    per_head = np.repeat(q_scale[:, None], 4, axis=1)
    assert np.array_equal(oracle.indexer_scores(q8, per_head, w, k8, k_scale),
                          oracle.indexer_scores(q8, q_scale, w, k8, k_scale))


def test_per_head_quantisation_tracks_heads_of_different_magnitude():
    # Float queries whose heads differ in size by 2^20, with all the weight on the smallest head.
    # One e4m3 scale per token (amax / 448) leaves that head below e4m3's normal range (its
    # values round to zero, below half the smallest subnormal 2^-9); one scale per (token, head)
    # keeps 3 mantissa bits for it.
    rs = np.random.default_rng(12)
    L, H_I, d_I = 24, 2, 32
    qf = rs.normal(size=(L, H_I, d_I)) * np.array([1.0, 2.0 ** -20])[None, :, None]
    kf = rs.normal(size=(L, d_I))
    w = np.tile(np.array([0.0, 2.0 ** 20]), (L, 1))
    exact = np.full((L, L), -np.inf)
    mag = np.zeros((L, L))
    for t in range(L):
        exact[t, : t + 1] = w[t] @ np.maximum(qf[t] @ kf[: t + 1].T, 0.0)
        mag[t, : t + 1] = w[t] @ (np.abs(qf[t]) @ np.abs(kf[: t + 1]).T)
    k8, ks = oracle.quantize_fp8_rows(kf)
    q8_h, qs_h = oracle.quantize_fp8_rows(qf.reshape(L * H_I, d_I))
    q8_t, qs_t = oracle.quantize_fp8_rows(qf.reshape(L, H_I * d_I))
    I_h = oracle.indexer_scores(q8_h.reshape(L, H_I, d_I), qs_h.reshape(L, H_I), w, k8, ks)
    I_t = oracle.indexer_scores(q8_t.reshape(L, H_I, d_I), qs_t, w, k8, ks)
    fin = np.isfinite(exact)
    err_h = np.abs(I_h[fin] - exact[fin]) / mag[fin]
    err_t = np.abs(I_t[fin] - exact[fin]) / mag[fin]
    # every dequantised element (normal range) is within 2^-4 of its value, relative, and ReLU
    # is 1-Lipschitz: |error| <= (2 * 2^-4 + 2^-8) * magnitude
    assert err_h.max() <= 2 * 2.0 ** -4 + 2.0 ** -8
    assert err_t.mean() > 10 * err_h.mean()


def test_single_head_unit_weight_is_scaled_relu_matmul():
    # H_I = 1, w = 1: I = ReLU(Q K^T) on the dequantised operands, causal-masked.
    rs = np.random.default_rng(5)
    L, d_I = 40, 16
    q8, q_scale, w, k8, k_scale = _random_case(rs, L=L, H_I=1, d_I=d_I)
    w[:] = 1.0
    tab = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float64)
    Q = tab[torch.from_numpy(q8[:, 0, :]).long()] * torch.from_numpy(q_scale)[:, None]
    K = tab[torch.from_numpy(k8).long()] * torch.from_numpy(k_scale)[:, None]
    ref = torch.relu(Q @ K.T)
    ref = ref.masked_fill(torch.triu(torch.ones(L, L, dtype=torch.bool), 1), float("-inf")).numpy()
    assert _close(oracle.indexer_scores(q8, q_scale, w, k8, k_scale), ref, rtol=1e-13)


def test_hand_worked_example():
    g = json.load(open(GOLDEN))["indexer"]
    got = oracle.indexer_scores(np.array(g["q8"], np.uint8), np.array(g["q_scale"]), np.array(g["w"]),
                                np.array(g["k8"], np.uint8), np.array(g["k_scale"]))
    exp = np.array([[float(x) for x in row] for row in g["expected_scores"]])
    assert np.array_equal(got, exp)


def test_causal_prefix_and_linearity_in_w():
    rs = np.random.default_rng(9)
    q8, q_scale, w, k8, k_scale = _random_case(rs, L=12, H_I=4, d_I=8)
    I = oracle.indexer_scores(q8, q_scale, w, k8, k_scale)
    assert all(np.isfinite(I[t, : t + 1]).all() and np.isneginf(I[t, t + 1:]).all() for t in range(12))
    w2 = rs.normal(size=w.shape)
    I2 = oracle.indexer_scores(q8, q_scale, w2, k8, k_scale)
    I12 = oracle.indexer_scores(q8, q_scale, w + w2, k8, k_scale)
    fin = np.isfinite(I)
    assert np.allclose(I12[fin], I[fin] + I2[fin], rtol=1e-12, atol=1e-12)


def test_relu_zeroes_negative_dot_products():
    # keys pointing against every head's query contribute nothing, whatever the weights
    q8 = np.full((2, 3, 4), 0x38, np.uint8)                      # every q entry = 1
    k8 = np.array([[0x38] * 4, [0xB8] * 4], np.uint8)            # key0 = +1s, key1 = -1s
    I = oracle.indexer_scores(q8, np.ones(2), np.array([[1.0, -2.0, 3.0]] * 2), k8, np.ones(2))
    assert I[1, 1] == 0.0 and I[1, 0] == 4.0 * (1 - 2 + 3)


def test_magnitude_bounds_score():
    rs = np.random.default_rng(3)
    q8, q_scale, w, k8, k_scale = _random_case(rs, L=8, H_I=4, d_I=8)
    for t in range(8):
        I = oracle.indexer_scores_query(q8[t], q_scale[t], w[t], k8[: t + 1], k_scale[: t + 1])
        A = oracle.indexer_magnitude_query(q8[t], q_scale[t], w[t], k8[: t + 1], k_scale[: t + 1])
        assert np.all(np.abs(I) <= A * (1 + 1e-12))


# ---- planted mistakes: each must be caught by a pin above -----------------------------------
def _mutant(kind):
    def f(q8, q_scale, w, k8, k_scale):
        L = k8.shape[0]
        tab = oracle.e4m3_table().copy()
        if kind == "bias8":
            tab = tab / 2.0
        out = np.full((L, L), -np.inf)
        for t in range(L):
            if q_scale.ndim == 2:
                qs = {"head_scale_first": np.full(q_scale.shape[1], q_scale[t, 0]),
                      "head_scale_reversed": q_scale[t, ::-1]}.get(kind, q_scale[t])
                q = tab[q8[t]] * qs[:, None]
            else:
                q = tab[q8[t]] * q_scale[t]
            k = tab[k8[: t + 1]] * k_scale[: t + 1, None]
            dots = q @ k.T
            if kind == "no_relu":
                act = dots
            elif kind == "abs":
                act = np.abs(dots)
            else:
                act = np.maximum(dots, 0)
            if kind == "w_transposed":
                out[t, : t + 1] = w[t][::-1] @ act          # weights paired with the wrong heads
            elif kind == "drop_kscale":
                out[t, : t + 1] = w[t] @ np.maximum(q @ (tab[k8[: t + 1]]).T, 0)
            else:
                out[t, : t + 1] = w[t] @ act
        return out
    return f


@pytest.mark.parametrize("kind", ["no_relu", "abs", "bias8", "w_transposed", "drop_kscale"])
def test_pins_catch_planted_mistakes(kind):
    args = _random_case(np.random.default_rng(0))
    assert not _close(_mutant(kind)(*args), _brute_force(*args))


@pytest.mark.parametrize("kind", ["head_scale_first", "head_scale_reversed", "no_relu", "w_transposed"])
def test_per_head_pins_catch_planted_mistakes(kind):
    args = _per_head_case(np.random.default_rng(3))
    assert _close(_mutant("none")(*args), _brute_force(*args))    # the unmutated copy passes
    assert not _close(_mutant(kind)(*args), _brute_force(*args))
