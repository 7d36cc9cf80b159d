"""Pins of the oracle's indexer training signals: the dense warm-up target and the indexer
backward.  Each pin rests on something other than the oracle's own formula: a library
attention routine, closed forms, and central finite differences of an independently written
forward."""
import math

import numpy as np
import pytest
import torch

import oracle


def _codes(rs, shape, lo=0x20, hi=0x48):
    """Random e4m3 codes of moderate magnitude with random signs."""
    c = rs.integers(lo, hi, size=shape).astype(np.uint8)
    return c | (rs.integers(0, 2, size=shape).astype(np.uint8) << 7)


# ---- dense warm-up target ---------------------------------------------------------------------
def test_dense_target_equals_library_attention_weights():
    rs = np.random.default_rng(1)
    H, n, D = 6, 37, 576
    q = rs.standard_normal((H, D)) * 0.05
    c = rs.standard_normal((n, D))
    sm = 1.0 / math.sqrt(D)
    got = oracle.attention_distribution_dense_token(q, c, sm)
    # scaled_dot_product_attention with identity values returns the attention weights
    qt = torch.tensor(q)[:, None, :]                        # [H, 1, D]
    kt = torch.tensor(c)[None].expand(H, n, D)
    vt = torch.eye(n, dtype=torch.float64)[None].expand(H, n, n)
    w = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=sm)[:, 0, :]   # [H, n]
    np.testing.assert_allclose(got, w.mean(0).numpy(), rtol=1e-12, atol=1e-15)
    assert abs(got.sum() - 1.0) < 1e-12


def test_dense_target_special_cases():
    rs = np.random.default_rng(2)
    c = rs.standard_normal((9, 8))
    assert np.allclose(oracle.attention_distribution_dense_token(np.zeros((3, 8)), c, 0.3), np.full(9, 1 / 9))
    # one head, two keys: softmax of two logits is the logistic function of their difference
    q = rs.standard_normal((1, 8))
    p = oracle.attention_distribution_dense_token(q, c[:2], 0.7)
    d = 0.7 * float(q[0] @ (c[0] - c[1]))
    assert abs(p[0] - 1.0 / (1.0 + math.exp(-d))) < 1e-14 and abs(p.sum() - 1) < 1e-14


# ---- indexer backward -------------------------------------------------------------------------
def _forward_real(qI, kI, w, g):
    """sum_s g[s] * sum_j w[j] * max(0, sum_d qI[j,d] * kI[s,d]), with explicit loops."""
    total = 0.0
    for s in range(kI.shape[0]):
        acc = 0.0
        for j in range(qI.shape[0]):
            a = 0.0
            for d in range(qI.shape[1]):
                a += qI[j, d] * kI[s, d]
            acc += w[j] * max(0.0, a)
        total += g[s] * acc
    return total


def _case(seed, H_I=3, d_I=5, n=4, per_head=False):
    rs = np.random.default_rng(seed)
    q8 = _codes(rs, (H_I, d_I))
    k8 = _codes(rs, (n, d_I))
    qs = rs.uniform(0.5, 2.0, size=H_I) if per_head else float(rs.uniform(0.5, 2.0))
    ks = rs.uniform(0.5, 2.0, size=n)
    w = rs.standard_normal(H_I)
    g = rs.standard_normal(n)
    qI = oracle.decode_e4m3(q8) * (np.asarray(qs)[:, None] if per_head else qs)
    kI = oracle.decode_e4m3(k8) * ks[:, None]
    return q8, qs, k8, ks, w, g, qI, kI


@pytest.mark.parametrize("per_head", [False, True])
def test_real_forward_equals_oracle_scores(per_head):
    q8, qs, k8, ks, w, g, qI, kI = _case(3, per_head=per_head)
    ref = float(g @ oracle.indexer_scores_query(q8, qs, w, k8, ks))
    assert abs(_forward_real(qI, kI, w, g) - ref) <= 1e-12 * max(1.0, abs(ref))


def _fd_grads(qI, kI, w, g, h=1e-6):
    def fd(arr, setter):
        out = np.zeros_like(arr)
        for ix in np.ndindex(arr.shape):
            a, b = arr.copy(), arr.copy()
            a[ix] += h
            b[ix] -= h
            out[ix] = (setter(a) - setter(b)) / (2 * h)
        return out
    dw = fd(w, lambda x: _forward_real(qI, kI, x, g))
    dq = fd(qI, lambda x: _forward_real(x, kI, w, g))
    dk = fd(kI, lambda x: _forward_real(qI, x, w, g))
    return dw, dq, dk


def _away_from_kinks(qI, kI, margin=1e-3):
    return np.abs(qI @ kI.T).min() > margin


@pytest.mark.parametrize("seed,per_head", [(4, False), (5, True), (6, False)])
def test_backward_matches_finite_differences(seed, per_head):
    q8, qs, k8, ks, w, g, qI, kI = _case(seed, per_head=per_head)
    assert _away_from_kinks(qI, kI)
    dw, dq, dk = oracle.indexer_backward_query(q8, qs, w, k8, ks, g)
    fw, fq, fk = _fd_grads(qI, kI, w, g)
    for got, ref in ((dw, fw), (dq, fq), (dk, fk)):
        np.testing.assert_allclose(got, ref, rtol=1e-6, atol=1e-8)


def test_planted_mistakes_fail_the_difference_check():
    """Plausible mistakes in the backward, each caught by the difference check."""
    q8, qs, k8, ks, w, g, qI, kI = _case(7)
    fw, fq, fk = _fd_grads(qI, kI, w, g)
    a = qI @ kI.T
    assert (a > 0).any() and (a < 0).any()
    m = (a > 0) * w[:, None] * g[None, :]
    np.testing.assert_allclose(m @ kI, fq, rtol=1e-6, atol=1e-8)          # the right form passes
    np.testing.assert_allclose(m.T @ qI, fk, rtol=1e-6, atol=1e-8)
    mutants = [
        ((w[:, None] * g[None, :]) @ kI, fq),                 # dq: ReLU mask dropped
        (((a > 0) * g[None, :]) @ kI, fq),                    # dq: head weight dropped
        ((w[:, None] * g[None, :]).T @ qI, fk),               # dk: ReLU mask dropped
        (m.T @ qI[::-1], fk),                                 # dk: heads paired with the wrong query rows
        (a @ g, fw),                                          # dw: ReLU dropped
        (np.maximum(a, 0) @ g[::-1], fw),                     # dw: keys paired with the wrong gradient
    ]
    for got, ref in mutants:
        assert not np.allclose(got, ref, rtol=1e-6, atol=1e-8)


def test_backward_closed_form_and_relu_off():
    # one head, one key: dw = g ReLU(a), dq = g w [a>0] k, dk = g w [a>0] q
    q8 = np.array([[0x38, 0x40, 0xB8]], dtype=np.uint8)    # 1, 2, -1
    k8 = np.array([[0x40, 0x38, 0x30]], dtype=np.uint8)    # 2, 1, 0.5
    dw, dq, dk = oracle.indexer_backward_query(q8, 1.0, np.array([3.0]), k8, np.array([1.0]), np.array([0.5]))
    a = 1 * 2 + 2 * 1 - 1 * 0.5
    assert dw[0] == 0.5 * a and np.array_equal(dq[0], 0.5 * 3.0 * np.array([2.0, 1.0, 0.5]))
    assert np.array_equal(dk[0], 0.5 * 3.0 * np.array([1.0, 2.0, -1.0]))
    # every dot product negative: no gradient anywhere
    dw, dq, dk = oracle.indexer_backward_query(q8 ^ 0x80, 1.0, np.array([3.0]), k8, np.array([1.0]), np.array([0.5]))
    assert not dw.any() and not dq.any() and not dk.any()


def test_sequence_backward_adds_key_gradients_over_queries():
    rs = np.random.default_rng(8)
    L, H_I, d_I, m = 12, 3, 4, 5
    q8 = _codes(rs, (L, H_I, d_I))
    k8 = _codes(rs, (L, d_I))
    qs = rs.uniform(0.5, 2.0, size=L)
    ks = rs.uniform(0.5, 2.0, size=L)
    w = rs.standard_normal((L, H_I))
    idx = np.full((L, m), -1, dtype=np.int64)
    for t in range(L):
        sel = np.sort(rs.choice(t + 1, size=min(m, t + 1), replace=False))
        idx[t, : sel.size] = sel
    grad = rs.standard_normal((L, m))
    dw, dq, dk = oracle.indexer_backward(q8, qs, w, k8, ks, idx, grad)
    # brute force: the same total as a sum of per-(token, key) one-key calls
    dk_ref = np.zeros_like(dk)
    for t in range(L):
        for i in range(m):
            s = idx[t, i]
            if s < 0:
                continue
            _, _, d1 = oracle.indexer_backward_query(q8[t], qs[t], w[t], k8[s:s + 1], ks[s:s + 1], grad[t, i:i + 1])
            dk_ref[s] += d1[0]
    np.testing.assert_allclose(dk, dk_ref, rtol=1e-12, atol=1e-12)
    # and the query gradients are those of the query alone
    for t in (0, 5, 11):
        v = idx[t] >= 0
        r = oracle.indexer_backward_query(q8[t], qs[t], w[t], k8[idx[t][v]], ks[idx[t][v]], grad[t][v])
        np.testing.assert_allclose(dw[t], r[0], rtol=1e-12)
        np.testing.assert_allclose(dq[t], r[1], rtol=1e-12)
