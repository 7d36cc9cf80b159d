"""Pins for the oracle's attention distribution over the selected rows and the indexer KL loss
(CPU only): properties and closed forms that a dropped term, a wrong sign or a transposed
operand would break."""
import math

import numpy as np

import oracle


def _case(seed, H=8, n=40, m=17, D=576):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((H, D)) / math.sqrt(D)
    lat = rng.standard_normal((n, D)) / math.sqrt(D) * 4
    sel = np.sort(rng.choice(n, size=m, replace=False))
    return q, lat, sel


def test_distribution_sums_to_one_and_is_head_mean():
    q, lat, sel = _case(1)
    sm = 1 / math.sqrt(576)
    p = oracle.attention_distribution_token(q, lat, sel, sm)
    assert abs(p.sum() - 1) < 1e-12 and np.all(p > 0)
    # one head: the softmax of its logits; the mean over heads of those
    per_head = []
    for h in range(q.shape[0]):
        z = sm * (lat[sel] @ q[h])
        e = np.exp(z - z.max())
        per_head.append(e / e.sum())
        p1 = oracle.attention_distribution_token(q[h:h + 1], lat, sel, sm)
        assert np.allclose(p1, per_head[-1], rtol=1e-12, atol=0)
    assert np.allclose(p, np.mean(per_head, axis=0), rtol=1e-12, atol=0)
    # invariant under a permutation of the heads; equal logits give the uniform distribution
    assert np.allclose(oracle.attention_distribution_token(q[::-1], lat, sel, sm), p, rtol=1e-12, atol=0)
    pu = oracle.attention_distribution_token(np.zeros_like(q), lat, sel, sm)
    assert np.allclose(pu, 1.0 / len(sel), rtol=0, atol=1e-15)


def test_kl_properties_and_gradient():
    rng = np.random.default_rng(3)
    p = rng.dirichlet(np.ones(12))
    s = rng.standard_normal(12) * 2
    loss, grad = oracle.indexer_kl(p, s)
    assert loss > 0
    assert abs(grad.sum()) < 1e-12
    # zero exactly at scores = log p + c
    l0, g0 = oracle.indexer_kl(p, np.log(p) + 3.7)
    assert abs(l0) < 1e-12 and np.max(np.abs(g0)) < 1e-12
    # central finite differences
    eps = 1e-6
    for i in range(12):
        sp, sn = s.copy(), s.copy()
        sp[i] += eps
        sn[i] -= eps
        fd = (oracle.indexer_kl(p, sp)[0] - oracle.indexer_kl(p, sn)[0]) / (2 * eps)
        assert abs(fd - grad[i]) < 1e-7
    # zero-probability targets contribute no loss term but keep their gradient q_i
    p2 = np.array([0.0, 1.0])
    l2, g2 = oracle.indexer_kl(p2, np.array([0.0, 0.0]))
    assert abs(l2 - math.log(2)) < 1e-12 and np.allclose(g2, [0.5, -0.5])
