"""Pins for the oracle's sparse MLA: k >= L equals dense causal attention (library routine),
closed forms, permutation invariance, paged decode == contiguous."""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example.json")


def _dense_causal_library(q, latent, sm_scale, dv):
    # MQA: one latent row per token serves as the key (all dims) and value (first dv dims)
    Q = torch.from_numpy(q).permute(1, 0, 2)                 # [H, L, D]
    K = torch.from_numpy(latent)[None].expand(Q.shape[0], -1, -1)
    V = torch.from_numpy(latent[:, :dv])[None].expand(Q.shape[0], -1, -1)
    out = torch.nn.functional.scaled_dot_product_attention(Q, K, V, is_causal=True, scale=sm_scale)
    return out.permute(1, 0, 2).numpy()


@pytest.mark.parametrize("L,H,D,dv", [(37, 3, 24, 16), (64, 2, 576, 512)])
def test_k_at_least_L_equals_dense_causal_attention(L, H, D, dv):
    rs = np.random.default_rng(L)
    q = rs.normal(size=(L, H, D))
    latent = rs.normal(size=(L, D))
    idx = np.full((L, L + 5), -1, np.int32)
    for t in range(L):
        idx[t, : t + 1] = np.arange(t + 1)
    sm = 1.0 / math.sqrt(D)
    out, _ = oracle.sparse_mla(q, latent, idx, sm, dv=dv)
    ref = _dense_causal_library(q, latent, sm, dv)
    assert np.abs(out - ref).max() < 1e-12


def test_closed_forms():
    rs = np.random.default_rng(4)
    H, D, dv = 4, 32, 24
    latent = rs.normal(size=(10, D))
    q = rs.normal(size=(H, D))
    # one selected row: output is its value, lse is its logit
    out, lse = oracle.sparse_mla_token(q, latent, [6], 0.3, dv)
    assert np.allclose(out, latent[6, :dv][None]) and np.allclose(lse, 0.3 * q @ latent[6])
    # all rows equal: output is that row's value, lse = logit + log m
    eq = np.repeat(latent[:1], 10, axis=0)
    out, lse = oracle.sparse_mla_token(q, eq, np.arange(7), 0.3, dv)
    assert np.allclose(out, eq[0, :dv][None]) and np.allclose(lse, 0.3 * q @ eq[0] + math.log(7))
    # zero query: uniform weights -> mean of the selected values, lse = log m
    out, lse = oracle.sparse_mla_token(np.zeros((H, D)), latent, [1, 4, 9], 1.0, dv)
    assert np.allclose(out, latent[[1, 4, 9], :dv].mean(0)[None]) and np.allclose(lse, math.log(3))


def test_hand_worked_example():
    g = json.load(open(GOLDEN))["attention"]
    out, lse = oracle.sparse_mla_token(np.array(g["q"]), np.array(g["latent"]), g["selected"], g["sm_scale"], g["dv"])
    assert np.allclose(out, g["expected_out"], rtol=1e-15) and np.allclose(lse, g["expected_lse"], rtol=1e-15)


def test_selection_order_and_padding_do_not_matter():
    rs = np.random.default_rng(8)
    L, H, D = 50, 3, 40
    q = rs.normal(size=(L, H, D))
    latent = rs.normal(size=(L, D))
    idx = np.full((L, 16), -1, np.int32)
    for t in range(L):
        sel = rs.choice(t + 1, size=min(10, t + 1), replace=False)
        idx[t, : len(sel)] = sel
    perm = idx.copy()
    for t in range(L):
        rs.shuffle(perm[t])
    a, la = oracle.sparse_mla(q, latent, idx, 0.2, dv=32)
    b, lb = oracle.sparse_mla(q, latent, perm, 0.2, dv=32)
    assert np.allclose(a, b, rtol=1e-12, atol=1e-14) and np.allclose(la, lb, rtol=1e-12)


def test_paged_decode_equals_contiguous_last_row():
    rs = np.random.default_rng(11)
    ctx, bs, H_I, d_I, H, D = 150, 16, 2, 8, 3, 40
    nb = (ctx + bs - 1) // bs
    pool = nb + 4
    perm = rs.permutation(pool)[:nb]
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], np.uint8)
    k8 = rs.choice(codes, size=(ctx, d_I)).astype(np.uint8)
    ks = rs.uniform(0.1, 1, size=ctx)
    lat = rs.normal(size=(ctx, D))
    kc = np.zeros((pool, bs, d_I), np.uint8)
    kscache = np.zeros((pool, bs))
    lc = np.zeros((pool, bs, D))
    for p in range(ctx):
        kc[perm[p // bs], p % bs] = k8[p]
        kscache[perm[p // bs], p % bs] = ks[p]
        lc[perm[p // bs], p % bs] = lat[p]
    q8 = rs.choice(codes, size=(H_I, d_I)).astype(np.uint8)
    w = rs.normal(size=H_I)
    q = rs.normal(size=(H, D))
    dec = oracle.dsa_decode(dict(q8=q8, q_scale=0.5, w=w, kcache8=kc, kscale_cache=kscache, latent_cache=lc,
                                 block_table=perm, ctx=ctx, q=q), k=32, sm_scale=0.1, dv=24)
    # contiguous reference: the last prefill row of the same sequence
    L = ctx
    q8_all = np.zeros((L, H_I, d_I), np.uint8)
    q8_all[-1] = q8
    qs = np.ones(L)
    qs[-1] = 0.5
    w_all = np.zeros((L, H_I))
    w_all[-1] = w
    q_all = np.zeros((L, H, D))
    q_all[-1] = q
    pre = oracle.dsa_prefill_rows(dict(q8=q8_all, q_scale=qs, w=w_all, k8=k8, k_scale=ks, q=q_all, latent=lat),
                                  k=32, sm_scale=0.1, rows=[L - 1], dv=24)
    assert np.array_equal(dec["idx"], pre["idx"][0])
    assert np.array_equal(dec["scores32"], pre["scores32"][0])
    assert np.allclose(dec["out"], pre["out"][0], rtol=1e-13, atol=1e-15)
