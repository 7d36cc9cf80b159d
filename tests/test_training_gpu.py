"""The indexer's training signals on the GPU against the oracle: the dense warm-up target
(dsa_attn_distribution_dense) and the indexer backward (dsa_indexer_backward).

Dense target with the oracle's exact lse: as for the sparse target, each p is within 1e-4
relative (+1e-9) of the oracle; with the masked forward's own lse (within 1e-2) within 1.2e-2
relative, each row summing to 1 within that.

Backward on exact-arithmetic inputs (small-integer e4m3 codes, dyadic scales and weights): every
logit a = q_I . k_I is exact in fp32, so the ReLU masks equal the oracle's; the remaining error is
fp32 accumulation of the gradient sums (dk in an order set by atomic adds), bounded here by
1e-5 of the sum of the absolute terms."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import keys_desc, latent_desc, masked_mla_prefill, random_selection

pytestmark = pytest.mark.gpu
SM = 1.0 / math.sqrt(576)


def _dense_idx(seqlens, k):
    """Each row's whole causal prefix as a selection list (-1 beyond the row's position)."""
    rows = []
    for L in seqlens:
        pos = np.arange(k)[None, :]
        t = np.arange(L)[:, None]
        rows.append(np.where(pos <= t, pos, -1))
    return torch.from_numpy(np.concatenate(rows).astype(np.int32)).cuda()


def _oracle_lse_dense(seq, t):
    _, lse = oracle.sparse_mla_token(seq["q"][t], seq["latent"][: t + 1], np.arange(t + 1), SM)
    return lse


@pytest.mark.parametrize("seqlens,block", [([300, 129, 700], (0, 1129)), ([300, 129, 700], (250, 460))])
def test_dense_distribution_matches_oracle(seqlens, block):
    import sparse_attention_09_b200 as dsa
    cfg = dict(synth.WORKLOADS["tiny_256"])
    cfg["seqlens"] = seqlens
    inp = synth.prefill_inputs(device="cuda", **cfg)
    T, H = inp["q"].shape[0], inp["q"].shape[1]
    cu = inp["cu_seqlens"].cpu().numpy()
    r0, r1 = block
    lse = np.zeros((T, H), np.float32)
    checks = []
    for b, L in enumerate(seqlens):
        seq = synth.seq_slice_numpy(inp, b)
        for t in range(L):
            g = cu[b] + t
            if r0 <= g < r1 and (t < 70 or t % 37 == 0 or t == L - 1):
                lse[g] = _oracle_lse_dense(seq, t)
                checks.append((g, t, oracle.attention_distribution_dense_token(seq["q"][t], seq["latent"][: t + 1], SM)))
    ld = 704
    p = torch.full((r1 - r0, ld), float("nan"), device="cuda")
    dsa.dsa_attn_distribution_dense(inp["q"], latent_desc(inp), torch.from_numpy(lse).cuda(), len(seqlens), H, r0, r1,
                                    SM, p)
    assert dsa.dsa_device_error() == 0
    p = p.cpu().numpy()
    for g, t, ref in checks:
        got = p[g - r0]
        assert np.all(np.abs(got[: t + 1] - ref) <= 1e-4 * ref + 1e-9), f"row {g}"
        assert np.all(got[t + 1:] == 0.0), f"row {g}: entries past the prefix"


def test_dense_distribution_with_masked_forward_lse_and_long_prefix():
    import sparse_attention_09_b200 as dsa
    L, k = 1900, 1920
    cfg = dict(synth.WORKLOADS["prefill_8k"])
    cfg["seqlens"] = [L]
    inp = synth.prefill_inputs(device="cuda", **cfg)
    H = inp["q"].shape[1]
    _, lse = masked_mla_prefill(inp, _dense_idx([L], k), k, SM)   # dense causal attention's lse
    rows = [0, 1, 63, 64, 1000, L - 1]
    seq = synth.seq_slice_numpy(inp, 0, rows=rows)
    for t in rows:
        p = torch.full((1, L), float("nan"), device="cuda")
        dsa.dsa_attn_distribution_dense(inp["q"], latent_desc(inp), lse, 1, H, t, t + 1, SM, p)
        assert dsa.dsa_device_error() == 0
        got = p[0].cpu().numpy()
        ref = oracle.attention_distribution_dense_token(seq["q"][t], seq["latent"][: t + 1], SM)
        assert np.all(np.abs(got[: t + 1] - ref) <= 1.2e-2 * ref + 1e-9), f"row {t}"
        assert abs(got.sum() - 1.0) <= 1.2e-2 and np.all(got[t + 1:] == 0.0)


def test_dense_kl_through_indexer_kl_matches_oracle():
    """The dense stage's loss and gradient: dsa_indexer_kl over prefix-length rows."""
    import sparse_attention_09_b200 as dsa
    seqlens = [200]
    cfg = dict(synth.WORKLOADS["tiny_256"])
    cfg["seqlens"] = seqlens
    inp = synth.prefill_inputs(device="cuda", **cfg)
    T, H = inp["q"].shape[0], inp["q"].shape[1]
    seq = synth.seq_slice_numpy(inp, 0)
    lse = np.stack([_oracle_lse_dense(seq, t) for t in range(T)]).astype(np.float32)
    ld = 256
    p = torch.zeros((T, ld), device="cuda")
    dsa.dsa_attn_distribution_dense(inp["q"], latent_desc(inp), torch.from_numpy(lse).cuda(), 1, H, 0, T, SM, p)
    S = torch.full((T, ld), float("-inf"), device="cuda")
    dsa.dsa_indexer_scores(inp["q8"], inp["q_scale"], inp["w"], keys_desc(inp), 1, cfg["H_I"], cfg["d_I"], 0, T, S)
    idx = _dense_idx(seqlens, ld)
    loss = torch.empty(T, device="cuda")
    grad = torch.empty((T, ld), device="cuda")
    dsa.dsa_indexer_kl(p, S, idx, loss, grad)
    assert dsa.dsa_device_error() == 0
    p_h, S_h, loss_h, grad_h = (x.cpu().numpy() for x in (p, S, loss, grad))
    for t in (0, 1, 50, T - 1):
        ref_loss, ref_grad = oracle.indexer_kl(p_h[t, : t + 1], S_h[t, : t + 1])
        assert abs(loss_h[t] - ref_loss) <= 1e-4 * abs(ref_loss) + 1e-6, f"row {t}"
        assert np.all(np.abs(grad_h[t, : t + 1] - ref_grad) <= 1e-6), f"row {t}"
        assert np.all(grad_h[t, t + 1:] == 0.0)


def _magnitudes(seq, idx, grad):
    """Sums of the absolute terms of each gradient (the scale of its fp32 rounding)."""
    qs = np.asarray(seq["q_scale"], np.float64)
    qI = oracle.decode_e4m3(seq["q8"]) * (qs[:, :, None] if qs.ndim == 2 else qs[:, None, None])
    kI = oracle.decode_e4m3(seq["k8"]) * seq["k_scale"][:, None]
    L = qI.shape[0]
    mw = np.zeros((L, qI.shape[1]))
    mq = np.zeros(qI.shape)
    mk = np.zeros(kI.shape)
    for t in range(L):
        v = idx[t] >= 0
        sel, g = idx[t][v], np.abs(grad[t][v])
        a = qI[t] @ kI[sel].T
        m = (a > 0) * np.abs(seq["w"][t])[:, None] * g[None, :]
        mw[t] = np.maximum(a, 0.0) @ g
        mq[t] = m @ np.abs(kI[sel])
        np.add.at(mk, sel, m.T @ np.abs(qI[t]))
    return mw, mq, mk


@pytest.mark.parametrize("H_I,d_I,seqlens,k,per_head", [
    (64, 128, [300, 129], 64, False),
    (64, 64, [250], 128, True),
    (4, 128, [200, 77], 64, False),
    (4, 64, [190], 256, False),     # k >= L: the dense stage's whole-prefix entries
])
def test_indexer_backward_matches_oracle(H_I, d_I, seqlens, k, per_head):
    import sparse_attention_09_b200 as dsa
    inp = synth.exact_prefill_inputs(seqlens, H_I, d_I, 16, seed=H_I + d_I + k, device="cuda",
                                     q_scale_per_head=per_head)
    T = sum(seqlens)
    idx = random_selection(seqlens, k, seed=5 + k, scatter_pad=True)
    rs = np.random.default_rng(k)
    grad = torch.from_numpy(rs.standard_normal((T, k)).astype(np.float32)).cuda()
    dw = torch.full((T, H_I), float("nan"), device="cuda")
    dq = torch.full((T, H_I, d_I), float("nan"), device="cuda")
    dk = torch.full((T, d_I), float("nan"), device="cuda")
    dsa.dsa_indexer_backward(inp["q8"], inp["q_scale"], inp["w"], keys_desc(inp), len(seqlens), H_I, d_I, idx, grad,
                             dw, dq, dk)
    assert dsa.dsa_device_error() == 0
    dw, dq, dk = (x.cpu().numpy().astype(np.float64) for x in (dw, dq, dk))
    idx_h, grad_h = idx.cpu().numpy(), grad.cpu().numpy().astype(np.float64)
    cu = inp["cu_seqlens"].cpu().numpy()
    for b, L in enumerate(seqlens):
        seq = synth.seq_slice_numpy(inp, b)
        s0 = cu[b]
        rw, rq, rk = oracle.indexer_backward(seq["q8"], seq["q_scale"], seq["w"], seq["k8"], seq["k_scale"],
                                             idx_h[s0:s0 + L], grad_h[s0:s0 + L])
        mw, mq, mk = _magnitudes(seq, idx_h[s0:s0 + L], grad_h[s0:s0 + L])
        assert np.all(np.abs(dw[s0:s0 + L] - rw) <= 1e-5 * mw + 1e-30), f"dw, seq {b}"
        assert np.all(np.abs(dq[s0:s0 + L] - rq) <= 1e-5 * mq + 1e-30), f"dq, seq {b}"
        assert np.all(np.abs(dk[s0:s0 + L] - rk) <= 1e-5 * mk + 1e-30), f"dk, seq {b}"
        assert np.abs(rk).max() > 0 and np.abs(rq).max() > 0


def test_indexer_backward_reports_and_skips_entries_outside_the_sequence():
    import sparse_attention_09_b200 as dsa
    seqlens = [120, 90]
    inp = synth.exact_prefill_inputs(seqlens, 64, 128, 16, seed=3, device="cuda")
    idx = random_selection(seqlens, 64, seed=2)
    grad = torch.randn((210, 64), generator=torch.Generator(device="cuda").manual_seed(1), device="cuda")

    def run(sel):
        outs = (torch.empty((210, 64), device="cuda"), torch.empty((210, 64, 128), device="cuda"),
                torch.empty((210, 128), device="cuda"))
        dsa.dsa_indexer_backward(inp["q8"], inp["q_scale"], inp["w"], keys_desc(inp), 2, 64, 128, sel, grad, *outs)
        return outs, dsa.dsa_device_error()

    masked, bad = idx.clone(), idx.clone()
    for (t, i, v) in [(10, 3, 130), (125, 0, -9), (200, 5, 90)]:   # past the sequence, negative, past sequence 1
        assert idx[t, i] >= 0
        bad[t, i] = v
        masked[t, i] = -1
    ref, err = run(masked)
    assert err == dsa.DSA_OK
    got, err = run(bad)
    assert err == dsa.DSA_ERR_DEVICE_CHECK
    # dw and dq: the same per-token arithmetic, bit for bit; dk: atomic adds in any order
    assert torch.equal(got[0], ref[0]) and torch.equal(got[1], ref[1])
    assert (got[2] - ref[2]).abs().max() <= 1e-5 * ref[2].abs().max()
