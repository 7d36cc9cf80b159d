"""The fused indexer top-k under heavy ties, on rows far longer than its candidate capacity.

The method keeps the top-k = 2048 scores per query with ties going to the lower index.  The
fused kernel streams each row through a bounded candidate set (for sequences of up to 128K keys:
capacity max(2k, k + 2560), at most 4608) and cuts it to a superset of the current top k whenever
it fills; when the boundary
bucket holds many equal keys the cut splits them by index.  These inputs make that happen on
most rows: every key is one of three e4m3 patterns, so a row's scores take three values and the
k-th position falls inside a tied class of thousands; a quarter of the rows have w = 0, so all
their scores are equal and the selection must be exactly 0..k-1.

The inputs are exact (small-integer e4m3 codes, w a multiple of 1/16, scales powers of two),
so the GPU's fp32 scores equal the oracle's bit for bit (checked on sampled rows) and the
selection must equal the oracle's top-k of those scores bit for bit."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import indexer_scores, indexer_topk, keys_desc, latent_desc

pytestmark = pytest.mark.gpu


def _three_level_inputs(seqlens, seed):
    inp = synth.exact_prefill_inputs(seqlens, 64, 128, 16, seed=seed, device="cuda", small_scores=True)
    T = sum(seqlens)
    rs = np.random.default_rng(seed)
    pats = inp["k8"][:3].clone()
    inp["k8"] = pats[torch.from_numpy(rs.integers(0, 3, size=T)).to("cuda")].contiguous()
    inp["k_scale"] = torch.ones(T, device="cuda")
    zero = torch.from_numpy(rs.random(T) < 0.25).to("cuda")
    inp["w"] = torch.where(zero[:, None], torch.zeros_like(inp["w"]), inp["w"]).contiguous()
    return inp, zero.cpu().numpy()


def _capacity(k):
    """Candidates per token of the fused top-k for sequences of at most 128K keys (d_I = 128)."""
    return min(max(2 * k, k + 2560), 4608)


def _straddles(row, m):
    """Whether the m-th largest value of the row is shared by selected and unselected entries."""
    kth = np.sort(row)[::-1][m - 1]
    return (row > kth).sum() < m < (row >= kth).sum()


def _check_rows(inp, zero, idx, rows, k, S_rows):
    """S_rows[i]: the GPU's scores of local row rows[i] (one sequence starting at packed row 0)."""
    seq = synth.seq_slice_numpy(inp, 0, rows=rows[:3])
    for t, srow in zip(rows[:3], S_rows[:3]):   # exact inputs: bit-identical to the oracle
        ref = oracle.indexer_scores_query(seq["q8"][t], seq["q_scale"][t], seq["w"][t], seq["k8"][: t + 1],
                                          seq["k_scale"][: t + 1]).astype(np.float32)
        assert np.array_equal(srow[: t + 1], ref), f"row {t}: scores differ from the oracle's"
    straddle = 0
    for t, srow in zip(rows, S_rows):
        row = srow[: t + 1]
        exp = oracle.topk_rows(row[None, :], np.array([t + 1]), k)[0]
        assert np.array_equal(idx[t], exp), f"row {t}: selection != oracle top-k (ties to the lower index)"
        m = min(k, t + 1)
        if zero[t]:
            assert np.array_equal(idx[t][:m], np.arange(m)), f"row {t}: all-equal row must select 0..{m - 1}"
        if t + 1 > _capacity(k) and _straddles(row.astype(np.float64), m):
            straddle += 1
    return straddle


@pytest.mark.parametrize("k", [64, 512, 2048])
def test_fused_topk_three_level_ties_8k(k):
    L = 8192
    inp, zero = _three_level_inputs([L], seed=40 + k)
    idx = indexer_topk(inp, k).cpu().numpy()
    S = indexer_scores(inp).cpu().numpy()
    rows = list(range(L))
    straddle = _check_rows(inp, zero, idx, rows, k, [S[t] for t in rows])
    # the tie-splitting cut ran: long rows whose k-th value is shared across the boundary
    assert straddle > L // 4, f"only {straddle} rows split a tied class past the candidate capacity"


def test_forward_selection_equals_fused_topk_under_ties():
    import sparse_attention_09_b200 as dsa
    L, k = 8192, 2048
    inp, zero = _three_level_inputs([L], seed=77)
    idx = indexer_topk(inp, k)
    T, H = inp["q"].shape[0], inp["q"].shape[1]
    out = torch.empty((T, H, 512), dtype=torch.bfloat16, device="cuda")
    idx_f = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    dsa.dsa_forward(dsa.DSA_MODE_PREFILL, inp["q8"], inp["q_scale"], inp["w"], keys_desc(inp), inp["q"],
                    latent_desc(inp), 1, 64, 128, H, k, 1.0 / math.sqrt(576), out, None, idx_f)
    assert dsa.dsa_device_error() == 0
    assert torch.equal(idx_f, idx)
    assert torch.isfinite(out.float()).all()
    rows = [0, 1, 2047, 2048, 4095, 4096, 8191]
    S_rows = [indexer_scores(inp, row_begin=t, row_end=t + 1)[0].cpu().numpy() for t in rows]
    _check_rows(inp, zero, idx_f.cpu().numpy(), rows, k, S_rows)


@pytest.mark.parametrize("k", [64, 2048])
def test_fused_topk_three_level_ties_2x32k_sampled(k):
    seqlens = [32768, 32768]
    inp, zero = _three_level_inputs(seqlens, seed=90 + k)
    idx = indexer_topk(inp, k).cpu().numpy()
    straddle = 0
    for b, L in enumerate(seqlens):
        g0 = b * 32768
        rows = sorted(set([0, 1, k - 1, k, _capacity(k), _capacity(k) + 1, L - 1] +
                          list(synth.sample_rows(L, k, 40, seed=b + k))))
        S_rows = [indexer_scores(inp, row_begin=g0 + t, row_end=g0 + t + 1)[0].cpu().numpy() for t in rows]
        sub = synth.seq_slice_numpy(inp, b, rows=rows[-3:])
        for t, srow in zip(rows[-3:], S_rows[-3:]):
            ref = oracle.indexer_scores_query(sub["q8"][t], sub["q_scale"][t], sub["w"][t], sub["k8"][: t + 1],
                                              sub["k_scale"][: t + 1]).astype(np.float32)
            assert np.array_equal(srow[: t + 1], ref), f"seq {b} row {t}: scores differ from the oracle's"
        for t, srow in zip(rows, S_rows):
            row = srow[: t + 1]
            exp = oracle.topk_rows(row[None, :], np.array([t + 1]), k)[0]
            assert np.array_equal(idx[g0 + t], exp), f"seq {b} row {t}: selection != oracle top-k"
            m = min(k, t + 1)
            if zero[g0 + t]:
                assert np.array_equal(idx[g0 + t][:m], np.arange(m))
            if t + 1 > _capacity(k) and _straddles(row.astype(np.float64), m):
                straddle += 1
    assert straddle > 20, f"only {straddle} sampled rows split a tied class past the candidate capacity"


@pytest.mark.parametrize("d_I,L", [(64, 66000), (64, 65536)])
def test_fused_topk_both_ring_configurations(d_I, L):
    """Up to 2^16 keys at d_I = 64 (2^17 at d_I = 128) the fused top-k runs a 2-stage key ring
    with 4608 candidates per token; one key more and it takes the 3-stage ring with 4096 (the
    emission bitmap needs the third stage).  Both give the oracle's top-k of the GPU scores."""
    k = 512
    inp = synth.exact_prefill_inputs([L], 4, d_I, 16, seed=L % 97, device="cuda", small_scores=True)
    idx = indexer_topk(inp, k).cpu().numpy()
    rows = [0, k - 1, k, 3000, 40000, L - 2, L - 1]
    for t in rows:
        S = indexer_scores(inp, row_begin=t, row_end=t + 1)[0].cpu().numpy()
        exp = oracle.topk_rows(S[None, : t + 1], np.array([t + 1]), k)[0]
        assert np.array_equal(idx[t], exp), f"row {t}"
