"""The fused decode selection (dsa_indexer_topk_decode): paged indexer, then the per-sequence
top-k that reads only the 16-key groups whose maximum reaches the k-th largest group maximum
and keeps their scores at or above it.

The selection must equal the oracle's top-k (ties to the lower position, ascending) of the
GPU's own scores bit for bit: dsa_indexer_scores runs the same kernel and fp32 arithmetic, and
those scores are checked against the oracle's in test_indexer_gpu.py and below.  The cases
cover every path of the selection kernel:
  - contexts of at most k keys (every position is selected);
  - fewer 16-key groups than k (the group maxima bound nothing; every score is a candidate);
  - the group-maximum bound with its candidates held on chip, at 128K keys;
  - a tie class straddling the k-th position whose members fit on chip;
  - a tie class of tens of thousands (the on-chip candidate buffer overflows: the full radix
    select over the row in global memory runs instead)."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu
CAP = 8192          # candidates the selection holds on chip per row


def _run(d, k, max_ctx=None, scan_reports=True):
    import sparse_attention_09_b200 as dsa
    B = d["B"]
    max_ctx = d["max_ctx"] if max_ctx is None else max_ctx
    keys = dsa.paged_desc(d["kcache8"], d["block_table"], d["ctx"], max_ctx, scale=d["kscale_cache"])
    ws = torch.empty(dsa.dsa_decode_select_workspace_size(B, max_ctx), dtype=torch.uint8, device="cuda")
    idx = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
    dsa.dsa_indexer_topk_decode(d["q8"], d["q_scale"], d["w"], keys, B, 64, 128, k, idx, ws)
    err = dsa.dsa_device_error()
    ld = (max_ctx + 3) // 4 * 4
    S = torch.full((B, ld), float("nan"), device="cuda")
    dsa.dsa_indexer_scores(d["q8"], d["q_scale"], d["w"], keys, B, 64, 128, 0, B, S)
    # the scan alone reports what the fused call reported (NaN scores only the selection does)
    assert dsa.dsa_device_error() == (err if scan_reports else dsa.DSA_OK)
    return idx.cpu().numpy(), S.cpu().numpy(), err


def _check(idx, S, ctx, k):
    for b, n in enumerate(ctx):
        exp = oracle.topk_rows(S[b:b + 1, :n], np.array([n]), k)[0]
        assert np.array_equal(idx[b], exp), f"sequence {b} (ctx {n}): selection != oracle top-k of the scores"


def _patterned(d, patterns, seed):
    """Every cached key becomes one of `patterns` e4m3 rows (k_scale 1), so a query's scores
    take at most `patterns` distinct values: tie classes of ~ctx/patterns keys."""
    rs = np.random.default_rng(seed)
    nb, bs, dI = d["kcache8"].shape
    pats = d["kcache8"].reshape(-1, dI)[: patterns].clone()
    pick = torch.from_numpy(rs.integers(0, patterns, size=nb * bs)).to("cuda")
    d["kcache8"] = pats[pick].reshape(nb, bs, dI).contiguous()
    d["kscale_cache"] = torch.ones_like(d["kscale_cache"])
    return d


@pytest.mark.parametrize("k", [64, 512, 2048])
def test_selection_equals_topk_of_scores_across_paths(k):
    g = 16 * k   # contexts below this have fewer 16-key groups than k
    ctx = sorted(set([1, 100, k - 1, k, k + 1, g - 1, g, g + 1, g + 17, 70001, 131072]))
    d = synth.decode_inputs(B=len(ctx), ctx_lo=1, ctx_hi=131072, H_I=64, d_I=128, H=16, seed=50 + k,
                            device="cuda", ctx=ctx)
    idx, S, err = _run(d, k)
    assert err == 0
    _check(idx, S, ctx, k)
    for b, n in enumerate(ctx):
        m = min(k, n)
        assert (idx[b, :m] >= 0).all() and (idx[b, m:] == -1).all()
        assert (np.diff(idx[b, :m]) > 0).all(), "indices must be ascending"


def test_scores_behind_the_selection_match_oracle():
    ctx = [3000, 40000]
    d = synth.decode_inputs(B=2, ctx_lo=1, ctx_hi=40000, H_I=64, d_I=128, H=16, seed=61, device="cuda", ctx=ctx)
    idx, S, err = _run(d, 2048)
    assert err == 0
    for b in range(2):
        seq = synth.decode_seq_numpy(d, b)
        ref = oracle.decode_indexer_scores(seq["q8"], seq["q_scale"], seq["w"], seq["kcache8"],
                                           seq["kscale_cache"], seq["block_table"], seq["ctx"])
        k8 = oracle.paged_gather(seq["kcache8"], seq["block_table"], seq["ctx"])
        ks = oracle.paged_gather(seq["kscale_cache"], seq["block_table"], seq["ctx"])
        mag = oracle.indexer_magnitude_query(seq["q8"], seq["q_scale"], seq["w"], k8, ks)
        assert np.all(np.abs(S[b, : ctx[b]] - ref) <= 1e-3 * mag + 1e-30), f"seq {b}"
        # the selection against the oracle's own scores: any difference is a near-tie
        sel, sel_ref = set(idx[b][idx[b] >= 0].tolist()), set(oracle.topk_indices(ref, 2048).tolist())
        kth = np.sort(ref)[::-1][2047]
        for s in sel ^ sel_ref:
            assert abs(ref[s] - kth) <= 2e-3 * max(mag[s], 1e-30) + 2e-3 * abs(kth), (b, s)


@pytest.mark.parametrize("patterns,ctx", [(32, [131072, 100000, 90000]), (3, [131072, 120000])])
def test_tie_classes_at_the_boundary(patterns, ctx):
    """32 patterns: the top class (~2.8-4K keys) holds the k-th position and fits on chip;
    3 patterns: the top class (~40K keys) overflows the candidate buffer (full radix select)."""
    k = 2048
    d = _patterned(synth.decode_inputs(B=len(ctx), ctx_lo=1, ctx_hi=131072, H_I=64, d_I=128, H=16,
                                       seed=70 + patterns, device="cuda", ctx=ctx), patterns, seed=patterns)
    idx, S, err = _run(d, k)
    assert err == 0
    _check(idx, S, ctx, k)
    for b, n in enumerate(ctx):
        row = S[b, :n].astype(np.float64)
        assert len(np.unique(row)) <= patterns
        kth = np.sort(row)[::-1][k - 1]
        above, tied = int((row > kth).sum()), int((row == kth).sum())
        assert above < k < above + tied, "the k-th position must fall inside a tie class"
        if patterns == 3:   # the candidates (at least the whole tie class) exceed the buffer
            assert above + tied > CAP
        else:
            assert above + tied <= CAP


def test_all_equal_scores_select_the_first_k_positions():
    """w = 0: every score is 0.  Below 16k keys every score is a candidate and fits on chip;
    at 32K and 128K every group passes the bound and the candidates overflow."""
    k = 2048
    ctx = [5000, 32768, 131072]
    d = synth.decode_inputs(B=3, ctx_lo=1, ctx_hi=131072, H_I=64, d_I=128, H=16, seed=80, device="cuda", ctx=ctx)
    d["w"] = torch.zeros_like(d["w"])
    idx, S, err = _run(d, k)
    assert err == 0
    for b in range(3):
        assert np.array_equal(idx[b], np.arange(k))


def test_context_longer_than_declared_is_reported_and_clamped():
    import sparse_attention_09_b200 as dsa
    k = 512
    d = synth.decode_inputs(B=2, ctx_lo=1, ctx_hi=20000, H_I=64, d_I=128, H=16, seed=81, device="cuda",
                            ctx=[9000, 20000])
    idx, S, err = _run(d, k, max_ctx=12000)   # sequence 1 holds 20000 keys
    assert err == dsa.DSA_ERR_DEVICE_CHECK
    _check(idx, S, [9000, 12000], k)


def test_blocks_outside_the_pool_score_minus_inf_and_are_not_selected():
    import sparse_attention_09_b200 as dsa
    k = 2048
    d = synth.decode_inputs(B=2, ctx_lo=1, ctx_hi=60000, H_I=64, d_I=128, H=16, seed=82, device="cuda",
                            ctx=[60000, 40000])
    d["block_table"] = d["block_table"].clone()
    d["block_table"][0, 100] = d["num_blocks"] + 3
    d["block_table"][1, 0] = -2
    idx, S, err = _run(d, k)
    assert err == dsa.DSA_ERR_DEVICE_CHECK
    assert np.isneginf(S[0, 6400:6464]).all() and np.isneginf(S[1, :64]).all()
    _check(idx, S, [60000, 40000], k)
    assert not ((idx[0] >= 6400) & (idx[0] < 6464)).any() and not ((idx[1] >= 0) & (idx[1] < 64)).any()


def test_nan_score_is_reported():
    """A NaN key scale makes a NaN score; its group counts as passing the bound, so the
    selection reads it and reports DSA_ERR_DEVICE_CHECK."""
    import sparse_attention_09_b200 as dsa
    d = synth.decode_inputs(B=2, ctx_lo=1, ctx_hi=60000, H_I=64, d_I=128, H=16, seed=83, device="cuda",
                            ctx=[60000, 40000])
    blk = int(d["block_table"][1, 300].item())   # sequence 1, position 300 * 64 + 5
    d["kscale_cache"] = d["kscale_cache"].clone()
    d["kscale_cache"][blk, 5] = float("nan")
    idx, S, err = _run(d, 2048, scan_reports=False)
    assert err == dsa.DSA_ERR_DEVICE_CHECK
    assert np.isnan(S[1, 300 * 64 + 5])
    _check(idx[:1], S[:1], [60000], 2048)   # the other sequence is untouched
