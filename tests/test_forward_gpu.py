"""dsa_forward end to end (fused indexer + top-k, then sparse MLA; or the paged decode chain)
against the oracle.

Selection: the forward's idx must equal the oracle's top-k of the scores dsa_indexer_scores
writes for the same rows (bit for bit: same fp32 arithmetic), and every index that differs
from the oracle's top-k of its own float64 scores must be a near-tie at the k-th value.
Outputs: within the attention bar of the oracle run on the GPU's selection."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_attention_close, assert_scores_close, indexer_scores, keys_desc, latent_desc, oracle_scores

pytestmark = pytest.mark.gpu
SM = 1.0 / math.sqrt(576)


def _forward_prefill(inp, k):
    import sparse_attention_09_b200 as dsa
    T, H = inp["q"].shape[0], inp["q"].shape[1]
    out = torch.full((T, H, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((T, H), device="cuda")
    idx = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    dsa.dsa_forward(dsa.DSA_MODE_PREFILL, inp["q8"], inp["q_scale"], inp["w"], keys_desc(inp), inp["q"],
                    latent_desc(inp), len(inp["seqlens"]), inp["H_I"], inp["d_I"], H, k, SM, out, lse, idx)
    assert dsa.dsa_device_error() == 0
    return out, lse, idx


def _check_prefill(inp, k, rows_per_seq, out, idx):
    cu = inp["cu_seqlens"].cpu().numpy()
    for b, rows in enumerate(rows_per_seq):
        g0 = int(cu[b])
        seq = synth.seq_slice_numpy(inp, b, rows=rows)
        # GPU scores of exactly these rows, then the oracle's selection of them
        I_gpu = [indexer_scores(inp, row_begin=g0 + t, row_end=g0 + t + 1)[0].cpu().numpy() for t in rows]
        I_ref, A_ref = oracle_scores(seq, rows)
        L = int(cu[b + 1] - cu[b])
        for t, sg, ir, ar in zip(rows, I_gpu, I_ref, A_ref):
            assert_scores_close(sg, ir, ar, t, L)   # the indexer's scores of this row, element by element
            got = idx[g0 + t].cpu().numpy()
            exp = oracle.topk_rows(sg[None, : t + 1], np.array([t + 1]), k)[0]
            assert np.array_equal(got, exp), f"seq {b} row {t}: selection != top-k of GPU scores"
            sel_ref = set(oracle.topk_indices(ir.astype(np.float32), k).tolist())
            m = min(k, t + 1)
            kth = np.sort(ir)[::-1][m - 1]
            for s in set(got[got >= 0].tolist()) ^ sel_ref:
                assert abs(ir[s] - kth) <= 2e-3 * ar[s] + 2e-3 * abs(kth) + 1e-30, (b, t, s)
            sel = got[got >= 0]
            ref, _ = oracle.sparse_mla_token(seq["q"][t], seq["latent"], sel, SM)
            assert_attention_close(out[g0 + t].float().cpu().numpy(), ref, f"seq {b} row {t}")


@pytest.mark.parametrize("name,seqlens,k,rows", [
    ("tiny_256", [256], 64, None),
    ("tiny_256", [90, 256, 7], 64, None),
    ("prefill_8k", [2500], 2048, [0, 5, 2047, 2048, 2499]),
    ("prefill_8k", [1200, 3300], 1024, [0, 1023, 1024, 1199, 3299]),
])
def test_prefill_forward(name, seqlens, k, rows):
    cfg = dict(synth.WORKLOADS[name])
    cfg["seqlens"] = seqlens
    inp = synth.prefill_inputs(device="cuda", **cfg)
    out, lse, idx = _forward_prefill(inp, k)
    rows_per_seq = [list(range(L)) if rows is None else [r for r in rows if r < L] for L in seqlens]
    _check_prefill(inp, k, rows_per_seq, out, idx)


def test_prefill_forward_per_head_scales():
    # one query scale per (token, head); heads drawn up to 128x apart in size
    cfg = dict(synth.WORKLOADS["prefill_8k"])
    cfg["seqlens"] = [1500, 700]
    inp = synth.prefill_inputs(device="cuda", q_scale_per_head=True, **cfg)
    out, lse, idx = _forward_prefill(inp, 1024)
    _check_prefill(inp, 1024, [[0, 1023, 1024, 1499], [0, 350, 699]], out, idx)


@pytest.mark.parametrize("name", ["prefill_8k", "prefill_2x32k", "prefill_128k"])
def test_prefill_forward_full_size_sampled(name):
    cfg = dict(synth.WORKLOADS[name])
    inp = synth.prefill_inputs(device="cuda", **cfg)
    out, lse, idx = _forward_prefill(inp, cfg["k"])
    rows = [synth.sample_rows(L, cfg["k"], 6, seed=7 + b) for b, L in enumerate(cfg["seqlens"])]
    _check_prefill(inp, cfg["k"], rows, out, idx)
    assert torch.isfinite(out.float()).all()


def _decode(d, k):
    import sparse_attention_09_b200 as dsa
    B = d["B"]
    keys = dsa.paged_desc(d["kcache8"], d["block_table"], d["ctx"], d["max_ctx"], scale=d["kscale_cache"])
    latent = dsa.paged_desc(d["latent_cache"], d["block_table"], d["ctx"], d["max_ctx"])
    ws = torch.empty(dsa.dsa_workspace_size(dsa.DSA_MODE_DECODE, B, 0, d["max_ctx"], 128, k), dtype=torch.uint8,
                     device="cuda")
    out = torch.full((B, 128, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    idx = torch.full((B, k), -7, dtype=torch.int32, device="cuda")
    dsa.dsa_forward(dsa.DSA_MODE_DECODE, d["q8"], d["q_scale"], d["w"], keys, d["q"], latent, B, 64, 128, 128, k, SM,
                    out, None, idx, ws)
    assert dsa.dsa_device_error() == 0
    return out, idx, keys


@pytest.mark.parametrize("full,per_head", [(False, False), (True, False), (False, True)])
def test_decode_forward(full, per_head):
    import sparse_attention_09_b200 as dsa
    k = 2048
    if full:
        cfg = dict(synth.WORKLOADS["decode_64"])
        d = synth.decode_inputs(device="cuda", **cfg)
        check = [0, 17, 63]
    else:
        d = synth.decode_inputs(B=6, ctx_lo=1, ctx_hi=9000, H_I=64, d_I=128, H=128, seed=8, device="cuda",
                                ctx=[1, 64, 2047, 2048, 2049, 8999], q_scale_per_head=per_head)
        check = range(6)
    out, idx, keys = _decode(d, k)
    ld = ((d["max_ctx"] + 3) // 4) * 4
    S = torch.empty((d["B"], ld), device="cuda")
    dsa.dsa_indexer_scores(d["q8"], d["q_scale"], d["w"], keys, d["B"], 64, 128, 0, d["B"], S)
    for b in check:
        seq = synth.decode_seq_numpy(d, b)
        ctx = seq["ctx"]
        sg = S[b, :ctx].cpu().numpy()
        got = idx[b].cpu().numpy()
        assert np.array_equal(got, oracle.topk_rows(sg[None], np.array([ctx]), k)[0]), f"seq {b} selection"
        lat = oracle.paged_gather(seq["latent_cache"], seq["block_table"], ctx)
        ref, _ = oracle.sparse_mla_token(seq["q"], lat, got[got >= 0], SM)
        assert_attention_close(out[b].float().cpu().numpy(), ref, f"seq {b}")
