"""Device-side input checks: inputs that only the GPU sees (selection entries, block tables,
context and row lengths) and that lie outside what the host arguments declare are masked or
clamped by the kernels' own bounds checks, reported as DSA_ERR_DEVICE_CHECK through
dsa_device_error, and leave every other result as a clean run computes it.

Each case was checked by reading the kernels first: a bad block id reaches the TMA key loads
only as a row coordinate (out-of-range coordinates read the fill value), and the plain loads
and the row gather it would address are skipped; clamped lengths stay within the caller's
buffers."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_attention_close, random_selection

pytestmark = pytest.mark.gpu
SM = 1.0 / math.sqrt(576)
K = 2048


def _decode(d, block_table, max_ctx):
    import sparse_attention_09_b200 as dsa
    B = d["B"]
    keys = dsa.paged_desc(d["kcache8"], block_table, d["ctx"], max_ctx, scale=d["kscale_cache"])
    lat = dsa.paged_desc(d["latent_cache"], block_table, d["ctx"], max_ctx)
    ws = torch.empty(dsa.dsa_workspace_size(dsa.DSA_MODE_DECODE, B, 0, max_ctx, 128, K), dtype=torch.uint8,
                     device="cuda")
    out = torch.full((B, 128, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    idx = torch.full((B, K), -7, dtype=torch.int32, device="cuda")
    dsa.dsa_forward(dsa.DSA_MODE_DECODE, d["q8"], d["q_scale"], d["w"], keys, d["q"], lat, B, 64, 128, 128, K, SM,
                    out, None, idx, ws)
    return out, idx, dsa.dsa_device_error()


def test_block_ids_outside_the_pool_are_reported_and_masked():
    import sparse_attention_09_b200 as dsa
    d = synth.decode_inputs(B=4, ctx_lo=1, ctx_hi=5000, H_I=64, d_I=128, H=128, seed=21, device="cuda",
                            ctx=[900, 3000, 2500, 4000])
    clean_out, clean_idx, err = _decode(d, d["block_table"], d["max_ctx"])
    assert err == dsa.DSA_OK
    bad = d["block_table"].clone()
    bad[1, 5] = d["num_blocks"] + 7   # inside sequence 1's context, past the pool
    bad[2, 0] = -5                    # sequence 2's first block (also its padding row's source)
    out, idx, err = _decode(d, bad, d["max_ctx"])
    assert err == dsa.DSA_ERR_DEVICE_CHECK
    for b in (0, 3):                  # sequences with valid tables: exactly the clean results
        assert torch.equal(idx[b], clean_idx[b]) and torch.equal(out[b], clean_out[b]), f"seq {b}"
    assert torch.isfinite(out[1].float()).all() and torch.isfinite(out[2].float()).all()
    # keys of a block outside the pool score -inf, so with more than K valid keys left in the
    # context none of them is selected
    sel1, sel2 = idx[1].cpu().numpy(), idx[2].cpu().numpy()
    assert not ((sel1 >= 5 * 64) & (sel1 < 6 * 64)).any(), "a key of the bad block of sequence 1 was selected"
    assert not ((sel2 >= 0) & (sel2 < 64)).any(), "a key of the bad block of sequence 2 was selected"
    assert (sel1 >= 0).sum() == min(K, 3000) and (sel2 >= 0).sum() == min(K, 2500)
    assert dsa.dsa_device_error() == dsa.DSA_OK  # the read cleared the word


def test_empty_context_gives_zero_output_without_error():
    import sparse_attention_09_b200 as dsa
    d = synth.decode_inputs(B=3, ctx_lo=1, ctx_hi=5000, H_I=64, d_I=128, H=128, seed=22, device="cuda",
                            ctx=[0, 700, 2500])
    assert (d["block_table"][0] == -1).all()  # no blocks: every table entry is unused
    out, idx, err = _decode(d, d["block_table"], d["max_ctx"])
    assert err == dsa.DSA_OK
    assert (idx[0] == -1).all()
    assert (out[0].float() == 0).all()
    for b in (1, 2):
        seq = synth.decode_seq_numpy(d, b)
        sel = idx[b].cpu().numpy()
        lat = oracle.paged_gather(seq["latent_cache"], seq["block_table"], seq["ctx"])
        ref, _ = oracle.sparse_mla_token(seq["q"], lat, sel[sel >= 0], SM)
        assert_attention_close(out[b].float().cpu().numpy(), ref, f"seq {b}")


def test_context_longer_than_declared_is_reported_and_clamped():
    import sparse_attention_09_b200 as dsa
    d = synth.decode_inputs(B=3, ctx_lo=1, ctx_hi=5000, H_I=64, d_I=128, H=128, seed=23, device="cuda",
                            ctx=[500, 1000, 3000])
    clean_out, clean_idx, err = _decode(d, d["block_table"], d["max_ctx"])
    assert err == dsa.DSA_OK
    out, idx, err = _decode(d, d["block_table"], 2000)  # declares 2000; sequence 2 holds 3000
    assert err == dsa.DSA_ERR_DEVICE_CHECK
    for b in (0, 1):
        assert torch.equal(idx[b], clean_idx[b]) and torch.equal(out[b], clean_out[b]), f"seq {b}"
    sel = idx[2].cpu().numpy()
    # clamped to the declared 2000 positions, fewer than k: every one of them is selected
    assert np.array_equal(sel[:2000], np.arange(2000)) and (sel[2000:] == -1).all()


def test_prefill_selection_entries_outside_the_sequence_are_reported_and_masked():
    import sparse_attention_09_b200 as dsa
    cfg = dict(synth.WORKLOADS["tiny_256"])
    inp = synth.prefill_inputs(device="cuda", **cfg)
    L, H, k = 256, cfg["H"], cfg["k"]
    lat = dsa.contiguous_desc(inp["latent"], inp["cu_seqlens"], L)
    good = random_selection([L], k, seed=9)
    bad = good.clone()
    masked = good.clone()
    for (t, i, v) in [(10, 3, 300), (20, 0, -7), (100, 5, L)]:
        assert good[t, i] >= 0
        bad[t, i] = v
        masked[t, i] = -1

    def run(idx):
        out = torch.full((L, H, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((L, H), float("nan"), device="cuda")
        dsa.dsa_sparse_mla_prefill(inp["q"], lat, idx, 1, H, k, SM, out, lse)
        return out, lse, dsa.dsa_device_error()

    out_m, lse_m, err = run(masked)
    assert err == dsa.DSA_OK
    out_b, lse_b, err = run(bad)
    assert err == dsa.DSA_ERR_DEVICE_CHECK
    assert torch.equal(out_b, out_m) and torch.equal(lse_b, lse_m)


def test_topk_row_lengths_outside_the_row_are_reported_and_clamped():
    import sparse_attention_09_b200 as dsa
    g = torch.Generator(device="cuda").manual_seed(4)
    scores = torch.randn((4, 64), generator=g, device="cuda")
    k = 8
    idx = torch.full((4, k), -7, dtype=torch.int32, device="cuda")
    dsa.dsa_topk(scores, torch.tensor([10, 64, 100, -3], dtype=torch.int32, device="cuda"), k, idx)
    assert dsa.dsa_device_error() == dsa.DSA_ERR_DEVICE_CHECK
    ref = oracle.topk_rows(scores.cpu().numpy(), np.array([10, 64, 64, 0]), k)
    assert np.array_equal(idx.cpu().numpy(), ref)
