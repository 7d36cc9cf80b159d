"""Masked dense mode of sparse MLA (short-prefill mode) against the oracle: the selection
restricts the softmax exactly as in the sparse path, so the oracle is the same
(oracle.sparse_mla_token on the selected rows) and so are the bars (max-abs 2e-2, mean-abs
2e-3 after bf16, relative 1e-2; lse within 1e-2, see test_sparse_mla_gpu).  Also checked:
agreement with the sparse path on the same inputs, and varlen packing (a chunk of the last
tokens of one sequence reaches into the next; those keys are never selected)."""
import math

import numpy as np
import pytest

import oracle
import synth
from helpers import assert_attention_close, masked_mla_prefill, random_selection, sparse_mla_prefill

pytestmark = pytest.mark.gpu

LSE_TOL = 1e-2


@pytest.mark.parametrize("name,seqlens,k,rows", [
    ("tiny_256", [256], 64, None),
    ("tiny_256", [100, 37, 256], 64, None),
    ("prefill_8k", [2048], 2048, [0, 1, 63, 64, 65, 1000, 2047]),        # every causal key selected
    ("prefill_8k", [1500, 700], 512, [0, 511, 512, 699, 1499]),
    ("prefill_8k", [4096], 1024, [0, 1023, 1024, 3000, 4095]),
])
def test_masked_matches_oracle(name, seqlens, k, rows):
    cfg = dict(synth.WORKLOADS[name])
    cfg["seqlens"] = seqlens
    inp = synth.prefill_inputs(device="cuda", **cfg)
    idx = random_selection(seqlens, k, seed=7 * len(seqlens) + k)
    sm = 1.0 / math.sqrt(576)
    out, lse = masked_mla_prefill(inp, idx, k, sm)
    cu = inp["cu_seqlens"].cpu().numpy()
    idx_h = idx.cpu().numpy()
    out_h = out.float().cpu().numpy()
    lse_h = lse.cpu().numpy()
    for b, L in enumerate(seqlens):
        rr = list(range(L)) if rows is None else [r for r in rows if r < L]
        seq = synth.seq_slice_numpy(inp, b, rows=rr)
        for t in rr:
            g = cu[b] + t
            sel = idx_h[g][idx_h[g] >= 0]
            ref, ref_lse = oracle.sparse_mla_token(seq["q"][t], seq["latent"], sel, sm)
            assert_attention_close(out_h[g], ref, f"seq {b} row {t}")
            assert np.allclose(lse_h[g], ref_lse, rtol=0, atol=LSE_TOL), f"lse seq {b} row {t}"


def test_masked_agrees_with_sparse_path():
    cfg = dict(synth.WORKLOADS["prefill_8k"])
    cfg["seqlens"] = [3000]
    inp = synth.prefill_inputs(device="cuda", **cfg)
    k = 2048
    idx = random_selection([3000], k, seed=99)
    sm = 1.0 / math.sqrt(576)
    out_m, lse_m = masked_mla_prefill(inp, idx, k, sm)
    out_s, lse_s = sparse_mla_prefill(inp, idx, k, sm)
    d = (out_m.float() - out_s.float()).abs()
    assert d.max().item() <= 2e-2 and d.mean().item() <= 2e-3
    assert (lse_m - lse_s).abs().max().item() <= 2 * LSE_TOL
