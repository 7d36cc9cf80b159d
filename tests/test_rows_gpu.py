"""Row-block entry points (query rows of one sequence, for sharding a prefill over GPUs):
every block's indices must equal the whole-sequence call's rows bit for bit, and its
attention output and lse must equal them exactly (the same arithmetic per row).  Sampled
rows of a block inside the sequence are also checked against the oracle directly."""
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_attention_close, assert_scores_close, indexer_scores, oracle_scores

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("splits", [[0, 4096, 8192], [0, 1, 4097, 6001, 8192], [0, 3000, 3000, 8192]])
def test_row_blocks_equal_whole_sequence(splits):
    import sparse_attention_09_b200 as dsa
    cfg = dict(synth.WORKLOADS["prefill_8k"])
    inp = synth.prefill_inputs(device="cuda", **cfg)
    L, k, H, H_I, d_I = 8192, cfg["k"], cfg["H"], cfg["H_I"], cfg["d_I"]
    sm = 1.0 / math.sqrt(576)
    keys = dsa.contiguous_desc(inp["k8"], inp["cu_seqlens"], L, scale=inp["k_scale"])
    lat = dsa.contiguous_desc(inp["latent"], inp["cu_seqlens"], L)
    idx = torch.empty((L, k), dtype=torch.int32, device="cuda")
    dsa.dsa_indexer_topk(inp["q8"], inp["q_scale"], inp["w"], keys, 1, H_I, d_I, k, idx)
    out = torch.empty((L, H, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((L, H), device="cuda")
    dsa.dsa_sparse_mla_prefill(inp["q"], lat, idx, 1, H, k, sm, out, lse)
    for rb, re in zip(splits[:-1], splits[1:]):
        R = re - rb
        ib = torch.full((max(R, 1), k), -7, dtype=torch.int32, device="cuda")
        dsa.dsa_indexer_topk_rows(inp["q8"][rb:re].contiguous(), inp["q_scale"][rb:re].contiguous(),
                                  inp["w"][rb:re].contiguous(), keys, H_I, d_I, k, rb, re, ib)
        ob = torch.empty((max(R, 1), H, 512), dtype=torch.bfloat16, device="cuda")
        lb = torch.empty((max(R, 1), H), device="cuda")
        dsa.dsa_sparse_mla_prefill_rows(inp["q"][rb:re].contiguous(), lat, ib, H, k, sm, rb, re, ob, lb)
        torch.cuda.synchronize()
        if R == 0:
            assert (ib == -7).all()          # an empty block writes nothing
            continue
        assert torch.equal(ib[:R], idx[rb:re]), f"indices of rows [{rb}, {re})"
        assert torch.equal(ob[:R], out[rb:re]), f"output of rows [{rb}, {re})"
        assert torch.equal(lb[:R], lse[rb:re]), f"lse of rows [{rb}, {re})"
    assert dsa.dsa_device_error() == 0


def test_row_block_inside_the_sequence_matches_oracle():
    import sparse_attention_09_b200 as dsa
    cfg = dict(synth.WORKLOADS["prefill_8k"])
    inp = synth.prefill_inputs(device="cuda", **cfg)
    L, k, H, H_I, d_I = 8192, cfg["k"], cfg["H"], cfg["H_I"], cfg["d_I"]
    sm = 1.0 / math.sqrt(576)
    rb, re = 3000, 6001
    R = re - rb
    keys = dsa.contiguous_desc(inp["k8"], inp["cu_seqlens"], L, scale=inp["k_scale"])
    lat = dsa.contiguous_desc(inp["latent"], inp["cu_seqlens"], L)
    ib = torch.full((R, k), -7, dtype=torch.int32, device="cuda")
    dsa.dsa_indexer_topk_rows(inp["q8"][rb:re].contiguous(), inp["q_scale"][rb:re].contiguous(),
                              inp["w"][rb:re].contiguous(), keys, H_I, d_I, k, rb, re, ib)
    ob = torch.empty((R, H, 512), dtype=torch.bfloat16, device="cuda")
    lb = torch.empty((R, H), device="cuda")
    dsa.dsa_sparse_mla_prefill_rows(inp["q"][rb:re].contiguous(), lat, ib, H, k, sm, rb, re, ob, lb)
    assert dsa.dsa_device_error() == 0
    rows = [3000, 3001, 4095, 5000, 6000]
    seq = synth.seq_slice_numpy(inp, 0, rows=rows)
    I_ref, A_ref = oracle_scores(seq, rows)
    ib_h, ob_h, lb_h = ib.cpu().numpy(), ob.float().cpu().numpy(), lb.cpu().numpy()
    for t, ir, ar in zip(rows, I_ref, A_ref):
        sg = indexer_scores(inp, row_begin=t, row_end=t + 1)[0].cpu().numpy()
        assert_scores_close(sg, ir, ar, t, L)
        got = ib_h[t - rb]
        assert np.array_equal(got, oracle.topk_rows(sg[None, : t + 1], np.array([t + 1]), k)[0]), f"row {t}"
        kth = np.sort(ir)[::-1][min(k, t + 1) - 1]
        for s in set(got[got >= 0].tolist()) ^ set(oracle.topk_indices(ir.astype(np.float32), k).tolist()):
            assert abs(ir[s] - kth) <= 2e-3 * ar[s] + 2e-3 * abs(kth) + 1e-30, (t, s)
        ref, ref_lse = oracle.sparse_mla_token(seq["q"][t], seq["latent"], got[got >= 0], sm)
        assert_attention_close(ob_h[t - rb], ref, f"row {t}")
        assert np.allclose(lb_h[t - rb], ref_lse, rtol=0, atol=1e-2), f"lse row {t}"
