"""Shared helpers for the GPU parity tests: run the library on synth inputs, run the oracle on
host copies of the same inputs, and compare under the tolerances the method states."""

import numpy as np
import torch

import oracle


def lib():
    import sparse_attention_09_b200 as dsa
    return dsa


def keys_desc(inp):
    dsa = lib()
    return dsa.contiguous_desc(inp["k8"], inp["cu_seqlens"], max(inp["seqlens"]), scale=inp["k_scale"])


def latent_desc(inp):
    dsa = lib()
    return dsa.contiguous_desc(inp["latent"], inp["cu_seqlens"], max(inp["seqlens"]))


def indexer_scores(inp, row_begin=0, row_end=None, ld=None):
    dsa = lib()
    T = inp["q8"].shape[0]
    row_end = T if row_end is None else row_end
    L = max(inp["seqlens"])
    ld = ld or ((L + 3) // 4) * 4
    scores = torch.full((row_end - row_begin, ld), float("nan"), device="cuda")
    dsa.dsa_indexer_scores(inp["q8"], inp["q_scale"], inp["w"], keys_desc(inp), len(inp["seqlens"]), inp["H_I"],
                           inp["d_I"], row_begin, row_end, scores)
    assert dsa.dsa_device_error() == 0
    return scores


def indexer_topk(inp, k):
    dsa = lib()
    T = inp["q8"].shape[0]
    idx = torch.full((T, k), -7, dtype=torch.int32, device="cuda")
    dsa.dsa_indexer_topk(inp["q8"], inp["q_scale"], inp["w"], keys_desc(inp), len(inp["seqlens"]), inp["H_I"],
                         inp["d_I"], k, idx)
    assert dsa.dsa_device_error() == 0
    return idx


def random_selection(seqlens, k, seed, device="cuda", scatter_pad=False):
    """A valid selection per token: min(k, t+1) distinct causal positions, ascending, -1 padded
    (or, with scatter_pad, the -1 entries shuffled among the valid ones)."""
    g = torch.Generator(device=device).manual_seed(seed)
    rows = []
    for L in seqlens:
        r = torch.rand(L, L, generator=g, device=device)
        r = r.masked_fill(torch.ones(L, L, dtype=torch.bool, device=device).triu(1), -1.0)
        kk = min(k, L)
        top = torch.topk(r, kk, dim=1).indices
        vals = torch.gather(r, 1, top)
        top = torch.where(vals >= 0, top, torch.full_like(top, 1 << 30))
        top = torch.sort(top, dim=1).values
        top = torch.where(top >= (1 << 30), torch.full_like(top, -1), top).to(torch.int32)
        sel = torch.full((L, k), -1, dtype=torch.int32, device=device)
        sel[:, :kk] = top
        if scatter_pad:
            perm = torch.argsort(torch.rand(L, k, generator=g, device=device), dim=1)
            sel = torch.gather(sel, 1, perm)
        rows.append(sel)
    return torch.cat(rows, 0).contiguous()


def sparse_mla_prefill(inp, idx, k, sm_scale, with_lse=True):
    dsa = lib()
    T, H = inp["q"].shape[0], inp["q"].shape[1]
    out = torch.full((T, H, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((T, H), float("nan"), device="cuda") if with_lse else None
    dsa.dsa_sparse_mla_prefill(inp["q"], latent_desc(inp), idx, len(inp["seqlens"]), H, k, sm_scale, out, lse)
    assert dsa.dsa_device_error() == 0
    return out, lse


def masked_mla_prefill(inp, idx, k, sm_scale, with_lse=True):
    dsa = lib()
    T, H = inp["q"].shape[0], inp["q"].shape[1]
    out = torch.full((T, H, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((T, H), float("nan"), device="cuda") if with_lse else None
    dsa.dsa_masked_mla_prefill(inp["q"], latent_desc(inp), idx, len(inp["seqlens"]), H, k, sm_scale, out, lse)
    assert dsa.dsa_device_error() == 0
    return out, lse


def assert_attention_close(got, ref, what=""):
    """The stated bar (max-abs 2e-2, mean-abs 2e-3 after bf16 rounding) plus a relative bar
    (1e-2 of the reference norm), since the synthetic outputs are only ~1e-2 in size."""
    g = np.asarray(got, dtype=np.float64)
    r = np.asarray(torch.from_numpy(np.asarray(ref, dtype=np.float32)).to(torch.bfloat16).float().numpy(),
                   dtype=np.float64)
    d = np.abs(g - r)
    assert d.max() <= 2e-2, f"{what} max-abs {d.max():.3e}"
    assert d.mean() <= 2e-3, f"{what} mean-abs {d.mean():.3e}"
    rel = np.linalg.norm(g - r) / max(np.linalg.norm(r), 1e-30)
    assert rel <= 1e-2, f"{what} relative {rel:.3e}"


def oracle_scores(seq_np, rows):
    """float64 scores and magnitudes of the given local rows (full causal prefix)."""
    I, A = [], []
    for t in rows:
        I.append(oracle.indexer_scores_query(seq_np["q8"][t], seq_np["q_scale"][t], seq_np["w"][t],
                                             seq_np["k8"][: t + 1], seq_np["k_scale"][: t + 1]))
        A.append(oracle.indexer_magnitude_query(seq_np["q8"][t], seq_np["q_scale"][t], seq_np["w"][t],
                                                seq_np["k8"][: t + 1], seq_np["k_scale"][: t + 1]))
    return I, A


def assert_scores_close(gpu_row, ref, mag, t, L):
    """|I_gpu - I_ref| <= 1e-3 * A + 1e-30 on s <= t; -inf on t < s < L."""
    g = np.asarray(gpu_row, dtype=np.float64)
    err = np.abs(g[: t + 1] - ref)
    bound = 1e-3 * mag + 1e-30
    bad = np.nonzero(err > bound)[0]
    assert bad.size == 0, f"row {t}: {bad.size} scores off, first s={bad[0]} gpu={g[bad[0]]} ref={ref[bad[0]]}"
    assert np.all(np.isneginf(g[t + 1: L])), f"row {t}: causal mask not -inf"
