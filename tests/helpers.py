"""Shared helpers for the GPU parity tests: run the library on synth inputs, run the oracle on
host copies of the same inputs, and compare under the tolerances the method states."""
import math

import numpy as np
import torch

import oracle
import synth


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
    lib_fn = dsa._lib.dsa_indexer_topk
    import ctypes
    st = lib_fn(ctypes.c_void_p(inp["q8"].data_ptr()), ctypes.c_void_p(inp["q_scale"].data_ptr()),
                ctypes.c_void_p(inp["w"].data_ptr()), keys_desc(inp).ref(), len(inp["seqlens"]), inp["H_I"],
                inp["d_I"], k, ctypes.c_void_p(idx.data_ptr()),
                ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == 0, dsa.dsa_status_string(st)
    assert dsa.dsa_device_error() == 0
    return idx


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
