"""dsa_topk (CUDA radix select) against the oracle on the same fp32 score buffers: bit-exact."""
import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


def _run(scores, row_len, k):
    import sparse_attention_09_b200 as dsa
    idx = torch.full((scores.shape[0], k), -7, dtype=torch.int32, device="cuda")
    dsa.dsa_topk(scores, row_len, k, idx)
    assert dsa.dsa_device_error() == 0
    return idx.cpu().numpy()


def _check(scores, row_len, k):
    got = _run(scores, row_len, k)
    exp = oracle.topk_rows(scores.cpu().numpy(), row_len.cpu().numpy(), k)
    bad = np.nonzero((got != exp).any(axis=1))[0]
    assert bad.size == 0, f"rows differ: {bad[:10]}"


@pytest.mark.parametrize("n,k", [(256, 64), (8192, 2048), (5000, 2048), (131072, 2048), (1000, 1)])
def test_random_rows(n, k):
    g = torch.Generator(device="cuda").manual_seed(n + k)
    rows = 24
    scores = torch.randn(rows, n, device="cuda", generator=g)
    row_len = torch.randint(1, n + 1, (rows,), device="cuda", generator=g, dtype=torch.int32)
    row_len[0] = n
    row_len[1] = min(k, n)
    row_len[2] = min(k + 1, n)
    _check(scores, row_len, k)


@pytest.mark.parametrize("levels", [2, 3, 16])
def test_tie_heavy_rows(levels):
    scores = synth.tie_heavy_scores(40, 6000, levels, seed=levels, device="cuda")
    row_len = torch.tensor(np.random.default_rng(levels).integers(1, 6001, size=40), dtype=torch.int32,
                           device="cuda")
    _check(scores, row_len, 2048)


def test_causal_rows_with_masked_tail_and_ragged_ld():
    L, k = 3000, 512
    ld = 3004
    buf = torch.full((L, ld), float("-inf"), device="cuda")
    g = torch.Generator(device="cuda").manual_seed(3)
    for t0 in range(0, L, 500):
        blk = torch.randn(min(500, L - t0), L, device="cuda", generator=g)
        buf[t0:t0 + blk.shape[0], :L] = blk
    buf[:, :L] = torch.where(torch.ones(L, L, device="cuda", dtype=torch.bool).tril(), buf[:, :L],
                             torch.full_like(buf[:, :L], float("-inf")))
    row_len = torch.arange(1, L + 1, dtype=torch.int32, device="cuda")
    _check(buf, row_len, k)


def test_special_values():
    s = torch.tensor([[0.0, -0.0, 0.0, -0.0, 1.0, float("-inf"), float("inf"), -1e-45, 1e-45, 0.0] * 30],
                     device="cuda")
    row_len = torch.tensor([s.shape[1]], dtype=torch.int32, device="cuda")
    for k in (1, 3, 7, 64, 150, 300, 512):
        _check(s, row_len, k)


def test_nan_sets_device_check():
    import sparse_attention_09_b200 as dsa
    s = torch.randn(2, 4096, device="cuda")
    s[1, 77] = float("nan")
    idx = torch.empty(2, 64, dtype=torch.int32, device="cuda")
    dsa.dsa_topk(s, torch.tensor([4096, 4096], dtype=torch.int32, device="cuda"), 64, idx)
    assert dsa.dsa_device_error() == dsa.DSA_ERR_DEVICE_CHECK
    assert dsa.dsa_device_error() == 0
