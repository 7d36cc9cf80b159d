"""Failure detection without a GPU fault: a kernel whose barrier never completes ends by itself
after its time limit, the device error word reports DSA_ERR_TIMEOUT, and the context keeps
working (a following top-k runs and the error word is clear again)."""
import time

import pytest
import torch

pytestmark = pytest.mark.gpu


def test_bounded_wait_times_out_and_context_stays_usable():
    import sparse_attention_09_b200 as dsa
    assert dsa.dsa_device_error() == 0            # clear
    t0 = time.perf_counter()
    dsa.dsa_selftest_wait_timeout(20000)          # 20 ms limit
    code = dsa.dsa_device_error()                 # synchronises
    elapsed = time.perf_counter() - t0
    assert code == dsa.DSA_ERR_TIMEOUT
    assert elapsed < 5.0                          # the kernel ended by itself
    assert dsa.dsa_device_error() == 0            # reading clears the word
    scores = torch.randn(4, 512, device="cuda")
    row_len = torch.full((4,), 512, dtype=torch.int32, device="cuda")
    idx = torch.empty(4, 64, dtype=torch.int32, device="cuda")
    dsa.dsa_topk(scores, row_len, 64, idx)
    torch.cuda.synchronize()
    assert dsa.dsa_device_error() == 0
    want = torch.sort(torch.topk(scores, 64, dim=1).indices, dim=1).values.int()
    assert torch.equal(idx, want)


def test_selftest_rejects_bad_limits():
    import sparse_attention_09_b200 as dsa
    with pytest.raises(dsa.DSAError):
        dsa.dsa_selftest_wait_timeout(0)
    with pytest.raises(dsa.DSAError):
        dsa.dsa_selftest_wait_timeout(3_000_000)
