"""The C-ABI library loads, exports every entry point include/dsa.h declares, and validates
arguments on the host (no GPU work is launched by these calls)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "dsa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(dsa_[a-z_0-9]+)\s*\(", src)))


def test_library_exports_every_declared_symbol():
    import sparse_attention_09_b200 as dsa
    lib = ctypes.CDLL(dsa.lib_path())
    names = _declared()
    assert len(names) >= 8
    for n in names:
        assert hasattr(lib, n), n
    assert set(dsa.EXPORTED) <= set(names)


def test_status_strings():
    import sparse_attention_09_b200 as dsa
    assert dsa.dsa_status_string(0) == "ok"
    assert "timed out" in dsa.dsa_status_string(dsa.DSA_ERR_TIMEOUT)
    assert dsa.dsa_status_string(999) == "unknown status"


def test_host_validation_rejects_bad_arguments_before_launch():
    import sparse_attention_09_b200 as dsa
    lib = dsa._lib
    null = ctypes.c_void_p(0)
    # NULL scores / bad k / misaligned leading dimension
    assert lib.dsa_topk(null, 8, 4, null, 4, null, null) == dsa.DSA_ERR_INVALID_ARGUMENT
    assert lib.dsa_topk(ctypes.c_void_p(256), 8, 4, ctypes.c_void_p(256), 0, ctypes.c_void_p(256), null) == \
        dsa.DSA_ERR_INVALID_ARGUMENT
    assert lib.dsa_topk(ctypes.c_void_p(256), 6, 4, ctypes.c_void_p(256), 4, ctypes.c_void_p(256), null) == \
        dsa.DSA_ERR_INVALID_ARGUMENT
    assert lib.dsa_topk(ctypes.c_void_p(260), 8, 4, ctypes.c_void_p(256), 4, ctypes.c_void_p(256), null) == \
        dsa.DSA_ERR_INVALID_ARGUMENT
    # zero rows is a no-op
    assert lib.dsa_topk(null, 8, 0, null, 4, null, null) == dsa.DSA_OK


def test_quantiser_host_validation():
    import sparse_attention_09_b200 as dsa
    lib = dsa._lib
    null = ctypes.c_void_p(0)
    a = ctypes.c_void_p(4096)
    assert lib.dsa_quantize_fp8(null, 0, 0, null, null, null) == dsa.DSA_OK            # zero rows: no-op
    assert lib.dsa_quantize_fp8(a, -1, 8, a, a, null) == dsa.DSA_ERR_INVALID_ARGUMENT
    assert lib.dsa_quantize_fp8(a, 4, 12, a, a, null) == dsa.DSA_ERR_INVALID_ARGUMENT   # cols % 8
    assert lib.dsa_quantize_fp8(a, 4, 0, a, a, null) == dsa.DSA_ERR_INVALID_ARGUMENT
    assert lib.dsa_quantize_fp8(null, 4, 8, a, a, null) == dsa.DSA_ERR_INVALID_ARGUMENT
    assert lib.dsa_quantize_fp8(ctypes.c_void_p(4104), 4, 8, a, a, null) == dsa.DSA_ERR_INVALID_ARGUMENT  # 16 B
    assert lib.dsa_quantize_fp8(a, 4, 8, ctypes.c_void_p(4100), a, null) == dsa.DSA_ERR_INVALID_ARGUMENT  # 8 B


def test_row_block_entries_host_validation():
    import sparse_attention_09_b200 as dsa
    lib = dsa._lib
    null = ctypes.c_void_p(0)
    cu = ctypes.c_void_p(4096)
    d = dsa.KVDesc(dsa.DSA_KV_CONTIGUOUS, 4096, 4096, 4096, 0, 0, 100, 100, 0, 0, 0)
    ref = ctypes.byref(d)
    # empty blocks are no-ops even with NULL row arrays
    assert lib.dsa_indexer_topk_rows(null, null, 1, null, ref, 64, 128, 2048, 40, 40, null, null) == dsa.DSA_OK
    assert lib.dsa_sparse_mla_prefill_rows(null, ref, null, 128, 2048, ctypes.c_float(0.04), 40, 40, null, null,
                                           null) == dsa.DSA_OK
    # bad ranges
    assert lib.dsa_indexer_topk_rows(cu, cu, 1, cu, ref, 64, 128, 2048, 50, 40, cu, null) == dsa.DSA_ERR_INVALID_ARGUMENT
    assert lib.dsa_indexer_topk_rows(cu, cu, 1, cu, ref, 64, 128, 2048, 0, 101, cu, null) == dsa.DSA_ERR_INVALID_ARGUMENT
    # the query-scale granularity is 1 (per token) or H_I (per token and head), nothing else
    for heads in (0, 2, 63, 65, -1):
        assert lib.dsa_indexer_topk_rows(cu, cu, heads, cu, ref, 64, 128, 2048, 0, 40, cu, null) == \
            dsa.DSA_ERR_INVALID_ARGUMENT
    assert lib.dsa_sparse_mla_prefill_rows(cu, ref, cu, 128, 2048, ctypes.c_float(0.04), -1, 4, cu, null,
                                           null) == dsa.DSA_ERR_INVALID_ARGUMENT


def test_q_scale_heads_from_shape():
    import torch

    import sparse_attention_09_b200 as dsa
    assert dsa._q_scale_heads(torch.ones(10), 64) == 1
    assert dsa._q_scale_heads(torch.ones(10, 64), 64) == 64
    with pytest.raises(ValueError):
        dsa._q_scale_heads(torch.ones(10, 4), 64)


def test_decode_split_rule_through_workspace_size():
    # Decode splits each selection into the largest power of two s of parts with B * s <= 74
    # (CTA pairs: one round) and s <= k / 64, at least 1.  The workspace holds, per (sequence,
    # split, head), 512 fp32 partial outputs and 2 fp32 (max, sum), then the scores
    # (max_ctx = 0 here: none) and the selection.
    import sparse_attention_09_b200 as dsa

    def a256(x):
        return (x + 255) // 256 * 256

    def expected(B, H, k, s):
        return a256(B * s * H * 512 * 4) + a256(B * s * H * 2 * 4) + a256(B * k * 4)

    table = {1: 32, 2: 32, 3: 16, 5: 8, 9: 8, 10: 4, 18: 4, 19: 2, 37: 2, 38: 1, 64: 1, 200: 1}
    for B, s in table.items():
        assert dsa.dsa_workspace_size(dsa.DSA_MODE_DECODE, B, 0, 0, 128, 2048) == expected(B, 128, 2048, s), B
    # k / 64 caps the count: two 64-row chunks allow two splits
    assert dsa.dsa_workspace_size(dsa.DSA_MODE_DECODE, 1, 0, 0, 128, 128) == expected(1, 128, 128, 2)


def test_decode_split_count_partitions_every_selection():
    # Decode split sp of a sequence takes the 64-row chunks [floor(sp * per / 64),
    # floor((sp + 1) * per / 64)) with per = k / splits.  For every batch size and every
    # supported k, the split count the library picks (read back through the workspace size)
    # must divide k and leave no split empty, so the splits partition the selection's chunks
    # exactly: an empty split would be made to repeat a chunk.
    import sparse_attention_09_b200 as dsa

    def a256(x):
        return (x + 255) // 256 * 256

    for k in range(64, 2049, 64):
        for B in range(1, 257):
            ws = dsa.dsa_workspace_size(dsa.DSA_MODE_DECODE, B, 0, 0, 128, k)
            base = a256(B * k * 4)
            s = next(s for s in (1, 2, 4, 8, 16, 32)
                     if a256(B * s * 128 * 512 * 4) + a256(B * s * 128 * 2 * 4) + base == ws)
            assert k % s == 0 and s <= k // 64, (B, k, s)
            per = k // s
            bounds = [sp * per // 64 for sp in range(s)] + [k // 64]
            assert all(bounds[i] < bounds[i + 1] for i in range(s)), (B, k, s)
            assert B * s <= 74 or s == 1, (B, k, s)   # one round on the CTA pairs
