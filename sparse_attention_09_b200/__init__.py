"""Python binding of libdsa (the B200 DeepSeek Sparse Attention library).

Argument marshalling only: every function passes device pointers (``tensor.data_ptr()``),
sizes and the current CUDA stream to the C ABI declared in ``include/dsa.h`` and raises
``DSAError`` on a non-zero status.  All computation happens in the library's CUDA kernels;
there is no fallback.  Importing fails if the library has not been built
(``python sparse_attention_09_b200/build.py``).
"""

from __future__ import annotations

import ctypes
import os

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libdsa.so")
if not os.path.exists(_LIB_PATH):
    raise ImportError(f"libdsa.so is not built ({_LIB_PATH}); run: python sparse_attention_09_b200/build.py")
_lib = ctypes.CDLL(_LIB_PATH)

DSA_OK = 0
DSA_ERR_INVALID_ARGUMENT = 1
DSA_ERR_UNSUPPORTED = 2
DSA_ERR_WORKSPACE_TOO_SMALL = 3
DSA_ERR_CUDA = 4
DSA_ERR_TIMEOUT = 5
DSA_ERR_DEVICE_CHECK = 6
DSA_KV_CONTIGUOUS = 0
DSA_KV_PAGED = 1
DSA_MODE_PREFILL = 0
DSA_MODE_DECODE = 1

EXPORTED = ("dsa_indexer_scores", "dsa_indexer_topk", "dsa_topk", "dsa_sparse_mla_prefill", "dsa_sparse_mla_decode",
            "dsa_forward", "dsa_workspace_size", "dsa_status_string", "dsa_device_error",
            "dsa_sparse_mla_decode_noalloc", "dsa_quantize_fp8", "dsa_masked_mla_prefill",
            "dsa_indexer_topk_rows", "dsa_sparse_mla_prefill_rows", "dsa_attn_distribution", "dsa_indexer_kl",
            "dsa_selftest_wait_timeout", "dsa_row_partition", "dsa_indexer_topk_decode",
            "dsa_decode_select_workspace_size", "dsa_attn_distribution_dense", "dsa_indexer_backward")


class KVDesc(ctypes.Structure):
    _fields_ = [
        ("kind", ctypes.c_int32),
        ("data", ctypes.c_void_p),
        ("scale", ctypes.c_void_p),
        ("cu_seqlens", ctypes.c_void_p),
        ("block_table", ctypes.c_void_p),
        ("context_lens", ctypes.c_void_p),
        ("total_tokens", ctypes.c_int64),
        ("max_seqlen", ctypes.c_int32),
        ("num_blocks", ctypes.c_int32),
        ("block_size", ctypes.c_int32),
        ("max_blocks_per_seq", ctypes.c_int32),
    ]


_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_F32 = ctypes.c_float
_SZ = ctypes.c_size_t
_DESC = ctypes.POINTER(KVDesc)

_lib.dsa_status_string.argtypes = [_I32]
_lib.dsa_status_string.restype = ctypes.c_char_p
_lib.dsa_device_error.argtypes = [ctypes.POINTER(_I32), _P]
_lib.dsa_device_error.restype = _I32
_lib.dsa_topk.argtypes = [_P, _I64, _I64, _P, _I32, _P, _P]
_lib.dsa_topk.restype = _I32
_lib.dsa_indexer_scores.argtypes = [_P, _P, _I32, _P, _DESC, _I32, _I32, _I32, _I64, _I64, _P, _I64, _P]
_lib.dsa_indexer_scores.restype = _I32
_lib.dsa_sparse_mla_prefill.argtypes = [_P, _DESC, _P, _I32, _I32, _I32, _F32, _P, _P, _P]
_lib.dsa_sparse_mla_prefill.restype = _I32
_lib.dsa_sparse_mla_decode.argtypes = [_P, _DESC, _P, _I32, _I32, _I32, _F32, _P, _P, _P, _SZ, _P]
_lib.dsa_sparse_mla_decode.restype = _I32
_lib.dsa_forward.argtypes = [_I32, _P, _P, _I32, _P, _DESC, _P, _DESC, _I32, _I32, _I32, _I32, _I32, _F32, _P, _P, _P,
                             _P, _SZ, _P]
_lib.dsa_forward.restype = _I32
_lib.dsa_indexer_topk.argtypes = [_P, _P, _I32, _P, _DESC, _I32, _I32, _I32, _I32, _P, _P]
_lib.dsa_indexer_topk.restype = _I32
_lib.dsa_sparse_mla_decode_noalloc.argtypes = [_P, _DESC, _P, _I32, _I32, _I32, _F32, _P, _P, _P]
_lib.dsa_sparse_mla_decode_noalloc.restype = _I32
_lib.dsa_attn_distribution.argtypes = [_P, _DESC, _P, _P, _I32, _I32, _I32, _F32, _P, _P]
_lib.dsa_attn_distribution.restype = _I32
_lib.dsa_indexer_kl.argtypes = [_P, _P, _P, _I64, _I32, _P, _P, _P]
_lib.dsa_indexer_kl.restype = _I32
_lib.dsa_selftest_wait_timeout.argtypes = [_I32, _P]
_lib.dsa_selftest_wait_timeout.restype = _I32
_lib.dsa_indexer_topk_rows.argtypes = [_P, _P, _I32, _P, _DESC, _I32, _I32, _I32, _I64, _I64, _P, _P]
_lib.dsa_indexer_topk_rows.restype = _I32
_lib.dsa_sparse_mla_prefill_rows.argtypes = [_P, _DESC, _P, _I32, _I32, _F32, _I64, _I64, _P, _P, _P]
_lib.dsa_row_partition.argtypes = [_I64, _I32, _I32, ctypes.c_double, ctypes.c_double, ctypes.POINTER(_I64)]
_lib.dsa_row_partition.restype = _I32
_lib.dsa_sparse_mla_prefill_rows.restype = _I32
_lib.dsa_masked_mla_prefill.argtypes = [_P, _DESC, _P, _I32, _I32, _I32, _F32, _P, _P, _P]
_lib.dsa_masked_mla_prefill.restype = _I32
_lib.dsa_quantize_fp8.argtypes = [_P, _I64, _I32, _P, _P, _P]
_lib.dsa_quantize_fp8.restype = _I32
_lib.dsa_workspace_size.argtypes = [_I32, _I32, _I64, _I32, _I32, _I32]
_lib.dsa_workspace_size.restype = _SZ
_lib.dsa_indexer_topk_decode.argtypes = [_P, _P, _I32, _P, _DESC, _I32, _I32, _I32, _I32, _P, _P, _SZ, _P]
_lib.dsa_indexer_topk_decode.restype = _I32
_lib.dsa_decode_select_workspace_size.argtypes = [_I32, _I32]
_lib.dsa_decode_select_workspace_size.restype = _SZ
_lib.dsa_attn_distribution_dense.argtypes = [_P, _DESC, _P, _I32, _I32, _I64, _I64, _F32, _P, _I64, _P]
_lib.dsa_attn_distribution_dense.restype = _I32
_lib.dsa_indexer_backward.argtypes = [_P, _P, _I32, _P, _DESC, _I32, _I32, _I32, _P, _P, _I32, _P, _P, _P, _P]
_lib.dsa_indexer_backward.restype = _I32


class DSAError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = int(status)
        super().__init__(f"{where}: {dsa_status_string(status)} (status {status})")


def lib_path() -> str:
    return _LIB_PATH


def dsa_status_string(status: int) -> str:
    return _lib.dsa_status_string(int(status)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status, where):
    if status != DSA_OK:
        raise DSAError(status, where)


class Desc:
    """A dsa_kv_desc plus references to the tensors it points at."""

    def __init__(self, struct: KVDesc, refs):
        self.struct = struct
        self._refs = refs

    def ref(self):
        return ctypes.byref(self.struct)


def contiguous_desc(data, cu_seqlens, max_seqlen, scale=None) -> Desc:
    """Contiguous per-token operand: data [T, D] (e4m3 bytes with scale [T], or bf16 latent)."""
    s = KVDesc(kind=DSA_KV_CONTIGUOUS, data=data.data_ptr(), scale=None if scale is None else scale.data_ptr(),
               cu_seqlens=cu_seqlens.data_ptr(), block_table=None, context_lens=None,
               total_tokens=int(data.shape[0]), max_seqlen=int(max_seqlen), num_blocks=0, block_size=0,
               max_blocks_per_seq=0)
    return Desc(s, (data, scale, cu_seqlens))


def paged_desc(data, block_table, context_lens, max_ctx, scale=None) -> Desc:
    """Paged operand: data [num_blocks, block_size, D]; block_table [B, max_blocks]; context_lens [B]."""
    s = KVDesc(kind=DSA_KV_PAGED, data=data.data_ptr(), scale=None if scale is None else scale.data_ptr(),
               cu_seqlens=None, block_table=block_table.data_ptr(), context_lens=context_lens.data_ptr(),
               total_tokens=0, max_seqlen=int(max_ctx), num_blocks=int(data.shape[0]),
               block_size=int(data.shape[1]), max_blocks_per_seq=int(block_table.shape[1]))
    return Desc(s, (data, scale, block_table, context_lens))


def dsa_quantize_fp8(x, codes, scale, stream=None):
    """codes[r, :] = e4m3(x[r, :] / scale[r]) with scale[r] = amax|x[r, :]| / 448 (per token)."""
    rows = x.shape[0]
    cols = x.numel() // rows if rows else 0
    _check(_lib.dsa_quantize_fp8(_ptr(x), rows, cols, _ptr(codes), _ptr(scale), _stream(stream)), "dsa_quantize_fp8")
    return codes, scale


def dsa_topk(scores, row_len, k, idx, stream=None):
    """idx[r, :] = top-k indices (ascending, -1 padded) of scores[r, :row_len[r]]."""
    _check(_lib.dsa_topk(_ptr(scores), scores.stride(0), scores.shape[0], _ptr(row_len), int(k), _ptr(idx),
                         _stream(stream)), "dsa_topk")
    return idx


def _q_scale_heads(q_scale, H_I) -> int:
    """The C ABI's q_scale_heads from the scale tensor's shape: [rows] -> 1 (one scale per
    token), [rows, H_I] -> H_I (one per token and indexer head)."""
    if q_scale is not None and q_scale.dim() == 2:
        if q_scale.shape[1] != int(H_I):
            raise ValueError(f"q_scale has {q_scale.shape[1]} columns, expected H_I = {H_I}")
        return int(H_I)
    return 1


def dsa_indexer_scores(q_fp8, q_scale, w, keys: Desc, B, H_I, d_I, row_begin, row_end, scores, stream=None):
    _check(_lib.dsa_indexer_scores(_ptr(q_fp8), _ptr(q_scale), _q_scale_heads(q_scale, H_I), _ptr(w), keys.ref(),
                                   int(B), int(H_I), int(d_I), int(row_begin), int(row_end), _ptr(scores),
                                   scores.stride(0), _stream(stream)),
           "dsa_indexer_scores")
    return scores


def dsa_attn_distribution(q, latent: Desc, idx, lse, B, H, k, sm_scale, p_out, stream=None):
    """p_out[t, i] = head-averaged attention probability of the selected row idx[t, i]."""
    _check(_lib.dsa_attn_distribution(_ptr(q), latent.ref(), _ptr(idx), _ptr(lse), int(B), int(H), int(k),
                                      float(sm_scale), _ptr(p_out), _stream(stream)), "dsa_attn_distribution")
    return p_out


def dsa_indexer_kl(p, scores, idx, loss, grad, stream=None):
    """loss[r] = KL(p[r] || softmax(scores[r])) over valid entries; grad = softmax(scores) - p."""
    rows, k = p.shape
    _check(_lib.dsa_indexer_kl(_ptr(p), _ptr(scores), _ptr(idx), int(rows), int(k), _ptr(loss), _ptr(grad),
                               _stream(stream)), "dsa_indexer_kl")
    return loss, grad


def dsa_selftest_wait_timeout(limit_us, stream=None):
    """Runs the bounded-wait self-test kernel (it records DSA_ERR_TIMEOUT and returns)."""
    _check(_lib.dsa_selftest_wait_timeout(int(limit_us), _stream(stream)), "dsa_selftest_wait_timeout")


def dsa_indexer_topk_rows(q_fp8, q_scale, w, keys: Desc, H_I, d_I, k, row_begin, row_end, idx, stream=None):
    """Fused indexer + top-k for query rows [row_begin, row_end) of one sequence; the query
    arrays and idx hold just those rows."""
    _check(_lib.dsa_indexer_topk_rows(_ptr(q_fp8), _ptr(q_scale), _q_scale_heads(q_scale, H_I), _ptr(w),
                                      keys.ref(), int(H_I), int(d_I), int(k), int(row_begin), int(row_end),
                                      _ptr(idx), _stream(stream)), "dsa_indexer_topk_rows")
    return idx


def dsa_sparse_mla_prefill_rows(q, latent: Desc, idx, H, k, sm_scale, row_begin, row_end, out, lse=None, stream=None):
    """Sparse MLA prefill for query rows [row_begin, row_end) of one sequence."""
    _check(_lib.dsa_sparse_mla_prefill_rows(_ptr(q), latent.ref(), _ptr(idx), int(H), int(k), float(sm_scale),
                                            int(row_begin), int(row_end), _ptr(out), _ptr(lse), _stream(stream)),
           "dsa_sparse_mla_prefill_rows")
    return out


def dsa_masked_mla_prefill(q, latent: Desc, idx, B, H, k, sm_scale, out, lse=None, stream=None):
    """Same result as dsa_sparse_mla_prefill, computed densely over the causal prefix with a mask."""
    _check(_lib.dsa_masked_mla_prefill(_ptr(q), latent.ref(), _ptr(idx), int(B), int(H), int(k), float(sm_scale),
                                       _ptr(out), _ptr(lse), _stream(stream)), "dsa_masked_mla_prefill")
    return out


def dsa_sparse_mla_prefill(q, latent: Desc, idx, B, H, k, sm_scale, out, lse=None, stream=None):
    _check(_lib.dsa_sparse_mla_prefill(_ptr(q), latent.ref(), _ptr(idx), int(B), int(H), int(k), float(sm_scale),
                                       _ptr(out), _ptr(lse), _stream(stream)), "dsa_sparse_mla_prefill")
    return out


def dsa_sparse_mla_decode(q, latent: Desc, idx, B, H, k, sm_scale, out, lse=None, workspace=None, stream=None):
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.dsa_sparse_mla_decode(_ptr(q), latent.ref(), _ptr(idx), int(B), int(H), int(k), float(sm_scale),
                                      _ptr(out), _ptr(lse), _ptr(workspace), ws_bytes, _stream(stream)),
           "dsa_sparse_mla_decode")
    return out


def dsa_forward(mode, q_fp8, q_scale, w, keys: Desc, q, latent: Desc, B, H_I, d_I, H, k, sm_scale, out, lse=None,
                idx_out=None, workspace=None, stream=None):
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(_lib.dsa_forward(int(mode), _ptr(q_fp8), _ptr(q_scale), _q_scale_heads(q_scale, H_I), _ptr(w), keys.ref(),
                            _ptr(q), latent.ref(),
                            int(B), int(H_I), int(d_I), int(H), int(k), float(sm_scale), _ptr(out), _ptr(lse),
                            _ptr(idx_out), _ptr(workspace), ws_bytes, _stream(stream)), "dsa_forward")
    return out


def dsa_workspace_size(mode, B, total_tokens, max_ctx, H, k) -> int:
    return int(_lib.dsa_workspace_size(int(mode), int(B), int(total_tokens), int(max_ctx), int(H), int(k)))


def dsa_attn_distribution_dense(q, latent: Desc, lse, B, H, row_begin, row_end, sm_scale, p_out, stream=None):
    """p_out [row_end - row_begin, ld]: head-averaged attention over each row's causal prefix."""
    _check(_lib.dsa_attn_distribution_dense(_ptr(q), latent.ref(), _ptr(lse), int(B), int(H), int(row_begin),
                                            int(row_end), float(sm_scale), _ptr(p_out), p_out.stride(0),
                                            _stream(stream)), "dsa_attn_distribution_dense")
    return p_out


def dsa_indexer_backward(q_fp8, q_scale, w, keys: Desc, B, H_I, d_I, idx, grad, dw, dq, dk, stream=None):
    """Gradients of the indexer's inputs (dw [T, H_I], dq [T, H_I, d_I], dk [T, d_I], fp32) from
    d loss / d I on each token's entries (idx / grad [T, k])."""
    _check(_lib.dsa_indexer_backward(_ptr(q_fp8), _ptr(q_scale), _q_scale_heads(q_scale, H_I), _ptr(w), keys.ref(),
                                     int(B), int(H_I), int(d_I), _ptr(idx), _ptr(grad), idx.shape[1], _ptr(dw),
                                     _ptr(dq), _ptr(dk), _stream(stream)), "dsa_indexer_backward")
    return dw, dq, dk


def dsa_decode_select_workspace_size(B, max_ctx) -> int:
    return int(_lib.dsa_decode_select_workspace_size(int(B), int(max_ctx)))


def dsa_indexer_topk_decode(q_fp8, q_scale, w, keys: Desc, B, H_I, d_I, k, idx_out, workspace, stream=None):
    """Fused decode selection: paged indexer + per-sequence top-k; idx_out [B, k] (ascending,
    -1 padded); workspace is a uint8 device tensor of dsa_decode_select_workspace_size bytes."""
    _check(_lib.dsa_indexer_topk_decode(_ptr(q_fp8), _ptr(q_scale), _q_scale_heads(q_scale, H_I), _ptr(w),
                                        keys.ref(), int(B), int(H_I), int(d_I), int(k), _ptr(idx_out),
                                        _ptr(workspace), workspace.numel() * workspace.element_size(),
                                        _stream(stream)), "dsa_indexer_topk_decode")
    return idx_out


def dsa_device_error(stream=None) -> int:
    code = _I32(0)
    _check(_lib.dsa_device_error(ctypes.byref(code), _stream(stream)), "dsa_device_error")
    return int(code.value)


def dsa_indexer_topk(q_fp8, q_scale, w, keys: Desc, B, H_I, d_I, k, idx_out, stream=None):
    """Fused indexer + top-k for prefill: idx_out [T, k] (ascending, -1 padded)."""
    _check(_lib.dsa_indexer_topk(_ptr(q_fp8), _ptr(q_scale), _q_scale_heads(q_scale, H_I), _ptr(w), keys.ref(),
                                 int(B), int(H_I), int(d_I), int(k),
                                 _ptr(idx_out), _stream(stream)), "dsa_indexer_topk")
    return idx_out


def dsa_sparse_mla_decode_noalloc(q, latent: Desc, idx, B, H, k, sm_scale, out, lse=None, stream=None):
    """Decode sparse MLA that allocates nothing: partial results go to the library's own
    per-device scratch array.  Calls that overlap on the GPU share that array and race."""
    _check(_lib.dsa_sparse_mla_decode_noalloc(_ptr(q), latent.ref(), _ptr(idx), int(B), int(H), int(k),
                                              float(sm_scale), _ptr(out), _ptr(lse), _stream(stream)),
           "dsa_sparse_mla_decode_noalloc")
    return out


def dsa_row_partition(L, k, parts, indexer_cost, mla_cost):
    """Row-block boundaries [0, ..., L] of balanced estimated cost for sharding one prefill of
    length L over `parts` GPUs (host only; see dsa_row_partition in include/dsa.h)."""
    out = (_I64 * (int(parts) + 1))()
    _check(_lib.dsa_row_partition(int(L), int(k), int(parts), float(indexer_cost), float(mla_cost), out),
           "dsa_row_partition")
    return [int(x) for x in out]
