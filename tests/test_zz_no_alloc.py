"""The decode entry point that allocates nothing (its split partials live in a scratch array
the library holds in device memory) must give the same result as the workspace entry point,
call after call.  This file is collected last on purpose."""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
import synth
from helpers import assert_attention_close

pytestmark = pytest.mark.gpu


def _inputs():
    B, k = 5, 2048
    d = synth.decode_inputs(B=B, ctx_lo=1, ctx_hi=5000, H_I=64, d_I=128, H=128, seed=12, device="cuda",
                            ctx=[1, 777, 2048, 3000, 4999])
    idx = torch.full((B, k), -1, dtype=torch.int32, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(5)
    for b, c in enumerate(d["ctx_host"]):
        m = min(k, c)
        idx[b, :m] = torch.sort(torch.randperm(c, generator=g, device="cuda")[:m]).values.to(torch.int32)
    return d, idx, B, k


def test_noalloc_decode_matches_workspace_decode_twice():
    import sparse_attention_09_b200 as dsa
    d, idx, B, k = _inputs()
    sm = 1.0 / math.sqrt(576)
    latent = dsa.paged_desc(d["latent_cache"], d["block_table"], d["ctx"], d["max_ctx"])
    ws = torch.empty(dsa.dsa_workspace_size(dsa.DSA_MODE_DECODE, B, 0, d["max_ctx"], 128, k), dtype=torch.uint8,
                     device="cuda")
    ref = torch.empty((B, 128, 512), dtype=torch.bfloat16, device="cuda")
    ref_lse = torch.empty((B, 128), device="cuda")
    dsa.dsa_sparse_mla_decode(d["q"], latent, idx, B, 128, k, sm, ref, ref_lse, ws)
    for call in range(2):
        out = torch.full((B, 128, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((B, 128), float("nan"), device="cuda")
        st = dsa._lib.dsa_sparse_mla_decode_noalloc(
            ctypes.c_void_p(d["q"].data_ptr()), latent.ref(), ctypes.c_void_p(idx.data_ptr()), B, 128, k,
            ctypes.c_float(sm), ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(lse.data_ptr()),
            ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == dsa.DSA_OK, dsa.dsa_status_string(st)
        assert dsa.dsa_device_error() == 0
        for b in range(B):
            assert_attention_close(out[b].float().cpu().numpy(), ref[b].float().cpu().numpy(), f"call {call} seq {b}")
        assert np.allclose(lse.cpu().numpy(), ref_lse.cpu().numpy(), rtol=0, atol=1e-2)


def test_noalloc_decode_rejects_sizes_beyond_its_scratch():
    import sparse_attention_09_b200 as dsa
    d, idx, B, k = _inputs()
    latent = dsa.paged_desc(d["latent_cache"], d["block_table"], d["ctx"], d["max_ctx"])
    big_B = 4096  # partials of 4096 x 128 heads (1 split) need 1.08 GB: more than the fixed scratch
    st = dsa._lib.dsa_sparse_mla_decode_noalloc(
        ctypes.c_void_p(d["q"].data_ptr()), latent.ref(), ctypes.c_void_p(idx.data_ptr()), big_B, 128, k,
        ctypes.c_float(0.04), ctypes.c_void_p(d["q"].data_ptr()), None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == dsa.DSA_ERR_UNSUPPORTED


def test_noalloc_decode_size_edge_at_128_heads():
    """At H = 128 the partials of B = 127 sequences (one split each) fit the scratch array and
    B = 128 do not: the last size that fits runs, equals the workspace call and agrees with the
    oracle on sampled sequences; the first that does not is refused before any launch."""
    import sparse_attention_09_b200 as dsa
    B, k = 127, 2048
    d = synth.decode_inputs(B=B, ctx_lo=1, ctx_hi=2500, H_I=64, d_I=128, H=128, seed=31, device="cuda")
    idx = torch.full((B, k), -1, dtype=torch.int32, device="cuda")
    g = torch.Generator(device="cuda").manual_seed(8)
    for b, c in enumerate(d["ctx_host"]):
        m = min(k, c)
        idx[b, :m] = torch.sort(torch.randperm(c, generator=g, device="cuda")[:m]).values.to(torch.int32)
    sm = 1.0 / math.sqrt(576)
    latent = dsa.paged_desc(d["latent_cache"], d["block_table"], d["ctx"], d["max_ctx"])
    ws = torch.empty(dsa.dsa_workspace_size(dsa.DSA_MODE_DECODE, B, 0, d["max_ctx"], 128, k), dtype=torch.uint8,
                     device="cuda")
    ref = torch.empty((B, 128, 512), dtype=torch.bfloat16, device="cuda")
    dsa.dsa_sparse_mla_decode(d["q"], latent, idx, B, 128, k, sm, ref, None, ws)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    out = torch.full((B, 128, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
    st = dsa._lib.dsa_sparse_mla_decode_noalloc(ctypes.c_void_p(d["q"].data_ptr()), latent.ref(),
                                                ctypes.c_void_p(idx.data_ptr()), B, 128, k, ctypes.c_float(sm),
                                                ctypes.c_void_p(out.data_ptr()), None, stream)
    assert st == dsa.DSA_OK, dsa.dsa_status_string(st)
    assert dsa.dsa_device_error() == 0
    assert torch.equal(out, ref)  # the same kernels on the same inputs
    for b in (0, 63, B - 1):        # and the oracle on the selected latent rows
        seq = synth.decode_seq_numpy(d, b)
        lat = oracle.paged_gather(seq["latent_cache"], seq["block_table"], seq["ctx"])
        sel = idx[b].cpu().numpy()
        want, _ = oracle.sparse_mla_token(seq["q"], lat, sel[sel >= 0], sm)
        assert_attention_close(out[b].float().cpu().numpy(), want, f"seq {b}")
    poison = out.clone()
    st = dsa._lib.dsa_sparse_mla_decode_noalloc(ctypes.c_void_p(d["q"].data_ptr()), latent.ref(),
                                                ctypes.c_void_p(idx.data_ptr()), B + 1, 128, k, ctypes.c_float(sm),
                                                ctypes.c_void_p(out.data_ptr()), None, stream)
    assert st == dsa.DSA_ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert torch.equal(out, poison)  # nothing was launched
