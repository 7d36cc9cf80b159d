"""Per-token FP8 quantiser kernel (dsa_quantize_fp8) against the oracle: codes and scales
bit-exact, on small shapes with edge rows and on sampled rows of the full q_I of the
L=131072 prefill ([131072, 64 x 128] bf16)."""

import numpy as np
import pytest
import torch

import oracle
import synth

pytestmark = pytest.mark.gpu


def _run(x):
    import sparse_attention_09_b200 as dsa
    rows = x.shape[0]
    cols = x.numel() // max(rows, 1)
    codes = torch.empty((rows, cols), dtype=torch.uint8, device="cuda")
    scale = torch.empty((rows,), dtype=torch.float32, device="cuda")
    dsa.dsa_quantize_fp8(x, codes, scale)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scale.cpu().numpy()


def _check(x_gpu, rows=None):
    codes, scale = _run(x_gpu)
    xr = x_gpu.float().cpu().numpy().reshape(x_gpu.shape[0], -1)
    sel = np.arange(xr.shape[0]) if rows is None else np.asarray(rows)
    ref_codes, ref_scale = oracle.quantize_fp8_rows(xr[sel])
    assert np.array_equal(scale[sel].view(np.uint32), ref_scale.view(np.uint32)), "scales differ"
    assert np.array_equal(codes[sel], ref_codes), "codes differ"


@pytest.mark.parametrize("rows,cols", [(1, 8), (3, 16), (37, 128), (64, 256), (300, 8192), (9, 136), (7, 2048),
                                       (5, 4104), (3, 8184), (2, 8200)])
def test_quantiser_random_rows(rows, cols):
    g = torch.Generator(device="cuda")
    g.manual_seed(rows * 1000 + cols)
    mag = torch.exp(torch.randn((rows, 1), generator=g, device="cuda") * 4)   # scales over many decades
    x = (torch.randn((rows, cols), generator=g, device="cuda") * mag).to(torch.bfloat16)
    _check(x)


def test_quantiser_edge_rows():
    cols = 64
    x = torch.randn((8, cols), device="cuda").to(torch.bfloat16)
    x[0] = 0                                            # all zero -> scale 1, codes 0
    x[1] = -0.0                                         # negative zeros keep their sign bit
    x[2, 5] = 3e38                                      # one huge element dominates
    x[3] = 1e-38                                        # tiny row
    x[4] = torch.tensor([1.0, -1.0] * (cols // 2))      # exact ties at the largest code
    x[5, 7] = float("nan")                              # NaN ignored by the maximum, encodes NaN
    x[6] = torch.linspace(-448, 448, cols)
    x[7, :] = 2.0 ** -20                                # constant row
    _check(x)


def test_quantiser_full_q_index_shape_sampled_rows():
    g = torch.Generator(device="cuda")
    g.manual_seed(41)
    T, H_I, d_I = 131072, 64, 128
    x = torch.empty((T, H_I, d_I), dtype=torch.bfloat16, device="cuda")
    for t0 in range(0, T, 8192):
        x[t0:t0 + 8192] = torch.randn((8192, H_I, d_I), generator=g, device="cuda").to(torch.bfloat16)
    codes = torch.empty((T, H_I * d_I), dtype=torch.uint8, device="cuda")
    scale = torch.empty((T,), dtype=torch.float32, device="cuda")
    import sparse_attention_09_b200 as dsa
    dsa.dsa_quantize_fp8(x, codes, scale)
    torch.cuda.synchronize()
    rows = synth.sample_rows(T, 1, 48, seed=4)
    xr = x.reshape(T, -1)[torch.as_tensor(rows, device="cuda")].float().cpu().numpy()
    ref_codes, ref_scale = oracle.quantize_fp8_rows(xr)
    got_codes = codes[torch.as_tensor(rows, device="cuda")].cpu().numpy()
    got_scale = scale[torch.as_tensor(rows, device="cuda")].cpu().numpy()
    assert np.array_equal(got_scale.view(np.uint32), ref_scale.view(np.uint32))
    assert np.array_equal(got_codes, ref_codes)
