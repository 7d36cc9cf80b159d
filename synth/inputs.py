"""Input recipes for the DSA workloads.

Workloads (shapes of the DSA prefill/decode cases the library is measured on):

* ``tiny_256``      batch 1, L=256, indexer 4 heads x d_I=64, top-k 64, 16 query heads.
* ``prefill_8k``    batch 1, L=8192, indexer 64 heads x d_I=128 (FP8), top-k 2048, 128 heads.
* ``prefill_2x32k`` batch 2, L=32768 each (packed by cu_seqlens), otherwise as prefill_8k.
* ``decode_64``     64 sequences, one query each, context ~ U[8192, 131072], paged caches with
                    64-token blocks drawn from a seeded permutation of the block pool.
* ``prefill_128k``  batch 1, L=131072, as prefill_8k plus 5% of the indexer keys at 4x norm.

Distributions: indexer queries/keys N(0,1) (tiny_256: N(0,1)/sqrt(64) rounded to bf16),
quantised per token to e4m3 with scale = amax/448 (scale 1 for an all-zero token); head
weights w ~ N(0,1)/8 (tiny_256: U(0,1)); q and the latent ~ N(0,1)/sqrt(576) in bf16.
The latent is one 576-d row per token (512 "nope" + 64 "rope" dims), contiguous per sequence
in prefill and paged in decode.

All draws come from torch generators seeded per tensor; the tensors are produced on the
device that will consume them and copied to the host for the oracle.
"""

from __future__ import annotations

import math

import numpy as np
import torch

E4M3_MAX = 448.0
D_QK = 576
D_V = 512

WORKLOADS = {
    "tiny_256": dict(kind="prefill", seqlens=[256], H_I=4, d_I=64, k=64, H=16, w_dist="uniform",
                     idx_std=1.0 / math.sqrt(64), idx_bf16=True, planted=0.0, seed=1),
    "prefill_8k": dict(kind="prefill", seqlens=[8192], H_I=64, d_I=128, k=2048, H=128,
                       w_dist="normal8", idx_std=1.0, idx_bf16=False, planted=0.0, seed=11),
    "prefill_2x32k": dict(kind="prefill", seqlens=[32768, 32768], H_I=64, d_I=128, k=2048, H=128,
                          w_dist="normal8", idx_std=1.0, idx_bf16=False, planted=0.0, seed=21),
    "decode_64": dict(kind="decode", B=64, ctx_lo=8192, ctx_hi=131072, block_size=64, H_I=64,
                      d_I=128, k=2048, H=128, w_dist="normal8", idx_std=1.0, seed=31),
    "prefill_128k": dict(kind="prefill", seqlens=[131072], H_I=64, d_I=128, k=2048, H=128,
                         w_dist="normal8", idx_std=1.0, idx_bf16=False, planted=0.05, seed=41),
}

_CHUNK = 2048  # tokens per generator call, so that large tensors are drawn without fp32 copies


def _gen(device, seed: int, stream: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) * 1000003 + int(stream))
    return g


def quantize_e4m3_per_token(x: torch.Tensor):
    """Per-token e4m3 encoding of x [T, ...]: scale = amax/448 (1 for an all-zero token),
    codes = round-to-nearest-even(x / scale).  Returns (codes uint8 [T, ...], scale f32 [T])."""
    xf = x.float()
    amax = xf.abs().reshape(xf.shape[0], -1).amax(dim=1)
    scale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax))
    shape = (-1,) + (1,) * (xf.dim() - 1)
    y = (xf / scale.reshape(shape)).clamp_(-E4M3_MAX, E4M3_MAX)
    codes = y.to(torch.float8_e4m3fn).view(torch.uint8)
    return codes.contiguous(), scale.float().contiguous()


def _normal_bf16(shape, std, g, device):
    """N(0, std^2) drawn in token chunks straight into a bf16 tensor."""
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    T = shape[0]
    for t0 in range(0, T, _CHUNK):
        t1 = min(T, t0 + _CHUNK)
        out[t0:t1] = (torch.randn((t1 - t0,) + tuple(shape[1:]), generator=g, device=device) * std).to(torch.bfloat16)
    return out


def _indexer_operand(shape, std, as_bf16, g, device, planted=0.0, g_plant=None, per_head=False):
    """e4m3 codes and fp32 scales of a seeded normal operand [T, ...]: one scale per token, or
    with per_head (shape [T, H_I, d_I]) one per (token, head), head j drawn 2^-(j mod 8) times
    smaller so that the heads' scales differ."""
    T = shape[0]
    codes = torch.empty(shape, dtype=torch.uint8, device=device)
    scales = torch.empty((T, shape[1]) if per_head else (T,), dtype=torch.float32, device=device)
    for t0 in range(0, T, _CHUNK):
        t1 = min(T, t0 + _CHUNK)
        x = torch.randn((t1 - t0,) + tuple(shape[1:]), generator=g, device=device) * std
        if per_head:
            x *= (2.0 ** -(torch.arange(shape[1], device=device) % 8)).reshape(1, -1, 1)
        if as_bf16:
            x = x.to(torch.bfloat16).float()
        if planted > 0:
            hot = torch.rand((t1 - t0,), generator=g_plant, device=device) < planted
            x[hot] *= 4.0
        if per_head:
            c, s = quantize_e4m3_per_token(x.reshape(-1, shape[2]))
            c, s = c.reshape(x.shape), s.reshape(t1 - t0, shape[1])
        else:
            c, s = quantize_e4m3_per_token(x)
        codes[t0:t1] = c
        scales[t0:t1] = s
    return codes, scales


def _weights(shape, dist, g, device):
    if dist == "uniform":
        return torch.rand(shape, generator=g, device=device, dtype=torch.float32)
    if dist == "normal8":
        return torch.randn(shape, generator=g, device=device, dtype=torch.float32) / 8.0
    raise ValueError(dist)


def prefill_inputs(seqlens, H_I, d_I, H, *, seed, device, w_dist="normal8", idx_std=1.0,
                   idx_bf16=False, planted=0.0, q_scale_per_head=False, **_):
    """Packed prefill inputs for sequences of the given lengths (queries == keys per sequence).

    Returns a dict of device tensors: cu_seqlens [B+1] i32, q8 [T,H_I,d_I] u8, q_scale [T]
    (or [T,H_I] with q_scale_per_head), w [T,H_I], k8 [T,d_I] u8, k_scale [T], q [T,H,576]
    bf16, latent [T,576] bf16, plus the host-side ``seqlens`` list.
    """
    seqlens = [int(x) for x in seqlens]
    T = sum(seqlens)
    cu = torch.tensor(np.concatenate([[0], np.cumsum(seqlens)]), dtype=torch.int32, device=device)
    q8, q_scale = _indexer_operand((T, H_I, d_I), idx_std, idx_bf16, _gen(device, seed, 1), device,
                                   per_head=q_scale_per_head)
    k8, k_scale = _indexer_operand((T, d_I), idx_std, idx_bf16, _gen(device, seed, 2), device,
                                   planted=planted, g_plant=_gen(device, seed, 7))
    w = _weights((T, H_I), w_dist, _gen(device, seed, 3), device)
    q = _normal_bf16((T, H, D_QK), 1.0 / math.sqrt(D_QK), _gen(device, seed, 4), device)
    latent = _normal_bf16((T, D_QK), 1.0 / math.sqrt(D_QK), _gen(device, seed, 5), device)
    return dict(cu_seqlens=cu, seqlens=seqlens, q8=q8, q_scale=q_scale, w=w, k8=k8,
                k_scale=k_scale, q=q, latent=latent, H_I=H_I, d_I=d_I, H=H)


def prefill_block_inputs(L, row_begin, row_end, H_I, d_I, H, *, seed, device, w_dist="normal8", idx_std=1.0,
                         planted=0.0, mla=True, **_):
    """Inputs for a block of query rows [row_begin, row_end) of ONE sequence of length L: the keys
    (k8, k_scale) and latent of the whole sequence, the query-side tensors (q8, q_scale, w, q) of
    the block only, with the distributions prefill_inputs draws (a small-footprint case of the
    same workload for counter captures; the values are not those rows of prefill_inputs).
    With mla=False the attention operands (q, latent) are left out (None): indexer-only cases."""
    R = int(row_end) - int(row_begin)
    cu = torch.tensor([0, int(L)], dtype=torch.int32, device=device)
    q8, q_scale = _indexer_operand((R, H_I, d_I), idx_std, False, _gen(device, seed, 11), device)
    k8, k_scale = _indexer_operand((int(L), d_I), idx_std, False, _gen(device, seed, 12), device,
                                   planted=planted, g_plant=_gen(device, seed, 17))
    w = _weights((R, H_I), w_dist, _gen(device, seed, 13), device)
    q = _normal_bf16((R, H, D_QK), 1.0 / math.sqrt(D_QK), _gen(device, seed, 14), device) if mla else None
    latent = _normal_bf16((int(L), D_QK), 1.0 / math.sqrt(D_QK), _gen(device, seed, 15), device) if mla else None
    return dict(cu_seqlens=cu, seqlens=[int(L)], q8=q8, q_scale=q_scale, w=w, k8=k8, k_scale=k_scale, q=q,
                latent=latent, H_I=H_I, d_I=d_I, H=H, row_begin=int(row_begin), row_end=int(row_end))


def decode_inputs(B, ctx_lo, ctx_hi, H_I, d_I, H, *, seed, device, block_size=64, w_dist="normal8",
                  idx_std=1.0, ctx=None, spare_blocks=3, q_scale_per_head=False, **_):
    """Paged decode inputs: one query per sequence over a cache of ctx[b] tokens.

    Blocks of ``block_size`` tokens are taken from a pool in the order of a seeded
    permutation, so a sequence's blocks are scattered.  Returns device tensors ctx [B] i32,
    block_table [B,max_blocks] i32 (unused entries -1), kcache8 [nb,bs,d_I] u8,
    kscale_cache [nb,bs] f32, latent_cache [nb,bs,576] bf16, q8 [B,H_I,d_I], q_scale [B]
    (or [B,H_I] with q_scale_per_head), w [B,H_I], q [B,H,576], plus host copies ``ctx_host``
    and ``max_ctx``.
    """
    rs = np.random.default_rng(int(seed))
    if ctx is None:
        ctx = rs.integers(int(ctx_lo), int(ctx_hi) + 1, size=int(B))
    ctx = np.asarray(ctx, dtype=np.int64)
    nblk_seq = (ctx + block_size - 1) // block_size
    max_blocks = int(nblk_seq.max())
    num_blocks = int(nblk_seq.sum()) + int(spare_blocks)
    perm = rs.permutation(num_blocks)
    bt = np.full((int(B), max_blocks), -1, dtype=np.int32)
    off = 0
    for b in range(int(B)):
        n = int(nblk_seq[b])
        bt[b, :n] = perm[off:off + n]
        off += n
    kcache8, kscale = _indexer_operand((num_blocks * block_size, d_I), idx_std, False, _gen(device, seed, 2), device)
    kcache8 = kcache8.reshape(num_blocks, block_size, d_I)
    kscale = kscale.reshape(num_blocks, block_size)
    latent = _normal_bf16((num_blocks * block_size, D_QK), 1.0 / math.sqrt(D_QK), _gen(device, seed, 5), device)
    latent = latent.reshape(num_blocks, block_size, D_QK)
    q8, q_scale = _indexer_operand((int(B), H_I, d_I), idx_std, False, _gen(device, seed, 1), device,
                                   per_head=q_scale_per_head)
    w = _weights((int(B), H_I), w_dist, _gen(device, seed, 3), device)
    q = _normal_bf16((int(B), H, D_QK), 1.0 / math.sqrt(D_QK), _gen(device, seed, 4), device)
    return dict(ctx=torch.tensor(ctx, dtype=torch.int32, device=device), ctx_host=ctx.tolist(),
                max_ctx=int(ctx.max()), block_table=torch.tensor(bt, device=device),
                kcache8=kcache8, kscale_cache=kscale, latent_cache=latent, q8=q8, q_scale=q_scale,
                w=w, q=q, block_size=block_size, num_blocks=num_blocks, H_I=H_I, d_I=d_I, H=H, B=int(B))


def exact_prefill_inputs(seqlens, H_I, d_I, H, *, seed, device, small_scores=False, q_scale_per_head=False):
    """Inputs on which every float32 partial sum of the indexer is exact.

    e4m3 codes of small integers |x| <= 4 (dots of 128 terms stay below 2^11), head weights
    multiples of 1/16 in [-1, 1], per-token scales powers of two.  Every partial sum of
    w * ReLU(dot) then needs at most 21 significant bits, so float32 accumulation in any
    order is exact and GPU and CPU scores agree bit for bit.
    With small_scores the integers are in [-1, 1] (few distinct scores, many ties).  With
    q_scale_per_head the query scales are drawn per (token, head), [T, H_I].
    """
    seqlens = [int(x) for x in seqlens]
    T = sum(seqlens)
    rs = np.random.default_rng(int(seed))
    lim = 1 if small_scores else 4
    ints_q = rs.integers(-lim, lim + 1, size=(T, H_I, d_I)).astype(np.float32)
    ints_k = rs.integers(-lim, lim + 1, size=(T, d_I)).astype(np.float32)
    q8 = torch.from_numpy(ints_q).to(torch.float8_e4m3fn).view(torch.uint8)
    k8 = torch.from_numpy(ints_k).to(torch.float8_e4m3fn).view(torch.uint8)
    q_scale = torch.from_numpy(2.0 ** rs.integers(-3, 2, size=T)).float()
    k_scale = torch.from_numpy(2.0 ** rs.integers(-3, 2, size=T)).float()
    if q_scale_per_head:
        q_scale = torch.from_numpy(2.0 ** rs.integers(-3, 2, size=(T, H_I))).float()
    w = torch.from_numpy(rs.integers(-16, 17, size=(T, H_I)) / 16.0).float()
    base = prefill_inputs(seqlens, H_I, d_I, H, seed=seed, device=device)
    base.update(q8=q8.to(device), k8=k8.to(device), q_scale=q_scale.to(device),
                k_scale=k_scale.to(device), w=w.to(device))
    return base


def tie_heavy_scores(rows, n, levels, *, seed, device):
    """Score buffer whose entries take only `levels` distinct values (including -0.0/+0.0)."""
    rs = np.random.default_rng(int(seed))
    vals = np.linspace(-1.0, 1.0, int(levels)).astype(np.float32)
    s = vals[rs.integers(0, int(levels), size=(int(rows), int(n)))]
    zero = s == 0
    s[zero & (rs.random(s.shape) < 0.5)] = -0.0
    return torch.from_numpy(s).to(device)


def sample_rows(L: int, k: int, count: int, seed: int):
    """Stratified query rows of a length-L sequence: 0, k-1, k, L-1 plus seeded random rows."""
    rs = np.random.default_rng(int(seed))
    fixed = [0, min(k - 1, L - 1), min(k, L - 1), L - 1]
    rest = rs.choice(L, size=max(0, count - len(fixed)), replace=False).tolist()
    return sorted(set(fixed + rest))


class SampledRows:
    """The rows of a per-token array for a sample of tokens only: ``x[t]`` is token t's row
    (a KeyError for a token outside the sample) and ``shape`` is the whole array's, so code
    written against the whole array reads the sample without it being allocated."""

    def __init__(self, rows: dict, shape):
        self._rows = {int(t): v for t, v in rows.items()}
        self.shape = tuple(shape)

    def __getitem__(self, t):
        return self._rows[int(t)]


def seq_slice_numpy(inp: dict, b: int, rows=None):
    """Host copies (numpy) of sequence b of prefill inputs, for the oracle.

    rows restricts q and the indexer queries to those local rows (keys stay whole); q is then
    a SampledRows (a whole [L, H, 576] float64 q of a long sequence would take tens of GB)."""
    s0 = int(inp["cu_seqlens"][b].item())
    s1 = int(inp["cu_seqlens"][b + 1].item())
    out = dict(k8=inp["k8"][s0:s1].cpu().numpy(), k_scale=inp["k_scale"][s0:s1].double().cpu().numpy(),
               latent=inp["latent"][s0:s1].float().cpu().numpy().astype(np.float64), L=s1 - s0, start=s0)
    if rows is None:
        out.update(q8=inp["q8"][s0:s1].cpu().numpy(), q_scale=inp["q_scale"][s0:s1].double().cpu().numpy(),
                   w=inp["w"][s0:s1].double().cpu().numpy(), q=inp["q"][s0:s1].float().cpu().numpy().astype(np.float64))
    else:
        L = s1 - s0
        r = torch.as_tensor(list(rows), dtype=torch.long, device=inp["q8"].device) + s0
        H_I, d_I = inp["q8"].shape[1], inp["q8"].shape[2]
        H = inp["q"].shape[1]
        q8 = np.zeros((L, H_I, d_I), np.uint8)
        qs = np.ones((L,) + tuple(inp["q_scale"].shape[1:]))
        w = np.zeros((L, H_I))
        rl = list(rows)
        q8[rl] = inp["q8"][r].cpu().numpy()
        qs[rl] = inp["q_scale"][r].double().cpu().numpy()
        w[rl] = inp["w"][r].double().cpu().numpy()
        qr = inp["q"][r].float().cpu().numpy().astype(np.float64)
        q = SampledRows({t: qr[i] for i, t in enumerate(rl)}, (L, H, D_QK))
        out.update(q8=q8, q_scale=qs, w=w, q=q)
    return out


def decode_seq_numpy(inp: dict, b: int, keep_paging: bool = True):
    """Host copies (numpy) of decode sequence b, for the oracle.

    Only the blocks the sequence uses are copied.  With keep_paging they keep their pool
    order and the block table is remapped onto the copied subset (so the oracle still reads
    through a scattered table); otherwise the blocks are copied in logical order.
    """
    bs = inp["block_size"]
    nb_used = max(1, (inp["ctx_host"][b] + bs - 1) // bs)
    bt = inp["block_table"][b, :nb_used].long()
    if keep_paging:
        pool = torch.unique(bt)                       # sorted physical ids
        local = torch.searchsorted(pool, bt)          # table over the copied subset
    else:
        pool = bt
        local = torch.arange(nb_used, device=bt.device)
    qs = inp["q_scale"][b]
    return dict(q8=inp["q8"][b].cpu().numpy(),
                q_scale=float(qs.item()) if qs.dim() == 0 else qs.double().cpu().numpy(),
                w=inp["w"][b].double().cpu().numpy(), kcache8=inp["kcache8"][pool].cpu().numpy(),
                kscale_cache=inp["kscale_cache"][pool].double().cpu().numpy(),
                latent_cache=inp["latent_cache"][pool].float().cpu().numpy().astype(np.float64),
                block_table=local.cpu().numpy(), ctx=inp["ctx_host"][b],
                q=inp["q"][b].float().cpu().numpy().astype(np.float64))
