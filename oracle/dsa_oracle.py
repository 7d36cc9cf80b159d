"""Plain float64 definition of the DSA hot path: lightning indexer -> top-k -> sparse MLA (MQA).

TEST INFRASTRUCTURE ONLY (see the package docstring for who may use it and for the page
citations [MZ], [JD], [36], [DP], [TW]).

Nothing here is blocked, fused or reordered beyond the definitions; numpy's float64 matmul
is the only library primitive used as a step.  Readings taken where the pages are silent:

* FP8 means OCP E4M3FN (bias 7, subnormals, max 448, S.1111.111 = NaN, no infinities).
* Dequantisation is per token: q_I[t,j,:] = e4m3(q8[t,j,:]) * q_scale[t],
  k_I[s,:] = e4m3(k8[s,:]) * k_scale[s]; or, for queries quantised per (token, head),
  q_I[t,j,:] = e4m3(q8[t,j,:]) * q_scale[t,j].
* "All preceding tokens" is the causal prefix s <= t (the query's own key included), so a
  prefill row keeps min(k, t+1) entries; a decode query sits at position ctx-1 and sees all
  ctx cached keys.
* Scores are computed in float64 and rounded once to float32 (round to nearest even) before
  selection; selection orders by score descending, ties to the lower index, -0.0 == +0.0.
* Selected indices are emitted in ascending order, padded with -1.
* Attention: logits = sm_scale * q[t,h,:576] . c[i,:576], softmax over the selected i, value
  = c[i,:512] (the first 512 latent dims); lse is the natural-log sum of exp(logits).
"""

from __future__ import annotations

import numpy as np

E4M3_MAX = 448.0


# ---------------------------------------------------------------------------------------------
# FP8 e4m3 ([MZ] "工作原理": the indexer may run in FP8; [JD] 2.1: low-precision FP8 compute)
# ---------------------------------------------------------------------------------------------
def e4m3_table() -> np.ndarray:
    """Value of every byte under OCP E4M3FN, written from the format definition.

    Bit 7 is the sign, bits 6..3 the exponent (bias 7), bits 2..0 the mantissa.  Exponent 0
    encodes subnormals m/8 * 2^-6; exponent 15 with mantissa 7 is NaN; there is no infinity.
    """
    table = np.empty(256, dtype=np.float64)
    for code in range(256):
        sign = -1.0 if code & 0x80 else 1.0
        exponent = (code >> 3) & 0xF
        mantissa = code & 0x7
        if exponent == 0xF and mantissa == 0x7:
            table[code] = np.nan
        elif exponent == 0:
            table[code] = sign * (mantissa / 8.0) * 2.0 ** (1 - 7)
        else:
            table[code] = sign * (1.0 + mantissa / 8.0) * 2.0 ** (exponent - 7)
    return table


_E4M3 = e4m3_table()


def decode_e4m3(codes: np.ndarray) -> np.ndarray:
    """float64 values of an array of e4m3 bytes."""
    return _E4M3[np.asarray(codes, dtype=np.uint8)]


def encode_e4m3(y: np.ndarray) -> np.ndarray:
    """e4m3 bytes of the values y: nearest representable value, ties to the even mantissa
    (round to nearest even), magnitudes >= 448 saturate to 448, NaN -> 0x7F with its sign
    bit; the sign of zero is kept.

    Written from the format definition: the 127 non-negative finite values (codes 0..126)
    increase with the code, so a magnitude is bracketed by two consecutive codes and the
    nearer one (the even one on a tie) is taken.
    """
    y = np.asarray(y, dtype=np.float64)
    mag = np.abs(y)
    pos = _E4M3[:127]                                   # codes 0..126, increasing
    lo = np.clip(np.searchsorted(pos, mag, side="right") - 1, 0, 126)
    hi = np.minimum(lo + 1, 126)
    dlo = mag - pos[lo]
    dhi = pos[hi] - mag
    pick_hi = (dhi < dlo) | ((dhi == dlo) & (lo % 2 == 1))
    code = np.where(pick_hi, hi, lo)
    code = np.where(mag >= E4M3_MAX, 126, code)         # saturation (and +-inf)
    code = np.where(np.isnan(y), 0x7F, code)
    sign = np.where(np.signbit(y), 0x80, 0)
    return (code | sign).astype(np.uint8)


def quantize_fp8_rows(x: np.ndarray):
    """Per-token FP8 quantiser ([MZ] "工作原理": the indexer runs in FP8 with per-token
    scales): for each row, scale = amax|x| / 448 in IEEE float32 (1 for an all-zero row) and
    codes = e4m3(x / scale) with the quotient in IEEE float32.  NaN elements take no part in
    the maximum.  x: [rows, cols] values exactly representable in float32 (bf16 inputs are).
    Returns (codes uint8 [rows, cols], scale float32 [rows]).
    """
    x32 = np.asarray(x, dtype=np.float32)
    a = np.abs(x32)
    a = np.where(np.isnan(a), np.float32(0.0), a)
    amax = a.max(axis=1) if x32.shape[1] else np.zeros(x32.shape[0], np.float32)
    scale = np.where(amax > 0, amax / np.float32(E4M3_MAX), np.float32(1.0)).astype(np.float32)
    with np.errstate(invalid="ignore", divide="ignore"):
        y = (x32 / scale[:, None]).astype(np.float32)
    return encode_e4m3(y), scale


# ---------------------------------------------------------------------------------------------
# Lightning indexer ([MZ] "工作原理"; [36] "第一步：Lightning Indexer"; [DP] 二)
# ---------------------------------------------------------------------------------------------
def indexer_scores_query(q8: np.ndarray, q_scale: float, w: np.ndarray, k8: np.ndarray,
                         k_scale: np.ndarray) -> np.ndarray:
    """Index scores of one query token against a set of keys.

    I[s] = sum_j w[j] * ReLU(q_I[j] . k_I[s]) with q_I[j] = e4m3(q8[j]) * q_scale (one scale
    for the token, or q_scale[j] when given one per head) and k_I = e4m3(k8) * k_scale.
    q8: [H_I, d_I] bytes, q_scale: scalar or [H_I], w: [H_I], k8: [n, d_I] bytes,
    k_scale: [n].  Returns float64 [n].
    """
    qs = np.asarray(q_scale, np.float64)
    q = decode_e4m3(q8) * (qs[:, None] if qs.ndim == 1 else qs)   # [H_I, d_I], dequantised
    k = decode_e4m3(k8) * np.asarray(k_scale, np.float64)[:, None]  # [n, d_I]
    dots = q @ k.T                                              # [H_I, n]
    return np.asarray(w, np.float64) @ np.maximum(dots, 0.0)    # sum over indexer heads j


def indexer_magnitude_query(q8, q_scale, w, k8, k_scale) -> np.ndarray:
    """A[s] = sum_j |w[j]| * ReLU(q_I[j] . k_I[s]): the size of the terms that make up I[s].

    Used as the denominator of the relative score tolerance, since I itself can cancel when
    the head weights have mixed signs.
    """
    return indexer_scores_query(q8, q_scale, np.abs(np.asarray(w, np.float64)), k8, k_scale)


def indexer_scores(q8: np.ndarray, q_scale: np.ndarray, w: np.ndarray, k8: np.ndarray,
                   k_scale: np.ndarray, rows=None) -> np.ndarray:
    """Prefill index scores of one sequence, for the causal prefix of each query row.

    q8: [L, H_I, d_I], q_scale: [L] or [L, H_I], w: [L, H_I], k8: [L, d_I], k_scale: [L].
    Returns float64 [len(rows), L]: I[t, s] for s <= t and -inf for s > t.
    """
    L = k8.shape[0]
    rows = list(range(L)) if rows is None else list(rows)
    out = np.full((len(rows), L), -np.inf)
    for r, t in enumerate(rows):
        out[r, : t + 1] = indexer_scores_query(q8[t], q_scale[t], w[t], k8[: t + 1], k_scale[: t + 1])
    return out


# ---------------------------------------------------------------------------------------------
# Fine-grained token selection ([MZ] "工作原理": each query keeps the top-k entries, k = 2048;
# [36] "第二步：Fine-grained Token Selection"; [DP] 二)
# ---------------------------------------------------------------------------------------------
def order_key_f32(scores_f32: np.ndarray) -> np.ndarray:
    """Map float32 scores to uint32 keys whose unsigned order is the score order (-0 == +0)."""
    s = np.asarray(scores_f32, dtype=np.float32).copy()
    s[s == 0] = 0.0                                   # canonical +0
    u = s.view(np.uint32).astype(np.uint64)
    neg = (u & 0x80000000) != 0
    key = np.where(neg, (~u) & 0xFFFFFFFF, u | 0x80000000)
    return key.astype(np.uint32)


def topk_indices(scores: np.ndarray, m: int) -> np.ndarray:
    """Indices of the m largest entries of a score row (ties to the lower index), ascending.

    scores holds only the valid entries of the row (the causal prefix).  NaN is rejected.
    """
    s = np.asarray(scores, dtype=np.float64)
    if np.isnan(s).any():
        raise ValueError("NaN score")
    m = min(int(m), s.shape[0])
    order = np.lexsort((np.arange(s.shape[0]), -s))   # primary: score desc; secondary: index asc
    return np.sort(order[:m])


def topk_rows(scores: np.ndarray, row_len: np.ndarray, k: int) -> np.ndarray:
    """Row-wise top-k over the first row_len[r] entries of each row; int32 [rows, k], -1 padded."""
    scores = np.asarray(scores)
    out = np.full((scores.shape[0], k), -1, dtype=np.int32)
    for r in range(scores.shape[0]):
        sel = topk_indices(scores[r, : int(row_len[r])], k)
        out[r, : sel.shape[0]] = sel
    return out


# ---------------------------------------------------------------------------------------------
# Sparse MLA in MQA mode ([MZ] "挂在 MLA 上": every latent vector is shared by all query heads
# of a token; [JD] 2.1: MLA compresses K/V into a latent vector space; [MZ] "工作原理": attention
# runs only over the selected top-k entries)
# ---------------------------------------------------------------------------------------------
def sparse_mla_token(q: np.ndarray, latent: np.ndarray, sel: np.ndarray, sm_scale: float,
                     dv: int = 512):
    """Attention of all heads of one query over its selected latent rows.

    q: [H, D] (D = 576), latent: [n, D], sel: selected row indices (no padding).
    Key = the full 576-d latent row, value = its first dv dims.
    Returns (out [H, dv] float64, lse [H] float64, natural log).
    """
    c = np.asarray(latent, np.float64)[np.asarray(sel, np.int64)]   # [m, D]
    logits = float(sm_scale) * (np.asarray(q, np.float64) @ c.T)     # [H, m]
    mx = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - mx)
    z = e.sum(axis=1, keepdims=True)
    out = (e / z) @ c[:, :dv]
    lse = mx[:, 0] + np.log(z[:, 0])
    return out, lse


def attention_distribution_token(q: np.ndarray, latent: np.ndarray, sel: np.ndarray, sm_scale: float):
    """The main attention's distribution over a token's selected rows, aggregated over heads:
    p[i] = (1/H) sum_h softmax_i(sm_scale * q[h] . c[sel_i]) -- the target the indexer's
    distribution is aligned to by the KL loss ([MZ] 二, the two training stages of the indexer:
    a KL-divergence loss pulls the indexer's output distribution towards the main attention's;
    in the sparse stage over the selected set).
    Reading: "the main attention's distribution" of a query = its per-head attention
    probabilities summed over heads and normalised to total 1 (= the mean over heads).
    q: [H, D], latent: [n, D], sel: selected rows (no padding).  Returns float64 [len(sel)].
    """
    c = np.asarray(latent, np.float64)[np.asarray(sel, np.int64)]
    logits = float(sm_scale) * (np.asarray(q, np.float64) @ c.T)     # [H, m]
    mx = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - mx)
    return (e / e.sum(axis=1, keepdims=True)).mean(axis=0)


def indexer_kl(p: np.ndarray, scores: np.ndarray):
    """KL alignment loss of one token and its gradient ([MZ] 二, training of the indexer):
    q = softmax(scores) over the same rows as the target p;
    loss = KL(p || q) = sum_i p_i (log p_i - log q_i) (terms with p_i = 0 contribute 0);
    d loss / d scores_i = q_i - p_i.  Returns (loss float64, grad float64 [m])."""
    p = np.asarray(p, np.float64)
    s = np.asarray(scores, np.float64)
    mx = s.max()
    logq = s - mx - np.log(np.exp(s - mx).sum())
    pos = p > 0
    loss = float(np.sum(p[pos] * (np.log(p[pos]) - logq[pos])))
    return loss, np.exp(logq) - p


def attention_distribution_dense_token(q: np.ndarray, latent_prefix: np.ndarray, sm_scale: float):
    """Target of the dense warm-up stage for one query: the main attention's distribution over
    the query's whole causal prefix, averaged over heads ([MZ] 二 "两阶段继续预训练", dense
    warm-up: attention stays dense and the indexer alone is trained, by a KL loss, to match the
    main attention's output distribution; [36] "DSA 訓練的兩個階段", stage one).
    Reading: the same aggregation as the sparse stage (mean over heads of the per-head softmax),
    taken over every preceding token (rows 0..t) instead of the selected set.
    q: [H, D], latent_prefix: [t+1, D].  Returns float64 [t+1]."""
    c = np.asarray(latent_prefix, np.float64)
    logits = float(sm_scale) * (np.asarray(q, np.float64) @ c.T)     # [H, t+1]
    mx = logits.max(axis=1, keepdims=True)
    e = np.exp(logits - mx)
    return (e / e.sum(axis=1, keepdims=True)).mean(axis=0)


def indexer_backward_query(q8: np.ndarray, q_scale, w: np.ndarray, k8: np.ndarray, k_scale: np.ndarray,
                           g: np.ndarray):
    """Backward of the indexer for one query token ([MZ] 二 "两阶段继续预训练": the indexer is
    trained by the KL loss alone, with its input detached from the main model's graph).

    Given g[s] = d loss / d I[s] over a set of keys (the KL gradient, q_s - p_s), returns the
    gradient of sum_s g[s] * I[s] with I[s] = sum_j w[j] * ReLU(q_I[j] . k_I[s]):
      dw[j]    = sum_s g[s] * ReLU(a[j,s]),                 a[j,s] = q_I[j] . k_I[s]
      dq_I[j]  = sum_s g[s] * w[j] * [a[j,s] > 0] * k_I[s]
      dk_I[s]  = g[s] * sum_j w[j] * [a[j,s] > 0] * q_I[j]
    Readings: the gradient is taken with respect to the dequantised operands q_I =
    e4m3(q8) * q_scale and k_I = e4m3(k8) * k_scale (the real values the FP8 codes stand for;
    the quantiser passes it through); ReLU'(0) = 0.
    q8: [H_I, d_I], q_scale: scalar or [H_I], w: [H_I], k8: [n, d_I], k_scale: [n], g: [n].
    Returns (dw [H_I], dq [H_I, d_I], dk [n, d_I]), float64."""
    qs = np.asarray(q_scale, np.float64)
    q = decode_e4m3(q8) * (qs[:, None] if qs.ndim == 1 else qs)   # [H_I, d_I]
    k = decode_e4m3(k8) * np.asarray(k_scale, np.float64)[:, None]  # [n, d_I]
    g = np.asarray(g, np.float64)
    w = np.asarray(w, np.float64)
    a = q @ k.T                                                 # [H_I, n]
    dw = np.maximum(a, 0.0) @ g
    m = (a > 0.0) * w[:, None] * g[None, :]                     # d loss / d a[j, s]
    return dw, m @ k, m.T @ q


def indexer_backward(q8: np.ndarray, q_scale: np.ndarray, w: np.ndarray, k8: np.ndarray, k_scale: np.ndarray,
                     idx: np.ndarray, grad: np.ndarray):
    """Backward of the indexer over one sequence: token t's gradient grad[t, i] = d loss /
    d I[t, idx[t, i]] on its selected keys (idx -1 padded; in the dense stage the selection is
    the whole prefix).  Key gradients add up over every query that selected the key.
    q8: [L, H_I, d_I], q_scale: [L] or [L, H_I], w: [L, H_I], k8: [L, d_I], k_scale: [L],
    idx / grad: [L, m].  Returns (dw [L, H_I], dq [L, H_I, d_I], dk [L, d_I]), float64."""
    L, H_I, d_I = q8.shape
    dw = np.zeros((L, H_I))
    dq = np.zeros((L, H_I, d_I))
    dk = np.zeros((k8.shape[0], d_I))
    for t in range(L):
        valid = idx[t] >= 0
        sel = np.asarray(idx[t][valid], np.int64)
        if sel.size == 0:
            continue
        dw[t], dq[t], dks = indexer_backward_query(q8[t], q_scale[t], w[t], k8[sel], k_scale[sel],
                                                   np.asarray(grad[t], np.float64)[valid])
        np.add.at(dk, sel, dks)
    return dw, dq, dk


def sparse_mla(q: np.ndarray, latent: np.ndarray, idx: np.ndarray, sm_scale: float, rows=None,
               dv: int = 512):
    """Prefill sparse MLA of one sequence for the given rows; idx [L, k] is -1 padded.

    Returns (out [len(rows), H, dv], lse [len(rows), H]).
    """
    L = idx.shape[0]
    rows = list(range(L)) if rows is None else list(rows)
    H = q.shape[1]
    out = np.zeros((len(rows), H, dv))
    lse = np.zeros((len(rows), H))
    for r, t in enumerate(rows):
        sel = idx[t][idx[t] >= 0]
        out[r], lse[r] = sparse_mla_token(q[t], latent, sel, sm_scale, dv)
    return out, lse


# ---------------------------------------------------------------------------------------------
# Decode over a paged cache ([MZ] "等性能验证": decoding cost at 128K; paged layout is the
# library's decode input contract)
# ---------------------------------------------------------------------------------------------
def paged_gather(cache: np.ndarray, block_table_row: np.ndarray, ctx: int) -> np.ndarray:
    """Rows 0..ctx-1 of one sequence from a paged cache [num_blocks, block_size, ...]."""
    block_size = cache.shape[1]
    pos = np.arange(int(ctx))
    return cache[np.asarray(block_table_row)[pos // block_size], pos % block_size]


def decode_indexer_scores(q8, q_scale, w, kcache8, kscale_cache, block_table_row, ctx):
    """Index scores of the decode query (position ctx-1) over all ctx cached keys; float64 [ctx]."""
    k8 = paged_gather(kcache8, block_table_row, ctx)
    ks = paged_gather(kscale_cache, block_table_row, ctx)
    return indexer_scores_query(q8, q_scale, w, k8, ks)


# ---------------------------------------------------------------------------------------------
# Whole path
# ---------------------------------------------------------------------------------------------
def dsa_prefill_rows(seq: dict, k: int, sm_scale: float, rows, dv: int = 512):
    """DSA prefill of one sequence for the given query rows.

    seq holds numpy arrays: q8 [L,H_I,d_I], q_scale [L] or [L,H_I], w [L,H_I], k8 [L,d_I], k_scale [L],
    q [L,H,D], latent [L,D].  Returns dict(scores32 per row, idx [rows,k], out, lse).
    """
    rows = list(rows)
    scores = indexer_scores(seq["q8"], seq["q_scale"], seq["w"], seq["k8"], seq["k_scale"], rows)
    scores32 = scores.astype(np.float32)
    idx = np.full((len(rows), k), -1, dtype=np.int32)
    out = np.zeros((len(rows), seq["q"].shape[1], dv))
    lse = np.zeros((len(rows), seq["q"].shape[1]))
    for r, t in enumerate(rows):
        sel = topk_indices(scores32[r, : t + 1], k)
        idx[r, : sel.shape[0]] = sel
        out[r], lse[r] = sparse_mla_token(seq["q"][t], seq["latent"], sel, sm_scale, dv)
    return {"scores32": scores32, "idx": idx, "out": out, "lse": lse}


def dsa_decode(seq: dict, k: int, sm_scale: float, dv: int = 512):
    """DSA decode step of one sequence: indexer over the paged FP8 keys, top-k, sparse MLA over
    the paged latent cache.

    seq holds numpy arrays: q8 [H_I,d_I], q_scale (scalar, or [H_I] per head), w [H_I], kcache8 [nb,bs,d_I],
    kscale_cache [nb,bs], latent_cache [nb,bs,D], block_table [max_blocks], ctx, q [H,D].
    """
    ctx = int(seq["ctx"])
    scores = decode_indexer_scores(seq["q8"], seq["q_scale"], seq["w"], seq["kcache8"],
                                   seq["kscale_cache"], seq["block_table"], ctx)
    scores32 = scores.astype(np.float32)
    sel = topk_indices(scores32, k)
    latent = paged_gather(seq["latent_cache"], seq["block_table"], ctx)
    out, lse = sparse_mla_token(seq["q"], latent, sel, sm_scale, dv)
    idx = np.full(k, -1, dtype=np.int32)
    idx[: sel.shape[0]] = sel
    return {"scores32": scores32, "idx": idx, "out": out, "lse": lse}
