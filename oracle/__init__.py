"""Oracle for DeepSeek Sparse Attention (DSA): a plain, slow, float64 CPU implementation.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import it.  The product path
(the CUDA library and its Python binding) never imports, calls or links anything here, and
this package imports nothing from the product.

Every function cites the passage of the source pages it follows.  The pages are five web
pages about the DeepSeek-V3.2 technical report; citations name the page's title and section:

* [MZ] "DeepSeek-V3.2 论文解读：稀疏注意力加疯狂的 RL，把开源带到 IMO 金牌"
  (mizuki-eaf.pages.dev), section 二 "DeepSeek Sparse Attention（稀疏注意力）":
  subsections "工作原理" (indexer + top-k), "挂在 MLA 上" (MQA mode, shared latent),
  "等性能验证" (H800 cost curves, masked-MHA short-prefill mode), and the table
  "附：DSA 关键参数".
* [JD] "DeepSeek V3.2 ..." (jienda.com), section 2.1 "DeepSeek稀疏注意力（DSA）：长上下文处理的范式转移".
* [36] report digest (36881.com.cn), section "DSA：把注意力從 O(L2) 降到 O(Lk)".
* [DP] news article (digipub.cc), section 二 "基于DeepSeek-V3.1最終版打造，DSA讓模型計算更聰明".
* [TW] techwalker.com article, section 一 "突破效率瓶颈的稀疏注意力机制".

The indexer formula I[t,s] = sum_j w[t,j] * ReLU(q_I[t,j] . k_I[s]), the 576-d latent
(512 + 64) with a 512-d value, FP8 e4m3 operands with per-token fp32 scales and the
lower-index tie rule are the method's stated problem definition (the hot-path statement
this library implements); the pages themselves give the structure in words only.

Parity status per function (what pins it, in ``tests/test_oracle_*.py``):

* ``e4m3_table`` / ``decode_e4m3``: pinned (all 256 codes against an independent library
  decoder, plus hand-checked code points).
* ``indexer_scores_query`` / ``indexer_scores``: pinned (exact rational brute force on tiny
  inputs, single-head closed form against a library matmul, hand-worked golden example,
  causal-mask and ReLU invariants).
* ``topk_indices``: pinned (brute-force sort, invariants, argmax and all-equal special cases).
* ``sparse_mla_token`` / ``sparse_mla``: pinned (k >= L equals dense causal attention from a
  library routine; single-row, equal-rows and uniform-logit closed forms; permutation
  invariance).
* ``paged_gather`` / decode functions: pinned (paged layout equals the contiguous result).
* ``attention_distribution_token`` / ``indexer_kl``: pinned (a distribution summing to 1, one
  head = the softmax of its logits, equal logits = uniform, head-permutation invariance; KL >= 0,
  0 exactly when the scores are log p plus a constant, the gradient sums to 0 and matches
  central finite differences of the loss, and a two-point closed form).
* ``attention_distribution_dense_token``: pinned (equals the attention weights a library
  scaled-dot-product attention returns with identity values, averaged over heads; sums to 1;
  a zero query gives the uniform distribution; two keys of one head give the logistic closed form).
* ``indexer_backward_query`` / ``indexer_backward``: pinned (every component matches central
  finite differences of an independently written real-valued forward that itself equals
  ``indexer_scores_query`` on dequantised codes; closed form for one head and one key; zero
  where every ReLU is off; planted mistakes -- a dropped ReLU mask, a dropped head weight, a
  transposed key gradient -- fail the difference check; the sequence form adds key gradients
  over the queries that selected the key).
* ``encode_e4m3`` / ``quantize_fp8_rows``: pinned (every finite code round-trips; midpoints
  between neighbouring values go to the even code; saturation and NaN; agreement with torch's
  float8_e4m3fn cast on random values; the per-row scale rule and its error bound).
* Agreement with DeepSeek's trained model: parity unpinned (no weights, no printed values).
"""

from .dsa_oracle import (  # noqa: F401
    E4M3_MAX,
    e4m3_table,
    decode_e4m3,
    encode_e4m3,
    quantize_fp8_rows,
    indexer_scores_query,
    indexer_scores,
    indexer_magnitude_query,
    order_key_f32,
    topk_indices,
    topk_rows,
    sparse_mla_token,
    sparse_mla,
    attention_distribution_token,
    attention_distribution_dense_token,
    indexer_kl,
    indexer_backward_query,
    indexer_backward,
    paged_gather,
    decode_indexer_scores,
    dsa_prefill_rows,
    dsa_decode,
)
