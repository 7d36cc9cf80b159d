/*
 * dsa.h — C ABI of the B200 (sm_100a) DeepSeek Sparse Attention hot path.
 *
 * The method (DeepSeek-V3.2 technical report, as described on the source pages):
 *   1. a lightning indexer scores every query token t against each token s of its causal
 *      prefix, I[t,s] = sum_j w[t,j] * ReLU(q_I[t,j] . k_I[s]), with few heads, ReLU and FP8
 *      operands ("DeepSeek-V3.2 论文解读", section 二 "DeepSeek Sparse Attention", subsection
 *      "工作原理"; 36881.com.cn digest, section "DSA：把注意力從 O(L2) 降到 O(Lk)",
 *      "第一步：Lightning Indexer");
 *   2. fine-grained token selection keeps the top-k (k = 2048) index scores of each query
 *      (same subsections; "第二步：Fine-grained Token Selection");
 *   3. attention runs only over the selected entries, on MLA in MQA mode: one 576-d latent
 *      row per token (512 "nope" + 64 "rope" dims) serves as the key of every query head, and
 *      its first 512 dims are the value ("DeepSeek-V3.2 论文解读", subsection "挂在 MLA 上";
 *      jienda.com section 2.1 on MLA's latent compression of K/V).
 *
 * Conventions for every entry point:
 *   - Tensor pointers are DEVICE pointers owned by the caller; the library never allocates,
 *     frees or synchronises (dsa_device_error is the one call that synchronises).  All work
 *     is enqueued on `stream` (a cudaStream_t; NULL = the legacy default stream).
 *   - Layouts are row-major and dense unless a leading dimension is given.  bf16 tensors are
 *     passed as `const void*`.  FP8 operands are OCP e4m3 bytes with fp32 scales: one per token,
 *     or for indexer queries optionally one per (token, head) (dequantised value = e4m3(byte) * scale).
 *   - Indices are sequence-local token positions.  A prefill query at local position t has
 *     the causal prefix 0..t (min(k, t+1) entries are selected); a decode query sits at
 *     position ctx-1 and sees all ctx cached tokens.
 *   - Selected indices are written in ascending order and padded with -1.  Ties in the
 *     index score go to the lower index; -0.0 equals +0.0.
 *   - Host-side validation runs before any launch: NULL or misaligned pointers and
 *     inconsistent sizes return DSA_ERR_INVALID_ARGUMENT, shapes outside the supported set
 *     return DSA_ERR_UNSUPPORTED, a launch failure returns DSA_ERR_CUDA.  Errors found on the
 *     device are recorded in a per-process device error word and reported by
 *     dsa_device_error(): a bounded wait that expired (DSA_ERR_TIMEOUT), or an input only the
 *     GPU reads that contradicts the host arguments (DSA_ERR_DEVICE_CHECK): a NaN index score;
 *     a selection entry that is neither -1 nor a position of its sequence (the entry is
 *     masked); a block-table entry of a position inside the context that is not a block of the
 *     pool (that position is masked: no load is made through it); a context length above the
 *     descriptor's max_seqlen, or a top-k row length outside [0, ld_scores] (clamped).  Results
 *     that do not depend on the offending input are those of a clean call.
 *   - Supported shapes: indexer heads H_I in {4, 64} with d_I in {64, 128}; query heads
 *     H = 128 (prefill and decode) or 16 (prefill only); latent dim 576 with value dim 512;
 *     1 <= k <= 2048 with k a multiple of 64 for attention; paged block size 64.
 */
#ifndef DSA_B200_H_
#define DSA_B200_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARGUMENT = 1,
  DSA_ERR_UNSUPPORTED = 2,
  DSA_ERR_WORKSPACE_TOO_SMALL = 3,
  DSA_ERR_CUDA = 4,
  DSA_ERR_TIMEOUT = 5,      /* a device-side bounded wait expired */
  DSA_ERR_DEVICE_CHECK = 6  /* a device-side input check failed (NaN score, index or length out of range) */
} dsa_status;

typedef enum { DSA_KV_CONTIGUOUS = 0, DSA_KV_PAGED = 1 } dsa_kv_kind;
typedef enum { DSA_MODE_PREFILL = 0, DSA_MODE_DECODE = 1 } dsa_mode;

/*
 * Describes one per-token operand: the FP8 indexer keys (data = e4m3 bytes, scale = fp32 per
 * token) or the bf16 latent (scale = NULL).
 *   contiguous: data [total_tokens, D]; scale [total_tokens]; cu_seqlens [B+1] (device) gives
 *               each sequence's token range; in prefill the queries are the same tokens.
 *   paged:      data [num_blocks, block_size, D]; scale [num_blocks, block_size];
 *               block_table [B, max_blocks_per_seq] (device) maps a sequence's logical block
 *               p/block_size to a physical block; context_lens [B] (device) = ctx per sequence.
 * total_tokens and max_seqlen are host copies (max_seqlen: longest sequence or context).
 */
typedef struct {
  int32_t kind;
  const void* data;
  const float* scale;
  const int32_t* cu_seqlens;
  const int32_t* block_table;
  const int32_t* context_lens;
  int64_t total_tokens;
  int32_t max_seqlen;
  int32_t num_blocks;
  int32_t block_size;
  int32_t max_blocks_per_seq;
} dsa_kv_desc;

/*
 * Query scale granularity (q_scale_heads), shared by every call that runs the indexer (the
 * indexer runs in FP8: "DeepSeek-V3.2 论文解读", section 二, subsection "工作原理"):
 *   1    q_scale holds one fp32 scale per query row, shared by its H_I heads ([rows]);
 *   H_I  q_scale holds one scale per (query row, indexer head) ([rows, H_I], row-major),
 *        as a per-(token, head) FP8 quantisation of q_I produces (dsa_quantize_fp8 over
 *        rows * H_I rows of d_I columns).
 * The dequantised query of head j is e4m3(q_fp8[r, j, :]) * q_scale[r] (resp. q_scale[r, j]).
 * Scales must be finite and positive; any other q_scale_heads -> DSA_ERR_INVALID_ARGUMENT.
 *
 * Lightning indexer scores (method step 1), written to HBM for a range of query rows.
 *   prefill (keys contiguous): rows are packed query tokens [row_begin, row_end) of
 *     q_fp8 [T, H_I, d_I], q_scale [T] or [T, H_I], w [T, H_I]; row r (local position t in a sequence
 *     of length n) gets scores[(r-row_begin)*ld_scores + s] = I[t,s] for s <= t and -INFINITY
 *     for t < s < n.  ld_scores >= keys->max_seqlen and a multiple of 4.
 *   decode (keys paged): rows are sequences b in [row_begin, row_end) with q_fp8 [B, H_I, d_I],
 *     q_scale [B] or [B, H_I], w [B, H_I]; scores[(b-row_begin)*ld_scores + s] = I for s < ctx[b].
 * Scores are fp32, accumulated in fp32 on the tensor cores (e4m3 x e4m3).
 */
dsa_status dsa_indexer_scores(const uint8_t* q_fp8, const float* q_scale, int32_t q_scale_heads, const float* w,
                              const dsa_kv_desc* keys, int32_t B, int32_t H_I, int32_t d_I,
                              int64_t row_begin, int64_t row_end, float* scores, int64_t ld_scores,
                              void* stream);

/*
 * Fused lightning indexer + top-k for prefill (method steps 1 and 2 together): for every
 * packed query token of q_fp8 [T, H_I, d_I] (keys contiguous, queries == keys per sequence),
 * idx_out[t*k ...] receives the min(k, t+1) highest-scoring causal-prefix positions,
 * ascending, -1 padded.  Scores stay on chip: each CTA keeps a per-token candidate set in
 * shared memory with a rising threshold.  The selection equals dsa_topk applied to the
 * scores dsa_indexer_scores writes (same fp32 arithmetic).  keys->max_seqlen <= 196608 (d_I = 128) or 98304 (d_I = 64).
 */
dsa_status dsa_indexer_topk(const uint8_t* q_fp8, const float* q_scale, int32_t q_scale_heads, const float* w,
                            const dsa_kv_desc* keys, int32_t B, int32_t H_I, int32_t d_I, int32_t k, int32_t* idx_out,
                            void* stream);

/*
 * Fused decode selection (method steps 1 and 2 for one decode query per sequence): the paged
 * lightning indexer over each sequence's context (as dsa_indexer_scores, decode form, rows
 * 0..B-1), then the per-sequence top-k.  idx_out [B, k] receives, for sequence b, the indices
 * of the min(k, ctx_b) highest-scoring context positions, ties to the lower position,
 * ascending, -1 padded, with ctx_b = min(context_lens[b], keys->max_seqlen) -- the result
 * dsa_topk gives on the scores dsa_indexer_scores writes.  While it scans, the indexer
 * records the largest score of every 16 consecutive keys; the k-th largest of those maxima
 * bounds the k-th largest score from below, so the selection reads each score row once and
 * keeps only the scores at or above that bound (falling back to a full radix select of the
 * row when they do not fit on chip).  keys must be paged (else DSA_ERR_UNSUPPORTED).
 * workspace (device, 256-byte aligned, caller-owned, contents unspecified on return) holds
 * the score rows and group maxima: ws_bytes >= dsa_decode_select_workspace_size(B,
 * keys->max_seqlen), else DSA_ERR_WORKSPACE_TOO_SMALL.  A context longer than
 * keys->max_seqlen and NaN scores set DSA_ERR_DEVICE_CHECK in the device error word.
 */
dsa_status dsa_indexer_topk_decode(const uint8_t* q_fp8, const float* q_scale, int32_t q_scale_heads, const float* w,
                                   const dsa_kv_desc* keys, int32_t B, int32_t H_I, int32_t d_I, int32_t k,
                                   int32_t* idx_out, void* workspace, size_t ws_bytes, void* stream);

/* Workspace bytes of dsa_indexer_topk_decode for B sequences of at most max_ctx keys (0 when
 * B or max_ctx is not positive). */
size_t dsa_decode_select_workspace_size(int32_t B, int32_t max_ctx);

/*
 * Top-k selection (method step 2: the index scores pick the k = 2048 highest-scoring tokens
 * of each query -- "DeepSeek-V3.2 论文解读", section 二, subsection "工作原理" and table
 * "附：DSA 关键参数"; 36881.com.cn digest, "第二步：Fine-grained Token Selection") over score
 * rows: for row r the first row_len[r] entries
 * of scores[r*ld_scores ...] are candidates; idx[r*k ...] receives the indices of the
 * min(k, row_len[r]) largest (ties -> lower index), ascending, -1 padded.  row_len is a device
 * array.  scores must be 16-byte aligned and ld_scores a multiple of 4.  NaN scores set
 * DSA_ERR_DEVICE_CHECK in the device error word.
 */
dsa_status dsa_topk(const float* scores, int64_t ld_scores, int64_t rows, const int32_t* row_len,
                    int32_t k, int32_t* idx, void* stream);

/*
 * Row blocks of one sequence, for sharding a long prefill over GPUs by query rows (each GPU
 * holds every key and latent row -- gathered from the others -- and its own block of query
 * rows).  keys / latent describe ONE contiguous sequence (cu_seqlens = {0, L}).
 *   dsa_indexer_topk_rows: like dsa_indexer_topk for query rows [row_begin, row_end) only;
 *     q_fp8 [R, H_I, d_I], q_scale [R] or [R, H_I], w [R, H_I] and idx_out [R, k] hold just those
 *     R = row_end - row_begin rows (row 0 = query row_begin).
 *   dsa_sparse_mla_prefill_rows: like dsa_sparse_mla_prefill for rows [row_begin, row_end);
 *     q [R, H, 576], idx [R, k], out [R, H, 512], lse [R, H] hold just those rows.
 * Each block's results equal the corresponding rows of the whole-sequence call.  row_begin ==
 * row_end is a no-op; 0 <= row_begin <= row_end <= L, else DSA_ERR_INVALID_ARGUMENT.
 */
/*
 * Row blocks of balanced cost for sharding one prefill of length L over `parts` GPUs (host
 * only, no device work): bounds[0] = 0 < bounds[1] < ... < bounds[parts] = L, every block
 * non-empty.  Query row t costs indexer_cost * (t+1) / sum_t (t+1) -- the indexer scans its
 * causal prefix -- plus mla_cost * min(t+1, k) / sum_t min(t+1, k) -- sparse MLA over its
 * selection; pass the two kernels' measured times of one whole-sequence step (any unit, both
 * >= 0, not both 0).  Block r ends at the first row where the cumulative cost reaches r/parts
 * of the total.  The pages describe no parallelism; this is a scale-out helper for the row-block
 * entry points below.  DSA_ERR_INVALID_ARGUMENT for bounds == NULL, L < 1, k < 1,
 * parts outside [1, L] or costs as above.
 */
dsa_status dsa_row_partition(int64_t L, int32_t k, int32_t parts, double indexer_cost, double mla_cost,
                             int64_t* bounds);

dsa_status dsa_indexer_topk_rows(const uint8_t* q_fp8, const float* q_scale, int32_t q_scale_heads, const float* w,
                                 const dsa_kv_desc* keys, int32_t H_I, int32_t d_I, int32_t k,
                                 int64_t row_begin, int64_t row_end, int32_t* idx_out, void* stream);
dsa_status dsa_sparse_mla_prefill_rows(const void* q, const dsa_kv_desc* latent, const int32_t* idx, int32_t H,
                                       int32_t k, float sm_scale, int64_t row_begin, int64_t row_end, void* out,
                                       float* lse, void* stream);

/*
 * Masked dense mode of sparse MLA prefill, for short sequences ("DeepSeek-V3.2 论文解读",
 * section 二, subsection "等性能验证": for short prefill a masked MHA mode simulates DSA): the same out/lse as
 * dsa_sparse_mla_prefill for the same arguments, computed by walking every causal 64-key chunk
 * of the contiguous latent (rows read in order, none through idx) and masking the keys idx does
 * not select.  Cost grows with L^2 instead of L*k, so it pays only when most causal keys are
 * selected (L up to ~2k).  idx rows must be strictly ascending with the -1 padding at the end
 * (as the top-k entry points write them); entries outside [0, t] are ignored (not reported).
 * Same layouts, alignment and errors as dsa_sparse_mla_prefill.
 */
dsa_status dsa_masked_mla_prefill(const void* q, const dsa_kv_desc* latent, const int32_t* idx, int32_t B,
                                  int32_t H, int32_t k, float sm_scale, void* out, float* lse, void* stream);

/*
 * Sparse MLA prefill (method step 3: attention runs only over the selected entries, on MLA in
 * MQA mode, where one latent row per token is the key of every query head and its first 512
 * dims are the value -- "DeepSeek-V3.2 论文解读", section 二, subsection "挂在 MLA 上"; jienda.com
 * section 2.1 on MLA's latent K/V): for every packed query token t and head h,
 *   out[t,h,:] = sum_i softmax_i(sm_scale * q[t,h,:] . c[idx[t,i],:]) * c[idx[t,i], 0:512]
 * over the valid (>= 0) entries of idx [T, k]; c is the contiguous latent of t's sequence.
 * q [T, H, 576] bf16, out [T, H, 512] bf16, lse [T, H] fp32 natural log (may be NULL).
 * A row without a valid index gets out = 0 and lse = -INFINITY.
 */
dsa_status dsa_sparse_mla_prefill(const void* q, const dsa_kv_desc* latent, const int32_t* idx,
                                  int32_t B, int32_t H, int32_t k, float sm_scale, void* out,
                                  float* lse, void* stream);

/*
 * Sparse MLA decode (method step 3 for the decode step the pages' long-context cost curves
 * measure -- "DeepSeek-V3.2 论文解读", section 二, subsection "等性能验证"; techwalker.com,
 * section 五 "成本效益与部署优势"): one query per sequence, q [B, H, 576]; idx [B, k] holds logical positions
 * (< ctx[b]) resolved through the paged latent cache (latent->kind == DSA_KV_PAGED).  The work
 * is split over the k selected rows (into more parts for fewer sequences, so that all the
 * parts run in one round on the GPU); partial results go to `workspace`
 * (dsa_workspace_size(DSA_MODE_DECODE, ...) bytes) and are merged by log-sum-exp.  When the
 * sequences alone fill the GPU (one part each) the kernel writes out and lse directly.
 */
dsa_status dsa_sparse_mla_decode(const void* q, const dsa_kv_desc* latent, const int32_t* idx,
                                 int32_t B, int32_t H, int32_t k, float sm_scale, void* out,
                                 float* lse, void* workspace, size_t ws_bytes, void* stream);

/*
 * Same as dsa_sparse_mla_decode, but it allocates nothing and takes no workspace: the split
 * partial results live in a scratch array that the library itself holds in device memory
 * (DSA_NOALLOC_SCRATCH_BYTES per GPU that loads the library, kept until the process exits).
 * This entry point has no counterpart in the method's description; it exists for callers that
 * cannot allocate device memory on the call path, for example a serving engine that hands
 * all device memory to its own pool at start-up, or a latency-critical loop that cannot
 * afford cudaMalloc's implicit device-wide synchronisation.
 *   - The first call on a device looks up the array's device address (with that device
 *     current); make that first call before any stream capture.  The address is cached for the
 *     life of the device's primary context: after cudaDeviceReset (or anything else that tears
 *     that context down) this entry point must not be called again in the process.
 *   - Every call on a device shares the one array, which keeps the last call's contents: calls
 *     whose kernels overlap on the GPU (different streams, no ordering) race with each other.
 *   - Sizes whose partial results do not fit (B * H * splits * 2056 bytes; splits is the largest
 *     power of two s with B * s <= 74 and s <= k/64, at least 1, so B * splits <= 74 for B <= 74)
 *     return DSA_ERR_UNSUPPORTED before any launch: at H = 128 every B <= 127 fits and B = 128
 *     does not.
 */
#define DSA_NOALLOC_SCRATCH_BYTES (32u << 20)
dsa_status dsa_sparse_mla_decode_noalloc(const void* q, const dsa_kv_desc* latent, const int32_t* idx, int32_t B,
                                         int32_t H, int32_t k, float sm_scale, void* out, float* lse,
                                         void* stream);

/*
 * Whole DSA forward (method steps 1-3: lightning indexer, fine-grained top-k selection, sparse
 * MLA in MQA mode -- "DeepSeek-V3.2 论文解读", section 二, subsections "工作原理" and "挂在 MLA
 * 上"; prefill and decode as in its subsection "等性能验证").
 *   DSA_MODE_PREFILL: indexer and top-k run fused (no score matrix is written to HBM), then
 *     sparse MLA.  keys/latent contiguous with the same cu_seqlens; q_fp8 [T, H_I, d_I], etc.
 *   DSA_MODE_DECODE: the fused decode selection (dsa_indexer_topk_decode), then split
 *     sparse MLA with a log-sum-exp merge.
 * idx_out [rows, k] receives the selection when not NULL (otherwise it lives in workspace).
 */
dsa_status dsa_forward(int32_t mode, const uint8_t* q_fp8, const float* q_scale, int32_t q_scale_heads,
                       const float* w, const dsa_kv_desc* keys, const void* q, const dsa_kv_desc* latent, int32_t B,
                       int32_t H_I, int32_t d_I, int32_t H, int32_t k, float sm_scale, void* out,
                       float* lse, int32_t* idx_out, void* workspace, size_t ws_bytes, void* stream);

/* Bytes of workspace dsa_forward / dsa_sparse_mla_decode need (0 when none): prefill, the
 * selection [total_tokens, k] int32; decode, the split partials of B sequences with H heads,
 * the decode selection's workspace (dsa_decode_select_workspace_size) and the selection [B, k]. */
size_t dsa_workspace_size(int32_t mode, int32_t B, int64_t total_tokens, int32_t max_ctx, int32_t H, int32_t k);

/* Static description of a status code. */
const char* dsa_status_string(int32_t status);

/*
 * Synchronises `stream`, then reads and clears the device error word of the current device.
 * *code receives DSA_OK or the first DSA_ERR_TIMEOUT / DSA_ERR_DEVICE_CHECK recorded since the
 * last call.  Returns DSA_ERR_CUDA if synchronisation failed.
 */
dsa_status dsa_device_error(int32_t* code, void* stream);

/*
 * Indexer KL alignment (the training-side step next to the indexer; "DeepSeek-V3.2 论文解读",
 * section 二: a KL loss aligns the indexer's distribution with the main attention's; in the
 * sparse stage over each token's selected rows).
 *   dsa_attn_distribution: p_out[t*k + i] = (1/H) sum_h exp(sm_scale * q[t,h,:] . c[idx[t,i],:]
 *     - lse[t,h]) for valid entries (idx >= 0 and inside the sequence), 0 otherwise: the
 *     head-averaged attention distribution over the selected rows.  q [T, H, 576] bf16, latent
 *     contiguous [T, 576] bf16 with cu_seqlens, idx [T, k] (k a multiple of 64, <= 2048), lse
 *     [T, H] fp32 natural log as dsa_sparse_mla_prefill writes it; p_out [T, k] fp32.
 *   dsa_indexer_kl: per row r over the valid entries (idx >= 0): q = softmax(scores[r,:]),
 *     loss[r] = sum_i p_i (log p_i - log q_i) (p_i = 0 adds nothing), grad[r*k + i] = q_i - p_i
 *     (0 for invalid entries); a row without valid entries gets loss 0.  fp32 [rows, k] inputs.
 * Device pointers, caller-owned outputs, asynchronous on `stream`; DSA_ERR_INVALID_ARGUMENT for
 * NULL / misaligned pointers, DSA_ERR_UNSUPPORTED outside the stated shapes.
 */
dsa_status dsa_attn_distribution(const void* q, const dsa_kv_desc* latent, const int32_t* idx, const float* lse,
                                 int32_t B, int32_t H, int32_t k, float sm_scale, float* p_out, void* stream);
dsa_status dsa_indexer_kl(const float* p, const float* scores, const int32_t* idx, int64_t rows, int32_t k,
                          float* loss, float* grad, void* stream);

/*
 * Dense warm-up target and the indexer backward (the two training stages of the indexer:
 * "DeepSeek-V3.2 论文解读", section 二, subsection "两阶段继续预训练" -- a dense warm-up in
 * which attention stays dense and only the indexer learns, by a KL loss towards the main
 * attention's distribution, then sparse training in which the indexer, its input detached,
 * still learns from the KL loss alone).
 *   dsa_attn_distribution_dense: for packed query tokens r in [row_begin, row_end) (position t
 *     in a sequence of the contiguous latent, cu_seqlens), p_out[(r-row_begin)*ld_p + s] =
 *     (1/H) sum_h exp(sm_scale * q[r,h,:] . c[s,:] - lse[r,h]) for s <= t and 0 for
 *     t < s < ld_p: the head-averaged attention distribution over the whole causal prefix.
 *     q [T, H, 576] bf16, lse [T, H] fp32 natural log of a dense causal attention over the
 *     prefix (dsa_masked_mla_prefill writes it), ld_p >= latent->max_seqlen; 1 <= H <= 128.
 *     With p_out, the KL loss and its gradient of the dense stage are dsa_indexer_kl over rows
 *     of ld_p entries whose idx lists the prefix positions (-1 beyond).
 *   dsa_indexer_backward: given grad[t*k + i] = d loss / d I[t, idx[t*k + i]] (idx -1 padded,
 *     as dsa_indexer_kl writes it), writes the gradients of the indexer's inputs, taken with
 *     respect to the dequantised operands q_I = e4m3(q_fp8) * q_scale and k_I = e4m3(k8) *
 *     k_scale, through the ReLU (derivative 0 at 0), in fp32:
 *       dw [T, H_I]:      dw[t,j] = sum_i g_i ReLU(a_j(s_i)),   a_j(s) = q_I[t,j,:] . k_I[s,:]
 *       dq [T, H_I, d_I]: dq[t,j,:] = sum_i g_i w[t,j] [a_j(s_i) > 0] k_I[s_i,:]
 *       dk [T, d_I]:      dk[s,:] = sum over (t, i) with idx = s of g_i sum_j w[t,j] [a_j(s) > 0] q_I[t,j,:]
 *     keys contiguous (cu_seqlens, total_tokens T; queries are the packed tokens); dk is zeroed
 *     by the call and accumulated with atomic adds (summation order, and so the last bits,
 *     vary between runs).  Entries outside their sequence (other than -1) are skipped and set
 *     DSA_ERR_DEVICE_CHECK.  H_I in {4, 64}, d_I in {64, 128}.
 * Device pointers, caller-owned outputs, asynchronous on `stream`; DSA_ERR_INVALID_ARGUMENT for
 * NULL / misaligned pointers (dq and dk 16-byte aligned) or ranges outside the arrays,
 * DSA_ERR_UNSUPPORTED outside the stated shapes.
 */
dsa_status dsa_attn_distribution_dense(const void* q, const dsa_kv_desc* latent, const float* lse, int32_t B,
                                       int32_t H, int64_t row_begin, int64_t row_end, float sm_scale, float* p_out,
                                       int64_t ld_p, void* stream);
dsa_status dsa_indexer_backward(const uint8_t* q_fp8, const float* q_scale, int32_t q_scale_heads, const float* w,
                                const dsa_kv_desc* keys, int32_t B, int32_t H_I, int32_t d_I, const int32_t* idx,
                                const float* grad, int32_t k, float* dw, float* dq, float* dk, void* stream);

/*
 * Self-test of failure detection (no counterpart on the pages): launches a kernel that waits on
 * a barrier nothing completes, with the same bounded-wait scheme as every pipeline wait of this
 * library but a limit of limit_us microseconds (1 .. 2000000); the kernel then records
 * DSA_ERR_TIMEOUT in the device error word and returns normally, so a following
 * dsa_device_error reports 5 and the context stays usable.  Asynchronous on `stream`.
 */
dsa_status dsa_selftest_wait_timeout(int32_t limit_us, void* stream);

/*
 * Per-row FP8 quantiser for the indexer operands (the step that produces the indexer's input
 * contract; "DeepSeek-V3.2 论文解读", section 二, subsection "工作原理": the indexer runs in
 * FP8).  For each row r of x [rows, cols] bf16 (row-major, contiguous), where a row is a key of
 * k_I, or the queries of one token (all H_I heads: one q scale per token, q_scale_heads = 1),
 * or one (token, head) query of q_I passed as [T * H_I, d_I] (one q scale per head,
 * q_scale_heads = H_I):
 *   scale[r] = amax_c |x[r,c]| / 448 in IEEE fp32 (1 for an all-zero row),
 *   codes[r*cols + c] = e4m3(x[r,c] / scale[r]), the quotient in IEEE fp32 rounded to the
 *   nearest e4m3 value (ties to even), saturating at +-448.  NaN elements take no part in
 *   the maximum and encode as NaN.
 * Device pointers; x 16-byte aligned, codes 8-byte aligned, cols a positive multiple of 8.
 * rows == 0 is a no-op.  Outputs are caller-owned; nothing is allocated.
 * Errors: DSA_ERR_INVALID_ARGUMENT for null/misaligned pointers or a bad cols; the call is
 * asynchronous on `stream` (launch errors are returned, execution errors surface later).
 */
dsa_status dsa_quantize_fp8(const void* x_bf16, int64_t rows, int32_t cols, uint8_t* codes, float* scale,
                            void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DSA_B200_H_ */
