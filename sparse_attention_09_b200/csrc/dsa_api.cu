// Host side of the C ABI declared in include/dsa.h: argument validation, TMA descriptor
// encoding and kernel launches.  Every entry point enqueues on the caller's stream and
// returns without synchronising.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/dsa.h"
#include "common.cuh"
#include "indexer.cuh"
#include "quantize.cuh"
#include "attn_probs.cuh"
#include "indexer_bwd.cuh"
#include "indexer_kl.cuh"
#include "selftest.cuh"
#include "mla_common.cuh"
#include "sparse_mla_pair.cuh"
#include "topk.cuh"

namespace dsa {
namespace {

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

inline dsa_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

// ---- TMA descriptors (encoded on the host through the driver entry point) -------------------
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static std::once_flag once;
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// 2-D map over a row-major [rows, cols] tensor; box = [box_rows, box_cols].
bool make_map_2d(CUtensorMap* m, const void* base, CUtensorMapDataType dt, uint64_t cols, uint64_t rows,
                 uint64_t row_bytes, uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t es[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---- lightning indexer -------------------------------------------------------------------
constexpr int kIdxStages = 4;      // key-tile ring depth, scores mode
// Fused top-k mode: the candidate sets need the shared memory.  Up to 128K keys (d_I = 128) the
// key ring has 2 stages and a token holds up to 4608 candidates; longer sequences need the
// third stage for the emission bitmap (which reuses the ring) and hold 4096.  Measured at
// L = 131072: 130.9 ms against 135.4 ms with 3 stages and 4096 (fewer streaming cuts).
constexpr int kIdxStagesTopkShort = 2, kIdxCapShort = 4608, kIdxCapExtraShort = 2560;
constexpr int kIdxStagesTopkLong = 3, kIdxCapLong = 4096, kIdxCapExtraLong = 1024;
constexpr int kIdxTok = 4;            // prefill query tokens per CTA
constexpr int kDecodeTilesPerCta = 32;  // decode: 4096 keys per CTA (measured: 16 -> 32 tiles, -3 % at 64 x ~71K keys, -12 % at 8 x ~127K)

template <int D_I, int H_I, int TOK, int MODE, bool PAGED, int STAGES>
dsa_status launch_indexer_s(const CUtensorMap& qm, const CUtensorMap& km, const IndexerParams& p, dim3 grid,
                            cudaStream_t s) {
  auto kern = indexer_kernel<D_I, H_I, TOK, MODE, PAGED, STAGES>;
  const int smem = indexer_smem_bytes<D_I, H_I, TOK, MODE, STAGES>(p.cap) + 1024;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return DSA_ERR_CUDA;
  kern<<<grid, IdxGroups<TOK>::kThreads, smem, s>>>(qm, km, p);
  return launch_status();
}

// Scores mode: kIdxStages; fused top-k mode: the ring depth `stages` (2 or 3, see above).
template <int D_I, int H_I, int TOK, int MODE, bool PAGED>
dsa_status launch_indexer_t(const CUtensorMap& qm, const CUtensorMap& km, const IndexerParams& p, dim3 grid,
                            cudaStream_t s, int stages) {
  if constexpr (MODE == kIdxTopk) {
    if (stages == kIdxStagesTopkShort)
      return launch_indexer_s<D_I, H_I, TOK, MODE, PAGED, kIdxStagesTopkShort>(qm, km, p, grid, s);
    return launch_indexer_s<D_I, H_I, TOK, MODE, PAGED, kIdxStagesTopkLong>(qm, km, p, grid, s);
  } else {
    return launch_indexer_s<D_I, H_I, TOK, MODE, PAGED, kIdxStages>(qm, km, p, grid, s);
  }
}

// Ring depth and candidate capacity of the fused top-k for sequences of up to max_seqlen keys
// (the final ascending emission uses a bitmap of the causal prefix inside the key ring, half of
// it per epilogue group); DSA_ERR_UNSUPPORTED when the bitmap does not fit three stages.
dsa_status topk_config(int d_I, int max_seqlen, int k, int* stages, int* cap) {
  const int64_t bitmap_bytes = (static_cast<int64_t>(max_seqlen) + 31) / 32 * 4;
  const int64_t stage_bytes = 128 * static_cast<int64_t>(d_I);
  if (max_seqlen > (1 << 24)) return DSA_ERR_UNSUPPORTED;
  int extra, cmax;
  if (bitmap_bytes <= kIdxStagesTopkShort * stage_bytes / 2) {
    *stages = kIdxStagesTopkShort;
    extra = kIdxCapExtraShort;
    cmax = kIdxCapShort;
  } else if (bitmap_bytes <= kIdxStagesTopkLong * stage_bytes / 2) {
    *stages = kIdxStagesTopkLong;
    extra = kIdxCapExtraLong;
    cmax = kIdxCapLong;
  } else {
    return DSA_ERR_UNSUPPORTED;
  }
  *cap = k + extra < 2 * k ? 2 * k : k + extra;
  if (*cap > cmax) *cap = cmax;
  return DSA_OK;
}

template <int MODE, bool PAGED>
dsa_status launch_indexer(int d_I, int H_I, const CUtensorMap& qm, const CUtensorMap& km, const IndexerParams& p,
                          dim3 grid, cudaStream_t s, int stages = 0) {
  constexpr int TOK = PAGED ? 1 : kIdxTok;
  if constexpr (PAGED) {
    if (H_I != 64) return DSA_ERR_UNSUPPORTED;
    if (d_I == 128) return launch_indexer_t<128, 64, TOK, MODE, PAGED>(qm, km, p, grid, s, stages);
    if (d_I == 64) return launch_indexer_t<64, 64, TOK, MODE, PAGED>(qm, km, p, grid, s, stages);
    return DSA_ERR_UNSUPPORTED;
  } else {
    if (d_I == 128 && H_I == 64) return launch_indexer_t<128, 64, TOK, MODE, PAGED>(qm, km, p, grid, s, stages);
  if (d_I == 64 && H_I == 64) return launch_indexer_t<64, 64, TOK, MODE, PAGED>(qm, km, p, grid, s, stages);
  if (d_I == 128 && H_I == 4) return launch_indexer_t<128, 4, TOK, MODE, PAGED>(qm, km, p, grid, s, stages);
  if (d_I == 64 && H_I == 4) return launch_indexer_t<64, 4, TOK, MODE, PAGED>(qm, km, p, grid, s, stages);
  return DSA_ERR_UNSUPPORTED;
  }
}

bool indexer_shape_ok(int H_I, int d_I) { return (H_I == 4 || H_I == 64) && (d_I == 64 || d_I == 128); }

// Validates the common indexer arguments and builds the Q / K tensor maps.
// q_rows: rows held by the query arrays (prefill: the packed tokens they cover; 0 = all of them)
dsa_status indexer_common(const uint8_t* q_fp8, const float* q_scale, int32_t q_scale_heads, const float* w,
                          const dsa_kv_desc* keys, int32_t B, int32_t H_I, int32_t d_I, CUtensorMap* qm,
                          CUtensorMap* km, IndexerParams* p, int64_t q_rows = 0) {
  if (q_fp8 == nullptr || q_scale == nullptr || w == nullptr || keys == nullptr || keys->data == nullptr ||
      keys->scale == nullptr || B <= 0)
    return DSA_ERR_INVALID_ARGUMENT;
  if (q_scale_heads != 1 && q_scale_heads != H_I) return DSA_ERR_INVALID_ARGUMENT;
  if (!aligned(q_fp8, 16) || !aligned(keys->data, 16)) return DSA_ERR_INVALID_ARGUMENT;
  if (!indexer_shape_ok(H_I, d_I)) return DSA_ERR_UNSUPPORTED;
  const CUtensorMapSwizzle sw = d_I == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B;
  std::memset(p, 0, sizeof(*p));
  p->tok_begin = 0;
  p->tok_end = 0x7FFFFFFF;
  p->q_row0 = 0;
  p->q_scale = q_scale;
  p->q_scale_heads = q_scale_heads;
  p->w = w;
  p->k_scale = keys->scale;
  if (keys->kind == DSA_KV_CONTIGUOUS) {
    if (keys->cu_seqlens == nullptr || keys->total_tokens <= 0 || keys->max_seqlen <= 0) return DSA_ERR_INVALID_ARGUMENT;
    if (keys->total_tokens * H_I > 0x7FFFFFFFLL) return DSA_ERR_UNSUPPORTED;
    const uint64_t T = static_cast<uint64_t>(keys->total_tokens);
    const uint64_t TQ = q_rows > 0 ? static_cast<uint64_t>(q_rows) : T;
    if (!make_map_2d(qm, q_fp8, CU_TENSOR_MAP_DATA_TYPE_UINT8, d_I, TQ * H_I, d_I, d_I, kIdxTok * H_I, sw) ||
        !make_map_2d(km, keys->data, CU_TENSOR_MAP_DATA_TYPE_UINT8, d_I, T, d_I, d_I, 128, sw))
      return DSA_ERR_INVALID_ARGUMENT;
    p->cu_seqlens = keys->cu_seqlens;
  } else if (keys->kind == DSA_KV_PAGED) {
    if (keys->block_table == nullptr || keys->context_lens == nullptr || keys->num_blocks <= 0 ||
        keys->max_blocks_per_seq <= 0 || keys->max_seqlen <= 0)
      return DSA_ERR_INVALID_ARGUMENT;
    if (keys->block_size != 64 || H_I != 64) return DSA_ERR_UNSUPPORTED;
    if (static_cast<int64_t>(keys->max_seqlen) > static_cast<int64_t>(keys->max_blocks_per_seq) * 64)
      return DSA_ERR_INVALID_ARGUMENT;
    if (static_cast<int64_t>(keys->num_blocks) * 64 > 0x7FFFFFFFLL) return DSA_ERR_UNSUPPORTED;
    const uint64_t rows = static_cast<uint64_t>(keys->num_blocks) * 64;
    if (!make_map_2d(qm, q_fp8, CU_TENSOR_MAP_DATA_TYPE_UINT8, d_I, static_cast<uint64_t>(B) * H_I, d_I, d_I, H_I,
                     sw) ||
        !make_map_2d(km, keys->data, CU_TENSOR_MAP_DATA_TYPE_UINT8, d_I, rows, d_I, d_I, 64, sw))
      return DSA_ERR_INVALID_ARGUMENT;
    p->block_table = keys->block_table;
    p->context_lens = keys->context_lens;
    p->max_blocks_per_seq = keys->max_blocks_per_seq;
    p->num_blocks = keys->num_blocks;
    p->max_len = keys->max_seqlen;  // validated above: 0 < max_seqlen <= 64 * max_blocks_per_seq
    p->tiles_per_cta = kDecodeTilesPerCta;
  } else {
    return DSA_ERR_INVALID_ARGUMENT;
  }
  return DSA_OK;
}

// ---- sparse MLA ------------------------------------------------------------------------------
constexpr int kMlaClusters = 74;   // one CTA pair per two SMs of a 148-SM B200
constexpr int kLatentDim = 576, kValueDim = 512;

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

size_t decode_partials_bytes(int B, int H, int splits) {
  return align256(static_cast<size_t>(B) * splits * H * kValueDim * 4) + align256(static_cast<size_t>(B) * splits * H * 2 * 4);
}

// Decode divides each sequence's selection into `splits` work units of whole 64-row chunks,
// merged afterwards by a log-sum-exp combine.  Splitting pays only while the units still fit
// one round on the CTA pairs: each unit costs a Q load, an O readout and fp32 partials, and
// every chunk of a unit is one step of the same latency chain.  So splits is the largest power
// of two s with B * s <= the number of CTA pairs (one round) and s <= k / 64 (a chunk per
// unit), at least 1.  With one split the kernel writes out and lse itself (no partials, no
// combine).  Measured on a B200 for 64 sequences, k = 2048 (MLA + combine, the latent-split
// kernel that preceded the head-split pair): 1 split 100 us, 2 splits 117 us, 4 splits 151 us,
// 8 splits 221 us.
int decode_splits(int B, int k) {
  int s = 1;
  while (2 * s <= k / 64 && static_cast<int64_t>(B) * 2 * s <= kMlaClusters) s *= 2;
  return s;
}

// Sparse prefill, masked prefill and decode: the head-split pair kernel.  Q is read by TMA as a
// [q_rows * H, 576] bf16 matrix in 64 x 64 tiles (128-byte swizzle).
template <bool DECODE, bool MASKED = false>
dsa_status launch_mla_pair(const void* latent, const void* q, int64_t q_rows, const MlaParams& p, int64_t units,
                           cudaStream_t s) {
  CUtensorMap qm;
  if (!make_map_2d(&qm, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, kLatentDim, static_cast<uint64_t>(q_rows) * p.H,
                   kLatentDim * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B))
    return DSA_ERR_INVALID_ARGUMENT;
  auto kern = sparse_mla_pair_kernel<DECODE, MASKED>;
  const int smem = mlap::kSmemBytes + 1024;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return DSA_ERR_CUDA;
  const int clusters = static_cast<int>(units < kMlaClusters ? units : kMlaClusters);
  kern<<<2 * clusters, mlap::kThreads, smem, s>>>(static_cast<const __nv_bfloat16*>(latent), p, qm);
  return launch_status();
}

bool mla_shape_ok(int H, int k) { return H >= 1 && H <= 128 && k >= 64 && k <= 2048 && k % 64 == 0; }

// ---- decode with library-held scratch (no allocation on the call path) ---------------------
// One array per device, in this translation unit.  Host code cannot pass the symbol itself to
// a kernel (on the host it is only a stand-in), so each device's address is looked up once,
// with that device current, and cached.
static __device__ __align__(256) uint8_t g_noalloc_scratch[DSA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 256;

dsa_status noalloc_scratch(void** ptr) {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return DSA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return DSA_ERR_CUDA;
    addr[dev] = p;
  }
  *ptr = addr[dev];
  return DSA_OK;
}

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" {

const char* dsa_status_string(int32_t status) {
  switch (status) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARGUMENT: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported shape or configuration";
    case DSA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case DSA_ERR_CUDA: return "CUDA error";
    case DSA_ERR_TIMEOUT: return "device-side wait timed out";
    case DSA_ERR_DEVICE_CHECK: return "device-side input check failed";
    default: return "unknown status";
  }
}

dsa_status dsa_device_error(int32_t* code, void* stream) {
  if (code == nullptr) return DSA_ERR_INVALID_ARGUMENT;
  cudaStream_t s = as_stream(stream);
  int32_t v = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_device_error, sizeof(v), 0, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return DSA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return DSA_ERR_CUDA;
  const int32_t zero = 0;
  if (cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return DSA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return DSA_ERR_CUDA;
  *code = v;
  return DSA_OK;
}

dsa_status dsa_attn_distribution(const void* q, const dsa_kv_desc* latent, const int32_t* idx, const float* lse,
                                 int32_t B, int32_t H, int32_t k, float sm_scale, float* p_out, void* stream) {
  if (q == nullptr || latent == nullptr || latent->data == nullptr || idx == nullptr || lse == nullptr ||
      p_out == nullptr || B <= 0)
    return DSA_ERR_INVALID_ARGUMENT;
  if (latent->kind != DSA_KV_CONTIGUOUS || latent->cu_seqlens == nullptr || latent->total_tokens <= 0)
    return DSA_ERR_INVALID_ARGUMENT;
  if (!aligned(q, 16) || !aligned(latent->data, 16)) return DSA_ERR_INVALID_ARGUMENT;
  if (H < 1 || H > 128 || k < 64 || k > 2048 || k % 64 != 0) return DSA_ERR_UNSUPPORTED;
  ProbsParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.idx = idx;
  p.lse = lse;
  p.cu_seqlens = latent->cu_seqlens;
  p.B = B;
  p.H = H;
  p.k = k;
  p.rows = latent->total_tokens;
  p.scale_log2 = sm_scale * 1.4426950408889634f;
  p.p = p_out;
  const int smem = probs::kSmemBytes + 1024;
  if (cudaFuncSetAttribute(attn_probs_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return DSA_ERR_CUDA;
  const int64_t grid = p.rows < 148 ? p.rows : 148;
  attn_probs_kernel<false><<<static_cast<unsigned>(grid), probs::kThreads, smem, as_stream(stream)>>>(
      static_cast<const __nv_bfloat16*>(latent->data), p);
  return launch_status();
}

dsa_status dsa_attn_distribution_dense(const void* q, const dsa_kv_desc* latent, const float* lse, int32_t B,
                                       int32_t H, int64_t row_begin, int64_t row_end, float sm_scale, float* p_out,
                                       int64_t ld_p, void* stream) {
  if (latent == nullptr || row_begin < 0 || row_end < row_begin) return DSA_ERR_INVALID_ARGUMENT;
  if (row_end == row_begin) return DSA_OK;
  if (q == nullptr || latent->data == nullptr || lse == nullptr || p_out == nullptr || B <= 0)
    return DSA_ERR_INVALID_ARGUMENT;
  if (latent->kind != DSA_KV_CONTIGUOUS || latent->cu_seqlens == nullptr || latent->total_tokens <= 0)
    return DSA_ERR_INVALID_ARGUMENT;
  if (row_end > latent->total_tokens || ld_p < latent->max_seqlen) return DSA_ERR_INVALID_ARGUMENT;
  if (!aligned(q, 16) || !aligned(latent->data, 16)) return DSA_ERR_INVALID_ARGUMENT;
  if (H < 1 || H > 128) return DSA_ERR_UNSUPPORTED;
  ProbsParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.lse = lse;
  p.cu_seqlens = latent->cu_seqlens;
  p.B = B;
  p.H = H;
  p.rows = row_end - row_begin;
  p.row0 = row_begin;
  p.ld = ld_p;
  p.scale_log2 = sm_scale * 1.4426950408889634f;
  p.p = p_out;
  const int smem = probs::kSmemBytes + 1024;
  if (cudaFuncSetAttribute(attn_probs_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
    return DSA_ERR_CUDA;
  const int64_t grid = p.rows < 148 ? p.rows : 148;
  attn_probs_kernel<true><<<static_cast<unsigned>(grid), probs::kThreads, smem, as_stream(stream)>>>(
      static_cast<const __nv_bfloat16*>(latent->data), p);
  return launch_status();
}

dsa_status dsa_indexer_backward(const uint8_t* q_fp8, const float* q_scale, int32_t q_scale_heads, const float* w,
                                const dsa_kv_desc* keys, int32_t B, int32_t H_I, int32_t d_I, const int32_t* idx,
                                const float* grad, int32_t k, float* dw, float* dq, float* dk, void* stream) {
  if (keys == nullptr || k <= 0 || B <= 0) return DSA_ERR_INVALID_ARGUMENT;
  if (keys->kind != DSA_KV_CONTIGUOUS) return DSA_ERR_UNSUPPORTED;
  if (q_fp8 == nullptr || q_scale == nullptr || w == nullptr || keys->data == nullptr || keys->scale == nullptr ||
      keys->cu_seqlens == nullptr || keys->total_tokens <= 0 || idx == nullptr || grad == nullptr || dw == nullptr ||
      dq == nullptr || dk == nullptr)
    return DSA_ERR_INVALID_ARGUMENT;
  if (q_scale_heads != 1 && q_scale_heads != H_I) return DSA_ERR_INVALID_ARGUMENT;
  if (!aligned(keys->data, 4) || !aligned(dk, 16) || !aligned(dq, 16)) return DSA_ERR_INVALID_ARGUMENT;
  if (!indexer_shape_ok(H_I, d_I)) return DSA_ERR_UNSUPPORTED;
  IdxBwdParams p;
  std::memset(&p, 0, sizeof(p));
  p.q8 = q_fp8;
  p.q_scale = q_scale;
  p.q_scale_heads = q_scale_heads;
  p.w = w;
  p.k8 = static_cast<const uint8_t*>(keys->data);
  p.k_scale = keys->scale;
  p.cu_seqlens = keys->cu_seqlens;
  p.B = B;
  p.idx = idx;
  p.grad = grad;
  p.k = k;
  p.rows = keys->total_tokens;
  p.dw = dw;
  p.dq = dq;
  p.dk = dk;
  cudaStream_t s = as_stream(stream);
  if (cudaMemsetAsync(dk, 0, static_cast<size_t>(keys->total_tokens) * d_I * sizeof(float), s) != cudaSuccess)
    return DSA_ERR_CUDA;
  auto launch = [&](auto kern, int smem) -> dsa_status {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess)
      return DSA_ERR_CUDA;
    const int64_t grid = p.rows < 2 * 148 ? p.rows : 2 * 148;
    kern<<<static_cast<unsigned>(grid), ibwd::kThreads, smem, s>>>(p);
    return launch_status();
  };
  if (H_I == 64 && d_I == 128) return launch(indexer_backward_h64_kernel<128>, ibwd::Layout64<128>::kSmemBytes);
  if (H_I == 64 && d_I == 64) return launch(indexer_backward_h64_kernel<64>, ibwd::Layout64<64>::kSmemBytes);
  if (H_I == 4 && d_I == 128) return launch(indexer_backward_kernel<4, 128>, ibwd::Layout<4, 128>::kSmemBytes);
  return launch(indexer_backward_kernel<4, 64>, ibwd::Layout<4, 64>::kSmemBytes);
}

dsa_status dsa_indexer_kl(const float* p, const float* scores, const int32_t* idx, int64_t rows, int32_t k,
                          float* loss, float* grad, void* stream) {
  if (rows < 0 || k <= 0) return DSA_ERR_INVALID_ARGUMENT;
  if (rows == 0) return DSA_OK;
  if (p == nullptr || scores == nullptr || idx == nullptr || loss == nullptr || grad == nullptr)
    return DSA_ERR_INVALID_ARGUMENT;
  if (rows > 0x7FFFFFFFLL) return DSA_ERR_UNSUPPORTED;
  indexer_kl_kernel<<<static_cast<unsigned>(rows), kl::kThreads, 0, as_stream(stream)>>>(p, scores, idx, k, loss, grad);
  return launch_status();
}

dsa_status dsa_selftest_wait_timeout(int32_t limit_us, void* stream) {
  if (limit_us <= 0 || limit_us > 2000000) return DSA_ERR_INVALID_ARGUMENT;
  wait_timeout_selftest_kernel<<<1, 32, 0, as_stream(stream)>>>(static_cast<uint64_t>(limit_us) * 1000u);
  return launch_status();
}

dsa_status dsa_quantize_fp8(const void* x_bf16, int64_t rows, int32_t cols, uint8_t* codes, float* scale,
                            void* stream) {
  if (rows < 0) return DSA_ERR_INVALID_ARGUMENT;
  if (rows == 0) return DSA_OK;
  if (cols <= 0 || (cols % 8) != 0) return DSA_ERR_INVALID_ARGUMENT;
  if (x_bf16 == nullptr || codes == nullptr || scale == nullptr || !aligned(x_bf16, 16) || !aligned(codes, 8))
    return DSA_ERR_INVALID_ARGUMENT;
  if (cols >= 2048 && cols <= quant::kWideThreads * quant::kWideMaxChunks * 8) {
    if (rows > 0x7FFFFFFFLL) return DSA_ERR_UNSUPPORTED;
    quantize_fp8_wide_kernel<<<static_cast<unsigned>(rows), quant::kWideThreads, 0, as_stream(stream)>>>(
        static_cast<const __nv_bfloat16*>(x_bf16), cols, codes, scale);
    return launch_status();
  }
  const int64_t blocks = (rows + quant::kWarps - 1) / quant::kWarps;
  if (blocks > 0x7FFFFFFFLL) return DSA_ERR_UNSUPPORTED;
  quantize_fp8_rows_kernel<<<static_cast<unsigned>(blocks), quant::kWarps * 32, 0, as_stream(stream)>>>(
      static_cast<const __nv_bfloat16*>(x_bf16), rows, cols, codes, scale);
  return launch_status();
}

dsa_status dsa_topk(const float* scores, int64_t ld_scores, int64_t rows, const int32_t* row_len, int32_t k,
                    int32_t* idx, void* stream) {
  if (rows < 0 || k <= 0 || ld_scores <= 0 || (ld_scores % 4) != 0) return DSA_ERR_INVALID_ARGUMENT;
  if (rows == 0) return DSA_OK;
  if (scores == nullptr || row_len == nullptr || idx == nullptr || !aligned(scores, 16))
    return DSA_ERR_INVALID_ARGUMENT;
  if (rows > 0x7FFFFFFFLL || ld_scores > 0x7FFFFFFFLL) return DSA_ERR_UNSUPPORTED;
  if (rows * kTopkCluster > 0x7FFFFFFFLL) return DSA_ERR_UNSUPPORTED;
  topk_rows_cluster_kernel<<<static_cast<unsigned>(rows * kTopkCluster), kTopkThreads, 0, as_stream(stream)>>>(
      scores, ld_scores, row_len, k, idx);
  return launch_status();
}

dsa_status dsa_indexer_scores(const uint8_t* q_fp8, const float* q_scale, int32_t q_scale_heads, const float* w,
                              const dsa_kv_desc* keys, int32_t B, int32_t H_I, int32_t d_I, int64_t row_begin,
                              int64_t row_end, float* scores, int64_t ld_scores, void* stream) {
  if (scores == nullptr || row_begin < 0 || row_end < row_begin) return DSA_ERR_INVALID_ARGUMENT;
  if (keys == nullptr) return DSA_ERR_INVALID_ARGUMENT;
  if (row_end == row_begin) return DSA_OK;
  CUtensorMap qm, km;
  IndexerParams p;
  dsa_status st = indexer_common(q_fp8, q_scale, q_scale_heads, w, keys, B, H_I, d_I, &qm, &km, &p);
  if (st != DSA_OK) return st;
  if (ld_scores < keys->max_seqlen) return DSA_ERR_INVALID_ARGUMENT;
  p.scores = scores;
  p.ld = ld_scores;
  p.row_begin = row_begin;
  p.row_end = row_end;
  if (keys->kind == DSA_KV_CONTIGUOUS) {
    if (row_end > keys->total_tokens) return DSA_ERR_INVALID_ARGUMENT;
    dim3 grid((keys->max_seqlen + kIdxTok - 1) / kIdxTok, B);
    return launch_indexer<kIdxScores, false>(d_I, H_I, qm, km, p, grid, as_stream(stream));
  }
  if (row_end > B) return DSA_ERR_INVALID_ARGUMENT;
  dim3 grid((keys->max_seqlen + 128 * kDecodeTilesPerCta - 1) / (128 * kDecodeTilesPerCta), B);
  return launch_indexer<kIdxScores, true>(d_I, H_I, qm, km, p, grid, as_stream(stream));
}

dsa_status dsa_indexer_topk(const uint8_t* q_fp8, const float* q_scale, int32_t q_scale_heads, const float* w,
                            const dsa_kv_desc* keys, int32_t B, int32_t H_I, int32_t d_I, int32_t k, int32_t* idx_out,
                            void* stream) {
  if (idx_out == nullptr || keys == nullptr || k <= 0) return DSA_ERR_INVALID_ARGUMENT;
  if (keys->kind != DSA_KV_CONTIGUOUS) return DSA_ERR_UNSUPPORTED;
  if (k > 2048) return DSA_ERR_UNSUPPORTED;
  CUtensorMap qm, km;
  IndexerParams p;
  dsa_status st = indexer_common(q_fp8, q_scale, q_scale_heads, w, keys, B, H_I, d_I, &qm, &km, &p);
  if (st != DSA_OK) return st;
  int stages;
  st = topk_config(d_I, keys->max_seqlen, k, &stages, &p.cap);
  if (st != DSA_OK) return st;
  p.idx_out = idx_out;
  p.k = k;
  dim3 grid((keys->max_seqlen + kIdxTok - 1) / kIdxTok, B);
  return launch_indexer<kIdxTopk, false>(d_I, H_I, qm, km, p, grid, as_stream(stream), stages);
}

dsa_status dsa_indexer_topk_rows(const uint8_t* q_fp8, const float* q_scale, int32_t q_scale_heads, const float* w,
                                 const dsa_kv_desc* keys, int32_t H_I, int32_t d_I, int32_t k, int64_t row_begin,
                                 int64_t row_end, int32_t* idx_out, void* stream) {
  if (keys == nullptr || k <= 0 || row_begin < 0 || row_end < row_begin) return DSA_ERR_INVALID_ARGUMENT;
  if (keys->kind != DSA_KV_CONTIGUOUS) return DSA_ERR_UNSUPPORTED;
  if (k > 2048) return DSA_ERR_UNSUPPORTED;
  if (row_end > keys->total_tokens) return DSA_ERR_INVALID_ARGUMENT;
  if (row_end == row_begin) return DSA_OK;  // an empty block: nothing to read or write
  if (idx_out == nullptr) return DSA_ERR_INVALID_ARGUMENT;
  CUtensorMap qm, km;
  IndexerParams p;
  dsa_status st = indexer_common(q_fp8, q_scale, q_scale_heads, w, keys, 1, H_I, d_I, &qm, &km, &p,
                                 row_end - row_begin);
  if (st != DSA_OK) return st;
  int stages;
  st = topk_config(d_I, keys->max_seqlen, k, &stages, &p.cap);
  if (st != DSA_OK) return st;
  p.idx_out = idx_out;
  p.k = k;
  p.tok_begin = static_cast<int32_t>(row_begin);
  p.tok_end = static_cast<int32_t>(row_end);
  p.q_row0 = row_begin;
  dim3 grid(static_cast<unsigned>((row_end - row_begin + kIdxTok - 1) / kIdxTok), 1);
  return launch_indexer<kIdxTopk, false>(d_I, H_I, qm, km, p, grid, as_stream(stream), stages);
}

size_t dsa_decode_select_workspace_size(int32_t B, int32_t max_ctx) {
  if (B <= 0 || max_ctx <= 0) return 0;
  const int64_t ld = (static_cast<int64_t>(max_ctx) + 3) / 4 * 4;
  const int64_t ld16 = ((static_cast<int64_t>(max_ctx) + kSelGroup - 1) / kSelGroup + 3) / 4 * 4;
  return align256(static_cast<size_t>(B) * ld * 4) + align256(static_cast<size_t>(B) * ld16 * 4);
}

dsa_status dsa_indexer_topk_decode(const uint8_t* q_fp8, const float* q_scale, int32_t q_scale_heads, const float* w,
                                   const dsa_kv_desc* keys, int32_t B, int32_t H_I, int32_t d_I, int32_t k,
                                   int32_t* idx_out, void* workspace, size_t ws_bytes, void* stream) {
  if (keys == nullptr || idx_out == nullptr || k <= 0 || B <= 0) return DSA_ERR_INVALID_ARGUMENT;
  if (keys->kind != DSA_KV_PAGED) return DSA_ERR_UNSUPPORTED;
  if (workspace == nullptr || !aligned(workspace, 256)) return DSA_ERR_INVALID_ARGUMENT;
  if (static_cast<int64_t>(B) * kTopkCluster > 0x7FFFFFFFLL) return DSA_ERR_UNSUPPORTED;
  CUtensorMap qm, km;
  IndexerParams p;
  dsa_status st = indexer_common(q_fp8, q_scale, q_scale_heads, w, keys, B, H_I, d_I, &qm, &km, &p);
  if (st != DSA_OK) return st;
  if (ws_bytes < dsa_decode_select_workspace_size(B, keys->max_seqlen)) return DSA_ERR_WORKSPACE_TOO_SMALL;
  // workspace: [scores B x ld fp32][group maxima B x ld16 u32]
  const int64_t ld = (static_cast<int64_t>(keys->max_seqlen) + 3) / 4 * 4;
  const int64_t ld16 = ((static_cast<int64_t>(keys->max_seqlen) + kSelGroup - 1) / kSelGroup + 3) / 4 * 4;
  p.scores = static_cast<float*>(workspace);
  p.ld = ld;
  p.row_begin = 0;
  p.row_end = B;
  p.gmax = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + align256(static_cast<size_t>(B) * ld * 4));
  p.ld16 = ld16;
  cudaStream_t s = as_stream(stream);
  dim3 grid((keys->max_seqlen + 128 * kDecodeTilesPerCta - 1) / (128 * kDecodeTilesPerCta), B);
  st = launch_indexer<kIdxScores, true>(d_I, H_I, qm, km, p, grid, s);
  if (st != DSA_OK) return st;
  if (cudaFuncSetAttribute(topk_decode_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSelSmemBytes) !=
      cudaSuccess)
    return DSA_ERR_CUDA;
  topk_decode_select_kernel<<<static_cast<unsigned>(B * kTopkCluster), kTopkThreads, kSelSmemBytes, s>>>(
      p.scores, ld, p.gmax, ld16, keys->context_lens, keys->max_seqlen, k, idx_out);
  return launch_status();
}

dsa_status dsa_sparse_mla_prefill_rows(const void* q, const dsa_kv_desc* latent, const int32_t* idx, int32_t H,
                                       int32_t k, float sm_scale, int64_t row_begin, int64_t row_end, void* out,
                                       float* lse, void* stream) {
  if (latent == nullptr || latent->kind != DSA_KV_CONTIGUOUS || latent->cu_seqlens == nullptr ||
      latent->total_tokens <= 0)
    return DSA_ERR_INVALID_ARGUMENT;
  if (row_begin < 0 || row_end < row_begin || row_end > latent->total_tokens) return DSA_ERR_INVALID_ARGUMENT;
  if (row_end == row_begin) return DSA_OK;  // an empty block: nothing to read or write
  if (q == nullptr || latent->data == nullptr || idx == nullptr || out == nullptr) return DSA_ERR_INVALID_ARGUMENT;
  if (!aligned(q, 16) || !aligned(latent->data, 16) || !aligned(idx, 16) || !aligned(out, 16))
    return DSA_ERR_INVALID_ARGUMENT;
  if (!mla_shape_ok(H, k)) return DSA_ERR_UNSUPPORTED;
  if (latent->total_tokens > 0x7FFFFFFFLL) return DSA_ERR_UNSUPPORTED;
  MlaParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.idx = idx;
  p.cu_seqlens = latent->cu_seqlens;
  p.B = 1;
  p.H = H;
  p.k = k;
  p.rows = row_end - row_begin;
  p.unit0 = row_begin;
  p.splits = 1;
  p.scale_log2 = sm_scale * 1.4426950408889634f;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  return launch_mla_pair<false>(latent->data, q, p.rows, p, p.rows, as_stream(stream));
}

dsa_status dsa_sparse_mla_prefill(const void* q, const dsa_kv_desc* latent, const int32_t* idx, int32_t B, int32_t H,
                                  int32_t k, float sm_scale, void* out, float* lse, void* stream) {
  if (q == nullptr || latent == nullptr || latent->data == nullptr || idx == nullptr || out == nullptr || B <= 0)
    return DSA_ERR_INVALID_ARGUMENT;
  if (latent->kind != DSA_KV_CONTIGUOUS || latent->cu_seqlens == nullptr || latent->total_tokens <= 0)
    return DSA_ERR_INVALID_ARGUMENT;
  if (!aligned(q, 16) || !aligned(latent->data, 16) || !aligned(idx, 16) || !aligned(out, 16))
    return DSA_ERR_INVALID_ARGUMENT;
  if (!mla_shape_ok(H, k)) return DSA_ERR_UNSUPPORTED;
  if (latent->total_tokens > 0x7FFFFFFFLL) return DSA_ERR_UNSUPPORTED;
  MlaParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.idx = idx;
  p.cu_seqlens = latent->cu_seqlens;
  p.B = B;
  p.H = H;
  p.k = k;
  p.rows = latent->total_tokens;
  p.splits = 1;
  p.scale_log2 = sm_scale * 1.4426950408889634f;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  return launch_mla_pair<false>(latent->data, q, p.rows, p, p.rows, as_stream(stream));
}

dsa_status dsa_masked_mla_prefill(const void* q, const dsa_kv_desc* latent, const int32_t* idx, int32_t B, int32_t H,
                                  int32_t k, float sm_scale, void* out, float* lse, void* stream) {
  if (q == nullptr || latent == nullptr || latent->data == nullptr || idx == nullptr || out == nullptr || B <= 0)
    return DSA_ERR_INVALID_ARGUMENT;
  if (latent->kind != DSA_KV_CONTIGUOUS || latent->cu_seqlens == nullptr || latent->total_tokens <= 0)
    return DSA_ERR_INVALID_ARGUMENT;
  if (!aligned(q, 16) || !aligned(latent->data, 16) || !aligned(idx, 16) || !aligned(out, 16))
    return DSA_ERR_INVALID_ARGUMENT;
  if (!mla_shape_ok(H, k)) return DSA_ERR_UNSUPPORTED;
  if (latent->total_tokens > 0x7FFFFFFFLL) return DSA_ERR_UNSUPPORTED;
  MlaParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.idx = idx;
  p.cu_seqlens = latent->cu_seqlens;
  p.B = B;
  p.H = H;
  p.k = k;
  p.rows = latent->total_tokens;
  p.splits = 1;
  p.scale_log2 = sm_scale * 1.4426950408889634f;
  p.out = static_cast<__nv_bfloat16*>(out);
  p.lse = lse;
  return launch_mla_pair<false, true>(latent->data, q, p.rows, p, p.rows, as_stream(stream));
}

dsa_status dsa_sparse_mla_decode(const void* q, const dsa_kv_desc* latent, const int32_t* idx, int32_t B, int32_t H,
                                 int32_t k, float sm_scale, void* out, float* lse, void* workspace, size_t ws_bytes,
                                 void* stream) {
  if (q == nullptr || latent == nullptr || latent->data == nullptr || idx == nullptr || out == nullptr || B <= 0)
    return DSA_ERR_INVALID_ARGUMENT;
  if (latent->kind != DSA_KV_PAGED || latent->block_table == nullptr || latent->context_lens == nullptr ||
      latent->num_blocks <= 0 || latent->max_blocks_per_seq <= 0)
    return DSA_ERR_INVALID_ARGUMENT;
  if (latent->block_size != 64) return DSA_ERR_UNSUPPORTED;
  if (!aligned(q, 16) || !aligned(latent->data, 16) || !aligned(idx, 16) || !aligned(out, 16))
    return DSA_ERR_INVALID_ARGUMENT;
  if (!mla_shape_ok(H, k)) return DSA_ERR_UNSUPPORTED;
  if (static_cast<int64_t>(latent->num_blocks) * 64 > 0x7FFFFFFFLL) return DSA_ERR_UNSUPPORTED;
  const int splits = decode_splits(B, k);
  if (workspace == nullptr || ws_bytes < decode_partials_bytes(B, H, splits) || !aligned(workspace, 256))
    return workspace == nullptr ? DSA_ERR_INVALID_ARGUMENT : DSA_ERR_WORKSPACE_TOO_SMALL;
  MlaParams p;
  std::memset(&p, 0, sizeof(p));
  p.q = static_cast<const __nv_bfloat16*>(q);
  p.idx = idx;
  p.block_table = latent->block_table;
  p.context_lens = latent->context_lens;
  p.max_blocks_per_seq = latent->max_blocks_per_seq;
  p.num_blocks = latent->num_blocks;
  p.B = B;
  p.H = H;
  p.k = k;
  p.rows = B;
  p.splits = splits;
  p.scale_log2 = sm_scale * 1.4426950408889634f;
  p.part_o = static_cast<float*>(workspace);
  p.part_ml = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                       align256(static_cast<size_t>(B) * splits * H * kValueDim * 4));
  p.out = static_cast<__nv_bfloat16*>(out);  // one split: the kernel writes out / lse itself
  p.lse = lse;
  cudaStream_t s = as_stream(stream);
  dsa_status st = launch_mla_pair<true>(latent->data, q, B, p, static_cast<int64_t>(B) * splits, s);
  if (st != DSA_OK) return st;
  if (splits == 1) return DSA_OK;
  mla_combine_kernel<<<dim3(H, B), 128, 0, s>>>(p.part_o, p.part_ml, splits, H, static_cast<__nv_bfloat16*>(out), lse);
  return launch_status();
}

dsa_status dsa_sparse_mla_decode_noalloc(const void* q, const dsa_kv_desc* latent, const int32_t* idx, int32_t B,
                                         int32_t H, int32_t k, float sm_scale, void* out, float* lse, void* stream) {
  if (B <= 0) return DSA_ERR_INVALID_ARGUMENT;
  if (!mla_shape_ok(H, k)) return DSA_ERR_UNSUPPORTED;
  if (decode_partials_bytes(B, H, decode_splits(B, k)) > DSA_NOALLOC_SCRATCH_BYTES) return DSA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  const dsa_status st = noalloc_scratch(&scratch);
  if (st != DSA_OK) return st;
  return dsa_sparse_mla_decode(q, latent, idx, B, H, k, sm_scale, out, lse, scratch, DSA_NOALLOC_SCRATCH_BYTES,
                               stream);
}

dsa_status dsa_forward(int32_t mode, const uint8_t* q_fp8, const float* q_scale, int32_t q_scale_heads,
                       const float* w, const dsa_kv_desc* keys, const void* q, const dsa_kv_desc* latent, int32_t B,
                       int32_t H_I, int32_t d_I, int32_t H, int32_t k, float sm_scale, void* out, float* lse,
                       int32_t* idx_out, void* workspace, size_t ws_bytes, void* stream) {
  if (keys == nullptr || latent == nullptr || B <= 0) return DSA_ERR_INVALID_ARGUMENT;
  if (!mla_shape_ok(H, k)) return DSA_ERR_UNSUPPORTED;
  const size_t need = dsa_workspace_size(mode, B, keys->total_tokens, keys->max_seqlen, H, k);
  if (mode == DSA_MODE_PREFILL) {
    if (keys->kind != DSA_KV_CONTIGUOUS || latent->kind != DSA_KV_CONTIGUOUS) return DSA_ERR_INVALID_ARGUMENT;
    int32_t* idx = idx_out;
    if (idx == nullptr) {
      if (workspace == nullptr) return DSA_ERR_INVALID_ARGUMENT;
      if (ws_bytes < need) return DSA_ERR_WORKSPACE_TOO_SMALL;
      idx = static_cast<int32_t*>(workspace);
    }
    dsa_status st = dsa_indexer_topk(q_fp8, q_scale, q_scale_heads, w, keys, B, H_I, d_I, k, idx, stream);
    if (st != DSA_OK) return st;
    return dsa_sparse_mla_prefill(q, latent, idx, B, H, k, sm_scale, out, lse, stream);
  }
  if (mode != DSA_MODE_DECODE) return DSA_ERR_INVALID_ARGUMENT;
  if (keys->kind != DSA_KV_PAGED || latent->kind != DSA_KV_PAGED) return DSA_ERR_INVALID_ARGUMENT;
  if (workspace == nullptr) return DSA_ERR_INVALID_ARGUMENT;
  if (ws_bytes < need || !aligned(workspace, 256)) return DSA_ERR_WORKSPACE_TOO_SMALL;
  // workspace: [decode partials][selection workspace: scores, group maxima][selection B x k]
  const int splits = decode_splits(B, k);
  const size_t part = decode_partials_bytes(B, H, splits);
  const size_t sel = dsa_decode_select_workspace_size(B, keys->max_seqlen);
  int32_t* idx = idx_out != nullptr ? idx_out
                                    : reinterpret_cast<int32_t*>(static_cast<uint8_t*>(workspace) + part + sel);
  dsa_status st = dsa_indexer_topk_decode(q_fp8, q_scale, q_scale_heads, w, keys, B, H_I, d_I, k, idx,
                                          static_cast<uint8_t*>(workspace) + part, sel, stream);
  if (st != DSA_OK) return st;
  return dsa_sparse_mla_decode(q, latent, idx, B, H, k, sm_scale, out, lse, workspace, part, stream);
}

dsa_status dsa_row_partition(int64_t L, int32_t k, int32_t parts, double indexer_cost, double mla_cost,
                             int64_t* bounds) {
  if (bounds == nullptr || L < 1 || k < 1 || parts < 1 || parts > L) return DSA_ERR_INVALID_ARGUMENT;
  if (!(indexer_cost >= 0.0) || !(mla_cost >= 0.0) || !(indexer_cost + mla_cost > 0.0)) return DSA_ERR_INVALID_ARGUMENT;
  // cost of rows [0, n): indexer_cost * C(n) / C(L) + mla_cost * M(n) / M(L), with
  // C(n) = sum_{t<n} (t+1) (the causal prefixes the indexer scans) and
  // M(n) = sum_{t<n} min(t+1, k) (the rows sparse MLA attends to)
  const double kk = static_cast<double>(k);
  auto C = [](double n) { return n * (n + 1.0) / 2.0; };
  auto M = [&](double n) { return n <= kk ? n * (n + 1.0) / 2.0 : kk * (kk + 1.0) / 2.0 + (n - kk) * kk; };
  const double Lf = static_cast<double>(L), CL = C(Lf), ML = M(Lf);
  auto cost = [&](int64_t n) {
    const double x = static_cast<double>(n);
    return indexer_cost * C(x) / CL + mla_cost * M(x) / ML;
  };
  const double total = cost(L);
  bounds[0] = 0;
  for (int32_t r = 1; r < parts; ++r) {
    const double target = total * static_cast<double>(r) / static_cast<double>(parts);
    int64_t lo = bounds[r - 1] + 1, hi = L - (parts - r);  // every block keeps at least one row
    if (lo > hi) return DSA_ERR_INVALID_ARGUMENT;
    while (lo < hi) {  // the first boundary whose cost reaches the target
      const int64_t mid = lo + (hi - lo) / 2;
      if (cost(mid) >= target) hi = mid;
      else lo = mid + 1;
    }
    bounds[r] = lo;
  }
  bounds[parts] = L;
  return DSA_OK;
}

size_t dsa_workspace_size(int32_t mode, int32_t B, int64_t total_tokens, int32_t max_ctx, int32_t H, int32_t k) {
  if (B <= 0 || k <= 0 || H <= 0) return 0;
  if (mode == DSA_MODE_PREFILL) return align256(static_cast<size_t>(total_tokens > 0 ? total_tokens : 0) * k * 4);
  return decode_partials_bytes(B, H, decode_splits(B, k)) + dsa_decode_select_workspace_size(B, max_ctx) +
         align256(static_cast<size_t>(B) * k * 4);
}

}  // extern "C"
