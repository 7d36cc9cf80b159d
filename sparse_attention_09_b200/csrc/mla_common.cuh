// Parameters and small device helpers shared by the sparse MLA paths (the head-split pair
// kernel in its sparse, masked and decode forms), and the log-sum-exp merge of split decode
// selections.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace dsa {

struct MlaParams {
  const __nv_bfloat16* q;     // [rows, H, 576]
  const int32_t* idx;         // [rows, k]
  const int32_t* cu_seqlens;  // prefill [B+1]
  const int32_t* block_table; // decode [B, max_blocks_per_seq]
  const int32_t* context_lens;// decode [B]
  int32_t max_blocks_per_seq;
  int32_t num_blocks;         // decode: blocks in the paged latent pool
  int32_t B;
  int32_t H;                  // query heads (<= 128; rows >= H are padding)
  int32_t k;                  // selected entries per row (multiple of 64)
  int64_t rows;               // prefill: tokens (units) to process; decode: B
  int64_t unit0;              // prefill: packed token of unit 0 (row 0 of q, idx, out, lse)
  int32_t splits;             // decode: selection splits per sequence
  float scale_log2;           // sm_scale * log2(e)
  __nv_bfloat16* out;         // prefill: [rows, H, 512]
  float* lse;                 // prefill: [rows, H] natural log (nullable)
  float* part_o;              // decode: [B, splits, H, 512] unnormalised
  float* part_ml;             // decode: [B, splits, H, 2] (M in log2 units, l)
};

namespace mla {

constexpr int kChunk = 64;  // selection entries per pipeline step

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Number of 64-entry chunks up to the last valid (>= 0) index of a selection row, computed by
// one warp (all roles compute it the same way from the same row).
__device__ __forceinline__ int active_chunks(const int32_t* row, int k) {
  const int lane = threadIdx.x & 31;
  int last = -1;
  for (int j = lane; j < k; j += 32)
    if (row[j] >= 0) last = j;
  last = __reduce_max_sync(0xffffffffu, last);
  return last < 0 ? 1 : last / kChunk + 1;
}

}  // namespace mla

// Merges the per-split partial results of decode: out = sum_s 2^(M_s - M) O_s / sum_s 2^(M_s - M) l_s.
__global__ void __launch_bounds__(128) mla_combine_kernel(const float* __restrict__ part_o,
                                                          const float* __restrict__ part_ml, int splits, int H,
                                                          __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
  const int b = blockIdx.y, h = blockIdx.x;
  float Mmax = -INFINITY;
  for (int s = 0; s < splits; ++s) {
    const float* ml = part_ml + ((static_cast<int64_t>(b) * splits + s) * H + h) * 2;
    if (ml[1] > 0.f) Mmax = fmaxf(Mmax, ml[0]);
  }
  float wsum = 0.f;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int s = 0; s < splits; ++s) {
    const float* ml = part_ml + ((static_cast<int64_t>(b) * splits + s) * H + h) * 2;
    if (!(ml[1] > 0.f)) continue;
    const float wgt = exp2f(ml[0] - Mmax);
    wsum += wgt * ml[1];
    const float4 o = *reinterpret_cast<const float4*>(part_o + ((static_cast<int64_t>(b) * splits + s) * H + h) * 512 +
                                                      4 * threadIdx.x);
    acc[0] += wgt * o.x;
    acc[1] += wgt * o.y;
    acc[2] += wgt * o.z;
    acc[3] += wgt * o.w;
  }
  const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
  __nv_bfloat16* orow = out + (static_cast<int64_t>(b) * H + h) * 512 + 4 * threadIdx.x;
  const uint32_t lo = dev::pack_bf16x2(acc[0] * inv, acc[1] * inv), hi = dev::pack_bf16x2(acc[2] * inv, acc[3] * inv);
  *reinterpret_cast<uint2*>(orow) = make_uint2(lo, hi);
  if (lse != nullptr && threadIdx.x == 0)
    lse[static_cast<int64_t>(b) * H + h] = wsum > 0.f ? (Mmax + log2f(wsum)) * 0.69314718055994531f : -INFINITY;
}

}  // namespace dsa
