// Per-token FP8 (e4m3) quantiser for the lightning indexer's operands.
//
// The indexer runs in FP8 with one fp32 scale per token ("DeepSeek-V3.2 论文解读", section 二,
// subsection "工作原理": the indexer may run in FP8).  For a token row x (all of its indexer heads for
// q_I, its single key for k_I):
//   scale = amax(|x|) / 448   (1 for an all-zero row),   codes = e4m3(x / scale)
// with both divisions in IEEE fp32 and the e4m3 encoding rounding to nearest-even, saturating
// at +-448 (the largest finite e4m3 value); NaN stays NaN.
//
// HBM-bound.  Wide rows (2048..8192 columns, e.g. a token's 64 x 128 q_I): one CTA per row
// holds the row in registers, so it is read from HBM once.  Narrow rows (k_I's 128 columns):
// one warp per row reads the row twice (the second read is served by L1) and writes one byte
// per element plus the scale; lane l handles the 16-byte chunks l, l+32, ...
#pragma once

#include <cuda_bf16.h>

#include "common.cuh"

namespace dsa {

namespace quant {
constexpr int kWarps = 8;  // rows per CTA
constexpr float kE4m3Max = 448.f;

// Two fp32 values to two e4m3 bytes (first value in the low byte), round-to-nearest-even,
// saturating to the largest finite magnitude.
__device__ __forceinline__ uint16_t to_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// 8 bf16 values (one 16-byte chunk) divided by s and encoded, as 8 bytes.
__device__ __forceinline__ uint2 encode_chunk(const uint4 v, float s) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t out[2];
#pragma unroll
  for (int i = 0; i < 4; i += 2) {
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i + 1]));
    const uint32_t lo = to_e4m3x2(__fdiv_rn(a.x, s), __fdiv_rn(a.y, s));
    const uint32_t hi = to_e4m3x2(__fdiv_rn(b.x, s), __fdiv_rn(b.y, s));
    out[i / 2] = lo | (hi << 16);
  }
  return make_uint2(out[0], out[1]);
}

__device__ __forceinline__ float chunk_amax(const uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  float m = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[i]));
    m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));  // a NaN element never wins fmaxf
  }
  return m;
}

constexpr int kWideThreads = 256;
constexpr int kWideMaxChunks = 4;  // per thread: rows up to 256 x 4 x 8 = 8192 columns
}  // namespace quant

// One CTA per row, the row held in registers (cols a multiple of 8, 2048 <= cols <= 8192).
__global__ void __launch_bounds__(quant::kWideThreads)
    quantize_fp8_wide_kernel(const __nv_bfloat16* __restrict__ x, int cols, uint8_t* __restrict__ codes,
                             float* __restrict__ scale) {
  const int64_t row = blockIdx.x;
  const int nchunks = cols / 8;
  const uint4* src = reinterpret_cast<const uint4*>(x + row * cols);
  uint4 v[quant::kWideMaxChunks];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < quant::kWideMaxChunks; ++i) {
    const int c = threadIdx.x + i * quant::kWideThreads;
    if (c < nchunks) {
      v[i] = __ldg(src + c);
      amax = fmaxf(amax, quant::chunk_amax(v[i]));
    }
  }
  __shared__ uint32_t red[quant::kWideThreads / 32];
  const uint32_t wmax = __reduce_max_sync(0xffffffffu, __float_as_uint(amax));  // non-negative: bit order
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = wmax;
  __syncthreads();
  uint32_t m = red[0];
#pragma unroll
  for (int i = 1; i < quant::kWideThreads / 32; ++i) m = max(m, red[i]);
  amax = __uint_as_float(m);
  const float s = amax > 0.f ? __fdiv_rn(amax, quant::kE4m3Max) : 1.f;
  if (threadIdx.x == 0) scale[row] = s;
  uint2* dst = reinterpret_cast<uint2*>(codes + row * cols);
#pragma unroll
  for (int i = 0; i < quant::kWideMaxChunks; ++i) {
    const int c = threadIdx.x + i * quant::kWideThreads;
    if (c < nchunks) dst[c] = quant::encode_chunk(v[i], s);
  }
}

__global__ void __launch_bounds__(quant::kWarps * 32)
    quantize_fp8_rows_kernel(const __nv_bfloat16* __restrict__ x, int64_t rows, int cols,
                             uint8_t* __restrict__ codes, float* __restrict__ scale) {
  const int lane = threadIdx.x & 31;
  const int64_t row = static_cast<int64_t>(blockIdx.x) * quant::kWarps + (threadIdx.x >> 5);
  if (row >= rows) return;
  const int nchunks = cols / 8;
  const uint4* src = reinterpret_cast<const uint4*>(x + row * cols);
  float amax = 0.f;
  for (int c = lane; c < nchunks; c += 32) amax = fmaxf(amax, quant::chunk_amax(__ldg(src + c)));
  // non-negative floats order like their bit patterns
  amax = __uint_as_float(__reduce_max_sync(0xffffffffu, __float_as_uint(amax)));
  const float s = amax > 0.f ? __fdiv_rn(amax, quant::kE4m3Max) : 1.f;
  if (lane == 0) scale[row] = s;
  uint2* dst = reinterpret_cast<uint2*>(codes + row * cols);
  for (int c = lane; c < nchunks; c += 32) dst[c] = quant::encode_chunk(__ldg(src + c), s);
}

}  // namespace dsa
