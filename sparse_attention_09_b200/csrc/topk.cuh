// Row-wise top-k over fp32 index scores (fine-grained token selection).
//
// One CTA per row.  A 4-pass radix select over the order-preserving 32-bit keys of the
// scores (8 bits per pass, warp-private histograms) finds the key of the k-th largest entry
// and how many entries equal to it are still needed; an emit pass then walks the row in
// index order and writes the selected indices with a block-wide scan, so the output is
// ascending and ties at the boundary go to the lowest indices.  Each thread takes 16
// consecutive scores per step (four 16-byte loads in flight), so a step covers 8192 scores.
#pragma once

#include "common.cuh"

namespace dsa {

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkVec = 4;                               // float4 loads per thread per step
constexpr int kTopkTile = 4 * kTopkVec * kTopkThreads;    // scores per step

// The 16 scores [i0, i0 + 16) of a row of length n (entries past n are not loaded; a row
// buffer of ld >= n elements, ld % 4 == 0, holds every float4 that starts before n).
__device__ __forceinline__ void topk_load16(const float* row, int i0, int n, float (&f)[16]) {
#pragma unroll
  for (int v = 0; v < kTopkVec; ++v) {
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (i0 + 4 * v < n) x = *reinterpret_cast<const float4*>(row + i0 + 4 * v);
    f[4 * v] = x.x;
    f[4 * v + 1] = x.y;
    f[4 * v + 2] = x.z;
    f[4 * v + 3] = x.w;
  }
}

__global__ void __launch_bounds__(kTopkThreads) topk_rows_kernel(const float* __restrict__ scores, int64_t ld,
                                                                 const int32_t* __restrict__ row_len, int32_t k,
                                                                 int32_t* __restrict__ idx) {
  __shared__ uint32_t hist[kTopkWarps][256];
  __shared__ uint32_t total[256];
  __shared__ int scan_scratch[kTopkWarps];
  __shared__ uint32_t s_bin, s_remaining;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t r = blockIdx.x;
  const float* row = scores + r * ld;
  int32_t* out = idx + r * static_cast<int64_t>(k);
  const int n = row_len[r];

  if (n <= k) {  // every candidate is selected
    for (int i = tid; i < k; i += kTopkThreads) out[i] = i < n ? i : -1;
    return;
  }

  uint32_t prefix = 0, mask = 0, remaining = static_cast<uint32_t>(k);
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < kTopkWarps * 256; i += kTopkThreads) (&hist[0][0])[i] = 0u;
    __syncthreads();
#pragma unroll 1
    for (int base = 0; base < n; base += kTopkTile) {
      const int i0 = base + 16 * tid;
      if (i0 < n) {
        float f[16];
        topk_load16(row, i0, n, f);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if (i0 + j < n) {
            if (pass == 0 && is_nan_bits(__float_as_uint(f[j]))) record_device_error(DSA_ERR_DEVICE_CHECK);
            const uint32_t key = order_key(f[j]);
            if ((key & mask) == prefix) atomicAdd(&hist[warp][(key >> shift) & 255u], 1u);
          }
        }
      }
    }
    __syncthreads();
    if (tid < 256) {
      uint32_t s = 0;
#pragma unroll
      for (int w = 0; w < kTopkWarps; ++w) s += hist[w][tid];
      total[tid] = s;
    }
    __syncthreads();
    if (warp == 0) {
      // Lane l owns bins 255-8l-7 .. 255-8l, visited from the top down.
      uint32_t c[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = total[255 - (8 * lane + j)];
        sum += c[j];
      }
      const uint32_t inc = static_cast<uint32_t>(warp_inclusive_scan(static_cast<int>(sum)));
      const uint32_t before = inc - sum;
      if (before < remaining && remaining <= inc) {
        uint32_t acc = before;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (acc + c[j] >= remaining) {
            s_bin = 255u - static_cast<uint32_t>(8 * lane + j);
            s_remaining = remaining - acc;
            break;
          }
          acc += c[j];
        }
      }
    }
    __syncthreads();
    prefix |= s_bin << shift;
    mask |= 255u << shift;
    remaining = s_remaining;
    __syncthreads();
  }

  // Emit in index order: keys above the threshold, plus the first `remaining` equal keys.
  const uint32_t thr = prefix;
  const int need_eq = static_cast<int>(remaining);
  int eq_taken = 0, out_pos = 0;
#pragma unroll 1
  for (int base = 0; base < n && out_pos < k; base += kTopkTile) {
    const int i0 = base + 16 * tid;
    uint32_t gbits = 0u, ebits = 0u;  // bit j: score i0 + j is above / equal to the threshold
    if (i0 < n) {
      float f[16];
      topk_load16(row, i0, n, f);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (i0 + j < n) {
          const uint32_t key = order_key(f[j]);
          gbits |= static_cast<uint32_t>(key > thr) << j;
          ebits |= static_cast<uint32_t>(key == thr) << j;
        }
      }
    }
    int tie_total;
    int tie_rank = eq_taken + block_exclusive_scan<kTopkWarps>(__popc(ebits), scan_scratch, tie_total);
    uint32_t sbits = gbits;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if ((ebits >> j) & 1u) {
        if (tie_rank < need_eq) sbits |= 1u << j;
        ++tie_rank;
      }
    }
    int sel_total;
    int pos = out_pos + block_exclusive_scan<kTopkWarps>(__popc(sbits), scan_scratch, sel_total);
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if ((sbits >> j) & 1u) out[pos++] = i0 + j;
    eq_taken += tie_total;
    out_pos += sel_total;
  }
}

}  // namespace dsa
