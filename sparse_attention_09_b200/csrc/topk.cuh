// Row-wise top-k over fp32 index scores (fine-grained token selection).
//
// One CTA per row.  A 4-pass radix select over the order-preserving 32-bit keys of the
// scores (8 bits per pass, warp-private histograms) finds the key of the k-th largest entry
// and how many entries equal to it are still needed; an emit pass then walks the row in
// index order and writes the selected indices with a block-wide scan, so the output is
// ascending and ties at the boundary go to the lowest indices.
#pragma once

#include "common.cuh"

namespace dsa {

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkTile = 4 * kTopkThreads;  // one float4 per thread per step

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
      const int i0 = base + 4 * tid;
      if (i0 < n) {
        const float4 v = *reinterpret_cast<const float4*>(row + i0);
        const float f[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
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
    const int i0 = base + 4 * tid;
    bool g[4] = {false, false, false, false}, e[4] = {false, false, false, false};
    if (i0 < n) {
      const float4 v = *reinterpret_cast<const float4*>(row + i0);
      const float f[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        if (i0 + j < n) {
          const uint32_t key = order_key(f[j]);
          g[j] = key > thr;
          e[j] = key == thr;
        }
      }
    }
    const int ne = int(e[0]) + int(e[1]) + int(e[2]) + int(e[3]);
    int tie_total;
    int tie_rank = eq_taken + block_exclusive_scan<kTopkWarps>(ne, scan_scratch, tie_total);
    bool sel[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      sel[j] = g[j];
      if (e[j]) {
        sel[j] = tie_rank < need_eq;
        ++tie_rank;
      }
    }
    const int ns = int(sel[0]) + int(sel[1]) + int(sel[2]) + int(sel[3]);
    int sel_total;
    int pos = out_pos + block_exclusive_scan<kTopkWarps>(ns, scan_scratch, sel_total);
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (sel[j]) out[pos++] = i0 + j;
    eq_taken += tie_total;
    out_pos += sel_total;
  }
}

}  // namespace dsa
