// Row-wise top-k over fp32 index scores (fine-grained token selection).
//
// A 4-pass radix select over the order-preserving 32-bit keys of the
// scores (8 bits per pass, warp-private histograms) finds the key of the k-th largest entry
// and how many entries equal to it are still needed; an emit pass then walks the row in
// index order and writes the selected indices with a block-wide scan, so the output is
// ascending and ties at the boundary go to the lowest indices.  Each thread takes 16
// consecutive scores per step (four 16-byte loads in flight), so a step covers 8192 scores.
// A row is handled by a cluster of CTAs (below).
#pragma once

#include "common.cuh"
#include "sm100.cuh"

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

// A cluster of C CTAs per row, each taking a contiguous segment of it
// (a multiple of 16 scores).  Every radix pass merges the C segment histograms through
// distributed shared memory, so all CTAs take the same decision; each CTA also counts, from
// its own histograms, its scores above the final threshold and its scores equal to it.  In
// the emit pass CTA c writes at the offset of the selected scores of the segments before it,
// taking as many ties as the row still needs after theirs (ties go to the lowest indices).
namespace topk_detail {
__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}
}  // namespace topk_detail

constexpr int kTopkCluster = 4;

__global__ void __cluster_dims__(kTopkCluster, 1, 1) __launch_bounds__(kTopkThreads)
    topk_rows_cluster_kernel(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ row_len,
                             int32_t k, int32_t* __restrict__ idx) {
  constexpr int C = kTopkCluster;
  __shared__ uint32_t hist[kTopkWarps][256];
  __shared__ uint32_t total[2][256];   // this CTA's histogram of a pass (double-buffered: peers read it)
  __shared__ uint32_t gtotal[256];     // the row's histogram of the pass
  __shared__ int scan_scratch[kTopkWarps];
  __shared__ uint32_t s_bin, s_remaining, s_above;
  __shared__ uint32_t s_cnt[2];        // this CTA's scores above / equal to the threshold

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t rank = dev::cluster_ctarank();
  const int64_t r = blockIdx.x / C;
  const float* row = scores + r * ld;
  int32_t* out = idx + r * static_cast<int64_t>(k);
  int n = row_len[r];
  if (n < 0 || n > ld) {  // a row length outside [0, ld] is an input error; the row is clamped
    if (threadIdx.x == 0 && rank == 0) record_device_error(DSA_ERR_DEVICE_CHECK);
    n = n < 0 ? 0 : static_cast<int>(ld);
  }

  if (n <= k) {  // every candidate is selected (the same decision in every CTA of the row)
    if (rank == 0)
      for (int i = tid; i < k; i += kTopkThreads) out[i] = i < n ? i : -1;
    return;
  }
  const int per = ((n + C - 1) / C + 15) / 16 * 16;
  const int seg0 = min(n, static_cast<int>(rank) * per), seg1 = min(n, seg0 + per);

  uint32_t prefix = 0, mask = 0, remaining = static_cast<uint32_t>(k);
  if (tid == 0) s_above = 0u;  // this segment's scores known to be above the threshold
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < kTopkWarps * 256; i += kTopkThreads) (&hist[0][0])[i] = 0u;
    __syncthreads();
#pragma unroll 1
    for (int base = seg0; base < seg1; base += kTopkTile) {
      const int i0 = base + 16 * tid;
      if (i0 < seg1) {
        float f[16];
        topk_load16(row, i0, seg1, f);
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if (i0 + j < seg1) {
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
      total[pass & 1][tid] = s;
    }
    dev::cluster_sync();  // every CTA's histogram of this pass is complete
    if (tid < 256) {
      const uint32_t a = dev::smem_addr(&total[pass & 1][tid]);
      uint32_t s = 0;
#pragma unroll
      for (int c = 0; c < C; ++c) s += topk_detail::ld_cluster_u32(dev::map_to_rank(a, c));
      gtotal[tid] = s;
    }
    __syncthreads();
    if (warp == 0) {
      uint32_t c[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = gtotal[255 - (8 * lane + j)];
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
    const uint32_t bin = s_bin;
    // this segment's scores of this pass's prefix in bins above the chosen one are above the
    // threshold; in the last pass, those in the chosen bin are equal to it
    if (tid < 256 && static_cast<uint32_t>(tid) > bin) atomicAdd(&s_above, total[pass & 1][tid]);
    if (pass == 3 && tid == 0) s_cnt[1] = total[pass & 1][bin];
    prefix |= bin << shift;
    mask |= 255u << shift;
    remaining = s_remaining;
    __syncthreads();
  }
  if (tid == 0) s_cnt[0] = s_above;
  dev::cluster_sync();  // the segment counts are published
  // this CTA's output offset and tie quota from the segments before it
  const int need_eq = static_cast<int>(remaining);
  int offset = 0, ties_before = 0;
  for (int c = 0; c < static_cast<int>(rank); ++c) {
    const int g = static_cast<int>(topk_detail::ld_cluster_u32(dev::map_to_rank(dev::smem_addr(&s_cnt[0]), c)));
    const int e = static_cast<int>(topk_detail::ld_cluster_u32(dev::map_to_rank(dev::smem_addr(&s_cnt[1]), c)));
    offset += g + min(e, max(0, need_eq - ties_before));
    ties_before += e;
  }
  const int quota = max(0, need_eq - ties_before);  // ties this segment may still take
  const int my_total = static_cast<int>(s_cnt[0]) + min(static_cast<int>(s_cnt[1]), quota);

  const uint32_t thr = prefix;
  int eq_taken = 0, out_pos = offset;
#pragma unroll 1
  for (int base = seg0; base < seg1 && out_pos < offset + my_total; base += kTopkTile) {
    const int i0 = base + 16 * tid;
    uint32_t gbits = 0u, ebits = 0u;
    if (i0 < seg1) {
      float f[16];
      topk_load16(row, i0, seg1, f);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (i0 + j < seg1) {
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
        if (tie_rank < quota) sbits |= 1u << j;
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
  dev::cluster_sync();  // no CTA leaves while a peer may still read its shared memory
}

}  // namespace dsa
