// Row-wise top-k over fp32 index scores (fine-grained token selection: the k largest index
// scores of a query, ties to the lower key index, indices written ascending).
//
// Core: a 4-pass radix select over the order-preserving 32-bit keys of the scores (8 bits per
// pass, warp-private histograms merged over a cluster of CTAs through distributed shared
// memory) finds the key of the k-th largest entry and how many entries equal to it are still
// needed; an emit pass then walks the entries in index order and writes the selected indices
// with a block-wide scan, so the output is ascending and ties at the boundary go to the lowest
// indices.  The core reads its entries through a source (a segment of a score row in global
// memory, or candidates in shared memory) and is generic over the CTAs that share a row.
// dsa_topk runs it on a cluster of kTopkCluster CTAs per row.
//
// Decode selection (topk_decode_select_kernel): the paged indexer also writes, per 16 keys,
// the largest key of the group.  tau = the k-th largest group maximum is a lower bound of the
// row's k-th largest score: at least k groups have a maximum >= tau and each holds one score
// >= tau.  The row's scores >= tau (~2-3K of a 128K-key row) are gathered, in index order, into
// one CTA's shared memory, where the exact k-th largest is found and the selection emitted.
// A row whose candidates overflow that buffer takes the core over the row in global memory, in
// the same kernel (same result, slower).
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace dsa {

constexpr int kTopkThreads = 512;
constexpr int kTopkWarps = kTopkThreads / 32;
constexpr int kTopkVec = 4;                               // float4 loads per thread per step
constexpr int kTopkTile = 4 * kTopkVec * kTopkThreads;    // entries per step
constexpr int kTopkCluster = 4;

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

namespace topk_detail {

__device__ __forceinline__ uint32_t ld_cluster_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared::cluster.u32 %0, [%1];" : "=r"(v) : "r"(addr) : "memory");
  return v;
}

struct Shared {
  uint32_t hist[kTopkWarps][256];
  uint32_t total[2][256];   // this CTA's histogram of a pass (double-buffered: peers read it)
  uint32_t gtotal[256];     // the row's histogram of the pass
  int scan_scratch[kTopkWarps];
  uint32_t s_bin, s_remaining, s_above;
  uint32_t s_cnt[2];        // this CTA's entries above / equal to the threshold
};

// Entries [begin, end) of a score row in global memory; the index of entry i is i.
struct RowSource {
  const float* row;
  int begin, end;
  bool nan_check;  // report NaN scores (first pass only)
  __device__ __forceinline__ void load16(int i0, bool first_pass, uint32_t (&key)[16], int32_t (&idx)[16]) const {
    float f[16];
    topk_load16(row, i0, end, f);
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if (nan_check && first_pass && i0 + j < end && is_nan_bits(__float_as_uint(f[j])))
        record_device_error(DSA_ERR_DEVICE_CHECK);
      key[j] = order_key(f[j]);
      idx[j] = i0 + j;
    }
  }
};

// Candidates [0, end) held in shared memory as (order key, index), in index order.
struct CandSource {
  const uint32_t* key;
  const int32_t* idx;
  int begin, end;
  __device__ __forceinline__ void load16(int i0, bool, uint32_t (&k)[16], int32_t (&ix)[16]) const {
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      uint4 a = make_uint4(0u, 0u, 0u, 0u);
      int4 b = make_int4(0, 0, 0, 0);
      if (i0 + 4 * v < end) {  // the buffers are padded to a multiple of 16 entries
        a = *reinterpret_cast<const uint4*>(key + i0 + 4 * v);
        b = *reinterpret_cast<const int4*>(idx + i0 + 4 * v);
      }
      k[4 * v] = a.x; k[4 * v + 1] = a.y; k[4 * v + 2] = a.z; k[4 * v + 3] = a.w;
      ix[4 * v] = b.x; ix[4 * v + 1] = b.y; ix[4 * v + 2] = b.z; ix[4 * v + 3] = b.w;
    }
  }
};

// Barrier over the C CTAs that share a row (C = 1: the CTA alone).
template <int C>
__device__ __forceinline__ void row_sync() {
  if constexpr (C == 1) __syncthreads();
  else dev::cluster_sync();
}

// A shared-memory word of CTA c of the row's cluster (C = 1: this CTA's own).
template <int C>
__device__ __forceinline__ uint32_t row_ld(const uint32_t* local, int c) {
  if constexpr (C == 1) return *reinterpret_cast<const volatile uint32_t*>(local);
  else return ld_cluster_u32(dev::map_to_rank(dev::smem_addr(local), static_cast<uint32_t>(c)));
}

// The radix select and ordered emission over the C CTAs of a cluster (or one CTA, C = 1), each
// holding the entries [src.begin, src.end) of the row (CTA c's entries precede CTA c+1's in
// index order).  Every CTA of the cluster calls it with the same k; it ends with a barrier over
// the C CTAs, so no CTA leaves while a peer may still read its shared memory.
template <int C, class Src>
__device__ void radix_select_emit(const Src& src, int k, int32_t* __restrict__ out, Shared& sh) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t rank = C == 1 ? 0u : dev::cluster_ctarank();
  uint32_t prefix = 0, mask = 0, remaining = static_cast<uint32_t>(k);
  if (tid == 0) sh.s_above = 0u;  // this segment's entries known to be above the threshold
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < kTopkWarps * 256; i += kTopkThreads) (&sh.hist[0][0])[i] = 0u;
    __syncthreads();
#pragma unroll 1
    for (int base = src.begin; base < src.end; base += kTopkTile) {
      const int i0 = base + 16 * tid;
      if (i0 < src.end) {
        uint32_t key[16];
        int32_t ix[16];
        src.load16(i0, pass == 0, key, ix);
#pragma unroll
        for (int j = 0; j < 16; ++j)
          if (i0 + j < src.end && (key[j] & mask) == prefix) atomicAdd(&sh.hist[warp][(key[j] >> shift) & 255u], 1u);
      }
    }
    __syncthreads();
    if (tid < 256) {
      uint32_t s = 0;
#pragma unroll
      for (int w = 0; w < kTopkWarps; ++w) s += sh.hist[w][tid];
      sh.total[pass & 1][tid] = s;
    }
    row_sync<C>();  // every CTA's histogram of this pass is complete
    if (tid < 256) {
      uint32_t s = 0;
#pragma unroll
      for (int c = 0; c < C; ++c) s += row_ld<C>(&sh.total[pass & 1][tid], c);
      sh.gtotal[tid] = s;
    }
    __syncthreads();
    if (warp == 0) {
      uint32_t c[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = sh.gtotal[255 - (8 * lane + j)];
        sum += c[j];
      }
      const uint32_t inc = static_cast<uint32_t>(warp_inclusive_scan(static_cast<int>(sum)));
      const uint32_t before = inc - sum;
      if (before < remaining && remaining <= inc) {
        uint32_t acc = before;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (acc + c[j] >= remaining) {
            sh.s_bin = 255u - static_cast<uint32_t>(8 * lane + j);
            sh.s_remaining = remaining - acc;
            break;
          }
          acc += c[j];
        }
      }
    }
    __syncthreads();
    const uint32_t bin = sh.s_bin;
    // this segment's entries of this pass's prefix in bins above the chosen one are above the
    // threshold; in the last pass, those in the chosen bin are equal to it
    if (tid < 256 && static_cast<uint32_t>(tid) > bin) atomicAdd(&sh.s_above, sh.total[pass & 1][tid]);
    if (pass == 3 && tid == 0) sh.s_cnt[1] = sh.total[pass & 1][bin];
    prefix |= bin << shift;
    mask |= 255u << shift;
    remaining = sh.s_remaining;
    __syncthreads();
  }
  if (tid == 0) sh.s_cnt[0] = sh.s_above;
  row_sync<C>();  // the segment counts are published
  // this CTA's output offset and tie quota from the segments before it
  const int need_eq = static_cast<int>(remaining);
  int offset = 0, ties_before = 0;
  for (int c = 0; c < static_cast<int>(rank); ++c) {
    const int g = static_cast<int>(row_ld<C>(&sh.s_cnt[0], c));
    const int e = static_cast<int>(row_ld<C>(&sh.s_cnt[1], c));
    offset += g + min(e, max(0, need_eq - ties_before));
    ties_before += e;
  }
  const int quota = max(0, need_eq - ties_before);  // ties this segment may still take
  const int my_total = static_cast<int>(sh.s_cnt[0]) + min(static_cast<int>(sh.s_cnt[1]), quota);

  const uint32_t thr = prefix;
  int eq_taken = 0, out_pos = offset;
#pragma unroll 1
  for (int base = src.begin; base < src.end && out_pos < offset + my_total; base += kTopkTile) {
    const int i0 = base + 16 * tid;
    uint32_t gbits = 0u, ebits = 0u;
    int32_t ix[16];
    if (i0 < src.end) {
      uint32_t key[16];
      src.load16(i0, false, key, ix);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        if (i0 + j < src.end) {
          gbits |= static_cast<uint32_t>(key[j] > thr) << j;
          ebits |= static_cast<uint32_t>(key[j] == thr) << j;
        }
      }
    }
    int tie_total;
    int tie_rank = eq_taken + block_exclusive_scan<kTopkWarps>(__popc(ebits), sh.scan_scratch, tie_total);
    uint32_t sbits = gbits;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if ((ebits >> j) & 1u) {
        if (tie_rank < quota) sbits |= 1u << j;
        ++tie_rank;
      }
    }
    int sel_total;
    int pos = out_pos + block_exclusive_scan<kTopkWarps>(__popc(sbits), sh.scan_scratch, sel_total);
#pragma unroll
    for (int j = 0; j < 16; ++j)
      if ((sbits >> j) & 1u) out[pos++] = ix[j];
    eq_taken += tie_total;
    out_pos += sel_total;
  }
  row_sync<C>();  // no CTA leaves while a peer may still read its shared memory
}

// Row length check shared by the kernels: a length outside [0, cap] is an input error; the
// row is clamped.
__device__ __forceinline__ int checked_len(int n, int64_t cap, bool report) {
  if (n < 0 || n > cap) {
    if (report) record_device_error(DSA_ERR_DEVICE_CHECK);
    n = n < 0 ? 0 : static_cast<int>(cap);
  }
  return n;
}

}  // namespace topk_detail

// dsa_topk: one cluster per row over the scores in global memory.
__global__ void __cluster_dims__(kTopkCluster, 1, 1) __launch_bounds__(kTopkThreads)
    topk_rows_cluster_kernel(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ row_len,
                             int32_t k, int32_t* __restrict__ idx) {
  constexpr int C = kTopkCluster;
  __shared__ topk_detail::Shared sh;
  const int tid = threadIdx.x;
  const uint32_t rank = dev::cluster_ctarank();
  const int64_t r = blockIdx.x / C;
  int32_t* out = idx + r * static_cast<int64_t>(k);
  const int n = topk_detail::checked_len(row_len[r], ld, threadIdx.x == 0 && rank == 0);
  if (n <= k) {  // every candidate is selected (the same decision in every CTA of the row)
    if (rank == 0)
      for (int i = tid; i < k; i += kTopkThreads) out[i] = i < n ? i : -1;
    return;
  }
  const int per = ((n + C - 1) / C + 15) / 16 * 16;
  const int seg0 = min(n, static_cast<int>(rank) * per), seg1 = min(n, seg0 + per);
  topk_detail::radix_select_emit<C>(topk_detail::RowSource{scores + r * ld, seg0, seg1, true}, k, out, sh);
}

// ---- decode selection ------------------------------------------------------------------------
constexpr int kSelGroup = 16;       // scores per group maximum (written by the paged indexer)
constexpr int kSelCap = 8192;       // candidates of a row (key + index: 64 KB of shared memory)
constexpr int kSelBuckets = 4096;   // linear buckets over the group maxima's key range
constexpr int kSelCandBuckets = 2048;  // linear buckets over the candidates' key range
constexpr int kSelRankMax = 512;    // boundary-bucket members ranked directly (O(m^2))
constexpr int kSelDigit = 11;       // radix digit of the fallback select over the candidates
constexpr int kSelBatch = 8;        // 128-score steps a warp loads before using them
constexpr int kSelSmemBytes = kSelCap * 8;

namespace topk_detail {

__device__ __forceinline__ void st_cluster_u32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr), "r"(v) : "memory");
}

// The float whose order key is `key` (the inverse of order_key on its image); for a key whose
// inverse would be a NaN pattern, the infinity on its side, so that !(f < result) holds for
// every score f with order_key(f) >= key (a superset of them, never fewer).
__device__ __forceinline__ float key_floor_float(uint32_t key) {
  if (key > 0xFF800000u) return INFINITY;   // above order_key(+inf): positive NaN patterns
  if (key < 0x007FFFFFu) return -INFINITY;  // below order_key(-inf): negative NaN patterns
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// Block-wide reductions of one uint32 per thread (every thread receives the result).
template <class Op>
__device__ __forceinline__ uint32_t block_reduce_u32(uint32_t v, uint32_t* scratch, Op op) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) v = op(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();  // scratch is free
  if (lane == 0) scratch[warp] = v;
  __syncthreads();
  v = scratch[0];
#pragma unroll
  for (int w = 1; w < kTopkWarps; ++w) v = op(v, scratch[w]);
  return v;
}
struct MinOp { __device__ uint32_t operator()(uint32_t a, uint32_t b) const { return min(a, b); } };
struct MaxOp { __device__ uint32_t operator()(uint32_t a, uint32_t b) const { return max(a, b); } };
struct AndOp { __device__ uint32_t operator()(uint32_t a, uint32_t b) const { return a & b; } };
struct OrOp { __device__ uint32_t operator()(uint32_t a, uint32_t b) const { return a | b; } };

// Finds, counting from the top bin of hist[0..kBins), the bin where the count reaches `want`;
// returns it and sets `above` to the count in the bins above it.  Every thread calls it.
template <int kBins>
__device__ __forceinline__ int find_bin_from_top(const uint32_t* hist, uint32_t want, uint32_t& above, Shared& sh) {
  constexpr int BPT = kBins / kTopkThreads;
  const int tid = threadIdx.x;
  uint32_t c[BPT], sum = 0;
#pragma unroll
  for (int j = 0; j < BPT; ++j) {
    c[j] = hist[kBins - 1 - (BPT * tid + j)];
    sum += c[j];
  }
  int tot;
  const uint32_t before =
      static_cast<uint32_t>(block_exclusive_scan<kTopkWarps>(static_cast<int>(sum), sh.scan_scratch, tot));
  if (before < want && want <= before + sum) {
    uint32_t acc = before;
#pragma unroll
    for (int j = 0; j < BPT; ++j) {
      if (acc + c[j] >= want) {
        sh.s_bin = static_cast<uint32_t>(kBins - 1 - (BPT * tid + j));
        sh.s_above = acc;
        break;
      }
      acc += c[j];
    }
  }
  __syncthreads();
  const int bin = static_cast<int>(sh.s_bin);
  above = sh.s_above;
  __syncthreads();
  return bin;
}

// tau <= the k-th largest of the G group maxima gm[0..G) (G >= k).  The maxima's key range
// [lo, hi] is mapped linearly onto kSelBuckets buckets (any monotone map keeps the order; a
// linear one spreads the maxima, which crowd a few exponent bins, over many buckets); tau is
// the lower edge of the bucket below the one holding the k-th largest, so float rounding of
// the map cannot put tau above it.  Every thread of the CTA calls it; `hist` holds
// kSelBuckets counters.
__device__ uint32_t group_max_bound(const uint32_t* __restrict__ gm, int G, int k, uint32_t* hist, Shared& sh) {
  constexpr int V = 4;  // 16-byte loads per thread per step, all issued before the first use
  const int tid = threadIdx.x;
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
  // every load of a step is issued before any is used; a row of up to 8192 maxima (128K keys)
  // is one step, held in registers for both uses below
  uint32_t vv[4 * V];
  auto load_step = [&](int base) {
#pragma unroll
    for (int v = 0; v < V; ++v) {
      const int i = base + 4 * (v * kTopkThreads + tid);
      uint4 x = make_uint4(0u, 0u, 0u, 0u);
      if (i + 3 < G) {
        x = *reinterpret_cast<const uint4*>(gm + i);
      } else if (i < G) {
        x.x = gm[i];
        if (i + 1 < G) x.y = gm[i + 1];
        if (i + 2 < G) x.z = gm[i + 2];
      }
      vv[4 * v] = x.x;
      vv[4 * v + 1] = x.y;
      vv[4 * v + 2] = x.z;
      vv[4 * v + 3] = x.w;
    }
  };
  auto valid = [&](int base, int v, int j) { return base + 4 * (v * kTopkThreads + tid) + j < G; };
  constexpr int STEP = 4 * V * kTopkThreads;
#pragma unroll 1
  for (int base = 0; base < G; base += STEP) {
    load_step(base);
#pragma unroll
    for (int v = 0; v < V; ++v)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (valid(base, v, j)) {
          lo = min(lo, vv[4 * v + j]);
          hi = max(hi, vv[4 * v + j]);
        }
  }
  lo = block_reduce_u32(lo, reinterpret_cast<uint32_t*>(sh.scan_scratch), MinOp{});
  hi = block_reduce_u32(hi, reinterpret_cast<uint32_t*>(sh.scan_scratch), MaxOp{});
  if (hi == lo) return lo;  // every maximum is equal: all G >= k groups reach it
  const float inv = static_cast<float>(kSelBuckets) / (static_cast<float>(hi - lo) + 1.f);
  for (int i = tid; i < kSelBuckets; i += kTopkThreads) hist[i] = 0u;
  __syncthreads();
#pragma unroll 1
  for (int base = 0; base < G; base += STEP) {
    if (G > STEP) load_step(base);  // one step: the maxima are still in registers
#pragma unroll
    for (int v = 0; v < V; ++v)
#pragma unroll
      for (int j = 0; j < 4; ++j)
        if (valid(base, v, j)) {
          const int b = static_cast<int>(static_cast<float>(vv[4 * v + j] - lo) * inv);
          atomicAdd(&hist[b < kSelBuckets ? b : kSelBuckets - 1], 1u);
        }
  }
  __syncthreads();
  uint32_t above;
  const int b = find_bin_from_top<kSelBuckets>(hist, static_cast<uint32_t>(k), above, sh);
  const float edge = static_cast<float>(b - 1) / inv;  // one bucket of margin for the rounding
  return edge <= 0.f ? lo : lo + static_cast<uint32_t>(edge);
}

}  // namespace topk_detail

namespace topk_detail {

// The k-th largest of the n >= k candidate keys (thr) and how many keys equal to it are taken
// (quota), by radix passes of kSelDigit bits below the keys' common prefix.  The fallback of
// cand_threshold (many keys in its boundary bucket).
__device__ void cand_threshold_radix(const uint32_t* __restrict__ key, int n, int k, uint32_t* hist, Shared& sh,
                                     uint32_t& thr, int& quota) {
  constexpr int kBins = 1 << kSelDigit;
  const int tid = threadIdx.x;
  uint32_t a = 0xFFFFFFFFu, o = 0u;
  for (int i = tid; i < n; i += kTopkThreads) {
    a &= key[i];
    o |= key[i];
  }
  a = block_reduce_u32(a, reinterpret_cast<uint32_t*>(sh.scan_scratch), AndOp{});
  o = block_reduce_u32(o, reinterpret_cast<uint32_t*>(sh.scan_scratch), OrOp{});
  const int common = (a ^ o) == 0u ? 32 : __clz(a ^ o);  // leading bits every key shares
  uint32_t mask = common == 0 ? 0u : (0xFFFFFFFFu << (32 - common));
  uint32_t prefix = a & mask;
  uint32_t rem = static_cast<uint32_t>(k);
  int pos = 32 - common;
#pragma unroll 1
  while (pos > 0) {
    const int d = pos < kSelDigit ? pos : kSelDigit;
    const int shift = pos - d;
    const uint32_t dmask = (1u << d) - 1u;
    for (int i = tid; i < kBins; i += kTopkThreads) hist[i] = 0u;
    __syncthreads();
    for (int i = tid; i < n; i += kTopkThreads) {
      const uint32_t kk = key[i];
      if ((kk & mask) == prefix) atomicAdd(&hist[(kk >> shift) & dmask], 1u);
    }
    __syncthreads();
    uint32_t above;
    const uint32_t bin = static_cast<uint32_t>(find_bin_from_top<kBins>(hist, rem, above, sh));
    prefix |= bin << shift;
    mask |= dmask << shift;
    rem -= above;
    pos = shift;
  }
  thr = prefix;
  quota = static_cast<int>(rem);
}

// thr and quota as above.  The candidates' key range [lo, hi] is mapped linearly onto
// kSelCandBuckets buckets (monotone, so a higher bucket never holds a smaller key); the bucket
// where the count from the top reaches k usually holds a handful of keys, whose ranks are then
// counted directly.  Every thread of the CTA calls it; `hist` holds 2 * kSelCandBuckets words.
__device__ void cand_threshold(const uint32_t* __restrict__ key, int n, int k, uint32_t* hist, Shared& sh,
                               uint32_t& thr, int& quota) {
  const int tid = threadIdx.x;
  uint32_t lo = 0xFFFFFFFFu, hi = 0u;
  for (int i = tid; i < n; i += kTopkThreads) {
    lo = min(lo, key[i]);
    hi = max(hi, key[i]);
  }
  lo = block_reduce_u32(lo, reinterpret_cast<uint32_t*>(sh.scan_scratch), MinOp{});
  hi = block_reduce_u32(hi, reinterpret_cast<uint32_t*>(sh.scan_scratch), MaxOp{});
  if (hi == lo) {  // every key is equal
    thr = lo;
    quota = k;
    return;
  }
  const float inv = static_cast<float>(kSelCandBuckets) / (static_cast<float>(hi - lo) + 1.f);
  auto bucket = [&](uint32_t kk) {
    const int b = static_cast<int>(static_cast<float>(kk - lo) * inv);
    return b < kSelCandBuckets ? b : kSelCandBuckets - 1;
  };
  for (int i = tid; i < kSelCandBuckets; i += kTopkThreads) hist[i] = 0u;
  if (tid == 0) sh.s_cnt[0] = 0u;
  __syncthreads();
  for (int i = tid; i < n; i += kTopkThreads) atomicAdd(&hist[bucket(key[i])], 1u);
  __syncthreads();
  uint32_t above;
  const int bstar = find_bin_from_top<kSelCandBuckets>(hist, static_cast<uint32_t>(k), above, sh);
  const int m = static_cast<int>(hist[bstar]);
  const int rem = k - static_cast<int>(above);  // 1 <= rem <= m keys still needed from bucket bstar
  if (m > kSelRankMax) {  // a crowded boundary bucket (ties, or a narrow spike of keys)
    cand_threshold_radix(key, n, k, hist, sh, thr, quota);
    return;
  }
  uint32_t* members = hist + kSelCandBuckets;
  for (int i = tid; i < n; i += kTopkThreads) {
    const uint32_t kk = key[i];
    if (bucket(kk) == bstar) members[atomicAdd(&sh.s_cnt[0], 1u)] = kk;
  }
  __syncthreads();
  // the member whose rank (keys above it) is below rem and whose rank plus its equal keys reaches rem
  for (int i = tid; i < m; i += kTopkThreads) {
    const uint32_t kk = members[i];
    int g = 0, e = 0;
    for (int j = 0; j < m; ++j) {
      g += members[j] > kk ? 1 : 0;
      e += members[j] == kk ? 1 : 0;
    }
    if (g < rem && rem <= g + e) {  // every thread that gets here writes the same values
      sh.s_bin = kk;
      sh.s_remaining = static_cast<uint32_t>(rem - g);
    }
  }
  __syncthreads();
  thr = sh.s_bin;
  quota = static_cast<int>(sh.s_remaining);
  __syncthreads();
}

// Exact top-k of the n candidates (order key, index) that this CTA holds in index order,
// written ascending to out[0..k) (n >= k): keys above the k-th largest, and the first quota of
// the keys equal to it (the lowest indices).  Every thread of the CTA calls it.
__device__ void cand_select_emit(const uint32_t* __restrict__ key, const int32_t* __restrict__ idx, int n, int k,
                                 int32_t* __restrict__ out, uint32_t* hist, Shared& sh) {
  const int tid = threadIdx.x;
  uint32_t thr;
  int quota;
  cand_threshold(key, n, k, hist, sh, thr, quota);
  int eq_taken = 0, out_pos = 0;
#pragma unroll 1
  for (int base = 0; base < n; base += 4 * kTopkThreads) {
    const int i0 = base + 4 * tid;
    uint32_t gbits = 0u, ebits = 0u;
    int32_t ix[4] = {0, 0, 0, 0};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (i0 + j < n) {
        const uint32_t kk = key[i0 + j];
        ix[j] = idx[i0 + j];
        gbits |= static_cast<uint32_t>(kk > thr) << j;
        ebits |= static_cast<uint32_t>(kk == thr) << j;
      }
    }
    int tie_total;
    int tie_rank = eq_taken + block_exclusive_scan<kTopkWarps>(__popc(ebits), sh.scan_scratch, tie_total);
    uint32_t sbits = gbits;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if ((ebits >> j) & 1u) {
        if (tie_rank < quota) sbits |= 1u << j;
        ++tie_rank;
      }
    }
    int sel_total;
    int p = out_pos + block_exclusive_scan<kTopkWarps>(__popc(sbits), sh.scan_scratch, sel_total);
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if ((sbits >> j) & 1u) out[p++] = ix[j];
    eq_taken += tie_total;
    out_pos += sel_total;
  }
}

}  // namespace topk_detail

// Per-sequence selection after the paged indexer: scores [B, ld] (entries [0, n_b)), gmax
// [B, ld16] (order key of the largest score of entries [16 g, 16 g + 16) of the row), n_b =
// min(context_lens[b], max_len).  One cluster of kTopkCluster CTAs per row:
//   1. every CTA computes tau from the row's group maxima (the same value in each);
//   2. every CTA splits its quarter of the row into 16 warp slices and counts, with coalesced
//      16-byte loads, the scores >= tau of each slice;
//   3. the CTAs exchange their counts; unless the row's candidates exceed kSelCap, every warp
//      reads its slice again and writes its candidates, in index order, straight into CTA 0's
//      buffer at its offset (distributed shared memory), and CTA 0 alone selects and emits.
// With more than kSelCap candidates the cluster runs the full radix select over the row.
__global__ void __cluster_dims__(kTopkCluster, 1, 1) __launch_bounds__(kTopkThreads, 2)
    topk_decode_select_kernel(const float* __restrict__ scores, int64_t ld, const uint32_t* __restrict__ gmax,
                              int64_t ld16, const int32_t* __restrict__ context_lens, int32_t max_len, int32_t k,
                              int32_t* __restrict__ idx) {
  constexpr int C = kTopkCluster;
  extern __shared__ uint8_t sel_smem[];
  uint32_t* cand_key = reinterpret_cast<uint32_t*>(sel_smem);
  int32_t* cand_idx = reinterpret_cast<int32_t*>(cand_key + kSelCap);
  __shared__ topk_detail::Shared sh;
  __shared__ uint32_t s_count;
  __shared__ int s_wcount[kTopkWarps];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t rank = dev::cluster_ctarank();
  const int64_t r = blockIdx.x / C;
  int32_t* out = idx + r * static_cast<int64_t>(k);
  // the indexer reports a context longer than max_len; here it is clamped the same way
  const int n = topk_detail::checked_len(min(context_lens[r], max_len), ld, threadIdx.x == 0 && rank == 0);
  if (n <= k) {
    if (rank == 0)
      for (int i = tid; i < k; i += kTopkThreads) out[i] = i < n ? i : -1;
    return;
  }
  const float* row = scores + r * ld;
  const int G = (n + kSelGroup - 1) / kSelGroup;
  // 1. with fewer groups than k the maxima bound nothing: every score is a candidate
  const uint32_t tau = G >= k ? topk_detail::group_max_bound(gmax + r * ld16, G, k, &sh.hist[0][0], sh) : 0u;

  // 2. this CTA's segment, in 16 warp slices of whole 128-score steps (a float4 per lane)
  const int per = ((n + C - 1) / C + 15) / 16 * 16;
  const int seg0 = min(n, static_cast<int>(rank) * per), seg1 = min(n, seg0 + per);
  const int wlen = ((seg1 - seg0 + kTopkWarps - 1) / kTopkWarps + 127) / 128 * 128;
  const int w0 = min(seg1, seg0 + warp * wlen), w1 = min(seg1, w0 + wlen);
  // a warp reads its slice in batches of kSelBatch 128-score steps, every load of a batch
  // issued before the first is used (coalesced: a step is 512 contiguous bytes).  A score is a
  // candidate when !(score < tf), tf the float whose order key is tau: one compare per score,
  // the same set as order_key(score) >= tau for every non-NaN score, and a NaN score is always
  // a candidate (it is reported when the candidates are written).
  const float tf = topk_detail::key_floor_float(tau);
  int wcount = 0;
#pragma unroll 1
  for (int b0 = w0; b0 < w1; b0 += 128 * kSelBatch) {
    float4 x[kSelBatch];
#pragma unroll
    for (int m = 0; m < kSelBatch; ++m) {
      const int i = b0 + 128 * m + 4 * lane;
      x[m] = i < w1 ? *reinterpret_cast<const float4*>(row + i) : make_float4(0.f, 0.f, 0.f, 0.f);  // ld >= n, ld % 4 == 0
    }
#pragma unroll
    for (int m = 0; m < kSelBatch; ++m) {
      const int lim = w1 - (b0 + 128 * m + 4 * lane);  // scores of this float4 inside the slice
      if (lim >= 4) {
        wcount += (x[m].x < tf ? 0 : 1) + (x[m].y < tf ? 0 : 1) + (x[m].z < tf ? 0 : 1) + (x[m].w < tf ? 0 : 1);
      } else if (lim > 0) {
        const float f[4] = {x[m].x, x[m].y, x[m].z, x[m].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) wcount += (j < lim && !(f[j] < tf)) ? 1 : 0;
      }
    }
  }
  wcount = __reduce_add_sync(0xffffffffu, wcount);
  if (lane == 0) s_wcount[warp] = wcount;
  __syncthreads();
  int woff = 0, ccount = 0;
#pragma unroll
  for (int w = 0; w < kTopkWarps; ++w) {
    woff += w < warp ? s_wcount[w] : 0;
    ccount += s_wcount[w];
  }
  if (tid == 0) s_count = static_cast<uint32_t>(ccount);
  dev::cluster_sync();  // 3. the counts are published
  int total = 0, offset = 0;
  for (int c = 0; c < C; ++c) {
    const int cc = static_cast<int>(topk_detail::ld_cluster_u32(dev::map_to_rank(dev::smem_addr(&s_count), c)));
    if (c < static_cast<int>(rank)) offset += cc;
    total += cc;
  }
  if (total > kSelCap || total < k) {
    // too many candidates for one buffer (e.g. a tie class of thousands at the boundary):
    // the exact select over the row in global memory, on the whole cluster
    topk_detail::radix_select_emit<C>(topk_detail::RowSource{row, seg0, seg1, true}, k, out, sh);
    return;
  }
  {  // this warp's candidates, in index order, into CTA 0's buffer at offset + woff
    const uint32_t kdst = dev::map_to_rank(dev::smem_addr(cand_key), 0u);
    const uint32_t idst = dev::map_to_rank(dev::smem_addr(cand_idx), 0u);
    uint32_t at = static_cast<uint32_t>(offset + woff);
#pragma unroll 1
    for (int b0 = w0; b0 < w1; b0 += 128 * kSelBatch) {  // warp-uniform
      float4 x[kSelBatch];
#pragma unroll
      for (int m = 0; m < kSelBatch; ++m) {
        const int i = b0 + 128 * m + 4 * lane;
        x[m] = i < w1 ? *reinterpret_cast<const float4*>(row + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
#pragma unroll
      for (int m = 0; m < kSelBatch; ++m) {
        const int i = b0 + 128 * m + 4 * lane;
        const float f[4] = {x[m].x, x[m].y, x[m].z, x[m].w};
        const int lim = w1 - i;
        uint32_t keep = 0u;
#pragma unroll
        for (int j = 0; j < 4; ++j) keep |= static_cast<uint32_t>(j < lim && !(f[j] < tf)) << j;
        const int cnt = __popc(keep);
        const int incl = warp_inclusive_scan(cnt);
        uint32_t p = at + static_cast<uint32_t>(incl - cnt);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          if ((keep >> j) & 1u) {
            if (is_nan_bits(__float_as_uint(f[j]))) record_device_error(DSA_ERR_DEVICE_CHECK);
            topk_detail::st_cluster_u32(kdst + 4u * p, order_key(f[j]));
            topk_detail::st_cluster_u32(idst + 4u * p, static_cast<uint32_t>(i + j));
            ++p;
          }
        }
        at += static_cast<uint32_t>(__shfl_sync(0xffffffffu, incl, 31));
      }
    }
  }
  dev::cluster_sync();  // CTA 0 holds the row's candidates; the others are done
  if (rank != 0) return;
  topk_detail::cand_select_emit(cand_key, cand_idx, total, k, out, &sh.hist[0][0], sh);
}

}  // namespace dsa
