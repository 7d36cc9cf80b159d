// Lightning indexer on the 5th-generation tensor cores, with the selection fused in.
//
// I[t,s] = k_scale[s] * sum_j (w[t,j] * q_scale[t]) * ReLU(sum_d q8[t,j,d] * k8[s,d])
//
// The e4m3 x e4m3 products run as one tcgen05.mma (kind::f8f6f4, fp32 accumulate in TMEM)
// per 32-deep K slice with
//   M = 128 keys (A operand: a key tile, TMA-loaded, 128-byte swizzle, K-major),
//   N = TOK * H_I  (B operand: the indexer queries of TOK tokens x H_I heads, resident in SMEM).
// Keys on M put one key on each TMEM lane, so the epilogue thread that owns a lane reduces
// over heads in registers: ReLU, the per-head weight (w * q_scale), the head sum, k_scale and
// the causal mask all happen in the epilogue, straight out of TMEM.
//
// Warp roles (192 threads): warps 0-3 epilogue (thread e owns TMEM lane e = key e of the
// tile), warp 4 lane 0 TMA producer, warp 5 lane 0 MMA issuer (warp 5 also owns TMEM).
// Key tiles flow through a STAGES-deep SMEM ring; the accumulator is double-buffered in TMEM
// so the epilogue of tile i overlaps the MMA of tile i+1.
//
// Modes:
//   kIdxScores  write fp32 scores of the CTA's query rows to HBM (-inf beyond the causal
//               prefix), for dsa_indexer_scores (prefill rows or decode key ranges);
//   kIdxTopk    keep, per query token, a streaming candidate set in SMEM: a score enters
//               only if its key beats the running threshold; when the set is about to
//               overflow it is cut back to exactly k by a radix select (ties to the lower
//               index), which raises the threshold.  At the end the set is cut to
//               min(k, t+1) and written ascending through a bitmap.  No score leaves the SM.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace dsa {

enum { kIdxScores = 0, kIdxTopk = 1 };

struct IndexerParams {
  const float* q_scale;       // [rows]
  const float* w;             // [rows, H_I]
  const float* k_scale;       // contiguous [T] | paged [num_blocks * 64]
  const int32_t* cu_seqlens;  // prefill [B+1]
  const int32_t* block_table; // decode [B, max_blocks_per_seq]
  const int32_t* context_lens;// decode [B]
  int32_t max_blocks_per_seq;
  int32_t tiles_per_cta;      // decode: key tiles per CTA
  float* scores;              // kIdxScores output
  int64_t ld;
  int64_t row_begin, row_end;
  int32_t* idx_out;           // kIdxTopk output [T, k]
  int32_t k;
  int32_t cap;                // candidate capacity per token (kIdxTopk)
};

namespace idx_detail {

__device__ __forceinline__ void epi_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// Barrier over the 128 epilogue threads that also ORs a predicate across them, so that a
// decision to leave a loop is the same in every thread (a named barrier cannot time out).
__device__ __forceinline__ bool epi_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, 1, 128, q;\n\tselp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}

// Exclusive scan over the 128 epilogue threads (4 warps); `scratch` holds 4 ints.
__device__ __forceinline__ int epi_scan(int v, int* scratch, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int inc = warp_inclusive_scan(v);
  if (lane == 31) scratch[warp] = inc;
  epi_sync();
  const int w0 = scratch[0], w1 = scratch[1], w2 = scratch[2], w3 = scratch[3];
  total = w0 + w1 + w2 + w3;
  const int wprefix = (warp > 0 ? w0 : 0) + (warp > 1 ? w1 : 0) + (warp > 2 ? w2 : 0);
  epi_sync();
  return wprefix + inc - v;
}

// 16-byte shared-memory load that the compiler may not hoist out of the tile loop (the
// per-head weights of all TOK tokens would not fit in registers).
__device__ __forceinline__ float4 lds128(const float* p) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(dev::smem_addr(p)));
  return v;
}

struct SelectScratch {
  uint32_t hist[256];
  int scan[4];
  uint32_t bin, rem;
};

// Among n candidate (key, idx) pairs, keep exactly the m best (key descending, idx
// ascending) and compact them to the front.  Returns the key of the m-th best.
// Called by the 128 epilogue threads together; requires 1 <= m < n.
__device__ uint32_t select_compact(uint32_t* ck, int32_t* ci, int n, int m, SelectScratch& S) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // --- radix select on the key (descending) ---
  uint32_t prefix = 0, mask = 0, remaining = static_cast<uint32_t>(m);
#pragma unroll 1
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    S.hist[tid] = 0u;
    S.hist[tid + 128] = 0u;
    epi_sync();
    for (int e = tid; e < n; e += 128) {
      const uint32_t key = ck[e];
      if ((key & mask) == prefix) atomicAdd(&S.hist[(key >> shift) & 255u], 1u);
    }
    epi_sync();
    if (warp == 0) {
      uint32_t c[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = S.hist[255 - (8 * lane + j)];
        sum += c[j];
      }
      const uint32_t inc = static_cast<uint32_t>(warp_inclusive_scan(static_cast<int>(sum)));
      const uint32_t before = inc - sum;
      if (before < remaining && remaining <= inc) {
        uint32_t acc = before;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (acc + c[j] >= remaining) {
            S.bin = 255u - static_cast<uint32_t>(8 * lane + j);
            S.rem = remaining - acc;
            break;
          }
          acc += c[j];
        }
      }
    }
    epi_sync();
    prefix |= S.bin << shift;
    mask |= 255u << shift;
    remaining = S.rem;
  }
  const uint32_t kth = prefix;
  const uint32_t need_eq = remaining;
  // --- among keys equal to kth, the need_eq smallest indices (idx < 2^24) ---
  uint32_t iprefix = 0, imask = 0, irem = need_eq;
#pragma unroll 1
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = 16 - 8 * pass;
    S.hist[tid] = 0u;
    S.hist[tid + 128] = 0u;
    epi_sync();
    for (int e = tid; e < n; e += 128) {
      const uint32_t id = static_cast<uint32_t>(ci[e]);
      if (ck[e] == kth && (id & imask) == iprefix) atomicAdd(&S.hist[(id >> shift) & 255u], 1u);
    }
    epi_sync();
    if (warp == 0) {
      uint32_t c[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = S.hist[8 * lane + j];
        sum += c[j];
      }
      const uint32_t inc = static_cast<uint32_t>(warp_inclusive_scan(static_cast<int>(sum)));
      const uint32_t before = inc - sum;
      if (before < irem && irem <= inc) {
        uint32_t acc = before;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (acc + c[j] >= irem) {
            S.bin = static_cast<uint32_t>(8 * lane + j);
            S.rem = irem - acc;
            break;
          }
          acc += c[j];
        }
      }
    }
    epi_sync();
    iprefix |= S.bin << shift;
    imask |= 255u << shift;
    irem = S.rem;
  }
  const uint32_t idx_thr = iprefix;  // the need_eq-th smallest index among the ties
  // --- in-place compaction, one chunk of 128 entries at a time ---
  int base = 0;
#pragma unroll 1
  for (int c0 = 0; c0 < n; c0 += 128) {
    const int e = c0 + tid;
    uint32_t key = 0;
    int32_t id = 0;
    bool keep = false;
    if (e < n) {
      key = ck[e];
      id = ci[e];
      keep = key > kth || (key == kth && static_cast<uint32_t>(id) <= idx_thr);
    }
    int total;
    const int pos = base + epi_scan(keep ? 1 : 0, S.scan, total);
    if (keep) {
      ck[pos] = key;
      ci[pos] = id;
    }
    base += total;
  }
  epi_sync();
  return kth;
}

}  // namespace idx_detail

template <int D_I>
struct IdxLayout {
  static constexpr uint32_t kSwizzle = D_I == 128 ? dev::kSwizzle128B : dev::kSwizzle64B;
  static constexpr uint32_t kSBO = D_I == 128 ? 1024u : 512u;  // bytes between 8-row groups
  static constexpr int kKeyTileBytes = 128 * D_I;
};

// Shared-memory bytes the kernel needs (besides the 1 KB alignment slack).
template <int D_I, int H_I, int TOK, int MODE, int STAGES>
__host__ __device__ constexpr int indexer_smem_bytes(int cap) {
  return ((TOK * H_I * D_I + 1023) / 1024) * 1024 + STAGES * IdxLayout<D_I>::kKeyTileBytes + TOK * H_I * 4 +
         (MODE == kIdxTopk ? TOK * cap * 8 : 0);
}

template <int D_I, int H_I, int TOK, int MODE, bool PAGED, int STAGES>
__global__ void __launch_bounds__(192, 1)
    indexer_kernel(const __grid_constant__ CUtensorMap q_map, const __grid_constant__ CUtensorMap k_map,
                   const IndexerParams p) {
  using namespace dev;
  using L = IdxLayout<D_I>;
  constexpr int N = TOK * H_I;
  constexpr int Q_BYTES = N * D_I;
  constexpr int TMEM_COLS = (2 * N < 32) ? 32 : 2 * N;
  constexpr uint32_t IDESC = idesc_e4m3(128, N);
  static_assert(N % 16 == 0 && N <= 256, "MMA N must be a multiple of 16 in [16, 256]");

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem;
  uint8_t* sK = smem + ((Q_BYTES + 1023) / 1024) * 1024;
  float* sWq = reinterpret_cast<float*>(sK + STAGES * L::kKeyTileBytes);
  uint32_t* sCandKey = reinterpret_cast<uint32_t*>(sWq + N);
  int32_t* sCandIdx = reinterpret_cast<int32_t*>(sCandKey + (MODE == kIdxTopk ? TOK * p.cap : 0));

  __shared__ uint64_t bar_kfull[STAGES], bar_kempty[STAGES], bar_accfull[2], bar_accempty[2], bar_q;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ int s_cnt[TOK];
  __shared__ long long s_thr[TOK];
  __shared__ idx_detail::SelectScratch s_sel;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---------------- work item ----------------
  int b = blockIdx.y;
  int64_t key_row0;   // global row of local key 0 (contiguous keys)
  int t0, ntok, tile0, ntiles, len;
  int64_t q_row;      // row of the Q tile in the [rows * H_I, D_I] view
  if constexpr (!PAGED) {
    const int seq_start = p.cu_seqlens[b];
    len = p.cu_seqlens[b + 1] - seq_start;
    const int nblk = (len + TOK - 1) / TOK;
    const int tb = static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x);  // heavy blocks first
    if (tb >= nblk) return;
    t0 = tb * TOK;
    ntok = min(TOK, len - t0);
    if (MODE == kIdxScores) {
      const int64_t g0 = seq_start + t0, g1 = g0 + ntok;
      if (g1 <= p.row_begin || g0 >= p.row_end) return;
    }
    tile0 = 0;
    ntiles = (t0 + ntok - 1) / 128 + 1;
    key_row0 = seq_start;
    q_row = static_cast<int64_t>(seq_start + t0) * H_I;
  } else {
    if (b < p.row_begin || b >= p.row_end) return;
    len = min(p.context_lens[b], p.max_blocks_per_seq * 64);  // never read past the block table row
    tile0 = static_cast<int>(blockIdx.x) * p.tiles_per_cta;
    const int total_tiles = (len + 127) / 128;
    if (tile0 >= total_tiles) return;
    ntiles = min(p.tiles_per_cta, total_tiles - tile0);
    t0 = len - 1;  // the decode query sits at position ctx-1
    ntok = 1;
    key_row0 = 0;
    q_row = static_cast<int64_t>(b) * H_I;
  }

  // ---------------- setup ----------------
  if (tid == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&bar_kfull[i], 1);
      mbar_init(&bar_kempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_accfull[i], 1);
      mbar_init(&bar_accempty[i], 4);
    }
    mbar_init(&bar_q, 1);
    s_abort = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&s_tmem, TMEM_COLS);
    tmem_relinquish();
  }
  for (int i = tid; i < N; i += blockDim.x) {
    const int tt = i / H_I, j = i % H_I;
    float v = 0.f;
    if (tt < ntok) {
      const int64_t row = PAGED ? b : (p.cu_seqlens[b] + t0 + tt);
      v = p.w[row * H_I + j] * p.q_scale[row];
    }
    sWq[i] = v;
  }
  if (MODE == kIdxTopk && tid < TOK) {
    s_cnt[tid] = 0;
    s_thr[tid] = -1;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp == 4) {
    // ================= TMA producer =================
    if (lane == 0) {
      tma_prefetch_desc(&q_map);
      tma_prefetch_desc(&k_map);
      mbar_arrive_expect_tx(&bar_q, Q_BYTES);
      tma_load_2d(sQ, &q_map, &bar_q, 0, static_cast<int32_t>(q_row));
      const int nblocks_seq = PAGED ? (len + 63) / 64 : 0;
#pragma unroll 1
      for (int it = 0; it < ntiles; ++it) {
        const int stage = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        if (!mbar_wait(&bar_kempty[stage], ph ^ 1)) {
          record_device_error(DSA_ERR_TIMEOUT);
          s_abort = 1;
          break;
        }
        if (s_abort) break;
        mbar_arrive_expect_tx(&bar_kfull[stage], L::kKeyTileBytes);
        uint8_t* dst = sK + stage * L::kKeyTileBytes;
        if constexpr (!PAGED) {
          tma_load_2d(dst, &k_map, &bar_kfull[stage], 0, static_cast<int32_t>(key_row0 + (tile0 + it) * 128));
        } else {
          const int32_t* bt = p.block_table + static_cast<int64_t>(b) * p.max_blocks_per_seq;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const int lb = (tile0 + it) * 2 + h;
            const int phys = bt[lb < nblocks_seq ? lb : 0];
            tma_load_2d(dst + h * 64 * D_I, &k_map, &bar_kfull[stage], 0, phys * 64);
          }
        }
      }
    }
  } else if (warp == 5) {
    // ================= MMA issuer =================
    if (lane == 0) {
      bool ok = mbar_wait(&bar_q, 0);
      if (!ok) {
        record_device_error(DSA_ERR_TIMEOUT);
        s_abort = 1;
      }
#pragma unroll 1
      for (int it = 0; ok && it < ntiles; ++it) {
        const int stage = it % STAGES;
        const uint32_t ph = (it / STAGES) & 1;
        const int acc = it & 1;
        const uint32_t aph = (it >> 1) & 1;
        if (!mbar_wait(&bar_kfull[stage], ph) || !mbar_wait(&bar_accempty[acc], aph ^ 1)) {
          record_device_error(DSA_ERR_TIMEOUT);
          s_abort = 1;
          break;
        }
        if (s_abort) break;
        tc_fence_after();
        const uint32_t d = tmem + acc * N;
        const uint32_t a0 = smem_addr(sK + stage * L::kKeyTileBytes);
        const uint32_t b0 = smem_addr(sQ);
#pragma unroll
        for (int ks = 0; ks < D_I / 32; ++ks) {
          umma_e4m3_ss(d, make_smem_desc(a0 + ks * 32, 16, L::kSBO, L::kSwizzle),
                       make_smem_desc(b0 + ks * 32, 16, L::kSBO, L::kSwizzle), IDESC, ks > 0 ? 1u : 0u);
        }
        umma_commit(&bar_kempty[stage]);
        umma_commit(&bar_accfull[acc]);
      }
    }
  } else {
    // ================= epilogue (warps 0-3) =================
    const int e = tid;  // TMEM lane == key within the tile
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const int seq_start = PAGED ? 0 : p.cu_seqlens[b];
    const int32_t* bt = PAGED ? p.block_table + static_cast<int64_t>(b) * p.max_blocks_per_seq : nullptr;
    bool aborted = false;
#pragma unroll 1
    for (int it = 0; it < ntiles; ++it) {
      const int acc = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      const int s = (tile0 + it) * 128 + e;  // local key position
      // k_scale of this lane's key (0 beyond the sequence)
      float ksc = 0.f;
      if (s < len) {
        if constexpr (!PAGED) ksc = p.k_scale[seq_start + s];
        else ksc = p.k_scale[static_cast<int64_t>(bt[s >> 6]) * 64 + (s & 63)];
      }
      const bool ok = mbar_wait(&bar_accfull[acc], aph);
      if (!ok) record_device_error(DSA_ERR_TIMEOUT);
      if (idx_detail::epi_any(!ok)) {
        aborted = true;
        break;
      }
      tc_fence_after();
      float part[TOK][2];
#pragma unroll
      for (int tt = 0; tt < TOK; ++tt) part[tt][0] = part[tt][1] = 0.f;
      if constexpr (N == 16) {
        uint32_t r[16];
        tmem_ld16(lane_base + acc * N, r);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 16; c += 4) {
          const float4 w4 = idx_detail::lds128(sWq + c);
          const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
          for (int u = 0; u < 4; ++u)
            part[(c + u) / H_I][u & 1] =
                fmaf(wv[u], fmaxf(__uint_as_float(r[c + u]), 0.f), part[(c + u) / H_I][u & 1]);
        }
      } else {
#pragma unroll
        for (int c0 = 0; c0 < N; c0 += 32) {
          uint32_t r[32];
          tmem_ld32(lane_base + acc * N + c0, r);
          tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; c += 4) {
            const float4 w4 = idx_detail::lds128(sWq + c0 + c);
            const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const int col = c0 + c + u;
              part[col / H_I][u & 1] = fmaf(wv[u], fmaxf(__uint_as_float(r[c + u]), 0.f), part[col / H_I][u & 1]);
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_accempty[acc]);

      if constexpr (MODE == kIdxScores) {
#pragma unroll
        for (int tt = 0; tt < TOK; ++tt) {
          if (tt >= ntok) break;
          const int t = t0 + tt;
          const float score = (part[tt][0] + part[tt][1]) * ksc;
          if constexpr (!PAGED) {
            const int64_t g = seq_start + t;
            if (g >= p.row_begin && g < p.row_end && s < len)
              p.scores[(g - p.row_begin) * p.ld + s] = s <= t ? score : -INFINITY;
          } else {
            if (s < len) p.scores[(b - p.row_begin) * p.ld + s] = score;
          }
        }
      } else {
#pragma unroll
        for (int tt = 0; tt < TOK; ++tt) {
          if (tt >= ntok) break;
          const int t = t0 + tt;
          if (s <= t && s < len) {
            const float score = (part[tt][0] + part[tt][1]) * ksc;
            const uint32_t u = __float_as_uint(score);
            if (is_nan_bits(u)) record_device_error(DSA_ERR_DEVICE_CHECK);
            const uint32_t key = order_key(score);
            if (static_cast<long long>(key) > s_thr[tt]) {
              const int pos = atomicAdd(&s_cnt[tt], 1);
              sCandKey[tt * p.cap + pos] = key;
              sCandIdx[tt * p.cap + pos] = s;
            }
          }
        }
        idx_detail::epi_sync();
#pragma unroll 1
        for (int tt = 0; tt < ntok; ++tt) {
          const int n = s_cnt[tt];
          if (n > p.cap - 128) {
            const uint32_t kth = idx_detail::select_compact(sCandKey + tt * p.cap, sCandIdx + tt * p.cap, n, p.k,
                                                            s_sel);
            if (tid == 0) {
              s_cnt[tt] = p.k;
              s_thr[tt] = static_cast<long long>(kth);
            }
            idx_detail::epi_sync();
          }
        }
      }
    }

    if (!aborted) {
      if constexpr (MODE == kIdxScores && !PAGED) {
        // columns past the last computed tile are outside every causal prefix of this CTA
        const int s_begin = ntiles * 128;
        for (int tt = 0; tt < ntok; ++tt) {
          const int64_t g = seq_start + t0 + tt;
          if (g < p.row_begin || g >= p.row_end) continue;
          float* row = p.scores + (g - p.row_begin) * p.ld;
          for (int s = s_begin + e; s < len; s += 128) row[s] = -INFINITY;
        }
      }
      if constexpr (MODE == kIdxTopk) {
        // final cut to min(k, t+1) and ascending emission through a bitmap (aliases the key ring)
        uint32_t* bitmap = reinterpret_cast<uint32_t*>(sK);
#pragma unroll 1
        for (int tt = 0; tt < ntok; ++tt) {
          const int t = t0 + tt;
          const int m = min(p.k, t + 1);
          uint32_t* ck = sCandKey + tt * p.cap;
          int32_t* ci = sCandIdx + tt * p.cap;
          const int n = s_cnt[tt];
          if (n > m) idx_detail::select_compact(ck, ci, n, m, s_sel);
          const int nwords = (t + 1 + 31) / 32;
          for (int wd = e; wd < nwords; wd += 128) bitmap[wd] = 0u;
          idx_detail::epi_sync();
          for (int i = e; i < m; i += 128) atomicOr(&bitmap[ci[i] >> 5], 1u << (ci[i] & 31));
          idx_detail::epi_sync();
          const int per = (nwords + 127) / 128;
          const int w0 = min(nwords, e * per), w1 = min(nwords, w0 + per);
          int bits = 0;
          for (int wd = w0; wd < w1; ++wd) bits += __popc(bitmap[wd]);
          int total;
          int pos = idx_detail::epi_scan(bits, s_sel.scan, total);
          int32_t* out = p.idx_out + static_cast<int64_t>(seq_start + t) * p.k;
          for (int wd = w0; wd < w1; ++wd) {
            uint32_t word = bitmap[wd];
            while (word) {
              const int bit = __ffs(word) - 1;
              out[pos++] = wd * 32 + bit;
              word &= word - 1;
            }
          }
          for (int i = m + e; i < p.k; i += 128) out[i] = -1;
          idx_detail::epi_sync();
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace dsa
