// Lightning indexer on the 5th-generation tensor cores, with the selection fused in.
//
// I[t,s] = k_scale[s] * sum_j (w[t,j] * q_scale[t,j]) * ReLU(sum_d q8[t,j,d] * k8[s,d])
//
// with one query scale per token shared by its heads (q_scale[t,j] = q_scale[t]) or one per
// (token, head).  Every scale is positive, so it commutes with the ReLU and folds into the
// head weight once per CTA.
//
// The e4m3 x e4m3 products run as one tcgen05.mma (kind::f8f6f4, fp32 accumulate in TMEM)
// per 32-deep K slice with
//   M = 128 keys (A operand: a key tile, TMA-loaded, 128-byte swizzle, K-major),
//   N = TOK * H_I  (B operand: the indexer queries of TOK tokens x H_I heads, resident in SMEM).
// Keys on M put one key on each TMEM lane, so the epilogue thread that owns a lane reduces
// over heads in registers: ReLU, the per-head weight (w * q_scale), the head sum, k_scale and
// the causal mask all happen in the epilogue, straight out of TMEM.
//
// Warp roles: EG groups of 4 epilogue warps (warp q of a group owns TMEM lanes 32q..32q+31,
// i.e. keys 32q.. of the tile; group g owns tokens g*TOK/EG ..), then one TMA producer warp
// and one MMA-issuer warp (which also owns TMEM).  Prefill uses EG = 2 (8 epilogue warps,
// two tokens each), decode EG = 1.
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
#include "select.cuh"
#include "sm100.cuh"

namespace dsa {

enum { kIdxScores = 0, kIdxTopk = 1 };

struct IndexerParams {
  const float* q_scale;       // [rows] (q_scale_heads == 1) or [rows, H_I] (q_scale_heads == H_I)
  const float* w;             // [rows, H_I]
  const float* k_scale;       // contiguous [T] | paged [num_blocks * 64]
  const int32_t* cu_seqlens;  // prefill [B+1]
  const int32_t* block_table; // decode [B, max_blocks_per_seq]
  const int32_t* context_lens;// decode [B]
  int32_t max_blocks_per_seq;
  int32_t num_blocks;         // decode: blocks in the paged key pool
  int32_t max_len;            // decode: the declared longest context (<= 64 * max_blocks_per_seq)
  int32_t tiles_per_cta;      // decode: key tiles per CTA
  float* scores;              // kIdxScores output
  int64_t ld;
  uint32_t* gmax;             // paged kIdxScores, optional: [rows, ld16] order key of the largest
  int64_t ld16;               //   score of each 16 consecutive keys (for the decode selection)
  int64_t row_begin, row_end;
  int32_t* idx_out;           // kIdxTopk output [T, k]
  int32_t tok_begin, tok_end; // top-k prefill: token positions [tok_begin, tok_end) of each sequence
  int64_t q_row0;             // prefill: packed row held by row 0 of q / q_scale / w / idx_out
  int32_t k;
  int32_t cap;                // candidate capacity per token (kIdxTopk)
  int32_t q_scale_heads;      // 1: one query scale per token; H_I: one per (token, head)
};

namespace idx_detail {

// 16-byte shared-memory load that the compiler may not hoist out of the tile loop (the
// per-head weights of all TOK tokens would not fit in registers).
__device__ __forceinline__ float4 lds128(const float* p) {
  float4 v;
  asm volatile("ld.shared.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(dev::smem_addr(p)));
  return v;
}

}  // namespace idx_detail

template <int D_I>
struct IdxLayout {
  static constexpr uint32_t kSwizzle = D_I == 128 ? dev::kSwizzle128B : dev::kSwizzle64B;
  static constexpr uint32_t kSBO = D_I == 128 ? 1024u : 512u;  // bytes between 8-row groups
  static constexpr int kKeyTileBytes = 128 * D_I;
};

template <int TOK>
struct IdxGroups {
  static constexpr int kEG = TOK >= 2 ? 2 : 1;   // epilogue groups
  static constexpr int kThreads = (4 * kEG + 2) * 32;
};

// Shared-memory bytes the kernel needs (besides the 1 KB alignment slack).
template <int D_I, int H_I, int TOK, int MODE, int STAGES>
__host__ __device__ constexpr int indexer_smem_bytes(int cap) {
  return ((TOK * H_I * D_I + 1023) / 1024) * 1024 + STAGES * IdxLayout<D_I>::kKeyTileBytes + TOK * H_I * 4 +
         (MODE == kIdxTopk ? TOK * cap * 8 : 0);
}

template <int D_I, int H_I, int TOK, int MODE, bool PAGED, int STAGES>
__global__ void __launch_bounds__(IdxGroups<TOK>::kThreads, 1)
    indexer_kernel(const __grid_constant__ CUtensorMap q_map, const __grid_constant__ CUtensorMap k_map,
                   const IndexerParams p) {
  using namespace dev;
  using L = IdxLayout<D_I>;
  constexpr int EG = IdxGroups<TOK>::kEG;
  constexpr int TPG = TOK / EG;          // tokens per epilogue group
  constexpr int N = TOK * H_I;
  constexpr int NG = N / EG;             // accumulator columns per group
  constexpr int Q_BYTES = N * D_I;
  constexpr int TMEM_COLS = (2 * N < 32) ? 32 : 2 * N;
  constexpr uint32_t IDESC = idesc_e4m3(128, N);
  constexpr int PRODUCER_WARP = 4 * EG, MMA_WARP = 4 * EG + 1;
  static_assert(N % 16 == 0 && N <= 256, "MMA N must be a multiple of 16 in [16, 256]");
  static_assert(NG % 8 == 0, "group column slice must be a multiple of 8");

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
  __shared__ int s_cnt[TOK][4];       // candidate count per token and warp region
  __shared__ sel::Scratch s_sel[EG];

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  // ---------------- work item ----------------
  int b = blockIdx.y;
  int64_t key_row0;   // global row of local key 0 (contiguous keys)
  int t0, ntok, tile0, ntiles, len;
  int64_t q_row;      // row of the Q tile in the [rows * H_I, D_I] view
  if constexpr (!PAGED) {
    const int seq_start = p.cu_seqlens[b];
    len = p.cu_seqlens[b + 1] - seq_start;
    // tokens [tok_begin, min(len, tok_end)) of the sequence, TOK per CTA, heavy blocks first
    const int tend = min(len, p.tok_end);
    const int tb = static_cast<int>(gridDim.x) - 1 - static_cast<int>(blockIdx.x);
    t0 = p.tok_begin + tb * TOK;
    if (t0 >= tend) return;
    ntok = min(TOK, tend - t0);
    if (MODE == kIdxScores) {
      const int64_t g0 = seq_start + t0, g1 = g0 + ntok;
      if (g1 <= p.row_begin || g0 >= p.row_end) return;
    }
    tile0 = 0;
    ntiles = (t0 + ntok - 1) / 128 + 1;
    key_row0 = seq_start;
    q_row = (static_cast<int64_t>(seq_start + t0) - p.q_row0) * H_I;
  } else {
    if (b < p.row_begin || b >= p.row_end) return;
    // never read past the block table row nor write past the declared longest context (the
    // width of the caller's score rows): a longer context is an input error
    const int ctx = p.context_lens[b];
    if (ctx > p.max_len && blockIdx.x == 0 && threadIdx.x == 0) record_device_error(DSA_ERR_DEVICE_CHECK);
    len = min(ctx, p.max_len);
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
      mbar_init(&bar_accempty[i], 4 * EG);
    }
    mbar_init(&bar_q, 1);
    s_abort = 0;
    fence_mbar_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(&s_tmem, TMEM_COLS);
    tmem_relinquish();
  }
  for (int i = tid; i < N; i += blockDim.x) {
    const int tt = i / H_I, j = i % H_I;
    float v = 0.f;
    if (tt < ntok) {
      const int64_t row = PAGED ? b : (p.cu_seqlens[b] + t0 + tt - p.q_row0);
      v = p.w[row * H_I + j] * p.q_scale[p.q_scale_heads == 1 ? row : row * H_I + j];
    }
    sWq[i] = v;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  if (warp == PRODUCER_WARP) {
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
            int phys = bt[lb < nblocks_seq ? lb : 0];
            // a block id outside the key pool never reaches the TMA unit: block 0 is loaded in
            // its place and the epilogue scores the block's keys -inf (and reports them)
            if (phys < 0 || phys >= p.num_blocks) phys = 0;
            tma_load_2d(dst + h * 64 * D_I, &k_map, &bar_kfull[stage], 0, phys * 64);
          }
        }
      }
    }
  } else if (warp == MMA_WARP) {
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
    // ================= epilogue groups =================
    const int g = warp >> 2;                    // group
    const int q = warp & 3;                     // TMEM lane quadrant
    const sel::Group G{1 + g, tid - 128 * g};
    const int e = 32 * q + lane;                // key within the tile
    const int tg0 = g * TPG;                    // first token of this group
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(q * 32) << 16) + g * NG;
    const int seq_start = PAGED ? 0 : p.cu_seqlens[b];
    const int32_t* bt = PAGED ? p.block_table + static_cast<int64_t>(b) * p.max_blocks_per_seq : nullptr;
    const int Q = p.cap / 4;
    bool aborted = false;
    // fused top-k state in registers: this warp's region fill count, the acceptance
    // threshold (uniform), and the smallest / largest key this thread appended
    int wcnt[TPG];
    long long thr[TPG];
    uint32_t kmin[TPG], kmax[TPG];
#pragma unroll
    for (int tt = 0; tt < TPG; ++tt) {
      wcnt[tt] = 0;
      thr[tt] = -1;
      kmin[tt] = 0xFFFFFFFFu;
      kmax[tt] = 0u;
    }
#pragma unroll 1
    for (int it = 0; it < ntiles; ++it) {
      const int acc = it & 1;
      const uint32_t aph = (it >> 1) & 1;
      const int s = (tile0 + it) * 128 + e;  // local key position
      float ksc = 0.f;                       // k_scale of this lane's key (0 beyond the sequence)
      bool bad_blk = false;                  // paged: the key's block id lies outside the pool
      if (s < len) {
        if constexpr (!PAGED) ksc = p.k_scale[seq_start + s];
        else {
          const int blk = bt[s >> 6];
          if (blk >= 0 && blk < p.num_blocks) {
            ksc = p.k_scale[static_cast<int64_t>(blk) * 64 + (s & 63)];
          } else {
            bad_blk = true;
            record_device_error(DSA_ERR_DEVICE_CHECK);
          }
        }
      }
      const bool ok = mbar_wait(&bar_accfull[acc], aph);
      if (!ok) record_device_error(DSA_ERR_TIMEOUT);
      // top-k mode takes the abort decision at its group vote below (one barrier per two
      // tiles); reading a stale accumulator before it is harmless
      if (MODE == kIdxScores && sel::gany(G, !ok)) {
        aborted = true;
        break;
      }
      tc_fence_after();
      float part[TPG][2];
#pragma unroll
      for (int tt = 0; tt < TPG; ++tt) part[tt][0] = part[tt][1] = 0.f;
      const uint32_t abase = lane_base + acc * N;
      // part[tt] += w * ReLU(acc) over the 32 columns c0.. held in r
      auto accumulate32 = [&](const uint32_t(&r)[32], int c0) {
#pragma unroll
        for (int c = 0; c < 32; c += 4) {
          const float4 w4 = idx_detail::lds128(sWq + g * NG + c0 + c);
          const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int col = c0 + c + u;  // column inside the group's slice
            part[col / H_I][u & 1] = fmaf(wv[u], fmaxf(__uint_as_float(r[c + u]), 0.f), part[col / H_I][u & 1]);
          }
        }
      };
      if constexpr (NG >= 64 && NG % 64 == 0) {
        // Software pipeline over 32-column slices: the TMEM load of the next slice is in
        // flight while this one is summed (tcgen05.wait::ld waits for every load issued so
        // far, so each wait comes one slice of work after its load).  reg_fence keeps the
        // compiler from moving uses of the loaded registers above their wait.
        uint32_t ra[32], rb[32];
        tmem_ld32(abase, ra);
        tmem_wait_ld();
        reg_fence(ra);
#pragma unroll
        for (int c0 = 0; c0 < NG; c0 += 64) {
          tmem_ld32(abase + c0 + 32, rb);
          accumulate32(ra, c0);
          tmem_wait_ld();
          reg_fence(rb);
          if (c0 + 64 < NG) tmem_ld32(abase + c0 + 64, ra);
          accumulate32(rb, c0 + 32);
          if (c0 + 64 < NG) {
            tmem_wait_ld();
            reg_fence(ra);
          }
        }
      } else {
      constexpr int CH = NG >= 32 ? 32 : NG;
#pragma unroll
      for (int c0 = 0; c0 < NG; c0 += CH) {
        uint32_t r[32];
        if constexpr (CH == 32) {
          tmem_ld32(lane_base + acc * N + c0, *reinterpret_cast<uint32_t(*)[32]>(r));
        } else if constexpr (CH == 16) {
          tmem_ld16(lane_base + acc * N + c0, *reinterpret_cast<uint32_t(*)[16]>(r));
        } else {
          uint32_t r16[16];
          static_assert(CH == 8, "unsupported column slice");
          asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                       : "=r"(r16[0]), "=r"(r16[1]), "=r"(r16[2]), "=r"(r16[3]), "=r"(r16[4]), "=r"(r16[5]),
                         "=r"(r16[6]), "=r"(r16[7])
                       : "r"(lane_base + acc * N + c0));
#pragma unroll
          for (int u = 0; u < 8; ++u) r[u] = r16[u];
        }
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < CH; c += 4) {
          const float4 w4 = idx_detail::lds128(sWq + g * NG + c0 + c);
          const float wv[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int col = c0 + c + u;  // column inside the group's slice
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
        for (int tt = 0; tt < TPG; ++tt) {
          if (tg0 + tt >= ntok) break;
          const int t = t0 + tg0 + tt;
          const float score = (part[tt][0] + part[tt][1]) * ksc;
          if constexpr (!PAGED) {
            const int64_t gr = seq_start + t;
            if (gr >= p.row_begin && gr < p.row_end && s < len)
              p.scores[(gr - p.row_begin) * p.ld + s] = s <= t ? score : -INFINITY;
          } else {
            const float v = bad_blk ? -INFINITY : score;
            if (s < len) p.scores[(b - p.row_begin) * p.ld + s] = v;
            if (p.gmax != nullptr) {  // uniform: every lane takes part in the shuffles
              // the largest key of the 16 keys of this half-warp (lanes 16h .. 16h+15 hold keys
              // 16 * (s / 16) ..); keys past the context take no part
              uint32_t key = s < len ? order_key(v) : 0u;
#pragma unroll
              for (int o = 8; o > 0; o >>= 1) key = max(key, __shfl_xor_sync(0xffffffffu, key, o));
              if ((lane & 15) == 0 && s < len) p.gmax[(b - p.row_begin) * p.ld16 + (s >> 4)] = key;
            }
          }
        }
      } else {
        bool need_cut = false;
#pragma unroll
        for (int tt = 0; tt < TPG; ++tt) {
          const int t = t0 + tg0 + tt;
          const float score = (part[tt][0] + part[tt][1]) * ksc;
          const bool valid = tg0 + tt < ntok && s <= t && s < len;
          if (valid && is_nan_bits(__float_as_uint(score))) record_device_error(DSA_ERR_DEVICE_CHECK);
          const uint32_t key = order_key(score);
          const bool take = valid && static_cast<long long>(key) > thr[tt];
          const uint32_t m = __ballot_sync(0xffffffffu, take);
          if (take) {
            const int pos = (tg0 + tt) * p.cap + q * Q + wcnt[tt] + __popc(m & ((1u << lane) - 1u));
            sCandKey[pos] = key;
            sCandIdx[pos] = s;
            kmin[tt] = min(kmin[tt], key);
            kmax[tt] = max(kmax[tt], key);
          }
          wcnt[tt] += __popc(m);
          // the group votes after every second tile, and the two tiles after a vote add at most
          // 64 entries to a region: cut a token when one of its regions holds more than Q - 64
          need_cut |= wcnt[tt] > Q - 64;
        }
        if ((it & 1) && sel::gany(G, need_cut || !ok)) {
          if (sel::gany(G, !ok)) {
            aborted = true;
            break;
          }
          if (lane == 0) {
#pragma unroll
            for (int tt = 0; tt < TPG; ++tt) s_cnt[tg0 + tt][q] = wcnt[tt];
          }
          sel::gsync(G);
#pragma unroll
          for (int tt = 0; tt < TPG; ++tt) {
            const int tok = tg0 + tt;
            const bool full = s_cnt[tok][0] > Q - 64 || s_cnt[tok][1] > Q - 64 || s_cnt[tok][2] > Q - 64 ||
                              s_cnt[tok][3] > Q - 64;
            if (full) {  // uniform over the group
              uint32_t lo, hi;
              sel::group_minmax(G, s_sel[g], kmin[tt], kmax[tt], lo, hi);
              if (thr[tt] >= 0) lo = min(lo, static_cast<uint32_t>(thr[tt]));  // the smallest kept key
              sel::Cands C{sCandKey + tok * p.cap, sCandIdx + tok * p.cap, &s_cnt[tok][0], Q};
              const uint32_t nthr = sel::cut_stream(G, C, s_sel[g], p.k, p.cap - 512, lo, hi);
              thr[tt] = static_cast<long long>(nthr);
              kmin[tt] = 0xFFFFFFFFu;  // every later key is > thr
            }
            wcnt[tt] = s_cnt[tok][q];
          }
          sel::gsync(G);
        }
      }
    }

    if (!aborted) {
      if constexpr (MODE == kIdxScores && !PAGED) {
        // columns past the last computed tile are outside every causal prefix of this CTA
        const int s_begin = ntiles * 128;
        for (int tt = 0; tt < TPG; ++tt) {
          if (tg0 + tt >= ntok) break;
          const int64_t gr = seq_start + t0 + tg0 + tt;
          if (gr < p.row_begin || gr >= p.row_end) continue;
          float* row = p.scores + (gr - p.row_begin) * p.ld;
          for (int s = s_begin + e; s < len; s += 128) row[s] = -INFINITY;
        }
      }
      if constexpr (MODE == kIdxTopk) {
        // final cut to min(k, t+1) and ascending emission through a bitmap (aliases the key
        // ring; each group has its own half)
        if (lane == 0) {
#pragma unroll
          for (int tt = 0; tt < TPG; ++tt) s_cnt[tg0 + tt][q] = wcnt[tt];
        }
        sel::gsync(G);
        uint32_t* bitmap = reinterpret_cast<uint32_t*>(sK + g * (STAGES * L::kKeyTileBytes / EG));
#pragma unroll 1
        for (int tt = 0; tt < TPG; ++tt) {
          const int tok = tg0 + tt;
          if (tok >= ntok) break;
          const int t = t0 + tok;
          uint32_t lo, hi;
          sel::group_minmax(G, s_sel[g], kmin[tt], kmax[tt], lo, hi);
          if (thr[tt] >= 0) lo = min(lo, static_cast<uint32_t>(thr[tt]));  // the smallest kept key
          sel::Cands C{sCandKey + tok * p.cap, sCandIdx + tok * p.cap, &s_cnt[tok][0], Q};
          sel::cut_final(G, C, s_sel[g], min(p.k, t + 1), lo, hi);
          sel::emit_sorted(G, C, s_sel[g], bitmap, t + 1, p.idx_out + (static_cast<int64_t>(seq_start + t) - p.q_row0) * p.k, p.k);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

}  // namespace dsa
