// Sparse MLA in MQA mode on a CTA pair (thread-block cluster of 2).
//
// For a query token t with selected latent rows c_i (i over the top-k selection):
//   out[t,h,:] = sum_i softmax_i(sm_scale * q[t,h,:] . c_i) * c_i[0:512]
// Every head of the token shares the same 576-d latent rows (MQA mode), so one token is a
// [128 heads x 576] x [576 x k] product followed by a [128 x k] x [k x 512] product.
//
// Split over the pair (rank r = 0, 1), with no duplicated tensor-core work:
//   * rank r owns the latent dims D_r = [256r, 256r+256) u [512+32r, 512+32r+32): it holds
//     q[t, :, D_r] in TMEM (the A operand of Q.K^T), gathers only those 288 dims of each
//     selected row (TMA gather4, 128- and 64-byte swizzle), and computes the PARTIAL logits
//     S_r = q[:, D_r] . c[:, D_r];
//   * rank r owns the output half O_r = out[:, 256r : 256r+256] (the value dims it already
//     gathered) as a [128 x 256] fp32 accumulator in TMEM.
// The two partial logits are combined multiplicatively, which needs only one small exchange
// per 64-key chunk: each rank computes P_r = 2^(x*S_r - m_r) (x = sm_scale*log2 e, m_r its own
// running reference), rounds it to bf16 and sends it, with m_r, to its peer through
// distributed shared memory.  Both ranks then form the same P = P_0 * P_1 =
// 2^(x*(S_0+S_1) - (m_0+m_1)), i.e. the softmax numerator relative to M = m_0 + m_1, and
// accumulate O_r += P . V_r on the tensor cores.  M only moves when one rank's chunk maximum
// exceeds its reference by more than 2^8 (then O_r and the row sum are rescaled); both ranks
// see the same (m_0, m_1) and take the same decisions.
//
// Per CTA: warps 0-3 softmax/epilogue (thread h = head h = TMEM lane h), warp 4 TMA gather
// producer, warp 5 MMA issuer and TMEM owner.  TMEM columns: O_r [0,256), Q_r [256,400),
// S_r [400,464), P [464,496).  SMEM: a 4-stage ring of gathered chunks (64 rows x 576 B) and
// a double-buffered exchange area written by the peer.
//
// The same kernel serves decode: a work item is then (sequence, split of its selection) over
// a paged latent cache, and the unnormalised partial result (O, M, l) goes to a workspace
// that a small kernel merges by log-sum-exp.
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
  int32_t B;
  int32_t H;                  // query heads (<= 128; rows >= H are padding)
  int32_t k;                  // selected entries per row (multiple of 64)
  int64_t rows;               // prefill: total tokens; decode: B
  int32_t splits;             // decode: selection splits per sequence
  float scale_log2;           // sm_scale * log2(e)
  __nv_bfloat16* out;         // prefill: [rows, H, 512]
  float* lse;                 // prefill: [rows, H] natural log (nullable)
  float* part_o;              // decode: [B, splits, H, 512] unnormalised
  float* part_ml;             // decode: [B, splits, H, 2] (M in log2 units, l)
};

namespace mla {

constexpr int kChunk = 64;                         // selected rows per pipeline step
constexpr int kStages = 4;
constexpr int kNopeBlockBytes = kChunk * 128;      // 64 rows x 64 dims bf16, 128-byte swizzle
constexpr int kRopeBlockBytes = kChunk * 64;       // 64 rows x 32 dims bf16, 64-byte swizzle
constexpr int kStageBytes = 4 * kNopeBlockBytes + kRopeBlockBytes;  // 36864
constexpr int kXRowBytes = 144;                    // exchange row: 64 bf16 + m + pad
constexpr int kXBufBytes = 128 * kXRowBytes;
constexpr int kSmemBytes = kStages * kStageBytes + 2 * kXBufBytes;
constexpr uint32_t kColO = 0, kColQ = 256, kColS = 400, kColP = 464;
constexpr float kTau = 8.f;                        // lazy-rescale margin (log2 units)

__device__ __forceinline__ void sm_sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ bool sm_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, 1, 128, q;\n\tselp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
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

template <bool DECODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(192, 1)
    sparse_mla_kernel(const __grid_constant__ CUtensorMap lat128, const __grid_constant__ CUtensorMap lat64,
                      const MlaParams p) {
  using namespace dev;
  using namespace mla;
  constexpr uint32_t IDESC_QK = idesc_bf16(128, kChunk, false, false);
  constexpr uint32_t IDESC_PV = idesc_bf16(128, 256, false, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sKV = smem;                                     // [kStages][kStageBytes]
  uint8_t* sX = smem + kStages * kStageBytes;              // [2][128][kXRowBytes], written by the peer

  __shared__ uint64_t bar_kvfull[kStages], bar_kvempty[kStages];
  __shared__ uint64_t bar_qfull, bar_sfull, bar_sfree, bar_pfull, bar_pvdone, bar_ofree;
  __shared__ uint64_t bar_xfull[2], bar_xempty[2];
  __shared__ uint64_t s_vmask[kStages];                    // valid rows of each staged chunk
  __shared__ uint32_t s_tmem;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank(), peer = rank ^ 1u;
  const int cid = static_cast<int>(cluster_id_x()), ncl = static_cast<int>(num_clusters_x());
  const int64_t nunits = DECODE ? static_cast<int64_t>(p.B) * p.splits : p.rows;

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bar_kvfull[i], 1);
      mbar_init(&bar_kvempty[i], 1);
    }
    mbar_init(&bar_qfull, 128);
    mbar_init(&bar_sfull, 1);
    mbar_init(&bar_sfree, 4);
    mbar_init(&bar_pfull, 4);
    mbar_init(&bar_pvdone, 1);
    mbar_init(&bar_ofree, 4);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_xfull[i], 128);   // 128 remote arrivals from the peer's softmax threads
      mbar_init(&bar_xempty[i], 128);
    }
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(&s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // barriers of both CTAs are initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  // Work item -> (selection row, query row, key offset inside the row, key count, sequence).
  auto unit_info = [&](int64_t u, int64_t& qrow, int& kbeg, int& kend, int& seq, int& seq_start, int& seq_len) {
    if constexpr (DECODE) {
      seq = static_cast<int>(u / p.splits);
      const int sp = static_cast<int>(u % p.splits);
      const int per = p.k / p.splits;
      qrow = seq;
      kbeg = sp * per;
      kend = kbeg + per;
      seq_start = 0;
      seq_len = min(p.context_lens[seq], p.max_blocks_per_seq * 64);
    } else {
      qrow = u;
      kbeg = 0;
      kend = p.k;
      // sequence of token u: binary search in cu_seqlens
      int lo = 0, hi = p.B;
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (p.cu_seqlens[mid] <= u) lo = mid;
        else hi = mid;
      }
      seq = lo;
      seq_start = p.cu_seqlens[lo];
      seq_len = p.cu_seqlens[lo + 1] - seq_start;
    }
  };
  // chunks [c0, c1) of the selection row this unit processes
  auto unit_chunks = [&](int64_t qrow, int kbeg, int kend, int& c0, int& c1) {
    const int act = active_chunks(p.idx + qrow * p.k, p.k);
    c0 = kbeg / kChunk;
    c1 = min(kend / kChunk, act);
    if (c1 <= c0) c1 = c0 + 1;  // always at least one chunk (all masked if empty)
  };

  if (warp == 4) {
    // ================= gather producer =================
    uint32_t g = 0;
    bool ok = true;
    for (int64_t u = cid; ok && u < nunits; u += ncl) {
      int64_t qrow;
      int kbeg, kend, seq, seq_start, seq_len, c0, c1;
      unit_info(u, qrow, kbeg, kend, seq, seq_start, seq_len);
      unit_chunks(qrow, kbeg, kend, c0, c1);
      const int32_t* row = p.idx + qrow * p.k;
      const int32_t* bt = DECODE ? p.block_table + static_cast<int64_t>(seq) * p.max_blocks_per_seq : nullptr;
      for (int c = c0; c < c1; ++c, ++g) {
        const int stage = static_cast<int>(g % kStages);
        const uint32_t ph = (g / kStages) & 1u;
        if (!mbar_wait(&bar_kvempty[stage], ph ^ 1u)) {
          record_device_error(DSA_ERR_TIMEOUT);
          ok = false;
          break;
        }
        // lanes 0..15 each gather 4 rows
        int4 ix = make_int4(-1, -1, -1, -1);
        if (lane < 16) ix = *reinterpret_cast<const int4*>(row + c * kChunk + 4 * lane);
        int v[4] = {ix.x, ix.y, ix.z, ix.w};
        uint32_t valid4 = 0;
        int phys[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const bool okj = lane < 16 && v[j] >= 0 && v[j] < seq_len;
          valid4 |= okj ? (1u << j) : 0u;
          const int pos = okj ? v[j] : 0;
          if constexpr (DECODE) phys[j] = bt[pos >> 6] * 64 + (pos & 63);
          else phys[j] = seq_start + pos;
        }
        // 64-bit validity mask of the chunk: lane l contributes bits 4l..4l+3
        uint64_t mask = static_cast<uint64_t>(valid4) << (4 * (lane & 15));
        mask |= __shfl_xor_sync(0xffffffffu, mask, 1);
        mask |= __shfl_xor_sync(0xffffffffu, mask, 2);
        mask |= __shfl_xor_sync(0xffffffffu, mask, 4);
        mask |= __shfl_xor_sync(0xffffffffu, mask, 8);
        if (lane == 0) {
          s_vmask[stage] = mask;
          mbar_arrive_expect_tx(&bar_kvfull[stage], kStageBytes);
        }
        __syncwarp();
        if (lane < 16) {
          uint8_t* st = sKV + stage * kStageBytes;
#pragma unroll
          for (int j = 0; j < 4; ++j)
            tma_gather4(st + j * kNopeBlockBytes + lane * 512, &lat128, &bar_kvfull[stage],
                        static_cast<int32_t>(256 * rank + 64 * j), phys[0], phys[1], phys[2], phys[3]);
          tma_gather4(st + 4 * kNopeBlockBytes + lane * 256, &lat64, &bar_kvfull[stage],
                      static_cast<int32_t>(512 + 32 * rank), phys[0], phys[1], phys[2], phys[3]);
        }
        __syncwarp();
      }
    }
  } else if (warp == 5) {
    // ================= MMA issuer =================
    uint32_t g = 0, tok = 0;
    bool ok = true;
    int64_t pend = -1;           // chunk whose P.V is still to be issued
    bool pend_first = false;     // ... and whether it starts its unit
    uint32_t pend_tok = 0;
    auto issue_pv = [&]() -> bool {
      const uint32_t x = static_cast<uint32_t>(pend);
      if (!mbar_wait(&bar_pfull, x & 1u)) return false;
      if (pend_first && pend_tok > 0 && !mbar_wait(&bar_ofree, (pend_tok - 1) & 1u)) return false;
      tc_fence_after();
      if (lane == 0) {
        const uint32_t st = smem_addr(sKV + (x % kStages) * kStageBytes);
#pragma unroll
        for (int kk = 0; kk < kChunk / 16; ++kk)
          umma_bf16_ts(tmem + kColO, tmem + kColP + kk * 8, make_smem_desc(st + kk * 2048, 8192, 1024, kSwizzle128B),
                       IDESC_PV, (pend_first && kk == 0) ? 0u : 1u);
        umma_commit(&bar_pvdone);
        umma_commit(&bar_kvempty[x % kStages]);
      }
      __syncwarp();
      return true;
    };
    for (int64_t u = cid; ok && u < nunits; u += ncl, ++tok) {
      int64_t qrow;
      int kbeg, kend, seq, seq_start, seq_len, c0, c1;
      unit_info(u, qrow, kbeg, kend, seq, seq_start, seq_len);
      unit_chunks(qrow, kbeg, kend, c0, c1);
      for (int c = c0; c < c1; ++c, ++g) {
        const int stage = static_cast<int>(g % kStages);
        if (!mbar_wait(&bar_kvfull[stage], (g / kStages) & 1u) || (c == c0 && !mbar_wait(&bar_qfull, tok & 1u)) ||
            (g > 0 && !mbar_wait(&bar_sfree, (g - 1) & 1u))) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t st = smem_addr(sKV + stage * kStageBytes);
#pragma unroll
          for (int kk = 0; kk < 16; ++kk)  // 256 nope dims: 4 blocks x 4 steps of 16
            umma_bf16_ts(tmem + kColS, tmem + kColQ + kk * 8,
                         make_smem_desc(st + (kk >> 2) * kNopeBlockBytes + (kk & 3) * 32, 16, 1024, kSwizzle128B),
                         IDESC_QK, kk > 0 ? 1u : 0u);
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)   // 32 rope dims
            umma_bf16_ts(tmem + kColS, tmem + kColQ + (16 + kk) * 8,
                         make_smem_desc(st + 4 * kNopeBlockBytes + kk * 32, 16, 512, kSwizzle64B), IDESC_QK, 1u);
          umma_commit(&bar_sfull);
        }
        __syncwarp();
        if (pend >= 0 && !issue_pv()) {
          ok = false;
          break;
        }
        pend = g;
        pend_first = c == c0;
        pend_tok = tok;
      }
    }
    if (ok && pend >= 0) ok = issue_pv();
    if (!ok && lane == 0) record_device_error(DSA_ERR_TIMEOUT);
  } else {
    // ================= softmax / exchange / epilogue (warps 0-3) =================
    const int h = tid;  // head row == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const uint32_t x_peer = map_to_rank(smem_addr(sX), peer);
    uint32_t xbar_full_peer[2], xbar_empty_peer[2];
    for (int i = 0; i < 2; ++i) {
      xbar_full_peer[i] = map_to_rank(smem_addr(&bar_xfull[i]), peer);
      xbar_empty_peer[i] = map_to_rank(smem_addr(&bar_xempty[i]), peer);
    }
    // Q rows of this rank's dims into TMEM columns [kColQ, kColQ + 144)
    auto load_q = [&](int64_t qrow) {
      const __nv_bfloat16* qr = p.q + (qrow * p.H + h) * 576;
      const bool real = h < p.H;
#pragma unroll
      for (int c = 0; c < 144; c += 16) {
        uint32_t v[16];
#pragma unroll
        for (int j = 0; j < 16; j += 4) {
          const int col = c + j;  // packed column: dims 2col, 2col+1 of D_r
          const int d = 2 * col < 256 ? 256 * static_cast<int>(rank) + 2 * col
                                      : 512 + 32 * static_cast<int>(rank) + (2 * col - 256);
          uint4 w = make_uint4(0u, 0u, 0u, 0u);
          if (real) w = *reinterpret_cast<const uint4*>(qr + d);
          v[j] = w.x;
          v[j + 1] = w.y;
          v[j + 2] = w.z;
          v[j + 3] = w.w;
        }
        tmem_st16(lane_base + kColQ + c, v);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar_qfull);
    };

    uint32_t g = 0, tok = 0;
    bool aborted = false;
    if (cid < nunits) {
      int64_t qrow;
      int kbeg, kend, seq, ss, sl;
      unit_info(cid, qrow, kbeg, kend, seq, ss, sl);
      load_q(qrow);
    }
    for (int64_t u = cid; u < nunits; u += ncl, ++tok) {
      int64_t qrow;
      int kbeg, kend, seq, seq_start, seq_len, c0, c1;
      unit_info(u, qrow, kbeg, kend, seq, seq_start, seq_len);
      unit_chunks(qrow, kbeg, kend, c0, c1);
      float m_own = -INFINITY, m_peer = -INFINITY, M = -INFINITY, l = 0.f;
      for (int c = c0; c < c1; ++c, ++g) {
        const int stage = static_cast<int>(g % kStages);
        bool ok = mbar_wait(&bar_sfull, g & 1u);
        if (sm_any(!ok)) {
          aborted = true;
          break;
        }
        tc_fence_after();
        uint32_t sr[64];
        tmem_ld32(lane_base + kColS, *reinterpret_cast<uint32_t(*)[32]>(sr));
        tmem_ld32(lane_base + kColS + 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_sfree);
        if (c == c1 - 1 && u + ncl < nunits) {  // the last Q.K^T of this unit is done: stage the next Q
          int64_t nq;
          int a, bb, cc, dd, ee;
          unit_info(u + ncl, nq, a, bb, cc, dd, ee);
          load_q(nq);
        }
        // own partial logits (log2 units) and this chunk's maximum; the validity mask was
        // written by the producer before it armed this stage's barrier, so acquire that
        // barrier's (still current) phase before reading it
        ok = mbar_wait(&bar_kvfull[stage], (g / kStages) & 1u);
        if (sm_any(!ok)) {
          aborted = true;
          break;
        }
        const uint64_t vmask = s_vmask[stage];
        float cmax = -INFINITY;
#pragma unroll
        for (int i = 0; i < 64; ++i) {
          const float xv = __uint_as_float(sr[i]) * p.scale_log2;
          sr[i] = __float_as_uint(xv);
          if ((vmask >> i) & 1ull) cmax = fmaxf(cmax, xv);
        }
        if (cmax > m_own + kTau || (m_own == -INFINITY && cmax > -INFINITY)) m_own = cmax;
        uint32_t pown[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float a = ((vmask >> (2 * i)) & 1ull) ? exp2f(__uint_as_float(sr[2 * i]) - m_own) : 0.f;
          const float bq = ((vmask >> (2 * i + 1)) & 1ull) ? exp2f(__uint_as_float(sr[2 * i + 1]) - m_own) : 0.f;
          pown[i] = pack_bf16x2(a, bq);
        }
        // exchange with the peer: send my row, then read the peer's row of the same chunk
        const int xb = static_cast<int>(g & 1u);
        const uint32_t xuse = g >> 1;
        ok = mbar_wait_cluster(&bar_xempty[xb], (xuse & 1u) ^ 1u);  // the peer has read my previous row
        if (sm_any(!ok)) {
          aborted = true;
          break;
        }
        const uint32_t dst = x_peer + xb * kXBufBytes + h * kXRowBytes;
#pragma unroll
        for (int i = 0; i < 8; ++i)
          st_cluster_v4(dst + 16 * i, pown[4 * i], pown[4 * i + 1], pown[4 * i + 2], pown[4 * i + 3]);
        st_cluster_f32(dst + 128, m_own);
        mbar_arrive_remote(xbar_full_peer[xb]);
        ok = mbar_wait_cluster(&bar_xfull[xb], xuse & 1u);
        if (sm_any(!ok)) {
          aborted = true;
          break;
        }
        const uint8_t* src = sX + xb * kXBufBytes + h * kXRowBytes;
        uint32_t ppeer[32];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint4 w = *reinterpret_cast<const uint4*>(src + 16 * i);
          ppeer[4 * i] = w.x;
          ppeer[4 * i + 1] = w.y;
          ppeer[4 * i + 2] = w.z;
          ppeer[4 * i + 3] = w.w;
        }
        m_peer = *reinterpret_cast<const float*>(src + 128);
        mbar_arrive_remote(xbar_empty_peer[xb]);
        // P = P_own * P_peer relative to M = m_own + m_peer (identical in both ranks)
        const float Mn = m_own + m_peer;
        float psum = 0.f;
        uint32_t pp[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float2 a = unpack_bf16x2(pown[i]), bq = unpack_bf16x2(ppeer[i]);
          pp[i] = pack_bf16x2(a.x * bq.x, a.y * bq.y);
          const float2 r = unpack_bf16x2(pp[i]);
          psum += r.x + r.y;
        }
        // the previous chunk's P.V must be done before P is overwritten (and before O is rescaled)
        if (g > 0) {
          ok = mbar_wait(&bar_pvdone, (g - 1) & 1u);
          if (sm_any(!ok)) {
            aborted = true;
            break;
          }
          tc_fence_after();
        }
        // Rescale O_r when M moved.  tcgen05.ld/st are warp-collective, so the whole warp runs
        // the loop if any of its rows needs it (alpha = 1 for the others).
        const bool need_rescale = c > c0 && Mn != M && M > -INFINITY;
        if (__any_sync(0xffffffffu, need_rescale)) {
          const float alpha = need_rescale ? exp2f(M - Mn) : 1.f;
          l *= alpha;
#pragma unroll 1
          for (int c32 = 0; c32 < 256; c32 += 32) {
            uint32_t o[32];
            tmem_ld32(lane_base + kColO + c32, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(lane_base + kColO + c32, o);
          }
        }
        M = Mn;
        l += psum;
        tmem_st32(lane_base + kColP, pp);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_pfull);
      }
      if (aborted) break;
      // epilogue of the unit: O_r / l
      bool ok = mbar_wait(&bar_pvdone, (g - 1) & 1u);
      if (sm_any(!ok)) {
        aborted = true;
        break;
      }
      tc_fence_after();
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      if constexpr (!DECODE) {
        __nv_bfloat16* orow = p.out + (qrow * p.H + h) * 512 + 256 * rank;
#pragma unroll 1
        for (int c32 = 0; c32 < 256; c32 += 32) {
          uint32_t o[32];
          tmem_ld32(lane_base + kColO + c32, o);
          tmem_wait_ld();
          if (h < p.H) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              pk[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
#pragma unroll
            for (int i = 0; i < 4; ++i)
              *reinterpret_cast<uint4*>(orow + c32 + 8 * i) = make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
          }
        }
        if (rank == 0 && p.lse != nullptr && h < p.H)
          p.lse[qrow * p.H + h] = l > 0.f ? (M + log2f(l)) * 0.69314718055994531f : -INFINITY;
      } else {
        const int sp = static_cast<int>(u % p.splits);
        float* po = p.part_o + ((static_cast<int64_t>(seq) * p.splits + sp) * p.H + h) * 512 + 256 * rank;
#pragma unroll 1
        for (int c32 = 0; c32 < 256; c32 += 32) {
          uint32_t o[32];
          tmem_ld32(lane_base + kColO + c32, o);
          tmem_wait_ld();
          if (h < p.H) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              *reinterpret_cast<uint4*>(po + c32 + 4 * i) = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
          }
        }
        if (rank == 0 && h < p.H) {
          float* ml = p.part_ml + ((static_cast<int64_t>(seq) * p.splits + sp) * p.H + h) * 2;
          ml[0] = M;
          ml[1] = l;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_ofree);
    }
    if (aborted) record_device_error(DSA_ERR_TIMEOUT);
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer no longer writes into this CTA's shared memory
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

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
