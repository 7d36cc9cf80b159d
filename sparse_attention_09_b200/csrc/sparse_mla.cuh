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
//     selected row (into 128- and 64-byte-swizzled SMEM tiles), and computes the PARTIAL logits
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
// The row sums of P come from the tensor cores too: one more small MMA multiplies P by a tile
// of ones into 16 extra accumulator columns, so they are rescaled together with O_r.
//
// Per CTA: warps 0-7 softmax/epilogue (warps w and w+4 share head rows 32(w%4).. = their TMEM
// lanes; w takes keys 0-31 of each chunk and O columns 0-127, w+4 keys 32-63 and columns
// 128-255), warps 8-9 gather producers, warp 10 MMA issuer and TMEM owner.  The gather uses per-thread cp.async rather
// than TMA gather4: on B200 one gather4 instruction costs 65-130 cycles of the TMA engine, far
// too slow for 64 rows x 576 bytes per 64-key chunk, while a warp-wide cp.async moves one
// row's 512-byte nope segment in a single coalesced instruction.  TMEM columns: O_r [0,256), Q_r [256,400),
// S_r [400,464), P [464,496), row sums [496,512).  SMEM: a 4-stage ring of gathered chunks
// (64 rows x 576 B), a double-buffered exchange area written by the peer, the ones tile.
// The softmax warps run one chunk ahead: they compute and send their factor of chunk c+1
// before they wait for the peer's factor of chunk c, which hides the exchange latency.
//
// The same kernel serves decode: a work item is then (sequence, split of its selection) over
// a paged latent cache, and the unnormalised partial result (O, M, l) goes to a workspace
// that a small kernel merges by log-sum-exp.
//
// And the masked dense mode for short prefill (DENSE): the same attention over the selected
// rows, computed by walking every causal 64-key chunk of the contiguous latent (loaded with
// TMA tiles instead of a gather) and masking the keys the selection does not hold: the mode
// "DeepSeek-V3.2 论文解读" (section 二, subsection "等性能验证") describes for short prefill
// (dense attention with a mask that simulates the sparse pattern).  The selection rows must be ascending (as the top-k emits them).
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

constexpr int kChunk = 64;                         // selected rows per pipeline step
constexpr int kStages = 4;
constexpr int kNopeBlockBytes = kChunk * 128;      // 64 rows x 64 dims bf16, 128-byte swizzle
constexpr int kRopeBlockBytes = kChunk * 64;       // 64 rows x 32 dims bf16, 64-byte swizzle
constexpr int kStageBytes = 4 * kNopeBlockBytes + kRopeBlockBytes;  // 36864
constexpr int kXRowBytes = 144;                    // exchange row: 64 bf16 + m + pad
constexpr int kXBufBytes = 128 * kXRowBytes;
constexpr int kOnesBytes = 16 * 128;               // B tile of ones for the row sums
constexpr int kSmemBytes = kStages * kStageBytes + 4 * kXBufBytes + kOnesBytes;
constexpr uint32_t kColO = 0, kColQ = 256, kColS = 400, kColP = 464, kColL = 496;
constexpr float kTau = 8.f;                        // lazy-rescale margin (log2 units)
constexpr int kPolyPairsOf4 = 1;                   // exponentials by polynomial: this many of every 4 pairs
constexpr uint32_t kXBytesPerChunk = kXBufBytes;  // one bulk copy of the whole row block per chunk

// Named barriers: 1 = all softmax warps (256 threads), 2 + q = the two warps of lane quadrant q.
__device__ __forceinline__ void sm_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }
__device__ __forceinline__ void pair_sync(int q) { asm volatile("bar.sync %0, 64;" ::"r"(2 + q) : "memory"); }

__device__ __forceinline__ bool sm_any(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, 1, 256, q;\n\tselp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v))
      : "memory");
  return r != 0;
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 2^x on the FMA pipe, to take part of the exponentials off the special-function unit:
// Cody-Waite style range reduction x = n + f with n = round(x) (the 1.5*2^23 shifter leaves n in
// the low mantissa bits of t) and |f| <= 1/2, then a cubic for 2^f whose coefficients were fitted
// for least maximum relative error on [-1/2, 1/2] (7.5e-5, far below the bf16 rounding the
// result gets), and n added to the exponent field.  Inputs are clamped at -125 so the exponent
// never underflows; callers pass x <= 8 (the lazy-rescale margin).
__device__ __forceinline__ float exp2_poly(float x) {
  x = fmaxf(x, -125.f);
  const float t = x + 12582912.f;
  const float f = x - (t - 12582912.f);
  float p = fmaf(f, 0.0551716648f, 0.2426111251f);
  p = fmaf(p, f, 0.6932609677f);
  p = fmaf(p, f, 0.9999280572f);
  return __uint_as_float(__float_as_uint(p) + (__float_as_uint(t) << 23));
}

__device__ __forceinline__ uint32_t bf16x2_mul(uint32_t a, uint32_t b) {
  __nv_bfloat162 r = __hmul2(*reinterpret_cast<__nv_bfloat162*>(&a), *reinterpret_cast<__nv_bfloat162*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
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

namespace mla {
// 8 softmax warps (two per TMEM lane quadrant), 2 gather producers, 1 MMA issuer.
constexpr int kSoftmaxWarps = 8;
constexpr int kSoftmaxThreads = 32 * kSoftmaxWarps;
constexpr int kProducerWarps = 2;
constexpr int kFirstProducerWarp = kSoftmaxWarps;
constexpr int kMmaWarp = kSoftmaxWarps + kProducerWarps;
constexpr int kThreads = 32 * (kMmaWarp + 1);
}  // namespace mla

template <bool DECODE, bool DENSE = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(mla::kThreads, 1)
    sparse_mla_kernel(const __nv_bfloat16* __restrict__ latent, const MlaParams p,
                      const __grid_constant__ CUtensorMap nope_map, const __grid_constant__ CUtensorMap rope_map) {
  static_assert(!(DECODE && DENSE), "the dense mode is a prefill mode");
  using namespace dev;
  using namespace mla;
  constexpr uint32_t IDESC_QK = idesc_bf16(128, kChunk, false, false);
  constexpr uint32_t IDESC_PV = idesc_bf16(128, 256, false, true);
  constexpr uint32_t IDESC_L = idesc_bf16(128, 16, false, false);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sKV = smem;                                     // [kStages][kStageBytes]
  uint8_t* sX = smem + kStages * kStageBytes;              // [2][128][kXRowBytes], written by the peer
  uint8_t* sXout = sX + 2 * kXBufBytes;                    // [2][128][kXRowBytes], staged for the peer
  uint8_t* sOnes = sXout + 2 * kXBufBytes;                 // [16][64] bf16 ones (K-major, 1024-aligned)

  __shared__ uint64_t bar_kvfull[kStages], bar_kvempty[kStages];
  __shared__ uint64_t bar_qfull, bar_sfull, bar_sfree, bar_pfull, bar_pvdone, bar_ofree;
  __shared__ uint64_t bar_xfull[2], bar_xempty[2];
  __shared__ uint64_t s_vmask[kStages];                    // valid rows of each staged chunk (32 bits per producer warp)
  __shared__ uint32_t s_tmem;
  __shared__ float s_rmax[2][128];                         // per-half row maxima of the current chunk

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank(), peer = rank ^ 1u;
  const int cid = static_cast<int>(cluster_id_x()), ncl = static_cast<int>(num_clusters_x());
  const int64_t nunits = DECODE ? static_cast<int64_t>(p.B) * p.splits : p.rows;

  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      // every producer thread (plus its copies in flight); dense mode: one arrival + TMA bytes
      mbar_init(&bar_kvfull[i], DENSE ? 1 : 32 * kProducerWarps);
      mbar_init(&bar_kvempty[i], 1);
    }
    mbar_init(&bar_qfull, kSoftmaxThreads);
    mbar_init(&bar_sfull, 1);
    mbar_init(&bar_sfree, kSoftmaxWarps);
    mbar_init(&bar_pfull, kSoftmaxWarps);
    mbar_init(&bar_pvdone, 1);
    mbar_init(&bar_ofree, kSoftmaxWarps);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_xfull[i], 1);     // own arm (expect_tx) + the peer's asynchronous stores
      mbar_init(&bar_xempty[i], 1);    // one remote arrival: the peer has read this CTA's row block
    }
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&s_tmem, 512);
    tmem_relinquish();
  }
  if (tid < kOnesBytes / 16)  // bf16 1.0 everywhere: invariant under the 128-byte swizzle
    *reinterpret_cast<uint4*>(sOnes + 16 * tid) = make_uint4(0x3F803F80u, 0x3F803F80u, 0x3F803F80u, 0x3F803F80u);
  fence_proxy_async_smem();
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
      qrow = u;  // row of q, idx, out and lse
      kbeg = 0;
      kend = p.k;
      // sequence of packed token u + unit0: binary search in cu_seqlens
      const int64_t gtok = u + p.unit0;
      int lo = 0, hi = p.B;
      while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (p.cu_seqlens[mid] <= gtok) lo = mid;
        else hi = mid;
      }
      seq = lo;
      seq_start = p.cu_seqlens[lo];
      seq_len = p.cu_seqlens[lo + 1] - seq_start;
    }
  };
  // chunks [c0, c1) of the selection row this unit processes (dense mode: every causal chunk
  // of the token's sequence prefix)
  auto unit_chunks = [&](int64_t qrow, int kbeg, int kend, int seq_start, int& c0, int& c1) {
    if constexpr (DENSE) {
      c0 = 0;
      c1 = static_cast<int>(qrow + p.unit0 - seq_start) / kChunk + 1;
      return;
    }
    const int act = active_chunks(p.idx + qrow * p.k, p.k);
    c0 = kbeg / kChunk;
    c1 = min(kend / kChunk, act);
    if (c1 <= c0) c1 = c0 + 1;  // always at least one chunk (all masked if empty)
  };

  if (DENSE && warp >= kFirstProducerWarp && warp < kMmaWarp) {
    // ================= dense-mode producer =================
    // Producer warp 0: per chunk, the selection mask of its 64 keys from the (ascending)
    // selection row, then five TMA tiles of the contiguous latent (4 x 64 nope dims with the
    // 128-byte swizzle, 32 rope dims with the 64-byte swizzle) into the stage.
    if (warp == kFirstProducerWarp) {
      uint32_t g = 0;
      bool ok = true;
      if (lane == 0) {
        tma_prefetch_desc(&nope_map);
        tma_prefetch_desc(&rope_map);
      }
      for (int64_t u = cid; ok && u < nunits; u += ncl) {
        int64_t qrow;
        int kbeg, kend, seq, seq_start, seq_len, c0, c1;
        unit_info(u, qrow, kbeg, kend, seq, seq_start, seq_len);
        unit_chunks(qrow, kbeg, kend, seq_start, c0, c1);
        const int t = static_cast<int>(qrow + p.unit0 - seq_start);
        const int32_t* row = p.idx + qrow * p.k;
        int pos = 0;  // entries of the row consumed by earlier chunks
        for (int c = c0; c < c1; ++c, ++g) {
          const int stage = static_cast<int>(g % kStages);
          if (!mbar_wait(&bar_kvempty[stage], ((g / kStages) & 1u) ^ 1u)) {
            record_device_error(DSA_ERR_TIMEOUT);
            ok = false;
            break;
          }
          // the row's entries in [64c, 64c + 64) form one run starting at pos
          uint32_t lo = 0u, hi = 0u;
          while (true) {
            const int v = pos + lane < p.k ? row[pos + lane] : -1;
            const bool in = v >= kChunk * c && v < kChunk * (c + 1) && v <= t;
            const int n = __popc(__ballot_sync(0xffffffffu, in));
            if (in) {
              const int bit = v - kChunk * c;
              if (bit < 32) lo |= 1u << bit;
              else hi |= 1u << (bit - 32);
            }
            pos += n;
            if (n < 32) break;
          }
          lo = __reduce_or_sync(0xffffffffu, lo);
          hi = __reduce_or_sync(0xffffffffu, hi);
          if (lane == 0) {
            s_vmask[stage] = (static_cast<uint64_t>(hi) << 32) | lo;
            uint8_t* st = sKV + stage * kStageBytes;
            const int32_t y = seq_start + kChunk * c;
            mbar_arrive_expect_tx(&bar_kvfull[stage], kStageBytes);
#pragma unroll
            for (int j = 0; j < 4; ++j)
              tma_load_2d(st + j * kNopeBlockBytes, &nope_map, &bar_kvfull[stage], 256 * static_cast<int>(rank) + 64 * j, y);
            tma_load_2d(st + 4 * kNopeBlockBytes, &rope_map, &bar_kvfull[stage], 512 + 32 * static_cast<int>(rank), y);
          }
          __syncwarp();
        }
      }
    }
  } else if (!DENSE && warp >= kFirstProducerWarp && warp < kMmaWarp) {
    // ================= gather producers =================
    // Warp pw copies keys [32 pw, 32 pw + 32) of each 64-key chunk: one warp instruction per key
    // for its 512-byte nope segment (lane l -> 16-byte chunk l, written at its 128-byte-swizzle
    // position), four more for the 64-byte rope halves of the 32 keys (64-byte swizzle).  The
    // stage's barrier completes on its own once the copies have landed (an asynchronous
    // arrival per thread); the MMA warp fences the proxies before the tensor cores read it.
    // (Measured against announcing each stage after cp.async.wait_group, with or without an
    // early flush when the next slot is busy: this is the faster of the two on B200.)
    const int pw = warp - kFirstProducerWarp;
    uint32_t g = 0;
    bool ok = true;
    for (int64_t u = cid; ok && u < nunits; u += ncl) {
      int64_t qrow;
      int kbeg, kend, seq, seq_start, seq_len, c0, c1;
      unit_info(u, qrow, kbeg, kend, seq, seq_start, seq_len);
      unit_chunks(qrow, kbeg, kend, seq_start, c0, c1);
      const int32_t* row = p.idx + qrow * p.k;
      const int32_t* bt = DECODE ? p.block_table + static_cast<int64_t>(seq) * p.max_blocks_per_seq : nullptr;
      // masked rows still copy a real row (never NaN bits): the sequence's first key; in decode
      // the first row of its first block when that block id lies in the pool, else pool row 0
      int pad_row = seq_start;
      if constexpr (DECODE) {
        const int b0 = bt[0];
        pad_row = (b0 >= 0 && b0 < p.num_blocks) ? b0 * 64 : 0;
      }
      for (int c = c0; c < c1; ++c, ++g) {
        const int stage = static_cast<int>(g % kStages);
        if (!mbar_wait(&bar_kvempty[stage], ((g / kStages) & 1u) ^ 1u)) {
          record_device_error(DSA_ERR_TIMEOUT);
          ok = false;
          break;
        }
        const int v = row[c * kChunk + 32 * pw + lane];
        bool valid = v >= 0 && v < seq_len;
        bool bad = !valid && v != -1;  // neither padding nor a position of the sequence
        int prow = pad_row;
        if constexpr (DECODE) {
          const int blk = valid ? bt[v >> 6] : 0;
          const bool blk_ok = blk >= 0 && blk < p.num_blocks;  // a block id outside the pool
          bad = bad || (valid && !blk_ok);
          valid = valid && blk_ok;
          if (valid) prow = blk * 64 + (v & 63);
        } else {
          if (valid) prow = seq_start + v;
        }
        if (bad) record_device_error(DSA_ERR_DEVICE_CHECK);  // the entry is masked
        const uint32_t vbits = __ballot_sync(0xffffffffu, valid);
        if (lane == 0) reinterpret_cast<uint32_t*>(&s_vmask[stage])[pw] = vbits;
        const uint32_t st = smem_addr(sKV + stage * kStageBytes);
#pragma unroll 4
        for (int j = 0; j < 32; ++j) {  // nope: 32 lanes x 16 bytes of one key
          const int r = 32 * pw + j;
          const int kr = __shfl_sync(0xffffffffu, prow, j);
          const __nv_bfloat16* src = latent + static_cast<int64_t>(kr) * 576 + 256 * rank + 8 * lane;
          const int blk = lane >> 3, ch = lane & 7;
          cp_async16(st + blk * kNopeBlockBytes + r * 128 + ((ch ^ (r & 7)) << 4), src);
        }
#pragma unroll
        for (int h2 = 0; h2 < 4; ++h2) {  // rope: 8 keys x 4 chunks of 16 bytes per instruction
          const int j = 8 * h2 + (lane >> 2), ch = lane & 3;
          const int r = 32 * pw + j;
          const int kr = __shfl_sync(0xffffffffu, prow, j);
          const __nv_bfloat16* src = latent + static_cast<int64_t>(kr) * 576 + 512 + 32 * rank + 8 * ch;
          cp_async16(st + 4 * kNopeBlockBytes + r * 64 + ((ch ^ ((r >> 1) & 3)) << 4), src);
        }
        cp_async_commit();
        cp_async_mbar_arrive(&bar_kvfull[stage]);
        mbar_arrive(&bar_kvfull[stage]);  // releases the validity mask written above
      }
    }
    cp_async_wait<0>();
  } else if (warp == kMmaWarp) {
    // ================= MMA issuer =================
    // Two cursors walk the same chunk sequence: Q.K^T of a chunk is issued as soon as its keys
    // are staged and the single S buffer has been read, P.V as soon as P is ready, so the
    // tensor core computes the logits of the next chunk while the softmax warps work.
    struct Cursor {
      int64_t u;
      int c, c0, c1;
      uint32_t g, tok;
      bool valid;
    };
    auto enter_unit = [&](Cursor& cu) {
      cu.valid = cu.u < nunits;
      if (!cu.valid) return;
      int64_t qrow;
      int kbeg, kend, seq, seq_start, seq_len;
      unit_info(cu.u, qrow, kbeg, kend, seq, seq_start, seq_len);
      unit_chunks(qrow, kbeg, kend, seq_start, cu.c0, cu.c1);
      cu.c = cu.c0;
    };
    auto advance = [&](Cursor& cu) {
      ++cu.g;
      if (++cu.c >= cu.c1) {
        cu.u += ncl;
        ++cu.tok;
        enter_unit(cu);
      }
    };
    Cursor qk{cid, 0, 0, 0, 0, 0, false}, pv{cid, 0, 0, 0, 0, 0, false};
    enter_unit(qk);
    enter_unit(pv);
    bool ok = true;
    uint64_t idle_since = 0;
    while (pv.valid) {
      bool did = false;
      if (qk.valid) {
        const int stage = static_cast<int>(qk.g % kStages);
        bool ready = mbar_poll(smem_addr(&bar_kvfull[stage]), (qk.g / kStages) & 1u) &&
                     (qk.g == 0 || mbar_poll(smem_addr(&bar_sfree), (qk.g - 1) & 1u)) &&
                     (qk.c != qk.c0 || mbar_poll(smem_addr(&bar_qfull), qk.tok & 1u));
        ready = __shfl_sync(0xffffffffu, ready, 0);
        if (ready) {
          tc_fence_after();
          if (lane == 0) {
            fence_proxy_async_smem();  // the gathered rows were written through the generic proxy
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
          advance(qk);
          did = true;
        }
      }
      if (pv.g < qk.g) {
        const bool first = pv.c == pv.c0;
        bool ready = mbar_poll(smem_addr(&bar_pfull), pv.g & 1u) &&
                     (!first || pv.tok == 0 || mbar_poll(smem_addr(&bar_ofree), (pv.tok - 1) & 1u));
        ready = __shfl_sync(0xffffffffu, ready, 0);
        if (ready) {
          tc_fence_after();
          if (lane == 0) {
            const uint32_t st = smem_addr(sKV + (pv.g % kStages) * kStageBytes);
#pragma unroll
            for (int kk = 0; kk < kChunk / 16; ++kk)
              umma_bf16_ts(tmem + kColO, tmem + kColP + kk * 8,
                           make_smem_desc(st + kk * 2048, 8192, 1024, kSwizzle128B), IDESC_PV,
                           (first && kk == 0) ? 0u : 1u);
            const uint32_t ones = smem_addr(sOnes);
#pragma unroll
            for (int kk = 0; kk < kChunk / 16; ++kk)  // row sums of P
              umma_bf16_ts(tmem + kColL, tmem + kColP + kk * 8,
                           make_smem_desc(ones + kk * 32, 16, 1024, kSwizzle128B), IDESC_L,
                           (first && kk == 0) ? 0u : 1u);
            umma_commit(&bar_pvdone);
            umma_commit(&bar_kvempty[pv.g % kStages]);
          }
          __syncwarp();
          advance(pv);
          did = true;
        }
      }
      if (did) {
        idle_since = 0;
      } else {
        const uint64_t now = global_timer_ns();
        if (idle_since == 0) idle_since = now;
        else if (now - idle_since > kWaitLimitNs) {
          ok = false;
          break;
        }
      }
    }
    if (!ok && lane == 0) record_device_error(DSA_ERR_TIMEOUT);
  } else {
    // ================= softmax / exchange / epilogue (warps 0-7) =================
    // Warps w and w+4 own the same TMEM lanes (head rows 32(w%4)..+31); warp w takes keys 0-31
    // of every chunk and O columns 0-127, warp w+4 keys 32-63 and O columns 128-255.  The two
    // share the row maximum through shared memory, so both halves use one reference per row.
    const int q4 = warp & 3, hf = warp >> 2;
    const int h = 32 * q4 + lane;  // head row == TMEM lane
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(q4 * 32) << 16);
    const uint32_t x_peer = map_to_rank(smem_addr(sX), peer);
    uint32_t xbar_full_peer[2], xbar_empty_peer[2];
    for (int i = 0; i < 2; ++i) {
      xbar_full_peer[i] = map_to_rank(smem_addr(&bar_xfull[i]), peer);
      xbar_empty_peer[i] = map_to_rank(smem_addr(&bar_xempty[i]), peer);
    }
    // Q rows of this rank's dims into TMEM columns [kColQ, kColQ + 144), in 16-column groups:
    // half 0 stores groups 0-4, half 1 groups 5-8, each in batches of up to three groups whose
    // loads are all in flight together.
    auto load_q = [&](int64_t qrow) {
      const __nv_bfloat16* qr = p.q + (qrow * p.H + h) * 576;
      const bool real = h < p.H;
      const int gbeg = hf == 0 ? 0 : 5, gend = hf == 0 ? 5 : 9;
#pragma unroll 1
      for (int gb = gbeg; gb < gend; gb += 3) {
        uint32_t v[48];
#pragma unroll
        for (int j = 0; j < 12; ++j) {  // 12 x 16 bytes = three groups
          const int col = 16 * gb + 4 * j;  // packed column: dims 2col, 2col+1 of D_r
          const int d = 2 * col < 256 ? 256 * static_cast<int>(rank) + 2 * col
                                      : 512 + 32 * static_cast<int>(rank) + (2 * col - 256);
          uint4 w = make_uint4(0u, 0u, 0u, 0u);
          if (real && gb + j / 4 < gend) w = __ldg(reinterpret_cast<const uint4*>(qr + d));
          v[4 * j] = w.x;
          v[4 * j + 1] = w.y;
          v[4 * j + 2] = w.z;
          v[4 * j + 3] = w.w;
        }
#pragma unroll
        for (int j = 0; j < 3; ++j)
          if (gb + j < gend) tmem_st16(lane_base + kColQ + 16 * (gb + j), *reinterpret_cast<uint32_t(*)[16]>(v + 16 * j));
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
    // Stage A of chunk gg: read this half's partial logits, form this rank's factor
    // P_own = 2^(x*S_r - m_own) as bf16 and send it with m_own to the peer.
    auto stage_a = [&](uint32_t gg, bool last_of_unit, int64_t next_unit, float& m_own, uint32_t(&pown)[16],
                       float& m_sent) -> bool {
      const int stage = static_cast<int>(gg % kStages);
      bool ok = mbar_wait(&bar_sfull, gg & 1u);
      if (sm_any(!ok)) return false;
      tc_fence_after();
      uint32_t sr[32];
      tmem_ld32(lane_base + kColS + 32 * hf, sr);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_sfree);
      if (last_of_unit && next_unit < nunits) {  // the unit's last Q.K^T is done: stage the next Q
        int64_t nq;
        int a, bb, cc, dd, ee;
        unit_info(next_unit, nq, a, bb, cc, dd, ee);
        load_q(nq);
      }
      // the validity mask was written by the producer before it arrived on this stage's barrier;
      // producer warp hf gathered exactly this half's keys
      ok = mbar_wait(&bar_kvfull[stage], (gg / kStages) & 1u);
      if (sm_any(!ok)) return false;
      const uint32_t vmask = reinterpret_cast<const uint32_t*>(&s_vmask[stage])[hf];
      const bool full = vmask == ~0u;
      // row maximum over this half as 8 independent chains, then with the partner half
      float mx[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) mx[j] = -INFINITY;
      if (full) {
#pragma unroll
        for (int i = 0; i < 32; ++i) mx[i & 7] = fmaxf(mx[i & 7], __uint_as_float(sr[i]));
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if ((vmask >> i) & 1u) mx[i & 7] = fmaxf(mx[i & 7], __uint_as_float(sr[i]));
      }
      const float hmax = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      s_rmax[hf][h] = hmax;
      pair_sync(q4);
      const float smax = fmaxf(hmax, s_rmax[hf ^ 1][h]);
      const float cmax = smax * p.scale_log2;  // scale > 0
      if (cmax > m_own + kTau || (m_own == -INFINITY && cmax > -INFINITY)) m_own = cmax;
      const float neg_m = -m_own;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float xa = fmaf(__uint_as_float(sr[2 * i]), p.scale_log2, neg_m);
        const float xb = fmaf(__uint_as_float(sr[2 * i + 1]), p.scale_log2, neg_m);
        float a, bq;
        if ((i & 3) < kPolyPairsOf4) {  // this share of the pairs on the FMA pipe
          a = exp2_poly(xa);
          bq = exp2_poly(xb);
        } else {
          a = ex2_approx(xa);
          bq = ex2_approx(xb);
        }
        if (!full) {
          a = ((vmask >> (2 * i)) & 1u) ? a : 0.f;
          bq = ((vmask >> (2 * i + 1)) & 1u) ? bq : 0.f;
        }
        pown[i] = pack_bf16x2(a, bq);
      }
      // The peer has read the block of chunk gg-2 (so that copy, which read this staging
      // buffer, is complete): stage this half of the row locally and let the TMA engine push
      // the whole block to the peer, keeping the load/store path free.
      const int xb = static_cast<int>(gg & 1u);
      ok = mbar_wait_cluster(&bar_xempty[xb], ((gg >> 1) & 1u) ^ 1u);
      if (sm_any(!ok)) return false;
      uint8_t* row = sXout + xb * kXBufBytes + h * kXRowBytes;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        *reinterpret_cast<uint4*>(row + 64 * hf + 16 * i) =
            make_uint4(pown[4 * i], pown[4 * i + 1], pown[4 * i + 2], pown[4 * i + 3]);
      if (hf == 0) *reinterpret_cast<float*>(row + 128) = m_own;
      fence_proxy_async_smem();
      sm_sync();
      if (tid == 0)
        bulk_copy_to_peer(x_peer + xb * kXBufBytes, sXout + xb * kXBufBytes, kXBufBytes, xbar_full_peer[xb]);
      m_sent = m_own;
      return true;
    };
    // Stage B of chunk gg: receive the peer's factor, form P = P_own * P_peer relative to
    // M = m_own + m_peer (identical in both ranks and both halves), rescale this half's O
    // columns (and the row sums) if M moved, and hand this half of P to the tensor cores.
    auto stage_b = [&](uint32_t gg, bool first_of_unit, const uint32_t(&pown)[16], float m_sent, float& M) -> bool {
      const int xb = static_cast<int>(gg & 1u);
      if (tid == 0) mbar_arrive_expect_tx(&bar_xfull[xb], kXBytesPerChunk);  // may land before or after the data
      bool ok = mbar_wait_cluster(&bar_xfull[xb], (gg >> 1) & 1u);
      if (sm_any(!ok)) return false;
      const uint8_t* src = sX + xb * kXBufBytes + h * kXRowBytes;
      uint32_t pp[16];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 w = *reinterpret_cast<const uint4*>(src + 64 * hf + 16 * i);
        pp[4 * i] = bf16x2_mul(pown[4 * i], w.x);
        pp[4 * i + 1] = bf16x2_mul(pown[4 * i + 1], w.y);
        pp[4 * i + 2] = bf16x2_mul(pown[4 * i + 2], w.z);
        pp[4 * i + 3] = bf16x2_mul(pown[4 * i + 3], w.w);
      }
      const float m_peer = *reinterpret_cast<const float*>(src + 128);
      const float Mn = m_sent + m_peer;
      if (gg > 0) {  // the previous P.V must be done before P is overwritten or O rescaled
        ok = mbar_wait(&bar_pvdone, (gg - 1) & 1u);
        if (sm_any(!ok)) return false;
        tc_fence_after();
      } else {
        sm_sync();
      }
      // every thread has read its part of the peer's block (the barrier above): release it.
      // (Not thread 0: its cluster-scope release would also wait for the bulk copy it issued.)
      if (tid == 32) mbar_arrive_remote(xbar_empty_peer[xb]);
      // tcgen05.ld/st are warp-collective: the whole warp runs the rescale if any row needs it
      const bool need_rescale = !first_of_unit && Mn != M && M > -INFINITY;
      if (__any_sync(0xffffffffu, need_rescale)) {
        const float alpha = need_rescale ? exp2f(M - Mn) : 1.f;
#pragma unroll 1
        for (int c32 = 0; c32 < 128; c32 += 32) {
          uint32_t o[32];
          tmem_ld32(lane_base + kColO + 128 * hf + c32, o);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(lane_base + kColO + 128 * hf + c32, o);
        }
        if (hf == 0) {
          uint32_t lv[16];
          tmem_ld16(lane_base + kColL, lv);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 16; ++i) lv[i] = __float_as_uint(__uint_as_float(lv[i]) * alpha);
          tmem_st16(lane_base + kColL, lv);
        }
      }
      M = Mn;
      tmem_st16(lane_base + kColP + 16 * hf, pp);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_pfull);
      return true;
    };

    for (int64_t u = cid; u < nunits; u += ncl, ++tok) {
      int64_t qrow;
      int kbeg, kend, seq, seq_start, seq_len, c0, c1;
      unit_info(u, qrow, kbeg, kend, seq, seq_start, seq_len);
      unit_chunks(qrow, kbeg, kend, seq_start, c0, c1);
      if (u + ncl < nunits && h < p.H) {  // warm L2 with the next unit's Q row (loaded near this unit's end)
        int64_t nq;
        int a, bb, cc, dd, ee;
        unit_info(u + ncl, nq, a, bb, cc, dd, ee);
        const char* qn = reinterpret_cast<const char*>(p.q + (nq * p.H + h) * 576);
        if (hf == 0) {
#pragma unroll
          for (int i = 0; i < 4; ++i) prefetch_l2(qn + 512 * rank + 128 * i);
        } else {
          prefetch_l2(qn + 1024 + 64 * rank);
        }
      }
      float m_own = -INFINITY, M = -INFINITY, m_cur = -INFINITY, m_next = -INFINITY;
      uint32_t p_cur[16], p_next[16];
      if (!stage_a(g, c0 == c1 - 1, u + ncl, m_own, p_cur, m_cur)) {
        aborted = true;
        break;
      }
      for (int c = c0; c < c1; ++c, ++g) {
        if (c + 1 < c1 && !stage_a(g + 1, c + 1 == c1 - 1, u + ncl, m_own, p_next, m_next)) {
          aborted = true;
          break;
        }
        if (!stage_b(g, c == c0, p_cur, m_cur, M)) {
          aborted = true;
          break;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) p_cur[i] = p_next[i];
        m_cur = m_next;
      }
      if (aborted) break;
      // epilogue of the unit: this half's O columns / l
      bool ok = mbar_wait(&bar_pvdone, (g - 1) & 1u);
      if (sm_any(!ok)) {
        aborted = true;
        break;
      }
      tc_fence_after();
      uint32_t lv[16];
      tmem_ld16(lane_base + kColL, lv);
      tmem_wait_ld();
      const float l = __uint_as_float(lv[0]);
      const float inv_l = l > 0.f ? 1.f / l : 0.f;
      if constexpr (!DECODE) {
        __nv_bfloat16* orow = p.out + (qrow * p.H + h) * 512 + 256 * rank + 128 * hf;
#pragma unroll 1
        for (int c32 = 0; c32 < 128; c32 += 32) {
          uint32_t o[32];
          tmem_ld32(lane_base + kColO + 128 * hf + c32, o);
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
        if (rank == 0 && hf == 0 && p.lse != nullptr && h < p.H)
          p.lse[qrow * p.H + h] = l > 0.f ? (M + log2f(l)) * 0.69314718055994531f : -INFINITY;
      } else {
        const int sp = static_cast<int>(u % p.splits);
        float* po = p.part_o + ((static_cast<int64_t>(seq) * p.splits + sp) * p.H + h) * 512 + 256 * rank + 128 * hf;
#pragma unroll 1
        for (int c32 = 0; c32 < 128; c32 += 32) {
          uint32_t o[32];
          tmem_ld32(lane_base + kColO + 128 * hf + c32, o);
          tmem_wait_ld();
          if (h < p.H) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              *reinterpret_cast<uint4*>(po + c32 + 4 * i) = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
          }
        }
        if (rank == 0 && hf == 0 && h < p.H) {
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
  if (warp == kMmaWarp) {
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
