// Sparse MLA in MQA mode on a CTA pair that splits the HEADS (tcgen05 cta_group::2).
//
// For a query token t with selected latent rows c_i (i over the top-k selection):
//   out[t,h,:] = sum_i softmax_i(sm_scale * q[t,h,:] . c_i) * c_i[0:512]
// ("DeepSeek-V3.2 论文解读", section 二, subsection "挂在 MLA 上": every head of the token shares the
// same 576-d latent rows, MQA mode).  One token is a [128 heads x 576] x [576 x k] product followed
// by a [128 x k] x [k x 512] product.
//
// Split over the pair (rank r = 0, 1): CTA r owns heads [64r, 64r + 64).  Both products are
// issued once, from CTA 0, as pair MMAs with M = 128 (64 rows per CTA):
//   * logits  S = Q . K^T: A = this CTA's 64 query rows (all 576 dims, SMEM), B = the chunk's 64
//     selected rows split by N: CTA r stages its "own" 32 rows [32r, 32r + 32) with all 576 dims.
//     Each CTA's TMEM receives its 64 heads x 64 keys, keys 0-31 on lanes 0-63 and keys 32-63 on
//     lanes 64-127 (32 columns).
//   * output  O += P . V: A = this CTA's P (64 heads x 64 keys, bf16, SMEM), B = V split by N:
//     for each of the two N = 256 halves of the 512 value dims, CTA r stages dims
//     [256m + 128r, 256m + 128r + 128) of all 64 rows.  Each CTA's TMEM receives its 64 heads x
//     512 dims in 256 columns.
// The softmax of a head needs no data of the other CTA, so nothing is exchanged between the
// CTAs but barrier arrivals: the only cross-CTA dependencies are "both halves of the operands are
// staged" before an MMA and "both CTAs have read S / written P / read O" before the next MMA that
// overwrites them.
//
// Per CTA (11 warps; warp w issues on scheduler w % 4):
//   warps 0-3  softmax and epilogue.  Warp w reads TMEM lanes 32w..32w+31: warps 0 and 1 hold
//              keys 0-31 of heads 0-63, warps 2 and 3 keys 32-63 of the same heads; partners w
//              and w^2 share the row maximum and the row sum through SMEM;
//   warps 4-5  gather the own rows, warps 8-9 the value dims of all 64 rows (cp.async,
//              coalesced, into 128-byte-swizzled tiles; separate warps so the two rings refill
//              independently);
//   warp 6     loads Q by TMA;
//   warp 7     issues Q.K^T (CTA 0) or forwards CTA 1's "operands staged" signals (CTA 1);
//   warp 10    issues P.V (CTA 0).
// TMEM columns: O [0, 256), S double-buffered [256, 320).  SMEM: Q 72 KB, P 2 x 8 KB, own-row
// ring 2 x 36 KB, value ring 2 x 32 KB.  The value ring repeats the own rows' value dims (16 KB of
// the 32 KB) because the pair MMA reads both CTAs' B halves at one SMEM offset.
//
// What the measurements on B200 decided (prefill, L = 8192, k = 2048):
//   * MMAs are issued warp-collectively (one elected lane) with descriptors advanced by
//     addition: issued from a one-lane branch, an M = 128, N = 64 pair MMA cost 45 cycles
//     against 25 (the shared-memory operand rate);
//   * signals between the CTAs are CTA-scope barrier arrivals: cluster-scope release/acquire on
//     every signal added about 1K cycles per hand-off (527 -> 554 TFLOP/s; with the issue form
//     above 719);
//   * two issuing warps, one per product: with one, the warp issuing 44 MMAs per chunk was the
//     bottleneck (747 -> 828 TFLOP/s);
//   * Q stays in SMEM: holding 128 or 384 of its dims in tensor memory (loaded by tcgen05.cp)
//     made Q.K^T slower in the kernel (769 / 696 TFLOP/s), as did a third S buffer (823), eight
//     softmax warps, an index ring and a fixed issue order of the two products.
//
// The same kernel serves decode: a work item is then (sequence, split of its selection) over a
// paged latent cache.  A split selection's unnormalised partial results (O, M, l) go to a
// workspace that a small kernel merges by log-sum-exp; an unsplit one is written as out / lse
// directly, as in prefill.
//
// And the masked dense mode for short prefill (MASKED): the attention a dense MHA kernel gives
// under a mask that simulates the sparse pattern ("DeepSeek-V3.2 论文解读", section 二,
// subsection "等性能验证").  Chunk c of token t is then the 64 contiguous latent rows
// [64c, 64c + 64) of its sequence, for every c up to t / 64, and the keys that the (ascending)
// selection row does not hold, or that lie past t, are masked in the softmax.  The gather warps
// read no selection entries; each softmax warp walks the selection row with a cursor (the
// entries of chunk c are one run of at most 64 starting where chunk c - 1's run ended) and
// loads the next run while it works on the current chunk.
#pragma once

#include "common.cuh"
#include "mla_common.cuh"
#include "sm100.cuh"

namespace dsa {
namespace mlap {

constexpr int kChunk = 64;                          // selected rows per pipeline step
constexpr int kHeads = 64;                          // heads per CTA
constexpr int kQBlockBytes = kHeads * 128;          // 64 rows x 64 dims bf16, 128-byte swizzle
constexpr int kQBytes = 9 * kQBlockBytes;           // 576 dims
constexpr int kPBytes = kHeads * 128;               // 64 heads x 64 keys bf16
constexpr int kKQBlockBytes = 32 * 128;             // 32 own rows x 64 dims
constexpr int kKQBytes = 9 * kKQBlockBytes;         // 576 dims
constexpr int kVBlockBytes = kChunk * 128;          // 64 rows x 64 dims
constexpr int kVBytes = 4 * kVBlockBytes;           // 256 value dims
constexpr int kOffQ = 0;
constexpr int kOffP = kOffQ + kQBytes;
constexpr int kOffKQ = kOffP + 2 * kPBytes;
constexpr int kOffV = kOffKQ + 2 * kKQBytes;
constexpr int kSmemBytes = kOffV + 2 * kVBytes;     // 229376
constexpr uint32_t kColO = 0, kColS = 256;
constexpr int kSoftmaxWarps = 4;
constexpr int kProducerWarps = 2;      // per ring
constexpr int kFirstProducerWarp = 4;  // own rows: warps 4, 5
constexpr int kQWarp = 6;
constexpr int kMmaWarp = 7;            // Q.K^T issuer (CTA 0) / relay (CTA 1); owns the TMEM allocation
constexpr int kVWarp0 = 8;             // value rows: warps 8, 9
constexpr int kPvWarp = 10;            // P.V issuer (CTA 0)
constexpr int kThreads = 352;
constexpr float kTau = 8.f;                         // lazy-rescale margin (log2 units)

static_assert(kOffP % 1024 == 0 && kOffKQ % 1024 == 0 && kOffV % 1024 == 0, "swizzled tiles are 1024-aligned");

// Warps w and w^2 (same head rows, the two key halves) meet at named barrier 1 + (w & 1).
__device__ __forceinline__ void pair_sync(int w) { asm volatile("bar.sync %0, 64;" ::"r"(1 + (w & 1)) : "memory"); }
__device__ __forceinline__ bool pair_any(int w, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 q, %1, 0;\n\t"
      "bar.red.or.pred p, %2, 64, q;\n\tselp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(1 + (w & 1))
      : "memory");
  return r != 0;
}

// A work item: which rows of q / idx / out it uses, its sequence and its 64-entry chunks [c0, c1).
struct Unit {
  int64_t qrow;
  int seq, seq_start, seq_len, sp, c0, c1;
};

// Warp-collective (scans the selection row).  Masked mode: every causal chunk of the token.
template <bool DECODE, bool MASKED>
__device__ __forceinline__ Unit unit_of(const MlaParams& p, int64_t u) {
  Unit r;
  int kbeg, kend;
  if constexpr (DECODE) {
    r.seq = static_cast<int>(u / p.splits);
    r.sp = static_cast<int>(u % p.splits);
    const int per = p.k / p.splits;
    r.qrow = r.seq;
    kbeg = r.sp * per;
    kend = kbeg + per;
    r.seq_start = 0;
    r.seq_len = min(p.context_lens[r.seq], p.max_blocks_per_seq * 64);
  } else {
    r.qrow = u;
    r.sp = 0;
    kbeg = 0;
    kend = p.k;
    const int64_t gtok = u + p.unit0;  // packed token: binary search in cu_seqlens
    int lo = 0, hi = p.B;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (p.cu_seqlens[mid] <= gtok) lo = mid;
      else hi = mid;
    }
    r.seq = lo;
    r.seq_start = p.cu_seqlens[lo];
    r.seq_len = p.cu_seqlens[lo + 1] - r.seq_start;
  }
  if constexpr (MASKED) {
    r.c0 = 0;
    r.c1 = static_cast<int>(u + p.unit0 - r.seq_start) / kChunk + 1;
    return r;
  }
  const int act = mla::active_chunks(p.idx + r.qrow * p.k, p.k);
  r.c0 = kbeg / kChunk;
  r.c1 = min(kend / kChunk, act);
  if (r.c1 <= r.c0) r.c1 = r.c0 + 1;  // at least one chunk (all masked if empty)
  return r;
}

// Whether selection entry v of a unit names a row of its sequence, and that row of the latent
// array.  `bad` = neither the padding value -1 nor a usable position (or a block id outside the
// pool): such entries are masked and reported.  Producers and softmax use this same predicate.
template <bool DECODE>
__device__ __forceinline__ bool key_of(const MlaParams& p, const int32_t* bt, int v, const Unit& un, int& prow,
                                       bool& bad) {
  bool valid = v >= 0 && v < un.seq_len;
  bad = !valid && v != -1;
  if constexpr (DECODE) {
    const int blk = valid ? bt[v >> 6] : 0;
    const bool blk_ok = blk >= 0 && blk < p.num_blocks;
    bad = bad || (valid && !blk_ok);
    valid = valid && blk_ok;
    if (valid) prow = blk * 64 + (v & 63);
  } else {
    if (valid) prow = un.seq_start + v;
  }
  return valid;
}

}  // namespace mlap

template <bool DECODE, bool MASKED = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(mlap::kThreads, 1)
    sparse_mla_pair_kernel(const __nv_bfloat16* __restrict__ latent, const MlaParams p,
                           const __grid_constant__ CUtensorMap q_map) {
  using namespace dev;
  using namespace mlap;
  constexpr uint32_t IDESC_QK = idesc_bf16(128, kChunk, false, false);
  constexpr uint32_t IDESC_PV = idesc_bf16(128, 256, false, true);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = smem + kOffQ;
  uint8_t* sP = smem + kOffP;
  uint8_t* sKQ = smem + kOffKQ;
  uint8_t* sV = smem + kOffV;

  // local to each CTA
  __shared__ uint64_t bar_kq_full[2], bar_v_full[2];     // this CTA's rows of a slot have landed
  __shared__ uint64_t bar_kq_empty[2], bar_v_empty[2];   // the MMAs reading a slot are done
  __shared__ uint64_t bar_q_full, bar_q_empty;           // Q staged / the unit's last Q.K^T done
  __shared__ uint64_t bar_s_full[2], bar_pv_done[2];     // S of a slot written / P.V of a P slot done
  __shared__ uint64_t bar_mma_done;                      // every MMA of the kernel has completed
  // used in CTA 0 only: arrivals from both CTAs
  __shared__ uint64_t bar_s_free[2], bar_p_full[2], bar_o_free;
  __shared__ uint64_t bar_kq_peer[2], bar_v_peer[2], bar_q_peer;  // CTA 1's operands staged
  __shared__ uint32_t s_tmem;
  __shared__ float s_red[3][2][kHeads];                  // [buffer][key half][head] maxima / sums

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t rank = cluster_ctarank();
  const int cid = static_cast<int>(cluster_id_x()), ncl = static_cast<int>(num_clusters_x());
  const int64_t nunits = DECODE ? static_cast<int64_t>(p.B) * p.splits : p.rows;

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      // every producer thread (plus its copies in flight)
      mbar_init(&bar_kq_full[i], 32 * kProducerWarps);
      mbar_init(&bar_v_full[i], 32 * kProducerWarps);
      mbar_init(&bar_kq_empty[i], 1);
      mbar_init(&bar_v_empty[i], 1);
      mbar_init(&bar_s_full[i], 1);
      mbar_init(&bar_pv_done[i], 1);
      mbar_init(&bar_s_free[i], 2 * kSoftmaxWarps);
      mbar_init(&bar_p_full[i], 2 * kSoftmaxWarps);
      mbar_init(&bar_kq_peer[i], 1);
      mbar_init(&bar_v_peer[i], 1);
    }
    mbar_init(&bar_q_full, 1);
    mbar_init(&bar_q_empty, 1);
    mbar_init(&bar_mma_done, 2);
    mbar_init(&bar_o_free, 2 * kSoftmaxWarps);
    mbar_init(&bar_q_peer, 1);
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc_pair(&s_tmem, 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers are initialised before any remote arrival
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  auto at_leader = [](uint64_t* bar) { return map_to_rank(smem_addr(bar), 0u); };

  if ((warp >= kFirstProducerWarp && warp < kFirstProducerWarp + kProducerWarps) || (warp >= kVWarp0 && warp < kVWarp0 + 2)) {
    const bool kqrole = warp < kVWarp0;
    // ================= gather producers =================
    // Own-row warps (4, 5): per chunk, this CTA's own 32 rows with all 576 dims (warp pw: rows
    // 16pw..16pw+15 of them, two warp instructions of 512 bytes per row plus the 128-byte rope
    // segments of four rows per instruction).  Value warps (8, 9): all 64 rows' value dims of this
    // CTA (warp pw: rows 32pw..32pw+31, one instruction per row covering its two 256-byte
    // segments).  Each ring slot's barrier completes on its own once the copies have landed.
    const int pw = kqrole ? warp - kFirstProducerWarp : warp - kVWarp0;
    uint32_t g = 0;
    bool ok = true;
    for (int64_t u = cid; ok && u < nunits; u += ncl) {
      const Unit un = unit_of<DECODE, MASKED>(p, u);
      const int32_t* row = p.idx + un.qrow * p.k;
      const int32_t* bt = DECODE ? p.block_table + static_cast<int64_t>(un.seq) * p.max_blocks_per_seq : nullptr;
      // masked entries still copy a real row (never NaN bits): the sequence's first key; in
      // decode the first row of its first block when that block id lies in the pool, else row 0
      int pad_row = un.seq_start;
      if constexpr (DECODE) {
        const int b0 = bt[0];
        pad_row = (b0 >= 0 && b0 < p.num_blocks) ? b0 * 64 : 0;
      }
      for (int c = un.c0; c < un.c1; ++c, ++g) {
        const int s = static_cast<int>(g & 1u);
        if (kqrole) {
          // ---- own rows, all dims (B of Q.K^T) ----
          if (!mbar_wait(&bar_kq_empty[s], ((g >> 1) & 1u) ^ 1u)) {
            ok = false;
            break;
          }
          int prow = pad_row;
          bool bad;
          const int e = c * kChunk + 32 * static_cast<int>(rank) + 16 * pw + (lane & 15);
          key_of<DECODE>(p, bt, MASKED ? e : row[e], un, prow, bad);
          if (!MASKED && bad && lane < 16) record_device_error(DSA_ERR_DEVICE_CHECK);  // the entry is masked
          const uint32_t kq = smem_addr(sKQ + s * kKQBytes);
#pragma unroll 4
          for (int j = 0; j < 16; ++j) {
            const int r = 16 * pw + j;
            const int kr = __shfl_sync(0xffffffffu, prow, j);
            const __nv_bfloat16* src = latent + static_cast<int64_t>(kr) * 576 + 8 * lane;
            const uint32_t off = r * 128 + (((lane & 7) ^ (r & 7)) << 4);
            cp_async16(kq + (lane >> 3) * kKQBlockBytes + off, src);
            cp_async16(kq + (4 + (lane >> 3)) * kKQBlockBytes + off, src + 256);
          }
#pragma unroll
          for (int i = 0; i < 4; ++i) {  // rope dims 512-575: four rows per instruction
            const int j = 4 * i + (lane >> 3), ch = lane & 7;
            const int r = 16 * pw + j;
            const int kr = __shfl_sync(0xffffffffu, prow, j);
            cp_async16(kq + 8 * kKQBlockBytes + r * 128 + ((ch ^ (r & 7)) << 4),
                       latent + static_cast<int64_t>(kr) * 576 + 512 + 8 * ch);
          }
          cp_async_commit();
          cp_async_mbar_arrive(&bar_kq_full[s]);
          mbar_arrive(&bar_kq_full[s]);
        } else {
          // ---- all rows, this CTA's value dims (B of P.V) ----
          if (!mbar_wait(&bar_v_empty[s], ((g >> 1) & 1u) ^ 1u)) {
            ok = false;
            break;
          }
          int prow = pad_row;
          bool bad;
          const int e = c * kChunk + 32 * pw + lane;
          key_of<DECODE>(p, bt, MASKED ? e : row[e], un, prow, bad);
          const uint32_t vb = smem_addr(sV + s * kVBytes);
          const int seg = lane >> 4, pc = lane & 15;  // segment m: dims 256m + 128 rank + 8 pc
          const int blk = 2 * seg + (pc >> 3), ch = pc & 7;
#pragma unroll 4
          for (int j = 0; j < 32; ++j) {
            const int n = 32 * pw + j;
            const int kr = __shfl_sync(0xffffffffu, prow, j);
            cp_async16(vb + blk * kVBlockBytes + n * 128 + ((ch ^ (n & 7)) << 4),
                       latent + static_cast<int64_t>(kr) * 576 + 256 * seg + 128 * static_cast<int>(rank) + 8 * pc);
          }
          cp_async_commit();
          cp_async_mbar_arrive(&bar_v_full[s]);
          mbar_arrive(&bar_v_full[s]);
        }
      }
    }
    cp_async_wait<0>();
    if (!ok) record_device_error(DSA_ERR_TIMEOUT);
  } else if (warp == kQWarp) {
    // ================= Q loader: this CTA's 64 query rows of each unit, nine TMA tiles =================
    uint32_t tok = 0;
    bool ok = true;
    if (lane == 0) tma_prefetch_desc(&q_map);
    for (int64_t u = cid; ok && u < nunits; u += ncl, ++tok) {
      const int64_t qrow = DECODE ? u / p.splits : u;
      if (lane == 0) {
        ok = mbar_wait(&bar_q_empty, (tok & 1u) ^ 1u);
        if (ok) {
          mbar_arrive_expect_tx(&bar_q_full, kQBytes);
          const int32_t y = static_cast<int32_t>(qrow * p.H + kHeads * static_cast<int64_t>(rank));
#pragma unroll
          for (int b = 0; b < 9; ++b) tma_load_2d(sQ + b * kQBlockBytes, &q_map, &bar_q_full, 64 * b, y);
        }
      }
      ok = __shfl_sync(0xffffffffu, ok, 0);
    }
    // the last load must have landed before the CTA may exit
    if (lane == 0 && ok && tok > 0 && !mbar_wait(&bar_q_full, (tok - 1) & 1u)) ok = false;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok && lane == 0) record_device_error(DSA_ERR_TIMEOUT);
  } else if (warp == kMmaWarp || warp == kPvWarp) {
    struct Cursor {
      int64_t u;
      int c, c0, c1;
      uint32_t g, tok;
      bool valid;
    };
    auto enter_unit = [&](Cursor& cu) {
      cu.valid = cu.u < nunits;
      if (!cu.valid) return;
      const Unit un = unit_of<DECODE, MASKED>(p, cu.u);
      cu.c0 = un.c0;
      cu.c1 = un.c1;
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
    bool ok = true;
    uint64_t idle_since = 0;
    if (rank == 0 && warp == kMmaWarp) {
      // ================= Q.K^T issuer (CTA 0, for the pair) =================
      Cursor qk{cid, 0, 0, 0, 0, 0, false};
      enter_unit(qk);
      while (qk.valid) {
        bool did = false;
        const int s = static_cast<int>(qk.g & 1u);
        const uint32_t par = (qk.g >> 1) & 1u;
        bool ready = mbar_poll(smem_addr(&bar_kq_full[s]), par) && mbar_poll(smem_addr(&bar_kq_peer[s]), par) &&
                     (qk.g < 2 || mbar_poll(smem_addr(&bar_s_free[s]), par ^ 1u)) &&
                     (qk.c != qk.c0 || (mbar_poll(smem_addr(&bar_q_full), qk.tok & 1u) &&
                                        mbar_poll(smem_addr(&bar_q_peer), qk.tok & 1u)));
        ready = __shfl_sync(0xffffffffu, ready, 0);
        if (ready) {
          tc_fence_after();
          if (lane == 0) fence_proxy_async_smem();  // the gathered rows were written through the generic proxy
          __syncwarp();
          const uint64_t ad = make_smem_desc(smem_addr(sQ), 16, 1024, kSwizzle128B);
          const uint64_t bd = make_smem_desc(smem_addr(sKQ + s * kKQBytes), 16, 1024, kSwizzle128B);
#pragma unroll
          for (int kk = 0; kk < 36; ++kk)
            umma_bf16_ss_pair_warp(tmem + kColS + 32 * s, ad + (((kk >> 2) * kQBlockBytes + (kk & 3) * 32) >> 4),
                                   bd + (((kk >> 2) * kKQBlockBytes + (kk & 3) * 32) >> 4), IDESC_QK, kk > 0 ? 1u : 0u);
          if (lane == 0) {
            umma_commit_pair(&bar_s_full[s], 3);
            umma_commit_pair(&bar_kq_empty[s], 3);
            if (qk.c == qk.c1 - 1) umma_commit_pair(&bar_q_empty, 3);
          }
          __syncwarp();
          advance(qk);
          did = true;
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
      if (lane == 0) umma_commit_pair(&bar_mma_done, 3);
      __syncwarp();
    } else if (rank == 0) {
      // ================= P.V issuer (CTA 0, for the pair) =================
      Cursor pv{cid, 0, 0, 0, 0, 0, false};
      enter_unit(pv);
      while (pv.valid) {
        bool did = false;
        const int s = static_cast<int>(pv.g & 1u);
        const uint32_t par = (pv.g >> 1) & 1u;
        const bool first = pv.c == pv.c0;
        bool ready = mbar_poll(smem_addr(&bar_p_full[s]), par) && mbar_poll(smem_addr(&bar_v_full[s]), par) &&
                     mbar_poll(smem_addr(&bar_v_peer[s]), par) &&
                     (!first || pv.tok == 0 || mbar_poll(smem_addr(&bar_o_free), (pv.tok - 1) & 1u));
        ready = __shfl_sync(0xffffffffu, ready, 0);
        if (ready) {
          tc_fence_after();
          if (lane == 0) fence_proxy_async_smem();  // P (st.shared) and the value rows (cp.async): generic proxy
          __syncwarp();
          const uint64_t ad = make_smem_desc(smem_addr(sP + s * kPBytes), 16, 1024, kSwizzle128B);
          const uint64_t bd = make_smem_desc(smem_addr(sV + s * kVBytes), kVBlockBytes, 1024, kSwizzle128B);
#pragma unroll
          for (int m = 0; m < 2; ++m)
#pragma unroll
            for (int kk = 0; kk < kChunk / 16; ++kk)
              umma_bf16_ss_pair_warp(tmem + kColO + 128 * m, ad + ((kk * 32) >> 4),
                                     bd + ((2 * m * kVBlockBytes + kk * 2048) >> 4), IDESC_PV, (first && kk == 0) ? 0u : 1u);
          if (lane == 0) {
            umma_commit_pair(&bar_pv_done[s], 3);
            umma_commit_pair(&bar_v_empty[s], 3);
          }
          __syncwarp();
          advance(pv);
          did = true;
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
      if (lane == 0) umma_commit_pair(&bar_mma_done, 3);
      __syncwarp();
    } else if (warp == kPvWarp) {
      // CTA 1 issues nothing: this warp only waits for the final commit below
    } else {
      // ================= relay (CTA 1): "this CTA's operands are staged" -> CTA 0 =================
      Cursor kq{cid, 0, 0, 0, 0, 0, false}, vc{cid, 0, 0, 0, 0, 0, false};
      enter_unit(kq);
      enter_unit(vc);
      int64_t uq = cid;
      uint32_t tq = 0;
      const uint32_t q_peer = at_leader(&bar_q_peer);
      while (kq.valid || vc.valid || uq < nunits) {
        bool did = false;
        if (uq < nunits) {
          bool ready = __shfl_sync(0xffffffffu, mbar_poll(smem_addr(&bar_q_full), tq & 1u), 0);
          if (ready) {
            if (lane == 0) mbar_arrive_peer(q_peer);
            uq += ncl;
            ++tq;
            did = true;
          }
        }
        if (kq.valid) {
          const int s = static_cast<int>(kq.g & 1u);
          bool ready = __shfl_sync(0xffffffffu, mbar_poll(smem_addr(&bar_kq_full[s]), (kq.g >> 1) & 1u), 0);
          if (ready) {
            if (lane == 0) {
              fence_proxy_async_smem();
              mbar_arrive_peer(at_leader(&bar_kq_peer[s]));
            }
            __syncwarp();
            advance(kq);
            did = true;
          }
        }
        if (vc.valid) {
          const int s = static_cast<int>(vc.g & 1u);
          bool ready = __shfl_sync(0xffffffffu, mbar_poll(smem_addr(&bar_v_full[s]), (vc.g >> 1) & 1u), 0);
          if (ready) {
            if (lane == 0) {
              fence_proxy_async_smem();
              mbar_arrive_peer(at_leader(&bar_v_peer[s]));
            }
            __syncwarp();
            advance(vc);
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
    }
    // both CTAs: wait for CTA 0's final commit (every MMA writing this CTA's TMEM has completed)
    if (lane == 0 && !mbar_wait(&bar_mma_done, 0)) ok = false;
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (!ok && lane == 0) record_device_error(DSA_ERR_TIMEOUT);
  } else {
    // ================= softmax / epilogue (warps 0-3) =================
    const int w = warp, kh = w >> 1;          // key half of each chunk this warp holds
    const int hl = 32 * (w & 1) + lane;       // head row within the CTA (TMEM lane 32w + lane)
    const int h = kHeads * static_cast<int>(rank) + hl;
    const bool real = h < p.H;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(32 * w) << 16);
    uint32_t s_free_l[2], p_full_l[2];
    for (int i = 0; i < 2; ++i) {
      s_free_l[i] = at_leader(&bar_s_free[i]);
      p_full_l[i] = at_leader(&bar_p_full[i]);
    }
    const uint32_t o_free_l = at_leader(&bar_o_free);
    // a bounded wait whose outcome both warps of the pair share, so that they leave together
    auto pair_wait = [&](uint64_t* bar, uint32_t parity) -> bool {
      const bool ok = mbar_wait(bar, parity);
      return !pair_any(w, !ok);
    };
    uint32_t g = 0;
    bool aborted = false;
    for (int64_t u = cid; !aborted && u < nunits; u += ncl) {
      const Unit un = unit_of<DECODE, MASKED>(p, u);
      const int32_t* row = p.idx + un.qrow * p.k;
      const int32_t* bt = DECODE ? p.block_table + static_cast<int64_t>(un.seq) * p.max_blocks_per_seq : nullptr;
      float m = -INFINITY, l = 0.f;
      // masked mode: the token's position, the selection cursor and the 64 entries from it
      const int t = MASKED ? static_cast<int>(u + p.unit0 - un.seq_start) : 0;
      int cur = 0, va = -1, vb = -1;
      if constexpr (MASKED) {
        va = row[lane];
        vb = row[32 + lane];
      }
      for (int c = un.c0; c < un.c1; ++c, ++g) {
        const int s = static_cast<int>(g & 1u);
        uint32_t vmask;
        if constexpr (MASKED) {
          // chunk c's entries are the run [cur, cur + n) of entries below 64c + 64 (at most 64
          // when the row is ascending and distinct); this warp keeps those of its key half that
          // lie in the causal prefix, then loads the 64 entries after the run
          const int lo = c * kChunk, half = lo + 32 * kh;
          const bool ina = va >= 0 && va < lo + kChunk, inb = vb >= 0 && vb < lo + kChunk;
          const int n = __popc(__ballot_sync(0xffffffffu, ina)) + __popc(__ballot_sync(0xffffffffu, inb));
          uint32_t bits = 0u;
          if (ina && va >= half && va < half + 32 && va <= t) bits |= 1u << (va - half);
          if (inb && vb >= half && vb < half + 32 && vb <= t) bits |= 1u << (vb - half);
          vmask = __reduce_or_sync(0xffffffffu, bits);
          cur += n;
          va = cur + lane < p.k ? row[cur + lane] : -1;
          vb = cur + 32 + lane < p.k ? row[cur + 32 + lane] : -1;
        } else {
          int prow_unused = 0;
          bool bad_unused;
          const bool valid = key_of<DECODE>(p, bt, row[c * kChunk + 32 * kh + lane], un, prow_unused, bad_unused);
          vmask = __ballot_sync(0xffffffffu, valid);
        }
        if (!pair_wait(&bar_s_full[s], (g >> 1) & 1u)) {
          aborted = true;
          break;
        }
        tc_fence_after();
        uint32_t sr[32];
        tmem_ld32(lane_base + kColS + 32 * s, sr);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_peer(s_free_l[s]);
        // row maximum over the valid keys of this half, then with the partner half
        float mx[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) mx[j] = -INFINITY;
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if ((vmask >> i) & 1u) mx[i & 7] = fmaxf(mx[i & 7], __uint_as_float(sr[i]));
        const float hmax = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])), fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
        const int buf = static_cast<int>(g & 1u);
        s_red[buf][kh][hl] = hmax;
        pair_sync(w);
        const float cmax = fmaxf(hmax, s_red[buf][kh ^ 1][hl]) * p.scale_log2;  // scale > 0
        bool rescale = false;
        float alpha = 1.f;
        if (c == un.c0) {
          m = cmax;
        } else if (cmax > m + kTau) {
          rescale = m > -INFINITY;  // nothing accumulated yet when every earlier key was masked
          alpha = rescale ? exp2f(m - cmax) : 1.f;
          m = cmax;
        }
        // tcgen05.ld/st are warp-collective: the whole warp runs the rescale if any row needs it
        // (the partner warp decides identically: same heads, same maxima)
        if (__any_sync(0xffffffffu, rescale)) {
          if (!pair_wait(&bar_pv_done[(g - 1) & 1u], ((g - 1) >> 1) & 1u)) {
            aborted = true;
            break;
          }
          tc_fence_after();
#pragma unroll 1
          for (int cc = 0; cc < 256; cc += 32) {
            uint32_t o[32];
            tmem_ld32(lane_base + kColO + cc, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(lane_base + kColO + cc, o);
          }
          tmem_wait_st();
          l *= alpha;
        }
        const float neg_m = -m;
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          float a = mla::ex2_approx(fmaf(__uint_as_float(sr[2 * i]), p.scale_log2, neg_m));
          float b = mla::ex2_approx(fmaf(__uint_as_float(sr[2 * i + 1]), p.scale_log2, neg_m));
          a = ((vmask >> (2 * i)) & 1u) ? a : 0.f;
          b = ((vmask >> (2 * i + 1)) & 1u) ? b : 0.f;
          pk[i] = pack_bf16x2(a, b);
          const float2 r = unpack_bf16x2(pk[i]);  // the row sum of the P that the tensor cores use
          l += r.x + r.y;
        }
        // P slot s is free once P.V of chunk g-2 has completed
        if (!pair_wait(&bar_pv_done[s], ((g >> 1) & 1u) ^ 1u)) {
          aborted = true;
          break;
        }
        uint8_t* prow = sP + s * kPBytes + hl * 128;
#pragma unroll
        for (int i = 0; i < 4; ++i)
          *reinterpret_cast<uint4*>(prow + (((4 * kh + i) ^ (hl & 7)) << 4)) =
              make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]);
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive_peer(p_full_l[s]);
      }
      if (aborted) break;
      // ---- epilogue of the unit: the row sum over both halves, then O / l ----
      s_red[2][kh][hl] = l;
      pair_sync(w);
      const float lt = l + s_red[2][kh ^ 1][hl];
      const uint32_t gl = g - 1;  // the unit's last chunk
      if (!pair_wait(&bar_pv_done[gl & 1u], (gl >> 1) & 1u)) {
        aborted = true;
        break;
      }
      tc_fence_after();
      if (!DECODE || p.splits == 1) {  // whole selection in this unit: O / l straight to out
        const float inv_l = lt > 0.f ? 1.f / lt : 0.f;
        __nv_bfloat16* orow = p.out + (un.qrow * p.H + h) * 512 + 128 * kh;
#pragma unroll 1
        for (int cc = 0; cc < 256; cc += 32) {
          uint32_t o[32];
          tmem_ld32(lane_base + kColO + cc, o);
          tmem_wait_ld();
          if (real) {
            uint32_t q16[16];
#pragma unroll
            for (int i = 0; i < 16; ++i)
              q16[i] = pack_bf16x2(__uint_as_float(o[2 * i]) * inv_l, __uint_as_float(o[2 * i + 1]) * inv_l);
            __nv_bfloat16* dst = orow + 256 * (cc >> 7) + (cc & 127);  // columns 128m + j: dims 256m + 128kh + j
#pragma unroll
            for (int i = 0; i < 4; ++i)
              *reinterpret_cast<uint4*>(dst + 8 * i) = make_uint4(q16[4 * i], q16[4 * i + 1], q16[4 * i + 2], q16[4 * i + 3]);
          }
        }
        if (kh == 0 && real && p.lse != nullptr)
          p.lse[un.qrow * p.H + h] = lt > 0.f ? (m + log2f(lt)) * 0.69314718055994531f : -INFINITY;
      } else {
        float* po = p.part_o + ((static_cast<int64_t>(un.seq) * p.splits + un.sp) * p.H + h) * 512 + 128 * kh;
#pragma unroll 1
        for (int cc = 0; cc < 256; cc += 32) {
          uint32_t o[32];
          tmem_ld32(lane_base + kColO + cc, o);
          tmem_wait_ld();
          if (real) {
            float* dst = po + 256 * (cc >> 7) + (cc & 127);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              *reinterpret_cast<uint4*>(dst + 4 * i) = make_uint4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
          }
        }
        if (kh == 0 && real) {
          float* ml = p.part_ml + ((static_cast<int64_t>(un.seq) * p.splits + un.sp) * p.H + h) * 2;
          ml[0] = m;
          ml[1] = lt;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_peer(o_free_l);
    }
    if (aborted) record_device_error(DSA_ERR_TIMEOUT);
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no CTA of the pair still signals or reads the other
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

}  // namespace dsa
