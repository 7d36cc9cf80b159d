// The main attention's distribution over each token's selected rows, averaged over heads:
//   p[t, i] = (1/H) sum_h 2^(x * q[t,h] . c[idx[t,i]] - lse2[t,h]),   x = sm_scale * log2(e),
// with lse2 = lse * log2(e) from the sparse MLA forward.  It is the target the indexer's
// distribution is aligned to by the KL loss in the sparse training stage ("DeepSeek-V3.2
// 论文解读", section 二: the indexer is trained with a KL loss towards the main attention).
//
// Dense mode (the dense warm-up stage's target): the same over every row of the token's causal
// prefix, p[t, s] for s <= t (the entries are the prefix positions themselves, no selection
// list), with lse from a dense (masked) attention forward; p rows hold ld entries, zero past t.
//
// One CTA per SM walks tokens.  Per CTA: warps 0-3 turn logits into probabilities and reduce
// them over heads (thread h = head h = TMEM lane h), warps 4-5 gather the selected latent rows
// (all 576 dims, cp.async into 9 blocks of 64 dims with the 128-byte swizzle), warp 6 issues
// Q.K^T (tcgen05, Q in TMEM columns [0, 288), S double-buffered in [288, 416)).  No value
// product, so there is no O accumulator and no cross-CTA exchange.
#pragma once

#include "common.cuh"
#include "sm100.cuh"

namespace dsa {

struct ProbsParams {
  const __nv_bfloat16* q;     // [rows, H, 576] (dense: [T, H, 576], packed tokens)
  const int32_t* idx;         // [rows, k] (sparse mode)
  const float* lse;           // [rows, H] natural log (dense: [T, H])
  const int32_t* cu_seqlens;  // [B+1]
  int32_t B, H, k;
  int64_t rows;               // units: sparse, rows of q / idx / p; dense, tokens row0 .. row0+rows-1
  int64_t row0;               // dense: packed token of unit 0
  int64_t ld;                 // dense: entries per row of p
  float scale_log2;           // sm_scale * log2(e)
  float* p;                   // [rows, k] (dense: [rows, ld])
};

namespace probs {
constexpr int kChunk = 64;
constexpr int kStages = 2;
constexpr int kBlockBytes = kChunk * 128;              // 64 rows x 64 dims bf16
constexpr int kBlocks = 9;                             // 576 dims
constexpr int kStageBytes = kBlocks * kBlockBytes;     // 73728
constexpr int kSmemBytes = kStages * kStageBytes;
constexpr uint32_t kColQ = 0, kColS = 288;             // S buffers at 288 and 352
constexpr int kProducerWarps = 2, kMmaWarp = 6, kThreads = 7 * 32;

__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

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

// Lane l receives sum over the 32 lanes of v[l] (v: 32 values per lane), by halving exchanges.
__device__ __forceinline__ float lane_transpose_sum(float (&v)[32]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int s = 16; s >= 1; s >>= 1) {
    const bool upper = (lane & s) != 0;
#pragma unroll
    for (int i = 0; i < s; ++i) {
      const float send = upper ? v[i] : v[i + s];
      const float keep = upper ? v[i + s] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
    }
  }
  return v[0];
}
}  // namespace probs

template <bool DENSE>
__global__ void __launch_bounds__(probs::kThreads, 1)
    attn_probs_kernel(const __nv_bfloat16* __restrict__ latent, const ProbsParams p) {
  using namespace dev;
  using namespace probs;
  constexpr uint32_t IDESC_QK = idesc_bf16(128, kChunk, false, false);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* sKV = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  __shared__ uint64_t bar_kvfull[kStages], bar_kvempty[kStages], bar_sfull[2], bar_sfree[2], bar_qfull;
  __shared__ float s_red[2][4][kChunk];
  __shared__ uint32_t s_tmem;

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t nunits = p.rows;
  if (tid == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&bar_kvfull[i], 32 * kProducerWarps);
      mbar_init(&bar_kvempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_sfull[i], 1);
      mbar_init(&bar_sfree[i], 4);
    }
    mbar_init(&bar_qfull, 128);
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;

  auto seq_of = [&](int64_t u, int& seq_start, int& seq_len) {
    int lo = 0, hi = p.B;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (p.cu_seqlens[mid] <= u) lo = mid;
      else hi = mid;
    }
    seq_start = p.cu_seqlens[lo];
    seq_len = p.cu_seqlens[lo + 1] - seq_start;
  };
  // chunks up to the last valid entry of the row (every role computes the same, warp-wide);
  // dense: up to the token's own position t
  auto unit_chunks = [&](int64_t u) {
    if constexpr (DENSE) {
      int seq_start, seq_len;
      seq_of(u + p.row0, seq_start, seq_len);
      return static_cast<int>(u + p.row0 - seq_start) / kChunk + 1;
    } else {
      const int32_t* row = p.idx + u * p.k;
      int last = -1;
      for (int j = lane; j < p.k; j += 32)
        if (row[j] >= 0) last = j;
      last = __reduce_max_sync(0xffffffffu, last);
      return last < 0 ? 1 : last / kChunk + 1;
    }
  };
  // entry j of a unit's row: its latent row position (and whether it is valid)
  auto entry = [&](int64_t u, int t, int seq_len, int j, bool& valid) {
    if constexpr (DENSE) {
      valid = j <= t;
      return j;
    } else {
      const int v = p.idx[u * p.k + j];
      valid = v >= 0 && v < seq_len;
      return v;
    }
  };

  if (warp >= 4 && warp < kMmaWarp) {
    // ================= gather producers =================
    // Warp pw copies keys [32 pw, 32 pw + 32) of each chunk: 32 keys x 72 chunks of 16 bytes,
    // 72 warp instructions; flat chunk f = 32 i + lane -> key f / 72, 16-byte piece f % 72.
    const int pw = warp - 4;
    uint32_t g = 0;
    bool ok = true;
    for (int64_t u = blockIdx.x; ok && u < nunits; u += gridDim.x) {
      int seq_start, seq_len;
      seq_of(DENSE ? u + p.row0 : u, seq_start, seq_len);
      const int t = DENSE ? static_cast<int>(u + p.row0 - seq_start) : 0;
      const int c1 = unit_chunks(u);
      for (int c = 0; c < c1; ++c, ++g) {
        const int stage = static_cast<int>(g % kStages);
        if (!mbar_wait(&bar_kvempty[stage], ((g / kStages) & 1u) ^ 1u)) {
          record_device_error(DSA_ERR_TIMEOUT);
          ok = false;
          break;
        }
        bool valid;
        const int v = entry(u, t, seq_len, c * kChunk + 32 * pw + lane, valid);
        const int prow = seq_start + (valid ? v : 0);  // masked rows still copy a real row
        const uint32_t st = smem_addr(sKV + stage * kStageBytes);
#pragma unroll 8
        for (int i = 0; i < 72; ++i) {
          const int f = 32 * i + lane;
          const int j = f / 72, piece = f % 72;
          const int kr = __shfl_sync(0xffffffffu, prow, j);
          const int r = 32 * pw + j;
          const int blk = piece >> 3, ch = piece & 7;
          cp_async16(st + blk * kBlockBytes + r * 128 + ((ch ^ (r & 7)) << 4),
                     latent + static_cast<int64_t>(kr) * 576 + 8 * piece);
        }
        cp_async_commit();
        cp_async_mbar_arrive(&bar_kvfull[stage]);
        mbar_arrive(&bar_kvfull[stage]);
      }
    }
    cp_async_wait<0>();
  } else if (warp == kMmaWarp) {
    // ================= MMA issuer =================
    // Chunks arrive in order; S is double-buffered, so Q.K^T of chunk g waits for its keys
    // and for the softmax warps to have read S of chunk g-2 (and, opening a unit, for its Q).
    bool ok = true;
    uint32_t g = 0, tok = 0;
    auto wait1 = [&](uint64_t* bar, uint32_t parity) -> bool {
      bool r = true;
      if (lane == 0) r = mbar_wait(bar, parity);
      return __shfl_sync(0xffffffffu, r, 0) != 0;
    };
    for (int64_t u = blockIdx.x; ok && u < nunits; u += gridDim.x, ++tok) {
      const int c1 = unit_chunks(u);
      for (int c = 0; c < c1; ++c, ++g) {
        const int stage = static_cast<int>(g % kStages), b = static_cast<int>(g & 1u);
        ok = wait1(&bar_kvfull[stage], (g / kStages) & 1u) && (g < 2 || wait1(&bar_sfree[b], ((g >> 1) - 1) & 1u)) &&
             (c != 0 || wait1(&bar_qfull, tok & 1u));
        if (!ok) break;
        tc_fence_after();
        if (lane == 0) {
          fence_proxy_async_smem();  // the gathered rows were written through the generic proxy
          const uint32_t st = smem_addr(sKV + stage * kStageBytes);
#pragma unroll
          for (int kk = 0; kk < 36; ++kk)  // 576 dims: 9 blocks x 4 steps of 16
            umma_bf16_ts(tmem + kColS + 64 * b, tmem + kColQ + kk * 8,
                         make_smem_desc(st + (kk >> 2) * kBlockBytes + (kk & 3) * 32, 16, 1024, kSwizzle128B),
                         IDESC_QK, kk > 0 ? 1u : 0u);
          umma_commit(&bar_sfull[b]);
          umma_commit(&bar_kvempty[stage]);
        }
        __syncwarp();
      }
    }
    if (!ok && lane == 0) record_device_error(DSA_ERR_TIMEOUT);
  } else {
    // ================= probabilities and the head sum (warps 0-3) =================
    const int h = tid;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    auto load_q = [&](int64_t u) {
      const __nv_bfloat16* qr = p.q + ((DENSE ? u + p.row0 : u) * p.H + h) * 576;
      const bool real = h < p.H;
#pragma unroll 1
      for (int c0 = 0; c0 < 288; c0 += 48) {
        uint32_t v[48];
#pragma unroll
        for (int j = 0; j < 12; ++j) {
          uint4 w = make_uint4(0u, 0u, 0u, 0u);
          if (real) w = __ldg(reinterpret_cast<const uint4*>(qr + 2 * (c0 + 4 * j)));
          v[4 * j] = w.x;
          v[4 * j + 1] = w.y;
          v[4 * j + 2] = w.z;
          v[4 * j + 3] = w.w;
        }
#pragma unroll
        for (int c = 0; c < 48; c += 16) tmem_st16(lane_base + kColQ + c0 + c, *reinterpret_cast<uint32_t(*)[16]>(v + c));
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar_qfull);
    };
    bool aborted = false;
    uint32_t g = 0;
    const float inv_h = 1.f / static_cast<float>(p.H);
    if (blockIdx.x < nunits) load_q(blockIdx.x);
    for (int64_t u = blockIdx.x; u < nunits; u += gridDim.x) {
      const int c1 = unit_chunks(u);
      int seq_start, seq_len;
      const int64_t gq = DENSE ? u + p.row0 : u;  // row of q and lse
      seq_of(gq, seq_start, seq_len);
      const int t = DENSE ? static_cast<int>(gq - seq_start) : 0;
      const float lse2 = h < p.H ? p.lse[gq * p.H + h] * 1.4426950408889634f : INFINITY;
      const int64_t row_len = DENSE ? p.ld : p.k;
      float* prow = p.p + u * row_len;
      for (int c = 0; c < c1; ++c, ++g) {
        const int b = static_cast<int>(g & 1u);
        // which of the chunk's 64 entries are valid: read here from the selection row (every
        // warp the same), so the mask needs no hand-over from the gather warps
        bool v0, v1;
        entry(u, t, seq_len, c * kChunk + lane, v0);
        entry(u, t, seq_len, c * kChunk + 32 + lane, v1);
        bool ok = mbar_wait(&bar_sfull[b], (g >> 1) & 1u);
        if (sm_any(!ok)) {
          aborted = true;
          break;
        }
        tc_fence_after();
        uint32_t sr[64];
        tmem_ld32(lane_base + kColS + 64 * b, *reinterpret_cast<uint32_t(*)[32]>(sr));
        tmem_ld32(lane_base + kColS + 64 * b + 32, *reinterpret_cast<uint32_t(*)[32]>(sr + 32));
        tmem_wait_ld();
        reg_fence(sr);
        const uint64_t vmask = static_cast<uint64_t>(__ballot_sync(0xffffffffu, v0)) |
                               (static_cast<uint64_t>(__ballot_sync(0xffffffffu, v1)) << 32);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar_sfree[b]);
        if (c == c1 - 1 && u + gridDim.x < nunits) load_q(u + gridDim.x);  // this unit's Q.K^T are done
        float half[2];
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const int j = 32 * hh + i;
            const float e = ex2f(fmaf(__uint_as_float(sr[j]), p.scale_log2, -lse2));
            v[i] = ((vmask >> j) & 1ull) ? e : 0.f;
          }
          half[hh] = lane_transpose_sum(v);  // this warp's 32 heads, key 32 hh + lane
        }
        s_red[g & 1u][warp][lane] = half[0];
        s_red[g & 1u][warp][32 + lane] = half[1];
        sm_sync();
        if (tid < kChunk && c * kChunk + tid < row_len) {  // a dense row may end inside the chunk
          const float s = (s_red[g & 1u][0][tid] + s_red[g & 1u][1][tid]) + (s_red[g & 1u][2][tid] + s_red[g & 1u][3][tid]);
          prow[c * kChunk + tid] = s * inv_h;
        }
      }
      if (aborted) break;
      for (int64_t j = c1 * kChunk + tid; j < row_len; j += 128) prow[j] = 0.f;  // past the last valid entry
    }
    if (aborted) record_device_error(DSA_ERR_TIMEOUT);
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace dsa
