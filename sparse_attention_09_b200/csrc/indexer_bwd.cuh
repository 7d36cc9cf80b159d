// Backward of the lightning indexer into its inputs, for training the indexer by the KL loss
// ("DeepSeek-V3.2 论文解读", section 二, subsection "两阶段继续预训练": in both training stages
// the indexer is trained by the KL loss alone, its input detached from the main model).
//
// Given g[t, i] = d loss / d I[t, idx[t, i]] on each token's entries (idx -1 padded; in the
// dense warm-up stage the entries are the whole causal prefix), with dequantised operands
//   q_I[t,j,:] = e4m3(q8[t,j,:]) * q_scale[t] (or q_scale[t,j]),  k_I[s,:] = e4m3(k8[s,:]) * k_scale[s],
//   a[j,s] = q_I[t,j,:] . k_I[s,:]:
//   dw[t,j]      = sum_i g[t,i] * ReLU(a[j, s_i])
//   dq_I[t,j,:]  = sum_i g[t,i] * w[t,j] * [a[j,s_i] > 0] * k_I[s_i,:]
//   dk_I[s,:]   += g[t,i] * sum_j w[t,j] * [a[j,s_i] > 0] * q_I[t,j,:]   (over every t selecting s)
// The FP8 codes are widened exactly and scaled in fp32; every product and sum is fp32 on the
// CUDA cores (no tensor-core rounding of the operands).
//
// One CTA of 256 threads per query token (grid-stride).  The token's q_I (H_I x d_I fp32) and
// w sit in shared memory; its entries go by in chunks of 32 keys: the k_I rows of a chunk are
// widened into shared memory, then (A) the H_I x 32 logits and the masked weights
// M[j,s] = [a > 0] w_j g_s, (B) dq += M K over the chunk (dq lives in registers, H_I*d_I/256
// values per thread), (C) the chunk's dk rows M^T Q, added to global memory with vector fp32
// reductions (tokens that selected the same key add concurrently).
#pragma once

#include <cuda_fp8.h>

#include "common.cuh"

namespace dsa {

struct IdxBwdParams {
  const uint8_t* q8;          // [T, H_I, d_I]
  const float* q_scale;       // [T] or [T, H_I]
  int32_t q_scale_heads;      // 1 or H_I
  const float* w;             // [T, H_I]
  const uint8_t* k8;          // [T, d_I]
  const float* k_scale;       // [T]
  const int32_t* cu_seqlens;  // [B+1]
  int32_t B;
  const int32_t* idx;         // [T, k]
  const float* grad;          // [T, k]
  int32_t k;
  int64_t rows;               // T
  float* dw;                  // [T, H_I]
  float* dq;                  // [T, H_I, d_I]
  float* dk;                  // [T, d_I], accumulated (zeroed by the host before the launch)
};

namespace ibwd {
constexpr int kThreads = 256;
constexpr int kKC = 32;  // keys per chunk

template <int H_I, int D_I>
struct Layout {
  static constexpr int kKStride = D_I + 1;  // padded k_I rows: lanes of phase A read different rows
  static constexpr int kQFloats = H_I * D_I;
  static constexpr int kKFloats = kKC * kKStride;
  static constexpr int kMFloats = H_I * kKC;
  static constexpr int kSmemBytes = 4 * (kQFloats + kKFloats + kMFloats + H_I + H_I + kKC) + 4 * kKC;
};

__device__ __forceinline__ float e4m3_to_f32(uint8_t c) {
  return __half2float(__half(__nv_cvt_fp8_to_halfraw(static_cast<__nv_fp8_storage_t>(c), __NV_E4M3)));
}
}  // namespace ibwd

template <int H_I, int D_I>
__global__ void __launch_bounds__(ibwd::kThreads) indexer_backward_kernel(const IdxBwdParams p) {
  using namespace ibwd;
  using Lay = Layout<H_I, D_I>;
  constexpr int EQ = H_I * D_I / kThreads;   // dq values per thread
  constexpr int PA = H_I * kKC / kThreads;   // logits per thread per chunk (0 when H_I * 32 < 256)
  constexpr int D4 = D_I / 4;
  static_assert((H_I * D_I) % kThreads == 0, "dq split");
  extern __shared__ __align__(16) float ibwd_smem[];
  float* sQ = ibwd_smem;                      // [H_I][D_I]
  float* sK = sQ + Lay::kQFloats;             // [kKC][D_I + 1]
  float* sM = sK + Lay::kKFloats;             // [H_I][kKC]
  float* sW = sM + Lay::kMFloats;             // [H_I]
  float* sDW = sW + H_I;                      // [H_I]
  float* sG = sDW + H_I;                      // [kKC]
  int* sV = reinterpret_cast<int*>(sG + kKC); // [kKC] key row (packed) or -1
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

  for (int64_t u = blockIdx.x; u < p.rows; u += gridDim.x) {
    int lo = 0, hi = p.B;  // the token's sequence
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (p.cu_seqlens[mid] <= u) lo = mid;
      else hi = mid;
    }
    const int seq_start = p.cu_seqlens[lo], seq_len = p.cu_seqlens[lo + 1] - seq_start;
    // the token's dequantised queries and head weights
    for (int e = tid; e < H_I * D_I; e += kThreads) {
      const int j = e / D_I;
      const float sc = p.q_scale[p.q_scale_heads == 1 ? u : u * H_I + j];
      sQ[e] = e4m3_to_f32(p.q8[u * H_I * D_I + e]) * sc;
    }
    for (int j = tid; j < H_I; j += kThreads) {
      sW[j] = p.w[u * H_I + j];
      sDW[j] = 0.f;
    }
    float dq[EQ];
#pragma unroll
    for (int r = 0; r < EQ; ++r) dq[r] = 0.f;
    // the entries up to the last valid one
    int last = -1;
    for (int i = tid; i < p.k; i += kThreads)
      if (p.idx[u * p.k + i] >= 0) last = i;
    last = __reduce_max_sync(0xffffffffu, last);
    __shared__ int s_last[kThreads / 32];
    if (lane == 0) s_last[warp] = last;
    __syncthreads();
    last = -1;
#pragma unroll
    for (int i = 0; i < kThreads / 32; ++i) last = max(last, s_last[i]);
    const int nchunks = (last + kKC) / kKC;

    for (int c = 0; c < nchunks; ++c) {
      if (tid < kKC) {
        const int i = c * kKC + tid;
        const int v = i < p.k ? p.idx[u * p.k + i] : -1;
        const bool valid = v >= 0 && v < seq_len;
        if (!valid && v != -1) record_device_error(DSA_ERR_DEVICE_CHECK);
        sV[tid] = valid ? seq_start + v : -1;
        sG[tid] = valid ? p.grad[u * p.k + i] : 0.f;
      }
      __syncthreads();
      // k_I rows of the chunk, widened and scaled (zero rows for invalid entries)
      for (int e = tid; e < kKC * D4; e += kThreads) {
        const int s = e / D4, d = 4 * (e % D4);
        const int row = sV[s];
        float* dst = sK + s * Lay::kKStride + d;
        if (row >= 0) {
          const uint32_t codes = *reinterpret_cast<const uint32_t*>(p.k8 + static_cast<int64_t>(row) * D_I + d);
          const float ks = p.k_scale[row];
#pragma unroll
          for (int b = 0; b < 4; ++b) dst[b] = e4m3_to_f32(static_cast<uint8_t>(codes >> (8 * b))) * ks;
        } else {
#pragma unroll
          for (int b = 0; b < 4; ++b) dst[b] = 0.f;
        }
      }
      __syncthreads();
      // (A) logits a[j,s] (a warp: one head, its 32 lanes the chunk's 32 keys), the masked
      // weights and the head-weight gradient
#pragma unroll
      for (int r = 0; r < (PA > 0 ? PA : 1); ++r) {
        const int pidx = tid + kThreads * r;
        if (pidx < H_I * kKC) {
          const int j = pidx / kKC, s = pidx % kKC;
          const float* qr = sQ + j * D_I;
          const float* kr = sK + s * Lay::kKStride;
          float a = 0.f;
#pragma unroll 16
          for (int d = 0; d < D_I; ++d) a = fmaf(qr[d], kr[d], a);
          const float gs = sG[s];
          sM[j * kKC + s] = a > 0.f ? sW[j] * gs : 0.f;
          float part = fmaxf(a, 0.f) * gs;
#pragma unroll
          for (int o = 16; o >= 1; o >>= 1) part += __shfl_xor_sync(0xffffffffu, part, o);
          if (lane == 0) sDW[j] += part;  // one warp per head per chunk
        }
      }
      __syncthreads();
      // (B) dq[j,d] += sum_s M[j,s] k_I[s,d]
#pragma unroll
      for (int r = 0; r < EQ; ++r) {
        const int e = tid + kThreads * r;
        const int j = e / D_I, d = e % D_I;
        const float* mr = sM + j * kKC;
        float acc = dq[r];
#pragma unroll
        for (int s = 0; s < kKC; ++s) acc = fmaf(mr[s], sK[s * Lay::kKStride + d], acc);
        dq[r] = acc;
      }
      // (C) dk[s, 4 dims] += sum_j M[j,s] q_I[j, 4 dims]
      for (int e = tid; e < kKC * D4; e += kThreads) {
        const int s = e / D4, d = 4 * (e % D4);
        const int row = sV[s];
        if (row < 0) continue;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll 8
        for (int j = 0; j < H_I; ++j) {
          const float m = sM[j * kKC + s];
          const float4 q4 = *reinterpret_cast<const float4*>(sQ + j * D_I + d);
          acc.x = fmaf(m, q4.x, acc.x);
          acc.y = fmaf(m, q4.y, acc.y);
          acc.z = fmaf(m, q4.z, acc.z);
          acc.w = fmaf(m, q4.w, acc.w);
        }
        atomicAdd(reinterpret_cast<float4*>(p.dk + static_cast<int64_t>(row) * D_I + d), acc);
      }
      __syncthreads();  // sK, sM, sV and sG are rewritten by the next chunk
    }
#pragma unroll
    for (int r = 0; r < EQ; ++r) p.dq[u * H_I * D_I + tid + kThreads * r] = dq[r];
    __syncthreads();
    for (int j = tid; j < H_I; j += kThreads) p.dw[u * H_I + j] = sDW[j];
    __syncthreads();  // sQ, sW and sDW are rewritten by the next token
  }
}

// The same computation for 64 heads, register-blocked: every shared-memory load is a 16-byte
// vector that feeds 8 (phase A) or 16-32 (phases B, C) fused multiply-adds.
//   A: thread (jb, sb) -> heads 2jb, 2jb+1 and keys sb + 8i (i < 4): 8 logits;
//   B: thread (jq, dq) -> heads 4jq..4jq+3, dims 4dq + 64c: dq accumulators in registers;
//   C: thread (sq, dq) -> keys 2sq, 2sq+1, dims 4dq + 64c: the chunk's dk rows.
// Rows of q_I and k_I are padded by 4 floats, so the 8 lanes that read 8 consecutive key rows
// (phase A) or heads 2 apart hit distinct banks.
namespace ibwd {
template <int D_I>
struct Layout64 {
  static constexpr int kQS = D_I + 4, kKS = D_I + 4;
  static constexpr int kFloats = 64 * kQS + kKC * kKS + 2 * 64 * kKC + 64 + 64 + kKC;
  static constexpr int kSmemBytes = 4 * kFloats + 4 * kKC;
};

__device__ __forceinline__ float dot4(const float4 a, const float4 b, float acc) {
  return fmaf(a.w, b.w, fmaf(a.z, b.z, fmaf(a.y, b.y, fmaf(a.x, b.x, acc))));
}
}  // namespace ibwd

template <int D_I>
__global__ void __launch_bounds__(ibwd::kThreads) indexer_backward_h64_kernel(const IdxBwdParams p) {
  using namespace ibwd;
  using Lay = Layout64<D_I>;
  constexpr int H_I = 64, QS = Lay::kQS, KS = Lay::kKS, D4 = D_I / 4, NC = D_I / 64;
  extern __shared__ __align__(16) float ibwd_smem[];
  float* sQ = ibwd_smem;                       // [64][QS]
  float* sK = sQ + 64 * QS;                    // [kKC][KS]
  float* sM = sK + kKC * KS;                   // [64][kKC]  M[j][s]
  float* sMT = sM + 64 * kKC;                  // [kKC][64]  M[j][s] transposed
  float* sW = sMT + kKC * 64;                  // [64]
  float* sDW = sW + 64;                        // [64]
  float* sG = sDW + 64;                        // [kKC]
  int* sV = reinterpret_cast<int*>(sG + kKC);  // [kKC]
  __shared__ int s_last[kThreads / 32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int jb = tid >> 3, sb = tid & 7;       // phase A
  const int jq = tid >> 4, dq4 = tid & 15;     // phase B (and sq = jq in phase C)

  for (int64_t u = blockIdx.x; u < p.rows; u += gridDim.x) {
    int lo = 0, hi = p.B;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (p.cu_seqlens[mid] <= u) lo = mid;
      else hi = mid;
    }
    const int seq_start = p.cu_seqlens[lo], seq_len = p.cu_seqlens[lo + 1] - seq_start;
    for (int e = tid; e < H_I * D_I; e += kThreads) {
      const int j = e / D_I, d = e % D_I;
      const float sc = p.q_scale[p.q_scale_heads == 1 ? u : u * H_I + j];
      sQ[j * QS + d] = e4m3_to_f32(p.q8[u * H_I * D_I + e]) * sc;
    }
    if (tid < H_I) {
      sW[tid] = p.w[u * H_I + tid];
      sDW[tid] = 0.f;
    }
    float dq[4][NC][4];
#pragma unroll
    for (int h = 0; h < 4; ++h)
#pragma unroll
      for (int c = 0; c < NC; ++c)
#pragma unroll
        for (int e = 0; e < 4; ++e) dq[h][c][e] = 0.f;
    int last = -1;
    for (int i = tid; i < p.k; i += kThreads)
      if (p.idx[u * p.k + i] >= 0) last = i;
    last = __reduce_max_sync(0xffffffffu, last);
    if (lane == 0) s_last[warp] = last;
    __syncthreads();
    last = -1;
#pragma unroll
    for (int i = 0; i < kThreads / 32; ++i) last = max(last, s_last[i]);
    const int nchunks = (last + kKC) / kKC;

    for (int c0 = 0; c0 < nchunks; ++c0) {
      if (tid < kKC) {
        const int i = c0 * kKC + tid;
        const int v = i < p.k ? p.idx[u * p.k + i] : -1;
        const bool valid = v >= 0 && v < seq_len;
        if (!valid && v != -1) record_device_error(DSA_ERR_DEVICE_CHECK);
        sV[tid] = valid ? seq_start + v : -1;
        sG[tid] = valid ? p.grad[u * p.k + i] : 0.f;
      }
      __syncthreads();
      for (int e = tid; e < kKC * D4; e += kThreads) {
        const int s = e / D4, d = 4 * (e % D4);
        const int row = sV[s];
        float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
        if (row >= 0) {
          const uint32_t codes = *reinterpret_cast<const uint32_t*>(p.k8 + static_cast<int64_t>(row) * D_I + d);
          const float ks = p.k_scale[row];
          x = make_float4(e4m3_to_f32(static_cast<uint8_t>(codes)) * ks, e4m3_to_f32(static_cast<uint8_t>(codes >> 8)) * ks,
                          e4m3_to_f32(static_cast<uint8_t>(codes >> 16)) * ks,
                          e4m3_to_f32(static_cast<uint8_t>(codes >> 24)) * ks);
        }
        *reinterpret_cast<float4*>(sK + s * KS + d) = x;
      }
      __syncthreads();
      // (A) logits of heads 2jb, 2jb+1 at keys sb + 8i
      {
        float a[2][4];
#pragma unroll
        for (int h = 0; h < 2; ++h)
#pragma unroll
          for (int i = 0; i < 4; ++i) a[h][i] = 0.f;
#pragma unroll 4
        for (int d4 = 0; d4 < D4; ++d4) {
          const float4 q0 = *reinterpret_cast<const float4*>(sQ + (2 * jb) * QS + 4 * d4);
          const float4 q1 = *reinterpret_cast<const float4*>(sQ + (2 * jb + 1) * QS + 4 * d4);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float4 kk = *reinterpret_cast<const float4*>(sK + (sb + 8 * i) * KS + 4 * d4);
            a[0][i] = dot4(q0, kk, a[0][i]);
            a[1][i] = dot4(q1, kk, a[1][i]);
          }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int j = 2 * jb + h;
          const float wj = sW[j];
          float part = 0.f;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const int s = sb + 8 * i;
            const float gs = sG[s];
            const float m = a[h][i] > 0.f ? wj * gs : 0.f;
            sM[j * kKC + s] = m;
            sMT[s * 64 + j] = m;
            part = fmaf(fmaxf(a[h][i], 0.f), gs, part);
          }
          // the 8 lanes of this head pair (same jb) hold its 32 keys
          part += __shfl_xor_sync(0xffffffffu, part, 1);
          part += __shfl_xor_sync(0xffffffffu, part, 2);
          part += __shfl_xor_sync(0xffffffffu, part, 4);
          if (sb == 0) sDW[j] += part;
        }
      }
      __syncthreads();
      // (B) dq[4jq + h, 4dq4 + 64c + e] += sum_s M[j,s] k_I[s, d]
#pragma unroll 4
      for (int s = 0; s < kKC; ++s) {
        const float4 m4 = *reinterpret_cast<const float4*>(sMT + s * 64 + 4 * jq);
        const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          const float4 kk = *reinterpret_cast<const float4*>(sK + s * KS + 4 * dq4 + 64 * c);
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            dq[h][c][0] = fmaf(mm[h], kk.x, dq[h][c][0]);
            dq[h][c][1] = fmaf(mm[h], kk.y, dq[h][c][1]);
            dq[h][c][2] = fmaf(mm[h], kk.z, dq[h][c][2]);
            dq[h][c][3] = fmaf(mm[h], kk.w, dq[h][c][3]);
          }
        }
      }
      // (C) dk rows of keys 2jq, 2jq+1: sum_j M[j,s] q_I[j, d]
      {
        float acc[2][NC][4];
#pragma unroll
        for (int r = 0; r < 2; ++r)
#pragma unroll
          for (int c = 0; c < NC; ++c)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[r][c][e] = 0.f;
#pragma unroll 4
        for (int j = 0; j < H_I; ++j) {
          const float2 m2 = *reinterpret_cast<const float2*>(sM + j * kKC + 2 * jq);
#pragma unroll
          for (int c = 0; c < NC; ++c) {
            const float4 qq = *reinterpret_cast<const float4*>(sQ + j * QS + 4 * dq4 + 64 * c);
            acc[0][c][0] = fmaf(m2.x, qq.x, acc[0][c][0]);
            acc[0][c][1] = fmaf(m2.x, qq.y, acc[0][c][1]);
            acc[0][c][2] = fmaf(m2.x, qq.z, acc[0][c][2]);
            acc[0][c][3] = fmaf(m2.x, qq.w, acc[0][c][3]);
            acc[1][c][0] = fmaf(m2.y, qq.x, acc[1][c][0]);
            acc[1][c][1] = fmaf(m2.y, qq.y, acc[1][c][1]);
            acc[1][c][2] = fmaf(m2.y, qq.z, acc[1][c][2]);
            acc[1][c][3] = fmaf(m2.y, qq.w, acc[1][c][3]);
          }
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int row = sV[2 * jq + r];
          if (row < 0) continue;
#pragma unroll
          for (int c = 0; c < NC; ++c)
            atomicAdd(reinterpret_cast<float4*>(p.dk + static_cast<int64_t>(row) * D_I + 4 * dq4 + 64 * c),
                      make_float4(acc[r][c][0], acc[r][c][1], acc[r][c][2], acc[r][c][3]));
        }
      }
      __syncthreads();  // sK, sM, sMT, sV and sG are rewritten by the next chunk
    }
#pragma unroll
    for (int h = 0; h < 4; ++h)
#pragma unroll
      for (int c = 0; c < NC; ++c)
        *reinterpret_cast<float4*>(p.dq + (u * H_I + 4 * jq + h) * D_I + 4 * dq4 + 64 * c) =
            make_float4(dq[h][c][0], dq[h][c][1], dq[h][c][2], dq[h][c][3]);
    __syncthreads();
    if (tid < H_I) p.dw[u * H_I + tid] = sDW[tid];
    __syncthreads();  // sQ, sW and sDW are rewritten by the next token
  }
}

}  // namespace dsa
