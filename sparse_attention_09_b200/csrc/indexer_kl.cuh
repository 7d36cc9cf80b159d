// KL alignment loss of the indexer and its gradient, per query token, over the token's
// selected rows ("DeepSeek-V3.2 论文解读", section 二: the indexer is trained with a KL loss
// towards the main attention's distribution; in the sparse stage over the selected set):
//   q = softmax(scores) over the valid entries (idx >= 0),
//   loss = sum_i p_i (log p_i - log q_i)  (entries with p_i = 0 add nothing),
//   grad_i = d loss / d scores_i = q_i - p_i  (0 for invalid entries).
// One CTA per row, fp32, three passes over the row (max, sum of exponentials, terms).
#pragma once

#include "common.cuh"

namespace dsa {

namespace kl {
constexpr int kThreads = 256;

template <bool MAX>
__device__ __forceinline__ float block_reduce(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const float w = __shfl_xor_sync(0xffffffffu, v, o);
    v = MAX ? fmaxf(v, w) : v + w;
  }
  __syncthreads();  // red is free (a previous reduction has been read)
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float r = red[0];
#pragma unroll
  for (int i = 1; i < kThreads / 32; ++i) r = MAX ? fmaxf(r, red[i]) : r + red[i];
  return r;
}
}  // namespace kl

__global__ void __launch_bounds__(kl::kThreads)
    indexer_kl_kernel(const float* __restrict__ p, const float* __restrict__ scores, const int32_t* __restrict__ idx,
                      int k, float* __restrict__ loss, float* __restrict__ grad) {
  __shared__ float red[kl::kThreads / 32];
  const int64_t row = blockIdx.x;
  const float* pr = p + row * k;
  const float* sr = scores + row * k;
  const int32_t* ir = idx + row * k;
  float* gr = grad + row * k;
  float mx = -INFINITY;
  for (int j = threadIdx.x; j < k; j += kl::kThreads)
    if (ir[j] >= 0) mx = fmaxf(mx, sr[j]);
  mx = kl::block_reduce<true>(mx, red);
  if (mx == -INFINITY) {  // no valid entry
    for (int j = threadIdx.x; j < k; j += kl::kThreads) gr[j] = 0.f;
    if (threadIdx.x == 0) loss[row] = 0.f;
    return;
  }
  float se = 0.f;
  for (int j = threadIdx.x; j < k; j += kl::kThreads)
    if (ir[j] >= 0) se += expf(sr[j] - mx);
  se = kl::block_reduce<false>(se, red);
  const float lz = mx + logf(se);  // log-sum-exp of the valid scores
  float l = 0.f;
  for (int j = threadIdx.x; j < k; j += kl::kThreads) {
    float g = 0.f;
    if (ir[j] >= 0) {
      const float lq = sr[j] - lz;
      const float pj = pr[j];
      if (pj > 0.f) l += pj * (logf(pj) - lq);
      g = expf(lq) - pj;
    }
    gr[j] = g;
  }
  l = kl::block_reduce<false>(l, red);
  if (threadIdx.x == 0) loss[row] = l;
}

}  // namespace dsa
