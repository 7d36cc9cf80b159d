// Shared device-side definitions: status codes, the device error word, score order keys,
// warp/block scans.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/dsa.h"

namespace dsa {

// Device error word: the first device-detected error since the last dsa_device_error().
__device__ int32_t g_device_error = 0;

__device__ __forceinline__ void record_device_error(int32_t code) {
  atomicCAS(&g_device_error, 0, code);
}

// Unsigned key whose order is the float order (-0.0 and +0.0 map to the same key).
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ bool is_nan_bits(uint32_t u) {
  return (u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu) != 0u;
}

// Inclusive warp scan of an int.
__device__ __forceinline__ int warp_inclusive_scan(int v) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    int n = __shfl_up_sync(0xffffffffu, v, o);
    if ((threadIdx.x & 31) >= o) v += n;
  }
  return v;
}

// Exclusive block scan of one int per thread; returns the prefix and writes the block total.
// `scratch` holds at least NWARPS ints.  Must be called by every thread of the block.
template <int NWARPS>
__device__ __forceinline__ int block_exclusive_scan(int v, int* scratch, int& total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int inc = warp_inclusive_scan(v);
  if (lane == 31) scratch[warp] = inc;
  __syncthreads();
  int wsum = (lane < NWARPS) ? scratch[lane] : 0;
  int winc = warp_inclusive_scan(wsum);
  int wprefix = __shfl_sync(0xffffffffu, winc - wsum, warp);
  total = __shfl_sync(0xffffffffu, winc, NWARPS - 1);
  __syncthreads();
  return wprefix + inc - v;
}

}  // namespace dsa
