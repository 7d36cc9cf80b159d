// Host side of the C ABI declared in include/dsa.h: argument validation, TMA descriptor
// encoding and kernel launches.  Every entry point enqueues on the caller's stream and
// returns without synchronising.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "../../include/dsa.h"
#include "common.cuh"
#include "topk.cuh"

namespace dsa {
namespace {

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

inline dsa_status launch_status() {
  return cudaGetLastError() == cudaSuccess ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace
}  // namespace dsa

using namespace dsa;

extern "C" {

const char* dsa_status_string(int32_t status) {
  switch (status) {
    case DSA_OK: return "ok";
    case DSA_ERR_INVALID_ARGUMENT: return "invalid argument";
    case DSA_ERR_UNSUPPORTED: return "unsupported shape or configuration";
    case DSA_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
    case DSA_ERR_CUDA: return "CUDA error";
    case DSA_ERR_TIMEOUT: return "device-side wait timed out";
    case DSA_ERR_DEVICE_CHECK: return "device-side input check failed";
    default: return "unknown status";
  }
}

dsa_status dsa_device_error(int32_t* code, void* stream) {
  if (code == nullptr) return DSA_ERR_INVALID_ARGUMENT;
  cudaStream_t s = as_stream(stream);
  int32_t v = 0;
  if (cudaMemcpyFromSymbolAsync(&v, g_device_error, sizeof(v), 0, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return DSA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return DSA_ERR_CUDA;
  const int32_t zero = 0;
  if (cudaMemcpyToSymbolAsync(g_device_error, &zero, sizeof(zero), 0, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return DSA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return DSA_ERR_CUDA;
  *code = v;
  return DSA_OK;
}

dsa_status dsa_topk(const float* scores, int64_t ld_scores, int64_t rows, const int32_t* row_len, int32_t k,
                    int32_t* idx, void* stream) {
  if (rows < 0 || k <= 0 || ld_scores <= 0 || (ld_scores % 4) != 0) return DSA_ERR_INVALID_ARGUMENT;
  if (rows == 0) return DSA_OK;
  if (scores == nullptr || row_len == nullptr || idx == nullptr || !aligned(scores, 16))
    return DSA_ERR_INVALID_ARGUMENT;
  if (rows > 0x7FFFFFFFLL || ld_scores > 0x7FFFFFFFLL) return DSA_ERR_UNSUPPORTED;
  topk_rows_kernel<<<static_cast<unsigned>(rows), kTopkThreads, 0, as_stream(stream)>>>(scores, ld_scores, row_len,
                                                                                       k, idx);
  return launch_status();
}

dsa_status dsa_indexer_scores(const uint8_t*, const float*, const float*, const dsa_kv_desc*, int32_t, int32_t,
                              int32_t, int64_t, int64_t, float*, int64_t, void*) {
  return DSA_ERR_UNSUPPORTED;
}

dsa_status dsa_sparse_mla_prefill(const void*, const dsa_kv_desc*, const int32_t*, int32_t, int32_t, int32_t, float,
                                  void*, float*, void*) {
  return DSA_ERR_UNSUPPORTED;
}

dsa_status dsa_sparse_mla_decode(const void*, const dsa_kv_desc*, const int32_t*, int32_t, int32_t, int32_t, float,
                                 void*, float*, void*, size_t, void*) {
  return DSA_ERR_UNSUPPORTED;
}

dsa_status dsa_forward(int32_t, const uint8_t*, const float*, const float*, const dsa_kv_desc*, const void*,
                       const dsa_kv_desc*, int32_t, int32_t, int32_t, int32_t, int32_t, float, void*, float*,
                       int32_t*, void*, size_t, void*) {
  return DSA_ERR_UNSUPPORTED;
}

size_t dsa_workspace_size(int32_t, int32_t, int64_t, int32_t, int32_t, int32_t, int32_t) { return 0; }

}  // extern "C"
