/*
 * A plain C99 program that uses the DSA library through include/dsa.h alone: no Python and
 * no torch, device memory from the CUDA runtime.
 *
 *   consumer host   host-side checks only, no GPU needed: status strings and the argument
 *                   validation of several entry points (each returns before any launch);
 *   consumer        the host checks, then a top-k (method step 2: per row the min(k, len)
 *                   largest scores, ties to the lower index, -0.0 == +0.0, ascending, -1
 *                   padded) over device score rows, compared with a brute-force selection
 *                   computed here, and the bounded-wait self-test reported through
 *                   dsa_device_error.
 * Exit status 0 and "dsa C consumer: ok" on success.
 */
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "dsa.h"

#define CHECK(cond, ...)                \
  do {                                  \
    if (!(cond)) {                      \
      fprintf(stderr, __VA_ARGS__);     \
      fputc('\n', stderr);              \
      return 1;                         \
    }                                   \
  } while (0)

#define CUDA_CHECK(call) CHECK((call) == cudaSuccess, "%s failed", #call)

enum { ROWS = 6, N = 700, K = 64 };

static int host_checks(void) {
  void* fake = (void*)(uintptr_t)4096; /* never dereferenced: every call below fails validation */
  CHECK(strlen(dsa_status_string(DSA_OK)) > 0, "empty status string");
  CHECK(strcmp(dsa_status_string(DSA_ERR_TIMEOUT), dsa_status_string(DSA_OK)) != 0, "status strings alike");
  CHECK(dsa_topk((const float*)fake, 8, 4, (const int32_t*)fake, 0, (int32_t*)fake, NULL) ==
            DSA_ERR_INVALID_ARGUMENT, "dsa_topk accepted k = 0");
  CHECK(dsa_topk((const float*)fake, 6, 4, (const int32_t*)fake, 4, (int32_t*)fake, NULL) ==
            DSA_ERR_INVALID_ARGUMENT, "dsa_topk accepted ld_scores not a multiple of 4");
  CHECK(dsa_topk(NULL, 8, 4, NULL, 4, NULL, NULL) == DSA_ERR_INVALID_ARGUMENT, "dsa_topk accepted NULL");
  CHECK(dsa_topk(NULL, 8, 0, NULL, 4, NULL, NULL) == DSA_OK, "zero rows is not a no-op");
  CHECK(dsa_quantize_fp8(fake, 4, 12, (uint8_t*)fake, (float*)fake, NULL) == DSA_ERR_INVALID_ARGUMENT,
        "dsa_quantize_fp8 accepted cols not a multiple of 8");
  CHECK(dsa_workspace_size(DSA_MODE_PREFILL, 0, 10, 10, 128, 2048) == 0, "workspace for B = 0");
  CHECK(dsa_workspace_size(DSA_MODE_PREFILL, 1, 1000, 1000, 128, 2048) >= (size_t)1000 * 2048 * 4,
        "prefill workspace smaller than the selection");
  return 0;
}

/* Brute-force selection of one row: index i is kept when fewer than m indices beat it. */
static void reference_topk(const float* s, int len, int k, int32_t* out) {
  int m = len < k ? len : k, n = 0, i, j;
  for (i = 0; i < len; ++i) {
    int beaten = 0;
    for (j = 0; j < len && beaten < m; ++j)
      if (s[j] > s[i] || (s[j] == s[i] && j < i)) ++beaten;
    if (beaten < m) out[n++] = i;
  }
  while (n < k) out[n++] = -1;
}

static int device_checks(void) {
  static const int32_t row_len[ROWS] = {1, 63, 64, 65, 333, N};
  static float h_scores[ROWS * N];
  static int32_t h_idx[ROWS * K], ref[K];
  float* d_scores = NULL;
  int32_t *d_len = NULL, *d_idx = NULL;
  int32_t code = -1;
  int r, i;
  /* few distinct values (many ties), with signed zeros mixed in */
  for (r = 0; r < ROWS; ++r)
    for (i = 0; i < N; ++i) {
      int v = (i * 37 + r * 11) % 29 - 14;
      h_scores[r * N + i] = (v == 0 && (i & 1)) ? -0.0f : (float)v * 0.25f;
    }
  CUDA_CHECK(cudaMalloc((void**)&d_scores, sizeof(h_scores)));
  CUDA_CHECK(cudaMalloc((void**)&d_len, sizeof(row_len)));
  CUDA_CHECK(cudaMalloc((void**)&d_idx, sizeof(h_idx)));
  CUDA_CHECK(cudaMemcpy(d_scores, h_scores, sizeof(h_scores), cudaMemcpyHostToDevice));
  CUDA_CHECK(cudaMemcpy(d_len, row_len, sizeof(row_len), cudaMemcpyHostToDevice));
  CHECK(dsa_topk(d_scores, N, ROWS, d_len, K, d_idx, NULL) == DSA_OK, "dsa_topk launch");
  CUDA_CHECK(cudaMemcpy(h_idx, d_idx, sizeof(h_idx), cudaMemcpyDeviceToHost));
  CHECK(dsa_device_error(&code, NULL) == DSA_OK && code == DSA_OK, "device error %d after dsa_topk", code);
  for (r = 0; r < ROWS; ++r) {
    reference_topk(h_scores + r * N, row_len[r], K, ref);
    CHECK(memcmp(ref, h_idx + r * K, sizeof(ref)) == 0, "row %d: selection differs from brute force", r);
  }
  /* a bounded wait that nothing completes: the kernel records DSA_ERR_TIMEOUT and returns */
  CHECK(dsa_selftest_wait_timeout(20000, NULL) == DSA_OK, "self-test launch");
  CHECK(dsa_device_error(&code, NULL) == DSA_OK && code == DSA_ERR_TIMEOUT, "self-test reported %d", code);
  CHECK(dsa_device_error(&code, NULL) == DSA_OK && code == DSA_OK, "device error word not cleared");
  CUDA_CHECK(cudaFree(d_scores));
  CUDA_CHECK(cudaFree(d_len));
  CUDA_CHECK(cudaFree(d_idx));
  return 0;
}

int main(int argc, char** argv) {
  int host_only = argc > 1 && strcmp(argv[1], "host") == 0;
  if (host_checks() != 0) return 1;
  if (!host_only && device_checks() != 0) return 1;
  printf("dsa C consumer: ok (%s)\n", host_only ? "host checks" : "host and device checks");
  return 0;
}
