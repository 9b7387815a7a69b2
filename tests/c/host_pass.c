/* Plain-C user of cpattn_ulysses_host on a GPU: Q/K/V rank shards in page-locked host
 * memory, O and LSE back into host memory, with caller-owned device work buffers.  The
 * result must equal, byte for byte, the device-resident path driven by hand (copies in,
 * cpattn_ulysses_fwd, copies out).  Uses only the CUDA runtime's C API.  Exit status 0 =
 * all checks passed; 77 = no CUDA device. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include <cuda_runtime_api.h>

#include "cpattn.h"

#define CHECK(x)                                                            \
  do {                                                                      \
    cudaError_t e_ = (x);                                                   \
    if (e_ != cudaSuccess) {                                                \
      fprintf(stderr, "%s: %s\n", #x, cudaGetErrorString(e_));              \
      return 1;                                                             \
    }                                                                       \
  } while (0)

/* bf16 bits of a value in about [-2, 2) from a 32-bit LCG (input data only) */
static uint16_t next_bf16(uint32_t* s) {
  *s = *s * 1664525u + 1013904223u;
  const uint32_t mant = (*s >> 9) & 0x7Fu, sign = (*s >> 31) & 1u;
  const uint32_t expo = 126u + ((*s >> 16) & 1u); /* 2^-1 or 2^0 */
  return (uint16_t)((sign << 15) | (expo << 7) | mant);
}

int main(void) {
  int n_dev = 0;
  if (cudaGetDeviceCount(&n_dev) != cudaSuccess || n_dev < 1) {
    printf("no CUDA device\n");
    return 77;
  }
  enum { P = 4, SL = 272, H = 8, D = 128 };
  const size_t n = (size_t)P * SL * H * D, n_lse = (size_t)H * P * SL;
  const size_t b_in = n * 2, b_lse = n_lse * 4;
  uint16_t *hq, *hk, *hv, *ho, *ho2;
  float *hl, *hl2;
  void *dq, *dk, *dv, *dout, *dq2, *dk2, *dv2, *dout2;
  float *dl, *dl2;
  CHECK(cudaMallocHost((void**)&hq, b_in));
  CHECK(cudaMallocHost((void**)&hk, b_in));
  CHECK(cudaMallocHost((void**)&hv, b_in));
  CHECK(cudaMallocHost((void**)&ho, b_in));
  CHECK(cudaMallocHost((void**)&ho2, b_in));
  CHECK(cudaMallocHost((void**)&hl, b_lse));
  CHECK(cudaMallocHost((void**)&hl2, b_lse));
  CHECK(cudaMalloc(&dq, b_in));
  CHECK(cudaMalloc(&dk, b_in));
  CHECK(cudaMalloc(&dv, b_in));
  CHECK(cudaMalloc(&dout, b_in));
  CHECK(cudaMalloc((void**)&dl, b_lse));
  CHECK(cudaMalloc(&dq2, b_in));
  CHECK(cudaMalloc(&dk2, b_in));
  CHECK(cudaMalloc(&dv2, b_in));
  CHECK(cudaMalloc(&dout2, b_in));
  CHECK(cudaMalloc((void**)&dl2, b_lse));
  uint32_t seed = 12345u;
  for (size_t i = 0; i < n; ++i) {
    hq[i] = next_bf16(&seed);
    hk[i] = next_bf16(&seed);
    hv[i] = next_bf16(&seed);
  }
  memset(ho, 0xFF, b_in);
  memset(hl, 0xFF, b_lse);
  cudaStream_t st;
  CHECK(cudaStreamCreate(&st));
  const float scale = 0.08838834764831845f; /* 1 / sqrt(128) */
  int rc = cpattn_ulysses_host(hq, hk, hv, ho, hl, dq, dk, dv, dout, dl, P, SL, H, D, scale,
                               CPATTN_BF16, 2, (cpattn_stream_t)st);
  if (rc != CPATTN_OK) {
    fprintf(stderr, "cpattn_ulysses_host: %s\n", cpattn_status_str(rc));
    return 1;
  }
  CHECK(cudaStreamSynchronize(st));
  /* the same layer by hand on separate buffers */
  CHECK(cudaMemcpy(dq2, hq, b_in, cudaMemcpyHostToDevice));
  CHECK(cudaMemcpy(dk2, hk, b_in, cudaMemcpyHostToDevice));
  CHECK(cudaMemcpy(dv2, hv, b_in, cudaMemcpyHostToDevice));
  rc = cpattn_ulysses_fwd(dq2, dk2, dv2, dout2, dl2, P, SL, H, D, scale, CPATTN_BF16,
                          (cpattn_stream_t)st);
  if (rc != CPATTN_OK) {
    fprintf(stderr, "cpattn_ulysses_fwd: %s\n", cpattn_status_str(rc));
    return 1;
  }
  CHECK(cudaStreamSynchronize(st));
  CHECK(cudaMemcpy(ho2, dout2, b_in, cudaMemcpyDeviceToHost));
  CHECK(cudaMemcpy(hl2, dl2, b_lse, cudaMemcpyDeviceToHost));
  if (cpattn_device_error() != CPATTN_OK) {
    fprintf(stderr, "a bounded wait ran out\n");
    return 1;
  }
  if (memcmp(ho, ho2, b_in) != 0 || memcmp(hl, hl2, b_lse) != 0) {
    fprintf(stderr, "host pass differs from the device path\n");
    return 1;
  }
  printf("cpattn_ulysses_host from C: all checks passed\n");
  return 0;
}
