// noalloc.cu -- split-KV attention for callers that cannot allocate device memory.
//
// cpattn_fwd_split needs a scratch workspace for its per-range partial results, and its
// caller provides that buffer.  Some callers have no way to obtain one: code that runs
// inside a host runtime that owns all device memory and offers no workspace hook (an
// inference-engine plugin, for instance), or a latency-critical loop that must not call
// cudaMalloc/cudaFree, which can synchronize the whole device.  This file gives them one
// more entry point whose scratch is a fixed device array compiled into the library.
#include <cuda_runtime.h>

#include <cstddef>
#include <mutex>

#include "cpattn.h"

namespace {

// The scratch: 64 MiB, enough for e.g. two key ranges of a [1][5520][16][128] bf16 query
// slice (46 MB) or eight ranges of [1][512][16][128] (17 MB).  Every GPU that loads this
// library holds it until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;

// Device address of g_noalloc_scratch on the current device.  In host code the name
// g_noalloc_scratch is only a host-side stand-in for the symbol, never a device address, so
// it is looked up with cudaGetSymbolAddress -- once per device, with that device current,
// on the first call made on it -- and only the looked-up pointer is handed to kernels.
// Under CUDA's lazy module loading (the default) this first lookup is also what loads the
// module holding the array, so the first call on a device may reserve its 64 MiB and
// synchronize; later calls only read the cached pointer.
void* scratch_on_current_device(int* status) {
  static void* addr[kMaxDevices] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *status = CPATTN_ERR_CUDA;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      *status = CPATTN_ERR_CUDA;
      return nullptr;
    }
    addr[dev] = p;
  }
  *status = CPATTN_OK;
  return addr[dev];
}

}  // namespace

extern "C" {

size_t cpattn_noalloc_scratch_bytes(void) { return kNoAllocScratchBytes; }

int cpattn_fwd_split_noalloc(const void* q, const void* k, const void* v, void* out, float* lse,
                             int B, int H, int Sq, int Skv, int D, float scale, int out_dtype,
                             int accumulate, int n_split, cpattn_stream_t stream) {
  // The size check comes first and needs no CUDA call: a request whose partials do not fit
  // in the fixed scratch is refused before anything is set up or launched.  It is made for
  // the split count cpattn_fwd_split will actually use: that call lowers n_split to the
  // number of 128-key blocks (every range holds at least one), so a request such as
  // n_split = 8 over 256 keys needs the scratch of two ranges, not eight.
  // For the tail split (n_split = 0) it is made for this call's own plan, which depends on
  // the key count: cpattn_fwd_split_workspace_kv gives the exact need either way.
  if (cpattn_fwd_split_workspace_kv(B, H, Sq, Skv, D, n_split, out_dtype) > kNoAllocScratchBytes)
    return CPATTN_ERR_SHAPE;
  int status = CPATTN_OK;
  void* scratch = scratch_on_current_device(&status);
  if (scratch == nullptr) return status;
  // Every byte of the scratch that a call reads is written earlier in the same call (each
  // key range writes all of its partial rows and LSEs before the combine reads them), so
  // nothing has to be cleared between calls.
  return cpattn_fwd_split(q, k, v, out, lse, B, H, Sq, Skv, D, scale, out_dtype, accumulate,
                          n_split, scratch, kNoAllocScratchBytes, stream);
}

}  // extern "C"
