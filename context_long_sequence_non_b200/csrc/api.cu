// api.cu -- the C ABI of include/cpattn.h: host-side argument checks, TMA tensor-map
// encoding, dispatch to the kernels, and the per-device error word.
#include <cuda.h>
#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "cpattn.h"
#include "kernels.h"
#include "sm100_ptx.cuh"

namespace {

// One word per device; kernels record bounded-wait timeouts here (atomicOr).
__device__ int g_cpattn_err;

constexpr int kMaxDevices = 64;

int* device_error_word() {
  static int* addr[kMaxDevices] = {nullptr};
  static std::mutex mu;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_cpattn_err) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<int*>(p);
  }
  return addr[dev];
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return nullptr;
    return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }();
  return fn;
}

// [B][S][H][D] bf16 tensor, box = 64 head-dim columns x 1 head x `box_rows` tokens x 1
// batch, 128-byte swizzle (the layout tcgen05 reads through a 128-byte-swizzle descriptor).
bool encode_bshd_bf16(CUtensorMap* map, const void* ptr, int B, int S, int H, int D,
                      unsigned box_rows = 128) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[4] = {cuuint64_t(D), cuuint64_t(H), cuuint64_t(S), cuuint64_t(B)};
  const cuuint64_t strides[3] = {cuuint64_t(D) * 2, cuuint64_t(H) * D * 2,
                                 cuuint64_t(S) * H * D * 2};
  const cuuint32_t box[4] = {64, 1, box_rows, 1};
  const cuuint32_t estr[4] = {1, 1, 1, 1};
  const CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(ptr), dims,
                        strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool overlap(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return x < y + nb && y < x + na;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? CPATTN_OK : CPATTN_ERR_CUDA; }

int elem_size(int dtype) { return dtype == CPATTN_BF16 ? 2 : (dtype == CPATTN_F32 ? 4 : 0); }

}  // namespace

extern "C" {

int cpattn_version(void) { return (1 << 16) | 0; }

const char* cpattn_status_str(int status) {
  switch (status) {
    case CPATTN_OK: return "CPATTN_OK";
    case CPATTN_ERR_NULL: return "CPATTN_ERR_NULL: a required pointer is NULL";
    case CPATTN_ERR_SHAPE: return "CPATTN_ERR_SHAPE: a size is out of range or inconsistent";
    case CPATTN_ERR_ALIGN: return "CPATTN_ERR_ALIGN: a pointer is not suitably aligned";
    case CPATTN_ERR_UNSUPPORTED: return "CPATTN_ERR_UNSUPPORTED: no kernel for this dtype/size";
    case CPATTN_ERR_CUDA: return "CPATTN_ERR_CUDA: a CUDA call or kernel launch failed";
    case CPATTN_ERR_DEVICE_TIMEOUT:
      return "CPATTN_ERR_DEVICE_TIMEOUT: a kernel's bounded wait ran out";
    default: return "CPATTN: unknown status";
  }
}

}  // extern "C"

namespace {

int fwd_impl(const void* q, const void* k, const void* v, void* out, float* lse, int B, int H,
             int Sq, int Skv, int D, float scale, int in_dtype, int out_dtype, bool accumulate,
             cpattn_stream_t stream) {
  if (B < 1 || H < 1 || Sq < 1 || Skv < 0 || D < 1) return CPATTN_ERR_SHAPE;
  if (!(std::isfinite(scale) && scale > 0.f)) return CPATTN_ERR_SHAPE;
  const int in_es = elem_size(in_dtype), out_es = elem_size(out_dtype);
  if (in_es == 0 || out_es == 0) return CPATTN_ERR_UNSUPPORTED;
  if (accumulate && in_dtype != CPATTN_BF16) return CPATTN_ERR_UNSUPPORTED;
  if (q == nullptr || out == nullptr) return CPATTN_ERR_NULL;
  if (accumulate && lse == nullptr) return CPATTN_ERR_NULL;
  if (Skv > 0 && (k == nullptr || v == nullptr)) return CPATTN_ERR_NULL;
  if (!aligned(q, 16) || !aligned(out, 16) || (Skv > 0 && (!aligned(k, 16) || !aligned(v, 16))) ||
      (lse != nullptr && !aligned(lse, 4)))
    return CPATTN_ERR_ALIGN;
  if (in_dtype == CPATTN_BF16 && D != 64 && D != 128) return CPATTN_ERR_UNSUPPORTED;
  if (in_dtype == CPATTN_F32 && D > 256) return CPATTN_ERR_UNSUPPORTED;
  if (B > 65535 || H > 65535) return CPATTN_ERR_SHAPE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const size_t out_bytes = size_t(B) * Sq * H * D * out_es;
  if (Skv == 0) {
    if (accumulate) return CPATTN_OK;  // merging an empty key set changes nothing
    if (out_bytes % 16 != 0) return CPATTN_ERR_SHAPE;
    return cuda_status(cpattn::launch_fill_empty(out, out_bytes, lse, size_t(B) * H * Sq, st));
  }
  if (in_dtype == CPATTN_BF16) {
    int* err = device_error_word();
    if (err == nullptr) return CPATTN_ERR_CUDA;
    CUtensorMap tq, tk, tv;
    if (!encode_bshd_bf16(&tq, q, B, Sq, H, D) || !encode_bshd_bf16(&tk, k, B, Skv, H, D) ||
        !encode_bshd_bf16(&tv, v, B, Skv, H, D))
      return CPATTN_ERR_CUDA;
    const float scale_log2 = float(double(scale) * 1.4426950408889634074);
    return cuda_status(cpattn::launch_attn_fwd_sm100(
        tq, tk, tv, out, lse, B, H, Sq, Skv, D, scale_log2, cpattn::kRescaleLog2,
        out_dtype == CPATTN_F32, accumulate, 1, err, cpattn::kDefaultWaitLimit, st));
  }
  // fp32 inputs: CUDA-core kernel
  return cuda_status(cpattn::launch_attn_fwd_f32(
      static_cast<const float*>(q), static_cast<const float*>(k), static_cast<const float*>(v),
      out, lse, B, H, Sq, Skv, D, scale, out_dtype == CPATTN_BF16, st));
}

}  // namespace

extern "C" {

int cpattn_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int B, int H,
               int Sq, int Skv, int D, float scale, int in_dtype, int out_dtype,
               cpattn_stream_t stream) {
  return fwd_impl(q, k, v, out, lse, B, H, Sq, Skv, D, scale, in_dtype, out_dtype, false, stream);
}

int cpattn_fwd_accumulate(const void* q, const void* k, const void* v, void* o_acc,
                          float* lse_acc, int B, int H, int Sq, int Skv, int D, float scale,
                          int in_dtype, int acc_dtype, cpattn_stream_t stream) {
  return fwd_impl(q, k, v, o_acc, lse_acc, B, H, Sq, Skv, D, scale, in_dtype, acc_dtype, true,
                  stream);
}

}  // extern "C"

namespace {

constexpr int kMaxSplit = 8;

size_t split_o_bytes(int B, int H, int Sq, int D, int n, int es) {
  const size_t o = size_t(n) * B * Sq * H * D * es;
  return (o + 255) & ~size_t(255);
}

size_t split_ws_bytes(int B, int H, int Sq, int D, int n, int es) {
  return split_o_bytes(B, H, Sq, D, n, es) + size_t(n) * B * H * Sq * sizeof(float);
}

}  // namespace

extern "C" {

size_t cpattn_fwd_split_workspace(int B, int H, int Sq, int D, int n_split, int out_dtype) {
  const int es = elem_size(out_dtype);
  if (B < 1 || H < 1 || Sq < 1 || D < 1 || n_split < 0 || n_split > kMaxSplit || es == 0)
    return 0;
  if (n_split == 0) {
    // tail split: the plan depends on the key count, which this query does not take; size
    // the workspace for the largest plan any key count can give
    if (D != 64 && D != 128) return 0;
    return cpattn::tail_split_workspace_bound(B, H, Sq, D);
  }
  return n_split == 1 ? 0 : split_ws_bytes(B, H, Sq, D, n_split, es);
}

size_t cpattn_fwd_split_workspace_kv(int B, int H, int Sq, int Skv, int D, int n_split,
                                     int out_dtype) {
  const int es = elem_size(out_dtype);
  if (B < 1 || H < 1 || Sq < 1 || Skv < 1 || D < 1 || n_split < 0 || n_split > kMaxSplit ||
      es == 0)
    return 0;
  if (n_split == 0) {
    if (D != 64 && D != 128) return 0;
    return cpattn::tail_split_workspace(cpattn::tail_split_plan(B, H, Sq, Skv), D);
  }
  const int n_kv = (Skv + 127) / 128;
  const int n = n_split > n_kv ? n_kv : n_split;  // the lowering cpattn_fwd_split applies
  return n <= 1 ? 0 : split_ws_bytes(B, H, Sq, D, n, es);
}

int cpattn_split_suggest(int B, int H, int Sq, int Skv) {
  if (B < 1 || H < 1 || Sq < 1 || Skv < 1) return 1;
  const long long ctas = (long long)((Sq + 255) / 256) * H * B;
  const int sms = cpattn::sm_count();
  const int n_kv = (Skv + 127) / 128;
  if (ctas >= 4LL * sms) return 1;  // already four or more waves: little tail to recover
  // modelled time per split count: waves of CTAs that each do 1/s of the key blocks, plus
  // a per-CTA start-up (prologue, pipeline fill, epilogue) worth ~10 key blocks -- measured:
  // a 352-CTA grid of 43-block CTAs gains nothing from two ranges -- and a combine pass of
  // ~1 block per split
  double best = 1e30;
  int best_s = 1;
  for (int sp = 1; sp <= kMaxSplit && n_kv / sp >= 4; ++sp) {
    const long long waves = (ctas * sp + sms - 1) / sms;
    const double t = double(waves) * (double(n_kv) / sp + 10.0) + (sp > 1 ? sp : 0);
    if (t < best * 0.97) {
      best = t;
      best_s = sp;
    }
  }
  return best_s;
}

int cpattn_fwd_split(const void* q, const void* k, const void* v, void* out, float* lse, int B,
                     int H, int Sq, int Skv, int D, float scale, int out_dtype, int accumulate,
                     int n_split, void* workspace, size_t workspace_bytes,
                     cpattn_stream_t stream) {
  if (n_split < 0 || n_split > kMaxSplit) return CPATTN_ERR_SHAPE;
  const int n_kv = Skv > 0 ? (Skv + 127) / 128 : 0;
  cpattn::TailSplit tail{};
  if (n_split == 0) {  // tail split: only the items of the last wave or two are split
    if (B >= 1 && H >= 1 && Sq >= 1 && Skv >= 1) tail = cpattn::tail_split_plan(B, H, Sq, Skv);
    if (tail.parts < 2) n_split = 1;
  } else if (n_split > n_kv) {
    n_split = n_kv > 0 ? n_kv : 1;  // every range holds a key block
  }
  if (n_split == 1)
    return fwd_impl(q, k, v, out, lse, B, H, Sq, Skv, D, scale, CPATTN_BF16, out_dtype,
                    accumulate != 0, stream);
  // validate the call exactly as the single-pass form would (no launch yet)
  if (B < 1 || H < 1 || Sq < 1 || D < 1) return CPATTN_ERR_SHAPE;
  if (!(std::isfinite(scale) && scale > 0.f)) return CPATTN_ERR_SHAPE;
  const int es = elem_size(out_dtype);
  if (es == 0) return CPATTN_ERR_UNSUPPORTED;
  if (D != 64 && D != 128) return CPATTN_ERR_UNSUPPORTED;
  if (B > 65535 || H > 65535) return CPATTN_ERR_SHAPE;
  if (!q || !k || !v || !out || !workspace) return CPATTN_ERR_NULL;
  if (accumulate && lse == nullptr) return CPATTN_ERR_NULL;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      !aligned(workspace, 256) || (lse != nullptr && !aligned(lse, 4)))
    return CPATTN_ERR_ALIGN;
  const size_t need = n_split == 0 ? cpattn::tail_split_workspace(tail, D)
                                    : split_ws_bytes(B, H, Sq, D, n_split, es);
  if (workspace_bytes < need) return CPATTN_ERR_SHAPE;
  if ((long long)B * Sq * H > 0x7fffffffLL) return CPATTN_ERR_SHAPE;  // 32-bit row index
  int* err = device_error_word();
  if (err == nullptr) return CPATTN_ERR_CUDA;
  CUtensorMap tq, tk, tv;
  if (!encode_bshd_bf16(&tq, q, B, Sq, H, D) || !encode_bshd_bf16(&tk, k, B, Skv, H, D) ||
      !encode_bshd_bf16(&tv, v, B, Skv, H, D))
    return CPATTN_ERR_CUDA;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  if (n_split == 0) {
    const float scale_log2 = float(double(scale) * 1.4426950408889634074);
    return cuda_status(cpattn::launch_attn_fwd_sm100_tail(
        tq, tk, tv, out, lse, B, H, Sq, Skv, D, scale_log2, cpattn::kRescaleLog2,
        out_dtype == CPATTN_F32, accumulate != 0, tail, workspace, err, cpattn::kDefaultWaitLimit,
        st));
  }
  void* part_o = workspace;
  float* part_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                             split_o_bytes(B, H, Sq, D, n_split, es));
  const float scale_log2 = float(double(scale) * 1.4426950408889634074);
  cudaError_t e = cpattn::launch_attn_fwd_sm100(
      tq, tk, tv, part_o, part_lse, B, H, Sq, Skv, D, scale_log2, cpattn::kRescaleLog2,
      out_dtype == CPATTN_F32, false, n_split, err, cpattn::kDefaultWaitLimit, st);
  if (e != cudaSuccess) return CPATTN_ERR_CUDA;
  return cuda_status(cpattn::launch_combine(part_o, part_lse, n_split, out, lse, B, H, Sq, D, es,
                                            accumulate != 0, st));
}

}  // extern "C"

namespace {

// Checks shared by the device and host Ulysses calls (no CUDA call).
int ulysses_args(const void* q, const void* k, const void* v, const void* out, const float* lse,
                 int P, int S_local, int H, int D, float scale, int out_dtype) {
  if (P < 1 || S_local < 1 || H < 1 || D < 1) return CPATTN_ERR_SHAPE;
  if (H % P != 0) return CPATTN_ERR_SHAPE;
  if ((long long)P * S_local > 0x7fffffffLL || P > 65535 || H / P > 65535) return CPATTN_ERR_SHAPE;
  if (!(std::isfinite(scale) && scale > 0.f)) return CPATTN_ERR_SHAPE;
  if (elem_size(out_dtype) == 0) return CPATTN_ERR_UNSUPPORTED;
  if (D != 64 && D != 128) return CPATTN_ERR_UNSUPPORTED;
  if (S_local % 16 != 0) return CPATTN_ERR_UNSUPPORTED;  // 16-row boxes may not cross shards
  if (!q || !k || !v || !out) return CPATTN_ERR_NULL;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16) ||
      (lse != nullptr && !aligned(lse, 4)))
    return CPATTN_ERR_ALIGN;
  return CPATTN_OK;
}

struct UlyssesMaps {
  CUtensorMap q, k, v, q16, k16, v16;
};

bool encode_ulysses(UlyssesMaps* m, const void* q, const void* k, const void* v, int P,
                    int S_local, int H, int D) {
  return encode_bshd_bf16(&m->q, q, P, S_local, H, D) && encode_bshd_bf16(&m->k, k, P, S_local, H, D) &&
         encode_bshd_bf16(&m->v, v, P, S_local, H, D) &&
         encode_bshd_bf16(&m->q16, q, P, S_local, H, D, 16) &&
         encode_bshd_bf16(&m->k16, k, P, S_local, H, D, 16) &&
         encode_bshd_bf16(&m->v16, v, P, S_local, H, D, 16);
}

// Per-device streams and events of the host-buffer pass, created on the first call on a
// device and kept until the process exits (no device memory is involved).  The mutex is
// held while a call enqueues its work, so that one event can be recorded and waited on
// again and again: every wait is enqueued right after the record it refers to.
struct HostPassResources {
  std::mutex mu;
  bool ready = false;
  cudaStream_t upload = nullptr, download = nullptr, compute2 = nullptr;
  cudaEvent_t start = nullptr, uploaded = nullptr, computed = nullptr, done = nullptr;
};

HostPassResources* host_pass_resources(int* status) {
  static HostPassResources res[kMaxDevices];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    *status = CPATTN_ERR_CUDA;
    return nullptr;
  }
  HostPassResources* r = &res[dev];
  *status = CPATTN_OK;
  return r;
}

bool host_pass_init(HostPassResources* r) {  // with r->mu held
  if (r->ready) return true;
  const unsigned sf = cudaStreamNonBlocking, ef = cudaEventDisableTiming;
  if (cudaStreamCreateWithFlags(&r->upload, sf) != cudaSuccess ||
      cudaStreamCreateWithFlags(&r->download, sf) != cudaSuccess ||
      cudaStreamCreateWithFlags(&r->compute2, sf) != cudaSuccess ||
      cudaEventCreateWithFlags(&r->start, ef) != cudaSuccess ||
      cudaEventCreateWithFlags(&r->uploaded, ef) != cudaSuccess ||
      cudaEventCreateWithFlags(&r->computed, ef) != cudaSuccess ||
      cudaEventCreateWithFlags(&r->done, ef) != cudaSuccess)
    return false;
  r->ready = true;
  return true;
}

}  // namespace

extern "C" {

int cpattn_ulysses_fwd(const void* q, const void* k, const void* v, void* out, float* lse, int P,
                       int S_local, int H, int D, float scale, int out_dtype,
                       cpattn_stream_t stream) {
  const int st = ulysses_args(q, k, v, out, lse, P, S_local, H, D, scale, out_dtype);
  if (st != CPATTN_OK) return st;
  int* err = device_error_word();
  if (err == nullptr) return CPATTN_ERR_CUDA;
  UlyssesMaps m;
  if (!encode_ulysses(&m, q, k, v, P, S_local, H, D)) return CPATTN_ERR_CUDA;
  const float scale_log2 = float(double(scale) * 1.4426950408889634074);
  return cuda_status(cpattn::launch_ulysses_fwd_sm100(
      m.q, m.k, m.v, m.q16, m.k16, m.v16, out, lse, P, S_local, H, D, scale_log2,
      cpattn::kRescaleLog2, out_dtype == CPATTN_F32, 0, P, err, cpattn::kDefaultWaitLimit,
      reinterpret_cast<cudaStream_t>(stream)));
}

size_t cpattn_ulysses_fwd_workspace(int P, int S_local, int H, int D, int out_dtype) {
  if (P < 1 || S_local < 1 || H < 1 || H % P != 0 || elem_size(out_dtype) == 0) return 0;
  if ((D != 64 && D != 128) || (long long)P * S_local > 0x7fffffffLL) return 0;
  const int S = P * S_local;
  return cpattn::tail_split_workspace(cpattn::tail_split_plan(P, H / P, S, S), D);
}

int cpattn_ulysses_fwd_split(const void* q, const void* k, const void* v, void* out, float* lse,
                             int P, int S_local, int H, int D, float scale, int out_dtype,
                             void* workspace, size_t workspace_bytes, cpattn_stream_t stream) {
  const int st = ulysses_args(q, k, v, out, lse, P, S_local, H, D, scale, out_dtype);
  if (st != CPATTN_OK) return st;
  const int S = P * S_local;
  const cpattn::TailSplit tail = cpattn::tail_split_plan(P, H / P, S, S);
  const size_t need = cpattn::tail_split_workspace(tail, D);
  if (need > 0) {
    if (workspace == nullptr) return CPATTN_ERR_NULL;
    if (!aligned(workspace, 256)) return CPATTN_ERR_ALIGN;
    if (workspace_bytes < need) return CPATTN_ERR_SHAPE;
    const size_t io = size_t(S) * H * D;
    const int es = elem_size(out_dtype);
    if (overlap(workspace, need, q, io * 2) || overlap(workspace, need, k, io * 2) ||
        overlap(workspace, need, v, io * 2) || overlap(workspace, need, out, io * es) ||
        (lse != nullptr && overlap(workspace, need, lse, size_t(H) * S * 4)))
      return CPATTN_ERR_SHAPE;
  }
  int* err = device_error_word();
  if (err == nullptr) return CPATTN_ERR_CUDA;
  UlyssesMaps m;
  if (!encode_ulysses(&m, q, k, v, P, S_local, H, D)) return CPATTN_ERR_CUDA;
  const float scale_log2 = float(double(scale) * 1.4426950408889634074);
  const cudaStream_t cs = reinterpret_cast<cudaStream_t>(stream);
  if (need == 0)
    return cuda_status(cpattn::launch_ulysses_fwd_sm100(
        m.q, m.k, m.v, m.q16, m.k16, m.v16, out, lse, P, S_local, H, D, scale_log2,
        cpattn::kRescaleLog2, out_dtype == CPATTN_F32, 0, P, err, cpattn::kDefaultWaitLimit, cs));
  return cuda_status(cpattn::launch_ulysses_fwd_sm100_tail(
      m.q, m.k, m.v, m.q16, m.k16, m.v16, out, lse, P, S_local, H, D, scale_log2,
      cpattn::kRescaleLog2, out_dtype == CPATTN_F32, tail, workspace, err,
      cpattn::kDefaultWaitLimit, cs));
}

int cpattn_ulysses_host(const void* h_q, const void* h_k, const void* h_v, void* h_out,
                        float* h_lse, void* d_q, void* d_k, void* d_v, void* d_out, float* d_lse,
                        int P, int S_local, int H, int D, float scale, int out_dtype, int n_chunks,
                        cpattn_stream_t stream) {
  const int st = ulysses_args(d_q, d_k, d_v, d_out, d_lse, P, S_local, H, D, scale, out_dtype);
  if (st != CPATTN_OK) return st;
  if (n_chunks < 1 || n_chunks > P) return CPATTN_ERR_SHAPE;
  if (!h_q || !h_k || !h_v || !h_out) return CPATTN_ERR_NULL;
  if ((h_lse == nullptr) != (d_lse == nullptr)) return CPATTN_ERR_NULL;
  const int es = elem_size(out_dtype);
  const size_t in_bytes = size_t(P) * S_local * H * D * 2, out_bytes = in_bytes / 2 * es;
  const size_t lse_bytes = size_t(H) * P * S_local * 4;
  const void* dev_bufs[5] = {d_q, d_k, d_v, d_out, d_lse};
  const size_t dev_sizes[5] = {in_bytes, in_bytes, in_bytes, out_bytes, lse_bytes};
  for (int a = 0; a < 5; ++a)
    for (int b = a + 1; b < 5; ++b)
      if (dev_bufs[a] && dev_bufs[b] && overlap(dev_bufs[a], dev_sizes[a], dev_bufs[b], dev_sizes[b]))
        return CPATTN_ERR_SHAPE;
  int* err = device_error_word();
  if (err == nullptr) return CPATTN_ERR_CUDA;
  UlyssesMaps m;
  if (!encode_ulysses(&m, d_q, d_k, d_v, P, S_local, H, D)) return CPATTN_ERR_CUDA;
  int rs = CPATTN_OK;
  HostPassResources* r = host_pass_resources(&rs);
  if (r == nullptr) return rs;
  std::lock_guard<std::mutex> lock(r->mu);
  if (!host_pass_init(r)) return CPATTN_ERR_CUDA;
  cudaStream_t cs[2] = {reinterpret_cast<cudaStream_t>(stream), r->compute2};
  const float scale_log2 = float(double(scale) * 1.4426950408889634074);
  const int Hp = H / P;
  const size_t rows = size_t(P) * S_local;  // token rows of every shard tensor
  // everything below is ordered after the work already on the caller's stream
  cudaError_t e = cudaEventRecord(r->start, cs[0]);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(r->upload, r->start, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(r->download, r->start, 0);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(cs[1], r->start, 0);
  for (int c = 0; e == cudaSuccess && c < n_chunks; ++c) {
    // chunk c = head groups [g0, g1): heads [g0*Hp, g1*Hp) of every token row, a strided
    // slab of each [P][S_l][H][D] tensor (one 2-D copy per tensor and direction)
    const int g0 = int((long long)c * P / n_chunks), g1 = int((long long)(c + 1) * P / n_chunks);
    const size_t in_off = size_t(g0) * Hp * D * 2, in_w = size_t(g1 - g0) * Hp * D * 2;
    const size_t in_pitch = size_t(H) * D * 2;
    const void* hs[3] = {h_q, h_k, h_v};
    void* ds[3] = {d_q, d_k, d_v};
    for (int t = 0; e == cudaSuccess && t < 3; ++t)
      e = cudaMemcpy2DAsync(static_cast<char*>(ds[t]) + in_off, in_pitch,
                            static_cast<const char*>(hs[t]) + in_off, in_pitch, in_w, rows,
                            cudaMemcpyHostToDevice, r->upload);
    if (e == cudaSuccess) e = cudaEventRecord(r->uploaded, r->upload);
    cudaStream_t s = cs[c & 1];  // neighbouring chunks overlap on two compute streams
    if (e == cudaSuccess) e = cudaStreamWaitEvent(s, r->uploaded, 0);
    if (e == cudaSuccess)
      e = cpattn::launch_ulysses_fwd_sm100(m.q, m.k, m.v, m.q16, m.k16, m.v16, d_out, d_lse, P,
                                           S_local, H, D, scale_log2, cpattn::kRescaleLog2,
                                           out_dtype == CPATTN_F32, g0, g1 - g0, err,
                                           cpattn::kDefaultWaitLimit, s);
    if (e == cudaSuccess) e = cudaEventRecord(r->computed, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(r->download, r->computed, 0);
    const size_t out_off = size_t(g0) * Hp * D * es, out_w = size_t(g1 - g0) * Hp * D * es;
    const size_t out_pitch = size_t(H) * D * es;
    if (e == cudaSuccess)
      e = cudaMemcpy2DAsync(static_cast<char*>(h_out) + out_off, out_pitch,
                            static_cast<const char*>(d_out) + out_off, out_pitch, out_w, rows,
                            cudaMemcpyDeviceToHost, r->download);
    if (e == cudaSuccess && h_lse != nullptr) {
      const size_t l_off = size_t(g0) * Hp * rows, l_n = size_t(g1 - g0) * Hp * rows;
      e = cudaMemcpyAsync(h_lse + l_off, d_lse + l_off, l_n * 4, cudaMemcpyDeviceToHost,
                          r->download);
    }
  }
  // the caller's stream resumes once the last copy to the host is done
  if (e == cudaSuccess) e = cudaEventRecord(r->done, r->download);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(cs[0], r->done, 0);
  return cuda_status(e);
}

int cpattn_merge(const void* o_a, const float* lse_a, const void* o_b, const float* lse_b, void* o,
                 float* lse, int B, int H, int S, int D, int dtype, cpattn_stream_t stream) {
  if (B < 1 || H < 1 || S < 1 || D < 1) return CPATTN_ERR_SHAPE;
  const int es = elem_size(dtype);
  if (es == 0) return CPATTN_ERR_UNSUPPORTED;
  if ((D * es) % 16 != 0 || D * es > 4096) return CPATTN_ERR_SHAPE;
  if ((long long)B * S * H > 0x7fffffffLL - 4096) return CPATTN_ERR_SHAPE;  // 32-bit row index
  if (!o_a || !lse_a || !o_b || !lse_b || !o || !lse) return CPATTN_ERR_NULL;
  if (!aligned(o_a, 16) || !aligned(o_b, 16) || !aligned(o, 16) || !aligned(lse_a, 4) ||
      !aligned(lse_b, 4) || !aligned(lse, 4))
    return CPATTN_ERR_ALIGN;
  const size_t ob = size_t(B) * S * H * D * es, lb = size_t(B) * H * S * 4;
  // o may be o_a exactly (in-place accumulate); any other overlap would race
  if ((o != o_a && overlap(o, ob, o_a, ob)) || overlap(o, ob, o_b, ob) ||
      (lse != lse_a && overlap(lse, lb, lse_a, lb)) || overlap(lse, lb, lse_b, lb))
    return CPATTN_ERR_SHAPE;
  return cuda_status(cpattn::launch_merge(o_a, lse_a, o_b, lse_b, o, lse, B, H, S, D, es,
                                          reinterpret_cast<cudaStream_t>(stream)));
}

static int permute_args(const void* src, void* dst, int P, int S_local, int H, int D,
                        int elem_bytes, long long* run_vec) {
  if (P < 1 || S_local < 1 || H < 1 || D < 1) return CPATTN_ERR_SHAPE;
  if (elem_bytes != 2 && elem_bytes != 4) return CPATTN_ERR_SHAPE;
  if (H % P != 0) return CPATTN_ERR_SHAPE;
  const long long run_bytes = (long long)(H / P) * D * elem_bytes;
  if (run_bytes % 16 != 0) return CPATTN_ERR_SHAPE;
  // item indices are 32-bit: rows x 32-vector chunks must stay below 2^31
  if ((long long)P * P * S_local * ((run_bytes / 16 + 31) / 32) > 0x7fffffffLL)
    return CPATTN_ERR_SHAPE;
  if (src == nullptr || dst == nullptr) return CPATTN_ERR_NULL;
  if (!aligned(src, 16) || !aligned(dst, 16)) return CPATTN_ERR_ALIGN;
  const size_t bytes = size_t(P) * S_local * H * D * elem_bytes;
  if (overlap(src, bytes, dst, bytes)) return CPATTN_ERR_SHAPE;
  *run_vec = run_bytes / 16;
  return CPATTN_OK;
}

int cpattn_seq2head(const void* src, void* dst, int P, int S_local, int H, int D, int elem_bytes,
                    cpattn_stream_t stream) {
  long long run_vec = 0;
  const int st = permute_args(src, dst, P, S_local, H, D, elem_bytes, &run_vec);
  if (st != CPATTN_OK) return st;
  return cuda_status(cpattn::launch_seq2head(src, dst, P, S_local, run_vec,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

int cpattn_seq2head_qkv(const void* q, const void* k, const void* v, void* qh, void* kh, void* vh,
                        int P, int S_local, int H, int D, int elem_bytes, cpattn_stream_t stream) {
  const void* src[3] = {q, k, v};
  void* dst[3] = {qh, kh, vh};
  long long run_vec = 0;
  for (int t = 0; t < 3; ++t) {
    const int st = permute_args(src[t], dst[t], P, S_local, H, D, elem_bytes, &run_vec);
    if (st != CPATTN_OK) return st;
  }
  // no destination may overlap another tensor's source or destination
  const size_t bytes = size_t(P) * S_local * H * D * elem_bytes;
  for (int a = 0; a < 3; ++a)
    for (int c = 0; c < 3; ++c)
      if ((a != c && overlap(dst[a], bytes, dst[c], bytes)) || overlap(dst[a], bytes, src[c], bytes))
        return CPATTN_ERR_SHAPE;
  return cuda_status(cpattn::launch_seq2head_n(src, dst, 3, P, S_local, run_vec,
                                               reinterpret_cast<cudaStream_t>(stream)));
}

static bool norm_dim_ok(int D) { return D >= 8 && D <= 256 && (D & (D - 1)) == 0; }

static int norm_scalars_ok(float eps, float out_scale) {
  if (!(eps >= 0.0f) || !std::isfinite(eps) || !std::isfinite(out_scale)) return CPATTN_ERR_SHAPE;
  return CPATTN_OK;
}

int cpattn_rmsnorm(const void* x, void* y, const float* gamma, int rows, int D, float eps,
                   float out_scale, cpattn_stream_t stream) {
  if (rows < 0 || !norm_dim_ok(D)) return CPATTN_ERR_SHAPE;
  const int sc = norm_scalars_ok(eps, out_scale);
  if (sc != CPATTN_OK) return sc;
  if (rows == 0) return CPATTN_OK;  // nothing is read or written: pointers are not checked
  if ((long long)rows * (D / 8) > 0x7fffffffLL - 256) return CPATTN_ERR_SHAPE;  // 32-bit vectors
  if (x == nullptr || y == nullptr || gamma == nullptr) return CPATTN_ERR_NULL;
  if (!aligned(x, 16) || !aligned(y, 16) || !aligned(gamma, 16)) return CPATTN_ERR_ALIGN;
  const size_t bytes = size_t(rows) * D * 2;
  if (x != y && overlap(x, bytes, y, bytes)) return CPATTN_ERR_SHAPE;  // in place or disjoint
  if (overlap(gamma, size_t(D) * 4, y, bytes)) return CPATTN_ERR_SHAPE;
  return cuda_status(cpattn::launch_rmsnorm(x, y, gamma, rows, D, eps, out_scale,
                                            reinterpret_cast<cudaStream_t>(stream)));
}

int cpattn_seq2head_qkv_norm(const void* q, const void* k, const void* v, void* qh, void* kh,
                             void* vh, const float* gamma_q, const float* gamma_k, int P,
                             int S_local, int H, int D, float eps, float out_scale,
                             cpattn_stream_t stream) {
  if (!norm_dim_ok(D)) return CPATTN_ERR_SHAPE;
  const int sc = norm_scalars_ok(eps, out_scale);
  if (sc != CPATTN_OK) return sc;
  const void* src[3] = {q, k, v};
  void* dst[3] = {qh, kh, vh};
  long long run_vec = 0;
  for (int t = 0; t < 3; ++t) {
    const int st = permute_args(src[t], dst[t], P, S_local, H, D, 2, &run_vec);
    if (st != CPATTN_OK) return st;
  }
  if (gamma_q == nullptr || gamma_k == nullptr) return CPATTN_ERR_NULL;
  if (!aligned(gamma_q, 16) || !aligned(gamma_k, 16)) return CPATTN_ERR_ALIGN;
  const size_t bytes = size_t(P) * S_local * H * D * 2;
  for (int a = 0; a < 3; ++a) {
    for (int c = 0; c < 3; ++c)
      if ((a != c && overlap(dst[a], bytes, dst[c], bytes)) || overlap(dst[a], bytes, src[c], bytes))
        return CPATTN_ERR_SHAPE;
    if (overlap(dst[a], bytes, gamma_q, size_t(D) * 4) || overlap(dst[a], bytes, gamma_k, size_t(D) * 4))
      return CPATTN_ERR_SHAPE;
  }
  return cuda_status(cpattn::launch_seq2head_qkv_norm(src, dst, gamma_q, gamma_k, P, S_local, D,
                                                      run_vec, eps, out_scale,
                                                      reinterpret_cast<cudaStream_t>(stream)));
}

int cpattn_head2seq(const void* src, void* dst, int P, int S_local, int H, int D, int elem_bytes,
                    cpattn_stream_t stream) {
  long long run_vec = 0;
  const int st = permute_args(src, dst, P, S_local, H, D, elem_bytes, &run_vec);
  if (st != CPATTN_OK) return st;
  return cuda_status(cpattn::launch_head2seq(src, dst, P, S_local, run_vec,
                                             reinterpret_cast<cudaStream_t>(stream)));
}

int cpattn_device_error(void) {
  if (cudaDeviceSynchronize() != cudaSuccess) return CPATTN_ERR_CUDA;
  int* addr = device_error_word();
  if (addr == nullptr) return CPATTN_ERR_CUDA;
  int word = 0;
  if (cudaMemcpyFromSymbol(&word, g_cpattn_err, sizeof(int)) != cudaSuccess) return CPATTN_ERR_CUDA;
  const int zero = 0;
  if (cudaMemcpyToSymbol(g_cpattn_err, &zero, sizeof(int)) != cudaSuccess) return CPATTN_ERR_CUDA;
  return (word & cpattn::kDevErrTimeout) ? CPATTN_ERR_DEVICE_TIMEOUT : CPATTN_OK;
}

int cpattn_selftest_wait_timeout(long long limit_cycles, cpattn_stream_t stream) {
  if (limit_cycles < 1 || limit_cycles > (1LL << 31)) return CPATTN_ERR_SHAPE;
  int* err = device_error_word();
  if (err == nullptr) return CPATTN_ERR_CUDA;
  return cuda_status(cpattn::launch_wait_timeout_selftest(err, limit_cycles,
                                                          reinterpret_cast<cudaStream_t>(stream)));
}

int cpattn_selftest_exp2(const float* t, float* out, int n, cpattn_stream_t stream) {
  if (n < 1) return CPATTN_ERR_SHAPE;
  if (t == nullptr || out == nullptr) return CPATTN_ERR_NULL;
  if (!aligned(t, 4) || !aligned(out, 4)) return CPATTN_ERR_ALIGN;
  return cuda_status(
      cpattn::launch_exp2_poly_selftest(t, out, n, reinterpret_cast<cudaStream_t>(stream)));
}

}  // extern "C"
