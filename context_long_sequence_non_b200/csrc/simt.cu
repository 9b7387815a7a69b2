// simt.cu -- the CUDA-core kernels of the path: fp32 attention, the (O, LSE) merge of the
// Ring Attention step, the two Ulysses permutes, the empty-key fill and the bounded-wait
// self-test.  Merge and permutes are HBM-bound streaming kernels: 16-byte vectors, each
// warp moving contiguous runs, several independent loads in flight per thread, grids
// sized in multiples of the SM count.
#include <cuda_runtime.h>

#include <cstdint>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace cpattn {
namespace {

// ------------------------------------------------------------------ dependent launches
// The bandwidth-bound kernels below are launched with programmatic stream serialization: a
// launch may be scheduled while the previous kernel on the stream is still finishing, and
// each CTA first waits (griddepcontrol.wait, a hardware dependency) until that kernel has
// completed and its writes are visible, then lets the next launch be scheduled.  A
// back-to-back burst (three seq2heads, a ring step's merges) then overlaps each launch's
// start-up with its predecessor's tail instead of paying it in full.  After a kernel that
// was not launched this way the wait returns at once and ordering is the stream's.
__device__ __forceinline__ void dependent_launch_gate() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, cudaStream_t stream,
                             Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// ------------------------------------------------------------------ fp32 attention
// One warp per query row (b, h, i); lane l holds q[d] for d = l, l + 32, ...  Keys are
// visited in order with an online softmax in fp32 (natural base, expf/logf).
template <int T>
__global__ void __launch_bounds__(256) attn_f32_kernel(const float* __restrict__ q,
                                                       const float* __restrict__ k,
                                                       const float* __restrict__ v, void* out,
                                                       float* lse, int B, int H, int Sq, int Skv,
                                                       int D, float scale, bool out_bf16) {
  const int lane = threadIdx.x & 31;
  const long long row = (long long)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const long long n_rows = (long long)B * H * Sq;
  if (row >= n_rows) return;
  const int i = int(row % Sq);
  const int h = int((row / Sq) % H);
  const int b = int(row / ((long long)Sq * H));
  float qv[T], acc[T];
  const float* qp = q + (((long long)b * Sq + i) * H + h) * D;
#pragma unroll
  for (int t = 0; t < T; ++t) {
    const int d = lane + 32 * t;
    qv[t] = d < D ? qp[d] : 0.f;
    acc[t] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  for (int j = 0; j < Skv; ++j) {
    const long long kv_off = (((long long)b * Skv + j) * H + h) * D;
    float part = 0.f;
#pragma unroll
    for (int t = 0; t < T; ++t) {
      const int d = lane + 32 * t;
      if (d < D) part = fmaf(qv[t], k[kv_off + d], part);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_down_sync(0xffffffffu, part, off);
    const float s = __shfl_sync(0xffffffffu, part, 0) * scale;
    if (s > m) {
      const float corr = expf(m - s);
      l *= corr;
#pragma unroll
      for (int t = 0; t < T; ++t) acc[t] *= corr;
      m = s;
    }
    const float p = expf(s - m);
    l += p;
#pragma unroll
    for (int t = 0; t < T; ++t) {
      const int d = lane + 32 * t;
      if (d < D) acc[t] = fmaf(p, v[kv_off + d], acc[t]);
    }
  }
  const float inv_l = 1.0f / l;
  const long long o_off = (((long long)b * Sq + i) * H + h) * D;
#pragma unroll
  for (int t = 0; t < T; ++t) {
    const int d = lane + 32 * t;
    if (d < D) {
      const float o = acc[t] * inv_l;
      if (out_bf16) {
        static_cast<uint16_t*>(out)[o_off + d] = uint16_t(pack_bf16x2(o, 0.f) & 0xFFFFu);
      } else {
        static_cast<float*>(out)[o_off + d] = o;
      }
    }
  }
  if (lane == 0 && lse != nullptr) lse[((long long)b * H + h) * Sq + i] = m + logf(l);
}

// ------------------------------------------------------------------ empty key set
__global__ void fill_empty_kernel(uint4* out, size_t n_vec, float* lse, size_t n_lse) {
  dependent_launch_gate();
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_vec; i += stride)
    out[i] = make_uint4(0u, 0u, 0u, 0u);
  if (lse != nullptr)
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n_lse; i += stride)
      lse[i] = -INFINITY;
}

// ------------------------------------------------------------------ (O, LSE) merge
// 16-byte vectors of O; a block covers whole (b, s, h) rows (blockDim = rows x
// vectors_per_row) and every thread handles kMergeRowsPerThread rows.  Every thread derives
// its rows' weights from the two LSEs itself (no shared-memory phase), so the loads of O and
// LSE for all its rows are in flight at once.
// The merged LSE is written after a block barrier by the row's first thread: every read of
// this block's LSE entries precedes every write, and each O vector is read and written by
// the same thread, so the result may overwrite partial a in place.
constexpr int kMergeThreads = 256;

__device__ __forceinline__ void merge_vec_bf16(const uint4& a, const uint4& b, float wa, float wb,
                                               uint4& o) {
  const uint32_t* pa = &a.x;
  const uint32_t* pb = &b.x;
  uint32_t* po = &o.x;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float a0 = __uint_as_float(pa[e] << 16), a1 = __uint_as_float(pa[e] & 0xFFFF0000u);
    const float b0 = __uint_as_float(pb[e] << 16), b1 = __uint_as_float(pb[e] & 0xFFFF0000u);
    po[e] = pack_bf16x2(fmaf(wa, a0, wb * b0), fmaf(wa, a1, wb * b1));
  }
}

__device__ __forceinline__ void merge_vec_f32(const uint4& a, const uint4& b, float wa, float wb,
                                              uint4& o) {
  o.x = __float_as_uint(fmaf(wa, __uint_as_float(a.x), wb * __uint_as_float(b.x)));
  o.y = __float_as_uint(fmaf(wa, __uint_as_float(a.y), wb * __uint_as_float(b.y)));
  o.z = __float_as_uint(fmaf(wa, __uint_as_float(a.z), wb * __uint_as_float(b.z)));
  o.w = __float_as_uint(fmaf(wa, __uint_as_float(a.w), wb * __uint_as_float(b.w)));
}

constexpr int kMergeRowsPerThread = 4;  // independent row vectors in flight per thread

template <bool kBf16>
__global__ void __launch_bounds__(kMergeThreads) merge_kernel(
    const uint4* o_a, const float* lse_a, const uint4* o_b, const float* lse_b, uint4* o,
    float* lse, int H, int S, long long n_rows, int vpr) {
  dependent_launch_gate();
  // a block covers kMergeRowsPerThread groups of (blockDim.x / vpr) consecutive rows; thread
  // (rl, v) takes vector v of row rl of every group, issuing all loads before any math
  const int rows_per_group = blockDim.x / vpr;
  const int rl = threadIdx.x / vpr;
  const int v = threadIdx.x - rl * vpr;
  const int row0 = int(blockIdx.x) * rows_per_group * kMergeRowsPerThread + rl;
  uint4 a[kMergeRowsPerThread], bb[kMergeRowsPerThread];
  float la[kMergeRowsPerThread], lb[kMergeRowsPerThread];
  int li[kMergeRowsPerThread];
  bool live[kMergeRowsPerThread];
#pragma unroll
  for (int u = 0; u < kMergeRowsPerThread; ++u) {
    const int row = row0 + u * rows_per_group;  // (b, s, h), h fastest; < 2^31
    live[u] = row < n_rows;
    const int bs = row / H;
    const int h = row - bs * H;
    const int b = bs / S;
    const int s = bs - b * S;
    li[u] = (b * H + h) * S + s;
    if (live[u]) {
      const long long idx = (long long)row * vpr + v;
      a[u] = o_a[idx];
      bb[u] = o_b[idx];
      la[u] = lse_a[li[u]];
      lb[u] = lse_b[li[u]];
    }
  }
  float L[kMergeRowsPerThread];
#pragma unroll
  for (int u = 0; u < kMergeRowsPerThread; ++u) {
    L[u] = -INFINITY;
    if (!live[u]) continue;
    const float mx = fmaxf(la[u], lb[u]);
    float wa = 0.f, wb = 0.f;
    if (mx != -INFINITY) {
      const float ea = expf(la[u] - mx), eb = expf(lb[u] - mx);
      const float tot = ea + eb;
      L[u] = mx + logf(tot);
      wa = ea / tot;
      wb = eb / tot;
    }
    uint4 r;
    if (kBf16) merge_vec_bf16(a[u], bb[u], wa, wb, r);
    else merge_vec_f32(a[u], bb[u], wa, wb, r);
    o[(long long)(row0 + u * rows_per_group) * vpr + v] = r;
  }
  // every read of this block's LSE entries precedes every write (in-place merge allowed)
  __syncthreads();
  if (v == 0) {
#pragma unroll
    for (int u = 0; u < kMergeRowsPerThread; ++u)
      if (live[u]) lse[li[u]] = L[u];
  }
}

// Rows of at most 32 vectors (bf16 D <= 256, fp32 D <= 128; vpr a power of two): warps
// stride over items of 32 consecutive vectors = 32/vpr whole rows, kMergeRowsPerThread items
// in flight, the grid a fixed multiple of the SM count (no tail wave).  A row's lanes all
// sit in one warp, so an in-place LSE update needs no block barrier, only a warp one: the
// __syncwarp() between the load loop and the store loop orders every lane's read of
// lse_a before the row leader's write of lse (which may be the same array).
template <bool kBf16>
__global__ void __launch_bounds__(kMergeThreads, 4) merge_rows_kernel(
    const uint4* o_a, const float* lse_a, const uint4* o_b, const float* lse_b, uint4* o,
    float* lse, int H, int S, int n_vec, int vpr_log2) {
  dependent_launch_gate();
  const int lane = threadIdx.x & 31;
  const int warp = int((blockIdx.x * kMergeThreads + threadIdx.x) >> 5);
  const int n_warps = int((gridDim.x * kMergeThreads) >> 5);
  const int n_items = (n_vec + 31) >> 5;
  const bool leader = (lane & ((1 << vpr_log2) - 1)) == 0;
  for (int it0 = warp * kMergeRowsPerThread; it0 < n_items; it0 += n_warps * kMergeRowsPerThread) {
    uint4 a[kMergeRowsPerThread], bb[kMergeRowsPerThread];
    float la[kMergeRowsPerThread], lb[kMergeRowsPerThread];
    int li[kMergeRowsPerThread];
    bool live[kMergeRowsPerThread];
#pragma unroll
    for (int u = 0; u < kMergeRowsPerThread; ++u) {
      const int idx = ((it0 + u) << 5) + lane;  // < 2^31 (checked by the launcher)
      live[u] = it0 + u < n_items && idx < n_vec;
      const int row = idx >> vpr_log2;  // (b, s, h), h fastest
      const int bs = row / H;
      const int h = row - bs * H;
      const int b = bs / S;
      li[u] = (b * H + h) * S + (bs - b * S);
      if (live[u]) {
        a[u] = o_a[idx];
        bb[u] = o_b[idx];
        la[u] = lse_a[li[u]];
        lb[u] = lse_b[li[u]];
      }
    }
    __syncwarp();  // every lane's LSE reads above precede the leaders' LSE writes below
#pragma unroll
    for (int u = 0; u < kMergeRowsPerThread; ++u) {
      if (!live[u]) continue;
      const float mx = fmaxf(la[u], lb[u]);
      float wa = 0.f, wb = 0.f, L = -INFINITY;
      if (mx != -INFINITY) {
        // CUDA's fast intrinsics: the arguments are <= 0 and tot is in [1, 2], where their
        // errors (a few float ulps) stay far below the merge's fp32 / LSE tolerances; every
        // lane of a row computes the same weights
        const float ea = __expf(la[u] - mx), eb = __expf(lb[u] - mx);
        const float tot = ea + eb;
        const float inv = __fdividef(1.0f, tot);
        L = mx + __logf(tot);
        wa = ea * inv;
        wb = eb * inv;
      }
      uint4 r;
      if (kBf16) merge_vec_bf16(a[u], bb[u], wa, wb, r);
      else merge_vec_f32(a[u], bb[u], wa, wb, r);
      o[((it0 + u) << 5) + lane] = r;
      if (leader) lse[li[u]] = L;
    }
  }
}

// ------------------------------------------------------------------ split-KV combine
// n partial results of the same queries over disjoint key ranges (split-KV), each a
// normalised O (dtype of out) with its LSE, are folded exactly -- optionally together with
// the running accumulator already in (out, lse) -- by the same merge formula generalised to
// n terms: L = max_s L_s + ln sum_s exp(L_s - max), O = sum_s exp(L_s - L) O_s.  Thread
// layout as the merge kernel: one 16-byte vector of the row per thread, whole rows per block,
// the output LSE written after a block barrier.
constexpr int kMaxSplit = 8;

template <bool kBf16, bool kAcc>
__global__ void __launch_bounds__(kMergeThreads) combine_kernel(
    const uint4* __restrict__ part_o, const float* __restrict__ part_lse, int n,
    long long o_stride, long long lse_stride, uint4* out, float* lse, int H, int S,
    long long n_rows, int vpr) {
  dependent_launch_gate();
  const int rows_per_block = blockDim.x / vpr;
  const int rl = threadIdx.x / vpr;
  const int v = threadIdx.x - rl * vpr;
  const int row = int(blockIdx.x) * rows_per_block + rl;  // (b, s, h), h fastest; < 2^31
  const bool live = row < n_rows;
  int li = 0;
  float L = -INFINITY;
  if (live) {
    const int bs = row / H;
    const int h = row - bs * H;
    const int b = bs / S;
    const int si = bs - b * S;
    li = (b * H + h) * S + si;
    const long long idx = (long long)row * vpr + v;
    float ls[kMaxSplit + 1];
    float mx = -INFINITY;
    for (int t = 0; t < n; ++t) {
      ls[t] = part_lse[t * lse_stride + li];
      mx = fmaxf(mx, ls[t]);
    }
    const float la = kAcc ? lse[li] : -INFINITY;
    mx = fmaxf(mx, la);
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    float tot = 0.f;
    if (mx != -INFINITY) {
      for (int t = 0; t <= n; ++t) {
        const float lt = t < n ? ls[t] : la;
        if (lt == -INFINITY) continue;  // an empty term contributes nothing (and is not read)
        const float wgt = expf(lt - mx);
        tot += wgt;
        const uint4 p = t < n ? part_o[t * o_stride + idx] : out[idx];
        if (kBf16) {
          const uint32_t pw[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            acc[2 * e] = fmaf(wgt, __uint_as_float(pw[e] << 16), acc[2 * e]);
            acc[2 * e + 1] = fmaf(wgt, __uint_as_float(pw[e] & 0xFFFF0000u), acc[2 * e + 1]);
          }
        } else {
          acc[0] = fmaf(wgt, __uint_as_float(p.x), acc[0]);
          acc[1] = fmaf(wgt, __uint_as_float(p.y), acc[1]);
          acc[2] = fmaf(wgt, __uint_as_float(p.z), acc[2]);
          acc[3] = fmaf(wgt, __uint_as_float(p.w), acc[3]);
        }
      }
      L = mx + logf(tot);
    }
    const float inv = tot > 0.f ? 1.0f / tot : 0.f;
    uint4 r;
    if (kBf16) {
      r.x = pack_bf16x2(acc[0] * inv, acc[1] * inv);
      r.y = pack_bf16x2(acc[2] * inv, acc[3] * inv);
      r.z = pack_bf16x2(acc[4] * inv, acc[5] * inv);
      r.w = pack_bf16x2(acc[6] * inv, acc[7] * inv);
    } else {
      r = make_uint4(__float_as_uint(acc[0] * inv), __float_as_uint(acc[1] * inv),
                     __float_as_uint(acc[2] * inv), __float_as_uint(acc[3] * inv));
    }
    out[idx] = r;
  }
  __syncthreads();
  if (live && v == 0 && lse != nullptr) lse[li] = L;
}

// ------------------------------------------------------------------ tail-split combine
// The items of the attention launch's last wave were split into `parts` key ranges; range p
// of tail item t left its normalised fp32 partial (O row, LSE) at workspace row
// (p * n_tail + t) * 256 + r.  One warp per query row folds them with the n-term merge
// L = max + ln sum_p exp(L_p - max), O = sum_p exp(L_p - L) O_p -- together with the running
// (out, lse) row when accumulating (a running LSE of -inf means an empty accumulator whose
// row is not read) -- and writes the row of out / lse.  Lane l holds D/32 consecutive
// elements of the row.
template <int VPL, bool kOutBf16, bool kAcc>
__global__ void __launch_bounds__(256) combine_tail_kernel(
    const float* __restrict__ ws_o, const float* __restrict__ ws_lse, int n_full, int n_tail,
    int parts, void* out, float* lse, int H, int Sq, long long batch_stride, int token_stride) {
  dependent_launch_gate();
  constexpr int D = 32 * VPL;
  const int lane = threadIdx.x & 31;
  const int wrow = int(blockIdx.x) * 8 + int(threadIdx.x >> 5);  // tail row (t, r)
  if (wrow >= n_tail * 256) return;
  const int t = wrow >> 8, r = wrow & 255;
  const int n_pairs = (Sq + 255) / 256;
  const int item = n_full + t;
  const int pair = item % n_pairs, h = (item / n_pairs) % H, b = item / n_pairs / H;
  const int q = pair * 256 + r;
  if (q >= Sq) return;  // rows past the end of the sequence were never written
  const size_t li = (size_t(b) * H + h) * Sq + q;
  const size_t orow =
      (size_t(b) * batch_stride + size_t(q) * token_stride + h) * D + lane * VPL;
  float lp[8];
  float mx = -INFINITY;
  for (int p = 0; p < parts; ++p) {
    lp[p] = ws_lse[size_t(p * n_tail + t) * 256 + r];
    mx = fmaxf(mx, lp[p]);
  }
  const float la = kAcc ? lse[li] : -INFINITY;
  mx = fmaxf(mx, la);
  float acc[VPL];
#pragma unroll
  for (int e = 0; e < VPL; ++e) acc[e] = 0.f;
  float tot = 0.f;
  for (int p = 0; p < parts; ++p) {
    const float w = expf(lp[p] - mx);
    tot += w;
    const float* src = ws_o + (size_t(p * n_tail + t) * 256 + r) * D + lane * VPL;
#pragma unroll
    for (int e = 0; e < VPL; ++e) acc[e] = fmaf(w, src[e], acc[e]);
  }
  if (kAcc && la != -INFINITY) {
    const float w = expf(la - mx);
    tot += w;
    if constexpr (kOutBf16) {
      const uint16_t* a = static_cast<const uint16_t*>(out) + orow;
#pragma unroll
      for (int e = 0; e < VPL; ++e) acc[e] = fmaf(w, __uint_as_float(uint32_t(a[e]) << 16), acc[e]);
    } else {
      const float* a = static_cast<const float*>(out) + orow;
#pragma unroll
      for (int e = 0; e < VPL; ++e) acc[e] = fmaf(w, a[e], acc[e]);
    }
  }
  const float inv = 1.0f / tot;
  if constexpr (kOutBf16) {
    uint32_t w2[VPL / 2];
#pragma unroll
    for (int e = 0; e < VPL / 2; ++e) w2[e] = pack_bf16x2(acc[2 * e] * inv, acc[2 * e + 1] * inv);
    uint32_t* dst = reinterpret_cast<uint32_t*>(static_cast<uint16_t*>(out) + orow);
#pragma unroll
    for (int e = 0; e < VPL / 2; ++e) dst[e] = w2[e];
  } else {
    float* dst = static_cast<float*>(out) + orow;
#pragma unroll
    for (int e = 0; e < VPL; ++e) dst[e] = acc[e] * inv;
  }
  __syncwarp();  // every lane's read of lse[li] precedes lane 0's write
  if (lane == 0 && lse != nullptr) lse[li] = mx + logf(tot);
}

// ------------------------------------------------------------------ Ulysses permutes
// Rows of Hp*D elements move as whole 16-byte-vector runs.  Head-grouped row index
// A(g, r, s) = (g*P + r)*S_l + s; sequence-sharded row index Bq(g, r, s) = (r*S_l + s)*P + g.
// seq2head: dst[A] = src[Bq]; head2seq: dst[Bq] = src[A].  Threads walk dst rows in order
// (coalesced stores); each warp moves kPermUnroll (row, 32-vector chunk) items at a time.
constexpr int kPermThreads = 256;
constexpr int kPermUnroll = 4;

// Up to three tensors share one launch (Q, K and V go through the same re-partition).
struct PermuteSet {
  const uint4* src[3];
  uint4* dst[3];
  // blocks [block_begin[t], block_begin[t + 1]) of the 1-D grid serve tensor t; the split
  // follows each tensor's work (a normalised tensor costs about twice a plain copy), so
  // all tensors finish together
  int block_begin[4];
};

// Optional RMSNorm of every head row on the way through (the Q/K norm of the
// attention_mdtrt sample, section 模型的核心结构): y = bf16(((x * r) * gamma[d]) * out_scale)
// with r = 1 / sqrt(mean(x^2) + eps), all in fp32.  A head row of D bf16 is row_vec = D/8
// vectors held by row_vec consecutive lanes (32 % row_vec == 0, and runs and 32-vector
// chunks start on head-row boundaries), so its sum of squares is a shuffle reduction and
// the head-dim slice a lane sees, (lane % row_vec) * 8 .. + 7, is the same for every item:
// its 8 weights are loaded once.
struct RowNorm {
  const float* gamma[3];  // per tensor of the set; nullptr = copied unchanged
  int row_vec;
  float inv_d, eps, out_scale;
};

// 1/sqrt(a) for a > 0: the special-function unit's estimate refined by one Newton step on
// f(y) = 1/y^2 - a (y' = y * (3 - a y^2) / 2), which brings it to about an ulp of the
// float32 1/sqrt(a) for every positive finite a (subnormal a included).
__device__ __forceinline__ float rsqrt_refined(float a) {
  float y;
  asm("rsqrt.approx.f32 %0, %1;" : "=f"(y) : "f"(a));
  const float hy = 0.5f * y;
  return fmaf(hy, fmaf(-a * y, y, 1.0f), y);  // y + (y/2)(1 - a y^2)
}

__device__ __forceinline__ void load_gamma8(const float* __restrict__ gamma, int d0, float (&g)[8]) {
  const float4 g0 = __ldg(reinterpret_cast<const float4*>(gamma + d0));
  const float4 g1 = __ldg(reinterpret_cast<const float4*>(gamma + d0 + 4));
  g[0] = g0.x; g[1] = g0.y; g[2] = g0.z; g[3] = g0.w;
  g[4] = g1.x; g[5] = g1.y; g[6] = g1.z; g[7] = g1.w;
}

// Normalise the 8 elements of one 16-byte vector; every lane of the warp must call it.  A
// head row (kRowVec lanes) is always either wholly live or wholly dead -- items are
// warp-uniform and runs are whole head rows -- so a dead lane (whose input is zero, never
// stored) never mixes into a live row's sum.
template <int kRowVec>
__device__ __forceinline__ uint4 rms_normalise(uint4 in, float inv_d, float eps,
                                               float out_scale, const float (&g)[8]) {
  const uint32_t w[4] = {in.x, in.y, in.z, in.w};
  float f[8];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    f[2 * t] = __uint_as_float(w[t] << 16);  // bf16 -> fp32 is exact
    f[2 * t + 1] = __uint_as_float(w[t] & 0xFFFF0000u);
  }
  // packed fp32x2 arithmetic: per lane the same IEEE operations as the scalar forms, in
  // half the issue slots (the fused permute is issue-bound)
  float2 ss2 = make_float2(0.f, 0.f);
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    const float2 fe = make_float2(f[e], f[e + 1]);
    ss2 = ffma2(fe, fe, ss2);
  }
  float ss = ss2.x + ss2.y;
#pragma unroll
  for (int o = 1; o < kRowVec; o <<= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float a = ss * inv_d + eps;
  const float r = a > 0.f ? rsqrt_refined(a) : 0.f;  // an all-zero row with eps = 0 stays 0
  const float2 r2 = make_float2(r, r), s2 = make_float2(out_scale, out_scale);
  uint32_t w_out[4];
#pragma unroll
  for (int t = 0; t < 4; ++t) {
    float2 y = fmul2(fmul2(make_float2(f[2 * t], f[2 * t + 1]), r2),
                     make_float2(g[2 * t], g[2 * t + 1]));
    if (out_scale != 1.0f) y = fmul2(y, s2);
    w_out[t] = pack_bf16x2(y.x, y.y);
  }
  return make_uint4(w_out[0], w_out[1], w_out[2], w_out[3]);
}

// kRowVec: 16-byte vectors per head row for the normalising form (D / 8), 0 for a copy.
// The normalising form takes 4 blocks per SM (its registers without spilling), the copy 5.
template <bool kToHead, bool kNorm, int kRowVec>
__global__ void __launch_bounds__(kPermThreads, kNorm ? 4 : 5) permute_kernel(const __grid_constant__ PermuteSet set,
                                                                const __grid_constant__ RowNorm nrm,
                                                                int P, int S_l, int run_vec,
                                                                int chunks, int n_items) {
  dependent_launch_gate();
  // blockIdx.y picks the tensor (uniform per block); item = (dst row, 32-vector chunk)
  const int bx = int(blockIdx.x);
  const int tsr = int(bx >= set.block_begin[1]) + int(bx >= set.block_begin[2]);  // tensor
  const int local_block = bx - set.block_begin[tsr];
  const int n_blocks = set.block_begin[tsr + 1] - set.block_begin[tsr];
  const uint4* __restrict__ src = set.src[tsr];
  uint4* __restrict__ dst = set.dst[tsr];
  const int lane = threadIdx.x & 31;
  const int warp = (local_block * kPermThreads + int(threadIdx.x)) >> 5;
  const int n_warps = (n_blocks * kPermThreads) >> 5;
  const float* __restrict__ gamma = kNorm ? nrm.gamma[tsr] : nullptr;  // per block
  float g[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (kNorm && gamma != nullptr) load_gamma8(gamma, (lane % nrm.row_vec) * 8, g);
  for (int it0 = warp * kPermUnroll; it0 < n_items; it0 += n_warps * kPermUnroll) {
    uint4 buf[kPermUnroll];
    long long dst_off[kPermUnroll];
    bool live[kPermUnroll];
    // The warp's items it0 .. it0+kPermUnroll-1 are consecutive: divide once for the
    // first, then step the mixed-radix digits of the dst row.  seq2head: n = A(g, r, s),
    // digits (d0, d1, d2) = (s, r, g); head2seq: n = Bq(g, r, s), digits (g, s, r).
    int n = it0 / chunks;  // dst row
    int c = it0 - n * chunks;
    int d0, d1, d2;
    if (kToHead) {
      const int q = n / S_l;
      d0 = n - q * S_l;
      d2 = q / P;
      d1 = q - d2 * P;
    } else {
      const int q = n / P;
      d0 = n - q * P;
      d2 = q / S_l;
      d1 = q - d2 * S_l;
    }
    const int R0 = kToHead ? S_l : P, R1 = kToHead ? P : S_l;
#pragma unroll
    for (int u = 0; u < kPermUnroll; ++u) {
      const int v = c * 32 + lane;
      live[u] = it0 + u < n_items && v < run_vec;
      const int src_row = kToHead ? (d1 * S_l + d0) * P + d2   // Bq(g, r, s)
                                  : (d0 * P + d2) * S_l + d1;  // A(g, r, s)
      dst_off[u] = (long long)n * run_vec + v;
      if constexpr (kNorm) buf[u] = make_uint4(0u, 0u, 0u, 0u);
      if (live[u]) buf[u] = src[(long long)src_row * run_vec + v];
      if (++c == chunks) {  // next item: next chunk, else the next dst row
        c = 0;
        ++n;
        if (++d0 == R0) {
          d0 = 0;
          if (++d1 == R1) {
            d1 = 0;
            ++d2;
          }
        }
      }
    }
    if constexpr (kNorm) {
      if (gamma != nullptr) {
#pragma unroll
        for (int u = 0; u < kPermUnroll; ++u)
          buf[u] = rms_normalise<kRowVec>(buf[u], nrm.inv_d, nrm.eps, nrm.out_scale, g);
      }
    }
#pragma unroll
    for (int u = 0; u < kPermUnroll; ++u)
      if (live[u]) dst[dst_off[u]] = buf[u];
  }
}

// ------------------------------------------------------------------ exp2 polynomial self-test
__global__ void exp2_poly_selftest_kernel(const float* __restrict__ t, float* __restrict__ out,
                                          int n) {
  const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float2 in = make_float2(t[i], i + 1 < n ? t[i + 1] : 0.f);
  const float2 r = exp2_poly2(in);
  out[i] = r.x;
  if (i + 1 < n) out[i + 1] = r.y;
}

// ------------------------------------------------------------------ bounded-wait self-test
__global__ void wait_timeout_selftest_kernel(int* err, long long limit) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_sh;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_sh = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // nothing ever arrives on `bar`: the wait must run out and record the timeout
  mbar_wait(smem_u32(&bar), 0, &abort_sh, err, limit);
  __syncthreads();
}

long long grid_for(long long work_items, int threads, int waves_per_sm) {
  const long long per_block = threads;
  long long blocks = (work_items + per_block - 1) / per_block;
  const long long cap = (long long)sm_count() * waves_per_sm;
  if (blocks > cap) blocks = cap;
  return blocks < 1 ? 1 : blocks;
}

}  // namespace

int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (cached[dev] == 0) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
      n = 148;
    cached[dev] = n;
  }
  return cached[dev];
}

cudaError_t launch_attn_fwd_f32(const float* q, const float* k, const float* v, void* out,
                                float* lse, int B, int H, int Sq, int Skv, int D, float scale,
                                bool out_bf16, cudaStream_t stream) {
  const long long rows = (long long)B * H * Sq;
  const int warps = 8;
  const long long blocks = (rows + warps - 1) / warps;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const int T = (D + 31) / 32;
#define CPATTN_F32_CASE(TT)                                                                   \
  case TT:                                                                                    \
    attn_f32_kernel<TT><<<unsigned(blocks), warps * 32, 0, stream>>>(q, k, v, out, lse, B, H, \
                                                                     Sq, Skv, D, scale,       \
                                                                     out_bf16);               \
    break;
  switch (T) {
    CPATTN_F32_CASE(1)
    CPATTN_F32_CASE(2)
    CPATTN_F32_CASE(3)
    CPATTN_F32_CASE(4)
    CPATTN_F32_CASE(5)
    CPATTN_F32_CASE(6)
    CPATTN_F32_CASE(7)
    CPATTN_F32_CASE(8)
    default:
      return cudaErrorInvalidValue;
  }
#undef CPATTN_F32_CASE
  return cudaGetLastError();
}

cudaError_t launch_fill_empty(void* out, size_t out_bytes, float* lse, size_t n_lse,
                              cudaStream_t stream) {
  const size_t n_vec = out_bytes / 16;
  const long long work = (long long)(n_vec > n_lse ? n_vec : n_lse);
  return launch_dependent(fill_empty_kernel, dim3(unsigned(grid_for(work, 256, 8))), dim3(256),
                          stream, static_cast<uint4*>(out), n_vec, lse, n_lse);
}

cudaError_t launch_merge(const void* o_a, const float* lse_a, const void* o_b, const float* lse_b,
                         void* o, float* lse, int B, int H, int S, int D, int elem_bytes,
                         cudaStream_t stream) {
  const long long n_rows = (long long)B * S * H;
  const int vpr = D * elem_bytes / 16;  // 16-byte vectors per row (validated: 1..256)
  const long long n_vec = n_rows * vpr;
  if (vpr <= 32 && (vpr & (vpr - 1)) == 0 && n_vec <= 0x7fffffffLL - 32 * (kMergeRowsPerThread + 1)) {
    int vpr_log2 = 0;
    while ((1 << vpr_log2) < vpr) ++vpr_log2;
    const long long items = (n_vec + 31) / 32;
    const long long warps_needed = (items + kMergeRowsPerThread - 1) / kMergeRowsPerThread;
    const long long blocks_needed = (warps_needed * 32 + kMergeThreads - 1) / kMergeThreads;
    const long long cap = (long long)sm_count() * 4;  // all resident (64 registers a thread)
    const unsigned blocks = unsigned(blocks_needed < cap ? blocks_needed : cap);
    return launch_dependent(elem_bytes == 2 ? merge_rows_kernel<true> : merge_rows_kernel<false>,
                            dim3(blocks), dim3(kMergeThreads), stream,
                            static_cast<const uint4*>(o_a), lse_a, static_cast<const uint4*>(o_b),
                            lse_b, static_cast<uint4*>(o), lse, H, S, int(n_vec), vpr_log2);
  }
  const int rows_per_group = vpr >= kMergeThreads ? 1 : kMergeThreads / vpr;
  const long long rows_per_block = (long long)rows_per_group * kMergeRowsPerThread;
  const long long blocks = (n_rows + rows_per_block - 1) / rows_per_block;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const int threads = rows_per_group * vpr;
  return launch_dependent(elem_bytes == 2 ? merge_kernel<true> : merge_kernel<false>,
                          dim3(unsigned(blocks)), dim3(threads), stream,
                          static_cast<const uint4*>(o_a), lse_a, static_cast<const uint4*>(o_b),
                          lse_b, static_cast<uint4*>(o), lse, H, S, n_rows, vpr);
}

cudaError_t launch_combine(const void* part_o, const float* part_lse, int n, void* out, float* lse,
                           int B, int H, int S, int D, int elem_bytes, bool accumulate,
                           cudaStream_t stream) {
  if (n < 1 || n > kMaxSplit) return cudaErrorInvalidValue;
  const long long n_rows = (long long)B * S * H;
  const int vpr = D * elem_bytes / 16;
  const int rows_per_block = vpr >= kMergeThreads ? 1 : kMergeThreads / vpr;
  const long long blocks = (n_rows + rows_per_block - 1) / rows_per_block;
  if (blocks > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const int threads = rows_per_block * vpr;
  const long long o_stride = n_rows * vpr;  // 16-byte vectors per partial
  const long long lse_stride = (long long)B * H * S;
  const uint4* po = static_cast<const uint4*>(part_o);
  uint4* o = static_cast<uint4*>(out);
  auto kernel = elem_bytes == 2 ? (accumulate ? combine_kernel<true, true> : combine_kernel<true, false>)
                                : (accumulate ? combine_kernel<false, true> : combine_kernel<false, false>);
  return launch_dependent(kernel, dim3(unsigned(blocks)), dim3(threads), stream, po, part_lse, n,
                          o_stride, lse_stride, o, lse, H, S, n_rows, vpr);
}

cudaError_t launch_combine_tail(const float* ws_o, const float* ws_lse, int n_full, int n_tail,
                                int parts, void* out, float* lse, int B, int H, int Sq, int D,
                                int out_bytes, bool accumulate, long long batch_stride,
                                int token_stride, cudaStream_t stream) {
  (void)B;
  if (parts < 1 || parts > 8 || n_tail < 1 || (D != 64 && D != 128)) return cudaErrorInvalidValue;
  const unsigned blocks = unsigned((n_tail * 256 + 7) / 8);
  const bool bf = out_bytes == 2;
  auto kernel = D == 128
      ? (bf ? (accumulate ? combine_tail_kernel<4, true, true> : combine_tail_kernel<4, true, false>)
            : (accumulate ? combine_tail_kernel<4, false, true> : combine_tail_kernel<4, false, false>))
      : (bf ? (accumulate ? combine_tail_kernel<2, true, true> : combine_tail_kernel<2, true, false>)
            : (accumulate ? combine_tail_kernel<2, false, true> : combine_tail_kernel<2, false, false>));
  return launch_dependent(kernel, dim3(blocks), dim3(256), stream, ws_o, ws_lse, n_full, n_tail,
                          parts, out, lse, H, Sq, batch_stride, token_stride);
}

static cudaError_t launch_permute(bool to_head, const void* const* src, void* const* dst,
                                  int n_tensors, int P, int S_local, long long run_vec,
                                  cudaStream_t stream, const RowNorm* nrm = nullptr) {
  PermuteSet set{};
  for (int t = 0; t < 3; ++t) {
    const int u = t < n_tensors ? t : 0;
    set.src[t] = static_cast<const uint4*>(src[u]);
    set.dst[t] = static_cast<uint4*>(dst[u]);
  }
  const long long n_rows = (long long)P * P * S_local;
  const int chunks = int((run_vec + 31) / 32);
  const long long n_items = n_rows * chunks;
  if (n_items > 0x7fffffffLL) return cudaErrorInvalidValue;  // 32-bit item index
  const long long warps_needed = (n_items + kPermUnroll - 1) / kPermUnroll;
  const long long blocks_needed = (warps_needed * 32 + kPermThreads - 1) / kPermThreads;
  // about 8 resident blocks per SM in total, shared out by each tensor's cost
  int weight[3] = {0, 0, 0}, weight_sum = 0;
  for (int t = 0; t < n_tensors; ++t) {
    weight[t] = (nrm != nullptr && nrm->gamma[t] != nullptr) ? 2 : 1;
    weight_sum += weight[t];
  }
  const long long total = (long long)sm_count() * 8;
  set.block_begin[0] = 0;
  for (int t = 0; t < 3; ++t) {
    long long b = 0;
    if (t < n_tensors) {
      b = total * weight[t] / weight_sum;
      if (b > blocks_needed) b = blocks_needed;
      if (b < 1) b = 1;
    }
    set.block_begin[t + 1] = set.block_begin[t] + int(b);
  }
  const dim3 grid{unsigned(set.block_begin[3]), 1u, 1u};
  const RowNorm none{};
  auto kernel = to_head ? permute_kernel<true, false, 0> : permute_kernel<false, false, 0>;
  if (nrm != nullptr) {
    switch (nrm->row_vec) {  // D / 8 for D a power of two in [8, 256]
      case 1: kernel = permute_kernel<true, true, 1>; break;
      case 2: kernel = permute_kernel<true, true, 2>; break;
      case 4: kernel = permute_kernel<true, true, 4>; break;
      case 8: kernel = permute_kernel<true, true, 8>; break;
      case 16: kernel = permute_kernel<true, true, 16>; break;
      case 32: kernel = permute_kernel<true, true, 32>; break;
      default: return cudaErrorInvalidValue;
    }
  }
  return launch_dependent(kernel, grid, dim3(kPermThreads), stream, set,
                          nrm != nullptr ? *nrm : none, P, S_local, int(run_vec), chunks,
                          int(n_items));
}

static RowNorm row_norm(const float* g0, const float* g1, const float* g2, int D, float eps,
                        float out_scale) {
  RowNorm n{};
  n.gamma[0] = g0;
  n.gamma[1] = g1;
  n.gamma[2] = g2;
  n.row_vec = D / 8;
  n.inv_d = 1.0f / float(D);  // D is a power of two: x * inv_d == x / D exactly
  n.eps = eps;
  n.out_scale = out_scale;
  return n;
}

cudaError_t launch_seq2head_qkv_norm(const void* const* src, void* const* dst, const float* gamma_q,
                                     const float* gamma_k, int P, int S_local, int D,
                                     long long run_vec, float eps, float out_scale,
                                     cudaStream_t stream) {
  const RowNorm n = row_norm(gamma_q, gamma_k, nullptr, D, eps, out_scale);
  return launch_permute(true, src, dst, 3, P, S_local, run_vec, stream, &n);
}

// Standalone RMSNorm over a flat [rows][D] array: item = 32 consecutive vectors (32/row_vec
// whole head rows), kPermUnroll items per warp in flight; same arithmetic as the fused form.
template <int kRowVec>
__global__ void __launch_bounds__(kPermThreads, 5) rmsnorm_kernel(const uint4* __restrict__ x,
                                                                  uint4* __restrict__ y,
                                                                  const float* __restrict__ gamma,
                                                                  int n_vec, int row_vec,
                                                                  float inv_d, float eps,
                                                                  float out_scale) {
  dependent_launch_gate();
  const int lane = threadIdx.x & 31;
  const int warp = int((blockIdx.x * kPermThreads + threadIdx.x) >> 5);
  const int n_warps = int((gridDim.x * kPermThreads) >> 5);
  float g[8];
  load_gamma8(gamma, (lane % row_vec) * 8, g);
  const int n_items = (n_vec + 31) >> 5;
  for (int it0 = warp * kPermUnroll; it0 < n_items; it0 += n_warps * kPermUnroll) {
    uint4 buf[kPermUnroll];
    bool live[kPermUnroll];
#pragma unroll
    for (int u = 0; u < kPermUnroll; ++u) {
      const int v = ((it0 + u) << 5) + lane;  // < 2^31: n_vec + 31 + 32 * kPermUnroll fits
      live[u] = it0 + u < n_items && v < n_vec;
      buf[u] = make_uint4(0u, 0u, 0u, 0u);
      if (live[u]) buf[u] = x[v];
    }
#pragma unroll
    for (int u = 0; u < kPermUnroll; ++u)
      buf[u] = rms_normalise<kRowVec>(buf[u], inv_d, eps, out_scale, g);
#pragma unroll
    for (int u = 0; u < kPermUnroll; ++u)
      if (live[u]) y[((it0 + u) << 5) + lane] = buf[u];
  }
}

cudaError_t launch_rmsnorm(const void* x, void* y, const float* gamma, long long rows, int D,
                           float eps, float out_scale, cudaStream_t stream) {
  const int row_vec = D / 8;
  const long long n_vec = rows * row_vec;
  // 32-bit vector indices, with room for a warp's last partial item
  if (n_vec > 0x7fffffffLL - 32 * (kPermUnroll + 1)) return cudaErrorInvalidValue;
  const long long warps_needed = ((n_vec + 31) / 32 + kPermUnroll - 1) / kPermUnroll;
  const long long blocks_needed = (warps_needed * 32 + kPermThreads - 1) / kPermThreads;
  const long long cap = (long long)sm_count() * 8;
  const long long blocks = blocks_needed < cap ? blocks_needed : cap;
  void (*kernel)(const uint4*, uint4*, const float*, int, int, float, float, float) = nullptr;
  switch (row_vec) {  // D / 8 for D a power of two in [8, 256]
    case 1: kernel = rmsnorm_kernel<1>; break;
    case 2: kernel = rmsnorm_kernel<2>; break;
    case 4: kernel = rmsnorm_kernel<4>; break;
    case 8: kernel = rmsnorm_kernel<8>; break;
    case 16: kernel = rmsnorm_kernel<16>; break;
    case 32: kernel = rmsnorm_kernel<32>; break;
    default: return cudaErrorInvalidValue;
  }
  return launch_dependent(kernel, dim3(unsigned(blocks)), dim3(kPermThreads), stream,
                          static_cast<const uint4*>(x), static_cast<uint4*>(y), gamma, int(n_vec),
                          row_vec, 1.0f / float(D), eps, out_scale);
}

cudaError_t launch_seq2head(const void* src, void* dst, int P, int S_local, long long run_vec,
                            cudaStream_t stream) {
  const void* s[1] = {src};
  void* d[1] = {dst};
  return launch_permute(true, s, d, 1, P, S_local, run_vec, stream);
}

cudaError_t launch_head2seq(const void* src, void* dst, int P, int S_local, long long run_vec,
                            cudaStream_t stream) {
  const void* s[1] = {src};
  void* d[1] = {dst};
  return launch_permute(false, s, d, 1, P, S_local, run_vec, stream);
}

cudaError_t launch_seq2head_n(const void* const* src, void* const* dst, int n, int P, int S_local,
                              long long run_vec, cudaStream_t stream) {
  return launch_permute(true, src, dst, n, P, S_local, run_vec, stream);
}

cudaError_t launch_exp2_poly_selftest(const float* t, float* out, int n, cudaStream_t stream) {
  const int pairs = (n + 1) / 2;
  exp2_poly_selftest_kernel<<<(pairs + 255) / 256, 256, 0, stream>>>(t, out, n);
  return cudaGetLastError();
}

cudaError_t launch_wait_timeout_selftest(int* err, long long limit, cudaStream_t stream) {
  wait_timeout_selftest_kernel<<<1, 32, 0, stream>>>(err, limit);
  return cudaGetLastError();
}

}  // namespace cpattn
