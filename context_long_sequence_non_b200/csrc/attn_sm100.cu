// attn_sm100.cu -- non-causal attention forward on B200 tensor cores (tcgen05 + TMEM + TMA).
//
// What it computes (AllGather KV / 环形注意力 Ring Attention sections of "Scaling AI
// Inference Across Multiple GPUs Using NVIDIA TensorRT with Multi-Device Inference
// Support", Figs. 2-3): for every (b, h, query row i)
//   O_i = sum_j softmax_j(scale * q_i . k_j) v_j,   LSE_i = ln sum_j exp(scale * q_i . k_j)
// streamed over 128-key blocks with an online softmax, so that the (O, LSE) of separate
// key chunks merge exactly afterwards (the Ring Attention step).
//
// Work decomposition.  A work item is 256 query rows (two 128-row Q tiles) of one (b, h)
// against a range of key blocks.  Two grid forms:
//   3-D grid (pairs * n_split, H, B): every item over all keys (n_split = 1), or over one of
//     n_split equal key ranges (split-KV, each range's partial written to its own slice);
//   1-D grid of n_full + n_tail * tail_parts CTAs ("tail split"): the first n_full items --
//     whole waves of the GPU -- over all keys, then the n_tail items of the last, partial
//     wave each split into tail_parts key ranges, so that the last wave is short instead
//     of mostly idle.  A tail part writes its normalised partial (O, LSE) in fp32 to a
//     workspace slot; a combine kernel folds the parts (and the running accumulator) after.
//
// Design (one CTA = 256 query rows of one (b, h), 12 warps):
//   warps 0-3  softmax for Q tile 0  (TMEM lanes 0..127, one thread per query row)
//   warps 4-7  softmax for Q tile 1
//   warp  8    TMA producer: Q0, Q1 once, then K_0, V_0, K_1, V_1, ... into a 4-slot ring
//   warp  9    TMEM allocator + single-thread tcgen05.mma issuer
// TMEM (512 columns): S0 | S1 (128 fp32 columns each; P_i is written back over S_i as
// bf16 pairs) | O0 | O1 (D fp32 columns each).  S = Q K^T runs smem x smem; O += P V
// takes P from TMEM and V from smem (MN-major).  While softmax works on one Q tile the
// tensor core runs the other tile's MMAs (ping-pong), and TMA prefetches ahead.
// Softmax works in base 2: x = s * scale * log2(e).  The row's reference max m is raised
// to a block's row max when that exceeds m by more than `rescale_log2` (2^8), or when a key
// above m could carry 1/8 or more of the row's final weight.  Any reference is exact in
// real arithmetic (the final normalisation uses the same m); the rule keeps every key that
// can dominate a row at P = 1 exactly in bf16 (so its rounding costs nothing), while the
// many small increases of the max in rows without a dominant key -- ~30 % of key blocks
// for iid logits -- no longer cost an O rescale.  O is rescaled in TMEM by the softmax
// warps when m moves.
// Every wait is bounded (mbar_wait): a stalled pipeline sets the device error word and
// the CTA drains and exits instead of hanging.
#include <cuda_runtime.h>

#include "kernels.h"
#include "sm100_ptx.cuh"

namespace cpattn {
namespace {

constexpr int kBlockM = 128;     // query rows per Q tile = TMEM lanes
constexpr int kBlockN = 128;     // keys per K/V tile
constexpr int kSlots = 4;        // K/V ring slots (K_j and V_j alternate)
constexpr int kThreads = 384;
constexpr int kWarpProducer = 8;
constexpr int kWarpMma = 9;
// Register split (setmaxnreg): the CTA launches with 168 x 384 = 64512 registers; the two
// softmax warpgroups take 216 each per thread and the producer/MMA warpgroup 72:
// 2 x 128 x 216 + 128 x 72 = 64512.  ptxas reports no spills for D = 64 and an 8-byte
// stack slot for D = 128 (8 B stored, 24 B loaded, in the producer/issuer warps' code,
// outside the per-key-block loop of the softmax warps).
constexpr uint32_t kRegsLaunch = 168, kRegsSoftmax = 216, kRegsOther = 72;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsOther <= kRegsLaunch * kThreads,
              "register split exceeds the launch allocation");
constexpr uint32_t kTmemCols = 512;
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;
// exp2 work split: of every 8 column pairs, this many go through the FMA-pipe polynomial
// and the rest through the special-function unit (ex2), which would otherwise be
// co-critical with the tensor core (one ex2 per score, 16 per clock per SM).
constexpr int kPolyPairs = 2;
// A key above the running reference max whose final weight in the row can reach
// 1/kMinorWeightInv moves the reference (and rescales O); lighter ones do not.
constexpr int kMinorWeightInv = 8;
// P handoff granularity: each block's P is stored and handed to the issuer in this many
// key chunks, so that O += P V of the first chunks runs while the rest of P is computed.
constexpr int kPChunks = 2;
constexpr int kChunkPairs = kBlockN / 2 / kPChunks;  // bf16 pairs (TMEM columns) per chunk
static_assert(kChunkPairs == 16 || kChunkPairs == 32, "P chunks of 32 or 64 keys");

template <int D>
struct Geometry {
  static constexpr int kBox = 64;                       // bf16 columns per TMA box (128 B)
  static constexpr int kBoxBytes = kBlockN * kBox * 2;  // 16 KB: 128 rows x 128 B
  static constexpr int kBoxes = D / kBox;
  static constexpr int kTileBytes = kBoxes * kBoxBytes; // one 128-row tile of Q, K or V
  static constexpr int kOffQ = 0;
  static constexpr int kOffSlots = 2 * kTileBytes;
  static constexpr int kBytes = kOffSlots + kSlots * kTileBytes;
  // + slack for 1024-B alignment; never below 120 KB so that one CTA, which takes all
  // 512 TMEM columns, is the only one resident on its SM
  static constexpr int kDynSmem = (kBytes + 1024) > 120 * 1024 ? (kBytes + 1024) : 120 * 1024;
};

struct __align__(8) Barriers {
  uint64_t q_full;
  uint64_t full[kSlots];
  uint64_t empty[kSlots];
  uint64_t s_full[2];
  uint64_t p_part[2][kPChunks];  // P chunk c of Q tile t stored (chunk 0: O rescaled too)
  uint64_t o_full;
  uint64_t drain;
};

// Addressing/epilogue modes of the kernel.
enum Mode : int {
  kPlain = 0,    // [B][S][H][D] in, O and LSE written
  kAccum = 1,    // as kPlain, but (O, LSE) merged into the running accumulator in place
  kSharded = 2,  // Ulysses fused: Q/K/V/O are [P][S_l][H*P][D] rank shards (see below)
};

template <int D, bool kOutF32, int kMode>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_sm100_kernel(const __grid_constant__ CUtensorMap tm_q,
                          const __grid_constant__ CUtensorMap tm_k,
                          const __grid_constant__ CUtensorMap tm_v,
                          const __grid_constant__ CUtensorMap tm_q16,
                          const __grid_constant__ CUtensorMap tm_k16,
                          const __grid_constant__ CUtensorMap tm_v16, void* __restrict__ out,
                          float* __restrict__ lse, int H, int Sq, int Skv, float scale_log2,
                          float rescale_log2, int s_local, int n_split, int b_first, int n_full,
                          int n_tail, int tail_parts, float* __restrict__ ws_o,
                          float* __restrict__ ws_lse, int* err, long long wait_limit) {
  using G = Geometry<D>;
  constexpr bool kAcc = kMode == kAccum;
  // kSharded: the DeepSpeed Ulysses path in one kernel.  The grid's z is the head group g
  // (P of them), y the head j inside it (H = heads per group); head g*H + j of the full
  // sequence is read straight from the sequence shards [P][S_l][H*P][D] (token t lives in
  // shard t / S_l, row t % S_l) with 16-row TMA boxes, so no box crosses a shard boundary
  // (S_l % 16 == 0), and O goes back to the same sharded layout: the all-to-alls become
  // addressing.  A tile inside one shard is a single 128-row box (tm_q/k/v); only tiles
  // that straddle a shard boundary use the 16-row maps (tm_q16/k16/v16).
  constexpr bool kShard = kMode == kSharded;
  extern __shared__ uint8_t smem_raw[];
  __shared__ Barriers bars;
  __shared__ uint32_t tmem_base_sh;
  __shared__ int abort_sh;

  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const uint32_t smem_base = smem_u32(smem);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  int pair, h, b, split, n_ranges;
  int slot = -1;  // tail split: this CTA's workspace slot (-1: writes the output itself)
  if (n_full < 0) {
    // 3-D grid.  split-KV: blockIdx.x = (query tile pair) * n_split + split; range `split`
    // writes its partial (O, LSE) to its own slice of out / lse
    split = n_split > 1 ? int(blockIdx.x % unsigned(n_split)) : 0;
    n_ranges = n_split;
    pair = int(blockIdx.x / unsigned(n_split));
    h = blockIdx.y;
    b = b_first + int(blockIdx.z);
    if (n_split > 1) {
      out = static_cast<char*>(out) + size_t(split) * gridDim.z * Sq * H * D * (kOutF32 ? 4 : 2);
      lse += size_t(split) * gridDim.z * H * Sq;
    }
  } else {
    // 1-D grid: whole items first, then the tail items' key ranges (items numbered tile
    // pair fastest, then head, then batch)
    const int x = int(blockIdx.x);
    int item = x;
    split = 0;
    n_ranges = 1;
    if (x >= n_full) {
      const int t = (x - n_full) / tail_parts;
      split = (x - n_full) - t * tail_parts;
      n_ranges = tail_parts;
      item = n_full + t;
      slot = split * n_tail + t;
    }
    const int n_pairs = (Sq + 2 * kBlockM - 1) / (2 * kBlockM);
    pair = item % n_pairs;
    h = (item / n_pairs) % H;
    b = b_first + item / n_pairs / H;
  }
  const int q_first = pair * (2 * kBlockM);
  const int head_coord = kShard ? b * H + h : h;  // head coordinate in the tensor maps
  const int n_kv_all = (Skv + kBlockN - 1) / kBlockN;
  const int kv_base = n_kv_all / n_ranges, kv_rem = n_kv_all % n_ranges;
  const int j0 = split * kv_base + (split < kv_rem ? split : kv_rem);  // first key block
  const int n_kv = kv_base + (split < kv_rem ? 1 : 0);                 // key blocks here
  volatile int* abort_flag = &abort_sh;

  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bars.q_full), 1);
    for (int s = 0; s < kSlots; ++s) {
      mbar_init(smem_u32(&bars.full[s]), 1);
      mbar_init(smem_u32(&bars.empty[s]), 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(smem_u32(&bars.s_full[t]), 1);
      for (int c = 0; c < kPChunks; ++c)
        mbar_init(smem_u32(&bars.p_part[t][c]), 4);  // one arrive per softmax warp
    }
    mbar_init(smem_u32(&bars.o_full), 1);
    mbar_init(smem_u32(&bars.drain), 1);
    abort_sh = 0;
    fence_mbar_init();
  }
  if (warp == kWarpProducer && lane == 0) {
    tma_prefetch_desc(&tm_q);
    tma_prefetch_desc(&tm_k);
    tma_prefetch_desc(&tm_v);
    if (kShard) {
      tma_prefetch_desc(&tm_q16);
      tma_prefetch_desc(&tm_k16);
      tma_prefetch_desc(&tm_v16);
    }
  }
  if (warp == kWarpMma) {
    tmem_alloc(smem_u32(&tmem_base_sh), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_base_sh;
  // The launch is a dependent one: the set-up above may overlap the previous kernel's last
  // wave, nothing below reads or writes global memory before that kernel has completed, and
  // the next kernel may be scheduled from here on (it waits the same way).
  griddep_wait();
  griddep_release();

  if (warp < 8) {
    // ------------------------------------------------------------------ softmax warps
    regs_inc<kRegsSoftmax>();
    const int tile = warp >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;  // row within the Q tile == TMEM lane
    const uint32_t lane_bits = uint32_t(quarter * 32) << 16;
    const uint32_t t_s = tmem + lane_bits + uint32_t(tile * kBlockN);
    const uint32_t t_o = tmem + lane_bits + uint32_t(2 * kBlockN + tile * D);
    const uint32_t bar_s = smem_u32(&bars.s_full[tile]);
    const uint32_t bar_p0 = smem_u32(&bars.p_part[tile][0]);  // chunk c at + 8 c
    float m = -INFINITY;  // running (possibly stale) max of x = s * scale * log2(e)
    float l = 0.f;        // running sum of 2^(x - m)
    bool ok = true;

    for (int j = 0; j < n_kv; ++j) {
      ok = mbar_wait(bar_s, j & 1, abort_flag, err, wait_limit);
      if (!__all_sync(0xffffffffu, ok)) { ok = false; break; }
      tc_fence_after();

      float x[kBlockN];
      {
        uint32_t r[kBlockN];
        tmem_ld128(t_s, r);  // the whole S row, one wait
#pragma unroll
        for (int c = 0; c < kBlockN; ++c) x[c] = __uint_as_float(r[c]);
      }
      const int valid = Skv - (j0 + j) * kBlockN;  // keys of this block inside the sequence
      if (valid < kBlockN) {
#pragma unroll
        for (int c = 0; c < kBlockN; ++c)
          if (c >= valid) x[c] = -INFINITY;
      }
      // row maximum of the raw logits (scale > 0 is a precondition of the call): a tree of
      // three-input max, 64 instructions and 5 levels deep (a chain would be latency-bound)
      float mx;
      {
        float l1[44];
#pragma unroll
        for (int i = 0; i < 42; ++i) l1[i] = max3(x[3 * i], x[3 * i + 1], x[3 * i + 2]);
        l1[42] = x[126];
        l1[43] = x[127];
        float l2[16];
#pragma unroll
        for (int i = 0; i < 14; ++i) l2[i] = max3(l1[3 * i], l1[3 * i + 1], l1[3 * i + 2]);
        l2[14] = l1[42];
        l2[15] = l1[43];
        float l3[6];
#pragma unroll
        for (int i = 0; i < 5; ++i) l3[i] = max3(l2[3 * i], l2[3 * i + 1], l2[3 * i + 2]);
        l3[5] = l2[15];
        mx = fmaxf(max3(l3[0], l3[1], l3[2]), max3(l3[3], l3[4], l3[5]));
      }
      const float m_tile = mx * scale_log2;
      float alpha = 1.0f;
      bool rescale = false;
      if (j == 0) {
        m = m_tile;
      } else {
        // The reference m moves to the block max (O rescaled in TMEM) when the block max
        // exceeds it by more than rescale_log2, or when a key above it could carry
        // 1/kMinorWeightInv or more of the row's final weight: such a key's final weight is
        // at most 2^d / (l + 2^d) with d = m_tile - m (l only grows afterwards), and after
        // the move it gets P = 1 exactly.  A key below that weight leaves the reference
        // where it is: its P in (1, 2^rescale_log2] is rounded to bf16 like any other P, at
        // a share of the result under 1/kMinorWeightInv.
        const float d = m_tile - m;
        bool grow = d > rescale_log2;
        if (!grow && d > 0.f) grow = ex2(d) * float(kMinorWeightInv - 1) >= l;
        rescale = __any_sync(0xffffffffu, grow);
        if (rescale) {
          const float m_new = grow ? m_tile : m;
          alpha = ex2(m - m_new);
          m = m_new;
          l *= alpha;
        }
      }
      // p = 2^(x * scale_log2 - m): most pairs on the special-function unit, kPolyPairs of
      // every 8 pairs on the FMA pipe (exp2_poly2); p rounded to bf16 for the PV product and
      // written over S as bf16 pairs; the row sum keeps the unrounded fp32 p.  The keys go
      // in kPChunks chunks with one handoff each, so that the issuer runs O += P V of the
      // first chunks while the rest of P is computed.
      const float2 sl2 = make_float2(scale_log2, scale_log2);
      const float2 nm2 = make_float2(-m, -m);
      float2 acc0 = make_float2(0.f, 0.f), acc1 = make_float2(0.f, 0.f);
#pragma unroll
      for (int part = 0; part < kPChunks; ++part) {
        uint32_t pk[kChunkPairs];
#pragma unroll
        for (int e = 0; e < kChunkPairs; ++e) {
          const int c = 2 * (part * kChunkPairs + e);
          const float2 t = ffma2(make_float2(x[c], x[c + 1]), sl2, nm2);
          float2 pv;
          if ((e & 7) >= 8 - kPolyPairs) {
            pv = exp2_poly2(t);
          } else {
            pv.x = ex2(t.x);
            pv.y = ex2(t.y);
          }
          if (e & 1) acc1 = fadd2(acc1, pv);
          else acc0 = fadd2(acc0, pv);
          pk[e] = pack_bf16x2(pv.x, pv.y);
        }
        tmem_st_any(t_s + part * kChunkPairs, pk);
        if (part == 0 && rescale) {
          // rescale this warp's O rows by alpha before the first PV chunk accumulates into
          // them: PV of the previous block has completed (the issuer committed this
          // block's S after it), and no PV of this block starts before the arrive below
          const float2 a2 = make_float2(alpha, alpha);
#pragma unroll
          for (int oc = 0; oc < D / 32; ++oc) {
            uint32_t r[32];
            tmem_ld32(t_o + oc * 32, r);
#pragma unroll
            for (int c = 0; c < 32; c += 2) {
              const float2 o =
                  fmul2(make_float2(__uint_as_float(r[c]), __uint_as_float(r[c + 1])), a2);
              r[c] = __float_as_uint(o.x);
              r[c + 1] = __float_as_uint(o.y);
            }
            tmem_st32(t_o + oc * 32, r);
          }
        }
        // hand this chunk over: every lane's TMEM stores complete, then one arrive per warp
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar_p0 + 8 * part);
      }
      const float2 acc = fadd2(acc0, acc1);
      l += acc.x + acc.y;
    }

    // ------------------------------------------------------------------ epilogue
    const int q = q_first + tile * kBlockM + row;
    const bool in_range = q < Sq;
    const int qr = in_range ? q : 0;
    // sharded layout: token q = r * S_l + s sits at row q of the flattened [P][S_l] shards
    // (P = Sq / S_l head groups in all, whichever of them this launch covers)
    const size_t row_off = kShard ? (size_t(qr) * (H * (Sq / s_local)) + head_coord) * size_t(D)
                                  : ((size_t(b) * Sq + qr) * H + h) * size_t(D);
    const size_t lse_idx = (size_t(b) * H + h) * Sq + (in_range ? q : 0);
    // bf16 accumulate: the running row and its LSE are loaded now, before the last
    // O += P V has completed, so that one memory round trip overlaps it instead of one per
    // 32-column chunk after it.  (An empty accumulator's row may hold anything: it is
    // loaded but never used.)
    constexpr bool kPreload = kAcc && !kOutF32;
    uint4 acc_row[kPreload ? D / 8 : 1];
    float la_pre = -INFINITY;
    if constexpr (kPreload) {
      if (ok && slot < 0 && in_range) {
        la_pre = lse[lse_idx];
        const uint4* src = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(out) + row_off);
#pragma unroll
        for (int e = 0; e < D / 8; ++e) acc_row[e] = src[e];
      }
    }
    if (ok) {
      ok = mbar_wait(smem_u32(&bars.o_full), 0, abort_flag, err, wait_limit);
      ok = __all_sync(0xffffffffu, ok);
    }
    if (ok) {
      tc_fence_after();
      // this block's result: O_c = O_tmem / l, LSE_c = ln(2^m * l) = (m + log2 l) * ln 2
      const float lc2 = m + log2f(l);  // LSE_c in base 2
      float fa = 0.f, fc = 1.0f / l;   // written row = fa * O_acc + fc * O_tmem
      float lse_out = lc2 * kLn2;
      if (slot >= 0) {
        // tail split: the normalised partial of this key range, fp32, to workspace row
        // (slot, tile * 128 + row); the combine kernel folds the ranges afterwards
        const size_t wrow = size_t(slot) * (2 * kBlockM) + tile * kBlockM + row;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(t_o + c * 32, r);
          if (in_range) {
            float4* dst = reinterpret_cast<float4*>(ws_o + wrow * D + c * 32);
#pragma unroll
            for (int e = 0; e < 8; ++e)
              dst[e] = make_float4(__uint_as_float(r[4 * e]) * fc, __uint_as_float(r[4 * e + 1]) * fc,
                                   __uint_as_float(r[4 * e + 2]) * fc, __uint_as_float(r[4 * e + 3]) * fc);
          }
        }
        if (in_range) ws_lse[wrow] = lse_out;
      } else {
        if constexpr (kAcc) {
          // Ring Attention step fused into the epilogue: merge (O_c, LSE_c) into the running
          // (O_acc, LSE_acc) in place; an empty accumulator (LSE_acc = -inf) takes O_c
          if (in_range) {
            const float la2 = (kPreload ? la_pre : lse[lse_idx]) * kLog2e;
            const float mx = fmaxf(la2, lc2);
            const float wa = exp2f(la2 - mx), wc = exp2f(lc2 - mx);
            const float tot = wa + wc;
            fa = wa / tot;
            fc = wc / (tot * l);
            lse_out = (mx + log2f(tot)) * kLn2;
          }
        }
        // one 32-column chunk of the row: scaled (and merged into the accumulator) and stored
        auto store_chunk = [&](int c, const uint32_t (&r)[32]) {
          if (!in_range) return;
          if constexpr (kOutF32) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + row_off + c * 32);
  #pragma unroll
            for (int e = 0; e < 8; ++e) {
              float4 v = make_float4(__uint_as_float(r[4 * e]) * fc, __uint_as_float(r[4 * e + 1]) * fc,
                                     __uint_as_float(r[4 * e + 2]) * fc, __uint_as_float(r[4 * e + 3]) * fc);
              if (kAcc && fa != 0.f) {  // an empty accumulator row is never read
                const float4 a = dst[e];
                v.x = fmaf(fa, a.x, v.x);
                v.y = fmaf(fa, a.y, v.y);
                v.z = fmaf(fa, a.z, v.z);
                v.w = fmaf(fa, a.w, v.w);
              }
              dst[e] = v;
            }
          } else {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + row_off + c * 32);
  #pragma unroll
            for (int e = 0; e < 4; ++e) {
              float o[8];
  #pragma unroll
              for (int t = 0; t < 8; ++t) o[t] = __uint_as_float(r[8 * e + t]) * fc;
              if (kAcc && fa != 0.f) {  // an empty accumulator's row is not used
                uint4 a;
                if constexpr (kPreload) a = acc_row[c * 4 + e];
                else a = dst[e];
                const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
  #pragma unroll
                for (int t = 0; t < 4; ++t) {
                  o[2 * t] = fmaf(fa, __uint_as_float(aw[t] << 16), o[2 * t]);
                  o[2 * t + 1] = fmaf(fa, __uint_as_float(aw[t] & 0xFFFF0000u), o[2 * t + 1]);
                }
              }
              uint4 v;
              v.x = pack_bf16x2(o[0], o[1]);
              v.y = pack_bf16x2(o[2], o[3]);
              v.z = pack_bf16x2(o[4], o[5]);
              v.w = pack_bf16x2(o[6], o[7]);
              dst[e] = v;
            }
          }
        };
        if constexpr (kPreload) {
  #pragma unroll
          for (int c = 0; c < D / 32; ++c) {  // unrolled: acc_row is indexed statically
            uint32_t r[32];
            tmem_ld32(t_o + c * 32, r);
            store_chunk(c, r);
          }
        } else {
  #pragma unroll 1
          for (int c = 0; c < D / 32; ++c) {
            uint32_t r[32];
            tmem_ld32(t_o + c * 32, r);
            store_chunk(c, r);
          }
        }
        if (in_range && lse != nullptr) lse[lse_idx] = lse_out;
      }
    }
  } else {
    regs_dec<kRegsOther>();
  }
  if (warp == kWarpProducer) {
    // ------------------------------------------------------------------ TMA producer
    if (elect_one()) {
      // one 128-row tile starting at token t0 into `dst`: a 64-column box per 128-byte
      // column block; sharded inputs take eight 16-row boxes, each inside one rank shard
      auto load_tile = [&](const CUtensorMap* map, const CUtensorMap* map16, uint32_t dst,
                           uint32_t bar, int t0) {
        if constexpr (!kShard) {
#pragma unroll
          for (int bx = 0; bx < G::kBoxes; ++bx)
            tma_load_4d(dst + bx * G::kBoxBytes, map, bar, bx * G::kBox, head_coord, t0, b);
        } else {
          int r = t0 / s_local;  // rank shard (== P past the end: zero-filled)
          int sr = t0 - r * s_local;
          if (sr + kBlockN <= s_local) {
#pragma unroll
            for (int bx = 0; bx < G::kBoxes; ++bx)
              tma_load_4d(dst + bx * G::kBoxBytes, map, bar, bx * G::kBox, head_coord, sr, r);
          } else {
#pragma unroll 1
            for (int i = 0; i < kBlockN / 16; ++i) {
#pragma unroll
              for (int bx = 0; bx < G::kBoxes; ++bx)
                tma_load_4d(dst + bx * G::kBoxBytes + i * 16 * 128, map16, bar, bx * G::kBox,
                            head_coord, sr, r);
              sr += 16;
              if (sr >= s_local) {
                sr -= s_local;
                ++r;
              }
            }
          }
        }
      };
      const uint32_t bar_q = smem_u32(&bars.q_full);
      mbar_arrive_expect_tx(bar_q, 2 * G::kTileBytes);
#pragma unroll
      for (int t = 0; t < 2; ++t)
        load_tile(&tm_q, &tm_q16, smem_base + G::kOffQ + t * G::kTileBytes, bar_q,
                  q_first + t * kBlockM);
      int issued = 0;
      for (int use = 0; use < 2 * n_kv; ++use) {
        const int slot = use % kSlots;
        const uint32_t ph = uint32_t(use / kSlots) & 1u;
        if (!mbar_wait(smem_u32(&bars.empty[slot]), ph ^ 1u, abort_flag, err, wait_limit)) break;
        const uint32_t bar_f = smem_u32(&bars.full[slot]);
        mbar_arrive_expect_tx(bar_f, G::kTileBytes);
        load_tile((use & 1) ? &tm_v : &tm_k, (use & 1) ? &tm_v16 : &tm_k16,
                  smem_base + G::kOffSlots + slot * G::kTileBytes, bar_f,
                  (j0 + (use >> 1)) * kBlockN);
        issued = use + 1;
      }
      // drain: every issued copy must have landed before the CTA's shared memory is
      // released (immediate on the normal path, where the consumer already saw them)
      drain_wait(bar_q, 0, wait_limit);
      for (int use = issued - kSlots < 0 ? 0 : issued - kSlots; use < issued; ++use)
        drain_wait(smem_u32(&bars.full[use % kSlots]), uint32_t(use / kSlots) & 1u, wait_limit);
    }
    __syncwarp();
  } else if (warp == kWarpMma) {
    // ------------------------------------------------------------------ MMA issuer
    if (elect_one()) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBlockM, kBlockN, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBlockM, D, true);
      const uint32_t q_addr[2] = {smem_base + G::kOffQ, smem_base + G::kOffQ + G::kTileBytes};
      const uint32_t t_s[2] = {tmem, tmem + kBlockN};
      const uint32_t t_o[2] = {tmem + 2 * kBlockN, tmem + 2 * kBlockN + D};

      // S_t = Q_t K^T over D in K=16 steps; K-major 128-B swizzled operands: 32 B per
      // step inside a 128-B row, the next 64 columns in the next box
      auto issue_qk = [&](int t, uint32_t k_addr) {
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * G::kBoxBytes + (kk & 3) * 32;
          mma_ss(t_s[t], sdesc_sw128(q_addr[t] + off, 16, 1024),
                 sdesc_sw128(k_addr + off, 16, 1024), idesc_qk, kk > 0 ? 1u : 0u);
        }
      };
      // O_t += P_t V over the 128 keys in K=16 steps; P from TMEM (8 columns = 16 bf16
      // per step), V MN-major: 16 key rows = 2 KB per step, the d halves one box apart
      constexpr int kStepsPerChunk = kBlockN / 16 / kPChunks;
      auto issue_pv_chunk = [&](int t, uint32_t v_addr, bool accumulate, int part) {
#pragma unroll
        for (int kk = part * kStepsPerChunk; kk < (part + 1) * kStepsPerChunk; ++kk) {
          mma_ts(t_o[t], t_s[t] + kk * 8, sdesc_sw128(v_addr + kk * 16 * 128, G::kBoxBytes, 1024),
                 idesc_pv, (accumulate || kk > 0) ? 1u : 0u);
        }
      };
      auto slot_addr = [&](int use) {
        return smem_base + G::kOffSlots + (use % kSlots) * G::kTileBytes;
      };
      // O_t += P_t V, chunk by chunk as the softmax warps hand P over
      auto issue_pv = [&](int t, uint32_t v_addr, int j) {
#pragma unroll
        for (int part = 0; part < kPChunks; ++part) {
          if (!mbar_wait(smem_u32(&bars.p_part[t][part]), uint32_t(j) & 1u, abort_flag, err,
                         wait_limit))
            return false;
          tc_fence_after();
          issue_pv_chunk(t, v_addr, j > 0 || part > 0, part);
        }
        return true;
      };
      auto wait_full = [&](int use) {
        return mbar_wait(smem_u32(&bars.full[use % kSlots]), uint32_t(use / kSlots) & 1u,
                         abort_flag, err, wait_limit);
      };

      bool ok = mbar_wait(smem_u32(&bars.q_full), 0, abort_flag, err, wait_limit) && wait_full(0);
      if (ok) {
        tc_fence_after();
        issue_qk(0, slot_addr(0));
        tc_commit(smem_u32(&bars.s_full[0]));
        issue_qk(1, slot_addr(0));
        tc_commit(smem_u32(&bars.s_full[1]));
        tc_commit(smem_u32(&bars.empty[0]));
      }
      for (int j = 0; ok && j < n_kv; ++j) {
        const int use_v = 2 * j + 1, use_k = 2 * j + 2;
        const bool more = j + 1 < n_kv;
        if (!(ok = wait_full(use_v))) break;
        if (!(ok = issue_pv(0, slot_addr(use_v), j))) break;
        if (more) {
          if (!(ok = wait_full(use_k))) break;
          tc_fence_after();
          issue_qk(0, slot_addr(use_k));
          tc_commit(smem_u32(&bars.s_full[0]));
        }
        if (!(ok = issue_pv(1, slot_addr(use_v), j))) break;
        tc_commit(smem_u32(&bars.empty[use_v % kSlots]));
        if (more) {
          issue_qk(1, slot_addr(use_k));
          tc_commit(smem_u32(&bars.s_full[1]));
          tc_commit(smem_u32(&bars.empty[use_k % kSlots]));
        }
      }
      if (ok) tc_commit(smem_u32(&bars.o_full));
      // drain: no MMA may still be writing TMEM when it is freed
      tc_commit(smem_u32(&bars.drain));
      drain_wait(smem_u32(&bars.drain), 0, wait_limit);
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kWarpMma) tmem_dealloc(tmem, kTmemCols);
}

// Launch arguments shared by every mode and grid form.
struct Launch {
  dim3 grid;
  int H, Sq, Skv, s_local, n_split, b_first;
  int n_full, n_tail, tail_parts;  // n_full < 0: 3-D grid form
  float* ws_o;
  float* ws_lse;
  float scale_log2, rescale_log2;
  int* err;
  long long wait_limit;
};

template <int D, bool kOutF32, int kMode>
cudaError_t launch(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                   const CUtensorMap& tq16, const CUtensorMap& tk16, const CUtensorMap& tv16,
                   void* out, float* lse, const Launch& a, cudaStream_t stream) {
  using G = Geometry<D>;
  auto kernel = attn_fwd_sm100_kernel<D, kOutF32, kMode>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       G::kDynSmem);
  if (e != cudaSuccess) return e;
  // launched as a dependent of the previous kernel on the stream (see griddep_wait)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = a.grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = G::kDynSmem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, tq, tk, tv, tq16, tk16, tv16, out, lse, a.H, a.Sq, a.Skv,
                            a.scale_log2, a.rescale_log2, a.s_local, a.n_split, a.b_first,
                            a.n_full, a.n_tail, a.tail_parts, a.ws_o, a.ws_lse, a.err,
                            a.wait_limit);
}

template <int D, int kMode>
cudaError_t launch_o(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     const CUtensorMap& tq16, const CUtensorMap& tk16, const CUtensorMap& tv16,
                     void* out, float* lse, const Launch& a, bool out_f32, cudaStream_t stream) {
  return out_f32 ? launch<D, true, kMode>(tq, tk, tv, tq16, tk16, tv16, out, lse, a, stream)
                 : launch<D, false, kMode>(tq, tk, tv, tq16, tk16, tv16, out, lse, a, stream);
}

template <int D>
cudaError_t launch_m(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                     const CUtensorMap& tq16, const CUtensorMap& tk16, const CUtensorMap& tv16,
                     void* out, float* lse, const Launch& a, bool out_f32, int mode,
                     cudaStream_t stream) {
  switch (mode) {
    case kAccum:
      return launch_o<D, kAccum>(tq, tk, tv, tq16, tk16, tv16, out, lse, a, out_f32, stream);
    case kSharded:
      return launch_o<D, kSharded>(tq, tk, tv, tq16, tk16, tv16, out, lse, a, out_f32, stream);
    default:
      return launch_o<D, kPlain>(tq, tk, tv, tq16, tk16, tv16, out, lse, a, out_f32, stream);
  }
}

cudaError_t launch_any(const CUtensorMap& tq, const CUtensorMap& tk, const CUtensorMap& tv,
                       const CUtensorMap& tq16, const CUtensorMap& tk16, const CUtensorMap& tv16,
                       void* out, float* lse, int D, const Launch& a, bool out_f32, int mode,
                       cudaStream_t stream) {
  if (D == 128) return launch_m<128>(tq, tk, tv, tq16, tk16, tv16, out, lse, a, out_f32, mode, stream);
  return launch_m<64>(tq, tk, tv, tq16, tk16, tv16, out, lse, a, out_f32, mode, stream);
}

}  // namespace

cudaError_t launch_attn_fwd_sm100(const CUtensorMap& tq, const CUtensorMap& tk,
                                  const CUtensorMap& tv, void* out, float* lse, int B, int H,
                                  int Sq, int Skv, int D, float scale_log2, float rescale_log2,
                                  bool out_f32, bool accumulate, int n_split, int* err,
                                  long long wait_limit, cudaStream_t stream) {
  Launch a{};
  a.grid = dim3(((Sq + 2 * kBlockM - 1) / (2 * kBlockM)) * n_split, H, B);
  a.H = H, a.Sq = Sq, a.Skv = Skv, a.s_local = 0, a.n_split = n_split, a.b_first = 0;
  a.n_full = -1, a.n_tail = 0, a.tail_parts = 1, a.ws_o = nullptr, a.ws_lse = nullptr;
  a.scale_log2 = scale_log2, a.rescale_log2 = rescale_log2, a.err = err, a.wait_limit = wait_limit;
  return launch_any(tq, tk, tv, tq, tk, tv, out, lse, D, a, out_f32, accumulate ? kAccum : kPlain,
                    stream);
}

cudaError_t launch_attn_fwd_sm100_tail(const CUtensorMap& tq, const CUtensorMap& tk,
                                       const CUtensorMap& tv, void* out, float* lse, int B, int H,
                                       int Sq, int Skv, int D, float scale_log2,
                                       float rescale_log2, bool out_f32, bool accumulate,
                                       const TailSplit& t, void* workspace, int* err,
                                       long long wait_limit, cudaStream_t stream) {
  const size_t rows = size_t(t.parts) * t.n_tail * (2 * kBlockM);
  Launch a{};
  a.grid = dim3(unsigned(t.n_full + t.n_tail * t.parts), 1, 1);
  a.H = H, a.Sq = Sq, a.Skv = Skv, a.s_local = 0, a.n_split = 1, a.b_first = 0;
  a.n_full = t.n_full, a.n_tail = t.n_tail, a.tail_parts = t.parts;
  a.ws_o = static_cast<float*>(workspace);
  a.ws_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                      ((rows * D * 4 + 255) & ~size_t(255)));
  a.scale_log2 = scale_log2, a.rescale_log2 = rescale_log2, a.err = err, a.wait_limit = wait_limit;
  cudaError_t e = launch_any(tq, tk, tv, tq, tk, tv, out, lse, D, a, out_f32,
                             accumulate ? kAccum : kPlain, stream);
  if (e != cudaSuccess) return e;
  return launch_combine_tail(a.ws_o, a.ws_lse, t.n_full, t.n_tail, t.parts, out, lse, B, H, Sq,
                             D, out_f32 ? 4 : 2, accumulate, /*batch_stride=*/Sq * H,
                             /*token_stride=*/H, stream);
}

cudaError_t launch_ulysses_fwd_sm100_tail(const CUtensorMap& tq, const CUtensorMap& tk,
                                          const CUtensorMap& tv, const CUtensorMap& tq16,
                                          const CUtensorMap& tk16, const CUtensorMap& tv16,
                                          void* out, float* lse, int P, int S_local, int H, int D,
                                          float scale_log2, float rescale_log2, bool out_f32,
                                          const TailSplit& t, void* workspace, int* err,
                                          long long wait_limit, cudaStream_t stream) {
  const int S = P * S_local, Hp = H / P;
  const size_t rows = size_t(t.parts) * t.n_tail * (2 * kBlockM);
  Launch a{};
  a.grid = dim3(unsigned(t.n_full + t.n_tail * t.parts), 1, 1);
  a.H = Hp, a.Sq = S, a.Skv = S, a.s_local = S_local, a.n_split = 1, a.b_first = 0;
  a.n_full = t.n_full, a.n_tail = t.n_tail, a.tail_parts = t.parts;
  a.ws_o = static_cast<float*>(workspace);
  a.ws_lse = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                      ((rows * D * 4 + 255) & ~size_t(255)));
  a.scale_log2 = scale_log2, a.rescale_log2 = rescale_log2, a.err = err, a.wait_limit = wait_limit;
  cudaError_t e = launch_any(tq, tk, tv, tq16, tk16, tv16, out, lse, D, a, out_f32, kSharded,
                             stream);
  if (e != cudaSuccess) return e;
  // token q of head group g, head j: row q of the flattened [P][S_local] shards, head g*Hp + j
  return launch_combine_tail(a.ws_o, a.ws_lse, t.n_full, t.n_tail, t.parts, out, lse, P, Hp, S,
                             D, out_f32 ? 4 : 2, false, /*batch_stride=*/Hp, /*token_stride=*/H,
                             stream);
}

cudaError_t launch_ulysses_fwd_sm100(const CUtensorMap& tq, const CUtensorMap& tk,
                                     const CUtensorMap& tv, const CUtensorMap& tq16,
                                     const CUtensorMap& tk16, const CUtensorMap& tv16, void* out,
                                     float* lse, int P, int S_local, int H, int D,
                                     float scale_log2, float rescale_log2, bool out_f32,
                                     int g_first, int n_groups, int* err, long long wait_limit,
                                     cudaStream_t stream) {
  const int S = P * S_local, Hp = H / P;
  Launch a{};
  a.grid = dim3((S + 2 * kBlockM - 1) / (2 * kBlockM), Hp, n_groups);
  a.H = Hp, a.Sq = S, a.Skv = S, a.s_local = S_local, a.n_split = 1, a.b_first = g_first;
  a.n_full = -1, a.n_tail = 0, a.tail_parts = 1, a.ws_o = nullptr, a.ws_lse = nullptr;
  a.scale_log2 = scale_log2, a.rescale_log2 = rescale_log2, a.err = err, a.wait_limit = wait_limit;
  return launch_any(tq, tk, tv, tq16, tk16, tv16, out, lse, D, a, out_f32, kSharded, stream);
}

}  // namespace cpattn
