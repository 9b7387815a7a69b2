// kernels.h -- internal launchers behind the C ABI (include/cpattn.h).  Each returns the
// CUDA error of its launch; argument validation happens in api.cu before any of them runs.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

namespace cpattn {

// Default bounded-wait limit in SM clock cycles (about one second at 1.9 GHz).
constexpr long long kDefaultWaitLimit = 2000000000LL;

// tcgen05 attention, bf16 in, D in {64, 128}; tensor maps describe [B][S][H][D] bf16
// tensors with a 64 x 1 x 128 x 1 box and 128-byte swizzle.  With `accumulate` the result
// is merged into (out, lse) in place (the Ring Attention step) instead of overwriting it.
// With n_split > 1 the key blocks are divided into n_split contiguous ranges, one CTA per
// (query tile pair, range); range s writes its partial to out + s * B*Sq*H*D elements and
// lse + s * B*H*Sq (combine them with launch_combine).
cudaError_t launch_attn_fwd_sm100(const CUtensorMap& tq, const CUtensorMap& tk,
                                  const CUtensorMap& tv, void* out, float* lse, int B, int H,
                                  int Sq, int Skv, int D, float scale_log2, float rescale_log2,
                                  bool out_f32, bool accumulate, int n_split, int* err,
                                  long long wait_limit, cudaStream_t stream);

// Tail split of a single-pass attention launch: the first n_full work items (256-row tile
// pair x head x batch; whole waves of one CTA per SM) run over all keys, the last n_tail
// items -- the partial last wave, or that wave and the whole one before it -- each as
// `parts` key ranges whose fp32 partials go to a workspace and are folded by a combine
// kernel.  The plan minimises the modelled makespan; parts < 2: nothing to gain, run the
// plain launch.
struct TailSplit {
  int n_full, n_tail, parts;
};
TailSplit tail_split_plan(int B, int H, int Sq, int Skv);
size_t tail_split_workspace(const TailSplit& t, int D);  // bytes (0 when parts < 2)
// The largest workspace any key length can make the plan of (B, H, Sq) need.
size_t tail_split_workspace_bound(int B, int H, int Sq, int D);

// The attention (plain or accumulate) with a tail split, then the combine of the tail
// items' partials into (out, lse) -- with `accumulate`, merged into the running (out, lse).
cudaError_t launch_attn_fwd_sm100_tail(const CUtensorMap& tq, const CUtensorMap& tk,
                                       const CUtensorMap& tv, void* out, float* lse, int B, int H,
                                       int Sq, int Skv, int D, float scale_log2,
                                       float rescale_log2, bool out_f32, bool accumulate,
                                       const TailSplit& t, void* workspace, int* err,
                                       long long wait_limit, cudaStream_t stream);

// Fold the tail items' key-range partials (fp32 O rows [parts][n_tail][256][D], LSE
// [parts][n_tail][256]) -- and with `accumulate` the running (out, lse) -- into out / lse.
// Row (b, q, h) of out starts at element (b * batch_stride + q * token_stride + h) * D:
// [B][Sq][H][D] has batch_stride = Sq * H and token_stride = H; the Ulysses shards (b the
// head group, H its heads) have batch_stride = H and token_stride = H * B.  LSE is
// [B][H][Sq] either way.
cudaError_t launch_combine_tail(const float* ws_o, const float* ws_lse, int n_full, int n_tail,
                                int parts, void* out, float* lse, int B, int H, int Sq, int D,
                                int out_bytes, bool accumulate, long long batch_stride,
                                int token_stride, cudaStream_t stream);

// The fused Ulysses pass over all P head groups with a tail split (work items numbered tile
// pair fastest, then head, then group), then the combine of the tail items' partials.
cudaError_t launch_ulysses_fwd_sm100_tail(const CUtensorMap& tq, const CUtensorMap& tk,
                                          const CUtensorMap& tv, const CUtensorMap& tq16,
                                          const CUtensorMap& tk16, const CUtensorMap& tv16,
                                          void* out, float* lse, int P, int S_local, int H, int D,
                                          float scale_log2, float rescale_log2, bool out_f32,
                                          const TailSplit& t, void* workspace, int* err,
                                          long long wait_limit, cudaStream_t stream);

// Ulysses fused: q/k/v/out are [P][S_local][H][D] rank shards, each described by two tensor
// maps over dims (D, H, S_local, P): a 64 x 1 x 128 x 1 box and a 64 x 1 x 16 x 1 box (for
// tiles that straddle two shards); LSE is [P][H/P][P*S_local].  The launch computes head
// groups g_first .. g_first + n_groups - 1 (all P for the whole pass); it reads and writes
// only those groups' heads.
cudaError_t launch_ulysses_fwd_sm100(const CUtensorMap& tq, const CUtensorMap& tk,
                                     const CUtensorMap& tv, const CUtensorMap& tq16,
                                     const CUtensorMap& tk16, const CUtensorMap& tv16, void* out,
                                     float* lse, int P,
                                     int S_local, int H, int D, float scale_log2,
                                     float rescale_log2, bool out_f32, int g_first, int n_groups,
                                     int* err, long long wait_limit, cudaStream_t stream);

// Running-max policy of the tensor-core kernel: the reference max of a row moves (and O is
// rescaled) when a block's max exceeds it by more than this (log2 units), or when a key
// above it could weigh 1/8 or more of the row's result (see attn_sm100.cu).
constexpr float kRescaleLog2 = 8.0f;

// fp32 CUDA-core attention, D <= 256.
cudaError_t launch_attn_fwd_f32(const float* q, const float* k, const float* v, void* out,
                                float* lse, int B, int H, int Sq, int Skv, int D, float scale,
                                bool out_bf16, cudaStream_t stream);

// out = 0 and lse = -inf (the empty key set).
cudaError_t launch_fill_empty(void* out, size_t out_bytes, float* lse, size_t n_lse,
                              cudaStream_t stream);

// (O, LSE) merge; elem_bytes 2 (bf16) or 4 (f32).
cudaError_t launch_merge(const void* o_a, const float* lse_a, const void* o_b, const float* lse_b,
                         void* o, float* lse, int B, int H, int S, int D, int elem_bytes,
                         cudaStream_t stream);

// Fold n (1..8) split-KV partials [n][B][S][H][D] (elem_bytes dtype) + LSE [n][B][H][S]
// into (out, lse); with `accumulate` the running (out, lse) is one more term.
cudaError_t launch_combine(const void* part_o, const float* part_lse, int n, void* out, float* lse,
                           int B, int H, int S, int D, int elem_bytes, bool accumulate,
                           cudaStream_t stream);

// Ulysses permutes over 16-byte words; `run_vec` = Hp*D*elem_bytes/16.
cudaError_t launch_seq2head(const void* src, void* dst, int P, int S_local, long long run_vec,
                            cudaStream_t stream);
cudaError_t launch_head2seq(const void* src, void* dst, int P, int S_local, long long run_vec,
                            cudaStream_t stream);
// seq2head of n (1..3) same-shaped tensors in one launch.
cudaError_t launch_seq2head_n(const void* const* src, void* const* dst, int n, int P, int S_local,
                              long long run_vec, cudaStream_t stream);
// seq2head of Q, K, V in one launch with the RMSNorm of every Q and K head row fused in
// (src/dst: 3 tensors; D a power of two with D/8 dividing 32).
cudaError_t launch_seq2head_qkv_norm(const void* const* src, void* const* dst, const float* gamma_q,
                                     const float* gamma_k, int P, int S_local, int D,
                                     long long run_vec, float eps, float out_scale,
                                     cudaStream_t stream);
// RMSNorm of `rows` head rows of D bf16 (x and y may be the same buffer).
cudaError_t launch_rmsnorm(const void* x, void* y, const float* gamma, long long rows, int D,
                           float eps, float out_scale, cudaStream_t stream);

// One CTA waiting on an mbarrier nothing completes, with the attention kernel's bounded wait.
cudaError_t launch_wait_timeout_selftest(int* err, long long limit, cudaStream_t stream);

// The attention kernel's FMA-pipe 2^t (exp2_poly2) applied to n floats.
cudaError_t launch_exp2_poly_selftest(const float* t, float* out, int n, cudaStream_t stream);

int sm_count();

}  // namespace cpattn
