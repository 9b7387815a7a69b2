/*
 * cpattn.h -- C ABI of the per-rank context-parallel attention hot path (B200, sm_100a).
 *
 * The operations come from the context-parallel attention strategies described in
 * "Scaling AI Inference Across Multiple GPUs Using NVIDIA TensorRT with Multi-Device
 * Inference Support" (NVIDIA developer blog): AllGather KV (Fig. 2), 环形注意力 /
 * Ring Attention with online softmax (Fig. 3) and DeepSpeed Ulysses (Fig. 4).  The
 * pages print no interface for this compute; the calls below are this library's own.
 *
 * Layout of every activation tensor (reading of the (seq, batch, heads, dim) reshape in
 * the attention_mdtrt guide "TensorRT 多设备注意力推理实战", section 模型的核心结构):
 *   Q, K, V, O : [B][S][H][D] row-major (token-major, heads interleaved, D contiguous)
 *   LSE        : [B][H][Sq]  float32, natural log of the sum of exp of the scaled logits
 *
 * Conventions shared by every call
 *   - Ownership: the caller allocates and owns every buffer (device memory unless a
 *     call says otherwise).  The library allocates nothing per call; it keeps one
 *     device error word per device for bounded-wait timeouts.
 *   - Asynchrony: work is enqueued on `stream` (NULL = legacy default stream) and the
 *     call returns without waiting.  Argument errors are detected on the host, before
 *     anything is launched, and nothing is written then.
 *   - Return value: a cpattn_status.  CPATTN_ERR_CUDA means a launch failed; the CUDA
 *     error is left for the caller's next CUDA call to report as well.
 *   - Tensor pointers (Q, K, V, O, permute buffers) must be 16-byte aligned and LSE
 *     pointers 4-byte aligned (CPATTN_ERR_ALIGN otherwise).
 *   - Every argument is checked before the first CUDA call, so argument errors are
 *     reported the same way with or without a GPU.
 *   - Stream capture: a call that takes a stream only launches kernels on it (kernels
 *     launched as programmatic dependents of the previous one), so it can be recorded
 *     into a CUDA graph and replayed; the graph keeps the pointers and sizes of the
 *     recorded call.  Make one ordinary call first: the first call on a device loads the
 *     module and looks up the device error word.  Not capturable: cpattn_ulysses_host
 *     (its own streams and events), cpattn_device_error (synchronises the device), and
 *     the first cpattn_fwd_split_noalloc call on a device (see there).
 */
#ifndef CPATTN_H
#define CPATTN_H

#include <stddef.h>

#if defined(__GNUC__)
#define CPATTN_API __attribute__((visibility("default")))
#else
#define CPATTN_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same object as cudaStream_t / CUstream; declared here so this header needs no CUDA
 * include. */
typedef struct CUstream_st* cpattn_stream_t;

typedef enum {
  CPATTN_BF16 = 0, /* bfloat16, round-to-nearest-even on output */
  CPATTN_F32 = 1   /* IEEE float32 */
} cpattn_dtype;

typedef enum {
  CPATTN_OK = 0,
  CPATTN_ERR_NULL = 1,        /* a required pointer is NULL */
  CPATTN_ERR_SHAPE = 2,       /* a size is out of range or inconsistent */
  CPATTN_ERR_ALIGN = 3,       /* a pointer is not suitably aligned */
  CPATTN_ERR_UNSUPPORTED = 4, /* valid request the library has no kernel for */
  CPATTN_ERR_CUDA = 5,        /* a CUDA runtime/driver call or launch failed */
  CPATTN_ERR_DEVICE_TIMEOUT = 6 /* a kernel's bounded wait ran out (device error word) */
} cpattn_status;

/*
 * cpattn_fwd -- non-causal scaled dot-product attention with its log-sum-exp.
 *
 * Defines (AllGather KV and Ring Attention sections, Figs. 2-3; the QK^T -> Softmax ->
 * Attn*V core of the attention_mdtrt guide):
 *   s[b,h,i,j] = scale * sum_d q[b,i,h,d] * k[b,j,h,d]
 *   lse[b,h,i] = ln sum_j exp(s[b,h,i,j])
 *   out[b,i,h,:] = sum_j exp(s[b,h,i,j] - lse[b,h,i]) * v[b,j,h,:]
 * No mask.  With Sq != Skv this is one rank's AllGather-KV attention or one Ring
 * Attention chunk; the (out, lse) pair is what cpattn_merge folds.
 *
 * q   : [B][Sq][H][D]  in_dtype        k, v : [B][Skv][H][D] in_dtype
 * out : [B][Sq][H][D]  out_dtype       lse  : [B][H][Sq] float32, or NULL to skip it
 * B, H, Sq >= 1; Skv >= 0 (Skv = 0 gives out = 0, lse = -inf; k and v may be NULL).
 * scale must be finite and > 0 (the usual 1/sqrt(D)); the row maximum the kernel
 * subtracts for stability is taken on the unscaled logits.
 * in_dtype CPATTN_BF16: tensor-core kernel (tcgen05, TMEM accumulators, TMA-fed),
 *   D must be 64 or 128, fp32 accumulation and softmax; out_dtype BF16 (production)
 *   or F32 (same kernel, fp32 epilogue, for verification).
 * in_dtype CPATTN_F32: fp32 CUDA-core kernel, 1 <= D <= 256, out_dtype F32 or BF16.
 * Errors: CPATTN_ERR_NULL, _SHAPE, _ALIGN, _UNSUPPORTED (dtype/D combination),
 *   _CUDA.  A bounded wait that runs out inside the kernel is reported by
 *   cpattn_device_error(), not by this call (it returns before the kernel runs).
 */
CPATTN_API int cpattn_fwd(const void* q, const void* k, const void* v, void* out, float* lse,
               int B, int H, int Sq, int Skv, int D, float scale,
               int in_dtype, int out_dtype, cpattn_stream_t stream);

/*
 * cpattn_fwd_split -- cpattn_fwd (accumulate = 0) or cpattn_fwd_accumulate (accumulate = 1)
 * computed as n_split independent key ranges ("split-KV") whose partial (O, LSE) results
 * are then folded exactly by the merge formula of the Ring Attention step (Fig. 3) --
 * the online softmax makes partials over disjoint key sets combine losslessly.  It exists
 * for shapes with too few (query tile, head) work items to fill the GPU, e.g. one rank's
 * 5520-token query slice against a K/V chunk: 352 CTAs are 2.4 waves on 148 SMs, while
 * two key ranges give 704 CTAs.  Same arguments and results as the single-pass calls
 * (bf16 inputs, D in {64, 128}); with n_split = 1 it is exactly that call.
 * n_split = 0 is the tail split: work items (256 query rows x head x batch, one CTA each)
 * run over all keys, except the last, partial wave of them -- or that wave and the whole
 * wave before it -- whose items run as 2..8 key ranges each, as a makespan model of one CTA
 * per SM chooses (no split when none helps); their fp32 partials are folded afterwards.
 * n_split larger than the number of 128-key blocks is lowered to it.
 * workspace : caller-owned device buffer, 256-byte aligned, of at least
 *   cpattn_fwd_split_workspace(B, H, Sq, D, n_split, out_dtype) bytes; it receives the
 *   partials ([n_split][B][Sq][H][D] in out_dtype, then [n_split][B][H][Sq] float32; for
 *   n_split = 0, fp32 rows [parts][tail items][256][D], then their float32 LSEs).
 *   Concurrent calls must not share it.  May be NULL when no partials are needed.
 * Errors: as cpattn_fwd / cpattn_fwd_accumulate; CPATTN_ERR_SHAPE for n_split outside 0..8
 *   or a workspace that is too small; CPATTN_ERR_ALIGN for its alignment.
 */
CPATTN_API int cpattn_fwd_split(const void* q, const void* k, const void* v, void* out, float* lse,
                                int B, int H, int Sq, int Skv, int D, float scale, int out_dtype,
                                int accumulate, int n_split, void* workspace,
                                size_t workspace_bytes, cpattn_stream_t stream);

/* Workspace bytes cpattn_fwd_split needs (0 for n_split = 1 or invalid sizes).  For
 * n_split = 0 the plan also depends on the key count, which this query does not take: it
 * returns the largest workspace any key count can make the call need. */
CPATTN_API size_t cpattn_fwd_split_workspace(int B, int H, int Sq, int D, int n_split,
                                             int out_dtype);

/* Workspace bytes cpattn_fwd_split needs for this key count: exact, for every n_split
 * (after the call's lowering of n_split to the number of 128-key blocks); 0 when nothing
 * is split or the sizes are invalid. */
CPATTN_API size_t cpattn_fwd_split_workspace_kv(int B, int H, int Sq, int Skv, int D,
                                                int n_split, int out_dtype);

/*
 * cpattn_split_suggest -- split count (1..8) the library's wave model prefers for this
 * shape on the current device: 1 when the (query tile pair, head) grid already fills the
 * SMs for four or more waves.
 */
CPATTN_API int cpattn_split_suggest(int B, int H, int Sq, int Skv);

/*
 * cpattn_fwd_split_noalloc -- cpattn_fwd_split for callers that cannot allocate device
 * memory: code running inside a host runtime that owns all device memory and hands out no
 * workspace (an inference-engine plugin, for instance), or a latency-critical loop that
 * must not call cudaMalloc/cudaFree, which can synchronize the whole device.  The pages
 * have no counterpart to this call; it is a library convenience.
 * Same arguments and results as cpattn_fwd_split without the workspace arguments: the
 * partials go to a fixed scratch array compiled into the library,
 * cpattn_noalloc_scratch_bytes() = 64 MiB, which every GPU that loads the library holds
 * until the process exits.  The call itself allocates nothing: it makes no cudaMalloc,
 * cudaFree or other allocating call.
 * The first call on a device looks up that device's address of the array (with the device
 * current); make that first call before any stream capture.  Under CUDA's lazy module
 * loading (the default) that first call is also when the array's module is loaded, so it
 * may reserve the 64 MiB and synchronize the device: a caller that needs an
 * allocation-free loop makes one warm-up call first.
 * n_split is lowered exactly as cpattn_fwd_split lowers it (to the number of 128-key
 * blocks), and the size check uses the lowered count.
 * All calls on a device share the one array and it keeps the last call's contents (each
 * call writes every byte it reads first, so nothing needs clearing): calls that overlap on
 * the GPU -- on different streams, or from different threads -- race on it and must not
 * be issued.
 * Errors: as cpattn_fwd_split; CPATTN_ERR_SHAPE also when the partials need more than
 *   cpattn_noalloc_scratch_bytes() (cpattn_fwd_split_workspace_kv(B, H, Sq, Skv, D,
 *   n_split, out_dtype) tells), checked before anything is launched.
 */
CPATTN_API int cpattn_fwd_split_noalloc(const void* q, const void* k, const void* v, void* out,
                                        float* lse, int B, int H, int Sq, int Skv, int D,
                                        float scale, int out_dtype, int accumulate, int n_split,
                                        cpattn_stream_t stream);

/* Size in bytes of the fixed scratch behind cpattn_fwd_split_noalloc (64 MiB). */
CPATTN_API size_t cpattn_noalloc_scratch_bytes(void);

/*
 * cpattn_ulysses_fwd -- the whole DeepSpeed Ulysses attention of one layer in one kernel
 * (Fig. 4: all-to-all from sequence shards to head groups, full-sequence attention per head
 * group, all-to-all back), for P virtual ranks on one GPU.  The result equals
 *   cpattn_seq2head (Q, K, V) -> cpattn_fwd (B = P, H = H/P, S = P*S_local) -> cpattn_head2seq
 * but the re-partitions are done by the kernel's own addressing: every head is read over
 * the full sequence straight from the rank shards and O is written back to them.
 * q, k, v, out : [P][S_local][H][D] (q, k, v bf16; out BF16 or F32 per out_dtype).
 * lse : [P][H/P][P*S_local] float32 (head group, head within group, token), or NULL.
 * Requires H % P == 0, D in {64, 128}, S_local % 16 == 0 (the kernel reads 16-row boxes
 * that must not straddle two shards; CPATTN_ERR_UNSUPPORTED otherwise), 0 < scale.
 * Errors: CPATTN_ERR_NULL, _SHAPE, _ALIGN, _UNSUPPORTED, _CUDA.
 */
CPATTN_API int cpattn_ulysses_fwd(const void* q, const void* k, const void* v, void* out,
                                  float* lse, int P, int S_local, int H, int D, float scale,
                                  int out_dtype, cpattn_stream_t stream);

/*
 * cpattn_ulysses_fwd_split -- cpattn_ulysses_fwd with the tail split of cpattn_fwd_split
 * (n_split = 0): the work items (256 tokens x head, one CTA each; P * ceil(P*S_local/256) *
 * H/P of them) that fall in the last, partial wave of CTAs -- or in it and the whole wave
 * before -- run as 2..8 key ranges each, whose fp32 partials (O, LSE) are folded exactly
 * afterwards (the merge of the Ring Attention step, Fig. 3), so that the GPU's last wave is
 * short instead of partly idle.  Same arguments and result as cpattn_ulysses_fwd, to
 * rounding (each range subtracts its own row maximum before P is rounded to bf16, and the
 * fold runs in fp32), plus:
 * workspace : caller-owned device buffer, 256-byte aligned, of at least
 *   cpattn_ulysses_fwd_workspace(P, S_local, H, D, out_dtype) bytes (exact: the key count
 *   is the query's); NULL allowed when that is 0 (nothing to split: the call is then
 *   cpattn_ulysses_fwd).  It must not overlap q, k, v, out or lse.
 * Errors: as cpattn_ulysses_fwd; CPATTN_ERR_NULL / _ALIGN / _SHAPE for a missing,
 *   misaligned, too small or overlapping workspace.
 */
CPATTN_API int cpattn_ulysses_fwd_split(const void* q, const void* k, const void* v, void* out,
                                        float* lse, int P, int S_local, int H, int D,
                                        float scale, int out_dtype, void* workspace,
                                        size_t workspace_bytes, cpattn_stream_t stream);

/* Workspace bytes cpattn_ulysses_fwd_split needs (0: no split, or invalid sizes). */
CPATTN_API size_t cpattn_ulysses_fwd_workspace(int P, int S_local, int H, int D,
                                               int out_dtype);

/*
 * cpattn_ulysses_host -- cpattn_ulysses_fwd from host memory to host memory: one whole
 * Ulysses attention layer (Fig. 4) whose Q/K/V rank shards are in host memory and whose O
 * and LSE are wanted back in host memory, as in a host-driven inference loop (warm-up,
 * then timed iterations: the attention_mdtrt guide, section 推理程序运行机制).  The head
 * groups are processed in n_chunks chunks (chunk c = groups [c*P/n_chunks,
 * (c+1)*P/n_chunks)), pipelined so that the copies overlap the attention:
 *   upload stream:   Q, K, V heads of chunk c  host -> device  (one 2-D copy per tensor)
 *   compute streams: attention of chunk c      (the fused Ulysses kernel, chunk c only;
 *                    neighbouring chunks on two streams, so one chunk's last wave of work
 *                    overlaps the next chunk's first)
 *   download stream: O heads and LSE rows of chunk c  device -> host
 * ordered by events.  The result equals cpattn_ulysses_fwd on the same shards bit for bit.
 * h_q, h_k, h_v : [P][S_local][H][D] bf16 in host memory (page-locked, or the copies are
 *   not asynchronous); h_out : [P][S_local][H][D] out_dtype; h_lse : [P][H/P][P*S_local]
 *   float32, or NULL (then d_lse must be NULL too).
 * d_q, d_k, d_v, d_out, d_lse : caller-owned device buffers of the same shapes (the call
 *   allocates nothing), pairwise disjoint.
 * All work is ordered after the work already on `stream`, and `stream` waits for all of it
 * (the last copy to the host) before anything enqueued on it later; the call returns once
 * everything is enqueued.  Host outputs may be read, and host inputs reused, only after
 * `stream` has reached that point (cudaStreamSynchronize, or an event recorded on it).
 * The upload, download and second compute streams and four events per device are created
 * on the first call on that device and kept until the process exits; calls on one device
 * from several threads are enqueued one at a time.
 * n_chunks in 1..P (one chunk per head group, n_chunks = P, was fastest at P = 8); other
 * requirements and errors as cpattn_ulysses_fwd, plus CPATTN_ERR_SHAPE for n_chunks or
 * overlapping device buffers and CPATTN_ERR_NULL for a missing host pointer.
 */
CPATTN_API int cpattn_ulysses_host(const void* h_q, const void* h_k, const void* h_v,
                                   void* h_out, float* h_lse, void* d_q, void* d_k, void* d_v,
                                   void* d_out, float* d_lse, int P, int S_local, int H, int D,
                                   float scale, int out_dtype, int n_chunks,
                                   cpattn_stream_t stream);

/*
 * cpattn_fwd_accumulate -- one Ring Attention step with the merge fused into the attention
 * epilogue (环形注意力 / Ring Attention, Fig. 3: each rank folds every arriving K/V chunk
 * into its running result with the online softmax).  Computes the chunk's partial
 * (O_c, LSE_c) exactly as cpattn_fwd does and, instead of writing it out, merges it into
 * the running accumulator in place:
 *   L = max(L_acc, L_c) + ln(exp(L_acc - max) + exp(L_c - max))
 *   O_acc = exp(L_acc - L) * O_acc + exp(L_c - L) * O_c,   L_acc = L
 * Each accumulator row is read and rewritten by one thread, after the chunk is done.  A
 * row with L_acc = -inf is an empty accumulator: its o_acc row is not read (it may hold
 * anything, NaN included) and receives (O_c, L_c), so a ring step may start from an
 * uninitialised o_acc with lse_acc = -inf.
 * q : [B][Sq][H][D] bf16; k, v : [B][Skv][H][D] bf16 (the chunk); D in {64, 128}.
 * o_acc : [B][Sq][H][D] in acc_dtype (BF16 or F32), lse_acc : [B][H][Sq] float32, both
 * read and written.  Skv = 0 leaves the accumulator unchanged (nothing is launched).
 * Errors: CPATTN_ERR_NULL (lse_acc is required), _SHAPE, _ALIGN, _UNSUPPORTED (in_dtype
 * other than BF16, or D), _CUDA.
 */
CPATTN_API int cpattn_fwd_accumulate(const void* q, const void* k, const void* v, void* o_acc,
                                     float* lse_acc, int B, int H, int Sq, int Skv, int D,
                                     float scale, int in_dtype, int acc_dtype,
                                     cpattn_stream_t stream);

/*
 * cpattn_merge -- exact merge of two partial attention results over disjoint key sets
 * (the Ring Attention step: each rank folds each arriving K/V chunk's partial into its
 * running result with the online softmax, Fig. 3):
 *   L = max(La, Lb) + ln(exp(La - max) + exp(Lb - max))
 *   O = exp(La - L) * Oa + exp(Lb - L) * Ob
 * Two empty partials (La = Lb = -inf) give O = 0, L = -inf (never NaN).
 *
 * o_a, o_b, o : [B][S][H][D] in `dtype` (BF16 or F32); math in fp32.
 * lse_a, lse_b, lse : [B][H][S] float32.
 * o may alias o_a and lse may alias lse_a (in-place accumulate); no other overlap.
 * D must be a multiple of 8 (BF16) or 4 (F32) so rows move as 16-byte vectors, and a
 * row must fit in 4096 bytes (D <= 2048 BF16, 1024 F32); B*S*H < 2^31.
 * Errors: CPATTN_ERR_NULL, _SHAPE, _ALIGN, _UNSUPPORTED (dtype), _CUDA.
 */
CPATTN_API int cpattn_merge(const void* o_a, const float* lse_a, const void* o_b, const float* lse_b,
                 void* o, float* lse, int B, int H, int S, int D, int dtype,
                 cpattn_stream_t stream);

/*
 * cpattn_seq2head -- the DeepSpeed Ulysses first all-to-all (Fig. 4), run locally over
 * P virtual ranks: every rank's sequence shard becomes a full-sequence tensor of one
 * contiguous head group.  With Hp = H / P:
 *   dst[g][r*S_local + s][j][d] = src[r][s][g*Hp + j][d]
 * src : [P][S_local][H][D], dst : [P][P*S_local][Hp][D]; elements are copied as raw
 * `elem_bytes`-byte words (2 or 4), so the result is bit-exact.  dst is itself a
 * BSHD tensor with B = P, H = Hp, S = P*S_local, ready for cpattn_fwd.
 * Requires H % P == 0, Hp*D*elem_bytes a multiple of 16, src and dst not overlapping.
 * Errors: CPATTN_ERR_NULL, _SHAPE, _ALIGN, _CUDA.
 */
CPATTN_API int cpattn_seq2head(const void* src, void* dst, int P, int S_local, int H, int D,
                    int elem_bytes, cpattn_stream_t stream);

/*
 * cpattn_seq2head_qkv -- cpattn_seq2head of Q, K and V in one launch (the three
 * sequence->head all-to-alls that precede Ulysses attention, Fig. 4; the serving blog's
 * Cosmos 3 plan issues three all-to-alls per transformer layer).  Each of (q -> qh),
 * (k -> kh), (v -> vh) is exactly cpattn_seq2head with the same P, S_local, H, D and
 * elem_bytes; no destination may overlap any source or another destination.
 * Errors: as cpattn_seq2head.
 */
CPATTN_API int cpattn_seq2head_qkv(const void* q, const void* k, const void* v, void* qh, void* kh,
                                   void* vh, int P, int S_local, int H, int D, int elem_bytes,
                                   cpattn_stream_t stream);

/*
 * cpattn_rmsnorm -- the Q/K RMSNorm of the attention_mdtrt sample ("TensorRT 多设备注意力
 * 推理实战", section 模型的核心结构): after Q and K are split into heads, every head row
 * is normalised in fp32 as x * rsqrt(mean(x^2) + eps) (eps = 1e-6 there), multiplied by a
 * weight and cast back to 16 bits.  For each of `rows` head rows of D elements:
 *   r = 1 / sqrt(sum_d x[d]^2 / D + eps)                  (fp32: the hardware reciprocal
 *                                                           square-root estimate refined by
 *                                                           one Newton step, about an ulp of
 *                                                           the correctly rounded value)
 *   y[d] = bf16_rne(((x[d] * r) * gamma[d]) * out_scale)  (fp32 products)
 * `out_scale` is the sample's split scale sqrt(sqrt(1/D)) when the caller keeps Q and K
 * pre-scaled (then pass scale = 1 to cpattn_fwd); pass 1 to apply 1/sqrt(D) to the
 * logits through cpattn_fwd's `scale` instead (the same product in exact arithmetic).
 * x, y : [rows][D] bf16 (a [B][S][H][D] tensor is rows = B*S*H); y may be x itself (in
 * place) but must not overlap it otherwise.  gamma : D float32 weights in device memory,
 * caller-owned.  D a power of two in [8, 256]; rows >= 0 (rows = 0 is a no-op that reads
 * no pointer, so empty tensors may pass NULL); eps >= 0 and out_scale finite.  x, y, gamma 16-byte aligned.  The sum of squares is reduced in a
 * fixed order on the device, so y can differ from a float32 reference that sums in
 * another order by one bf16 unit in rare ties of the rounding.
 * Errors: CPATTN_ERR_NULL, _SHAPE, _ALIGN, _CUDA.
 */
CPATTN_API int cpattn_rmsnorm(const void* x, void* y, const float* gamma, int rows, int D,
                              float eps, float out_scale, cpattn_stream_t stream);

/*
 * cpattn_seq2head_qkv_norm -- cpattn_seq2head_qkv with the RMSNorm of cpattn_rmsnorm
 * applied to every Q head row (weights gamma_q) and K head row (gamma_k) while they are
 * copied; V is copied unchanged.  The norm acts on whole head rows and the permute moves
 * whole head rows, so qh = seq2head(rmsnorm(q)) bit for bit as the two separate calls
 * give it, at the bytes of the plain permute.  bf16 only (elem_bytes 2); D a power of
 * two in [8, 256]; other requirements as cpattn_seq2head_qkv and cpattn_rmsnorm.
 * Errors: CPATTN_ERR_NULL, _SHAPE, _ALIGN, _CUDA.
 */
CPATTN_API int cpattn_seq2head_qkv_norm(const void* q, const void* k, const void* v, void* qh,
                                        void* kh, void* vh, const float* gamma_q,
                                        const float* gamma_k, int P, int S_local, int H, int D,
                                        float eps, float out_scale, cpattn_stream_t stream);

/*
 * cpattn_head2seq -- the Ulysses second all-to-all (Fig. 4), exact inverse of
 * cpattn_seq2head:
 *   dst[r][s][g*Hp + j][d] = src[g][r*S_local + s][j][d]
 * src : [P][P*S_local][Hp][D] with Hp = H / P, dst : [P][S_local][H][D].
 * Same requirements and errors as cpattn_seq2head.
 */
CPATTN_API int cpattn_head2seq(const void* src, void* dst, int P, int S_local, int H, int D,
                    int elem_bytes, cpattn_stream_t stream);

/* Human-readable name of a cpattn_status value (static string, never NULL). */
CPATTN_API const char* cpattn_status_str(int status);

/*
 * cpattn_device_error -- synchronizes the current device, then reads and clears its
 * device error word.  Returns CPATTN_OK, or CPATTN_ERR_DEVICE_TIMEOUT if a kernel's
 * bounded wait (mbarrier / pipeline) ran out since the last call, or CPATTN_ERR_CUDA
 * if the synchronization itself failed.
 */
CPATTN_API int cpattn_device_error(void);

/*
 * cpattn_selftest_wait_timeout -- launches one CTA that waits on a pipeline barrier
 * nothing will ever complete, through the same bounded-wait routine the attention
 * kernel uses, with a limit of `limit_cycles` SM clock cycles (1 .. 2^31).  The wait
 * runs out, the kernel records the timeout in the device error word and returns, so
 * cpattn_device_error() must then report CPATTN_ERR_DEVICE_TIMEOUT.  Used by tests to
 * show a stalled pipeline ends in an error status instead of a hang.
 * Errors: CPATTN_ERR_SHAPE (limit out of range), _CUDA.
 */
CPATTN_API int cpattn_selftest_wait_timeout(long long limit_cycles, cpattn_stream_t stream);

/*
 * cpattn_selftest_exp2 -- evaluates, on the device, the polynomial 2^t the attention
 * kernel uses for a fixed share of its softmax exponentials (Cody-Waite range reduction
 * t = n + f, |f| <= 1/2, then a degree-3 polynomial with constant term exactly 1, fitted
 * by csrc/gen_exp2_poly.py; relative error <= 1.02e-4 for -125 <= t <= 8; t below -125
 * returns 2^-125).  t, out: n device floats.  For tests against the error bound.
 * Errors: CPATTN_ERR_SHAPE (n < 1), _NULL, _ALIGN, _CUDA.
 */
CPATTN_API int cpattn_selftest_exp2(const float* t, float* out, int n, cpattn_stream_t stream);

/* ABI version: (major << 16) | minor. */
CPATTN_API int cpattn_version(void);

#ifdef __cplusplus
}
#endif

#endif /* CPATTN_H */
