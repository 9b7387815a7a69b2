"""fp64 NumPy oracle for the per-rank context-parallel attention path (test infrastructure).

Layout reading (the pages reshape activations to (seq, batch, heads, dim) in the
attention_mdtrt guide, section 模型的核心结构; the Ulysses per-rank shard is a block of
tokens with all heads): Q, K, V, O are ``[B][S][H][D]`` (token-major, heads
interleaved), LSE is ``[B][H][Sq]``.

Everything is computed in float64 from the exact upcast of the caller's arrays (the
caller rounds to bf16 first when the kernel under test sees bf16).  There is no
blocking, fusion or reordering of the per-row arithmetic: query rows are independent,
and they are visited in row blocks only to bound memory.
"""

from __future__ import annotations

import os

import numpy as np

try:  # BLAS thread control; absent threadpoolctl simply leaves the default
    from threadpoolctl import threadpool_limits as _threadpool_limits
except Exception:  # pragma: no cover
    _threadpool_limits = None

_THREADS = None
_LIMITER = None


def set_threads(n: int | None = None) -> int:
    """Pin the BLAS thread count used by the oracle (default: all usable cores)."""
    global _THREADS, _LIMITER
    if n is None:
        n = len(os.sched_getaffinity(0))
    _THREADS = int(n)
    if _threadpool_limits is not None:
        _LIMITER = _threadpool_limits(limits=_THREADS, user_api="blas")
    return _THREADS


def threads() -> int:
    """BLAS threads the oracle runs with (set_threads() value, else usable cores)."""
    return _THREADS if _THREADS is not None else len(os.sched_getaffinity(0))


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # a torch tensor: exact upcast through float32/float64
        import torch

        t = x.detach().cpu()
        if t.dtype not in (torch.float32, torch.float64):
            t = t.to(torch.float32)  # bf16 -> f32 is exact
        x = t.numpy()
    return np.asarray(x, dtype=np.float64)


def _attention_head(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float):
    """One head: q [Sq][D], k [Skv][D], v [Skv][D] -> (o [Sq][D], lse [Sq]).

    Definition (Ring Attention / AllGather KV sections of the TensorRT multi-device
    blog; the softmax(QK^T)V core of the attention_mdtrt guide, 模型的核心结构):
        s_ij   = scale * sum_d q_id k_jd
        lse_i  = ln sum_j exp(s_ij)        (written as m_i + ln sum_j exp(s_ij - m_i),
                                            m_i = max_j s_ij, the usual stable form)
        o_i    = sum_j exp(s_ij - lse_i) v_j
    Non-causal: no mask.  Skv = 0 gives o = 0, lse = -inf (empty key set).
    """
    sq, d = q.shape
    skv = k.shape[0]
    if skv == 0:
        return np.zeros((sq, v.shape[1])), np.full(sq, -np.inf)
    o = np.empty((sq, v.shape[1]))
    lse = np.empty(sq)
    # row blocks sized so the score block stays near 64 MB of float64
    rows = max(1, min(sq, (8 << 20) // max(skv, 1)))
    for r0 in range(0, sq, rows):
        r1 = min(sq, r0 + rows)
        s = scale * (q[r0:r1] @ k.T)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        l = e.sum(axis=1, keepdims=True)
        lse[r0:r1] = (m + np.log(l))[:, 0]
        o[r0:r1] = (e @ v) / l
    return o, lse


def attention(q, k, v, scale: float):
    """Non-causal attention over ``[B][S][H][D]`` tensors.

    Returns ``(O [B][Sq][H][D] float64, LSE [B][H][Sq] float64)``.  LSE is the natural
    log of the sum of exponentials of the *scaled* logits (reading: the pages name the
    online softmax but print no formula; the natural-log convention makes the merge
    formula below exact).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    b_, sq, h_, d = q.shape
    skv = k.shape[1]
    assert k.shape == (b_, skv, h_, d) and v.shape[:3] == (b_, skv, h_)
    o = np.empty((b_, sq, h_, v.shape[3]))
    lse = np.empty((b_, h_, sq))
    for b in range(b_):
        for h in range(h_):
            o[b, :, h, :], lse[b, h, :] = _attention_head(
                q[b, :, h, :], k[b, :, h, :], v[b, :, h, :], scale
            )
    return o, lse


def attention_rows(q, k, v, scale: float, rows):
    """The same definition evaluated only at the listed query rows.

    ``rows`` is a sequence of ``(b, h, i)``.  Returns ``(O [n][D], LSE [n])`` in that
    order.  Used to check full-size GPU results on sampled outputs: each sampled row is
    exact, so sampling loses nothing per row.
    """
    rows = [tuple(int(t) for t in r) for r in rows]
    groups: dict[tuple[int, int], list[int]] = {}
    for n, (b, h, i) in enumerate(rows):
        groups.setdefault((b, h), []).append(n)
    dv = v.shape[3]
    o = np.empty((len(rows), dv))
    lse = np.empty(len(rows))
    for (b, h), idx in groups.items():
        qi = _f64(q[b, [rows[n][2] for n in idx], h, :])
        kh = _f64(k[b, :, h, :])
        vh = _f64(v[b, :, h, :])
        oo, ll = _attention_head(qi, kh, vh, scale)
        o[idx] = oo
        lse[idx] = ll
    return o, lse


def merge(o_a, lse_a, o_b, lse_b):
    """Exact merge of two partial attention results over disjoint key sets.

    Ring Attention (TensorRT multi-device blog, 环形注意力, Fig. 3) lets each rank keep
    its Q while K/V chunks travel round the ring and folds each chunk's result in with
    the online softmax.  For normalised partials (O_a, L_a), (O_b, L_b):
        L = max(L_a, L_b) + ln(exp(L_a - max) + exp(L_b - max))
        O = exp(L_a - L) O_a + exp(L_b - L) O_b
    Two empty partials (L = -inf on both sides) give O = 0, L = -inf.
    ``o_*`` are ``[B][S][H][D]``, ``lse_*`` are ``[B][H][S]``.
    """
    o_a, o_b = _f64(o_a), _f64(o_b)
    la, lb = _f64(lse_a), _f64(lse_b)
    mx = np.maximum(la, lb)
    both_empty = np.isneginf(la) & np.isneginf(lb)
    mx_safe = np.where(both_empty, 0.0, mx)
    ea = np.exp(la - mx_safe)
    eb = np.exp(lb - mx_safe)
    tot = ea + eb
    with np.errstate(divide="ignore"):
        lse = np.where(both_empty, -np.inf, mx_safe + np.log(np.where(both_empty, 1.0, tot)))
    wa = np.where(both_empty, 0.0, ea / np.where(both_empty, 1.0, tot))
    wb = np.where(both_empty, 0.0, eb / np.where(both_empty, 1.0, tot))
    # weights are [B][H][S]; O is [B][S][H][D]
    wa_o = np.transpose(wa, (0, 2, 1))[..., None]
    wb_o = np.transpose(wb, (0, 2, 1))[..., None]
    return wa_o * o_a + wb_o * o_b, lse


def merge_chunks(parts):
    """Left fold of ``merge`` over ``[(O_0, L_0), (O_1, L_1), ...]`` in ring order."""
    parts = list(parts)
    o, lse = _f64(parts[0][0]), _f64(parts[0][1])
    for o_c, l_c in parts[1:]:
        o, lse = merge(o, lse, o_c, l_c)
    return o, lse


def ring_attention(q, k_chunks, v_chunks, scale: float):
    """One rank's Ring Attention: attention against each K/V chunk, merged in order."""
    parts = [attention(q, kc, vc, scale) for kc, vc in zip(k_chunks, v_chunks)]
    return merge_chunks(parts)


def seq2head(src, p: int) -> np.ndarray:
    """Ulysses first all-to-all, run locally over ``p`` virtual ranks.

    DeepSpeed Ulysses section of the TensorRT multi-device blog (Fig. 4): before
    attention an all-to-all turns the sequence-sharded Q/K/V into full-sequence tensors
    holding a non-overlapping subset of heads on each rank.  Reading: head group g holds
    the contiguous heads [g*H/P, (g+1)*H/P); the full sequence is the rank shards
    concatenated in rank order.  With Hp = H/P:
        dst[g][r*S_l + s][j][d] = src[r][s][g*Hp + j][d]
    ``src`` is ``[P][S_l][H][D]``; the result is ``[P][P*S_l][Hp][D]`` (any dtype,
    values copied unchanged).
    """
    src = np.asarray(src)
    pp, s_l, h, d = src.shape
    assert pp == p and h % p == 0
    hp = h // p
    # axes of the view: (r, s, g, j, d) -> (g, r, s, j, d)
    return np.ascontiguousarray(
        src.reshape(p, s_l, p, hp, d).transpose(2, 0, 1, 3, 4).reshape(p, p * s_l, hp, d)
    )


def head2seq(src, p: int) -> np.ndarray:
    """Ulysses second all-to-all (the exact inverse of ``seq2head``).

    After attention the head-group results go back to sequence shards (DeepSpeed
    Ulysses section, Fig. 4):
        dst[r][s][g*Hp + j][d] = src[g][r*S_l + s][j][d]
    ``src`` is ``[P][P*S_l][Hp][D]``; the result is ``[P][S_l][P*Hp][D]``.
    """
    src = np.asarray(src)
    pp, s_full, hp, d = src.shape
    assert pp == p and s_full % p == 0
    s_l = s_full // p
    # axes of the view: (g, r, s, j, d) -> (r, s, g, j, d)
    return np.ascontiguousarray(
        src.reshape(p, p, s_l, hp, d).transpose(1, 2, 0, 3, 4).reshape(p, s_l, p * hp, d)
    )


def ulysses_attention(q_shards, k_shards, v_shards, p: int, scale: float):
    """Per-rank Ulysses path over P virtual ranks: seq2head x3, attention, head2seq.

    Inputs are ``[P][S_l][H][D]``.  The head-grouped buffers ``[P][P*S_l][H/P][D]`` are
    themselves BSHD tensors with B = P, so one attention call covers every group.
    Returns ``(O [P][S_l][H][D], LSE [P][H/P][P*S_l])``.
    """
    qh, kh, vh = (seq2head(_f64(x), p) for x in (q_shards, k_shards, v_shards))
    o, lse = attention(qh, kh, vh, scale)
    return head2seq(o, p), lse



def rmsnorm_heads(x, gamma, eps: float = 1e-6, out_scale: float = 1.0) -> np.ndarray:
    """RMSNorm of every head row of Q or K, as the attention_mdtrt sample applies it.

    "TensorRT 多设备注意力推理实战" (guide to the attention_mdtrt sample), section
    模型的核心结构: after Q and K are reshaped to heads (seq, batch, 32, 128), each is
    normalised in fp32 as x * rsqrt(mean(x^2) + eps) with eps = 1e-6, multiplied by a
    weight, and cast back to a 16-bit type; Q and K are then each scaled by
    sqrt(sqrt(1/HEAD_DIM)) before QK^T.

    Readings: the mean runs over the last axis (the head dimension D); one weight vector
    ``gamma[D]`` serves every head and token; the arithmetic is float32 because the page
    fixes it (x*r first, then *gamma, then *out_scale, each rounded to float32);
    ``out_scale`` is the optional split scale applied before the cast (1 when the scale
    is applied to the logits instead, as 1/sqrt(D)).  Returns float32 values *before*
    the cast to 16 bits; the caller rounds (bf16 round-to-nearest-even here, where the
    sample uses fp16).  ``x`` is ``[..., D]``.
    """
    x32 = np.asarray(_f64(x), dtype=np.float32)  # exact for bf16/fp32 inputs
    g32 = np.asarray(_f64(gamma), dtype=np.float32)
    assert g32.shape == (x32.shape[-1],)
    ms = np.mean(np.square(x32), axis=-1, dtype=np.float32, keepdims=True)
    r = np.float32(1.0) / np.sqrt(ms + np.float32(eps))
    y = (x32 * r) * g32
    if out_scale != 1.0:
        y = y * np.float32(out_scale)
    return y.astype(np.float32)
