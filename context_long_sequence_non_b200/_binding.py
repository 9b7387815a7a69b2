"""ctypes binding of libcpattn.so (include/cpattn.h).  Argument marshalling only: every
step of the path runs in the library's CUDA kernels.  PyTorch provides device memory and
the current stream; nothing here computes on the host.  There is no fallback: if the
library is missing or a call fails, an exception is raised.
"""

from __future__ import annotations

import ctypes
import math
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libcpattn.so")

BF16, F32 = 0, 1
OK, ERR_NULL, ERR_SHAPE, ERR_ALIGN, ERR_UNSUPPORTED, ERR_CUDA, ERR_DEVICE_TIMEOUT = range(7)

_lock = threading.Lock()
_lib = None


class CpattnError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {status_str(status)}")


def library_path() -> str:
    return LIB_PATH


def lib() -> ctypes.CDLL:
    """Load libcpattn.so (once).  Raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(
                    f"{LIB_PATH} is missing: build it with "
                    "`python -m context_long_sequence_non_b200.build` (no CPU fallback exists)")
            L = ctypes.CDLL(LIB_PATH)
            vp, i, f, ll = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_longlong
            L.cpattn_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp]
            L.cpattn_fwd_accumulate.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp]
            L.cpattn_ulysses_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp]
            L.cpattn_ulysses_fwd_split.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, f, i, vp,
                                                   ctypes.c_size_t, vp]
            L.cpattn_ulysses_fwd_workspace.argtypes = [i, i, i, i, i]
            L.cpattn_ulysses_fwd_workspace.restype = ctypes.c_size_t
            L.cpattn_ulysses_host.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i,
                                              f, i, i, vp]
            L.cpattn_fwd_split.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, i, vp,
                                           ctypes.c_size_t, vp]
            L.cpattn_fwd_split_workspace.argtypes = [i, i, i, i, i, i]
            L.cpattn_fwd_split_workspace.restype = ctypes.c_size_t
            L.cpattn_fwd_split_workspace_kv.argtypes = [i, i, i, i, i, i, i]
            L.cpattn_fwd_split_workspace_kv.restype = ctypes.c_size_t
            L.cpattn_split_suggest.argtypes = [i, i, i, i]
            L.cpattn_merge.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp]
            L.cpattn_seq2head.argtypes = [vp, vp, i, i, i, i, i, vp]
            L.cpattn_head2seq.argtypes = [vp, vp, i, i, i, i, i, vp]
            L.cpattn_seq2head_qkv.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, vp]
            L.cpattn_rmsnorm.argtypes = [vp, vp, vp, i, i, f, f, vp]
            L.cpattn_seq2head_qkv_norm.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, f,
                                                   f, vp]
            L.cpattn_status_str.argtypes = [i]
            L.cpattn_status_str.restype = ctypes.c_char_p
            L.cpattn_device_error.argtypes = []
            L.cpattn_selftest_wait_timeout.argtypes = [ll, vp]
            L.cpattn_version.argtypes = []
            L.cpattn_selftest_exp2.argtypes = [vp, vp, i, vp]
            for name in ("cpattn_fwd", "cpattn_fwd_accumulate", "cpattn_ulysses_fwd",
                         "cpattn_ulysses_fwd_split", "cpattn_ulysses_host",
                         "cpattn_fwd_split", "cpattn_split_suggest", "cpattn_merge", "cpattn_seq2head_qkv", "cpattn_seq2head", "cpattn_head2seq",
                         "cpattn_device_error", "cpattn_selftest_wait_timeout", "cpattn_version",
                         "cpattn_selftest_exp2"):
                getattr(L, name).restype = ctypes.c_int
            _lib = L
    return _lib


def status_str(status: int) -> str:
    return lib().cpattn_status_str(int(status)).decode()


def _check(status: int, what: str):
    if status != OK:
        raise CpattnError(status, what)


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return BF16
    if t == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need_cuda(*ts):
    for t in ts:
        if t is not None:
            if not t.is_cuda:
                raise ValueError("tensors must live on a CUDA device")
            if not t.is_contiguous():
                raise ValueError("tensors must be contiguous")


def _need_shape(t, shape, name, dtype=None):
    """A caller-provided output must have exactly the size the call writes: the library
    receives only its pointer."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, not {tuple(t.shape)}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, not {t.dtype}")


def _nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


def fwd(q, k, v, out=None, lse=None, scale=None, out_dtype=None, want_lse=True, stream=None):
    """Non-causal attention ``softmax(scale * Q K^T) V`` with its log-sum-exp.

    q: [B][Sq][H][D], k/v: [B][Skv][H][D] (bf16 -> tcgen05 kernel, fp32 -> CUDA-core
    kernel).  Returns ``(out [B][Sq][H][D], lse [B][H][Sq] float32)``.
    """
    B, Sq, H, D = q.shape
    Skv = k.shape[1]
    if k.shape != (B, Skv, H, D) or v.shape != (B, Skv, H, D):
        raise ValueError("k and v must be [B][Skv][H][D] matching q")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out_dtype is None:
        out_dtype = q.dtype
    if out is None:
        out = torch.empty((B, Sq, H, D), dtype=out_dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((B, H, Sq), dtype=torch.float32, device=q.device)
    _need_shape(out, (B, Sq, H, D), "out")
    _need_shape(lse, (B, H, Sq), "lse", torch.float32)
    _need_cuda(q, k, v, out, lse)
    st = lib().cpattn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Sq, Skv, D,
                          float(scale), _dtype_code(q.dtype), _dtype_code(out.dtype),
                          _stream(stream))
    _check(st, "cpattn_fwd")
    return out, lse


def ulysses_fwd(q, k, v, P, out=None, lse=None, scale=None, out_dtype=None, want_lse=True,
                stream=None):
    """Ulysses attention in one kernel: q/k/v/out are [P][S_l][H][D] rank shards; returns
    ``(out, lse [P][H/P][P*S_l])`` equal to seq2head -> fwd -> head2seq."""
    P_, S_l, H, D = q.shape
    if P_ != P or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must be same-shaped [P][S_l][H][D] shards")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty((P, S_l, H, D), dtype=out_dtype or q.dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((P, H // P, P * S_l), dtype=torch.float32, device=q.device)
    _need_shape(out, (P, S_l, H, D), "out")
    _need_shape(lse, (P, H // P, P * S_l), "lse", torch.float32)
    _need_cuda(q, k, v, out, lse)
    st = lib().cpattn_ulysses_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), P, S_l, H, D,
                                  float(scale), _dtype_code(out.dtype), _stream(stream))
    _check(st, "cpattn_ulysses_fwd")
    return out, lse


def ulysses_workspace_bytes(P, S_l, H, D, out_dtype=torch.bfloat16) -> int:
    """Workspace bytes of ulysses_fwd_split for these shards (0: nothing to split)."""
    return int(lib().cpattn_ulysses_fwd_workspace(P, S_l, H, D, _dtype_code(out_dtype)))


def ulysses_fwd_split(q, k, v, P, out=None, lse=None, scale=None, out_dtype=None,
                      want_lse=True, workspace=None, stream=None):
    """ulysses_fwd with the tail split (the items of the GPU's last wave or two computed
    as key ranges and folded exactly).  ``workspace``: a uint8 CUDA tensor of at least
    ``ulysses_workspace_bytes(...)`` bytes, allocated here (by PyTorch) when omitted."""
    P_, S_l, H, D = q.shape
    if P_ != P or k.shape != q.shape or v.shape != q.shape:
        raise ValueError("q, k, v must be same-shaped [P][S_l][H][D] shards")
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty((P, S_l, H, D), dtype=out_dtype or q.dtype, device=q.device)
    if lse is None and want_lse:
        lse = torch.empty((P, H // P, P * S_l), dtype=torch.float32, device=q.device)
    _need_shape(out, (P, S_l, H, D), "out")
    _need_shape(lse, (P, H // P, P * S_l), "lse", torch.float32)
    need = ulysses_workspace_bytes(P, S_l, H, D, out.dtype)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _need_cuda(q, k, v, out, lse, workspace)
    st = lib().cpattn_ulysses_fwd_split(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), P, S_l,
                                        H, D, float(scale), _dtype_code(out.dtype),
                                        _ptr(workspace), _nbytes(workspace), _stream(stream))
    _check(st, "cpattn_ulysses_fwd_split")
    return out, lse


def ulysses_host(hq, hk, hv, h_out, h_lse, dq, dk, dv, d_out, d_lse, P, scale=None,
                 n_chunks=None, stream=None):
    """Ulysses attention from host shards to host O/LSE through cpattn_ulysses_host: the
    copies are pipelined with the attention over head-group chunks.  h_*: CPU tensors
    (pinned for asynchronous copies); d_*: same-shaped CUDA work buffers.  The host
    outputs are valid once ``stream`` (default: the current stream) has passed the call."""
    P_, S_l, H, D = hq.shape
    for t in (hk, hv, dq, dk, dv):
        if t.shape != hq.shape:
            raise ValueError("all shard tensors must be [P][S_l][H][D]")
    if h_out.shape != hq.shape or d_out.shape != hq.shape or h_out.dtype != d_out.dtype:
        raise ValueError("h_out and d_out must be [P][S_l][H][D] of one dtype")
    if (h_lse is None) != (d_lse is None):
        raise ValueError("h_lse and d_lse go together")
    for t in (hq, hk, hv, h_out, h_lse):
        if t is not None and (t.is_cuda or not t.is_contiguous()):
            raise ValueError("host tensors must be contiguous CPU tensors")
    _need_cuda(dq, dk, dv, d_out, d_lse)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if n_chunks is None:
        n_chunks = P
    st = lib().cpattn_ulysses_host(_ptr(hq), _ptr(hk), _ptr(hv), _ptr(h_out), _ptr(h_lse),
                                   _ptr(dq), _ptr(dk), _ptr(dv), _ptr(d_out), _ptr(d_lse), P,
                                   S_l, H, D, float(scale), _dtype_code(d_out.dtype),
                                   int(n_chunks), _stream(stream))
    _check(st, "cpattn_ulysses_host")
    return h_out, h_lse


def split_workspace_bytes(B, H, Sq, D, n_split, out_dtype=torch.bfloat16, Skv=None) -> int:
    """Workspace bytes of fwd_split: exact for the key count ``Skv`` when given, else (for
    the tail split, n_split = 0) the largest any key count can need."""
    if Skv is not None:
        return int(lib().cpattn_fwd_split_workspace_kv(B, H, Sq, Skv, D, n_split,
                                                       _dtype_code(out_dtype)))
    return int(lib().cpattn_fwd_split_workspace(B, H, Sq, D, n_split, _dtype_code(out_dtype)))


def split_suggest(B, H, Sq, Skv) -> int:
    return int(lib().cpattn_split_suggest(B, H, Sq, Skv))


def fwd_split(q, k, v, out=None, lse=None, scale=None, out_dtype=None, accumulate=False,
              n_split=None, workspace=None, stream=None):
    """Split-KV attention: ``n_split`` key ranges computed as separate CTAs, their partials
    folded exactly (into the running (out, lse) when ``accumulate``).  ``workspace`` is a
    uint8 CUDA tensor of at least ``split_workspace_bytes(...)`` bytes (allocated here when
    omitted -- by PyTorch; the library allocates nothing)."""
    B_, Sq, H, D = q.shape
    Skv = k.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    if out is None:
        out = torch.empty((B_, Sq, H, D), dtype=out_dtype or q.dtype, device=q.device)
    if lse is None:
        lse = torch.empty((B_, H, Sq), dtype=torch.float32, device=q.device)
    if k.shape != (B_, Skv, H, D) or v.shape != (B_, Skv, H, D):
        raise ValueError("k and v must be [B][Skv][H][D] matching q")
    _need_shape(out, (B_, Sq, H, D), "out")
    _need_shape(lse, (B_, H, Sq), "lse", torch.float32)
    if n_split is None:
        n_split = split_suggest(B_, H, Sq, Skv)
    need = split_workspace_bytes(B_, H, Sq, D, n_split, out.dtype, Skv=Skv)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    _need_cuda(q, k, v, out, lse, workspace)
    st = lib().cpattn_fwd_split(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B_, H, Sq, Skv,
                                D, float(scale), _dtype_code(out.dtype), 1 if accumulate else 0,
                                int(n_split), _ptr(workspace), _nbytes(workspace),
                                _stream(stream))
    _check(st, "cpattn_fwd_split")
    return out, lse


def fwd_accumulate(q, k, v, o_acc, lse_acc, scale=None, stream=None):
    """Ring Attention step with the merge fused into the attention epilogue: attention of
    q over this K/V chunk, merged in place into the running (o_acc, lse_acc)."""
    B, Sq, H, D = q.shape
    Skv = k.shape[1]
    if k.shape != (B, Skv, H, D) or v.shape != (B, Skv, H, D):
        raise ValueError("k and v must be [B][Skv][H][D] matching q")
    if o_acc.shape != (B, Sq, H, D) or lse_acc.shape != (B, H, Sq):
        raise ValueError("o_acc must be [B][Sq][H][D] and lse_acc [B][H][Sq]")
    _need_shape(lse_acc, (B, H, Sq), "lse_acc", torch.float32)
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    _need_cuda(q, k, v, o_acc, lse_acc)
    st = lib().cpattn_fwd_accumulate(_ptr(q), _ptr(k), _ptr(v), _ptr(o_acc), _ptr(lse_acc), B, H,
                                     Sq, Skv, D, float(scale), _dtype_code(q.dtype),
                                     _dtype_code(o_acc.dtype), _stream(stream))
    _check(st, "cpattn_fwd_accumulate")
    return o_acc, lse_acc


def merge(o_a, lse_a, o_b, lse_b, out=None, lse=None, stream=None):
    """Exact merge of two partial (O, LSE) results; ``out``/``lse`` may be o_a/lse_a."""
    B, S, H, D = o_a.shape
    if out is None:
        out = torch.empty_like(o_a)
    if lse is None:
        lse = torch.empty_like(lse_a)
    _need_shape(o_b, (B, S, H, D), "o_b", o_a.dtype)
    _need_shape(out, (B, S, H, D), "out", o_a.dtype)
    for name, t in (("lse_a", lse_a), ("lse_b", lse_b), ("lse", lse)):
        _need_shape(t, (B, H, S), name, torch.float32)
    _need_cuda(o_a, lse_a, o_b, lse_b, out, lse)
    st = lib().cpattn_merge(_ptr(o_a), _ptr(lse_a), _ptr(o_b), _ptr(lse_b), _ptr(out), _ptr(lse),
                            B, H, S, D, _dtype_code(o_a.dtype), _stream(stream))
    _check(st, "cpattn_merge")
    return out, lse


def seq2head(src, P, out=None, stream=None):
    """[P][S_l][H][D] sequence shards -> [P][P*S_l][H/P][D] head groups (bit copy)."""
    P_, S_l, H, D = src.shape
    if P_ != P:
        raise ValueError("src.shape[0] must equal P")
    if out is None:
        out = torch.empty((P, P * S_l, H // P, D), dtype=src.dtype, device=src.device)
    _need_shape(out, (P, P * S_l, H // P, D), "out", src.dtype)
    _need_cuda(src, out)
    st = lib().cpattn_seq2head(_ptr(src), _ptr(out), P, S_l, H, D, src.element_size(),
                               _stream(stream))
    _check(st, "cpattn_seq2head")
    return out


def seq2head_qkv(q, k, v, P, out=None, stream=None):
    """seq2head of Q, K and V in one launch; ``out`` is an optional (qh, kh, vh) triple."""
    P_, S_l, H, D = q.shape
    if P_ != P or k.shape != q.shape or v.shape != q.shape or k.dtype != q.dtype or v.dtype != q.dtype:
        raise ValueError("q, k, v must be same-shaped [P][S_l][H][D] tensors")
    if out is None:
        out = tuple(torch.empty((P, P * S_l, H // P, D), dtype=q.dtype, device=q.device)
                    for _ in range(3))
    for i, t in enumerate(out):
        _need_shape(t, (P, P * S_l, H // P, D), f"out[{i}]", q.dtype)
    _need_cuda(q, k, v, *out)
    st = lib().cpattn_seq2head_qkv(_ptr(q), _ptr(k), _ptr(v), *(_ptr(t) for t in out), P, S_l, H,
                                   D, q.element_size(), _stream(stream))
    _check(st, "cpattn_seq2head_qkv")
    return out


def rmsnorm(x, gamma, eps=1e-6, out_scale=1.0, out=None, stream=None):
    """RMSNorm of every head row (last axis, D) of a bf16 tensor with fp32 weights
    ``gamma[D]``; ``out=x`` normalises in place.  See cpattn_rmsnorm."""
    if x.dtype != torch.bfloat16 or gamma.dtype != torch.float32 or gamma.shape != (x.shape[-1],):
        raise ValueError("x must be bf16 [..., D] and gamma float32 [D]")
    if out is None:
        out = torch.empty_like(x)
    if out.shape != x.shape or out.dtype != x.dtype:
        raise ValueError("out must match x")
    _need_cuda(x, gamma, out)
    D = x.shape[-1]
    st = lib().cpattn_rmsnorm(_ptr(x), _ptr(out), _ptr(gamma), x.numel() // D, D, float(eps),
                              float(out_scale), _stream(stream))
    _check(st, "cpattn_rmsnorm")
    return out


def seq2head_qkv_norm(q, k, v, P, gamma_q, gamma_k, eps=1e-6, out_scale=1.0, out=None,
                      stream=None):
    """seq2head of Q, K, V in one launch with Q and K head rows RMS-normalised on the way
    (weights gamma_q / gamma_k, float32 [D]); ``out`` is an optional (qh, kh, vh) triple."""
    P_, S_l, H, D = q.shape
    if P_ != P or k.shape != q.shape or v.shape != q.shape or any(
            t.dtype != torch.bfloat16 for t in (q, k, v)):
        raise ValueError("q, k, v must be same-shaped bf16 [P][S_l][H][D] tensors")
    for g in (gamma_q, gamma_k):
        if g.dtype != torch.float32 or g.shape != (D,):
            raise ValueError("gamma_q and gamma_k must be float32 [D]")
    if out is None:
        out = tuple(torch.empty((P, P * S_l, H // P, D), dtype=q.dtype, device=q.device)
                    for _ in range(3))
    for i, t in enumerate(out):
        _need_shape(t, (P, P * S_l, H // P, D), f"out[{i}]", q.dtype)
    _need_cuda(q, k, v, gamma_q, gamma_k, *out)
    st = lib().cpattn_seq2head_qkv_norm(_ptr(q), _ptr(k), _ptr(v), *(_ptr(t) for t in out),
                                        _ptr(gamma_q), _ptr(gamma_k), P, S_l, H, D, float(eps),
                                        float(out_scale), _stream(stream))
    _check(st, "cpattn_seq2head_qkv_norm")
    return out


def head2seq(src, P, out=None, stream=None):
    """[P][P*S_l][Hp][D] head groups -> [P][S_l][P*Hp][D] sequence shards (bit copy)."""
    P_, S_full, Hp, D = src.shape
    if P_ != P or S_full % P:
        raise ValueError("src must be [P][P*S_l][Hp][D]")
    S_l, H = S_full // P, Hp * P
    if out is None:
        out = torch.empty((P, S_l, H, D), dtype=src.dtype, device=src.device)
    _need_shape(out, (P, S_l, H, D), "out", src.dtype)
    _need_cuda(src, out)
    st = lib().cpattn_head2seq(_ptr(src), _ptr(out), P, S_l, H, D, src.element_size(),
                               _stream(stream))
    _check(st, "cpattn_head2seq")
    return out


def device_error() -> int:
    """Synchronize and read/clear the device error word (OK or ERR_DEVICE_TIMEOUT)."""
    return lib().cpattn_device_error()


def selftest_wait_timeout(limit_cycles: int, stream=None):
    _check(lib().cpattn_selftest_wait_timeout(int(limit_cycles), _stream(stream)),
           "cpattn_selftest_wait_timeout")


def selftest_exp2(t, out=None, stream=None):
    """The attention kernel's FMA-pipe 2^t on a float32 CUDA tensor (test hook)."""
    if out is None:
        out = torch.empty_like(t)
    _need_cuda(t, out)
    _check(lib().cpattn_selftest_exp2(_ptr(t), _ptr(out), t.numel(), _stream(stream)),
           "cpattn_selftest_exp2")
    return out


def version() -> int:
    return lib().cpattn_version()
