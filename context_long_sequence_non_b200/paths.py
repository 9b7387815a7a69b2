"""The two per-rank compositions of the hot path, built from the C-ABI calls.

* Ring Attention step (环形注意力 section of the TensorRT multi-device blog, Fig. 3): a
  rank keeps its Q slice and folds the partial (O, LSE) of each arriving K/V chunk into a
  running result with the exact online-softmax merge.
* DeepSpeed Ulysses (Fig. 4): all-to-all from sequence shards to head groups, attention
  over the full sequence per head group, all-to-all back; here the all-to-alls are local
  permutes over P virtual ranks on one GPU.

Buffers come from PyTorch (device memory only); every step is a libcpattn kernel.
"""

from __future__ import annotations

import math

import torch

from . import _binding as B


def ring_attention(q, k_chunks, v_chunks, scale=None, acc_dtype=None, fused=True, n_split=1,
                   stream=None):
    """One rank's ring step over K/V chunks in ring order.

    q: [B][Sq][H][D]; each chunk [B][S_c][H][D].  The running (O, LSE) is kept in
    ``acc_dtype`` (default: q's dtype).  ``fused=True`` (default) merges every chunk into
    the accumulator inside the attention epilogue (cpattn_fwd_accumulate); ``fused=False``
    writes each chunk's partial and folds it with the separate merge kernel.  With the fused
    form, ``n_split`` > 1 (or None: the library's suggestion) computes every chunk as that
    many key ranges folded straight into the accumulator (split-KV, for query slices too
    small to fill the GPU), and ``n_split = 0`` splits only the work items of each chunk's
    last wave or two of CTAs, as the library's makespan model chooses (tail split).
    Returns ``(O, LSE)``.
    """
    if scale is None:
        scale = 1.0 / math.sqrt(q.shape[3])
    acc_dtype = acc_dtype or q.dtype
    Bn, Sq, H, D = q.shape
    acc_o = torch.empty((Bn, Sq, H, D), dtype=acc_dtype, device=q.device)
    acc_l = torch.empty((Bn, H, Sq), dtype=torch.float32, device=q.device)
    if fused:
        if n_split is None:
            n_split = B.split_suggest(Bn, H, Sq, k_chunks[0].shape[1])
        if n_split != 1:
            need = max(B.split_workspace_bytes(Bn, H, Sq, D, n_split, acc_dtype, Skv=kc.shape[1])
                       for kc in k_chunks)
            ws = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
            acc_l.fill_(-math.inf)  # empty accumulator: its O rows are never read
            for kc, vc in zip(k_chunks, v_chunks):
                B.fwd_split(q, kc, vc, out=acc_o, lse=acc_l, scale=scale, accumulate=True,
                            n_split=n_split, workspace=ws, stream=stream)
            return acc_o, acc_l
        for c, (kc, vc) in enumerate(zip(k_chunks, v_chunks)):
            if c == 0:
                B.fwd(q, kc, vc, out=acc_o, lse=acc_l, scale=scale, stream=stream)
            else:
                B.fwd_accumulate(q, kc, vc, acc_o, acc_l, scale=scale, stream=stream)
        return acc_o, acc_l
    tmp_o = torch.empty_like(acc_o)
    tmp_l = torch.empty_like(acc_l)
    for c, (kc, vc) in enumerate(zip(k_chunks, v_chunks)):
        if c == 0:
            B.fwd(q, kc, vc, out=acc_o, lse=acc_l, scale=scale, stream=stream)
        else:
            B.fwd(q, kc, vc, out=tmp_o, lse=tmp_l, scale=scale, stream=stream)
            B.merge(acc_o, acc_l, tmp_o, tmp_l, out=acc_o, lse=acc_l, stream=stream)
    return acc_o, acc_l


class UlyssesPlan:
    """Preallocated buffers for the Ulysses path over P virtual ranks.

    Shards are [P][S_l][H][D]; head-grouped buffers [P][P*S_l][H/P][D].
    """

    def __init__(self, P, S_local, H, D, dtype=torch.bfloat16, device="cuda", batched=False,
                 qk_norm=None, norm_eps=1e-6):
        self.batched = batched  # one seq2head launch for Q, K, V together
        # (gamma_q, gamma_k) float32 [D]: the sample's Q/K RMSNorm fused into that launch
        self.qk_norm, self.norm_eps = qk_norm, norm_eps
        if H % P:
            raise ValueError("H must be divisible by P")
        self.P, self.S_local, self.H, self.D = P, S_local, H, D
        grouped = (P, P * S_local, H // P, D)
        self.qh = torch.empty(grouped, dtype=dtype, device=device)
        self.kh = torch.empty(grouped, dtype=dtype, device=device)
        self.vh = torch.empty(grouped, dtype=dtype, device=device)
        self.oh = torch.empty(grouped, dtype=dtype, device=device)
        self.lse = torch.empty((P, H // P, P * S_local), dtype=torch.float32, device=device)
        self.out = torch.empty((P, S_local, H, D), dtype=dtype, device=device)

    def run(self, q_shards, k_shards, v_shards, scale=None, stream=None):
        P = self.P
        if self.qk_norm is not None:
            B.seq2head_qkv_norm(q_shards, k_shards, v_shards, P, *self.qk_norm, eps=self.norm_eps,
                                out=(self.qh, self.kh, self.vh), stream=stream)
        elif self.batched:
            B.seq2head_qkv(q_shards, k_shards, v_shards, P, out=(self.qh, self.kh, self.vh),
                           stream=stream)
        else:
            B.seq2head(q_shards, P, out=self.qh, stream=stream)
            B.seq2head(k_shards, P, out=self.kh, stream=stream)
            B.seq2head(v_shards, P, out=self.vh, stream=stream)
        B.fwd(self.qh, self.kh, self.vh, out=self.oh, lse=self.lse, scale=scale, stream=stream)
        B.head2seq(self.oh, P, out=self.out, stream=stream)
        return self.out, self.lse


def ulysses_attention(q_shards, k_shards, v_shards, P, scale=None, stream=None):
    """seq2head x3 -> attention per head group -> head2seq.  Returns
    ``(O [P][S_l][H][D], LSE [P][H/P][P*S_l])``."""
    P_, S_l, H, D = q_shards.shape
    plan = UlyssesPlan(P, S_l, H, D, dtype=q_shards.dtype, device=q_shards.device)
    out, lse = plan.run(q_shards, k_shards, v_shards, scale=scale, stream=stream)
    return out, lse


class UlyssesStreamer:
    """Host-to-host Ulysses passes with the copies of neighbouring steps overlapped with
    compute.

    ``depth`` device buffer sets rotate.  Step i's Q/K/V go host -> device on an upload
    stream, its pass runs on the compute stream, and O and LSE go device -> host on a
    download stream.  Events order the three per buffer set:
    - upload i after the pass that last read set i % depth;
    - pass i after upload i and after the download that last emptied the set's outputs;
    - download i after pass i.

    So the upload of step i+1 and the download of step i-1 run while step i computes.
    Host buffers should be pinned, or the copies are not asynchronous.  ``submit`` returns
    the event that completes when step i's outputs are on the host.  The copies are
    asynchronous: a step's host inputs must not be modified, and its host outputs not
    read or reused, until that event has completed.
    """

    def __init__(self, P, S_local, H, D, dtype=torch.bfloat16, device="cuda", depth=2):
        if depth < 1:
            raise ValueError("depth must be at least 1 (2 or more to overlap copies)")
        self.depth = depth
        self.plans = [UlyssesPlan(P, S_local, H, D, dtype=dtype, device=device)
                      for _ in range(depth)]
        shard = (P, S_local, H, D)
        self.inputs = [tuple(torch.empty(shard, dtype=dtype, device=device) for _ in range(3))
                       for _ in range(depth)]
        self.compute = torch.cuda.current_stream(device)
        self.upload = torch.cuda.Stream(device)
        self.download = torch.cuda.Stream(device)
        ev = lambda: [torch.cuda.Event() for _ in range(depth)]
        self.uploaded, self.computed, self.downloaded = ev(), ev(), ev()
        self.step = 0

    def submit(self, hq, hk, hv, h_out, h_lse, scale=None):
        k = self.step % self.depth
        plan, (dq, dk, dv) = self.plans[k], self.inputs[k]
        if any(t.shape != dq.shape for t in (hq, hk, hv)):
            raise ValueError(f"host Q/K/V shards must be {tuple(dq.shape)}")
        if h_out.shape != plan.out.shape or h_lse.shape != plan.lse.shape:
            raise ValueError(f"h_out must be {tuple(plan.out.shape)} and h_lse "
                             f"{tuple(plan.lse.shape)}")
        # waiting on an event that was never recorded returns at once (first rotation)
        self.upload.wait_event(self.computed[k])
        with torch.cuda.stream(self.upload):
            dq.copy_(hq, non_blocking=True)
            dk.copy_(hk, non_blocking=True)
            dv.copy_(hv, non_blocking=True)
            self.uploaded[k].record(self.upload)
        self.compute.wait_event(self.uploaded[k])
        self.compute.wait_event(self.downloaded[k])
        plan.run(dq, dk, dv, scale=scale, stream=self.compute)
        self.computed[k].record(self.compute)
        self.download.wait_event(self.computed[k])
        with torch.cuda.stream(self.download):
            h_out.copy_(plan.out, non_blocking=True)
            h_lse.copy_(plan.lse, non_blocking=True)
            self.downloaded[k].record(self.download)
        self.step += 1
        return self.downloaded[k]


class UlyssesHostPass:
    """A whole Ulysses attention layer from host memory to host memory in one C-ABI call
    (cpattn_ulysses_host).  The device work buffers are allocated here once, by PyTorch;
    the library allocates nothing.  Inside the call the head groups go in ``n_chunks``
    chunks: the upload of chunk c+1 and the download of chunk c-1 overlap the attention of
    chunk c.  Host tensors should be pinned."""

    def __init__(self, P, S_local, H, D, out_dtype=torch.bfloat16, device="cuda", n_chunks=None,
                 with_lse=True):
        shard = (P, S_local, H, D)
        self.P, self.n_chunks = P, n_chunks if n_chunks is not None else P
        self.dq, self.dk, self.dv = (torch.empty(shard, dtype=torch.bfloat16, device=device)
                                     for _ in range(3))
        self.d_out = torch.empty(shard, dtype=out_dtype, device=device)
        self.d_lse = (torch.empty((P, H // P, P * S_local), dtype=torch.float32, device=device)
                      if with_lse else None)

    def run(self, hq, hk, hv, h_out, h_lse=None, scale=None, stream=None):
        """Enqueue one pass; h_out / h_lse are valid once ``stream`` has passed it."""
        return B.ulysses_host(hq, hk, hv, h_out, h_lse, self.dq, self.dk, self.dv, self.d_out,
                              self.d_lse if h_lse is not None else None, self.P, scale=scale,
                              n_chunks=self.n_chunks, stream=stream)
