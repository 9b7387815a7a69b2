"""Seeded synthetic workloads (input generation only; none of the method's arithmetic).

These generators feed both the CUDA path and the CPU oracle.  They draw iid normal
samples with ``torch.Generator('cpu')`` + ``torch.randn`` in float32, multiply by the
stated sigma and round to bf16 (round-to-nearest-even) where the workload is bf16.
Tensors Q, K, V are drawn in that order from one generator seeded per workload.

The shapes follow the workloads on the pages: the image-DiT joint sequence (4096 image
+ 512 text tokens), the Cosmos 3 Nano video latent of 44160 tokens split over 8 ranks
(5520 tokens per rank) and its 2992-token text path concatenated to it, with 16 heads
of 128 (the pages give 44160/5520 and 2992 tokens; head count and width are readings).
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    """One synthetic case.  ``kind`` selects how the hot path runs over it.

    * ``single``:  one attention call, Q [B][Sq][H][D], K/V [B][Skv][H][D].
    * ``chunked`` / ``ring``: the same Q against K/V split into ``chunks`` along the
      key sequence; per-chunk (O, LSE) merged in chunk order, compared with one pass.
    * ``ulysses``: P virtual ranks each hold [S_l][H][D] of Q, K, V; seq2head,
      attention per head group, head2seq.
    """

    key: int
    name: str
    kind: str
    B: int
    H: int
    Sq: int
    Skv: int
    D: int
    dtype: str  # "bf16" or "f32"
    seed: int
    sigma_qk: float = 1.0
    sigma_v: float = 1.0
    chunks: tuple = ()
    P: int = 1
    scale: float = field(default=float("nan"))

    @property
    def softmax_scale(self) -> float:
        return self.scale if not math.isnan(self.scale) else 1.0 / math.sqrt(self.D)

    @property
    def attn_flops(self) -> float:
        """4*B*H*Sq*Skv*D: the two matmuls of attention (exp work not counted)."""
        return 4.0 * self.B * self.H * self.Sq * self.Skv * self.D


WORKLOADS = {
    1: Workload(1, "tiny-fp32-chunked", "chunked", B=1, H=2, Sq=256, Skv=256, D=64,
                dtype="f32", seed=1000, chunks=(128, 128), scale=1.0 / 8.0),
    2: Workload(2, "image-dit-joint-4608", "single", B=1, H=24, Sq=4608, Skv=4608, D=128,
                dtype="bf16", seed=2000),
    3: Workload(3, "ring-step-5520x8x5520", "ring", B=1, H=16, Sq=5520, Skv=44160, D=128,
                dtype="bf16", seed=3000, chunks=(5520,) * 8),
    # Ulysses: attention runs over B = P head groups of H/P heads each, full sequence
    4: Workload(4, "ulysses-cp8-44160", "ulysses", B=8, H=2, Sq=44160, Skv=44160, D=128,
                dtype="bf16", seed=4000, P=8),
    5: Workload(5, "video-text-joint-47152-sigma3", "single", B=1, H=16, Sq=47152,
                Skv=47152, D=128, dtype="bf16", seed=5000, sigma_qk=3.0),
}

ULYSSES_LOCAL_TOKENS = 5520  # per-rank share of the 44160 video tokens at CP8
ULYSSES_HEADS = 16


def _torch_dtype(name: str):
    return {"bf16": torch.bfloat16, "f32": torch.float32}[name]


def randn(shape, gen: torch.Generator, sigma: float, dtype: str) -> torch.Tensor:
    """float32 N(0, sigma^2) samples, rounded to ``dtype`` (RNE for bf16)."""
    x = torch.randn(*shape, generator=gen, dtype=torch.float32)
    if sigma != 1.0:
        x.mul_(sigma)
    return x.to(_torch_dtype(dtype))


def make_inputs(w: Workload) -> dict:
    """CPU tensors for a workload: ``{"q", "k", "v"}`` (plus the chunk split)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed)
    if w.kind == "ulysses":
        s_l = w.Sq // w.P
        h_full = w.H * w.P
        shape = (w.P, s_l, h_full, w.D)  # [P][S_l][H][D] per-rank shards
        q = randn(shape, g, w.sigma_qk, w.dtype)
        k = randn(shape, g, w.sigma_qk, w.dtype)
        v = randn(shape, g, w.sigma_v, w.dtype)
        return {"q": q, "k": k, "v": v}
    q = randn((w.B, w.Sq, w.H, w.D), g, w.sigma_qk, w.dtype)
    k = randn((w.B, w.Skv, w.H, w.D), g, w.sigma_qk, w.dtype)
    v = randn((w.B, w.Skv, w.H, w.D), g, w.sigma_v, w.dtype)
    out = {"q": q, "k": k, "v": v}
    if w.chunks:
        assert sum(w.chunks) == w.Skv
        out["chunks"] = list(w.chunks)
    return out


def norm_weights(D: int, seed: int) -> torch.Tensor:
    """float32 [D] RMSNorm weights for the Q/K norm (the sample draws random weights):
    1 + 0.1 * N(0, 1), seeded."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return 1.0 + 0.1 * torch.randn(D, generator=g, dtype=torch.float32)


def random_case(seed: int, B: int, H: int, Sq: int, Skv: int, D: int, dtype: str = "bf16",
                sigma_qk: float = 1.0, sigma_v: float = 1.0):
    """Generic seeded case for parity tests of ragged and edge shapes."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    q = randn((B, Sq, H, D), g, sigma_qk, dtype)
    k = randn((B, Skv, H, D), g, sigma_qk, dtype)
    v = randn((B, Skv, H, D), g, sigma_v, dtype)
    return q, k, v


def sample_rows(B: int, H: int, S: int, n: int, seed: int, tile: int = 128):
    """(b, h, i) query rows to check at full size: row 0, the rows either side of every
    few tile boundaries, the last tile's rows (ragged tail) and seeded random rows."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    picks = set()
    for b in range(B):
        for h in range(H):
            for i in (0, 1, tile - 1, tile, S - 1):
                if 0 <= i < S:
                    picks.add((b, h, i))
    tail0 = (S // tile) * tile
    for i in range(max(0, tail0 - 2), S):
        picks.add((B - 1, H - 1, i))
    while len(picks) < n:
        b = int(torch.randint(0, B, (1,), generator=g))
        h = int(torch.randint(0, H, (1,), generator=g))
        i = int(torch.randint(0, S, (1,), generator=g))
        picks.add((b, h, i))
    return sorted(picks)
