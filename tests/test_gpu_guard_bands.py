"""Guard bands: every kernel that writes through computed indices writes inside its outputs
and nowhere else.

Each output (and the split-KV workspace) is carved out of a larger buffer whose bytes
before and after it hold a canary bit pattern (a NaN payload, so no computed value can
reproduce it by chance); after the call the canaries must be intact and the output must be
finite.  Shapes are ragged: query lengths that are not a multiple of the 256-row tile pair,
key lengths that end mid-block, permute shards whose length is not a multiple of 16 (where
the kernel allows it), and shards whose tiles straddle rank boundaries.
"""

import math

import pytest
import torch

import context_long_sequence_non_b200 as cp
from context_long_sequence_non_b200 import build as build_mod
from context_long_sequence_non_b200 import workloads as W

pytestmark = pytest.mark.gpu

DEV = "cuda"
GUARD_BYTES = 4096
CANARY = {2: 0x7FA5, 4: 0x7FC0A5A5}  # bf16 / float32 NaN payloads
INT_VIEW = {2: torch.int16, 4: torch.int32}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build_mod.build()
    cp.lib()
    yield
    assert cp.device_error() == 0


class Guarded:
    """A tensor of `shape` placed between two canary bands of GUARD_BYTES each."""

    def __init__(self, shape, dtype, init=None):
        es = torch.empty((), dtype=dtype).element_size()
        self.n = math.prod(shape)
        self.g = GUARD_BYTES // es
        self.es = es
        self.buf = torch.full((self.n + 2 * self.g,), CANARY[es], dtype=INT_VIEW[es], device=DEV)
        self.t = self.buf[self.g:self.g + self.n].view(dtype).view(shape)
        if init is not None:
            self.t.copy_(init)

    def intact(self):
        c = CANARY[self.es]
        return bool((self.buf[:self.g] == c).all()) and bool((self.buf[self.g + self.n:] == c).all())


def _check(*gs, finite=True):
    torch.cuda.synchronize()
    for i, g in enumerate(gs):
        assert g.intact(), f"output {i}: a canary byte was overwritten"
        if finite:
            assert torch.isfinite(g.t.float()).all(), f"output {i}: non-finite values"


@pytest.mark.parametrize("Bn,Sq,Skv,H,D", [(1, 300, 259, 3, 128), (2, 257, 1000, 2, 64)])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_guard_bands_attention_modes(Bn, Sq, Skv, H, D, out_dtype):
    q, k, v = (t.to(DEV) for t in W.random_case(Sq + Skv, Bn, H, Sq, Skv, D))
    o = Guarded((Bn, Sq, H, D), out_dtype)
    l = Guarded((Bn, H, Sq), torch.float32)
    cp.fwd(q, k, v, out=o.t, lse=l.t)
    _check(o, l)
    # accumulate a second chunk into the same guarded accumulator
    c = Skv // 3
    cp.fwd_accumulate(q, k[:, :c].contiguous(), v[:, :c].contiguous(), o.t, l.t)
    _check(o, l)
    # split-KV: guarded output and a guarded workspace of exactly the size asked for
    n = 3
    need = cp.split_workspace_bytes(Bn, H, Sq, D, n, out_dtype)
    # the workspace is bytes: its bands hold 0xA5
    wbuf = torch.full((need + 2 * GUARD_BYTES,), 0xA5, dtype=torch.uint8, device=DEV)
    wview = wbuf[GUARD_BYTES:GUARD_BYTES + need]
    o2 = Guarded((Bn, Sq, H, D), out_dtype)
    l2 = Guarded((Bn, H, Sq), torch.float32)
    cp.fwd_split(q, k, v, out=o2.t, lse=l2.t, n_split=n, workspace=wview)
    _check(o2, l2)
    assert bool((wbuf[:GUARD_BYTES] == 0xA5).all()) and bool((wbuf[GUARD_BYTES + need:] == 0xA5).all())
    cp.fwd_split(q, k, v, out=o2.t, lse=l2.t, n_split=n, workspace=wview, accumulate=True)
    _check(o2, l2)
    assert bool((wbuf[:GUARD_BYTES] == 0xA5).all()) and bool((wbuf[GUARD_BYTES + need:] == 0xA5).all())


@pytest.mark.parametrize("P,S_l,H,D", [(3, 48, 6, 128), (4, 400, 8, 64), (2, 272, 4, 128)])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_guard_bands_fused_ulysses(P, S_l, H, D, out_dtype):
    g = torch.Generator().manual_seed(P * 7 + S_l)
    shards = [W.randn((P, S_l, H, D), g, 1.0, "bf16").to(DEV) for _ in range(3)]
    o = Guarded((P, S_l, H, D), out_dtype)
    l = Guarded((P, H // P, P * S_l), torch.float32)
    cp.ulysses_fwd(*shards, P, out=o.t, lse=l.t)
    _check(o, l)


@pytest.mark.parametrize("P,S_l,H,D", [(4, 400, 64, 128), (3, 688, 24, 64)])
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_guard_bands_fused_ulysses_tail_split(P, S_l, H, D, out_dtype):
    g = torch.Generator().manual_seed(P * 11 + S_l)
    shards = [W.randn((P, S_l, H, D), g, 1.0, "bf16").to(DEV) for _ in range(3)]
    need = cp.ulysses_workspace_bytes(P, S_l, H, D, out_dtype)
    assert need > 0
    o = Guarded((P, S_l, H, D), out_dtype)
    l = Guarded((P, H // P, P * S_l), torch.float32)
    wbuf = torch.full((need + 2 * GUARD_BYTES,), 0xA5, dtype=torch.uint8, device=DEV)
    cp.ulysses_fwd_split(*shards, P, out=o.t, lse=l.t, workspace=wbuf[GUARD_BYTES:GUARD_BYTES + need])
    _check(o, l)
    assert bool((wbuf[:GUARD_BYTES] == 0xA5).all()) and bool((wbuf[GUARD_BYTES + need:] == 0xA5).all())


@pytest.mark.parametrize("Bn,S,H,D,dt", [(1, 301, 3, 128, torch.bfloat16), (2, 77, 2, 64, torch.float32),
                                         (1, 5, 1, 1024, torch.float32)])
def test_guard_bands_merge(Bn, S, H, D, dt):
    g = torch.Generator().manual_seed(S + D)
    oa, ob = (torch.randn(Bn, S, H, D, generator=g).to(dt).to(DEV) for _ in range(2))
    la, lb = (torch.randn(Bn, H, S, generator=g).to(DEV) for _ in range(2))
    o = Guarded((Bn, S, H, D), dt)
    l = Guarded((Bn, H, S), torch.float32)
    cp.merge(oa, la, ob, lb, out=o.t, lse=l.t)
    _check(o, l)
    # in place into a guarded accumulator
    acc_o = Guarded((Bn, S, H, D), dt, init=oa)
    acc_l = Guarded((Bn, H, S), torch.float32, init=la)
    cp.merge(acc_o.t, acc_l.t, ob, lb, out=acc_o.t, lse=acc_l.t)
    _check(acc_o, acc_l)


@pytest.mark.parametrize("P,S_l,H,D,dt", [(3, 37, 6, 8, torch.bfloat16), (8, 21, 16, 128, torch.bfloat16),
                                          (2, 5, 4, 16, torch.float32)])
def test_guard_bands_permutes(P, S_l, H, D, dt):
    g = torch.Generator().manual_seed(P + S_l + D)
    srcs = [torch.randn(P, S_l, H, D, generator=g).to(dt).to(DEV) for _ in range(3)]
    grouped = (P, P * S_l, H // P, D)
    d1 = Guarded(grouped, dt)
    cp.seq2head(srcs[0], P, out=d1.t)
    back = Guarded((P, S_l, H, D), dt)
    cp.head2seq(d1.t, P, out=back.t)
    _check(d1, back)
    assert torch.equal(back.t, srcs[0])
    outs = [Guarded(grouped, dt) for _ in range(3)]
    cp.seq2head_qkv(*srcs, P, out=tuple(o.t for o in outs))
    _check(*outs)
    if dt == torch.bfloat16:
        gq, gk = W.norm_weights(D, 1).to(DEV), W.norm_weights(D, 2).to(DEV)
        outs_n = [Guarded(grouped, dt) for _ in range(3)]
        cp.seq2head_qkv_norm(*srcs, P, gq, gk, out=tuple(o.t for o in outs_n))
        _check(*outs_n)


@pytest.mark.parametrize("rows,D", [(1001, 128), (37, 64), (5, 8)])
def test_guard_bands_rmsnorm(rows, D):
    g = torch.Generator().manual_seed(rows)
    x = torch.randn(rows, D, generator=g).to(torch.bfloat16).to(DEV)
    gamma = W.norm_weights(D, 3).to(DEV)
    y = Guarded((rows, D), torch.bfloat16)
    cp.rmsnorm(x, gamma, out=y.t)
    _check(y)
    xi = Guarded((rows, D), torch.bfloat16, init=x)  # in place
    cp.rmsnorm(xi.t, gamma, out=xi.t)
    _check(xi)
    assert torch.equal(xi.t, y.t)
