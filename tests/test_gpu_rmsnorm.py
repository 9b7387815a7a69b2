"""GPU parity of the Q/K RMSNorm (cpattn_rmsnorm) and of its fusion into the Ulysses
seq2head (cpattn_seq2head_qkv_norm), through the C ABI, against the oracle's float32
restatement of the attention_mdtrt sample's norm (模型的核心结构).

Both sides compute in float32 (the precision the page fixes) and round to bf16 (RNE); they
sum the squares in different orders, so a result may land on the other side of a bf16
rounding boundary.  The bar: every element bit-equal to the rounded oracle value except at
most max(2, 1e-4 * n) elements that differ by one bf16 unit and whose float32 oracle value
lies within 1e-6 (relative) of the midpoint between the two candidates -- a rounding tie,
never an arithmetic difference.
"""

import math

import numpy as np
import pytest
import torch

import context_long_sequence_non_b200 as cp
from context_long_sequence_non_b200 import build as build_mod
from context_long_sequence_non_b200 import workloads as W
from context_long_sequence_non_b200.paths import UlyssesPlan
from oracle import ref
from parity import check_lse, check_o

pytestmark = pytest.mark.gpu

DEV = "cuda"


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    build_mod.build()
    cp.lib()
    yield
    assert cp.device_error() == 0


def bits(t):
    return t.view(torch.int16)


def check_rounded(got, y32, what=""):
    """got: bf16 tensor; y32: the oracle's float32 values before the cast."""
    got = got.detach().cpu()
    exp = torch.from_numpy(np.ascontiguousarray(y32)).to(torch.bfloat16)
    gi, ei = bits(got).to(torch.int32), bits(exp).to(torch.int32)
    assert gi.shape == ei.shape, (gi.shape, ei.shape)
    diff = (gi - ei).abs()
    n = diff.numel()
    bad = diff != 0
    nbad = int(bad.sum())
    assert int(diff.max()) <= 1, f"{what}: a result differs by more than one bf16 unit"
    assert nbad <= max(2, int(1e-4 * n)), f"{what}: {nbad} of {n} results differ"
    if nbad:
        y = torch.from_numpy(np.ascontiguousarray(y32)).double()[bad]
        mid = (got[bad].double() + exp[bad].double()) / 2
        assert ((y - mid).abs() <= 1e-6 * y.abs()).all(), f"{what}: a mismatch is not a rounding tie"
    return nbad


@pytest.mark.parametrize("shape,sigma", [((1, 37, 3, 128), 1.0), ((2, 100, 5, 64), 30.0),
                                         ((1, 1, 1, 8), 1.0), ((3, 50, 2, 256), 0.01),
                                         ((1, 1000, 16, 128), 2.0), ((1, 7, 1, 16), 1.0),
                                         ((1, 5, 3, 32), 5.0)])
@pytest.mark.parametrize("mode", ["out_of_place", "in_place", "split_scale"])
def test_rmsnorm_matches_oracle(shape, sigma, mode):
    g = torch.Generator().manual_seed(sum(shape) + int(sigma * 10))
    x = W.randn(shape, g, sigma, "bf16")
    gamma = W.norm_weights(shape[-1], seed=shape[-1])
    out_scale = shape[-1] ** -0.25 if mode == "split_scale" else 1.0
    xd, gd = x.to(DEV), gamma.to(DEV)
    if mode == "in_place":
        y = cp.rmsnorm(xd, gd, out=xd)
        assert y.data_ptr() == xd.data_ptr()
    else:
        y = cp.rmsnorm(xd, gd, out_scale=out_scale)
    torch.cuda.synchronize()
    check_rounded(y, ref.rmsnorm_heads(x, gamma, 1e-6, out_scale), f"rmsnorm {shape} {mode}")


def test_rmsnorm_zero_rows_and_zero_input():
    gamma = W.norm_weights(128, seed=1).to(DEV)
    empty = torch.empty((0, 128), dtype=torch.bfloat16, device=DEV)
    cp.rmsnorm(empty, gamma)  # rows = 0: a no-op that returns OK
    z = torch.zeros((3, 4, 128), dtype=torch.bfloat16, device=DEV)
    y = cp.rmsnorm(z, gamma)  # mean(x^2) = 0: r = 1/sqrt(eps), y = 0 exactly
    torch.cuda.synchronize()
    assert torch.equal(bits(y), bits(z))


# (1, 9, 4, 256) has 2 KB rows (4 chunks of 32 vectors) and (2, 11, 24, 128) 3 KB rows
# (6 chunks): head rows in every chunk position.
@pytest.mark.parametrize("P,S_l,H,D", [(2, 3, 4, 8), (4, 33, 8, 128), (8, 17, 16, 128),
                                       (2, 5, 2, 64), (1, 9, 4, 256), (3, 7, 6, 32), (2, 11, 24, 128)])
def test_seq2head_qkv_norm_matches_oracle(P, S_l, H, D):
    g = torch.Generator().manual_seed(P * 31 + S_l)
    q, k, v = (W.randn((P, S_l, H, D), g, 3.0, "bf16") for _ in range(3))
    gq, gk = W.norm_weights(D, seed=10 + D), W.norm_weights(D, seed=20 + D)
    qd, kd, vd, gqd, gkd = (t.to(DEV) for t in (q, k, v, gq, gk))
    qh, kh, vh = cp.seq2head_qkv_norm(qd, kd, vd, P, gqd, gkd)
    # the same result from the two separate calls: same arithmetic, identical bits
    qh2 = cp.seq2head(cp.rmsnorm(qd, gqd), P)
    kh2 = cp.seq2head(cp.rmsnorm(kd, gkd), P)
    torch.cuda.synchronize()
    assert torch.equal(bits(qh), bits(qh2)) and torch.equal(bits(kh), bits(kh2))
    np.testing.assert_array_equal(bits(vh).cpu().numpy(), ref.seq2head(bits(v).numpy(), P))
    check_rounded(qh, ref.seq2head(ref.rmsnorm_heads(q, gq), P), "qh")
    check_rounded(kh, ref.seq2head(ref.rmsnorm_heads(k, gk), P), "kh")


def test_seq2head_qkv_norm_full_size():
    # the Cosmos-3 Ulysses shards: P = 8 x [5520][16][128]
    w = W.WORKLOADS[4]
    x = W.make_inputs(w)
    P = w.P
    gq, gk = W.norm_weights(w.D, seed=41), W.norm_weights(w.D, seed=42)
    q, k, v, gqd, gkd = (t.to(DEV) for t in (x["q"], x["k"], x["v"], gq, gk))
    qh, kh, vh = cp.seq2head_qkv_norm(q, k, v, P, gqd, gkd)
    qh2 = cp.seq2head(cp.rmsnorm(q, gqd), P)
    kh2 = cp.seq2head(cp.rmsnorm(k, gkd), P)
    vh2 = cp.seq2head(v, P)
    torch.cuda.synchronize()
    assert torch.equal(bits(qh), bits(qh2)) and torch.equal(bits(kh), bits(kh2))
    assert torch.equal(bits(vh), bits(vh2))
    # sampled head rows against the oracle: every 97th token of every rank, all heads
    tok = torch.arange(0, w.Sq // P, 97)
    for name, dev_buf, gamma in (("q", qh, gq), ("k", kh, gk)):
        src = x[name][:, tok]  # [P][n][H][D]
        want = ref.rmsnorm_heads(src, gamma)
        H = src.shape[2]
        hp = H // P
        got = dev_buf.cpu()  # [P][P*S_l][Hp][D]: group g row r*S_l + s holds src[r][s][g*Hp + j]
        sel = torch.stack([torch.stack([got[h // hp, r * (w.Sq // P) + tok, h % hp] for h in range(H)],
                                       dim=1) for r in range(P)])
        check_rounded(sel, want, f"{name}h sampled")


@pytest.mark.parametrize("P,S_l,H,D", [(2, 320, 4, 128), (4, 96, 8, 64)])
def test_ulysses_attention_with_qk_norm(P, S_l, H, D):
    g = torch.Generator().manual_seed(P * 7 + S_l)
    q, k, v = (W.randn((P, S_l, H, D), g, s, "bf16") for s in (4.0, 4.0, 1.0))
    gq, gk = W.norm_weights(D, seed=3), W.norm_weights(D, seed=4)
    plan = UlyssesPlan(P, S_l, H, D, qk_norm=(gq.to(DEV), gk.to(DEV)))
    out, lse = plan.run(q.to(DEV), k.to(DEV), v.to(DEV), scale=1 / math.sqrt(D))
    torch.cuda.synchronize()
    # single-device meaning: attention of the normalised (bf16) Q, K over the full sequence
    qn = torch.from_numpy(ref.rmsnorm_heads(q, gq)).to(torch.bfloat16)
    kn = torch.from_numpy(ref.rmsnorm_heads(k, gk)).to(torch.bfloat16)
    full = lambda t: t.reshape(1, P * S_l, H, D)
    o_ref, l_ref = ref.attention(full(qn), full(kn), full(v), 1 / math.sqrt(D))
    check_o(out.cpu().reshape(1, P * S_l, H, D), o_ref, "bf16_out", "ulysses + qk norm")
    hp = H // P
    check_lse(lse.cpu().reshape(H, P * S_l), l_ref[0].reshape(H, P * S_l), "ulysses + qk norm")
