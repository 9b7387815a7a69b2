"""Pins for the oracle's Q/K RMSNorm (the attention_mdtrt sample's 模型的核心结构 section:
fp32 x * rsqrt(mean(x^2) + eps), eps 1e-6, times a weight, split scale D^-1/4 on Q and K).

Closed forms, invariants and a loop brute force fix what the page fixes; planted mistakes
(eps outside the root, a sum for the mean, the wrong axis, a per-head weight) must each
fail at least one pin.
"""

import math

import numpy as np
import pytest

from oracle import brute, ref

EPS = 1e-6


def check_constant_row(fn):
    # x = c * 1: mean(x^2) = c^2, so y = c / sqrt(c^2 + eps) * gamma (c = 1e-3 puts c^2 = eps)
    d = 16
    g = np.linspace(0.25, 2.0, d)
    for c in (2.0, -0.5, 1e-3):
        y = np.asarray(fn(np.full((1, 1, 1, d), c), g, EPS), dtype=np.float64)[0, 0, 0]
        want = c / math.sqrt(c * c + EPS) * g
        assert np.allclose(y, want, rtol=2e-6, atol=0), (c, y[:3], want[:3])


def check_one_hot(fn):
    # x = a * e_k: mean(x^2) = a^2 / D, y_k = gamma_k * a / sqrt(a^2/D + eps), the rest 0
    d = 32
    g = np.linspace(1.0, 2.0, d)
    for k, a in ((0, 3.0), (5, -0.25), (31, 1e-2)):
        x = np.zeros((1, 1, 1, d))
        x[0, 0, 0, k] = a
        y = np.asarray(fn(x, g, EPS), dtype=np.float64)[0, 0, 0]
        want = np.zeros(d)
        want[k] = g[k] * a / math.sqrt(a * a / d + EPS)
        assert np.allclose(y, want, rtol=2e-6, atol=0), (k, a)


def check_unit_rms_per_head(fn):
    # heads of very different magnitude: every (b, s, h) row comes out with
    # mean(y^2) = ms / (ms + eps) under gamma = 1, whatever its neighbours are
    rng = np.random.default_rng(7)
    b, s, h, d = 2, 5, 4, 64
    mag = np.array([1e-3, 1.0, 30.0, 1e3])
    x = rng.standard_normal((b, s, h, d)) * mag[None, None, :, None]
    x = x.astype(np.float32).astype(np.float64)
    y = np.asarray(fn(x, np.ones(d), EPS), dtype=np.float64)
    ms = np.mean(x * x, axis=-1)
    assert np.allclose(np.mean(y * y, axis=-1), ms / (ms + EPS), rtol=1e-5, atol=0)


def check_weight_per_dim(fn):
    # gamma multiplies column d of every head row: y(gamma) = y(1) * gamma
    rng = np.random.default_rng(8)
    d = 32
    x = rng.standard_normal((2, 3, 4, d)).astype(np.float32)
    g = np.linspace(-2.0, 3.0, d)
    y1 = np.asarray(fn(x, np.ones(d), EPS), dtype=np.float64)
    yg = np.asarray(fn(x, g, EPS), dtype=np.float64)
    assert np.allclose(yg, y1 * g, rtol=1e-6, atol=1e-7)


def test_constant_row_closed_form():
    check_constant_row(ref.rmsnorm_heads)
    check_constant_row(brute.rmsnorm_heads)


def test_one_hot_closed_form():
    check_one_hot(ref.rmsnorm_heads)
    check_one_hot(brute.rmsnorm_heads)


def test_unit_rms_per_head_row():
    check_unit_rms_per_head(ref.rmsnorm_heads)


def test_weight_scales_each_head_dim():
    check_weight_per_dim(ref.rmsnorm_heads)


def test_scale_invariance():
    # y(4x) = y(x) up to the eps term (4 is a power of two: x*4 and its squares are exact)
    rng = np.random.default_rng(9)
    x = rng.standard_normal((3, 7, 2, 128)).astype(np.float32)
    g = rng.uniform(0.5, 1.5, 128)
    assert np.allclose(ref.rmsnorm_heads(4 * x, g), ref.rmsnorm_heads(x, g), rtol=2e-6, atol=1e-7)


def test_out_scale_is_a_plain_factor():
    rng = np.random.default_rng(10)
    x = rng.standard_normal((2, 3, 4, 128)).astype(np.float32)
    g = np.ones(128)
    s = 128 ** -0.25  # the sample's split scale sqrt(sqrt(1/HEAD_DIM))
    assert np.allclose(ref.rmsnorm_heads(x, g, out_scale=s), ref.rmsnorm_heads(x, g) * s,
                       rtol=1e-6, atol=0)


@pytest.mark.parametrize("shape", [(1, 1, 1, 8), (2, 3, 4, 16), (1, 5, 3, 64), (1, 2, 2, 128)])
def test_brute_force_agrees(shape):
    rng = np.random.default_rng(sum(shape))
    x = (rng.standard_normal(shape) * rng.uniform(0.01, 10.0)).astype(np.float32)
    g = rng.uniform(-1.5, 1.5, shape[-1])
    a = ref.rmsnorm_heads(x, g).astype(np.float64)
    b = np.array(brute.rmsnorm_heads(x.tolist(), g.tolist()))
    # float32 arithmetic (4 roundings after a float32 mean) against exact float64
    assert np.allclose(a, b, rtol=2e-6, atol=1e-30)


def test_norm_commutes_with_the_ulysses_permute():
    # the norm acts on whole head rows and seq2head moves whole head rows
    rng = np.random.default_rng(11)
    p, s_l, h, d = 4, 3, 8, 16
    x = rng.standard_normal((p, s_l, h, d)).astype(np.float32)
    g = rng.uniform(0.5, 1.5, d)
    a = ref.seq2head(ref.rmsnorm_heads(x, g), p)
    b = ref.rmsnorm_heads(ref.seq2head(x, p), g)
    assert np.array_equal(a, b)


def _mutant(kind):
    def bad(x, gamma, eps=1e-6, out_scale=1.0):
        x = np.asarray(x, dtype=np.float64)
        g = np.asarray(gamma, dtype=np.float64)
        if kind == "eps_outside_root":
            r = 1.0 / (np.sqrt(np.mean(x * x, axis=-1, keepdims=True)) + eps)
        elif kind == "sum_not_mean":
            r = 1.0 / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)
        elif kind == "over_heads":  # normalised over (heads, dim) instead of per head row
            r = 1.0 / np.sqrt(np.mean(x * x, axis=(-2, -1), keepdims=True) + eps)
        elif kind == "no_square_root":
            r = 1.0 / (np.mean(x * x, axis=-1, keepdims=True) + eps)
        elif kind == "weight_per_head":  # gamma indexed by the head instead of the dim
            r = 1.0 / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
            gh = np.resize(g, x.shape[-2])[:, None]
            return x * r * gh * out_scale
        return x * r * g * out_scale
    return bad


@pytest.mark.parametrize("kind", ["eps_outside_root", "sum_not_mean", "over_heads",
                                  "no_square_root", "weight_per_head"])
def test_planted_rmsnorm_mistake_is_caught(kind):
    fn = _mutant(kind)
    caught = 0
    for pin in (check_constant_row, check_one_hot, check_unit_rms_per_head, check_weight_per_dim):
        try:
            pin(fn)
        except AssertionError:
            caught += 1
    assert caught >= 1, f"no pin caught {kind!r}"
