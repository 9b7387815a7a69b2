"""Property-based pins of the oracle (hypothesis): random shapes, splits and scales checked
against invariants the mathematics fixes, independent of the worked examples:

* chunked attention merged in any order equals unchunked attention (the Ring step);
* the merge is commutative, and a chunk's result merged with itself adds ln 2 to LSE;
* seq2head / head2seq are mutually inverse permutations for every P dividing H;
* scaling all logits by c: LSE shifts as a log-sum-exp, O is the softmax-weighted mean;
* the Q/K RMSNorm output has unit RMS per head row (gamma = 1) for any magnitude.
"""

import math

import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

from oracle import ref

SETTINGS = settings(max_examples=40, deadline=None,
                    suppress_health_check=[HealthCheck.too_slow])


def _data(seed, b, sq, skv, h, d, sigma=1.0):
    r = np.random.default_rng(seed)
    q = r.standard_normal((b, sq, h, d)) * sigma
    k = r.standard_normal((b, skv, h, d)) * sigma
    v = r.standard_normal((b, skv, h, d))
    return q, k, v


@SETTINGS
@given(seed=st.integers(0, 2**31 - 1), skv=st.integers(1, 40), n_cuts=st.integers(0, 5),
       order_seed=st.integers(0, 1000))
def test_chunked_merge_in_any_order_equals_unchunked(seed, skv, n_cuts, order_seed):
    q, k, v = _data(seed, 1, 5, skv, 2, 4, sigma=1.5)
    r = np.random.default_rng(seed + 1)
    cuts = sorted(set([0, skv] + list(r.integers(0, skv + 1, size=n_cuts))))
    parts = [ref.attention(q, k[:, a:b], v[:, a:b], 0.3) for a, b in zip(cuts, cuts[1:])]
    np.random.default_rng(order_seed).shuffle(parts)  # the merge is order-independent
    o, lse = ref.merge_chunks(parts)
    o_full, l_full = ref.attention(q, k, v, 0.3)
    np.testing.assert_allclose(o, o_full, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse, l_full, rtol=1e-12, atol=1e-12)


@SETTINGS
@given(seed=st.integers(0, 2**31 - 1), sa=st.integers(1, 20), sb=st.integers(1, 20))
def test_merge_commutes_and_self_merge_adds_ln2(seed, sa, sb):
    q, k, v = _data(seed, 2, 3, sa + sb, 2, 3)
    pa = ref.attention(q, k[:, :sa], v[:, :sa], 0.5)
    pb = ref.attention(q, k[:, sa:], v[:, sa:], 0.5)
    o1, l1 = ref.merge(pa[0], pa[1], pb[0], pb[1])
    o2, l2 = ref.merge(pb[0], pb[1], pa[0], pa[1])
    np.testing.assert_allclose(o1, o2, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(l1, l2, rtol=1e-15, atol=1e-15)
    o3, l3 = ref.merge(pa[0], pa[1], pa[0], pa[1])
    np.testing.assert_allclose(o3, pa[0], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(l3 - pa[1], math.log(2.0), rtol=0, atol=1e-13)


@SETTINGS
@given(p=st.integers(1, 6), hp=st.integers(1, 4), s_l=st.integers(1, 9), d=st.integers(1, 5),
       seed=st.integers(0, 2**31 - 1))
def test_permutes_are_inverse_for_any_grouping(p, hp, s_l, d, seed):
    h = p * hp
    x = np.random.default_rng(seed).integers(-1000, 1000, size=(p, s_l, h, d))
    y = ref.seq2head(x, p)
    assert y.shape == (p, p * s_l, hp, d)
    np.testing.assert_array_equal(ref.head2seq(y, p), x)
    # a permutation: the multiset of values is unchanged
    np.testing.assert_array_equal(np.sort(y, axis=None), np.sort(x, axis=None))


@SETTINGS
@given(seed=st.integers(0, 2**31 - 1), c=st.floats(0.05, 4.0))
def test_lse_is_logsumexp_of_scaled_logits(seed, c):
    # LSE(scale) = logsumexp(scale * s) and O = softmax(scale * s) V, checked through the
    # row's own logits for any positive scale
    q, k, v = _data(seed, 1, 4, 9, 1, 6)
    o, lse = ref.attention(q, k, v, c)
    s = c * (q[0, :, 0] @ k[0, :, 0].T)
    mx = s.max(axis=1, keepdims=True)
    lse_direct = (mx + np.log(np.exp(s - mx).sum(axis=1, keepdims=True)))[:, 0]
    np.testing.assert_allclose(lse[0, 0], lse_direct, rtol=1e-13, atol=1e-13)
    w = np.exp(s - lse_direct[:, None])
    np.testing.assert_allclose(o[0, :, 0], w @ v[0, :, 0], rtol=1e-12, atol=1e-13)


@SETTINGS
@given(seed=st.integers(0, 2**31 - 1), log_mag=st.floats(-3.0, 3.0),
       d=st.sampled_from([8, 16, 64, 128]))
def test_rmsnorm_unit_rms_for_any_magnitude(seed, log_mag, d):
    x = (np.random.default_rng(seed).standard_normal((2, 3, 4, d)) * 10.0 ** log_mag)
    x = x.astype(np.float32)
    y = ref.rmsnorm_heads(x, np.ones(d)).astype(np.float64)
    ms = np.mean(x.astype(np.float64) ** 2, axis=-1)
    np.testing.assert_allclose(np.mean(y * y, axis=-1), ms / (ms + 1e-6), rtol=2e-5)
