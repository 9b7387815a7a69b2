"""Pins for the CPU oracle (no GPU).  Each test ties ``oracle`` to something other
than itself: hand-derived worked examples (tests/golden), closed forms, invariants,
library routines (scipy.special.softmax / logsumexp) and a loop-only brute force.
The last group plants plausible mistakes in the oracle and checks the pins catch them.
"""

import json
import math
import os

import numpy as np
import pytest
import scipy.special

from oracle import brute, ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _ev(expr):
    return float(eval(str(expr), {"__builtins__": {}}, {"ln": math.log}))


def _arr(case, name):
    if name in case:
        return np.asarray(case[name], dtype=np.float64)
    return np.vectorize(_ev, otypes=[np.float64])(np.asarray(case[name + "_expr"], dtype=object))


def _golden_cases():
    with open(os.path.join(GOLDEN, "attn_closed_form.json")) as f:
        return json.load(f)["cases"]


def _rng(seed):
    return np.random.default_rng(seed)


def _rand(seed, b, sq, skv, h, d, sigma=1.0):
    r = _rng(seed)
    q = r.standard_normal((b, sq, h, d)) * sigma
    k = r.standard_normal((b, skv, h, d)) * sigma
    v = r.standard_normal((b, skv, h, d))
    return q, k, v


# ----------------------------------------------------------------------------- attention


def check_golden(attention):
    for case in _golden_cases():
        q, k, v = _arr(case, "q"), _arr(case, "k"), _arr(case, "v")
        scale = _ev(case["scale_expr"])
        o, lse = attention(q, k, v, scale)
        np.testing.assert_allclose(o, _arr(case, "o"), rtol=0, atol=1e-12, err_msg=case["name"])
        np.testing.assert_allclose(lse, _arr(case, "lse"), rtol=0, atol=1e-12, err_msg=case["name"])


def test_golden_worked_examples_ref():
    check_golden(ref.attention)


def test_golden_worked_examples_brute():
    check_golden(lambda q, k, v, s: tuple(np.asarray(x) for x in brute.attention(q, k, v, s)))


def check_softmax_identity(attention):
    # V = I (Skv = D): O row i is the softmax row of the scaled logits; LSE is logsumexp
    for seed, (b, sq, h, d) in enumerate([(1, 7, 2, 5), (2, 3, 1, 9), (1, 12, 3, 4)]):
        r = _rng(100 + seed)
        q = r.standard_normal((b, sq, h, d))
        k = r.standard_normal((b, d, h, d))
        v = np.broadcast_to(np.eye(d)[None, :, None, :], (b, d, h, d)).copy()
        scale = 0.37 + seed
        o, lse = attention(q, k, v, scale)
        for bb in range(b):
            for hh in range(h):
                s = scale * q[bb, :, hh, :] @ k[bb, :, hh, :].T
                np.testing.assert_allclose(o[bb, :, hh, :], scipy.special.softmax(s, axis=1),
                                           rtol=1e-12, atol=1e-14)
                np.testing.assert_allclose(lse[bb, hh], scipy.special.logsumexp(s, axis=1),
                                           rtol=1e-13, atol=1e-13)


def test_v_identity_is_library_softmax():
    check_softmax_identity(ref.attention)


def test_q_zero_gives_mean_of_v():
    _, k, v = _rand(1, 2, 5, 37, 3, 8)
    q = np.zeros((2, 5, 3, 8))
    o, lse = ref.attention(q, k, v, 0.125)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=1, keepdims=True), o.shape),
                               rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, math.log(37), rtol=0, atol=1e-14)


def test_dominant_logit_selects_its_value_row():
    r = _rng(2)
    skv, d, jstar = 50, 16, 17
    k = r.standard_normal((1, skv, 1, d))
    k[0, :, 0, 0] = 0.0
    k[0, jstar, 0, 0] = 10.0
    v = r.standard_normal((1, skv, 1, d))
    q = np.zeros((1, 1, 1, d))
    q[0, 0, 0, 0] = 20.0  # with scale 1/4: s_j* = 50, every other s_j = 0
    o, lse = ref.attention(q, k, v, 0.25)
    # exact: o = (e^50 v* + sum_{j != j*} v_j) / (e^50 + 49); error below 50 e^-50
    np.testing.assert_allclose(o[0, 0, 0], v[0, jstar, 0], rtol=0, atol=1e-19 * 50)
    assert abs(lse[0, 0, 0] - 50.0) < 1e-19 * 50 + 1e-14


def test_key_permutation_invariance():
    q, k, v = _rand(3, 1, 9, 41, 2, 6)
    perm = _rng(4).permutation(41)
    o1, l1 = ref.attention(q, k, v, 0.3)
    o2, l2 = ref.attention(q, k[:, perm], v[:, perm], 0.3)
    np.testing.assert_allclose(o1, o2, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(l1, l2, rtol=1e-14, atol=1e-14)


def test_duplicated_keys_add_ln2():
    q, k, v = _rand(5, 2, 6, 13, 2, 4)
    o1, l1 = ref.attention(q, k, v, 0.7)
    o2, l2 = ref.attention(q, np.concatenate([k, k], 1), np.concatenate([v, v], 1), 0.7)
    np.testing.assert_allclose(o2, o1, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(l2, l1 + math.log(2.0), rtol=0, atol=1e-13)


def test_single_key():
    q, k, v = _rand(6, 1, 4, 1, 3, 5)
    o, lse = ref.attention(q, k, v, 0.9)
    np.testing.assert_array_equal(o, np.broadcast_to(v, o.shape))
    for h in range(3):
        np.testing.assert_allclose(lse[0, h], 0.9 * q[0, :, h] @ k[0, 0, h], rtol=0, atol=1e-14)


def test_ones_value_gives_ones():
    q, k, _ = _rand(7, 1, 5, 29, 2, 8, sigma=3.0)
    o, _ = ref.attention(q, k, np.ones((1, 29, 2, 8)), 1.0 / math.sqrt(8))
    np.testing.assert_allclose(o, 1.0, rtol=0, atol=1e-14)


def test_empty_key_set():
    q = np.ones((1, 3, 2, 4))
    o, lse = ref.attention(q, np.zeros((1, 0, 2, 4)), np.zeros((1, 0, 2, 4)), 0.5)
    assert np.all(o == 0) and np.all(np.isneginf(lse))


@pytest.mark.parametrize("shape", [(1, 1, 1, 1, 1), (2, 5, 7, 2, 3), (1, 9, 4, 3, 16),
                                   (2, 17, 33, 2, 8), (1, 33, 17, 1, 16)])
def test_brute_force_agrees(shape):
    b, sq, skv, h, d = shape
    q, k, v = _rand(sum(shape), b, sq, skv, h, d, sigma=2.0)
    scale = 1.0 / math.sqrt(d)
    o, lse = ref.attention(q, k, v, scale)
    ob, lb = brute.attention(q, k, v, scale)
    np.testing.assert_allclose(o, np.asarray(ob), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, np.asarray(lb), rtol=1e-13, atol=1e-13)


def test_large_logits_stay_finite():
    # sigma 3 Q and K at D=128: logits of std 9 (up to ~50); LSE matches scipy
    q, k, v = _rand(8, 1, 64, 300, 1, 128, sigma=3.0)
    scale = 1.0 / math.sqrt(128)
    o, lse = ref.attention(q, k, v, scale)
    s = scale * q[0, :, 0] @ k[0, :, 0].T
    np.testing.assert_allclose(lse[0, 0], scipy.special.logsumexp(s, axis=1), rtol=1e-14)
    assert np.isfinite(o).all()


def test_row_sampling_matches_full():
    q, k, v = _rand(9, 2, 40, 31, 3, 8)
    o, lse = ref.attention(q, k, v, 0.2)
    rows = [(0, 0, 0), (1, 2, 39), (0, 1, 17), (1, 0, 3), (1, 0, 4)]
    orr, lr = ref.attention_rows(q, k, v, 0.2, rows)
    for n, (b, h, i) in enumerate(rows):
        # BLAS may block a 2-row product differently from a 40-row one: rounding only
        np.testing.assert_allclose(orr[n], o[b, i, h], rtol=1e-13, atol=1e-15)
        assert abs(lr[n] - lse[b, h, i]) < 1e-14


# ----------------------------------------------------------------------------- merge


def _split_points(skv, r):
    cuts = sorted(r.integers(0, skv + 1, size=r.integers(1, 5)))
    return [0] + list(cuts) + [skv]


@pytest.mark.parametrize("seed", range(6))
def test_chunked_merge_equals_unchunked(seed):
    r = _rng(20 + seed)
    skv = int(r.integers(1, 60))
    q, k, v = _rand(30 + seed, 2, 7, skv, 2, 5, sigma=1.5)
    cuts = _split_points(skv, r)
    if seed == 0:
        cuts = [0, 0, 1, skv, skv]  # empty, size-1, rest, empty
    parts = [ref.attention(q, k[:, a:b], v[:, a:b], 0.4) for a, b in zip(cuts, cuts[1:])]
    o, lse = ref.merge_chunks(parts)
    o_full, l_full = ref.attention(q, k, v, 0.4)
    np.testing.assert_allclose(o, o_full, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, l_full, rtol=1e-13, atol=1e-12)


def test_merge_matches_brute_partials():
    q, k, v = _rand(40, 1, 4, 10, 2, 3)
    pa = [np.asarray(x) for x in brute.attention(q, k[:, :6], v[:, :6], 0.5)]
    pb = [np.asarray(x) for x in brute.attention(q, k[:, 6:], v[:, 6:], 0.5)]
    o, lse = ref.merge(pa[0], pa[1], pb[0], pb[1])
    ob, lb = brute.attention(q, k, v, 0.5)
    np.testing.assert_allclose(o, np.asarray(ob), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, np.asarray(lb), rtol=1e-13, atol=1e-13)


def test_merge_with_empty_is_identity_and_both_empty_is_zero():
    q, k, v = _rand(41, 1, 3, 5, 2, 4)
    o, lse = ref.attention(q, k, v, 0.5)
    oe, le = ref.attention(q, k[:, :0], v[:, :0], 0.5)
    for a, b in (((o, lse), (oe, le)), ((oe, le), (o, lse))):
        om, lm = ref.merge(a[0], a[1], b[0], b[1])
        np.testing.assert_array_equal(om, o)
        np.testing.assert_array_equal(lm, lse)
    om, lm = ref.merge(oe, le, oe, le)
    assert np.all(om == 0) and np.all(np.isneginf(lm)) and not np.isnan(om).any()


def test_merge_two_equal_halves_closed_form():
    # two partials with equal LSE L: merged LSE = L + ln 2, O = mean of the two
    r = _rng(42)
    oa, ob = r.standard_normal((1, 3, 2, 4)), r.standard_normal((1, 3, 2, 4))
    la = r.standard_normal((1, 2, 3)) * 10
    o, lse = ref.merge(oa, la, ob, la.copy())
    np.testing.assert_allclose(lse, la + math.log(2), rtol=0, atol=1e-13)
    np.testing.assert_allclose(o, 0.5 * (oa + ob), rtol=0, atol=1e-15)


# ----------------------------------------------------------------------------- permutes


def _ulysses_golden():
    with open(os.path.join(GOLDEN, "ulysses_tiny.json")) as f:
        return json.load(f)


def check_permute_golden(seq2head, head2seq):
    g = _ulysses_golden()
    src = np.asarray(g["src"], dtype=np.int64)
    dst = np.asarray(seq2head(src, g["P"]))
    np.testing.assert_array_equal(dst, np.asarray(g["seq2head"]))
    np.testing.assert_array_equal(np.asarray(head2seq(dst, g["P"])), src)


def test_permute_golden_numpy():
    check_permute_golden(ref.seq2head, ref.head2seq)


def test_permute_golden_brute():
    check_permute_golden(brute.seq2head, brute.head2seq)


@pytest.mark.parametrize("shape", [(2, 3, 4, 2), (4, 5, 8, 3), (1, 4, 3, 2), (3, 2, 6, 1)])
def test_permute_numpy_vs_loops_and_round_trip(shape):
    p, s_l, h, d = shape
    src = np.arange(p * s_l * h * d, dtype=np.int64).reshape(shape)
    dst = ref.seq2head(src, p)
    assert dst.shape == (p, p * s_l, h // p, d)
    np.testing.assert_array_equal(dst, np.asarray(brute.seq2head(src, p)))
    np.testing.assert_array_equal(ref.head2seq(dst, p), src)
    np.testing.assert_array_equal(np.asarray(brute.head2seq(dst, p)), src)
    # the other composition is the identity on the head-grouped layout too
    other = np.arange(dst.size, dtype=np.int64).reshape(dst.shape) * 7
    np.testing.assert_array_equal(ref.seq2head(ref.head2seq(other, p), p), other)
    # a permutation: every element appears exactly once
    assert np.array_equal(np.sort(dst.ravel()), np.sort(src.ravel()))


def test_permute_p1_is_identity():
    src = np.arange(5 * 3 * 2, dtype=np.int64).reshape(1, 5, 3, 2)
    np.testing.assert_array_equal(ref.seq2head(src, 1), src)
    np.testing.assert_array_equal(ref.head2seq(src, 1), src)


def test_ulysses_equals_single_device_attention():
    # the claim of the DeepSpeed Ulysses section: per-head attention over the full
    # sequence, computed by head groups and re-sharded, equals plain attention over the
    # concatenation of the rank shards
    p, s_l, h, d = 4, 6, 8, 5
    r = _rng(50)
    qs, ks, vs = (r.standard_normal((p, s_l, h, d)) for _ in range(3))
    o_u, lse_u = ref.ulysses_attention(qs, ks, vs, p, 0.45)
    full = lambda x: x.reshape(1, p * s_l, h, d)  # shards concatenated in rank order
    o_f, lse_f = ref.attention(full(qs), full(ks), full(vs), 0.45)
    np.testing.assert_allclose(o_u.reshape(1, p * s_l, h, d), o_f, rtol=1e-12, atol=1e-13)
    hp = h // p
    for g in range(p):
        for j in range(hp):
            np.testing.assert_allclose(lse_u[g, j], lse_f[0, g * hp + j], rtol=0, atol=1e-13)


# ----------------------------------------------------------------------------- planted mistakes


def _mutant_head(mistake):
    def head(q, k, v, scale):
        sq = q.shape[0]
        if k.shape[0] == 0:
            return np.zeros((sq, v.shape[1])), np.full(sq, -np.inf)
        s = (q @ k.T) * (1.0 if mistake == "no_scale" else scale)
        if mistake == "scale_sqrt":
            s = (q @ k.T) * math.sqrt(scale)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        l = e.sum(axis=1, keepdims=True)
        lse = (m + np.log(l))[:, 0]
        if mistake == "lse_log2":
            lse = (m / math.log(2) + np.log2(l))[:, 0]
        if mistake == "lse_no_max":
            lse = np.log(l)[:, 0]
        o = (e @ v) / l
        if mistake == "no_normalise":
            o = e @ v
        if mistake == "v_transposed" and v.shape[0] == v.shape[1]:
            o = (e @ v.T) / l
        if mistake == "k_for_v":
            o = (e @ k) / l
        if mistake == "max_not_subtracted_in_o":
            o = (np.exp(s) @ v) / l
        return o, lse

    return head


@pytest.mark.parametrize("mistake", ["no_scale", "scale_sqrt", "lse_log2", "lse_no_max",
                                     "no_normalise", "v_transposed", "k_for_v",
                                     "max_not_subtracted_in_o"])
def test_planted_attention_mistake_is_caught(monkeypatch, mistake):
    monkeypatch.setattr(ref, "_attention_head", _mutant_head(mistake))
    caught = 0
    for pin in (lambda: check_golden(ref.attention), lambda: check_softmax_identity(ref.attention),
                lambda: test_brute_force_agrees((2, 5, 7, 2, 3)),
                lambda: test_brute_force_agrees((1, 9, 4, 3, 16))):
        try:
            pin()
        except AssertionError:
            caught += 1
    assert caught >= 1, f"no pin caught the planted mistake {mistake!r}"


def test_planted_head_mixup_is_caught(monkeypatch):
    orig = ref.attention

    def mixed(q, k, v, scale):  # keys of the next head: a plausible indexing slip
        return orig(q, np.roll(np.asarray(k, dtype=np.float64), 1, axis=2), v, scale)

    with pytest.raises(AssertionError):
        check_golden(mixed)


@pytest.mark.parametrize("mistake", ["swap_weights", "no_max_in_lse", "ln2_base"])
def test_planted_merge_mistake_is_caught(monkeypatch, mistake):
    def bad_merge(o_a, lse_a, o_b, lse_b):
        o_a, o_b, la, lb = (np.asarray(x, dtype=np.float64) for x in (o_a, o_b, lse_a, lse_b))
        mx = np.maximum(la, lb)
        ea, eb = np.exp(la - mx), np.exp(lb - mx)
        lse = mx + np.log(ea + eb)
        if mistake == "no_max_in_lse":
            lse = np.log(ea + eb)
        if mistake == "ln2_base":
            lse = mx + np.log2(ea + eb)
        wa, wb = ea / (ea + eb), eb / (ea + eb)
        if mistake == "swap_weights":
            wa, wb = wb, wa
        t = lambda w: np.transpose(w, (0, 2, 1))[..., None]
        return t(wa) * o_a + t(wb) * o_b, lse

    monkeypatch.setattr(ref, "merge", bad_merge)
    with pytest.raises(AssertionError):
        for seed in range(1, 6):
            test_chunked_merge_equals_unchunked(seed)


@pytest.mark.parametrize("mistake", ["strided_groups", "reversed_ranks", "token_major_swap"])
def test_planted_permute_mistake_is_caught(mistake):
    def bad_seq2head(src, p):
        src = np.asarray(src)
        pp, s_l, h, d = src.shape
        hp = h // p
        if mistake == "strided_groups":  # heads g, g+P, ... instead of a contiguous block
            x = src.reshape(p, s_l, hp, p, d).transpose(3, 0, 1, 2, 4)
        elif mistake == "reversed_ranks":
            x = src[::-1].reshape(p, s_l, p, hp, d).transpose(2, 0, 1, 3, 4)
        else:  # sequence order inside the group taken as (s, r) instead of (r, s)
            x = src.reshape(p, s_l, p, hp, d).transpose(2, 1, 0, 3, 4)
        return np.ascontiguousarray(x.reshape(p, p * s_l, hp, d))

    with pytest.raises(AssertionError):
        check_permute_golden(bad_seq2head, ref.head2seq)


# ----------------------------------------------------------------------------- ring attention


def check_ring_attention(ring_attention, seed):
    """ring_attention over any split of the keys into chunks (empty, size-1, uneven) equals
    attention over the concatenated chunks: against the loop-only brute force (independent
    of ref.attention) and, for the closed form, a chunk repeated gives LSE + ln 2."""
    r = _rng(60 + seed)
    skv = int(r.integers(2, 24))
    q, k, v = _rand(70 + seed, 1, 5, skv, 2, 3, sigma=1.3)
    cuts = _split_points(skv, r)
    if seed == 0:
        cuts = [0, 1, 1, skv - 1, skv]  # size-1, empty, the bulk, size-1 tail
    kc = [k[:, a:b] for a, b in zip(cuts, cuts[1:])]
    vc = [v[:, a:b] for a, b in zip(cuts, cuts[1:])]
    o, lse = ring_attention(q, kc, vc, 0.45)
    ob, lb = brute.attention(q, k, v, 0.45)
    np.testing.assert_allclose(o, np.asarray(ob), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, np.asarray(lb), rtol=1e-13, atol=1e-13)
    # every chunk twice: the key multiset doubles, so O is unchanged and LSE gains ln 2
    o2, l2 = ring_attention(q, kc + kc, vc + vc, 0.45)
    np.testing.assert_allclose(o2, np.asarray(ob), rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(l2, np.asarray(lb) + math.log(2), rtol=1e-13, atol=1e-13)


@pytest.mark.parametrize("seed", range(5))
def test_ring_attention_equals_attention_over_concatenated_chunks(seed):
    check_ring_attention(ref.ring_attention, seed)


@pytest.mark.parametrize("mistake", ["drop_last_chunk", "kv_misaligned", "first_chunk_twice",
                                     "unmerged_last"])
def test_planted_ring_attention_mistake_is_caught(mistake):
    def bad_ring(q, k_chunks, v_chunks, scale):
        kc, vc = list(k_chunks), list(v_chunks)
        if mistake == "drop_last_chunk":  # an off-by-one in the ring loop
            kc, vc = kc[:-1], vc[:-1]
        elif mistake == "kv_misaligned":  # V of the previous chunk paired with K
            vc = vc[-1:] + vc[:-1]
        elif mistake == "first_chunk_twice":
            kc, vc = kc[:1] + kc, vc[:1] + vc
        parts = [ref.attention(q, a, b, scale) for a, b in zip(kc, vc)]
        if mistake == "unmerged_last":  # the last partial overwrites the running result
            return parts[-1]
        return ref.merge_chunks(parts)

    caught = 0
    for seed in range(5):
        try:
            check_ring_attention(bad_ring, seed)
        except AssertionError:
            caught += 1
    assert caught >= 1, f"no pin caught the planted mistake {mistake!r}"
