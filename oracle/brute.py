"""Loop-only brute force for tiny sizes (test infrastructure).

Pure Python: nested loops, ``math.fsum`` for every sum and ``math.exp`` / ``math.log``.
It shares nothing with ``oracle.ref`` except the definitions it restates (the
softmax(QK^T)V core of the attention_mdtrt guide, 模型的核心结构, and the Ulysses
re-partition of the TensorRT multi-device blog, Fig. 4), so the two can pin each
other.  Inputs are nested lists or arrays indexed ``[b][s][h][d]``.
"""

from __future__ import annotations

import math


def attention(q, k, v, scale):
    """Returns (O [B][Sq][H][D], LSE [B][H][Sq]) as nested lists of floats."""
    bn, sq, hn, dn = len(q), len(q[0]), len(q[0][0]), len(q[0][0][0])
    skv = len(k[0])
    dv = len(v[0][0][0]) if skv else dn
    o = [[[[0.0] * dv for _ in range(hn)] for _ in range(sq)] for _ in range(bn)]
    lse = [[[0.0] * sq for _ in range(hn)] for _ in range(bn)]
    for b in range(bn):
        for h in range(hn):
            for i in range(sq):
                if skv == 0:
                    lse[b][h][i] = -math.inf
                    continue
                s = [
                    scale * math.fsum(float(q[b][i][h][d]) * float(k[b][j][h][d]) for d in range(dn))
                    for j in range(skv)
                ]
                mx = max(s)
                tot = math.fsum(math.exp(x - mx) for x in s)
                l = mx + math.log(tot)
                lse[b][h][i] = l
                for d in range(dv):
                    o[b][i][h][d] = math.fsum(
                        math.exp(s[j] - l) * float(v[b][j][h][d]) for j in range(skv)
                    )
    return o, lse


def seq2head(src, p):
    """dst[g][r*S_l+s][j][d] = src[r][s][g*Hp+j][d], by explicit loops."""
    s_l, h, d = len(src[0]), len(src[0][0]), len(src[0][0][0])
    hp = h // p
    dst = [[[[None] * d for _ in range(hp)] for _ in range(p * s_l)] for _ in range(p)]
    for r in range(p):
        for s in range(s_l):
            for g in range(p):
                for j in range(hp):
                    for e in range(d):
                        dst[g][r * s_l + s][j][e] = src[r][s][g * hp + j][e]
    return dst


def head2seq(src, p):
    """dst[r][s][g*Hp+j][d] = src[g][r*S_l+s][j][d], by explicit loops."""
    s_full, hp, d = len(src[0]), len(src[0][0]), len(src[0][0][0])
    s_l = s_full // p
    dst = [[[[None] * d for _ in range(p * hp)] for _ in range(s_l)] for _ in range(p)]
    for g in range(p):
        for r in range(p):
            for s in range(s_l):
                for j in range(hp):
                    for e in range(d):
                        dst[r][s][g * hp + j][e] = src[g][r * s_l + s][j][e]
    return dst


def rmsnorm_heads(x, gamma, eps=1e-6, out_scale=1.0):
    """The attention_mdtrt sample's Q/K RMSNorm (模型的核心结构) by explicit loops in
    float64: y[..][d] = x[..][d] / sqrt(fsum(x^2) / D + eps) * gamma[d] * out_scale.
    ``x`` is a nested list whose innermost lists are head rows of length D."""
    if hasattr(x[0], "__len__"):  # not yet at a head row: recurse
        return [rmsnorm_heads(sub, gamma, eps, out_scale) for sub in x]
    row = [float(t) for t in x]
    dn = len(row)
    rms = math.sqrt(math.fsum(t * t for t in row) / dn + eps)
    return [row[d] / rms * float(gamma[d]) * out_scale for d in range(dn)]
