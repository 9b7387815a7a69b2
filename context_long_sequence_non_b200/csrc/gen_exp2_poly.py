"""Derives the polynomial the attention kernel uses for part of its 2^t evaluations.

Method (Cody-Waite range reduction followed by a polynomial): for t <= 0 split
t = n + f with n = round(t) and f in [-1/2, 1/2]; then 2^t = 2^n * 2^f, where 2^n is an
exponent-field add and 2^f ~= 1 + c1 f + c2 f^2 + c3 f^3.  The constant term is pinned to
1 so that t = 0 (the key holding the row maximum) gives exactly 1.  c1..c3 minimise the
maximum *relative* error over f in [-1/2, 1/2] (a linear program over a dense grid: the
discrete minimax fit), then are rounded to float32 and the error is re-measured with
float32 Horner arithmetic.

Run: ``python gen_exp2_poly.py`` -- prints the coefficients (decimal and hex) and the
measured relative error bound; the kernel's constants are copied from this output.
"""

from __future__ import annotations

import numpy as np
from scipy.optimize import linprog


def fit(degree: int = 3, n_grid: int = 4001):
    f = np.linspace(-0.5, 0.5, n_grid)
    target = np.exp2(f)
    # relative error r(f) = (1 + sum_k c_k f^k - 2^f) / 2^f; minimise t with |r| <= t
    cols = [f ** k / target for k in range(1, degree + 1)]
    A = np.stack(cols, axis=1)
    b = (target - 1.0) / target
    n = degree
    # variables: c_1..c_n, t ; minimise t
    c_obj = np.zeros(n + 1)
    c_obj[-1] = 1.0
    A_ub = np.block([[A, -np.ones((len(f), 1))], [-A, -np.ones((len(f), 1))]])
    b_ub = np.concatenate([b, -b])
    res = linprog(c_obj, A_ub=A_ub, b_ub=b_ub, bounds=[(None, None)] * n + [(0, None)],
                  method="highs")
    assert res.success, res.message
    return res.x[:n], res.x[-1]


def horner_f32(coef32, f32):
    acc = np.full_like(f32, coef32[-1])
    for c in coef32[-2::-1]:
        acc = np.float32(acc * f32 + c).astype(np.float32)
    return np.float32(acc * f32 + np.float32(1.0)).astype(np.float32)


def main():
    coef, t = fit()
    c32 = np.asarray(coef, dtype=np.float32)
    f = np.linspace(-0.5, 0.5, 200001, dtype=np.float32)
    p = horner_f32(c32, f)
    rel = np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1.0)
    print(f"LP minimax relative error (real coefficients): {t:.3e}")
    print(f"float32 Horner, float32 coefficients: max relative error {rel.max():.3e}")
    for k, c in enumerate(c32, start=1):
        print(f"c{k} = {float(c):.9g}f  (0x{c.view(np.uint32):08x})")


if __name__ == "__main__":
    main()
