"""The FMA-pipe 2^t used for part of the softmax exponentials: its coefficients are the
ones csrc/gen_exp2_poly.py derives (constrained minimax), and the algorithm, emulated in
float32 on the CPU, meets the stated relative error bound (no GPU)."""

import os
import re
import subprocess
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "context_long_sequence_non_b200", "csrc")


def _kernel_coefficients():
    with open(os.path.join(CSRC, "sm100_ptx.cuh")) as f:
        src = f.read()
    m = re.search(r"kC1 = ([0-9.eE+-]+)f, kC2 = ([0-9.eE+-]+)f, kC3 = ([0-9.eE+-]+)f", src)
    return np.array([float(x) for x in m.groups()], dtype=np.float32)


def test_coefficients_match_the_generator():
    out = subprocess.run([sys.executable, os.path.join(CSRC, "gen_exp2_poly.py")],
                         capture_output=True, text=True, check=True).stdout
    gen = np.array([float(x) for x in re.findall(r"c\d = ([0-9.eE+-]+)f", out)], dtype=np.float32)
    np.testing.assert_array_equal(gen, _kernel_coefficients())


def emulate(t):
    """float32 restatement of exp2_poly2: clamp, 1.5*2^23 shifter, Horner, exponent add."""
    c1, c2, c3 = _kernel_coefficients()
    f32 = np.float32
    t = np.maximum(t.astype(f32), f32(-125.0))
    shift = f32(12582912.0)
    j = (t + shift).astype(f32)
    n = (j - shift).astype(f32)
    f = (t - n).astype(f32)
    p = (f * c3 + c2).astype(f32)
    p = (p * f + c1).astype(f32)
    p = (p * f + f32(1.0)).astype(f32)
    bits = (p.view(np.uint32) + (j.view(np.uint32) << np.uint32(23))).astype(np.uint32)
    return bits.view(f32)


def test_emulated_polynomial_meets_bound():
    # the softmax's exponents lie in [-125, 8]: up to the 2^8 headroom of its reference max
    t = np.concatenate([np.linspace(-125, 8, 2_000_001, dtype=np.float32),
                        -np.abs(np.random.default_rng(0).standard_normal(100000).astype(np.float32)) * 20])
    out = emulate(t).astype(np.float64)
    rel = np.abs(out / np.exp2(t.astype(np.float64)) - 1)
    assert rel.max() <= 1.05e-4, rel.max()
    assert emulate(np.array([0.0], dtype=np.float32))[0] == 1.0
    assert emulate(np.array([-np.inf], dtype=np.float32))[0] == np.float32(2.0 ** -125)
