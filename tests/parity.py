"""Shared comparison rules for GPU-vs-oracle parity tests.

Tolerances (stated for this path): fp32 inputs -> max |O err| <= 1e-5; bf16 inputs ->
max |O err| <= 1e-2 and mean |O err| <= 1e-3 against the fp64 oracle on the same
bf16-rounded inputs, |LSE err| <= 1e-3.  A bf16 *output* cannot meet an absolute 1e-2
once |O| >= 4 (half an ulp there is 2^-6 = 0.0156), so a bf16 O is held to
1e-2 + half an ulp of bf16 at the reference value; the unrounded (fp32-epilogue) O of the
same kernel is held to the plain 1e-2 / 1e-3 bar.
"""

import numpy as np
import torch

F32_MAX_ERR = 1e-5
BF16_MAX_ERR = 1e-2
BF16_MEAN_ERR = 1e-3
LSE_ERR = 1e-3


def to64(t):
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu()
        if t.dtype not in (torch.float32, torch.float64):
            t = t.float()
        return t.double().numpy()
    return np.asarray(t, dtype=np.float64)


def half_ulp_bf16(x):
    """Half the bf16 spacing at |x| (bf16 keeps 8 significant bits)."""
    _, e = np.frexp(np.abs(x))  # |x| = m * 2^e, m in [0.5, 1)
    return np.where(x == 0, 0.0, np.ldexp(1.0, e - 9))


def check_o(o_gpu, o_ref, kind, what=""):
    o_gpu, o_ref = to64(o_gpu), to64(o_ref)
    assert o_gpu.shape == o_ref.shape, (o_gpu.shape, o_ref.shape)
    assert np.isfinite(o_gpu).all(), f"{what}: non-finite output"
    err = np.abs(o_gpu - o_ref)
    if kind == "f32":
        assert err.max() <= F32_MAX_ERR, f"{what}: max err {err.max():.3e}"
        return err
    bound = BF16_MAX_ERR + (half_ulp_bf16(o_ref) if kind == "bf16_out" else 0.0)
    worst = np.argmax(err - bound)
    assert (err <= bound).all(), (
        f"{what}: err {err.flat[worst]:.3e} > bound {np.broadcast_to(bound, err.shape).flat[worst]:.3e}"
        f" at {np.unravel_index(worst, err.shape)} (ref {o_ref.flat[worst]:.4f})")
    assert err.mean() <= BF16_MEAN_ERR, f"{what}: mean err {err.mean():.3e}"
    return err


def check_lse(l_gpu, l_ref, what="", tol=LSE_ERR):
    l_gpu, l_ref = to64(l_gpu), to64(l_ref)
    assert l_gpu.shape == l_ref.shape
    both_inf = np.isneginf(l_gpu) & np.isneginf(l_ref)
    err = np.where(both_inf, 0.0, np.abs(l_gpu - l_ref))
    assert err.max() <= tol, f"{what}: LSE max err {err.max():.3e}"
    return err


def rel_l2(o_gpu, o_ref):
    a, b = to64(o_gpu), to64(o_ref)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))
