"""GPU test of cpattn_fwd_split_noalloc, the split-KV entry point for callers that cannot
allocate device memory (its partials live in a fixed scratch array inside the library).

Called through the C ABI with ctypes and checked against cpattn_fwd_split given a
caller-allocated workspace, on two calls in a row: a plain pass, then an accumulating pass
that reuses the scratch the first call left behind.  Both entry points run the same
kernels on the same data with the same partial layout, so their results must be identical
bit for bit.  After a warm-up call, a further call must leave the device's free memory
unchanged (it allocates nothing).  Collected last so that a run stopping at the first
failure has already run every other test; it also passes on its own.
"""

import ctypes
import math

import pytest
import torch

pytestmark = pytest.mark.gpu

BF16, F32 = 0, 1
OK, ERR_SHAPE = 0, 2


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from context_long_sequence_non_b200 import build as build_mod

    build_mod.build()
    L = ctypes.CDLL(build_mod.LIB)
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    L.cpattn_fwd_split_noalloc.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, i, vp]
    L.cpattn_fwd_split_noalloc.restype = i
    L.cpattn_fwd_split.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, i, vp,
                                   ctypes.c_size_t, vp]
    L.cpattn_fwd_split.restype = i
    L.cpattn_fwd_split_workspace.argtypes = [i, i, i, i, i, i]
    L.cpattn_fwd_split_workspace.restype = ctypes.c_size_t
    L.cpattn_fwd_split_workspace_kv.argtypes = [i, i, i, i, i, i, i]
    L.cpattn_fwd_split_workspace_kv.restype = ctypes.c_size_t
    L.cpattn_noalloc_scratch_bytes.argtypes = []
    L.cpattn_noalloc_scratch_bytes.restype = ctypes.c_size_t
    L.cpattn_device_error.argtypes = []
    L.cpattn_device_error.restype = i
    return L


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


# (B, H, Sq, Skv, D, n_split requested, n_split the call uses)
CASES = [
    (1, 8, 300, 5000, 128, 4, 4),
    (2, 3, 257, 1300, 64, 3, 3),  # D = 64, ragged query tail
    # 8 ranges over 256 keys would need 65 MiB of partials; the call lowers the split to
    # the two 128-key blocks there are, and two ranges fit in the scratch
    (1, 8, 4096, 256, 128, 8, 2),
    # n_split = 0: only the items of the last, partial wave of CTAs are split (352 items on
    # 148 SMs leave 56, each computed as two key ranges)
    (1, 16, 5520, 2000, 128, 0, 0),
]


@pytest.mark.parametrize("case", CASES)
@pytest.mark.parametrize("out_dtype", [torch.bfloat16, torch.float32])
def test_noalloc_matches_workspace_entry_point(lib, case, out_dtype):
    B, H, Sq, Skv, D, n_split, n_used = case
    dt = BF16 if out_dtype == torch.bfloat16 else F32
    g = torch.Generator().manual_seed(123 + Sq)
    q, k, v = (torch.randn(B, s, H, D, generator=g).to(torch.bfloat16).cuda()
               for s in (Sq, Skv, Skv))
    k2, v2 = (torch.randn(B, Skv, H, D, generator=g).to(torch.bfloat16).cuda() for _ in range(2))
    scale = 1.0 / math.sqrt(D)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    need = lib.cpattn_fwd_split_workspace_kv(B, H, Sq, Skv, D, n_split, dt)  # exact
    assert 0 < need <= lib.cpattn_noalloc_scratch_bytes()
    assert need == lib.cpattn_fwd_split_workspace_kv(B, H, Sq, Skv, D, n_used, dt)
    if n_used != n_split:  # the unlowered request alone would not fit
        assert lib.cpattn_fwd_split_workspace(B, H, Sq, D, n_split, dt) > \
            lib.cpattn_noalloc_scratch_bytes()
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")

    o_ref = torch.empty(B, Sq, H, D, dtype=out_dtype, device="cuda")
    l_ref = torch.empty(B, H, Sq, device="cuda")
    o_na, l_na = torch.empty_like(o_ref), torch.empty_like(l_ref)
    for call, (kk, vv, acc) in enumerate(((k, v, 0), (k2, v2, 1))):
        # call 1: a plain pass; call 2: folds a second key set into the first call's result,
        # reading and rewriting (o, lse) while reusing the scratch call 1 left behind
        st = lib.cpattn_fwd_split(_p(q), _p(kk), _p(vv), _p(o_ref), _p(l_ref), B, H, Sq, Skv, D,
                                  scale, dt, acc, n_split, _p(ws), need, stream)
        assert st == OK, st
        st = lib.cpattn_fwd_split_noalloc(_p(q), _p(kk), _p(vv), _p(o_na), _p(l_na), B, H, Sq,
                                          Skv, D, scale, dt, acc, n_split, stream)
        assert st == OK, st
        torch.cuda.synchronize()
        # the same kernels on the same data and the same partial layout: identical bits
        assert torch.equal(o_na, o_ref), call
        assert torch.equal(l_na, l_ref), call
        assert torch.isfinite(o_na.float()).all() and torch.isfinite(l_na).all()
    assert lib.cpattn_device_error() == OK


def test_noalloc_call_allocates_nothing(lib):
    B, H, Sq, Skv, D, n_split = 1, 4, 500, 3000, 128, 4
    g = torch.Generator().manual_seed(5)
    q, k, v = (torch.randn(B, s, H, D, generator=g).to(torch.bfloat16).cuda()
               for s in (Sq, Skv, Skv))
    o = torch.empty(B, Sq, H, D, dtype=torch.bfloat16, device="cuda")
    l = torch.empty(B, H, Sq, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    args = (_p(q), _p(k), _p(v), _p(o), _p(l), B, H, Sq, Skv, D, 1.0 / math.sqrt(D), BF16, 0,
            n_split, stream)
    assert lib.cpattn_fwd_split_noalloc(*args) == OK  # warm-up: the first call on a device
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        assert lib.cpattn_fwd_split_noalloc(*args) == OK
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0, (free0, free1)
    assert lib.cpattn_device_error() == OK


def test_noalloc_refuses_requests_beyond_its_scratch(lib):
    # eight key ranges of a [1][44160][16][128] query would need ~720 MB of partials
    B, H, Sq, Skv, D = 1, 16, 44160, 44160, 128
    assert lib.cpattn_fwd_split_workspace(B, H, Sq, D, 8, BF16) > lib.cpattn_noalloc_scratch_bytes()
    fake = ctypes.c_void_p(0x10000)
    st = lib.cpattn_fwd_split_noalloc(fake, fake, fake, fake, fake, B, H, Sq, Skv, D, 0.1, BF16,
                                      0, 8, None)
    assert st == ERR_SHAPE
