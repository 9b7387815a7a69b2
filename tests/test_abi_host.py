"""Host-only checks of the C ABI (no GPU): the library builds and loads, exports every
symbol include/cpattn.h declares, and rejects bad arguments before any CUDA call."""

import ctypes
import os
import re

import pytest

from context_long_sequence_non_b200 import _binding as B
from context_long_sequence_non_b200 import build as build_mod

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    build_mod.build()
    return B.lib()


def _declared():
    names = []
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            with open(os.path.join(ROOT, "include", fn)) as f:
                names += re.findall(r"CPATTN_API\s+[\w\s\*]+?\b(cpattn_\w+)\s*\(", f.read())
    return names


def test_every_declared_symbol_is_exported(L):
    names = _declared()
    assert {"cpattn_fwd", "cpattn_merge", "cpattn_seq2head", "cpattn_head2seq",
            "cpattn_status_str", "cpattn_device_error"} <= set(names)
    for n in names:
        assert hasattr(L, n), n


def test_version_and_status_strings(L):
    assert B.version() >> 16 == 1
    for s in range(7):
        assert B.status_str(s).startswith("CPATTN")
    assert "unknown" in B.status_str(99)


FAKE = 0x10000  # 16-byte aligned, never dereferenced: every call below fails validation


def fwd(L, q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B_=1, H=2, Sq=8, Skv=8, D=128, scale=0.1,
        din=0, dout=0):
    vp = ctypes.c_void_p
    return L.cpattn_fwd(vp(q) if q else None, vp(k) if k else None, vp(v) if v else None,
                        vp(o) if o else None, vp(lse) if lse else None, B_, H, Sq, Skv, D,
                        scale, din, dout, None)


def test_fwd_argument_errors(L):
    assert fwd(L, Sq=0) == B.ERR_SHAPE
    assert fwd(L, Skv=-1) == B.ERR_SHAPE
    assert fwd(L, D=0) == B.ERR_SHAPE
    assert fwd(L, scale=0.0) == B.ERR_SHAPE
    assert fwd(L, scale=-1.0) == B.ERR_SHAPE
    assert fwd(L, scale=float("inf")) == B.ERR_SHAPE
    assert fwd(L, din=7) == B.ERR_UNSUPPORTED
    assert fwd(L, q=0) == B.ERR_NULL
    assert fwd(L, o=0) == B.ERR_NULL
    assert fwd(L, k=0) == B.ERR_NULL
    assert fwd(L, q=FAKE + 8) == B.ERR_ALIGN
    assert fwd(L, v=FAKE + 2) == B.ERR_ALIGN
    assert fwd(L, lse=FAKE + 2) == B.ERR_ALIGN
    assert fwd(L, D=96) == B.ERR_UNSUPPORTED  # bf16 tensor-core kernel: D in {64, 128}
    assert fwd(L, D=264, din=1, dout=1) == B.ERR_UNSUPPORTED  # fp32 kernel: D <= 256
    assert fwd(L, B_=70000) == B.ERR_SHAPE


def test_fwd_accumulate_argument_errors(L):
    vp = ctypes.c_void_p

    def acc(lse=FAKE, din=0, dout=0, D=128):
        return L.cpattn_fwd_accumulate(vp(FAKE), vp(FAKE), vp(FAKE), vp(FAKE),
                                       vp(lse) if lse else None, 1, 2, 8, 8, D, 0.1, din, dout,
                                       None)

    assert acc(lse=0) == B.ERR_NULL  # the running LSE is required
    assert acc(din=1, dout=1) == B.ERR_UNSUPPORTED  # tensor-core path only
    assert acc(D=96) == B.ERR_UNSUPPORTED
    assert acc(dout=3) == B.ERR_UNSUPPORTED


def test_ulysses_fwd_argument_errors(L):
    vp = ctypes.c_void_p

    def uf(P=2, S_l=32, H=4, D=128, dout=0, q=FAKE):
        return L.cpattn_ulysses_fwd(vp(q) if q else None, vp(FAKE), vp(FAKE), vp(FAKE), None, P,
                                    S_l, H, D, 0.1, dout, None)

    assert uf(H=5) == B.ERR_SHAPE          # H % P
    assert uf(S_l=24) == B.ERR_UNSUPPORTED  # 16-row boxes would straddle two shards
    assert uf(D=96) == B.ERR_UNSUPPORTED
    assert uf(q=0) == B.ERR_NULL
    assert uf(q=FAKE + 8) == B.ERR_ALIGN


def test_ulysses_fwd_split_plan_and_argument_errors(L):
    vp = ctypes.c_void_p
    # [8][5520][16][128]: 2768 items (8 groups x 2 heads x 173 tile pairs) on 148 SMs leave
    # 104 in the last wave; the makespan model splits them in 4 key ranges each (416 short
    # CTAs, 3 short waves of 1/4 of an item): fp32 rows of 4 * 104 * 256, then their LSEs
    rows = 4 * 104 * 256
    need = L.cpattn_ulysses_fwd_workspace(8, 5520, 16, 128, 0)
    assert need == rows * 128 * 4 + rows * 4
    assert L.cpattn_ulysses_fwd_workspace(8, 5520, 16, 128, 1) == need  # partials are fp32
    assert L.cpattn_ulysses_fwd_workspace(8, 5520, 16, 96, 0) == 0
    assert L.cpattn_ulysses_fwd_workspace(8, 5520, 15, 128, 0) == 0  # H % P
    # one rank of 9472 tokens x 16 heads: 37 tile pairs x 16 = 592 items, 4 whole waves
    assert L.cpattn_ulysses_fwd_workspace(1, 9472, 16, 128, 0) == 0

    def us(ws=FAKE + (1 << 30), ws_bytes=need, q=FAKE, S_l=5520):
        return L.cpattn_ulysses_fwd_split(vp(q) if q else None, vp(FAKE), vp(FAKE), vp(FAKE),
                                          None, 8, S_l, 16, 128, 0.1, 0,
                                          vp(ws) if ws else None, ws_bytes, None)

    assert us(ws=0) == B.ERR_NULL
    assert us(ws=FAKE + (1 << 30) + 16) == B.ERR_ALIGN
    assert us(ws_bytes=need - 1) == B.ERR_SHAPE
    assert us(ws=FAKE) == B.ERR_SHAPE      # overlaps q (and k, v, out at the same address)
    assert us(S_l=5512) == B.ERR_UNSUPPORTED  # S_l % 16
    assert us(q=0) == B.ERR_NULL


def test_ulysses_host_argument_errors(L):
    vp = ctypes.c_void_p
    H0, D0 = 0x7000000, 0x100000000  # fake host and device addresses (never dereferenced)
    step = 0x10000000

    def uh(P=2, S_l=32, H=4, D=128, n=1, hq=H0, hl=H0 + 5 * step, dl=D0 + 4 * step, dq=D0,
           dk=D0 + step, dout=0):
        return L.cpattn_ulysses_host(vp(hq) if hq else None, vp(H0 + step), vp(H0 + 2 * step),
                                     vp(H0 + 3 * step), vp(hl) if hl else None,
                                     vp(dq) if dq else None, vp(dk), vp(D0 + 2 * step),
                                     vp(D0 + 3 * step), vp(dl) if dl else None, P, S_l, H, D,
                                     0.1, dout, n, None)

    assert uh(H=5) == B.ERR_SHAPE
    assert uh(S_l=24) == B.ERR_UNSUPPORTED
    assert uh(n=0) == B.ERR_SHAPE and uh(n=3) == B.ERR_SHAPE  # chunks in 1..P
    assert uh(hq=0) == B.ERR_NULL
    assert uh(dq=0) == B.ERR_NULL
    assert uh(hl=0) == B.ERR_NULL  # h_lse and d_lse go together
    assert uh(dq=D0 + 8) == B.ERR_ALIGN
    assert uh(dk=D0 + 64) == B.ERR_SHAPE  # device buffers overlap
    assert uh(dout=5) == B.ERR_UNSUPPORTED


def test_fwd_split_argument_errors_and_sizes(L):
    vp = ctypes.c_void_p

    def fs(n=2, ws=FAKE, ws_bytes=1 << 30, lse=FAKE, acc=0, D=128):
        return L.cpattn_fwd_split(vp(FAKE), vp(FAKE), vp(FAKE), vp(FAKE), vp(lse) if lse else None,
                                  1, 2, 512, 4096, D, 0.1, 0, acc, n, vp(ws) if ws else None,
                                  ws_bytes, None)

    assert fs(n=9) == B.ERR_SHAPE
    assert fs(n=-1) == B.ERR_SHAPE
    assert fs(n=0, ws_bytes=1000) == B.ERR_SHAPE  # tail split: 4 items split 8 ways
    assert fs(n=0, ws=0) == B.ERR_NULL
    assert fs(ws=0) == B.ERR_NULL
    assert fs(ws=FAKE + 16) == B.ERR_ALIGN  # 256-byte alignment
    assert fs(ws_bytes=1000) == B.ERR_SHAPE  # too small
    assert fs(lse=0, acc=1) == B.ERR_NULL
    assert fs(D=96) == B.ERR_UNSUPPORTED
    need = L.cpattn_fwd_split_workspace(1, 2, 512, 128, 2, 0)
    assert need == 2 * 512 * 2 * 128 * 2 + 2 * 2 * 512 * 4
    assert L.cpattn_fwd_split_workspace(1, 2, 512, 128, 1, 0) == 0
    assert L.cpattn_fwd_split_workspace(1, 2, 512, 128, 9, 0) == 0
    # n_split = 0 (tail split) on 148 SMs: the query does not take the key count, so it
    # sizes the largest plan: the last wave's items in up to 8 ranges, or those and the
    # wave before in up to 4.  352 items of a [5520][16][128] query leave 56 in the last
    # wave: max(56 * 8, (56 + 148) * 4) = 816 tail ranges of 256 fp32 rows, then their LSEs
    rows = 816 * 256
    assert L.cpattn_fwd_split_workspace(1, 16, 5520, 128, 0, 0) == rows * 128 * 4 + rows * 4
    # 2768 items of [8][44160][2][128] leave 104: max(104 * 8, 252 * 4) = 1008 ranges
    rows = 1008 * 256
    assert L.cpattn_fwd_split_workspace(8, 2, 44160, 128, 0, 0) == rows * 128 * 4 + rows * 4
    assert L.cpattn_fwd_split_workspace(1, 16, 9472, 128, 0, 0) == 0  # 592 items: 4 whole waves
    assert L.cpattn_fwd_split_workspace(1, 16, 5520, 96, 0, 0) == 0
    # exact sizes for a key count: the ring chunk (5520 keys) splits its 56 items in 2 (one
    # short wave); the [8][44160][2][128] pass splits the last wave's 104 items in 4
    kv = L.cpattn_fwd_split_workspace_kv
    rows = 2 * 56 * 256
    assert kv(1, 16, 5520, 5520, 128, 0, 0) == rows * 128 * 4 + rows * 4
    rows = 4 * 104 * 256
    assert kv(8, 2, 44160, 44160, 128, 0, 0) == rows * 128 * 4 + rows * 4
    assert kv(1, 20, 3000, 3000, 128, 0, 0) == 0  # 24 key blocks: short ranges do not pay
    assert kv(1, 16, 5520, 300, 128, 0, 0) == 0  # 3 key blocks: ranges of 2 do not pay
    # split-KV: lowered to the key blocks there are, as the call lowers it
    assert kv(1, 8, 4096, 256, 128, 8, 0) == L.cpattn_fwd_split_workspace(1, 8, 4096, 128, 2, 0)
    assert kv(1, 8, 4096, 100, 128, 8, 0) == 0  # one key block: nothing to split
    assert kv(1, 2, 512, 0, 128, 2, 0) == 0


def test_split_suggestion_model():
    assert B.split_suggest(8, 2, 44160, 44160) == 1  # 2768 CTAs: many waves already
    assert B.split_suggest(1, 16, 512, 44160) >= 4   # 32 CTAs over 345 key blocks: split
    assert B.split_suggest(1, 16, 5520, 5520) == 1   # 352 CTAs of 43 blocks: start-up eats it
    assert B.split_suggest(1, 1, 128, 128) == 1       # too few key blocks to split


def test_merge_argument_errors(L):
    vp = ctypes.c_void_p
    base = [vp(FAKE), vp(FAKE + 0x100000), vp(FAKE + 0x200000), vp(FAKE + 0x300000),
            vp(FAKE + 0x400000), vp(FAKE + 0x500000)]

    def merge(ptrs=base, B_=1, H=2, S=4, D=128, dt=0):
        return L.cpattn_merge(*ptrs, B_, H, S, D, dt, None)

    assert merge(S=0) == B.ERR_SHAPE
    assert merge(D=12) == B.ERR_SHAPE  # 24 bytes: not a whole number of 16-byte vectors
    assert merge(D=2056) == B.ERR_SHAPE  # a row longer than 4096 bytes
    assert merge(dt=5) == B.ERR_UNSUPPORTED
    assert merge(ptrs=[None] + base[1:]) == B.ERR_NULL
    assert merge(ptrs=base[:4] + [vp(FAKE + 0x400008)] + base[5:]) == B.ERR_ALIGN
    # o overlapping o_b (not the allowed o == o_a in-place case)
    assert merge(ptrs=base[:4] + [vp(FAKE + 0x200000 + 16)] + base[5:]) == B.ERR_SHAPE


def test_permute_argument_errors(L):
    vp = ctypes.c_void_p
    s, d = vp(FAKE), vp(FAKE + 0x1000000)
    for fn in (L.cpattn_seq2head, L.cpattn_head2seq):
        assert fn(s, d, 3, 4, 16, 128, 2, None) == B.ERR_SHAPE  # H % P != 0
        assert fn(s, d, 2, 4, 16, 128, 3, None) == B.ERR_SHAPE  # elem_bytes
        assert fn(s, d, 16, 4, 16, 4, 2, None) == B.ERR_SHAPE   # 8-byte runs
        assert fn(None, d, 2, 4, 16, 128, 2, None) == B.ERR_NULL
        assert fn(vp(FAKE + 4), d, 2, 4, 16, 128, 2, None) == B.ERR_ALIGN
        assert fn(s, vp(FAKE + 64), 2, 4, 16, 128, 2, None) == B.ERR_SHAPE  # overlap


def test_seq2head_qkv_argument_errors(L):
    vp = ctypes.c_void_p
    big = 0x1000000
    ptrs = [vp(FAKE + i * big) for i in range(6)]
    f = L.cpattn_seq2head_qkv
    assert f(*ptrs, 3, 4, 16, 128, 2, None) == B.ERR_SHAPE  # H % P
    assert f(None, *ptrs[1:], 2, 4, 16, 128, 2, None) == B.ERR_NULL
    # kh overlapping vh
    bad = ptrs[:4] + [vp(FAKE + 5 * big + 32)] + ptrs[5:]
    assert f(*bad, 2, 4, 16, 128, 2, None) == B.ERR_SHAPE


def test_rmsnorm_argument_errors(L):
    vp = ctypes.c_void_p
    x, y, g = vp(FAKE), vp(FAKE + 0x1000000), vp(FAKE + 0x2000000)
    f = L.cpattn_rmsnorm
    for D in (0, 4, 48, 512, 100):  # powers of two in [8, 256] only
        assert f(x, y, g, 10, D, 1e-6, 1.0, None) == B.ERR_SHAPE, D
    assert f(x, y, g, -1, 128, 1e-6, 1.0, None) == B.ERR_SHAPE
    assert f(x, y, g, 10, 128, -1e-6, 1.0, None) == B.ERR_SHAPE       # eps < 0
    assert f(x, y, g, 10, 128, float("nan"), 1.0, None) == B.ERR_SHAPE
    assert f(x, y, g, 10, 128, 1e-6, float("inf"), None) == B.ERR_SHAPE
    assert f(None, y, g, 10, 128, 1e-6, 1.0, None) == B.ERR_NULL
    assert f(x, y, None, 10, 128, 1e-6, 1.0, None) == B.ERR_NULL
    assert f(x, y, vp(FAKE + 0x2000000 + 8), 10, 128, 1e-6, 1.0, None) == B.ERR_ALIGN
    assert f(x, vp(FAKE + 32), g, 10, 128, 1e-6, 1.0, None) == B.ERR_SHAPE  # partial overlap
    assert f(x, y, vp(FAKE + 0x1000000 + 64), 10, 128, 1e-6, 1.0, None) == B.ERR_SHAPE  # gamma in y
    assert f(x, y, g, 0, 128, 1e-6, 1.0, None) == B.OK  # nothing to do, nothing launched
    assert f(None, None, None, 0, 128, 1e-6, 1.0, None) == B.OK  # empty tensors may be NULL
    assert f(None, None, None, 0, 96, 1e-6, 1.0, None) == B.ERR_SHAPE  # shape still checked


def test_seq2head_qkv_norm_argument_errors(L):
    vp = ctypes.c_void_p
    big = 0x1000000
    ptrs = [vp(FAKE + i * big) for i in range(6)]
    gq, gk = vp(FAKE + 6 * big), vp(FAKE + 7 * big)
    f = L.cpattn_seq2head_qkv_norm
    assert f(*ptrs, gq, gk, 3, 4, 16, 128, 1e-6, 1.0, None) == B.ERR_SHAPE  # H % P
    assert f(*ptrs, gq, gk, 2, 4, 16, 96, 1e-6, 1.0, None) == B.ERR_SHAPE   # D not a power of 2
    assert f(*ptrs, gq, gk, 2, 4, 16, 128, -1.0, 1.0, None) == B.ERR_SHAPE  # eps
    assert f(*ptrs, None, gk, 2, 4, 16, 128, 1e-6, 1.0, None) == B.ERR_NULL
    assert f(*ptrs, gq, vp(FAKE + 7 * big + 4), 2, 4, 16, 128, 1e-6, 1.0, None) == B.ERR_ALIGN
    assert f(*ptrs, vp(FAKE + 3 * big + 256), gk, 2, 4, 16, 128, 1e-6, 1.0, None) == B.ERR_SHAPE
    bad = ptrs[:4] + [vp(FAKE + 5 * big + 32)] + ptrs[5:]
    assert f(*bad, gq, gk, 2, 4, 16, 128, 1e-6, 1.0, None) == B.ERR_SHAPE


def test_selftest_limit_checked(L):
    assert L.cpattn_selftest_wait_timeout(0, None) == B.ERR_SHAPE
    assert L.cpattn_selftest_wait_timeout((1 << 31) + 1, None) == B.ERR_SHAPE


def test_product_path_has_no_oracle_or_fallback():
    pkg = os.path.join(ROOT, "context_long_sequence_non_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                with open(os.path.join(dirpath, fn)) as f:
                    src = f.read()
                assert "import oracle" not in src and "from oracle" not in src, fn


def test_tail_split_workspace_bound_holds_for_every_key_count(L):
    # the n_split = 0 query takes no key count and promises an upper bound: the exact need
    # of every key count stays below it (a caller sizing by the bound never runs short)
    from hypothesis import given, settings
    from hypothesis import strategies as st

    @settings(max_examples=300, deadline=None)
    @given(st.integers(1, 8), st.integers(1, 64), st.integers(1, 60000), st.integers(1, 60000),
           st.sampled_from([64, 128]), st.sampled_from([0, 1]))
    def check(Bn, H, Sq, Skv, D, dt):
        exact = L.cpattn_fwd_split_workspace_kv(Bn, H, Sq, Skv, D, 0, dt)
        bound = L.cpattn_fwd_split_workspace(Bn, H, Sq, D, 0, dt)
        assert exact <= bound
        if exact:  # fp32 rows of 256 per range, then their LSEs
            rows = exact // (D * 4 + 4)
            assert rows % 256 == 0 and exact == rows * D * 4 + rows * 4

    check()


def test_ulysses_workspace_is_the_plain_plan_of_its_head_groups(L):
    # the fused pass splits the same work items as a [P][P*S_l][H/P][D] attention would
    from hypothesis import given, settings
    from hypothesis import strategies as st

    @settings(max_examples=200, deadline=None)
    @given(st.integers(1, 8), st.integers(1, 600), st.integers(1, 8), st.sampled_from([64, 128]))
    def check(P, s16, hp, D):
        S_l, H = 16 * s16, hp * P
        assert L.cpattn_ulysses_fwd_workspace(P, S_l, H, D, 0) == \
            L.cpattn_fwd_split_workspace_kv(P, hp, P * S_l, P * S_l, D, 0, 0)

    check()
