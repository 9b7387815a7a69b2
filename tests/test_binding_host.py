"""Host-only checks of the Python binding: a caller-provided output, LSE or workspace of the
wrong size is refused before its pointer reaches the library (which sees only pointers)."""

import pytest
import torch

import context_long_sequence_non_b200 as cp

bf = torch.bfloat16


def _t(*shape, dtype=bf):
    return torch.zeros(*shape, dtype=dtype)


def test_attention_outputs_checked():
    q, k, v = _t(1, 300, 2, 128), _t(1, 500, 2, 128), _t(1, 500, 2, 128)
    with pytest.raises(ValueError, match="out must have shape"):
        cp.fwd(q, k, v, out=_t(1, 299, 2, 128))
    with pytest.raises(ValueError, match="lse must have shape"):
        cp.fwd(q, k, v, lse=_t(1, 300, 2, dtype=torch.float32))
    with pytest.raises(ValueError, match="lse must be"):
        cp.fwd(q, k, v, lse=_t(1, 2, 300))
    with pytest.raises(ValueError, match="out must have shape"):
        cp.fwd_split(q, k, v, out=_t(1, 300, 2, 64), n_split=2)
    with pytest.raises(ValueError, match="k and v"):
        cp.fwd_split(q, _t(1, 500, 3, 128), v, n_split=2)
    with pytest.raises(ValueError, match="lse_acc must be"):
        cp.fwd_accumulate(q, k, v, _t(1, 300, 2, 128), _t(1, 2, 300))


def test_ulysses_outputs_checked():
    s = [_t(4, 32, 8, 128) for _ in range(3)]
    with pytest.raises(ValueError, match="out must have shape"):
        cp.ulysses_fwd(*s, 4, out=_t(4, 32, 8, 64))
    with pytest.raises(ValueError, match="lse must have shape"):
        cp.ulysses_fwd(*s, 4, lse=_t(4, 8, 128, dtype=torch.float32))
    with pytest.raises(ValueError, match="lse must have shape"):
        cp.ulysses_fwd_split(*s, 4, lse=_t(2, 4, 128, dtype=torch.float32))


def test_merge_and_permute_outputs_checked():
    oa, ob = _t(1, 10, 2, 64), _t(1, 10, 2, 64)
    la, lb = _t(1, 2, 10, dtype=torch.float32), _t(1, 2, 10, dtype=torch.float32)
    with pytest.raises(ValueError, match="o_b must have shape"):
        cp.merge(oa, la, _t(1, 11, 2, 64), lb)
    with pytest.raises(ValueError, match="lse_b must have shape"):
        cp.merge(oa, la, ob, _t(1, 10, 2, dtype=torch.float32))
    with pytest.raises(ValueError, match="out must be"):
        cp.merge(oa, la, ob, lb, out=_t(1, 10, 2, 64, dtype=torch.float32))
    src = _t(4, 8, 8, 16)
    with pytest.raises(ValueError, match="out must have shape"):
        cp.seq2head(src, 4, out=_t(4, 32, 4, 16))
    with pytest.raises(ValueError, match="out must be"):
        cp.seq2head(src, 4, out=_t(4, 32, 2, 16, dtype=torch.float32))
    with pytest.raises(ValueError, match=r"out\[1\] must have shape"):
        cp.seq2head_qkv(src, src, src, 4, out=(_t(4, 32, 2, 16), _t(4, 32, 2, 8), _t(4, 32, 2, 16)))
    with pytest.raises(ValueError, match="out must have shape"):
        cp.head2seq(_t(4, 32, 2, 16), 4, out=_t(4, 8, 8, 8))
