"""The Python binding refuses buffers whose shape differs from the problem shape (the kernels index
them by it); right shapes get past the check (on a CPU-only host they then stop at the CUDA-tensor
check, before any device work)."""

import pytest
import torch

import block_sparse_attention_attngate_b200 as S


def _shape():
    return S.Shape(2, 8, 2, 128, 64, 64, 16)


def test_kcomp_append_shapes():
    sh = _shape()
    good = dict(k_new=torch.zeros(2, 2, 128), seqlens=torch.zeros(2, dtype=torch.int32),
                state=torch.zeros(2, 2, 3, 128), valid_blocks=torch.zeros(2, 2, dtype=torch.int32),
                w_k=torch.zeros(2, 64, 384), kcomp=torch.zeros(2, 2, 16, 64))
    with pytest.raises(TypeError, match="CUDA tensor"):   # shapes accepted; CPU tensors refused next
        S.kcomp_append(sh, **good)
    for name, bad in (("state", torch.zeros(2, 2, 3, 64)), ("kcomp", torch.zeros(2, 2, 8, 64)),
                      ("k_new", torch.zeros(2, 128)), ("w_k", torch.zeros(2, 64, 256))):
        with pytest.raises(ValueError, match=name):
            S.kcomp_append(sh, **{**good, name: bad})


def test_kcomp_state_init_shapes():
    sh = _shape()
    with pytest.raises(ValueError, match="state"):
        S.kcomp_state_init(sh, None, torch.zeros(2, dtype=torch.int32), torch.zeros(2, 2, 3, 64))


def test_prefill_gt_shapes():
    sh = _shape()
    T = 300
    good = dict(q=torch.zeros(2, 8, T, 128), k=None, v=None, seqlens=torch.zeros(2, dtype=torch.int32),
                out=torch.zeros(2, 8, T, 128), gt=torch.zeros(2, 2, T, 16), workspace=torch.zeros(16),
                lse=torch.zeros(2, 8, T))
    with pytest.raises(TypeError, match="CUDA tensor"):
        S.prefill_gt(sh, **good)
    for name, bad in (("gt", torch.zeros(2, 2, T, 8)), ("out", torch.zeros(2, 8, T - 1, 128)),
                      ("lse", torch.zeros(2, 8, T + 1)), ("q", torch.zeros(2, 4, T, 128))):
        with pytest.raises(ValueError, match=name):
            S.prefill_gt(sh, **{**good, name: bad})
