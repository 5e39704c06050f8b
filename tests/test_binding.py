"""Argument checks of the Python binding that run before any library call
(CPU tensors, no device needed): shape, dtype and layout mismatches raise
ValueError."""
import pytest
import torch

import exact_io_aware_79_b200 as fa


def t(*shape, dtype=torch.bfloat16):
    return torch.zeros(*shape, dtype=dtype)


def test_bwd_rejects_mismatched_shapes():
    q, k = t(1, 8, 4, 64), t(1, 8, 2, 64)
    lse = torch.zeros(1, 4, 8)
    with pytest.raises(ValueError):
        fa.fa_bwd(q, k, k, q, lse, q, q, t(1, 8, 4, 64), k, 0.1)          # dk shaped like q
    with pytest.raises(ValueError):
        fa.fa_bwd(q, k, k, q, torch.zeros(1, 8, 4), q, q, k, k, 0.1)      # lse [B, Nq, H]
    with pytest.raises(ValueError):
        fa.fa_bwd(q, k, k, q, lse, q.half(), q, k, k, 0.1)                # mixed dtypes
    with pytest.raises(ValueError):
        fa.fa_bwd(q.transpose(1, 2), k, k, q, lse, q, q, k, k, 0.1)       # not contiguous


def test_bwd_varlen_rejects_bad_offsets_and_lse():
    q, k = t(20, 2, 64), t(30, 2, 64)
    cu = torch.tensor([0, 20], dtype=torch.int32)
    cuk = torch.tensor([0, 30], dtype=torch.int32)
    with pytest.raises(ValueError):
        fa.fa_bwd_varlen(q, k, k, q, torch.zeros(20, 2), q, q, k, k, cu, cuk, 20, 30, 0.1)   # lse [total, H]
    with pytest.raises(ValueError):
        fa.fa_bwd_varlen(q, k, k, q, torch.zeros(2, 20), q, q, k, k, cu.long(), cuk, 20, 30, 0.1)
    with pytest.raises(ValueError):
        fa.fa_bwd_varlen(q, k, k, q, torch.zeros(2, 20), q, q, k, k, cu, torch.tensor([0, 10, 30], dtype=torch.int32),
                         20, 30, 0.1)                                       # cu_seqlens_k of another batch


def test_bwd_qkvpacked_rejects_a_non_packed_tensor():
    qkv = t(1, 8, 2, 4, 64)                                                 # slot axis of 2, not 3
    out = t(1, 8, 4, 64)
    with pytest.raises(ValueError):
        fa.fa_bwd_qkvpacked(qkv, out, torch.zeros(1, 4, 8), out, qkv, 0.1)
    qkv = t(16, 3, 4, 64)
    with pytest.raises(ValueError):
        fa.fa_bwd_varlen_qkvpacked(qkv, t(16, 4, 64), torch.zeros(16, 4), t(16, 4, 64), qkv,
                                   torch.tensor([0, 16], dtype=torch.int32), 16, 0.1)


def test_attention_func_is_an_autograd_function():
    assert issubclass(fa._AttentionFn, torch.autograd.Function)
    assert callable(fa.attention_func)
