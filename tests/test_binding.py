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


@pytest.fixture
def no_library(monkeypatch):
    """Makes any library call fail the test, so a check that passes has
    raised before anything could be launched."""
    def boom():
        raise AssertionError("the library was called")
    monkeypatch.setattr(fa, "_lib_handle", boom)


def test_host_tensors_are_rejected_before_any_launch(no_library):
    """Host (CPU) tensors of valid shapes raise ValueError in every wrapper:
    their pointers would be illegal device addresses in the kernels."""
    B, N, H, d = 1, 8, 2, 64
    q, lse = t(B, N, H, d), torch.zeros(B, H, N)
    cu = torch.tensor([0, N], dtype=torch.int32)
    qp, qkv = t(N, H, d), t(B, N, 3, H, d)
    qkvp = t(N, 3, H, d)
    kc = t(4, 16, H, d)
    table = torch.zeros(B, 4, dtype=torch.int32)
    lens = torch.ones(B, dtype=torch.int32)
    one = t(B, 1, H, d)
    lse1 = torch.zeros(B, H, 1)
    calls = [
        lambda: fa.fa_fwd(q, q, q, q, lse, 0.1),
        lambda: fa.fa_fwd_gqa(q, q, q, q, lse, 0.1),
        lambda: fa.fa_fwd_varlen(qp, qp, qp, qp, torch.zeros(H, N), cu, cu, N, N, 0.1),
        lambda: fa.fa_fwd_qkvpacked(qkv, q, lse, 0.1),
        lambda: fa.fa_fwd_varlen_qkvpacked(qkvp, qp, torch.zeros(H, N), cu, N, 0.1),
        lambda: fa.fa_bwd(q, q, q, q, lse, q, q, q, q, 0.1),
        lambda: fa.fa_bwd_varlen(qp, qp, qp, qp, torch.zeros(H, N), qp, qp, qp, qp, cu, cu, N, N, 0.1),
        lambda: fa.fa_bwd_qkvpacked(qkv, q, lse, q, qkv, 0.1),
        lambda: fa.fa_bwd_varlen_qkvpacked(qkvp, qp, torch.zeros(H, N), qp, qkvp, cu, N, 0.1),
        lambda: fa.fa_fwd_kvcache(one, kc, kc, table, lens, one, lse1, 0.1),
        lambda: fa.fa_fwd_kvcache_gqa(one, kc, kc, table, lens, one, lse1, 0.1),
        lambda: fa.fa_fwd_kvcache_noalloc(one, kc, kc, table, lens, one, lse1, 0.1),
        lambda: fa.fa_kvcache_append(one, one, kc, kc, table, lens),
        lambda: fa.fa_fwd_fp8(q.to(torch.float8_e4m3fn), q.to(torch.float8_e4m3fn), q.to(torch.float8_e4m3fn),
                              t(B, N, H, d), lse, 0.1),
    ]
    for i, call in enumerate(calls):
        with pytest.raises(ValueError, match="CUDA"):
            call()


def test_decode_wrappers_reject_a_short_cache_seqlens(no_library):
    """cache_seqlens must hold one length per sequence: a shorter tensor
    would be read past its end on the device."""
    B, H, d = 3, 2, 64
    one, kc = t(B, 1, H, d), t(8, 16, H, d)
    table = torch.zeros(B, 4, dtype=torch.int32)
    short = torch.ones(B - 1, dtype=torch.int32)
    lse1 = torch.zeros(B, H, 1)
    for call in (lambda: fa.fa_fwd_kvcache(one, kc, kc, table, short, one, lse1, 0.1),
                 lambda: fa.fa_fwd_kvcache_gqa(one, kc, kc, table, short, one, lse1, 0.1),
                 lambda: fa.fa_fwd_kvcache_noalloc(one, kc, kc, table, short, one, lse1, 0.1),
                 lambda: fa.fa_kvcache_append(one, one, kc, kc, table, short)):
        with pytest.raises(ValueError, match="cache_seqlens"):
            call()


def test_device_check_covers_slopes_and_workspace():
    """The device check itself: host tensors, and slopes of the wrong length
    or type, raise (exercised here on host tensors only; the GPU tests pass
    device tensors through the same check)."""
    x = t(2, 3)
    with pytest.raises(ValueError, match="CUDA"):
        fa._on_device("f", (x,))
    with pytest.raises(ValueError, match="CUDA"):
        fa._on_device("f", (x,), workspace=torch.zeros(4, dtype=torch.uint8))
