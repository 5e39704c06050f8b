"""Exact IO-aware attention for B200 (sm_100a).

Python binding of the C ABI in include/fa.h (libfa_b200.so, built in-tree by
``python -m exact_io_aware_79_b200.build``). The binding only marshals
arguments: shapes are read off the torch tensors, pointers and the current
CUDA stream are passed through, and a non-OK status raises FaError. All
computation happens in the library's CUDA kernels; there is no fallback, and
every call raises if the library cannot be loaded.

Entry points with the C names:
    fa_fwd(q, k, v, out, lse, scale, causal, window_left, window_right,
           alibi_slopes, softcap)
    fa_fwd_fp8(q8, k8, v8, out, lse, scale, descale_q, descale_k, descale_v,
               causal, window_left, window_right, alibi_slopes, softcap,
               workspace)
    fa_fwd_kvcache(q, k_cache, v_cache, block_table, cache_seqlens, out, lse,
                   scale, window_left, alibi_slopes, softcap, num_splits,
                   workspace)
    fa_kvcache_num_splits(...), fa_kvcache_workspace_size(...),
    fa_status_string(code)
and allocating conveniences ``attention`` and ``decode``.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libfa_b200.so")

FA_FP16, FA_BF16 = 0, 1
FA_E4M3, FA_E5M2 = 0, 1
FA_MAX_SPLITS = 64
FA_NOALLOC_SCRATCH_BYTES = 32 << 20
STATUS = {
    0: "FA_OK", 1: "FA_ERR_NULL", 2: "FA_ERR_SHAPE", 3: "FA_ERR_DTYPE", 4: "FA_ERR_HEADDIM",
    5: "FA_ERR_ARG", 6: "FA_ERR_WORKSPACE", 7: "FA_ERR_CUDA", 8: "FA_ERR_DEVICE",
}


class FaError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__("%s failed: %s" % (where, _lib_handle().fa_status_string(code).decode()))


_LIB = None


def _lib_handle():
    global _LIB
    if _LIB is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError("libfa_b200.so not found at %s; build it with "
                              "`python -m exact_io_aware_79_b200.build`" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, i, vp, f, vp]
        L.fa_fwd.restype = i
        L.fa_fwd_gqa.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, i, i, vp, f, vp]
        L.fa_fwd_gqa.restype = i
        L.fa_fwd_fp8.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, f, f, f, i, i, i, vp, f, vp, sz, vp]
        L.fa_fwd_fp8.restype = i
        L.fa_fwd_fp8_workspace_size.argtypes = [i, i, i, i]
        L.fa_fwd_fp8_workspace_size.restype = sz
        L.fa_fwd_kvcache_gqa.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, f, i, vp, f, i, vp,
                                         sz, vp]
        L.fa_fwd_kvcache_gqa.restype = i
        L.fa_kvcache_append.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, vp]
        L.fa_kvcache_append.restype = i
        L.fa_fwd_qkvpacked.argtypes = [vp, vp, vp, i, i, i, i, i, f, i, i, i, vp, f, vp]
        L.fa_fwd_qkvpacked.restype = i
        L.fa_fwd_varlen_qkvpacked.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, i, vp, f, vp]
        L.fa_fwd_varlen_qkvpacked.restype = i
        L.fa_fwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, f, i, i, i, vp, f, vp]
        L.fa_fwd_varlen.restype = i
        L.fa_fwd_kvcache.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, vp, f, i, vp, sz,
                                     vp]
        L.fa_fwd_kvcache.restype = i
        L.fa_fwd_kvcache_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, vp, f, i,
                                             vp]
        L.fa_fwd_kvcache_noalloc.restype = i
        L.fa_kvcache_num_splits.argtypes = [i, i, i, i, i, i]
        L.fa_kvcache_num_splits.restype = i
        L.fa_kvcache_num_splits_gqa.argtypes = [i, i, i, i, i, i, i]
        L.fa_kvcache_num_splits_gqa.restype = i
        L.fa_kvcache_workspace_size.argtypes = [i, i, i, i, i, i]
        L.fa_kvcache_workspace_size.restype = sz
        L.fa_bwd_workspace_size.argtypes = [i, i, i, i]
        L.fa_bwd_workspace_size.restype = sz
        L.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, i, i, i, vp, f, i, vp, sz,
                             vp]
        L.fa_bwd.restype = i
        L.fa_bwd_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, i, i, f, i, i, i,
                                    vp, f, i, vp, sz, vp]
        L.fa_bwd_varlen.restype = i
        L.fa_bwd_qkvpacked.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, i, vp, f, i, vp, sz, vp]
        L.fa_bwd_qkvpacked.restype = i
        L.fa_bwd_varlen_qkvpacked.argtypes = [vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, i, i, vp, f, i, vp,
                                              sz, vp]
        L.fa_bwd_varlen_qkvpacked.restype = i
        L.fa_status_string.argtypes = [i]
        L.fa_status_string.restype = ctypes.c_char_p
        _LIB = L
    return _LIB


def library() -> ctypes.CDLL:
    """The loaded libfa_b200.so (raises ImportError if it is missing)."""
    return _lib_handle()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float16:
        return FA_FP16
    if t.dtype == torch.bfloat16:
        return FA_BF16
    return -1


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    if isinstance(stream, torch.cuda.Stream):
        return ctypes.c_void_p(stream.cuda_stream)
    return ctypes.c_void_p(int(stream))


def _check(code: int, where: str):
    if code != 0:
        raise FaError(code, where)


def _on_device(where: str, tensors, alibi_slopes=None, H: int = 0, workspace=None) -> None:
    """Checks, before anything is launched, that every tensor lives on the
    device of the first one (a CUDA device), and that alibi_slopes, when
    given, is a contiguous fp32 [H] tensor there: a host pointer or another
    GPU's pointer handed to a kernel would be an illegal device access, not
    an error the library could report."""
    ref = tensors[0]
    extra = [t for t in (alibi_slopes, workspace) if t is not None]
    for t in list(tensors) + extra:
        if not isinstance(t, torch.Tensor) or not t.is_cuda or t.device != ref.device:
            raise ValueError("%s: every tensor must be a CUDA tensor on %s" % (
                where, ref.device if ref.is_cuda else "one CUDA device"))
    if alibi_slopes is not None and (alibi_slopes.dtype != torch.float32 or tuple(alibi_slopes.shape) != (H,)
                                     or not alibi_slopes.is_contiguous()):
        raise ValueError("%s: alibi_slopes must be a contiguous fp32 tensor of shape [%d]" % (where, H))


def fa_status_string(code: int) -> str:
    return _lib_handle().fa_status_string(code).decode()


def fa_fwd(q, k, v, out, lse, scale: float, causal: bool = False, window_left: int = -1,
           window_right: int = -1, alibi_slopes=None, softcap: float = 0.0, stream=None) -> None:
    """q [B,Nq,H,d], k/v [B,Nk,H,d], out like q, lse fp32 [B,H,Nq]; all on the device."""
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    for t in (q, k, v, out, lse):
        if not t.is_contiguous():
            raise ValueError("fa_fwd needs contiguous tensors")
    if tuple(k.shape) != (B, Nk, H, d) or tuple(v.shape) != (B, Nk, H, d) or tuple(out.shape) != tuple(q.shape):
        raise ValueError("fa_fwd: shape mismatch")
    if tuple(lse.shape) != (B, H, Nq) or lse.dtype != torch.float32:
        raise ValueError("fa_fwd: lse must be fp32 [B, H, Nq]")
    if not (q.dtype == k.dtype == v.dtype == out.dtype):
        raise ValueError("fa_fwd: q, k, v, out must share one dtype")
    _on_device("fa_fwd", (q, k, v, out, lse), alibi_slopes, H)
    code = _lib_handle().fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, Nq, Nk, d,
                                _dtype_code(q), float(scale), int(bool(causal)), int(window_left),
                                int(window_right), _ptr(alibi_slopes), float(softcap), _stream(stream))
    _check(code, "fa_fwd")


def fa_fwd_gqa(q, k, v, out, lse, scale: float, causal: bool = False, window_left: int = -1,
               window_right: int = -1, alibi_slopes=None, softcap: float = 0.0, stream=None) -> None:
    """Grouped-query forward: q [B,Nq,H,d], k/v [B,Nk,H_kv,d] with H % H_kv == 0; out like q;
    lse fp32 [B,H,Nq]."""
    B, Nq, H, d = q.shape
    Nk, H_kv = k.shape[1], k.shape[2]
    for t in (q, k, v, out, lse):
        if not t.is_contiguous():
            raise ValueError("fa_fwd_gqa needs contiguous tensors")
    if tuple(k.shape) != (B, Nk, H_kv, d) or tuple(v.shape) != (B, Nk, H_kv, d) or \
            tuple(out.shape) != tuple(q.shape):
        raise ValueError("fa_fwd_gqa: shape mismatch")
    if tuple(lse.shape) != (B, H, Nq) or lse.dtype != torch.float32:
        raise ValueError("fa_fwd_gqa: lse must be fp32 [B, H, Nq]")
    if not (q.dtype == k.dtype == v.dtype == out.dtype):
        raise ValueError("fa_fwd_gqa: q, k, v, out must share one dtype")
    _on_device("fa_fwd_gqa", (q, k, v, out, lse), alibi_slopes, H)
    code = _lib_handle().fa_fwd_gqa(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, H_kv, Nq, Nk, d,
                                    _dtype_code(q), float(scale), int(bool(causal)), int(window_left),
                                    int(window_right), _ptr(alibi_slopes), float(softcap), _stream(stream))
    _check(code, "fa_fwd_gqa")


def _fp8_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float8_e4m3fn:
        return FA_E4M3
    if t.dtype == torch.float8_e5m2:
        return FA_E5M2
    return -1


def fa_fwd_fp8_workspace_size(B: int, H_kv: int, Nk: int, d: int) -> int:
    return int(_lib_handle().fa_fwd_fp8_workspace_size(B, H_kv, Nk, d))


def fa_fwd_fp8(q, k, v, out, lse, scale: float, descale_q: float = 1.0, descale_k: float = 1.0,
               descale_v: float = 1.0, causal: bool = False, window_left: int = -1, window_right: int = -1,
               alibi_slopes=None, softcap: float = 0.0, workspace: Optional[torch.Tensor] = None,
               stream=None) -> None:
    """8-bit forward: q [B,Nq,H,d], k/v [B,Nk,H_kv,d] float8_e4m3fn or float8_e5m2 (one format);
    out bf16 [B,Nq,H,d]; lse fp32 [B,H,Nq]; element x8 stands for x8 * descale_x; workspace a
    byte tensor of fa_fwd_fp8_workspace_size bytes (allocated here when None)."""
    B, Nq, H, d = q.shape
    Nk, H_kv = k.shape[1], k.shape[2]
    for t in (q, k, v, out, lse):
        if not t.is_contiguous():
            raise ValueError("fa_fwd_fp8 needs contiguous tensors")
    if tuple(k.shape) != (B, Nk, H_kv, d) or tuple(v.shape) != tuple(k.shape) or tuple(out.shape) != tuple(q.shape):
        raise ValueError("fa_fwd_fp8: shape mismatch")
    if out.dtype != torch.bfloat16 or tuple(lse.shape) != (B, H, Nq) or lse.dtype != torch.float32:
        raise ValueError("fa_fwd_fp8: out must be bf16 [B, Nq, H, d], lse fp32 [B, H, Nq]")
    if not (q.dtype == k.dtype == v.dtype) or _fp8_code(q) < 0:
        raise ValueError("fa_fwd_fp8: q, k, v must share one 8-bit float type")
    _on_device("fa_fwd_fp8", (q, k, v, out, lse), alibi_slopes, H, workspace=workspace)
    if workspace is None:
        workspace = torch.empty(max(fa_fwd_fp8_workspace_size(B, H_kv, Nk, d), 16), dtype=torch.uint8,
                                device=q.device)
    code = _lib_handle().fa_fwd_fp8(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, H, H_kv, Nq, Nk, d,
                                    _fp8_code(q), float(scale), float(descale_q), float(descale_k),
                                    float(descale_v), int(bool(causal)), int(window_left), int(window_right),
                                    _ptr(alibi_slopes), float(softcap), _ptr(workspace),
                                    workspace.numel() * workspace.element_size(), _stream(stream))
    _check(code, "fa_fwd_fp8")


def attention_fp8(q, k, v, scale: Optional[float] = None, descale_q: float = 1.0, descale_k: float = 1.0,
                  descale_v: float = 1.0, causal: bool = False, window_left: int = -1, window_right: int = -1,
                  alibi_slopes=None, softcap: float = 0.0):
    """Allocating form of fa_fwd_fp8; returns (out bf16, lse)."""
    B, Nq, H, d = q.shape
    out = torch.empty((B, Nq, H, d), dtype=torch.bfloat16, device=q.device)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    fa_fwd_fp8(q, k, v, out, lse, d ** -0.5 if scale is None else scale, descale_q, descale_k, descale_v, causal,
               window_left, window_right, alibi_slopes, softcap)
    return out, lse


def fa_bwd_workspace_size(B: int, H: int, Nq: int, d: int) -> int:
    return int(_lib_handle().fa_bwd_workspace_size(B, H, Nq, d))


def fa_bwd(q, k, v, out, lse, dout, dq, dk, dv, scale: float, causal: bool = False, window_left: int = -1,
           window_right: int = -1, alibi_slopes=None, softcap: float = 0.0, deterministic: bool = False,
           workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    """Backward of fa_fwd / fa_fwd_gqa: q, out, dout, dq [B,Nq,H,d]; k, v, dk, dv [B,Nk,H_kv,d];
    lse fp32 [B,H,Nq] from the forward; workspace a byte tensor of fa_bwd_workspace_size bytes
    (allocated here when None); deterministic: dq summed in a fixed order (bit-for-bit repeatable)."""
    B, Nq, H, d = q.shape
    Nk, H_kv = k.shape[1], k.shape[2]
    for t in (q, k, v, out, lse, dout, dq, dk, dv):
        if not t.is_contiguous():
            raise ValueError("fa_bwd needs contiguous tensors")
    if tuple(k.shape) != (B, Nk, H_kv, d) or tuple(v.shape) != tuple(k.shape) or \
            tuple(dk.shape) != tuple(k.shape) or tuple(dv.shape) != tuple(k.shape) or \
            tuple(out.shape) != tuple(q.shape) or tuple(dout.shape) != tuple(q.shape) or \
            tuple(dq.shape) != tuple(q.shape):
        raise ValueError("fa_bwd: shape mismatch")
    if tuple(lse.shape) != (B, H, Nq) or lse.dtype != torch.float32:
        raise ValueError("fa_bwd: lse must be fp32 [B, H, Nq]")
    if len({t.dtype for t in (q, k, v, out, dout, dq, dk, dv)}) != 1:
        raise ValueError("fa_bwd: q, k, v, out, dout, dq, dk, dv must share one dtype")
    _on_device("fa_bwd", (q, k, v, out, lse, dout, dq, dk, dv), alibi_slopes, H, workspace=workspace)
    need = fa_bwd_workspace_size(B, H, Nq, d)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    code = _lib_handle().fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk),
                                _ptr(dv), B, H, H_kv, Nq, Nk, d, _dtype_code(q), float(scale),
                                int(bool(causal)), int(window_left), int(window_right), _ptr(alibi_slopes),
                                float(softcap), int(bool(deterministic)), _ptr(workspace),
                                workspace.numel() * workspace.element_size(),
                                _stream(stream))
    _check(code, "fa_bwd")


def fa_bwd_varlen(q, k, v, out, lse, dout, dq, dk, dv, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int,
                  max_seqlen_k: int, scale: float, causal: bool = False, window_left: int = -1,
                  window_right: int = -1, alibi_slopes=None, softcap: float = 0.0, deterministic: bool = False,
                  workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    """Backward of fa_fwd_varlen: q, out, dout, dq [total_q,H,d]; k, v, dk, dv [total_k,H_kv,d];
    lse fp32 [H,total_q]; cu_seqlens_* int32 [B+1] on the device."""
    total_q, H, d = q.shape
    total_k, H_kv = k.shape[0], k.shape[1]
    B = cu_seqlens_q.numel() - 1
    for t in (q, k, v, out, lse, dout, dq, dk, dv, cu_seqlens_q, cu_seqlens_k):
        if not t.is_contiguous():
            raise ValueError("fa_bwd_varlen needs contiguous tensors")
    if tuple(k.shape) != (total_k, H_kv, d) or tuple(v.shape) != tuple(k.shape) or \
            tuple(dk.shape) != tuple(k.shape) or tuple(dv.shape) != tuple(k.shape) or \
            tuple(out.shape) != tuple(q.shape) or tuple(dout.shape) != tuple(q.shape) or \
            tuple(dq.shape) != tuple(q.shape) or cu_seqlens_k.numel() != B + 1:
        raise ValueError("fa_bwd_varlen: shape mismatch")
    if tuple(lse.shape) != (H, total_q) or lse.dtype != torch.float32:
        raise ValueError("fa_bwd_varlen: lse must be fp32 [H, total_q]")
    if cu_seqlens_q.dtype != torch.int32 or cu_seqlens_k.dtype != torch.int32:
        raise ValueError("fa_bwd_varlen: cu_seqlens must be int32")
    _on_device("fa_bwd_varlen", (q, k, v, out, lse, dout, dq, dk, dv, cu_seqlens_q, cu_seqlens_k),
               alibi_slopes, H, workspace=workspace)
    need = fa_bwd_workspace_size(1, H, total_q, d)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    code = _lib_handle().fa_bwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq),
                                       _ptr(dk), _ptr(dv), _ptr(cu_seqlens_q), _ptr(cu_seqlens_k), B, H, H_kv,
                                       int(max_seqlen_q), int(max_seqlen_k), total_q, total_k, d, _dtype_code(q),
                                       float(scale), int(bool(causal)), int(window_left), int(window_right),
                                       _ptr(alibi_slopes), float(softcap), int(bool(deterministic)),
                                       _ptr(workspace), workspace.numel() * workspace.element_size(),
                                       _stream(stream))
    _check(code, "fa_bwd_varlen")


def fa_bwd_qkvpacked(qkv, out, lse, dout, dqkv, scale: float, causal: bool = False, window_left: int = -1,
                     window_right: int = -1, alibi_slopes=None, softcap: float = 0.0, deterministic: bool = False,
                     workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    """Backward of fa_fwd_qkvpacked: qkv, dqkv [B,N,3,H,d]; out, dout [B,N,H,d]; lse fp32 [B,H,N]."""
    B, N, three, H, d = qkv.shape
    for t in (qkv, out, lse, dout, dqkv):
        if not t.is_contiguous():
            raise ValueError("fa_bwd_qkvpacked needs contiguous tensors")
    if three != 3 or tuple(dqkv.shape) != tuple(qkv.shape) or tuple(out.shape) != (B, N, H, d) or \
            tuple(dout.shape) != (B, N, H, d) or len({qkv.dtype, out.dtype, dout.dtype, dqkv.dtype}) != 1:
        raise ValueError("fa_bwd_qkvpacked: shape mismatch")
    if tuple(lse.shape) != (B, H, N) or lse.dtype != torch.float32:
        raise ValueError("fa_bwd_qkvpacked: lse must be fp32 [B, H, N]")
    _on_device("fa_bwd_qkvpacked", (qkv, out, lse, dout, dqkv), alibi_slopes, H, workspace=workspace)
    if workspace is None:
        workspace = torch.empty(max(fa_bwd_workspace_size(B, H, N, d), 16), dtype=torch.uint8, device=qkv.device)
    code = _lib_handle().fa_bwd_qkvpacked(_ptr(qkv), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dqkv), B, H, N, d,
                                          _dtype_code(qkv), float(scale), int(bool(causal)), int(window_left),
                                          int(window_right), _ptr(alibi_slopes), float(softcap),
                                          int(bool(deterministic)), _ptr(workspace),
                                          workspace.numel() * workspace.element_size(), _stream(stream))
    _check(code, "fa_bwd_qkvpacked")


def fa_bwd_varlen_qkvpacked(qkv, out, lse, dout, dqkv, cu_seqlens, max_seqlen: int, scale: float,
                            causal: bool = False, window_left: int = -1, window_right: int = -1, alibi_slopes=None,
                            softcap: float = 0.0, deterministic: bool = False,
                            workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    """Backward of fa_fwd_varlen_qkvpacked: qkv, dqkv [total,3,H,d]; out, dout [total,H,d];
    lse fp32 [H,total]; cu_seqlens int32 [B+1] on the device."""
    total, three, H, d = qkv.shape
    B = cu_seqlens.numel() - 1
    for t in (qkv, out, lse, dout, dqkv, cu_seqlens):
        if not t.is_contiguous():
            raise ValueError("fa_bwd_varlen_qkvpacked needs contiguous tensors")
    if three != 3 or tuple(dqkv.shape) != tuple(qkv.shape) or tuple(out.shape) != (total, H, d) or \
            tuple(dout.shape) != (total, H, d) or len({qkv.dtype, out.dtype, dout.dtype, dqkv.dtype}) != 1:
        raise ValueError("fa_bwd_varlen_qkvpacked: shape mismatch")
    if tuple(lse.shape) != (H, total) or lse.dtype != torch.float32 or cu_seqlens.dtype != torch.int32:
        raise ValueError("fa_bwd_varlen_qkvpacked: lse must be fp32 [H, total], cu_seqlens int32")
    _on_device("fa_bwd_varlen_qkvpacked", (qkv, out, lse, dout, dqkv, cu_seqlens),
               alibi_slopes, H, workspace=workspace)
    if workspace is None:
        workspace = torch.empty(max(fa_bwd_workspace_size(1, H, total, d), 16), dtype=torch.uint8,
                                device=qkv.device)
    code = _lib_handle().fa_bwd_varlen_qkvpacked(_ptr(qkv), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dqkv),
                                                 _ptr(cu_seqlens), B, H, int(max_seqlen), total, d,
                                                 _dtype_code(qkv), float(scale), int(bool(causal)),
                                                 int(window_left), int(window_right), _ptr(alibi_slopes),
                                                 float(softcap), int(bool(deterministic)), _ptr(workspace),
                                                 workspace.numel() * workspace.element_size(), _stream(stream))
    _check(code, "fa_bwd_varlen_qkvpacked")


def fa_fwd_qkvpacked(qkv, out, lse, scale: float, causal: bool = False, window_left: int = -1,
                     window_right: int = -1, alibi_slopes=None, softcap: float = 0.0, stream=None) -> None:
    """qkv [B,N,3,H,d] (slot 0 q, 1 k, 2 v); out [B,N,H,d]; lse fp32 [B,H,N]; all on the device."""
    B, N, three, H, d = qkv.shape
    for t in (qkv, out, lse):
        if not t.is_contiguous():
            raise ValueError("fa_fwd_qkvpacked needs contiguous tensors")
    if three != 3 or tuple(out.shape) != (B, N, H, d) or out.dtype != qkv.dtype:
        raise ValueError("fa_fwd_qkvpacked: shape mismatch")
    if tuple(lse.shape) != (B, H, N) or lse.dtype != torch.float32:
        raise ValueError("fa_fwd_qkvpacked: lse must be fp32 [B, H, N]")
    _on_device("fa_fwd_qkvpacked", (qkv, out, lse), alibi_slopes, H)
    code = _lib_handle().fa_fwd_qkvpacked(_ptr(qkv), _ptr(out), _ptr(lse), B, H, N, d, _dtype_code(qkv),
                                          float(scale), int(bool(causal)), int(window_left), int(window_right),
                                          _ptr(alibi_slopes), float(softcap), _stream(stream))
    _check(code, "fa_fwd_qkvpacked")


def fa_fwd_varlen_qkvpacked(qkv, out, lse, cu_seqlens, max_seqlen: int, scale: float, causal: bool = False,
                            window_left: int = -1, window_right: int = -1, alibi_slopes=None, softcap: float = 0.0,
                            stream=None) -> None:
    """qkv [total,3,H,d]; out [total,H,d]; lse fp32 [H,total]; cu_seqlens int32 [B+1] on the device."""
    total, three, H, d = qkv.shape
    B = cu_seqlens.numel() - 1
    for t in (qkv, out, lse, cu_seqlens):
        if not t.is_contiguous():
            raise ValueError("fa_fwd_varlen_qkvpacked needs contiguous tensors")
    if three != 3 or tuple(out.shape) != (total, H, d) or out.dtype != qkv.dtype:
        raise ValueError("fa_fwd_varlen_qkvpacked: shape mismatch")
    if tuple(lse.shape) != (H, total) or lse.dtype != torch.float32 or cu_seqlens.dtype != torch.int32:
        raise ValueError("fa_fwd_varlen_qkvpacked: lse must be fp32 [H, total], cu_seqlens int32")
    _on_device("fa_fwd_varlen_qkvpacked", (qkv, out, lse, cu_seqlens), alibi_slopes, H)
    code = _lib_handle().fa_fwd_varlen_qkvpacked(_ptr(qkv), _ptr(out), _ptr(lse), _ptr(cu_seqlens), B, H,
                                                 int(max_seqlen), total, d, _dtype_code(qkv), float(scale),
                                                 int(bool(causal)), int(window_left), int(window_right),
                                                 _ptr(alibi_slopes), float(softcap), _stream(stream))
    _check(code, "fa_fwd_varlen_qkvpacked")


def fa_fwd_varlen(q, k, v, out, lse, cu_seqlens_q, cu_seqlens_k, max_seqlen_q: int, max_seqlen_k: int,
                  scale: float, causal: bool = False, window_left: int = -1, window_right: int = -1,
                  alibi_slopes=None, softcap: float = 0.0, stream=None) -> None:
    """Packed sequences: q [total_q,H,d], k/v [total_k,H,d], out like q, lse fp32 [H,total_q];
    cu_seqlens_q / cu_seqlens_k int32 [B+1] row offsets on the device."""
    total_q, H, d = q.shape
    total_k = k.shape[0]
    B = cu_seqlens_q.numel() - 1
    for t in (q, k, v, out, lse, cu_seqlens_q, cu_seqlens_k):
        if not t.is_contiguous():
            raise ValueError("fa_fwd_varlen needs contiguous tensors")
    if tuple(k.shape) != (total_k, H, d) or tuple(v.shape) != (total_k, H, d) or tuple(out.shape) != tuple(q.shape):
        raise ValueError("fa_fwd_varlen: shape mismatch")
    if tuple(lse.shape) != (H, total_q) or lse.dtype != torch.float32:
        raise ValueError("fa_fwd_varlen: lse must be fp32 [H, total_q]")
    if cu_seqlens_q.dtype != torch.int32 or cu_seqlens_k.dtype != torch.int32 or cu_seqlens_k.numel() != B + 1:
        raise ValueError("fa_fwd_varlen: cu_seqlens must be int32 [B + 1]")
    if not (q.dtype == k.dtype == v.dtype == out.dtype):
        raise ValueError("fa_fwd_varlen: q, k, v, out must share one dtype")
    _on_device("fa_fwd_varlen", (q, k, v, out, lse, cu_seqlens_q, cu_seqlens_k), alibi_slopes, H)
    code = _lib_handle().fa_fwd_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(cu_seqlens_q),
                                       _ptr(cu_seqlens_k), B, H, int(max_seqlen_q), int(max_seqlen_k), total_q,
                                       total_k, d, _dtype_code(q), float(scale), int(bool(causal)),
                                       int(window_left), int(window_right), _ptr(alibi_slopes), float(softcap),
                                       _stream(stream))
    _check(code, "fa_fwd_varlen")


def fa_kvcache_num_splits(B: int, H: int, d: int, max_blocks: int, page_size: int, num_splits: int = 0) -> int:
    return int(_lib_handle().fa_kvcache_num_splits(B, H, d, max_blocks, page_size, num_splits))


def fa_kvcache_num_splits_gqa(B: int, H: int, H_kv: int, d: int, max_blocks: int, page_size: int,
                              num_splits: int = 0) -> int:
    """Split count fa_fwd_kvcache_gqa launches with H_kv cache heads."""
    return int(_lib_handle().fa_kvcache_num_splits_gqa(B, H, H_kv, d, max_blocks, page_size, num_splits))


def fa_kvcache_workspace_size(B: int, H: int, d: int, max_blocks: int, page_size: int,
                              num_splits: int = 0) -> int:
    return int(_lib_handle().fa_kvcache_workspace_size(B, H, d, max_blocks, page_size, num_splits))


def fa_fwd_kvcache(q, k_cache, v_cache, block_table, cache_seqlens, out, lse, scale: float,
                   window_left: int = -1, alibi_slopes=None, softcap: float = 0.0, num_splits: int = 0,
                   workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    """q [B,1,H,d]; caches [num_pages,page_size,H,d]; block_table int32 [B,max_blocks];
    cache_seqlens int32 [B]; out like q; lse fp32 [B,H,1]; workspace a byte tensor."""
    B, one, H, d = q.shape
    num_pages, page_size = k_cache.shape[0], k_cache.shape[1]
    max_blocks = block_table.shape[1]
    for t in (q, k_cache, v_cache, block_table, cache_seqlens, out, lse):
        if not t.is_contiguous():
            raise ValueError("fa_fwd_kvcache needs contiguous tensors")
    if one != 1 or tuple(k_cache.shape) != (num_pages, page_size, H, d) or \
            tuple(v_cache.shape) != tuple(k_cache.shape) or tuple(out.shape) != tuple(q.shape):
        raise ValueError("fa_fwd_kvcache: shape mismatch")
    if block_table.dtype != torch.int32 or cache_seqlens.dtype != torch.int32 or block_table.shape[0] != B or \
            tuple(cache_seqlens.shape) != (B,) or block_table.dim() != 2:
        raise ValueError("fa_fwd_kvcache: block_table must be int32 [B, max_blocks], cache_seqlens int32 [B]")
    if tuple(lse.shape) != (B, H, 1) or lse.dtype != torch.float32:
        raise ValueError("fa_fwd_kvcache: lse must be fp32 [B, H, 1]")
    _on_device("fa_fwd_kvcache", (q, k_cache, v_cache, block_table, cache_seqlens, out, lse),
               alibi_slopes, H, workspace=workspace)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    code = _lib_handle().fa_fwd_kvcache(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(cache_seqlens), _ptr(out), _ptr(lse),
        B, H, d, num_pages, page_size, max_blocks, _dtype_code(q), float(scale), int(window_left),
        _ptr(alibi_slopes), float(softcap), int(num_splits), _ptr(workspace), ws_bytes, _stream(stream))
    _check(code, "fa_fwd_kvcache")


def fa_fwd_kvcache_gqa(q, k_cache, v_cache, block_table, cache_seqlens, out, lse, scale: float,
                       window_left: int = -1, alibi_slopes=None, softcap: float = 0.0, num_splits: int = 0,
                       workspace: Optional[torch.Tensor] = None, stream=None) -> None:
    """Grouped-query decode: q [B,1,H,d]; caches [num_pages,page_size,H_kv,d] with H % H_kv == 0;
    the rest as fa_fwd_kvcache (the workspace size is that of H query heads)."""
    B, one, H, d = q.shape
    num_pages, page_size, H_kv = k_cache.shape[0], k_cache.shape[1], k_cache.shape[2]
    max_blocks = block_table.shape[1]
    for t in (q, k_cache, v_cache, block_table, cache_seqlens, out, lse):
        if not t.is_contiguous():
            raise ValueError("fa_fwd_kvcache_gqa needs contiguous tensors")
    if one != 1 or tuple(k_cache.shape) != (num_pages, page_size, H_kv, d) or \
            tuple(v_cache.shape) != tuple(k_cache.shape) or tuple(out.shape) != tuple(q.shape):
        raise ValueError("fa_fwd_kvcache_gqa: shape mismatch")
    if block_table.dtype != torch.int32 or cache_seqlens.dtype != torch.int32 or block_table.shape[0] != B or \
            tuple(cache_seqlens.shape) != (B,) or block_table.dim() != 2:
        raise ValueError("fa_fwd_kvcache_gqa: block_table must be int32 [B, max_blocks], cache_seqlens int32 [B]")
    if tuple(lse.shape) != (B, H, 1) or lse.dtype != torch.float32:
        raise ValueError("fa_fwd_kvcache_gqa: lse must be fp32 [B, H, 1]")
    _on_device("fa_fwd_kvcache_gqa", (q, k_cache, v_cache, block_table, cache_seqlens, out, lse),
               alibi_slopes, H, workspace=workspace)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    code = _lib_handle().fa_fwd_kvcache_gqa(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(cache_seqlens), _ptr(out), _ptr(lse),
        B, H, H_kv, d, num_pages, page_size, max_blocks, _dtype_code(q), float(scale), int(window_left),
        _ptr(alibi_slopes), float(softcap), int(num_splits), _ptr(workspace), ws_bytes, _stream(stream))
    _check(code, "fa_fwd_kvcache_gqa")


def fa_kvcache_append(k_new, v_new, k_cache, v_cache, block_table, cache_seqlens, stream=None) -> None:
    """Writes k_new/v_new [B,n_new,H_kv,d] into the paged caches [num_pages,page_size,H_kv,d] at
    positions cache_seqlens[b] .. + n_new - 1 (cache_seqlens is not advanced)."""
    B, n_new, H_kv, d = k_new.shape
    num_pages, page_size = k_cache.shape[0], k_cache.shape[1]
    max_blocks = block_table.shape[1]
    for t in (k_new, v_new, k_cache, v_cache, block_table, cache_seqlens):
        if not t.is_contiguous():
            raise ValueError("fa_kvcache_append needs contiguous tensors")
    if tuple(v_new.shape) != tuple(k_new.shape) or tuple(k_cache.shape) != (num_pages, page_size, H_kv, d) or \
            tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("fa_kvcache_append: shape mismatch")
    if block_table.dtype != torch.int32 or cache_seqlens.dtype != torch.int32 or block_table.shape[0] != B or \
            tuple(cache_seqlens.shape) != (B,) or block_table.dim() != 2:
        raise ValueError("fa_kvcache_append: block_table must be int32 [B, max_blocks], cache_seqlens int32 [B]")
    if not (k_new.dtype == v_new.dtype == k_cache.dtype == v_cache.dtype):
        raise ValueError("fa_kvcache_append: k/v and caches must share one dtype")
    _on_device("fa_kvcache_append", (k_new, v_new, k_cache, v_cache, block_table, cache_seqlens))
    code = _lib_handle().fa_kvcache_append(_ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache),
                                           _ptr(block_table), _ptr(cache_seqlens), B, n_new, H_kv, d, num_pages,
                                           page_size, max_blocks, _dtype_code(k_new), _stream(stream))
    _check(code, "fa_kvcache_append")


def fa_fwd_kvcache_noalloc(q, k_cache, v_cache, block_table, cache_seqlens, out, lse, scale: float,
                           window_left: int = -1, alibi_slopes=None, softcap: float = 0.0, num_splits: int = 0,
                           stream=None) -> None:
    """fa_fwd_kvcache without a workspace argument, for callers that cannot
    allocate device memory: the split partials live in the library's own
    fixed device array (FA_NOALLOC_SCRATCH_BYTES per GPU). Calls on one
    device share that array, so order them on one stream."""
    B, one, H, d = q.shape
    num_pages, page_size = k_cache.shape[0], k_cache.shape[1]
    max_blocks = block_table.shape[1]
    for t in (q, k_cache, v_cache, block_table, cache_seqlens, out, lse):
        if not t.is_contiguous():
            raise ValueError("fa_fwd_kvcache_noalloc needs contiguous tensors")
    if one != 1 or tuple(k_cache.shape) != (num_pages, page_size, H, d) or \
            tuple(v_cache.shape) != tuple(k_cache.shape) or tuple(out.shape) != tuple(q.shape):
        raise ValueError("fa_fwd_kvcache_noalloc: shape mismatch")
    if block_table.dtype != torch.int32 or cache_seqlens.dtype != torch.int32 or block_table.shape[0] != B or \
            tuple(cache_seqlens.shape) != (B,) or block_table.dim() != 2:
        raise ValueError("fa_fwd_kvcache_noalloc: block_table must be int32 [B, max_blocks], cache_seqlens int32 [B]")
    if tuple(lse.shape) != (B, H, 1) or lse.dtype != torch.float32:
        raise ValueError("fa_fwd_kvcache_noalloc: lse must be fp32 [B, H, 1]")
    _on_device("fa_fwd_kvcache_noalloc", (q, k_cache, v_cache, block_table, cache_seqlens, out, lse),
               alibi_slopes, H)
    code = _lib_handle().fa_fwd_kvcache_noalloc(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), _ptr(cache_seqlens), _ptr(out), _ptr(lse),
        B, H, d, num_pages, page_size, max_blocks, _dtype_code(q), float(scale), int(window_left),
        _ptr(alibi_slopes), float(softcap), int(num_splits), _stream(stream))
    _check(code, "fa_fwd_kvcache_noalloc")


def attention(q, k, v, scale: Optional[float] = None, causal: bool = False, window_left: int = -1,
              window_right: int = -1, alibi_slopes=None, softcap: float = 0.0):
    """Allocating form of fa_fwd; returns (out, lse)."""
    B, Nq, H, d = q.shape
    out = torch.empty_like(q)
    lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
    fa_fwd(q, k, v, out, lse, d ** -0.5 if scale is None else scale, causal, window_left, window_right,
           alibi_slopes, softcap)
    return out, lse


def decode(q, k_cache, v_cache, block_table, cache_seqlens, scale: Optional[float] = None,
           window_left: int = -1, alibi_slopes=None, softcap: float = 0.0, num_splits: int = 0):
    """Allocating form of fa_fwd_kvcache; returns (out, lse)."""
    B, _, H, d = q.shape
    out = torch.empty_like(q)
    lse = torch.empty((B, H, 1), dtype=torch.float32, device=q.device)
    nbytes = fa_kvcache_workspace_size(B, H, d, block_table.shape[1], k_cache.shape[1], num_splits)
    ws = torch.empty(max(nbytes, 1), dtype=torch.uint8, device=q.device) if nbytes else None
    fa_fwd_kvcache(q, k_cache, v_cache, block_table, cache_seqlens, out, lse,
                   d ** -0.5 if scale is None else scale, window_left, alibi_slopes, softcap, num_splits, ws)
    return out, lse


class _AttentionFn(torch.autograd.Function):
    """fa_fwd_gqa forward, fa_bwd backward (argument marshalling only)."""

    @staticmethod
    def forward(ctx, q, k, v, scale, causal, window_left, window_right, alibi_slopes, softcap, deterministic):
        q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
        B, Nq, H, d = q.shape
        out = torch.empty_like(q)
        lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
        fa_fwd_gqa(q, k, v, out, lse, scale, causal, window_left, window_right, alibi_slopes, softcap)
        ctx.save_for_backward(q, k, v, out, lse)
        ctx.opts = (scale, causal, window_left, window_right, alibi_slopes, softcap, deterministic)
        return out, lse

    @staticmethod
    def backward(ctx, dout, dlse):
        q, k, v, out, lse = ctx.saved_tensors
        scale, causal, window_left, window_right, alibi_slopes, softcap, deterministic = ctx.opts
        dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
        fa_bwd(q, k, v, out, lse, dout.contiguous(), dq, dk, dv, scale, causal, window_left, window_right,
               alibi_slopes, softcap, deterministic)
        return dq, dk, dv, None, None, None, None, None, None, None


def attention_func(q, k, v, scale: Optional[float] = None, causal: bool = False, window_left: int = -1,
                   window_right: int = -1, alibi_slopes=None, softcap: float = 0.0, deterministic: bool = False,
                   return_lse: bool = False):
    """Differentiable attention: q [B,Nq,H,d], k/v [B,Nk,H_kv,d] (H % H_kv == 0) on the device.
    Forward through fa_fwd_gqa, backward through fa_bwd (gradients for q, k, v; the LSE output
    carries no gradient). Returns out, or (out, lse) with return_lse."""
    d = q.shape[-1]
    out, lse = _AttentionFn.apply(q, k, v, d ** -0.5 if scale is None else float(scale), bool(causal),
                                  int(window_left), int(window_right), alibi_slopes, float(softcap),
                                  bool(deterministic))
    return (out, lse) if return_lse else out
