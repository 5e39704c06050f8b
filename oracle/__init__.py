"""fp64 CPU oracle for exact attention (test infrastructure).

Only the tests, the package smoke check and the benchmark's CPU-baseline leg
may import this package. It loads ``liboracle.so`` (built from
``attn_oracle.c``; see that file's header for the definition it follows and
the readings of the pages it takes) and shares no code with the CUDA path.

Inputs may be torch CPU tensors (fp16, bf16, float8_e4m3fn, float8_e5m2 or
fp64) or numpy arrays (float16 / float64, or uint16 / uint8 bit patterns
with an explicit ``dtype``).
Everything is returned as float64 numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

from . import build as _build

F16, BF16, F64, E4M3, E5M2 = 0, 1, 2, 3, 4

_lib = None


def load_library(path: Optional[str] = None):
    """(Re)binds the oracle to a compiled library; the default is the one
    built from attn_oracle.c. Tests use this to load deliberately broken
    copies of the oracle and check that the pins catch them."""
    global _lib
    _lib = None
    return lib(path)


def lib(path: Optional[str] = None):
    global _lib
    if _lib is None:
        path = path or _build.build()
        L = ctypes.CDLL(path)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int)
        vp = ctypes.c_void_p
        i, d = ctypes.c_int, ctypes.c_double
        L.oracle_attn_fwd.argtypes = [vp, vp, vp, i, dp, dp, dp, i, i, i, i, i, d, i, i, i, dp, d,
                                      ip, i, i]
        L.oracle_attn_fwd.restype = i
        L.oracle_attn_decode_paged.argtypes = [vp, vp, vp, i, ip, ip, dp, dp, i, i, i, i, i, i, d, i,
                                               dp, d, ip, i, i, i]
        L.oracle_attn_decode_paged.restype = i
        L.oracle_combine_splits.argtypes = [dp, dp, i, ctypes.c_long, i, dp, dp]
        L.oracle_combine_splits.restype = i
        L.oracle_widen.argtypes = [vp, i, dp, ctypes.c_long]
        L.oracle_widen.restype = i
        L.oracle_max_threads.restype = i
        _lib = L
    return _lib


def max_threads() -> int:
    return int(lib().oracle_max_threads())


def _as_storage(x, dtype_code: Optional[int] = None):
    """Returns (contiguous numpy array, storage code) for a tensor or array."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().contiguous()
            if x.dtype == torch.float8_e4m3fn:
                return x.view(torch.uint8).numpy(), E4M3
            if x.dtype == torch.float8_e5m2:
                return x.view(torch.uint8).numpy(), E5M2
            if x.dtype == torch.bfloat16:
                return x.view(torch.int16).numpy().view(np.uint16), BF16
            if x.dtype == torch.float16:
                return x.view(torch.int16).numpy().view(np.uint16), F16
            return np.ascontiguousarray(x.to(torch.float64).numpy()), F64
    except ImportError:  # pragma: no cover
        pass
    x = np.ascontiguousarray(x)
    if dtype_code is not None:
        return x, dtype_code
    if x.dtype == np.float16:
        return x.view(np.uint16), F16
    return np.ascontiguousarray(x, dtype=np.float64), F64


def _dptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _iptr(a: Optional[np.ndarray]):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int))


def _f64_vec(x) -> Optional[np.ndarray]:
    if x is None:
        return None
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().to(torch.float64).numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(x, dtype=np.float64)


def _i32_vec(x) -> Optional[np.ndarray]:
    if x is None:
        return None
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().cpu().numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(x, dtype=np.int32)


def widen(x, dtype_code: Optional[int] = None) -> np.ndarray:
    """The oracle's exact widening of fp16/bf16 storage to fp64."""
    a, code = _as_storage(x, dtype_code)
    out = np.empty(a.shape, dtype=np.float64)
    rc = lib().oracle_widen(a.ctypes.data, code, _dptr(out), a.size)
    if rc:
        raise ValueError("oracle_widen failed: %d" % rc)
    return out


def attn_fwd(q, k, v, scale: float, causal: bool = False, window_left: int = -1,
             window_right: int = -1, alibi_slopes=None, softcap: float = 0.0,
             rows: Optional[Sequence[int]] = None, return_probs: bool = False,
             num_threads: int = 0, dtype_code: Optional[int] = None):
    """Plain-definition attention. q [B,Nq,H,d], k/v [B,Nk,H,d].

    Returns (o [B,R,H,d], lse [B,H,R]) or (o, lse, p [B,H,R,Nk]) where R is
    len(rows) (all Nq rows when rows is None).
    """
    qa, code = _as_storage(q, dtype_code)
    ka, kc = _as_storage(k, dtype_code)
    va, vc = _as_storage(v, dtype_code)
    if not (code == kc == vc):
        raise ValueError("q, k, v must share one storage type")
    B, Nq, H, d = qa.shape
    Nk = ka.shape[1]
    if ka.shape != (B, Nk, H, d) or va.shape != ka.shape:
        raise ValueError("shape mismatch")
    r = _i32_vec(rows)
    R = Nq if r is None else len(r)
    o = np.empty((B, R, H, d), dtype=np.float64)
    lse = np.empty((B, H, R), dtype=np.float64)
    p = np.empty((B, H, R, Nk), dtype=np.float64) if return_probs else None
    slopes = _f64_vec(alibi_slopes)
    rc = lib().oracle_attn_fwd(qa.ctypes.data, ka.ctypes.data, va.ctypes.data, code, _dptr(o),
                               _dptr(lse), _dptr(p), B, H, Nq, Nk, d, float(scale), int(causal),
                               int(window_left), int(window_right), _dptr(slopes), float(softcap),
                               _iptr(r), R, int(num_threads))
    if rc:
        raise ValueError("oracle_attn_fwd failed: %d" % rc)
    return (o, lse, p) if return_probs else (o, lse)


def attn_fwd_fp8(q, k, v, scale: float, descale_q: float = 1.0, descale_k: float = 1.0, descale_v: float = 1.0,
                 causal: bool = False, window_left: int = -1, window_right: int = -1, alibi_slopes=None,
                 softcap: float = 0.0, rows: Optional[Sequence[int]] = None, num_threads: int = 0,
                 dtype_code: Optional[int] = None):
    """Attention on 8-bit inputs (the FP8 forward named in "FlashAttention深度解析：
    从算法创新到产业变革的全面影响", section 未来展望, and "IO感知技术革命", section
    H100架构的性能跃升; neither states the form): q, k, v hold E4M3 or E5M2
    values x8 standing for x8 * descale_x, so the result is attn_fwd of the
    dequantised inputs: the score scale becomes scale * descale_q * descale_k
    and O is multiplied by descale_v (O is linear in V; LSE is unchanged).
    Returns (o, lse) as attn_fwd."""
    qa, code = _as_storage(q, dtype_code)
    ka, kc = _as_storage(k, dtype_code)
    va, vc = _as_storage(v, dtype_code)
    if code not in (E4M3, E5M2) or not (code == kc == vc):
        raise ValueError("q, k, v must share one 8-bit storage type")
    o, lse = attn_fwd(qa, ka, va, float(scale) * float(descale_q) * float(descale_k), causal, window_left,
                      window_right, alibi_slopes, softcap, rows=rows, num_threads=num_threads, dtype_code=code)
    return o * float(descale_v), lse


def _expand_heads(a: np.ndarray, H: int, axis: int) -> np.ndarray:
    """Repeats each of the a.shape[axis] = H_kv heads H / H_kv times, so that
    query head h meets K/V head h // (H / H_kv)."""
    H_kv = a.shape[axis]
    if H_kv < 1 or H % H_kv:
        raise ValueError("H must be a multiple of the K/V head count")
    return np.ascontiguousarray(np.repeat(a, H // H_kv, axis=axis))


def attn_fwd_gqa(q, k, v, scale: float, causal: bool = False, window_left: int = -1,
                 window_right: int = -1, alibi_slopes=None, softcap: float = 0.0,
                 rows: Optional[Sequence[int]] = None, num_threads: int = 0,
                 dtype_code: Optional[int] = None):
    """Grouped-query attention: q [B,Nq,H,d], k/v [B,Nk,H_kv,d]; query head h
    attends with K/V head h // (H / H_kv) (the pages do not define the form;
    this is the plain reading). Returns (o [B,R,H,d], lse [B,H,R])."""
    qa, code = _as_storage(q, dtype_code)
    ka, kc = _as_storage(k, dtype_code)
    va, vc = _as_storage(v, dtype_code)
    H = qa.shape[2]
    return attn_fwd(qa, _expand_heads(ka, H, 2), _expand_heads(va, H, 2), scale, causal, window_left, window_right,
                    alibi_slopes, softcap, rows=rows, num_threads=num_threads, dtype_code=code)


def attn_fwd_qkvpacked(qkv, scale: float, causal: bool = False, window_left: int = -1, window_right: int = -1,
                       alibi_slopes=None, softcap: float = 0.0, rows: Optional[Sequence[int]] = None,
                       num_threads: int = 0, dtype_code: Optional[int] = None):
    """Packed layout of "FlashAttention深度解析：从算法创新到产业变革的全面影响"
    (flash_attn_qkvpacked_func): qkv [B,N,3,H,d] with slot 0 = q, 1 = k,
    2 = v; attention as attn_fwd on the three slots."""
    a, code = _as_storage(qkv, dtype_code)
    if a.ndim != 5 or a.shape[2] != 3:
        raise ValueError("qkv must be [B, N, 3, H, d]")
    q, k, v = (np.ascontiguousarray(a[:, :, i]) for i in range(3))
    return attn_fwd(q, k, v, scale, causal, window_left, window_right, alibi_slopes, softcap, rows=rows,
                    num_threads=num_threads, dtype_code=code)


def attn_fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, scale: float, causal: bool = False,
                    window_left: int = -1, window_right: int = -1, alibi_slopes=None, softcap: float = 0.0,
                    num_threads: int = 0, dtype_code: Optional[int] = None):
    """Packed variable-length attention. q [total_q,H,d], k/v [total_k,H,d];
    sequence b owns query rows cu_seqlens_q[b] .. cu_seqlens_q[b+1]-1 and
    key rows cu_seqlens_k[b] .. cu_seqlens_k[b+1]-1, and is attended on its
    own by the plain definition (attn_fwd with B = 1 and its own Nq, Nk).
    "FlashAttention深度解析：从算法创新到产业变革的全面影响" (section 未来展望)
    names variable sequence lengths without a formula; this is the reading
    that each sequence is its own problem.

    Returns (o [total_q,H,d], lse [H,total_q]); rows outside every sequence
    are NaN.
    """
    qa, code = _as_storage(q, dtype_code)
    ka, kc = _as_storage(k, dtype_code)
    va, vc = _as_storage(v, dtype_code)
    if not (code == kc == vc):
        raise ValueError("q, k, v must share one storage type")
    total_q, H, d = qa.shape
    total_k = ka.shape[0]
    if ka.shape != (total_k, H, d) or va.shape != ka.shape:
        raise ValueError("shape mismatch")
    cq = [int(x) for x in np.asarray(cu_seqlens_q).reshape(-1)]
    ck = [int(x) for x in np.asarray(cu_seqlens_k).reshape(-1)]
    if len(cq) != len(ck) or len(cq) < 1:
        raise ValueError("cu_seqlens_q and cu_seqlens_k need B + 1 entries each")
    o = np.full((total_q, H, d), np.nan)
    lse = np.full((H, total_q), np.nan)
    for b in range(len(cq) - 1):
        q0, q1, k0, k1 = cq[b], cq[b + 1], ck[b], ck[b + 1]
        if not (0 <= q0 <= q1 <= total_q and 0 <= k0 <= k1 <= total_k):
            raise ValueError("cu_seqlens entry %d out of range" % b)
        if q1 == q0:
            continue
        ob, lb = attn_fwd(qa[q0:q1][None], ka[k0:k1][None], va[k0:k1][None], scale, causal, window_left,
                          window_right, alibi_slopes, softcap, num_threads=num_threads, dtype_code=code)
        o[q0:q1] = ob[0]
        lse[:, q0:q1] = lb[0]
    return o, lse


def attn_decode_paged(q, k_cache, v_cache, block_table, cache_seqlens, scale: float,
                      window_left: int = -1, alibi_slopes=None, softcap: float = 0.0,
                      batch: Optional[Sequence[int]] = None, num_splits: int = 1,
                      num_threads: int = 0, dtype_code: Optional[int] = None):
    """Paged decode. q [B,1,H,d]; caches [num_pages,page_size,H,d].

    num_splits <= 1: returns (o [R,1,H,d], lse [R,H,1]).
    num_splits > 1: returns the split partials (o [S,R,H,d], lse [S,R,H]).
    R is len(batch) (all B sequences when batch is None).
    """
    qa, code = _as_storage(q, dtype_code)
    ka, kc = _as_storage(k_cache, dtype_code)
    va, vc = _as_storage(v_cache, dtype_code)
    if not (code == kc == vc):
        raise ValueError("q and caches must share one storage type")
    B, one, H, d = qa.shape
    num_pages, page_size = ka.shape[0], ka.shape[1]
    if one != 1 or ka.shape != (num_pages, page_size, H, d) or va.shape != ka.shape:
        raise ValueError("shape mismatch")
    bt = _i32_vec(block_table)
    sl = _i32_vec(cache_seqlens)
    max_blocks = bt.shape[1]
    bsel = _i32_vec(batch)
    R = B if bsel is None else len(bsel)
    S = max(1, int(num_splits))
    if S > 1:
        o = np.empty((S, R, H, d), dtype=np.float64)
        lse = np.empty((S, R, H), dtype=np.float64)
    else:
        o = np.empty((R, 1, H, d), dtype=np.float64)
        lse = np.empty((R, H, 1), dtype=np.float64)
    slopes = _f64_vec(alibi_slopes)
    rc = lib().oracle_attn_decode_paged(qa.ctypes.data, ka.ctypes.data, va.ctypes.data, code,
                                        _iptr(bt), _iptr(sl), _dptr(o), _dptr(lse), B, H, d,
                                        num_pages, page_size, max_blocks, float(scale),
                                        int(window_left), _dptr(slopes), float(softcap),
                                        _iptr(bsel), R, S, int(num_threads))
    if rc:
        raise ValueError("oracle_attn_decode_paged failed: %d" % rc)
    return o, lse


def attn_decode_paged_gqa(q, k_cache, v_cache, block_table, cache_seqlens, scale: float,
                          window_left: int = -1, alibi_slopes=None, softcap: float = 0.0,
                          batch: Optional[Sequence[int]] = None, num_splits: int = 1,
                          num_threads: int = 0, dtype_code: Optional[int] = None):
    """Grouped-query paged decode: q [B,1,H,d]; caches [num_pages,page_size,H_kv,d];
    query head h reads cache head h // (H / H_kv). Returns as attn_decode_paged."""
    qa, code = _as_storage(q, dtype_code)
    ka, _ = _as_storage(k_cache, dtype_code)
    va, _ = _as_storage(v_cache, dtype_code)
    H = qa.shape[2]
    return attn_decode_paged(qa, _expand_heads(ka, H, 2), _expand_heads(va, H, 2), block_table, cache_seqlens,
                             scale, window_left, alibi_slopes, softcap, batch=batch, num_splits=num_splits,
                             num_threads=num_threads, dtype_code=code)


def kvcache_append(k_new, v_new, k_cache, v_cache, block_table, cache_seqlens):
    """Returns copies of the caches with the new tokens written in: token i of
    sequence b goes to position t = cache_seqlens[b] + i, i.e. row
    t % page_size of page block_table[b][t // page_size] ("Flash-Attention
    v2.0 到 v2.7 更新", v2.5; "解密FlashAttention：如何让大语言模型推理速度翻倍",
    section 智能緩存機制); positions past
    the table and entries outside [0, num_pages) are skipped. Works on the
    raw storage (any element type), so the result is bit-exact."""
    kn, vn = np.asarray(k_new), np.asarray(v_new)
    kc, vc = np.array(k_cache, copy=True), np.array(v_cache, copy=True)
    bt = np.asarray(block_table, dtype=np.int64)
    sl = np.asarray(cache_seqlens, dtype=np.int64).reshape(-1)
    B, n_new = kn.shape[0], kn.shape[1]
    num_pages, page = kc.shape[0], kc.shape[1]
    cap = bt.shape[1] * page
    for b in range(B):
        for i in range(n_new):
            t = int(sl[b]) + i
            if sl[b] < 0 or t >= cap:
                continue
            pg = int(bt[b, t // page])
            if not 0 <= pg < num_pages:
                continue
            kc[pg, t % page] = kn[b, i]
            vc[pg, t % page] = vn[b, i]
    return kc, vc


def attn_bwd(q, k, v, dout, scale: float, causal: bool = False, window_left: int = -1,
             window_right: int = -1, alibi_slopes=None, softcap: float = 0.0,
             num_threads: int = 0, dtype_code: Optional[int] = None):
    """Gradients of L = sum(dout * O) with respect to q, k and v, where O is
    attn_fwd's output (grouped-query when k, v have fewer heads than q).

    The pages name the backward pass ("FlashAttention深度解析：从算法创新到产业
    变革的全面影响", section 技术演进, version 2.4; "Flash-Attention v2.0 到 v2.7
    更新", section v2.4: a deterministic backward) but give no formulas, so
    this is the chain rule through attn_fwd's definition, per (b, h):
      dV = P^T dO;  dP = dO V^T
      dZ_ij = P_ij (dP_ij - sum_k P_ik dP_ik)         (softmax Jacobian)
      dS_ij = dZ_ij * (1 - tanh(s_ij / c)^2)          if softcap c > 0, else dZ_ij
      dQ = scale * dS K;  dK = scale * dS^T Q
    with s_ij = scale * q_i . k_j and P the probabilities of attn_fwd (masked
    entries 0; the ALiBi term does not depend on q or k). Grouped-query K/V
    heads receive the sum over the query heads that read them.

    q, dout [B,Nq,H,d]; k, v [B,Nk,H_kv,d]. Returns (dq, dk, dv) as fp64
    arrays of the input shapes.
    """
    qa, code = _as_storage(q, dtype_code)
    ka, kc = _as_storage(k, dtype_code)
    va, vc = _as_storage(v, dtype_code)
    da, dc = _as_storage(dout, dtype_code)
    if not (code == kc == vc == dc):
        raise ValueError("q, k, v, dout must share one storage type")
    B, Nq, H, d = qa.shape
    Nk, H_kv = ka.shape[1], ka.shape[2]
    if da.shape != qa.shape or va.shape != ka.shape or ka.shape[0] != B or ka.shape[3] != d:
        raise ValueError("shape mismatch")
    ke, ve = _expand_heads(ka, H, 2), _expand_heads(va, H, 2)
    _, _, P = attn_fwd(qa, ke, ve, scale, causal, window_left, window_right, alibi_slopes, softcap,
                       return_probs=True, num_threads=num_threads, dtype_code=code)
    Q, K, V, DO = widen(qa, code), widen(ke, code), widen(ve, code), widen(da, code)
    dq = np.zeros((B, Nq, H, d))
    dk = np.zeros((B, Nk, H, d))
    dv = np.zeros((B, Nk, H, d))
    for b in range(B):
        for h in range(H):
            p = np.nan_to_num(P[b, h], nan=0.0)   # rows with no visible key carry no gradient
            qh, kh, vh, doh = Q[b, :, h], K[b, :, h], V[b, :, h], DO[b, :, h]
            dv[b, :, h] = p.T @ doh
            dp = doh @ vh.T
            dz = p * (dp - np.sum(p * dp, axis=1, keepdims=True))
            if softcap > 0.0:
                t = np.tanh(scale * (qh @ kh.T) / softcap)
                dz = dz * (1.0 - t * t)
            dq[b, :, h] = scale * (dz @ kh)
            dk[b, :, h] = scale * (dz.T @ qh)
    G = H // H_kv
    dk = dk.reshape(B, Nk, H_kv, G, d).sum(axis=3)
    dv = dv.reshape(B, Nk, H_kv, G, d).sum(axis=3)
    return dq, dk, dv


def combine_splits(o_part: np.ndarray, lse_part: np.ndarray):
    """Merge of split partials: o_part [S, ..., d], lse_part [S, ...]."""
    S = o_part.shape[0]
    d = o_part.shape[-1]
    rest = lse_part.shape[1:]
    n = int(np.prod(rest)) if rest else 1
    op = np.ascontiguousarray(o_part, dtype=np.float64).reshape(S, n, d)
    lp = np.ascontiguousarray(lse_part, dtype=np.float64).reshape(S, n)
    o = np.empty((n, d), dtype=np.float64)
    lse = np.empty((n,), dtype=np.float64)
    rc = lib().oracle_combine_splits(_dptr(op), _dptr(lp), S, n, d, _dptr(o), _dptr(lse))
    if rc:
        raise ValueError("oracle_combine_splits failed: %d" % rc)
    return o.reshape(rest + (d,)), lse.reshape(rest)
