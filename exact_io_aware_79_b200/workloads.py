"""Seeded synthetic workloads for the attention forward and the paged decode.

This module only draws inputs. It holds none of the attention arithmetic, so
both the CUDA path and the fp64 oracle can be fed from it without sharing any
of the method's code.

Workload recipe (the pages publish no dataset for this path, so every tensor
is synthetic):
  * Q, K, V are drawn i.i.d. N(0, 1) in fp32 from ``torch.Generator`` seeded
    per workload, multiplied by ``sigma`` and then rounded to fp16/bf16.
    Layout is [B, N, H, d], contiguous.
  * ALiBi slopes for head h of H heads are 2^(-8 (h + 1) / H).
  * The paged decode draws per-sequence cache lengths uniformly from
    [len_lo, len_hi] (inclusive), builds a K/V page pool of
    B * ceil(len_hi / page_size) pages of ``page_size`` tokens each and a
    block table that is a seeded random permutation of that pool, reshaped
    to [B, max_blocks].

Small workloads are drawn on the CPU. The full-size paged decode (34 GB of
K/V) is drawn directly on the device with a seeded CUDA generator; every
consumer (kernel and oracle) then reads the same tensor.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional

import torch


@dataclasses.dataclass(frozen=True)
class FwdWorkload:
    name: str
    B: int
    H: int
    Nq: int
    Nk: int
    d: int
    dtype: torch.dtype
    causal: bool = False
    window_left: int = -1
    window_right: int = -1
    alibi: bool = False
    softcap: float = 0.0
    sigma: float = 1.0
    seed: int = 0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    name: str
    B: int
    H: int
    d: int
    dtype: torch.dtype
    page_size: int
    len_lo: int
    len_hi: int
    window_left: int = -1
    alibi: bool = False
    softcap: float = 0.0
    sigma: float = 1.0
    seed: int = 4
    H_kv: int = 0  # cache heads (grouped-query attention); 0 means H

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def kv_heads(self) -> int:
        return self.H_kv or self.H

    @property
    def max_blocks(self) -> int:
        return -(-self.len_hi // self.page_size)

    @property
    def num_pages(self) -> int:
        return self.B * self.max_blocks


# The five workloads of the benchmark suite (tiny parity case, causal training
# shape, long sliding window and its Nq < Nk variant, ALiBi + softcap, paged
# decode).
TINY = FwdWorkload("tiny_fp16_b1h2n128d64", 1, 2, 128, 128, 64, torch.float16, seed=0)
CAUSAL_2K = FwdWorkload("causal_bf16_b8h16n2048d128", 8, 16, 2048, 2048, 128, torch.bfloat16,
                        causal=True, seed=1)
WINDOW_16K = FwdWorkload("window_bf16_b1h16n16384d128_wl4096", 1, 16, 16384, 16384, 128,
                         torch.bfloat16, causal=True, window_left=4096, window_right=0, seed=2)
WINDOW_Q4K_K16K = FwdWorkload("window_bf16_b1h16nq4096nk16384d128_wl4096", 1, 16, 4096, 16384, 128,
                              torch.bfloat16, causal=True, window_left=4096, window_right=0, seed=2)
CAUSAL_Q4K_K16K = FwdWorkload("causal_bf16_b1h16nq4096nk16384d128", 1, 16, 4096, 16384, 128,
                              torch.bfloat16, causal=True, seed=2)
ALIBI_SOFTCAP = FwdWorkload("alibi_softcap50_bf16_b4h32n4096d128", 4, 32, 4096, 4096, 128,
                            torch.bfloat16, causal=True, alibi=True, softcap=50.0, sigma=2.0, seed=3)
DECODE = DecodeWorkload("paged_decode_bf16_b64h32d128_page256", 64, 32, 128, torch.bfloat16,
                        page_size=256, len_lo=1024, len_hi=32768, seed=4)

# The decode workload with 4 sequences instead of 64 (same lengths law, pool of
# 512 pages = 2.1 GB of K/V): small enough for detailed profiler captures.
DECODE_SMALL = DecodeWorkload("paged_decode_bf16_b4h32d128_page256", 4, 32, 128, torch.bfloat16,
                              page_size=256, len_lo=1024, len_hi=32768, seed=4)

@dataclasses.dataclass(frozen=True)
class VarlenWorkload:
    """Packed sequences: B sequences with query and key lengths drawn
    uniformly from [len_lo, len_hi] (the same length for q and k)."""
    name: str
    B: int
    H: int
    d: int
    dtype: torch.dtype
    len_lo: int
    len_hi: int
    causal: bool = True
    sigma: float = 1.0
    seed: int = 5

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)


# Variable-length forward: 16 packed causal sequences of 256..4096 tokens
# (a training batch of documents of mixed length).
VARLEN = VarlenWorkload("varlen_causal_bf16_b16h16n256-4096d128", 16, 16, 128, torch.bfloat16, 256, 4096)

FWD_WORKLOADS = [TINY, CAUSAL_2K, WINDOW_16K, WINDOW_Q4K_K16K, CAUSAL_Q4K_K16K, ALIBI_SOFTCAP]
# Grouped-query decode: the same batch and lengths with 32 query heads over 8
# cache heads (groups of 4).
DECODE_GQA = DecodeWorkload("paged_decode_gqa_bf16_b64h32kv8d128_page256", 64, 32, 128, torch.bfloat16,
                            page_size=256, len_lo=1024, len_hi=32768, seed=4, H_kv=8)

# The grouped-query decode with 4 sequences (241 MB of unique K/V, above the
# 126 MB L2): the profiler-capture size of DECODE_GQA.
DECODE_GQA_SMALL = DecodeWorkload("paged_decode_gqa_bf16_b4h32kv8d128_page256", 4, 32, 128, torch.bfloat16,
                                  page_size=256, len_lo=1024, len_hi=32768, seed=4, H_kv=8)

DECODE_WORKLOADS = [DECODE, DECODE_SMALL, DECODE_GQA, DECODE_GQA_SMALL]


def alibi_slopes(H: int) -> torch.Tensor:
    """Per-head ALiBi slopes 2^(-8 (h + 1) / H), fp32, shape [H]."""
    h = torch.arange(H, dtype=torch.float64)
    return torch.pow(2.0, -8.0 * (h + 1.0) / H).to(torch.float32)


def _normal(shape, gen: torch.Generator, sigma: float, dtype: torch.dtype, device) -> torch.Tensor:
    x = torch.randn(*shape, generator=gen, dtype=torch.float32, device=device)
    if sigma != 1.0:
        x.mul_(sigma)
    return x.to(dtype)


def _normal_pages(shape, gen: torch.Generator, sigma: float, dtype: torch.dtype, device,
                  pages_per_draw: int = 256) -> torch.Tensor:
    """Like _normal for a page pool, drawn ``pages_per_draw`` pages at a time
    so the fp32 staging buffer stays small."""
    out = torch.empty(shape, dtype=dtype, device=device)
    for p0 in range(0, shape[0], pages_per_draw):
        p1 = min(shape[0], p0 + pages_per_draw)
        out[p0:p1] = _normal((p1 - p0,) + tuple(shape[1:]), gen, sigma, dtype, device)
    return out


def make_fwd_inputs(w: FwdWorkload, device="cpu", seed: Optional[int] = None):
    """Returns dict(q, k, v, slopes) for a forward workload.

    q is [B, Nq, H, d]; k, v are [B, Nk, H, d]; all ``w.dtype``; slopes is
    fp32 [H] or None. Values are drawn on the CPU so they do not depend on
    the device.
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(w.seed if seed is None else seed)
    q = _normal((w.B, w.Nq, w.H, w.d), gen, w.sigma, w.dtype, "cpu")
    k = _normal((w.B, w.Nk, w.H, w.d), gen, w.sigma, w.dtype, "cpu")
    v = _normal((w.B, w.Nk, w.H, w.d), gen, w.sigma, w.dtype, "cpu")
    slopes = alibi_slopes(w.H) if w.alibi else None
    out = dict(q=q.to(device), k=k.to(device), v=v.to(device),
               slopes=None if slopes is None else slopes.to(device))
    return out


def make_fwd_inputs_fp8(w: FwdWorkload, fmt: torch.dtype = torch.float8_e4m3fn, device="cpu",
                        seed: Optional[int] = None):
    """8-bit inputs for a forward workload: the fp32 draws of make_fwd_inputs
    (same seed, before rounding to w.dtype), each tensor scaled so that its
    largest magnitude maps to the format's largest finite value, then rounded
    to `fmt`. Returns dict(q, k, v, descale_q, descale_k, descale_v, slopes):
    element x8 stands for x8 * descale_x."""
    gen = torch.Generator(device="cpu")
    gen.manual_seed(w.seed if seed is None else seed)
    top = torch.finfo(fmt).max
    out = {}
    for name, n in (("q", w.Nq), ("k", w.Nk), ("v", w.Nk)):
        x = torch.randn((w.B, n, w.H, w.d), generator=gen, dtype=torch.float32) * w.sigma
        descale = float(x.abs().max()) / top if x.numel() else 1.0
        out[name] = (x / descale).to(fmt).to(device)
        out["descale_" + name] = descale
    slopes = alibi_slopes(w.H) if w.alibi else None
    out["slopes"] = None if slopes is None else slopes.to(device)
    return out


def make_varlen_inputs(w: VarlenWorkload, device="cpu", seed: Optional[int] = None):
    """Returns dict(q, k, v, cu_q, cu_k, max_q, max_k, lens).

    q, k, v are [total, H, d] (``w.dtype``); cu_q = cu_k are int32 [B + 1]
    row offsets; lens the B lengths (int64, CPU).
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(w.seed if seed is None else seed)
    lens = torch.randint(w.len_lo, w.len_hi + 1, (w.B,), generator=gen, dtype=torch.int64)
    cu = torch.zeros(w.B + 1, dtype=torch.int32)
    cu[1:] = torch.cumsum(lens, 0).to(torch.int32)
    total = int(cu[-1])
    q = _normal((total, w.H, w.d), gen, w.sigma, w.dtype, "cpu")
    k = _normal((total, w.H, w.d), gen, w.sigma, w.dtype, "cpu")
    v = _normal((total, w.H, w.d), gen, w.sigma, w.dtype, "cpu")
    return dict(q=q.to(device), k=k.to(device), v=v.to(device), cu_q=cu.to(device), cu_k=cu.clone().to(device),
                max_q=int(lens.max()), max_k=int(lens.max()), lens=lens)


def make_decode_inputs(w: DecodeWorkload, device="cpu", seed: Optional[int] = None,
                       seqlens: Optional[torch.Tensor] = None):
    """Returns dict(q, k_cache, v_cache, block_table, cache_seqlens, slopes).

    q is [B, 1, H, d]; k_cache, v_cache are [num_pages, page_size, H, d];
    block_table is int32 [B, max_blocks]; cache_seqlens is int32 [B].
    Integer tensors and q are drawn on the CPU; the K/V pool is drawn on
    ``device`` with a generator of that device (so the 34 GB pool of the
    full-size workload never passes through host memory).
    """
    s = w.seed if seed is None else seed
    gen = torch.Generator(device="cpu")
    gen.manual_seed(s)
    if seqlens is None:
        seqlens = torch.randint(w.len_lo, w.len_hi + 1, (w.B,), generator=gen, dtype=torch.int64)
    seqlens = seqlens.to(torch.int32)
    perm = torch.randperm(w.num_pages, generator=gen, dtype=torch.int64)
    block_table = perm.view(w.B, w.max_blocks).to(torch.int32)
    q = _normal((w.B, 1, w.H, w.d), gen, w.sigma, w.dtype, "cpu")
    dev = torch.device(device)
    kv_gen = torch.Generator(device=dev)
    kv_gen.manual_seed(s + 1000)
    shape = (w.num_pages, w.page_size, w.kv_heads, w.d)
    k_cache = _normal_pages(shape, kv_gen, w.sigma, w.dtype, dev)
    v_cache = _normal_pages(shape, kv_gen, w.sigma, w.dtype, dev)
    slopes = alibi_slopes(w.H) if w.alibi else None
    return dict(q=q.to(dev), k_cache=k_cache, v_cache=v_cache,
                block_table=block_table.to(dev), cache_seqlens=seqlens.to(dev),
                slopes=None if slopes is None else slopes.to(dev))
