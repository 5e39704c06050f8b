"""GPU parity of the grouped-query entry points and of the cache append
(through the C ABI) against the fp64 oracle.

fa_fwd_gqa and fa_fwd_kvcache_gqa use the forward / decode tolerances
(tests/parity.py); the append is a
copy and must match the oracle's scatter bit for bit, everywhere in the
caches.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import exact_io_aware_79_b200 as fa
from exact_io_aware_79_b200 import workloads as W
from tests import parity

pytestmark = pytest.mark.gpu


def compare(out, lse, o_ref, l_ref, dtype, what):
    return parity.check(out, lse, o_ref, l_ref, dtype, "gqa " + what)


FWD = [
    # (B, H, H_kv, Nq, Nk, d, dtype, causal, wl, wr, alibi, cap, sigma)
    (2, 8, 2, 300, 300, 128, torch.bfloat16, True, -1, -1, False, 0.0, 1.0),
    (1, 4, 1, 257, 513, 64, torch.float16, True, -1, -1, False, 0.0, 1.0),
    (1, 6, 3, 640, 640, 128, torch.bfloat16, True, 100, 0, True, 50.0, 2.0),
    (2, 4, 4, 129, 200, 128, torch.float16, False, -1, -1, False, 0.0, 1.0),
]


@pytest.mark.parametrize("case", FWD, ids=lambda c: "B%dH%dkv%dq%dk%dd%d_%s" % (c[:6] + (str(c[6])[6:],)))
def test_forward_gqa_matches_oracle(case):
    B, H, H_kv, Nq, Nk, d, dtype, causal, wl, wr, alibi, cap, sigma = case
    g = torch.Generator().manual_seed(Nq + 3 * H)
    q = (torch.randn(B, Nq, H, d, generator=g) * sigma).to(dtype)
    k = (torch.randn(B, Nk, H_kv, d, generator=g) * sigma).to(dtype)
    v = (torch.randn(B, Nk, H_kv, d, generator=g) * sigma).to(dtype)
    slopes = W.alibi_slopes(H) if alibi else None
    scale = 1.0 / math.sqrt(d)
    out = torch.empty_like(q, device="cuda")
    lse = torch.empty(B, H, Nq, dtype=torch.float32, device="cuda")
    fa.fa_fwd_gqa(q.cuda(), k.cuda(), v.cuda(), out, lse, scale, causal, wl, wr,
                  None if slopes is None else slopes.cuda(), cap)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.attn_fwd_gqa(q, k, v, scale, causal, wl, wr, slopes, cap)
    compare(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, dtype, str(case))


def decode_inputs(B, H, H_kv, d, page, mb, lens, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    num_pages = B * mb
    kc = torch.randn(num_pages, page, H_kv, d, generator=g).to(dtype)
    vc = torch.randn(num_pages, page, H_kv, d, generator=g).to(dtype)
    table = torch.randperm(num_pages, generator=g).view(B, mb).to(torch.int32)
    q = torch.randn(B, 1, H, d, generator=g).to(dtype)
    return q, kc, vc, table, torch.tensor(lens, dtype=torch.int32)


def run_decode_gqa(q, kc, vc, table, lens, scale, splits=0, wl=-1, slopes=None, cap=0.0):
    B, _, H, d = q.shape
    mb, page = table.shape[1], kc.shape[1]
    nbytes = fa.fa_kvcache_workspace_size(B, H, d, mb, page, splits)
    ws = torch.empty(max(nbytes, 16), dtype=torch.uint8, device="cuda")
    out = torch.empty(q.shape, dtype=q.dtype, device="cuda")
    lse = torch.empty(B, H, 1, dtype=torch.float32, device="cuda")
    fa.fa_fwd_kvcache_gqa(q.cuda(), kc.cuda(), vc.cuda(), table.cuda(), lens.cuda(), out, lse, scale, wl,
                          None if slopes is None else slopes.cuda(), cap, splits, ws)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), lse.cpu().numpy()


DEC = [
    # (B, H, H_kv, d, page, mb, lens, dtype, wl, alibi, cap)
    (3, 8, 2, 128, 256, 8, (2048, 300, 1), torch.bfloat16, -1, False, 0.0),
    (2, 4, 1, 64, 16, 20, (320, 77), torch.float16, -1, False, 0.0),
    (4, 6, 3, 128, 64, 12, (700, 0, 65, 768), torch.bfloat16, 100, False, 0.0),
    (2, 8, 2, 128, 256, 6, (1500, 257), torch.bfloat16, -1, True, 30.0),     # four heads a CTA, ALiBi + softcap
    (2, 4, 2, 64, 64, 10, (600, 90), torch.float16, 200, True, 0.0),         # two heads a CTA, ALiBi, window
    (2, 8, 1, 128, 128, 4, (500, 33), torch.bfloat16, -1, False, 5.0),       # MQA, eight heads a CTA, softcap
    (2, 32, 1, 128, 64, 6, (350, 129), torch.bfloat16, -1, True, 20.0),      # MQA, 16 heads a CTA (both row halves)
    (2, 12, 1, 64, 64, 5, (300, 64), torch.float16, -1, False, 0.0),         # 12 heads a CTA
    (2, 6, 2, 128, 128, 3, (380, 1), torch.bfloat16, 50, False, 0.0),        # an odd group of 3, window
]


@pytest.mark.parametrize("splits", [0, 1, 3, 8])
@pytest.mark.parametrize("case", DEC, ids=lambda c: "B%dH%dkv%dd%dp%d_a%d_s%g" % (c[:5] + (c[9], c[10])))
def test_decode_gqa_matches_oracle(case, splits):
    B, H, H_kv, d, page, mb, lens, dtype, wl, alibi, cap = case
    q, kc, vc, table, lens_t = decode_inputs(B, H, H_kv, d, page, mb, lens, dtype, seed=sum(lens) + H)
    slopes = W.alibi_slopes(H) if alibi else None
    scale = 1.0 / math.sqrt(d)
    out, lse = run_decode_gqa(q, kc, vc, table, lens_t, scale, splits, wl, slopes, cap)
    o_ref, l_ref = oracle.attn_decode_paged_gqa(q, kc, vc, table, lens_t, scale, wl, slopes, cap)
    compare(out, lse, o_ref, l_ref, dtype, "%s splits=%d" % (case, splits))


def test_append_matches_the_scatter_bit_for_bit():
    B, n_new, H_kv, d, page, mb = 5, 7, 2, 128, 16, 6
    g = torch.Generator().manual_seed(91)
    num_pages = B * mb
    kc = torch.randn(num_pages, page, H_kv, d, generator=g).to(torch.bfloat16)
    vc = torch.randn(num_pages, page, H_kv, d, generator=g).to(torch.bfloat16)
    table = torch.randperm(num_pages, generator=g).view(B, mb).to(torch.int32)
    table[3, 2] = num_pages + 5      # an entry outside the pool: its positions are skipped
    lens = torch.tensor([0, 15, 40, 30, 92], dtype=torch.int32)   # the last one ends past the table (96 slots)
    kn = torch.randn(B, n_new, H_kv, d, generator=g).to(torch.bfloat16)
    vn = torch.randn(B, n_new, H_kv, d, generator=g).to(torch.bfloat16)
    kd, vd = kc.cuda(), vc.cuda()
    fa.fa_kvcache_append(kn.cuda(), vn.cuda(), kd, vd, table.cuda(), lens.cuda())
    torch.cuda.synchronize()
    view = lambda t: t.view(torch.int16).numpy()
    k_ref, v_ref = oracle.kvcache_append(view(kn), view(vn), view(kc), view(vc), table.numpy(), lens.numpy())
    assert np.array_equal(view(kd.cpu()), k_ref)
    assert np.array_equal(view(vd.cpu()), v_ref)


def test_append_then_decode_sees_the_new_tokens():
    B, H, H_kv, d, page, mb = 2, 4, 2, 128, 64, 4
    q, kc, vc, table, lens = decode_inputs(B, H, H_kv, d, page, mb, (100, 63), torch.bfloat16, seed=5)
    g = torch.Generator().manual_seed(6)
    kn = torch.randn(B, 3, H_kv, d, generator=g).to(torch.bfloat16)
    vn = torch.randn(B, 3, H_kv, d, generator=g).to(torch.bfloat16)
    kd, vd = kc.cuda(), vc.cuda()
    fa.fa_kvcache_append(kn.cuda(), vn.cuda(), kd, vd, table.cuda(), lens.cuda())
    lens2 = lens + 3
    out, lse = run_decode_gqa(q, kd.cpu(), vd.cpu(), table, lens2, 0.1)
    k2, v2 = oracle.kvcache_append(kn.view(torch.int16).numpy(), vn.view(torch.int16).numpy(),
                                   kc.view(torch.int16).numpy(), vc.view(torch.int16).numpy(), table.numpy(),
                                   lens.numpy())
    o_ref, l_ref = oracle.attn_decode_paged_gqa(q, k2, v2, table, lens2, 0.1, dtype_code=oracle.BF16)
    compare(out, lse, o_ref, l_ref, torch.bfloat16, "append + decode")


def test_full_size_gqa_decode_sampled_sequences():
    w = W.DECODE_GQA
    xd = W.make_decode_inputs(w, device="cuda")
    B, H, d = w.B, w.H, w.d
    S = fa.fa_kvcache_num_splits_gqa(B, H, w.H_kv, d, w.max_blocks, w.page_size, 0)
    ws = torch.empty(max(fa.fa_kvcache_workspace_size(B, H, d, w.max_blocks, w.page_size, 0), 16),
                     dtype=torch.uint8, device="cuda")
    out = torch.empty_like(xd["q"])
    lse = torch.empty(B, H, 1, dtype=torch.float32, device="cuda")
    fa.fa_fwd_kvcache_gqa(xd["q"], xd["k_cache"], xd["v_cache"], xd["block_table"], xd["cache_seqlens"], out, lse,
                          w.scale, -1, None, 0.0, 0, ws)
    torch.cuda.synchronize()
    lens = xd["cache_seqlens"].cpu()
    table = xd["block_table"].cpu()
    picks = sorted({int(lens.argmin()), int(lens.argmax()), 17})
    for b in picks:
        n_pages = -(-int(lens[b]) // w.page_size)
        pages = table[b, :n_pages].long().cuda()
        kc = xd["k_cache"][pages].cpu()          # this sequence's pages, in order
        vc = xd["v_cache"][pages].cpu()
        ident = torch.arange(n_pages, dtype=torch.int32).view(1, n_pages)
        o_ref, l_ref = oracle.attn_decode_paged_gqa(xd["q"][b:b + 1].cpu(), kc, vc, ident, lens[b:b + 1], w.scale)
        compare(out[b:b + 1].float().cpu().numpy(), lse[b:b + 1].cpu().numpy(), o_ref, l_ref, w.dtype,
                "sequence %d (splits %d)" % (b, S))


@pytest.mark.parametrize("H_kv", [8, 2, 1])
def test_decode_staged_invalid_table_entry_and_length_give_nan_rows(H_kv):
    """Page size 64 (the TMA-staged kernels, one head or a group a CTA): a
    table entry past the pool and a length past the table are never
    dereferenced; those sequences' rows become NaN and the others match the
    oracle."""
    B, H, d, page, mb = 4, 8, 128, 64, 4
    q, kc, vc, table, lens = decode_inputs(B, H, H_kv, d, page, mb, (100, 200, 60, 7), torch.bfloat16, seed=9)
    bad_table = table.clone()
    bad_table[1, 2] = 10**6          # inside sequence 1's 200 tokens
    bad_lens = lens.clone()
    bad_lens[2] = mb * page + 1
    for splits in (1, 4):
        out, lse = run_decode_gqa(q, kc, vc, bad_table, bad_lens, 0.1, splits)
        assert np.isnan(out[1]).all() and np.isnan(lse[1]).all()
        assert np.isnan(out[2]).all() and np.isnan(lse[2]).all()
        good = [0, 3]
        o_ref, l_ref = oracle.attn_decode_paged_gqa(q[good], kc, vc, table[good], lens[good], 0.1)
        compare(out[good], lse[good], o_ref, l_ref, torch.bfloat16, "good rows, splits=%d" % splits)
