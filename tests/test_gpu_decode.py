"""GPU parity of fa_fwd_kvcache (through the C ABI) against the fp64 oracle.

Same tolerances as the forward (tests/parity.py). Block-table indexing is checked bit-exactly
with one-hot probes whose expected output is an integer code of the probed
token's logical index.
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


def case_inputs(B, H, d, page, max_blocks, lens, dtype, seed, sigma=1.0):
    g = torch.Generator().manual_seed(seed)
    num_pages = B * max_blocks
    kc = (torch.randn(num_pages, page, H, d, generator=g) * sigma).to(dtype)
    vc = (torch.randn(num_pages, page, H, d, generator=g) * sigma).to(dtype)
    table = torch.randperm(num_pages, generator=g).view(B, max_blocks).to(torch.int32)
    q = (torch.randn(B, 1, H, d, generator=g) * sigma).to(dtype)
    return q, kc, vc, table, torch.tensor(lens, dtype=torch.int32)


def run_gpu(q, kc, vc, table, lens, scale, wl=-1, slopes=None, cap=0.0, splits=0):
    c = lambda t: None if t is None else t.cuda()
    out, lse = fa.decode(c(q), c(kc), c(vc), c(table), c(lens), scale, wl, c(slopes), cap, splits)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), lse.cpu().numpy()


def compare(out, lse, o_ref, l_ref, dtype, what):
    return parity.check(out, lse, o_ref, l_ref, dtype, "decode " + what)


CASES = [
    # (B, H, d, page, max_blocks, lens, dtype, wl, alibi, cap, sigma)
    (3, 2, 128, 16, 20, (37, 320, 1), torch.bfloat16, -1, False, 0.0, 1.0),
    (4, 3, 64, 16, 9, (0, 5, 144, 100), torch.float16, -1, False, 0.0, 1.0),
    (2, 4, 128, 256, 8, (2048, 1500), torch.bfloat16, -1, True, 50.0, 2.0),
    (2, 2, 128, 256, 8, (2048, 777), torch.bfloat16, 300, False, 0.0, 1.0),
    (3, 2, 64, 32, 10, (320, 33, 17), torch.bfloat16, 40, True, 0.0, 1.0),
    (2, 2, 128, 256, 16, (4096, 3000), torch.float16, -1, False, 5.0, 1.5),
    (2, 3, 64, 64, 12, (700, 65), torch.bfloat16, -1, False, 0.0, 1.0),
    (3, 2, 128, 128, 6, (500, 129, 768), torch.float16, 100, True, 0.0, 1.0),
]


@pytest.mark.parametrize("splits", [0, 1, 2, 3, 4, 8, 16, 64])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dH%dd%dp%d_%s_w%d_a%d_s%g" % (
    c[0], c[1], c[2], c[3], str(c[6])[6:], c[7], c[8], c[9]))
def test_decode_matches_oracle(case, splits):
    B, H, d, page, mb, lens, dtype, wl, alibi, cap, sigma = case
    q, kc, vc, table, lens_t = case_inputs(B, H, d, page, mb, lens, dtype, seed=sum(lens) + d, sigma=sigma)
    slopes = W.alibi_slopes(H) if alibi else None
    scale = 1.0 / math.sqrt(d)
    out, lse = run_gpu(q, kc, vc, table, lens_t, scale, wl, slopes, cap, splits)
    o_ref, l_ref = oracle.attn_decode_paged(q, kc, vc, table, lens_t, scale, wl, slopes, cap)
    compare(out, lse, o_ref, l_ref, dtype, "%s splits=%d" % (case, splits))


def test_identity_table_equals_contiguous_forward():
    """Paged decode with an identity block table equals fa_fwd of the single
    query over the contiguous keys (both on the GPU, both against the oracle)."""
    B, H, d, page, mb = 2, 2, 128, 64, 8
    g = torch.Generator().manual_seed(11)
    k = torch.randn(B, mb * page, H, d, generator=g).to(torch.bfloat16)
    v = torch.randn(B, mb * page, H, d, generator=g).to(torch.bfloat16)
    q = torch.randn(B, 1, H, d, generator=g).to(torch.bfloat16)
    lens = torch.tensor([mb * page, 300], dtype=torch.int32)
    table = torch.arange(B * mb, dtype=torch.int32).view(B, mb)
    out, lse = run_gpu(q, k.view(B * mb, page, H, d), v.view(B * mb, page, H, d), table, lens, 0.1)
    for b in range(B):
        L = int(lens[b])
        o2, l2 = fa.attention(q[b:b + 1].cuda(), k[b:b + 1, :L].cuda(), v[b:b + 1, :L].cuda(), 0.1, causal=True)
        assert np.abs(out[b] - o2[0].float().cpu().numpy()).max() <= parity.O_SPEC[torch.bfloat16]
        assert np.abs(lse[b] - l2[0].cpu().numpy()).max() <= parity.LSE_SPEC


@pytest.mark.parametrize("splits", [1, 16])
def test_full_size_decode_on_sampled_sequences(splits):
    w = W.DECODE
    x = W.make_decode_inputs(w, device="cuda")
    out, lse = fa.decode(x["q"], x["k_cache"], x["v_cache"], x["block_table"], x["cache_seqlens"], w.scale,
                         num_splits=splits)
    torch.cuda.synchronize()
    assert torch.isfinite(out).all().item() and torch.isfinite(lse).all().item()
    lens = x["cache_seqlens"].cpu()
    picks = [int(torch.argmax(lens)), int(torch.argmin(lens)), 5, 37]
    # compact the referenced pages so the oracle reads only what it needs
    table = x["block_table"].cpu()
    used = sorted({int(p) for b in picks for p in table[b, :(int(lens[b]) + w.page_size - 1) // w.page_size]})
    remap = {p: i for i, p in enumerate(used)}
    idx = torch.tensor(used, device="cuda")
    kc = x["k_cache"].index_select(0, idx).cpu()
    vc = x["v_cache"].index_select(0, idx).cpu()
    sub_table = torch.zeros(len(picks), w.max_blocks, dtype=torch.int32)
    for r, b in enumerate(picks):
        n = (int(lens[b]) + w.page_size - 1) // w.page_size
        sub_table[r, :n] = torch.tensor([remap[int(p)] for p in table[b, :n]], dtype=torch.int32)
    sub_lens = lens[picks]
    o_ref, l_ref = oracle.attn_decode_paged(x["q"][picks].cpu(), kc, vc, sub_table, sub_lens, w.scale)
    compare(out[picks].float().cpu().numpy(), lse[picks].cpu().numpy(), o_ref, l_ref, w.dtype, "full decode")


@pytest.mark.parametrize("splits", [1, 5, 16])
def test_one_hot_probes_pin_block_table_indexing(splits):
    """For every (sequence, head) one logical token t gets K = 256 e0 while
    every other K is 0, and q = e0 with scale 1: the softmax collapses onto t
    exactly, and V holds the code (t // 64, t % 64) of each token's logical
    index, so O must equal t's code bit for bit."""
    B, H, d, page, mb = 6, 8, 128, 16, 40
    g = torch.Generator().manual_seed(21)
    lens = torch.tensor([640, 1, 17, 333, 600, 256], dtype=torch.int32)
    num_pages = B * mb
    table = torch.randperm(num_pages, generator=g).view(B, mb).to(torch.int32)
    kc = torch.zeros(num_pages, page, H, d)
    vc = torch.zeros(num_pages, page, H, d)
    for b in range(B):
        for t in range(int(lens[b])):
            pg, row = int(table[b, t // page]), t % page
            vc[pg, row, :, 0] = t // 64
            vc[pg, row, :, 1] = t % 64
    targets = torch.zeros(B, H, dtype=torch.int64)
    for b in range(B):
        targets[b] = torch.randint(0, int(lens[b]), (H,), generator=g)
        for h in range(H):
            t = int(targets[b, h])
            kc[int(table[b, t // page]), t % page, h, 0] = 256.0
    q = torch.zeros(B, 1, H, d)
    q[..., 0] = 1.0
    bf = torch.bfloat16
    out, lse = run_gpu(q.to(bf), kc.to(bf), vc.to(bf), table, lens, 1.0, splits=splits)
    want0 = (targets // 64).numpy().astype(np.float32)
    want1 = (targets % 64).numpy().astype(np.float32)
    assert np.array_equal(out[:, 0, :, 0], want0)
    assert np.array_equal(out[:, 0, :, 1], want1)
    assert np.all(out[:, 0, :, 2:] == 0)


def test_invalid_table_entry_and_length_give_nan_rows():
    """Out-of-range device-side values are never dereferenced; the affected
    sequence's outputs become NaN and the others are untouched."""
    q, kc, vc, table, lens = case_inputs(4, 2, 128, 16, 8, (40, 100, 60, 7), torch.bfloat16, seed=5)
    bad_table = table.clone()
    bad_table[1, 3] = 10**6          # page index past the pool, inside sequence 1's length
    bad_lens = lens.clone()
    bad_lens[2] = 8 * 16 + 1         # longer than max_blocks * page_size
    for splits in (1, 4):
        out, lse = run_gpu(q, kc, vc, bad_table, bad_lens, 0.1, splits=splits)
        assert np.isnan(out[1]).all() and np.isnan(lse[1]).all()
        assert np.isnan(out[2]).all() and np.isnan(lse[2]).all()
        good = [0, 3]
        o_ref, l_ref = oracle.attn_decode_paged(q[good], kc, vc, table[good], lens[good], 0.1)
        compare(out[good], lse[good], o_ref, l_ref, torch.bfloat16, "good rows")
