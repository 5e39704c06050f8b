"""fa_fwd_kvcache_noalloc: the paged decode for callers that cannot allocate
device memory (no device allocator of their own, or a memory pool owned by
another runtime), which keeps its split partials in the library's fixed
device array instead of a caller workspace.

The GPU test calls it through the C ABI twice in a row, on different inputs,
and checks each result bit for bit against fa_fwd_kvcache (which runs the
same kernels with a caller-allocated workspace), and the first one against
the fp64 oracle with the decode tolerances (tests/parity.py), on 64- and
256-token pages. This file is named so pytest collects it last.
"""
import ctypes

import numpy as np
import pytest
import torch

import exact_io_aware_79_b200 as fa

P = 0x10000  # fake aligned device address; the rejection happens before any device use


def test_noalloc_rejects_sizes_beyond_its_array():
    lib = fa.library()
    B, H, d, page, mb, splits = 1024, 64, 128, 256, 128, 8
    need = lib.fa_kvcache_workspace_size(B, H, d, mb, page, splits)
    assert need > fa.FA_NOALLOC_SCRATCH_BYTES
    rc = lib.fa_fwd_kvcache_noalloc(P, P, P, P, P, P, P, B, H, d, B * mb, page, mb, fa.FA_BF16, 0.1, -1, None,
                                    0.0, splits, None)
    assert rc == 6  # FA_ERR_WORKSPACE


def make_inputs(seed, B=5, H=4, d=128, page=64, mb=24):
    g = torch.Generator().manual_seed(seed)
    num_pages = B * mb
    kc = torch.randn(num_pages, page, H, d, generator=g).to(torch.bfloat16)
    vc = torch.randn(num_pages, page, H, d, generator=g).to(torch.bfloat16)
    table = torch.randperm(num_pages, generator=g).view(B, mb).to(torch.int32)
    lens = torch.randint(1, mb * page + 1, (B,), generator=g).to(torch.int32)
    lens[0] = 0
    q = torch.randn(B, 1, H, d, generator=g).to(torch.bfloat16)
    return q, kc, vc, table, lens


@pytest.mark.gpu
@pytest.mark.parametrize("page", [64, 256], ids=["page64", "page256"])
@pytest.mark.parametrize("num_splits", [0, 7])
def test_noalloc_matches_workspace_entry_point_on_two_calls(num_splits, page):
    """Two calls in a row on different inputs (the second reuses the array
    the first left its partials in). Same kernels, split count and inputs as
    fa_fwd_kvcache with a caller workspace, so the results must agree bit for
    bit; the first call's result is also checked against the fp64 oracle."""
    import oracle
    from tests import parity
    scale = 128 ** -0.5
    mb = 24 if page == 64 else 6
    for call, seed in enumerate((101, 202)):
        host = make_inputs(seed, page=page, mb=mb)
        q, kc, vc, table, lens = [t.cuda() for t in host]
        B, _, H, d = q.shape
        assert fa.fa_kvcache_workspace_size(B, H, d, table.shape[1], kc.shape[1], num_splits) > 0
        out = torch.empty_like(q)
        lse = torch.empty((B, H, 1), dtype=torch.float32, device="cuda")
        fa.fa_fwd_kvcache_noalloc(q, kc, vc, table, lens, out, lse, scale, num_splits=num_splits)
        ref_out, ref_lse = fa.decode(q, kc, vc, table, lens, scale, num_splits=num_splits)
        torch.cuda.synchronize()
        o, l = out.float().cpu().numpy(), lse.cpu().numpy()
        assert np.array_equal(o, ref_out.float().cpu().numpy()), "call %d: O differs from fa_fwd_kvcache" % call
        assert np.array_equal(l, ref_lse.cpu().numpy()), "call %d: LSE differs from fa_fwd_kvcache" % call
        if call == 0:
            o_ref, l_ref = oracle.attn_decode_paged(*host, scale)
            parity.check(o, l, o_ref, l_ref, torch.bfloat16, "noalloc page %d splits %d" % (page, num_splits))
