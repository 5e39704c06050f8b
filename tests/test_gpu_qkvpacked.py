"""GPU parity of the packed-QKV entry points (through the C ABI) against the
fp64 oracle, with the fa_fwd tolerances (tests/parity.py)."""
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
    return parity.check(out, lse, o_ref, l_ref, dtype, "qkvpacked " + what)


CASES = [
    # (B, H, N, d, dtype, causal, wl, wr, alibi, cap, sigma)
    (2, 3, 300, 128, torch.bfloat16, True, -1, -1, False, 0.0, 1.0),
    (1, 2, 129, 64, torch.float16, False, 40, 17, False, 0.0, 1.0),
    (1, 4, 384, 128, torch.bfloat16, True, -1, -1, True, 50.0, 2.0),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dH%dN%dd%d_%s" % (c[:4] + (str(c[4])[6:],)))
def test_qkvpacked_matches_oracle(case):
    B, H, N, d, dtype, causal, wl, wr, alibi, cap, sigma = case
    g = torch.Generator().manual_seed(N + H)
    qkv = (torch.randn(B, N, 3, H, d, generator=g) * sigma).to(dtype)
    slopes = W.alibi_slopes(H) if alibi else None
    scale = 1.0 / math.sqrt(d)
    out = torch.empty(B, N, H, d, dtype=dtype, device="cuda")
    lse = torch.empty(B, H, N, dtype=torch.float32, device="cuda")
    fa.fa_fwd_qkvpacked(qkv.cuda(), out, lse, scale, causal, wl, wr, None if slopes is None else slopes.cuda(), cap)
    torch.cuda.synchronize()
    o_ref, l_ref = oracle.attn_fwd_qkvpacked(qkv, scale, causal, wl, wr, slopes, cap)
    compare(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, dtype, str(case))


def test_varlen_qkvpacked_matches_oracle():
    lens = [1, 200, 0, 513, 128]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    total, H, d = int(cu[-1]), 2, 128
    g = torch.Generator().manual_seed(3)
    qkv = torch.randn(total, 3, H, d, generator=g).to(torch.bfloat16)
    out = torch.empty(total, H, d, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(H, total, dtype=torch.float32, device="cuda")
    scale = 1.0 / math.sqrt(d)
    fa.fa_fwd_varlen_qkvpacked(qkv.cuda(), out, lse, torch.from_numpy(cu).cuda(), max(lens), scale, causal=True)
    torch.cuda.synchronize()
    q, k, v = (qkv[:, i].contiguous() for i in range(3))
    o_ref, l_ref = oracle.attn_fwd_varlen(q, k, v, cu, cu, scale, True)
    compare(out.float().cpu().numpy(), lse.cpu().numpy(), o_ref, l_ref, torch.bfloat16, "varlen packed")
