"""GPU parity of fa_fwd_varlen (through the C ABI) against the fp64 oracle.

Every packed sequence must match the oracle's attention of that sequence
alone within the fa_fwd tolerances (tests/parity.py; empty rows exactly
O = 0, LSE = -inf). Rows
that no sequence owns, and sequences whose offsets break the contract, must
be left exactly as they were.
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
SENTINEL = 7.0
EXTRA = 3  # trailing query rows no sequence owns


def packed(lens_q, lens_k, H, d, dtype, seed, sigma=1.0):
    cq = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    ck = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn(int(cq[-1]) + EXTRA, H, d, generator=g) * sigma).to(dtype)
    k = (torch.randn(max(int(ck[-1]), 1), H, d, generator=g) * sigma).to(dtype)
    v = (torch.randn(max(int(ck[-1]), 1), H, d, generator=g) * sigma).to(dtype)
    return q, k, v, cq, ck


def run(q, k, v, cq, ck, max_q, max_k, scale, **kw):
    dev = "cuda"
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    out = torch.full(q.shape, SENTINEL, dtype=q.dtype, device=dev)
    lse = torch.full((q.shape[1], q.shape[0]), SENTINEL, dtype=torch.float32, device=dev)
    slopes = kw.pop("slopes", None)
    fa.fa_fwd_varlen(qd, kd, vd, out, lse, torch.from_numpy(cq).to(dev), torch.from_numpy(ck).to(dev), max_q, max_k,
                     scale, alibi_slopes=None if slopes is None else slopes.to(dev), **kw)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), lse.cpu().numpy()


def check_rows(out, lse, o_ref, l_ref, rows, dtype, what):
    o, l, orf, lrf = out[rows], lse[:, rows], o_ref[rows], l_ref[:, rows]
    fin = np.isfinite(lrf)
    if (~fin).any():
        assert np.all(o.transpose(1, 0, 2)[~fin] == 0.0), what + ": empty rows must be O = 0"
    parity.check(o, l, orf, lrf, dtype, "varlen " + what)


CASES = [
    # (lens_q, lens_k, H, d, dtype, causal, wl, wr, alibi, softcap, sigma)
    ([1, 127, 128, 129, 300, 513], [1, 127, 128, 129, 300, 513], 2, 128, torch.bfloat16, True, -1, -1, False, 0.0,
     1.0),
    ([200, 5, 0, 64], [700, 5, 17, 1000], 3, 64, torch.float16, True, -1, -1, False, 0.0, 1.0),
    ([700, 130, 9], [200, 1, 0], 2, 128, torch.bfloat16, True, -1, -1, False, 0.0, 1.0),
    ([1000, 257], [1000, 257], 2, 128, torch.bfloat16, True, 100, 0, False, 0.0, 1.0),
    ([640, 300], [640, 300], 4, 128, torch.bfloat16, True, -1, -1, True, 50.0, 2.0),
    ([513, 129], [513, 400], 2, 64, torch.float16, False, 50, 70, False, 0.0, 1.0),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "n%d_d%d_%s_c%d_w%d,%d_a%d_s%g" % (
    len(c[0]), c[3], str(c[4])[6:], c[5], c[6], c[7], c[8], c[9]))
def test_varlen_cases_match_oracle(case):
    lens_q, lens_k, H, d, dtype, causal, wl, wr, alibi, cap, sigma = case
    q, k, v, cq, ck = packed(lens_q, lens_k, H, d, dtype, seed=sum(lens_q) + 3 * sum(lens_k), sigma=sigma)
    slopes = W.alibi_slopes(H) if alibi else None
    scale = 1.0 / math.sqrt(d)
    out, lse = run(q, k, v, cq, ck, max(lens_q), max(lens_k + [0]), scale, causal=causal, window_left=wl,
                   window_right=wr, slopes=slopes, softcap=cap)
    o_ref, l_ref = oracle.attn_fwd_varlen(q, k[:int(ck[-1])], v[:int(ck[-1])], cq, ck, scale, causal, wl, wr,
                                          None if slopes is None else slopes.numpy(), cap)
    owned = np.arange(int(cq[-1]))
    check_rows(out, lse, o_ref, l_ref, owned, dtype, str(case))
    # rows past the last sequence are untouched
    assert np.all(out[int(cq[-1]):] == SENTINEL) and np.all(lse[:, int(cq[-1]):] == SENTINEL)


def test_many_random_sequences():
    g = np.random.default_rng(5)
    lens_q = [int(x) for x in g.integers(1, 400, 40)]
    lens_k = [n + int(x) for n, x in zip(lens_q, g.integers(0, 200, 40))]
    q, k, v, cq, ck = packed(lens_q, lens_k, 2, 128, torch.bfloat16, seed=77)
    scale = 1.0 / math.sqrt(128)
    out, lse = run(q, k, v, cq, ck, max(lens_q), max(lens_k), scale, causal=True)
    o_ref, l_ref = oracle.attn_fwd_varlen(q, k, v, cq, ck, scale, True)
    check_rows(out, lse, o_ref, l_ref, np.arange(int(cq[-1])), torch.bfloat16, "40 sequences")


def test_sequences_that_break_the_contract_are_skipped():
    # seq 0 is valid; seq 1 ends past total_q; seq 2 has a negative length;
    # seq 3 is longer than max_seqlen_k
    H, d = 2, 128
    g = torch.Generator().manual_seed(9)
    total_q, total_k = 250, 900
    q = torch.randn(total_q, H, d, generator=g).to(torch.bfloat16)
    k = torch.randn(total_k, H, d, generator=g).to(torch.bfloat16)
    v = torch.randn(total_k, H, d, generator=g).to(torch.bfloat16)
    cq = np.array([0, 100, 300, 200, 240], dtype=np.int32)
    ck = np.array([0, 120, 200, 260, 900], dtype=np.int32)
    scale = 1.0 / math.sqrt(d)
    out, lse = run(q, k, v, cq, ck, 200, 150, scale, causal=True)
    o_ref, l_ref = oracle.attn_fwd_varlen(q[:100], k[:120], v[:120], cq[:2], ck[:2], scale, True)
    check_rows(out, lse, o_ref, l_ref, np.arange(100), torch.bfloat16, "valid sequence")
    assert np.all(out[100:] == SENTINEL) and np.all(lse[:, 100:] == SENTINEL)


def test_full_size_varlen_workload_sampled_rows():
    w = W.VARLEN
    x = W.make_varlen_inputs(w, device="cuda")
    out = torch.empty_like(x["q"])
    lse = torch.empty((w.H, x["q"].shape[0]), dtype=torch.float32, device="cuda")
    fa.fa_fwd_varlen(x["q"], x["k"], x["v"], out, lse, x["cu_q"], x["cu_k"], x["max_q"], x["max_k"], w.scale,
                     w.causal)
    torch.cuda.synchronize()
    out_c, lse_c = out.float().cpu().numpy(), lse.cpu().numpy()
    qc, kc, vc = (x[n].cpu() for n in ("q", "k", "v"))
    cq, ck = x["cu_q"].cpu().numpy(), x["cu_k"].cpu().numpy()
    for b in range(len(cq) - 1):
        n = int(cq[b + 1] - cq[b])
        rows = sorted({0, n - 1, n // 2, min(127, n - 1), min(128, n - 1)})
        o_ref, l_ref = oracle.attn_fwd(qc[cq[b]:cq[b + 1]][None], kc[ck[b]:ck[b + 1]][None],
                                       vc[ck[b]:ck[b + 1]][None], w.scale, w.causal, rows=rows)
        got_o = out_c[cq[b] + np.array(rows)]
        got_l = lse_c[:, cq[b] + np.array(rows)]
        parity.check(got_o, got_l, o_ref[0], l_ref[0], w.dtype, "varlen full size, sequence %d" % b)
