"""GPU parity of fa_fwd_fp8 (through the C ABI) against the fp64 oracle.

The oracle computes attention of the dequantised 8-bit inputs exactly
(oracle.attn_fwd_fp8). The kernel rounds P to the input's 8-bit format
before the PV product and divides O by the sum of P as rounded, so with
w_j the exact weights of a row and p_j its unnormalised probabilities
(p_max >= 1, hence 1 / l <= w_max):

    O_gpu - O = sum_j (rho(p_j) - p_j) (v_j - O_gpu) / sum_j rho(p_j)

and the rounding rho of a normal value is within u p_j (u = 2^-4 for E4M3,
2^-3 for E5M2), of a value below the normal range within min(p_j, s) (s =
half the subnormal spacing: 2^-10 for E4M3, 2^-17 for E5M2). To first order

    |O_gpu - O| <= u sum_j w_j |v_j - O| + sum_j min(w_j, s w_max) |v_j - O|

per element; the test adds half a bf16 ulp of |O| (the output type) and
1e-4 (1 + |O|) for the fp32 arithmetic and the exponential's approximation,
and requires the LSE within 1e-3. Rows without visible keys must give O = 0,
LSE = -inf.
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

FMT = {torch.float8_e4m3fn: (2.0 ** -4, 2.0 ** -10), torch.float8_e5m2: (2.0 ** -3, 2.0 ** -17)}
LSE_TOL = 1e-3


def derived_bound(o_ref, p, v_deq, fmt):
    """Per-element bound [B,R,H,d] from the exact weights p [B,H,R,Nk] and
    the dequantised V [B,Nk,H,d] (heads already matched to the query heads)."""
    u, s = FMT[fmt]
    B, H, R, Nk = p.shape
    bound = np.zeros_like(o_ref)
    for b in range(B):
        for h in range(H):
            w = p[b, h]                                    # [R, Nk]
            wmax = w.max(axis=1, keepdims=True)
            coef = u * w + np.minimum(w, s * wmax)         # [R, Nk]
            for r0 in range(0, R, 64):                     # rows in chunks: [64, Nk, d] at a time
                dev = np.abs(v_deq[b, None, :, h, :] - o_ref[b, r0:r0 + 64, None, h, :])
                bound[b, r0:r0 + 64, h, :] = np.einsum("rk,rkd->rd", coef[r0:r0 + 64], dev)
    hu = parity.half_ulp(o_ref, torch.bfloat16)
    return bound + hu + 1e-4 * (1.0 + np.abs(o_ref))


def run_case(B, H, H_kv, Nq, Nk, fmt, causal, wl, wr, alibi, cap, sigma, seed, scale_sign=1.0):
    w = W.FwdWorkload("fp8case", B, H, Nq, Nk, 128, torch.bfloat16, causal=causal, window_left=wl,
                      window_right=wr, alibi=alibi, softcap=cap, sigma=sigma, seed=seed)
    x = W.make_fwd_inputs_fp8(w, fmt)
    # K/V with H_kv heads: keep the first H_kv heads of the draw (8-bit
    # tensors are moved around as their bytes)
    k8 = x["k"].view(torch.uint8)[:, :, :H_kv].contiguous().view(fmt)
    v8 = x["v"].view(torch.uint8)[:, :, :H_kv].contiguous().view(fmt)
    scale = scale_sign / math.sqrt(128)
    slopes = x["slopes"]
    out, lse = fa.attention_fp8(x["q"].cuda(), k8.cuda(), v8.cuda(), scale, x["descale_q"], x["descale_k"],
                                x["descale_v"], causal, wl, wr, None if slopes is None else slopes.cuda(), cap)
    torch.cuda.synchronize()
    # the oracle on query-head-matched K/V (query head h reads K/V head h // (H / H_kv))
    rep = H // H_kv
    k8h = k8.view(torch.uint8).repeat_interleave(rep, dim=2).view(fmt)
    v8h = v8.view(torch.uint8).repeat_interleave(rep, dim=2).view(fmt)
    o_ref, l_ref = oracle.attn_fwd_fp8(x["q"], k8h, v8h, scale, x["descale_q"], x["descale_k"], x["descale_v"],
                                       causal, wl, wr, slopes, cap)
    _, _, p = oracle.attn_fwd(x["q"], k8h, v8h, scale * x["descale_q"] * x["descale_k"], causal, wl, wr, slopes,
                              cap, return_probs=True)
    v_deq = oracle.widen(v8h) * x["descale_v"]
    o = out.float().cpu().numpy().astype(np.float64)
    l = lse.cpu().numpy().astype(np.float64)
    fin = np.isfinite(l_ref)
    assert np.array_equal(np.isfinite(l), fin), "empty-row pattern differs"
    assert np.all(l[~fin] == -np.inf)
    if (~fin).any():
        assert np.all(o.transpose(0, 2, 1, 3)[~fin] == 0.0)
    err = np.abs(o - o_ref)
    bound = derived_bound(o_ref, p, v_deq, fmt)
    ratio = float((err / bound).max()) if err.size else 0.0
    l_err = float(np.abs(l[fin] - l_ref[fin]).max()) if fin.any() else 0.0
    what = "fp8 %s B%d H%d/%d q%d k%d c%d w%d,%d a%d s%g" % (str(fmt)[-6:], B, H, H_kv, Nq, Nk, causal, wl, wr,
                                                             alibi, cap)
    parity.RECORD.append((what, float(err.max()) if err.size else 0.0, ratio, l_err))
    assert not np.isnan(o).any()
    assert ratio <= 1.0, "%s: O error %.3g is %.2f x its derived bound" % (what, float(err.max()), ratio)
    assert l_err <= LSE_TOL, "%s: LSE error %.3g" % (what, l_err)


CASES = [
    # (B, H, H_kv, Nq, Nk, fmt, causal, wl, wr, alibi, cap, sigma, seed)
    (1, 2, 2, 128, 128, torch.float8_e4m3fn, False, -1, -1, False, 0.0, 1.0, 1),
    (2, 3, 3, 300, 300, torch.float8_e4m3fn, True, -1, -1, False, 0.0, 1.0, 2),
    (1, 2, 2, 200, 700, torch.float8_e4m3fn, True, -1, -1, False, 0.0, 1.0, 3),
    (1, 2, 2, 700, 200, torch.float8_e4m3fn, True, -1, -1, False, 0.0, 1.0, 4),
    (1, 2, 2, 1000, 1000, torch.float8_e4m3fn, True, 100, 0, False, 0.0, 1.0, 5),
    (1, 4, 4, 640, 640, torch.float8_e4m3fn, True, -1, -1, True, 50.0, 2.0, 6),
    (1, 8, 2, 257, 385, torch.float8_e4m3fn, False, 50, 70, False, 0.0, 1.0, 7),
    (1, 2, 2, 384, 384, torch.float8_e5m2, True, -1, -1, False, 0.0, 1.0, 8),
    (1, 2, 1, 1, 333, torch.float8_e5m2, True, -1, -1, True, 5.0, 1.0, 9),
    (1, 2, 2, 2048, 2048, torch.float8_e4m3fn, True, -1, -1, False, 0.0, 1.0, 10),
    (1, 3, 3, 600, 450, torch.float8_e4m3fn, False, 200, 150, True, 30.0, 1.5, 12),
    (1, 2, 2, 257, 700, torch.float8_e4m3fn, False, -1, -1, True, 0.0, 1.0, 13),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dH%dkv%dq%dk%d_%s_c%d_w%d,%d_a%d_s%g" % (
    c[0], c[1], c[2], c[3], c[4], str(c[5])[-6:], c[6], c[7], c[8], c[9], c[10]))
def test_fp8_matches_oracle_within_derived_bound(case):
    run_case(*case)


def test_fp8_negative_scale():
    run_case(1, 2, 2, 300, 500, torch.float8_e4m3fn, True, 200, -1, False, 0.0, 1.0, 11, scale_sign=-1.0)


def test_fp8_no_keys_gives_empty_rows():
    q = torch.randn(1, 130, 2, 128).to(torch.float8_e4m3fn).cuda()
    k = torch.empty(1, 0, 2, 128, dtype=torch.float8_e4m3fn, device="cuda")
    out, lse = fa.attention_fp8(q, k, k, 0.1)
    torch.cuda.synchronize()
    assert torch.all(out == 0).item() and torch.all(lse == -float("inf")).item()


def test_fp8_rejects_other_head_dims_and_mixed_formats():
    q = torch.zeros(1, 16, 2, 64, dtype=torch.float8_e4m3fn, device="cuda")
    out = torch.empty(1, 16, 2, 64, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(1, 2, 16, dtype=torch.float32, device="cuda")
    with pytest.raises(fa.FaError):
        fa.fa_fwd_fp8(q, q, q, out, lse, 0.1)
    q = torch.zeros(1, 16, 2, 128, dtype=torch.float8_e4m3fn, device="cuda")
    k = torch.zeros(1, 16, 2, 128, dtype=torch.float8_e5m2, device="cuda")
    out = torch.empty(1, 16, 2, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(ValueError):
        fa.fa_fwd_fp8(q, k, k, out, lse, 0.1)
