"""GPU parity of the backward pass (fa_bwd, through the C ABI) against the
fp64 oracle's gradients.

Tolerance, from the arithmetic: the kernel rounds P and dS to the input type
before the products that consume them (dV = P^T dO; dK = dS^T Q; dQ = dS K)
and rounds dq, dk, dv to it at the end; every sum runs in fp32. Each term thus
carries a relative error of at most one unit in the last place of the input
type (2^-8 bf16, 2^-11 fp16), so a gradient entry is off by at most that
fraction of the sum of its terms' magnitudes, which for these inputs stays
within a few times the largest entry of the gradient. The bar is
max |got - want| <= tol * max |want| with tol = 2e-2 (bf16) and 5e-3 (fp16).
"""
import math

import numpy as np
import pytest
import torch

import oracle
import exact_io_aware_79_b200 as fa
from exact_io_aware_79_b200 import workloads as W

pytestmark = pytest.mark.gpu

TOL = {torch.bfloat16: 2e-2, torch.float16: 5e-3}


def inputs(B, H, H_kv, Nq, Nk, d, dtype, seed):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(B, Nq, H, d, generator=g).to(dtype)
    k = torch.randn(B, Nk, H_kv, d, generator=g).to(dtype)
    v = torch.randn(B, Nk, H_kv, d, generator=g).to(dtype)
    do = torch.randn(B, Nq, H, d, generator=g).to(dtype)
    return q, k, v, do


def run(q, k, v, do, scale, causal=False, wl=-1, wr=-1, slopes=None, cap=0.0, det=False):
    B, Nq, H, d = q.shape
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    out = torch.empty_like(qd)
    lse = torch.empty(B, H, Nq, dtype=torch.float32, device="cuda")
    sl = None if slopes is None else slopes.cuda()
    fa.fa_fwd_gqa(qd, kd, vd, out, lse, scale, causal, wl, wr, sl, cap)
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    fa.fa_bwd(qd, kd, vd, out, lse, dod, dq, dk, dv, scale, causal, wl, wr, sl, cap, deterministic=det)
    torch.cuda.synchronize()
    return dq, dk, dv


def check(got, want, dtype, what):
    got = got.float().cpu().numpy()
    err = float(np.abs(got - want).max())
    ref = float(np.abs(want).max())
    assert np.isfinite(got).all(), what
    assert err <= TOL[dtype] * max(ref, 1e-6), "%s: max error %.3g of max |want| %.3g" % (what, err, ref)


CASES = [
    # (B, H, H_kv, Nq, Nk, d, dtype, causal, wl, wr, alibi, cap)
    (2, 2, 2, 200, 200, 128, torch.bfloat16, True, -1, -1, False, 0.0),    # ragged, several blocks each way
    (1, 2, 2, 130, 257, 64, torch.float16, False, -1, -1, False, 0.0),     # Nq < Nk, no mask
    (1, 2, 1, 257, 129, 64, torch.float16, True, -1, -1, False, 0.0),      # Nq > Nk: rows without keys
    (1, 4, 2, 190, 190, 128, torch.bfloat16, True, 50, 0, True, 30.0),     # grouped, window, ALiBi, softcap
    (2, 2, 2, 64, 64, 128, torch.bfloat16, False, 10, 20, False, 0.0),     # two-sided window
    (1, 8, 2, 100, 300, 128, torch.float16, True, -1, -1, True, 0.0),      # groups of 4, ALiBi, Nq < Nk
    (1, 2, 2, 1, 70, 128, torch.bfloat16, True, -1, -1, False, 5.0),       # one query row, softcap
    (2, 4, 2, 300, 333, 64, torch.bfloat16, True, 100, 0, True, 30.0),     # d = 64 bf16: grouped, window, ALiBi, softcap
]


@pytest.mark.parametrize("det", [False, True], ids=["atomic_dq", "deterministic"])
@pytest.mark.parametrize("case", CASES, ids=lambda c: "B%dH%dkv%dq%dk%dd%d" % c[:6])
def test_bwd_matches_oracle(case, det):
    B, H, H_kv, Nq, Nk, d, dtype, causal, wl, wr, alibi, cap = case
    q, k, v, do = inputs(B, H, H_kv, Nq, Nk, d, dtype, seed=Nq + Nk + H)
    slopes = W.alibi_slopes(H) if alibi else None
    scale = 1.0 / math.sqrt(d)
    dq, dk, dv = run(q, k, v, do, scale, causal, wl, wr, slopes, cap, det)
    rq, rk, rv = oracle.attn_bwd(q, k, v, do, scale, causal, wl, wr, slopes, cap)
    check(dq, rq, dtype, "dq")
    check(dk, rk, dtype, "dk")
    check(dv, rv, dtype, "dv")


def test_bwd_dk_dv_are_reproducible_bit_for_bit():
    q, k, v, do = inputs(1, 4, 2, 300, 300, 128, torch.bfloat16, seed=3)
    a = run(q, k, v, do, 0.1, True)
    b = run(q, k, v, do, 0.1, True)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    assert (a[0].float() - b[0].float()).abs().max().item() <= 1e-2 * a[0].float().abs().max().item()


def test_bwd_deterministic_mode_repeats_every_output_bit_for_bit():
    q, k, v, do = inputs(1, 4, 2, 300, 300, 128, torch.bfloat16, seed=3)
    a = run(q, k, v, do, 0.1, True, det=True)
    b = run(q, k, v, do, 0.1, True, det=True)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    c = run(q, k, v, do, 0.1, True, det=False)   # same dK, dV as the atomic mode
    assert torch.equal(a[1], c[1]) and torch.equal(a[2], c[2])


def test_bwd_empty_sides():
    q, k, v, do = inputs(1, 2, 2, 0, 50, 64, torch.float16, seed=4)
    dq, dk, dv = run(q, k, v, do, 0.2, False)
    assert torch.count_nonzero(dk) == 0 and torch.count_nonzero(dv) == 0


def test_full_size_causal_bwd_on_sampled_heads():
    """The causal B8 H16 N2048 d128 workload, gradients of two (batch, head)
    pairs checked against the oracle on those heads alone (in MHA a head's
    gradients depend only on its own q, k, v, dout)."""
    w = W.CAUSAL_2K
    x = W.make_fwd_inputs(w, device="cuda")
    g = torch.Generator().manual_seed(77)
    do = torch.randn(x["q"].shape, generator=g).to(w.dtype).cuda()
    out = torch.empty_like(x["q"])
    lse = torch.empty(w.B, w.H, w.Nq, dtype=torch.float32, device="cuda")
    fa.fa_fwd(x["q"], x["k"], x["v"], out, lse, w.scale, True)
    dq, dk, dv = torch.empty_like(x["q"]), torch.empty_like(x["k"]), torch.empty_like(x["v"])
    fa.fa_bwd(x["q"], x["k"], x["v"], out, lse, do, dq, dk, dv, w.scale, True)
    torch.cuda.synchronize()
    for b, h in ((0, 0), (w.B - 1, w.H - 1)):
        sl = lambda t: t[b:b + 1, :, h:h + 1].cpu()
        rq, rk, rv = oracle.attn_bwd(sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(do), w.scale, True)
        check(sl(dq), rq, w.dtype, "dq (%d, %d)" % (b, h))
        check(sl(dk), rk, w.dtype, "dk (%d, %d)" % (b, h))
        check(sl(dv), rv, w.dtype, "dv (%d, %d)" % (b, h))


# ---------------------------------------------------------------- packed sequences

def _packed(lens, H, d, dtype, g):
    total = int(sum(lens))
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32)
    return torch.randn(total, H, d, generator=g).to(dtype), cu


def _varlen_reference(q, k, v, do, cu_q, cu_k, scale, **opts):
    """Per-sequence oracle gradients, stitched back into the packed layout."""
    dq = np.zeros(q.shape)
    dk = np.zeros(k.shape)
    dv = np.zeros(v.shape)
    for b in range(cu_q.numel() - 1):
        q0, q1, k0, k1 = int(cu_q[b]), int(cu_q[b + 1]), int(cu_k[b]), int(cu_k[b + 1])
        if q1 == q0 or k1 == k0:
            continue
        sl = lambda t, a, z: t[a:z].unsqueeze(0)
        rq, rk, rv = oracle.attn_bwd(sl(q, q0, q1), sl(k, k0, k1), sl(v, k0, k1), sl(do, q0, q1), scale, **opts)
        dq[q0:q1], dk[k0:k1], dv[k0:k1] = rq[0], rk[0], rv[0]
    return dq, dk, dv


VARLEN = [
    # (lens_q, lens_k, H, d, dtype, opts)
    ((130, 1, 257, 0, 64), (130, 1, 257, 0, 64), 2, 128, torch.bfloat16, {"causal": True}),
    ((50, 200), (120, 90), 2, 64, torch.float16, {"window_left": 30, "window_right": 10}),
    ((70, 190), (70, 190), 2, 128, torch.bfloat16, {"causal": True, "softcap": 20.0}),
]


@pytest.mark.parametrize("det", [False, True], ids=["atomic_dq", "deterministic"])
@pytest.mark.parametrize("case", VARLEN, ids=lambda c: "q%s_k%s" % ("-".join(map(str, c[0])), "-".join(map(str, c[1]))))
def test_bwd_varlen_matches_per_sequence_oracle(case, det):
    lens_q, lens_k, H, d, dtype, opts = case
    g = torch.Generator().manual_seed(sum(lens_q) + 7)
    q, cu_q = _packed(lens_q, H, d, dtype, g)
    k, cu_k = _packed(lens_k, H, d, dtype, g)
    v, _ = _packed(lens_k, H, d, dtype, g)
    do, _ = _packed(lens_q, H, d, dtype, g)
    scale = 1.0 / math.sqrt(d)
    qd, kd, vd, dod, cqd, ckd = (t.cuda() for t in (q, k, v, do, cu_q, cu_k))
    out = torch.empty_like(qd)
    lse = torch.empty(H, q.shape[0], dtype=torch.float32, device="cuda")
    fw = dict(causal=opts.get("causal", False), window_left=opts.get("window_left", -1),
              window_right=opts.get("window_right", -1), softcap=opts.get("softcap", 0.0))
    fa.fa_fwd_varlen(qd, kd, vd, out, lse, cqd, ckd, max(lens_q), max(lens_k), scale, **fw)
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    fa.fa_bwd_varlen(qd, kd, vd, out, lse, dod, dq, dk, dv, cqd, ckd, max(lens_q), max(lens_k), scale,
                     deterministic=det, **fw)
    torch.cuda.synchronize()
    rq, rk, rv = _varlen_reference(q, k, v, do, cu_q, cu_k, scale, **fw)
    check(dq, rq, dtype, "dq")
    check(dk, rk, dtype, "dk")
    check(dv, rv, dtype, "dv")


def test_bwd_varlen_grouped_heads_with_oracle_forward():
    """Grouped-query packed sequences; O and LSE come from the oracle's
    forward (rounded as a forward would return them)."""
    lens, H, H_kv, d, dtype = (100, 190), 4, 2, 128, torch.bfloat16
    g = torch.Generator().manual_seed(11)
    q, cu = _packed(lens, H, d, dtype, g)
    k, _ = _packed(lens, H_kv, d, dtype, g)
    v, _ = _packed(lens, H_kv, d, dtype, g)
    do, _ = _packed(lens, H, d, dtype, g)
    slopes = W.alibi_slopes(H)
    scale = 0.09
    out = torch.empty_like(q)
    lse = torch.empty(H, q.shape[0], dtype=torch.float32)
    for b in range(len(lens)):
        a, z = int(cu[b]), int(cu[b + 1])
        o, l = oracle.attn_fwd_gqa(q[a:z].unsqueeze(0), k[a:z].unsqueeze(0), v[a:z].unsqueeze(0), scale, True,
                                   alibi_slopes=slopes)
        out[a:z] = torch.from_numpy(o[0]).to(dtype)
        lse[:, a:z] = torch.from_numpy(l[0]).float()
    qd, kd, vd, dod, od, ld, cud = (t.cuda() for t in (q, k, v, do, out, lse, cu))
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(kd), torch.empty_like(vd)
    fa.fa_bwd_varlen(qd, kd, vd, od, ld, dod, dq, dk, dv, cud, cud, max(lens), max(lens), scale, True,
                     alibi_slopes=slopes.cuda())
    torch.cuda.synchronize()
    rq, rk, rv = _varlen_reference(q, k, v, do, cu, cu, scale, causal=True, alibi_slopes=slopes)
    check(dq, rq, dtype, "dq")
    check(dk, rk, dtype, "dk")
    check(dv, rv, dtype, "dv")


@pytest.mark.parametrize("det", [False, True], ids=["atomic_dq", "deterministic"])
def test_bwd_varlen_skips_a_sequence_with_broken_offsets(det):
    lens, H, d = (80, 120, 60), 2, 64
    g = torch.Generator().manual_seed(12)
    q, cu = _packed(lens, H, d, torch.float16, g)
    k, _ = _packed(lens, H, d, torch.float16, g)
    v, _ = _packed(lens, H, d, torch.float16, g)
    do, _ = _packed(lens, H, d, torch.float16, g)
    qd, kd, vd, dod, cud = (t.cuda() for t in (q, k, v, do, cu))
    out = torch.empty_like(qd)
    lse = torch.empty(H, q.shape[0], dtype=torch.float32, device="cuda")
    fa.fa_fwd_varlen(qd, kd, vd, out, lse, cud, cud, max(lens), max(lens), 0.125, causal=True)
    bad = cu.clone()
    bad[2] = 500                      # sequence 1 ends past total, sequence 2 starts there
    dq, dk, dv = torch.empty_like(qd), torch.full_like(kd, 7.0), torch.full_like(vd, 7.0)
    dq.fill_(float("nan"))            # every row of dq is written, valid sequence or not
    fa.fa_bwd_varlen(qd, kd, vd, out, lse, dod, dq, dk, dv, bad.cuda(), bad.cuda(), max(lens), max(lens), 0.125,
                     causal=True, deterministic=det)
    torch.cuda.synchronize()
    rq, rk, rv = _varlen_reference(q, k, v, do, cu, cu, 0.125, causal=True)
    a = int(cu[1])
    check(dq[:a], rq[:a], torch.float16, "dq of the valid sequence")
    check(dk[:a], rk[:a], torch.float16, "dk of the valid sequence")
    assert torch.all(dk[a:] == 7.0) and torch.all(dv[a:] == 7.0)    # skipped: left as they were
    assert torch.count_nonzero(dq[a:]) == 0                          # rows of no valid sequence


def test_attention_func_autograd_gradients_match_the_oracle():
    """loss = sum(out * dout) through attention_func; the gradients that
    autograd hands back are fa_bwd's and must match the oracle's."""
    B, H, H_kv, N, d, dtype = 1, 4, 2, 150, 64, torch.bfloat16
    q, k, v, do = inputs(B, H, H_kv, N, N, d, dtype, seed=21)
    qd, kd, vd = (t.cuda().requires_grad_(True) for t in (q, k, v))
    out = fa.attention_func(qd, kd, vd, causal=True, window_left=40, softcap=15.0)
    (out.float() * do.cuda().float()).sum().backward()
    rq, rk, rv = oracle.attn_bwd(q, k, v, do, d ** -0.5, True, 40, -1, None, 15.0)
    check(qd.grad, rq, dtype, "q.grad")
    check(kd.grad, rk, dtype, "k.grad")
    check(vd.grad, rv, dtype, "v.grad")


# ---------------------------------------------------------------- packed QKV

@pytest.mark.parametrize("det", [False, True], ids=["atomic_dq", "deterministic"])
def test_bwd_qkvpacked_matches_oracle(det):
    B, N, H, d, dtype = 2, 190, 2, 128, torch.bfloat16
    g = torch.Generator().manual_seed(31)
    qkv = torch.randn(B, N, 3, H, d, generator=g).to(dtype)
    do = torch.randn(B, N, H, d, generator=g).to(dtype)
    qkvd, dod = qkv.cuda(), do.cuda()
    out = torch.empty(B, N, H, d, dtype=dtype, device="cuda")
    lse = torch.empty(B, H, N, dtype=torch.float32, device="cuda")
    fa.fa_fwd_qkvpacked(qkvd, out, lse, 0.1, True, 60, -1)
    dqkv = torch.full_like(qkvd, 3.0)
    fa.fa_bwd_qkvpacked(qkvd, out, lse, dod, dqkv, 0.1, True, 60, -1, deterministic=det)
    torch.cuda.synchronize()
    refs = oracle.attn_bwd(qkv[:, :, 0], qkv[:, :, 1], qkv[:, :, 2], do, 0.1, True, 60, -1)
    for slot, (ref, name) in enumerate(zip(refs, ("dq", "dk", "dv"))):
        check(dqkv[:, :, slot], ref, dtype, name)


def test_bwd_varlen_qkvpacked_matches_per_sequence_oracle():
    lens, H, d, dtype = (120, 1, 200), 2, 64, torch.float16
    total = sum(lens)
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32)
    g = torch.Generator().manual_seed(32)
    qkv = torch.randn(total, 3, H, d, generator=g).to(dtype)
    do = torch.randn(total, H, d, generator=g).to(dtype)
    qkvd, dod, cud = qkv.cuda(), do.cuda(), cu.cuda()
    out = torch.empty(total, H, d, dtype=dtype, device="cuda")
    lse = torch.empty(H, total, dtype=torch.float32, device="cuda")
    fa.fa_fwd_varlen_qkvpacked(qkvd, out, lse, cud, max(lens), 0.125, causal=True)
    dqkv = torch.empty_like(qkvd)
    fa.fa_bwd_varlen_qkvpacked(qkvd, out, lse, dod, dqkv, cud, max(lens), 0.125, causal=True)
    torch.cuda.synchronize()
    rq, rk, rv = _varlen_reference(qkv[:, 0], qkv[:, 1], qkv[:, 2], do, cu, cu, 0.125, causal=True)
    check(dqkv[:, 0], rq, dtype, "dq")
    check(dqkv[:, 1], rk, dtype, "dk")
    check(dqkv[:, 2], rv, dtype, "dv")
