"""GPU parity of fa_fwd (through the C ABI) against the fp64 oracle.

Tolerances (tests/parity.py): |O_gpu - O_oracle| <= 1.6e-2 for bf16 and 4e-3
for fp16 element by element, widened by half an ulp of the output type only
where that half-ulp is at least half the bound (bf16 |O| >= 4, fp16
|O| >= 8), whatever the input scale; max |LSE_gpu - LSE_oracle| <= 1e-3 where
finite; rows the oracle finds empty must be exactly LSE = -inf. Mask membership is checked
bit-exactly on every row by the boundary probes.
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


def gpu_fwd(q, k, v, scale, causal=False, wl=-1, wr=-1, slopes=None, softcap=0.0):
    dev = "cuda"
    qd, kd, vd = q.to(dev), k.to(dev), v.to(dev)
    sd = None if slopes is None else slopes.to(dev)
    out, lse = fa.attention(qd, kd, vd, scale, causal, wl, wr, sd, softcap)
    torch.cuda.synchronize()
    return out.float().cpu().numpy(), lse.cpu().numpy()


def compare(out, lse, o_ref, l_ref, dtype, what=""):
    return parity.check(out, lse, o_ref, l_ref, dtype, "fwd " + what)


def make(B, H, Nq, Nk, d, dtype, seed, sigma=1.0):
    g = torch.Generator().manual_seed(seed)
    q = (torch.randn(B, Nq, H, d, generator=g) * sigma).to(dtype)
    k = (torch.randn(B, Nk, H, d, generator=g) * sigma).to(dtype)
    v = (torch.randn(B, Nk, H, d, generator=g) * sigma).to(dtype)
    return q, k, v


SMALL = [
    # (B, H, Nq, Nk, d, dtype, causal, wl, wr, alibi, softcap, sigma)
    (1, 2, 128, 128, 64, torch.float16, False, -1, -1, False, 0.0, 1.0),
    (2, 3, 300, 300, 128, torch.bfloat16, True, -1, -1, False, 0.0, 1.0),
    (1, 2, 200, 700, 128, torch.float16, True, -1, -1, False, 0.0, 1.0),
    (1, 2, 700, 200, 64, torch.bfloat16, True, -1, -1, False, 0.0, 1.0),
    (1, 2, 1000, 1000, 128, torch.bfloat16, True, 100, 0, False, 0.0, 1.0),
    (1, 2, 513, 513, 128, torch.bfloat16, False, 50, 70, False, 0.0, 1.0),
    (1, 4, 640, 640, 128, torch.bfloat16, True, -1, -1, True, 50.0, 2.0),
    (1, 3, 257, 385, 64, torch.float16, False, -1, -1, True, 0.0, 1.0),
    (1, 3, 600, 450, 128, torch.bfloat16, False, 200, 150, True, 30.0, 1.5),
    (1, 2, 384, 384, 128, torch.float16, True, 130, -1, False, 5.0, 1.5),
    (2, 2, 1, 1, 128, torch.bfloat16, True, -1, -1, False, 0.0, 1.0),
    (1, 1, 1, 333, 128, torch.bfloat16, True, -1, -1, True, 0.0, 1.0),
    (1, 2, 2048, 2048, 128, torch.bfloat16, True, -1, -1, False, 0.0, 1.0),
    (1, 2, 256, 4096, 128, torch.bfloat16, True, 1000, 0, False, 0.0, 1.0),
]


@pytest.mark.parametrize("case", SMALL, ids=lambda c: "B%dH%dq%dk%dd%d_%s_c%d_w%d,%d_a%d_s%g" % (
    c[0], c[1], c[2], c[3], c[4], str(c[5])[6:], c[6], c[7], c[8], c[9], c[10]))
def test_small_cases_match_oracle(case):
    B, H, Nq, Nk, d, dtype, causal, wl, wr, alibi, cap, sigma = case
    q, k, v = make(B, H, Nq, Nk, d, dtype, seed=Nq * 7 + Nk, sigma=sigma)
    slopes = W.alibi_slopes(H) if alibi else None
    scale = 1.0 / math.sqrt(d)
    out, lse = gpu_fwd(q, k, v, scale, causal, wl, wr, slopes, cap)
    o_ref, l_ref = oracle.attn_fwd(q, k, v, scale, causal, wl, wr, slopes, cap)
    compare(out, lse, o_ref, l_ref, dtype, str(case))


def test_no_keys_gives_empty_rows():
    q, _, _ = make(1, 2, 130, 1, 128, torch.bfloat16, seed=3)
    k = torch.empty(1, 0, 2, 128, dtype=torch.bfloat16)
    out, lse = gpu_fwd(q, k, k, 0.1)
    assert np.all(out == 0) and np.all(lse == -np.inf)


def test_empty_batch_is_a_no_op():
    q = torch.empty(0, 128, 2, 128, dtype=torch.bfloat16, device="cuda")
    out, lse = fa.attention(q, q, q)
    torch.cuda.synchronize()
    assert out.shape == q.shape and lse.shape == (0, 2, 128)


def sample_rows(Nq, seed, extra=24):
    rows = {0, 1, 127, 128, 255, 256, Nq // 2, Nq - 129, Nq - 128, Nq - 1}
    rng = np.random.default_rng(seed)
    rows |= set(rng.integers(0, Nq, size=extra).tolist())
    return sorted(r for r in rows if 0 <= r < Nq)


@pytest.mark.parametrize("w", [W.CAUSAL_2K, W.WINDOW_16K, W.WINDOW_Q4K_K16K, W.CAUSAL_Q4K_K16K, W.ALIBI_SOFTCAP,
                               W.TINY], ids=lambda w: w.name)
def test_full_size_workloads_on_sampled_rows(w):
    x = W.make_fwd_inputs(w)
    dev = {kk: (None if t is None else t.cuda()) for kk, t in x.items()}
    out, lse = fa.attention(dev["q"], dev["k"], dev["v"], w.scale, w.causal, w.window_left, w.window_right,
                            dev["slopes"], w.softcap)
    torch.cuda.synchronize()
    rows = sample_rows(w.Nq, w.seed)
    o_ref, l_ref = oracle.attn_fwd(x["q"], x["k"], x["v"], w.scale, w.causal, w.window_left, w.window_right,
                                   x["slopes"], w.softcap, rows=rows)
    o = out[:, rows].float().cpu().numpy()
    l = lse[:, :, rows].cpu().numpy()
    compare(o, l, o_ref, l_ref, w.dtype, w.name)
    assert torch.isfinite(out).all().item()


PROBE_SCALE = float(np.float32(1.0 / 1.4426950408889634))


def boundary_probe(B, H, Nq, Nk, d, causal, wl, wr, upper, dtype=torch.bfloat16):
    """Scores 128*j (upper) or -128*j (lower) for key j: each row's softmax
    collapses onto its largest (smallest) visible key, and V encodes the key
    index as (j // 64 + 1, j % 64 + 1), so O must equal that key's code
    exactly (the codes start at 1 so an empty row's O = 0 cannot pass for a
    key, and weights far below 2^-126 cannot disturb them).
    The scale is fp32(1 / log2 e), whose product with log2 e rounds to
    exactly 1 in fp32, so the scores in log2 units are the exact integers
    128*j: the top key's weight is exactly 1 and every other weight is
    2^-128 or less, which flushes to 0."""
    assert Nk <= 16384
    sign = 1.0 if upper else -1.0
    q = torch.zeros(B, Nq, H, d)
    q[..., 0] = sign * 8192.0
    q[..., 1] = sign * 128.0
    j = torch.arange(Nk, dtype=torch.float32)
    k = torch.zeros(B, Nk, H, d)
    k[..., 0] = (j // 64)[None, :, None]
    k[..., 1] = (j % 64)[None, :, None]
    v = torch.zeros(B, Nk, H, d)
    v[..., 0] = (j // 64 + 1)[None, :, None]
    v[..., 1] = (j % 64 + 1)[None, :, None]
    q, k, v = q.to(dtype), k.to(dtype), v.to(dtype)
    out, lse = gpu_fwd(q, k, v, PROBE_SCALE, causal, wl, wr)
    # expected visible interval of every row, by interval arithmetic
    i = np.arange(Nq)
    pos = i + Nk - Nq
    lo = np.zeros(Nq, dtype=np.int64) if wl < 0 else np.maximum(0, pos - wl)
    hi = np.full(Nq, Nk - 1, dtype=np.int64)
    if causal:
        hi = np.minimum(hi, pos)
    if wr >= 0:
        hi = np.minimum(hi, pos + wr)
    empty = lo > hi
    target = hi if upper else lo
    want0 = np.where(empty, 0, target // 64 + 1)
    want1 = np.where(empty, 0, target % 64 + 1)
    got0 = out[:, :, :, 0]
    got1 = out[:, :, :, 1]
    assert np.array_equal(got0, np.broadcast_to(want0[None, :, None], got0.shape))
    assert np.array_equal(got1, np.broadcast_to(want1[None, :, None], got1.shape))
    assert np.all(out[:, :, :, 2:] == 0)
    assert np.all(lse[:, :, empty] == -np.inf) and np.all(np.isfinite(lse[:, :, ~empty]))


PROBES = [
    (1, 2, 1000, 1000, 128, True, -1, -1),
    (1, 2, 300, 1000, 64, True, -1, -1),
    (1, 2, 1000, 300, 128, True, -1, -1),
    (1, 2, 2048, 2048, 128, True, 300, 0),
    (1, 2, 700, 900, 128, False, 77, 130),
    (1, 2, 513, 513, 64, False, 0, 0),
    (1, 2, 4096, 16384, 128, True, 4096, 0),
    (1, 1, 16384, 16384, 128, True, 4096, 0),
]


@pytest.mark.parametrize("case", PROBES, ids=lambda c: "q%dk%dd%d_c%d_w%d,%d" % c[2:])
@pytest.mark.parametrize("upper", [True, False], ids=["upper", "lower"])
def test_mask_boundaries_are_exact_on_every_row(case, upper):
    boundary_probe(*case, upper=upper)


@pytest.mark.parametrize("scale", [-0.09, 0.0])
@pytest.mark.parametrize("mods", [dict(), dict(alibi=True, softcap=5.0)], ids=["plain", "alibi_softcap"])
def test_negative_and_zero_scale(scale, mods):
    """A negative scale runs as -Q K^T on the tensor core with |scale|; a zero
    scale makes every visible score 0 (softcap and ALiBi still apply)."""
    B, H, Nq, Nk, d = 1, 2, 300, 500, 128
    q, k, v = make(B, H, Nq, Nk, d, torch.bfloat16, seed=77)
    slopes = W.alibi_slopes(H) if mods.get("alibi") else None
    cap = mods.get("softcap", 0.0)
    out, lse = gpu_fwd(q, k, v, scale, True, 200, -1, slopes, cap)
    o_ref, l_ref = oracle.attn_fwd(q, k, v, scale, True, 200, -1, slopes, cap)
    compare(out, lse, o_ref, l_ref, torch.bfloat16, "scale %g %s" % (scale, mods))


def test_slopes_must_be_fp32_of_length_h_on_the_device():
    q = torch.zeros(1, 16, 4, 64, dtype=torch.bfloat16, device="cuda")
    for bad in (torch.ones(3, device="cuda"), torch.ones(4, dtype=torch.float64, device="cuda"), torch.ones(4)):
        with pytest.raises(ValueError, match="alibi_slopes|CUDA"):
            fa.attention(q, q, q, 0.1, alibi_slopes=bad)
