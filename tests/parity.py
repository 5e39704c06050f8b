"""Shared parity check of the GPU outputs (O, LSE) against the fp64 oracle.

Bound on O, element by element: the stated max-abs bound (1.6e-2 for bf16
outputs, 4e-3 for fp16), plus half a unit in the last place of |O_oracle| in
the output type wherever that half-ulp is at least half the stated bound:
bf16 outputs with |O| >= 4 (half-ulp 2^-6 = 0.0156 on [4, 8), 2^-5 on
[8, 16)) and fp16 outputs with |O| >= 8 (2^-8 on [8, 16)). There, rounding
the exact value to the output type alone uses up half the stated bound or
more (on [4, 8) in bf16: 0.0156 of 0.016, leaving 3.75e-4, a relative 5e-5,
for the arithmetic, while the products take P rounded to bf16, a relative
2^-9 per weight), so the arithmetic keeps the stated bound and the final
rounding comes on top. Everywhere else the bound is the stated one, whatever
the input scale. LSE: max-abs 1e-3 where the oracle's LSE is finite; rows
the oracle finds empty must be exactly LSE = -inf.

Every check records its achieved maximum errors; the test session prints
them at the end (tests/conftest.py), so the margin left under the bounds is
visible in every GPU log.
"""
import numpy as np
import torch

O_SPEC = {torch.bfloat16: 1.6e-2, torch.float16: 4e-3}
LSE_SPEC = 1e-3
_MANT = {torch.bfloat16: 8, torch.float16: 11}      # significand bits, hidden bit included
_EMIN = {torch.bfloat16: -126, torch.float16: -14}  # exponent of the smallest normal

RECORD = []  # (what, o_err, o_err / bound (worst element), lse_err)


def half_ulp(x, dtype):
    """Half the spacing of `dtype` values around |x| (subnormal spacing below
    the smallest normal)."""
    a = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.where(a > 0, a, 2.0 ** _EMIN[dtype])))
    e = np.maximum(e, _EMIN[dtype])
    return np.ldexp(0.5, (e - (_MANT[dtype] - 1)).astype(np.int64))


def o_bound(o_ref, dtype):
    spec = O_SPEC[dtype]
    hu = half_ulp(o_ref, dtype)
    return spec + np.where(hu >= 0.5 * spec, hu, 0.0)


def check(out, lse, o_ref, l_ref, dtype, what=""):
    """Asserts the bounds above; out / lse are the GPU results as float
    arrays, o_ref / l_ref the oracle's. Returns (max O error, max LSE error)."""
    out = np.asarray(out, dtype=np.float64)
    o_ref = np.asarray(o_ref, dtype=np.float64)
    lse = np.asarray(lse, dtype=np.float64)
    l_ref = np.asarray(l_ref, dtype=np.float64)
    assert out.shape == o_ref.shape, "%s: O shape %s vs %s" % (what, out.shape, o_ref.shape)
    fin = np.isfinite(l_ref)
    assert np.array_equal(np.isfinite(lse), fin), what + ": empty-row pattern differs"
    assert np.all(lse[~fin] == -np.inf), what + ": an empty row's LSE is not -inf"
    err = np.abs(out - o_ref)
    o_err = float(err.max()) if err.size else 0.0
    ratio = float((err / o_bound(o_ref, dtype)).max()) if err.size else 0.0
    l_err = float(np.abs(lse[fin] - l_ref[fin]).max()) if fin.any() else 0.0
    RECORD.append((what, o_err, ratio, l_err))
    assert not np.isnan(err).any(), "%s: NaN in O" % what
    assert ratio <= 1.0, "%s: O max-abs error %.3g (%.2f x its bound)" % (what, o_err, ratio)
    assert l_err <= LSE_SPEC, "%s: LSE max-abs error %.3g" % (what, l_err)
    return o_err, l_err
