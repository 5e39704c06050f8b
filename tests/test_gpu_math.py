"""The hand-written math inside the attention kernels, on its own.

tanh_via_exp2 (the softcap's tanh in the decode and backward kernels) and
softcap_fma (the forward's softcap) are evaluated by test-only kernels
(tests/kernels/math_check.cu, compiled here with nvcc) on dense input
sweeps, against fp64 tanh evaluated on the device, and the worst errors are
asserted against the bounds their comments state:
  * tanh absolute error <= 2.5e-7 on +-10^[-8, 3] (log-spaced) and at 0;
  * the forward's folded softcap c tanh(x / s) + b (softcap_fma, the scale
    2 log2(e) / s folded into one multiply) within c (2.5e-7 + 2^-22) plus
    an ulp of c + |b| (the final rounding), for c, s = 50 (and the log2(e)
    scaled c the kernel uses) over the same range of x / s.
"""
import ctypes
import os
import subprocess

import numpy as np

import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
CSRC = os.path.join(ROOT, "exact_io_aware_79_b200", "csrc")


@pytest.fixture(scope="module")
def lib(tmp_path_factory):
    out = str(tmp_path_factory.mktemp("mathcheck") / "libmathcheck.so")
    subprocess.run([os.environ.get("NVCC", "nvcc"), "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                    "-std=c++17", "-Xcompiler", "-fPIC", "-shared", "-I", CSRC, "-o", out,
                    os.path.join(HERE, "kernels", "math_check.cu")], check=True)
    L = ctypes.CDLL(out)
    vp, d, i = ctypes.c_void_p, ctypes.c_double, ctypes.c_int
    L.check_tanh.argtypes = [vp, d, d, i, vp]
    L.check_softcap.argtypes = [vp, d, d, i, ctypes.c_float, ctypes.c_float, ctypes.c_float, vp]
    return L


def _run(fn, *args):
    worst = torch.zeros(4, dtype=torch.float32, device="cuda")
    s = torch.cuda.current_stream()
    assert fn(ctypes.c_void_p(worst.data_ptr()), *args, ctypes.c_void_p(s.cuda_stream)) == 0
    torch.cuda.synchronize()
    return worst.cpu().tolist()


def test_tanh_via_exp2_absolute_error(lib):
    n = 200000
    w = _run(lib.check_tanh, ctypes.c_double(-8.0), ctypes.c_double(11.0 / n), n)
    print("tanh_via_exp2: max absolute error: %.3e" % w[0])
    assert w[1] == 0.0, "NaN result"
    assert w[0] <= 2.5e-7


@pytest.mark.parametrize("c,b", [(50.0, 0.0), (50.0 * 1.4426950408889634, 0.0), (50.0 * 1.4426950408889634, -37.5)])
def test_softcap_fma_absolute_error(lib, c, b):
    n = 200000
    w = _run(lib.check_softcap, ctypes.c_double(-8.0), ctypes.c_double(11.0 / n), n, ctypes.c_float(50.0),
             ctypes.c_float(c), ctypes.c_float(b))
    ulp = np.spacing(np.float32(c + abs(b)))
    bound = c * (2.5e-7 + 2.0 ** -22) + float(ulp)
    print("softcap_fma(c=%g, b=%g): max absolute error %.3e (bound %.3e)" % (c, b, w[0], bound))
    assert w[1] == 0.0, "NaN result"
    assert w[0] <= bound
