"""C-ABI checks that need no GPU: symbols, status strings, argument validation,
split-count and workspace arithmetic.

Validation happens before any CUDA call, so on a machine without a device the
invalid calls return their own status and valid ones return FA_ERR_DEVICE.
Fake device addresses are passed for pointers; nothing dereferences them.
"""
import ctypes
import os
import re

import pytest

from exact_io_aware_79_b200 import build as fbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "fa.h")

OK, NULL, SHAPE, DTYPE, HEADDIM, ARG, WORKSPACE, CUDA, DEVICE = range(9)


@pytest.fixture(scope="module")
def lib():
    fbuild.build()
    import exact_io_aware_79_b200 as fa
    return fa.library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(fa_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    assert {"fa_fwd", "fa_fwd_varlen", "fa_fwd_qkvpacked", "fa_fwd_kvcache", "fa_kvcache_num_splits", "fa_kvcache_workspace_size",
            "fa_status_string"} <= set(names)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code in range(9):
        s = lib.fa_status_string(code).decode()
        assert s.startswith(["FA_OK", "FA_ERR_NULL", "FA_ERR_SHAPE", "FA_ERR_DTYPE", "FA_ERR_HEADDIM",
                             "FA_ERR_ARG", "FA_ERR_WORKSPACE", "FA_ERR_CUDA", "FA_ERR_DEVICE"][code])
    assert "unknown" in lib.fa_status_string(99).decode()


P = 0x10000  # fake 16-byte-aligned device address


def fwd(lib, q=P, k=P, v=P, out=P, lse=P, B=1, H=2, Nq=128, Nk=128, d=128, dtype=1, scale=0.1, causal=0,
        wl=-1, wr=-1, slopes=None, cap=0.0):
    return lib.fa_fwd(q, k, v, out, lse, B, H, Nq, Nk, d, dtype, scale, causal, wl, wr, slopes, cap, None)


def test_fwd_validation(lib):
    assert fwd(lib, d=96) == HEADDIM
    assert fwd(lib, d=256) == HEADDIM
    assert fwd(lib, dtype=2) == DTYPE
    assert fwd(lib, B=-1) == SHAPE
    assert fwd(lib, Nq=-3) == SHAPE
    assert fwd(lib, Nk=1 << 29) == SHAPE
    assert fwd(lib, wl=-2) == ARG
    assert fwd(lib, wr=-5) == ARG
    assert fwd(lib, cap=-1.0) == ARG
    assert fwd(lib, cap=float("inf")) == ARG
    assert fwd(lib, scale=float("nan")) == ARG
    assert fwd(lib, causal=2) == ARG
    assert fwd(lib, q=None) == NULL
    assert fwd(lib, lse=None) == NULL
    assert fwd(lib, k=None) == NULL
    assert fwd(lib, out=P + 8) == ARG          # misaligned
    # empty problems are no-ops, even with NULL pointers
    assert fwd(lib, B=0, q=None, k=None, v=None, out=None, lse=None) == OK
    assert fwd(lib, Nq=0) == OK
    # Nk == 0 needs no K/V pointers
    r = fwd(lib, Nk=0, k=None, v=None)
    assert r in (OK, DEVICE)


def test_fwd_reaches_the_device_check_without_gpu(lib):
    import torch
    if torch.cuda.is_available():
        pytest.skip("a device is present")
    assert fwd(lib) == DEVICE


def fwd_varlen(lib, q=P, k=P, v=P, out=P, lse=P, cq=P, ck=P, B=3, H=2, mq=300, mk=300, tq=600, tk=600, d=128,
               dtype=1, scale=0.1, causal=1, wl=-1, wr=-1, slopes=None, cap=0.0):
    return lib.fa_fwd_varlen(q, k, v, out, lse, cq, ck, B, H, mq, mk, tq, tk, d, dtype, scale, causal, wl, wr,
                             slopes, cap, None)


def test_fwd_varlen_validation(lib):
    assert fwd_varlen(lib, d=96) == HEADDIM
    assert fwd_varlen(lib, dtype=5) == DTYPE
    assert fwd_varlen(lib, B=-1) == SHAPE
    assert fwd_varlen(lib, tq=-1) == SHAPE
    assert fwd_varlen(lib, tk=1 << 29) == SHAPE
    assert fwd_varlen(lib, mq=-2) == SHAPE
    assert fwd_varlen(lib, wl=-3) == ARG
    assert fwd_varlen(lib, cap=-2.0) == ARG
    assert fwd_varlen(lib, causal=3) == ARG
    assert fwd_varlen(lib, cq=None) == NULL
    assert fwd_varlen(lib, ck=None) == NULL
    assert fwd_varlen(lib, q=None) == NULL
    assert fwd_varlen(lib, k=None) == NULL
    assert fwd_varlen(lib, lse=P + 4) == ARG
    # empty problems are no-ops
    assert fwd_varlen(lib, B=0, cq=None, ck=None, q=None) == OK
    assert fwd_varlen(lib, tq=0, q=None, out=None, lse=None) == OK
    assert fwd_varlen(lib, mq=0) == OK
    # no keys at all needs no K/V pointers
    assert fwd_varlen(lib, tk=0, mk=0, k=None, v=None) in (OK, DEVICE)
    assert fwd_varlen(lib) in (OK, DEVICE)


def kv(lib, q=P, kc=P, vc=P, bt=P, sl=P, out=P, lse=P, B=4, H=2, d=128, num_pages=64, page=256, mb=16,
       dtype=1, scale=0.1, wl=-1, slopes=None, cap=0.0, splits=1, ws=None, ws_bytes=0):
    return lib.fa_fwd_kvcache(q, kc, vc, bt, sl, out, lse, B, H, d, num_pages, page, mb, dtype, scale, wl,
                              slopes, cap, splits, ws, ws_bytes, None)


def test_kvcache_validation(lib):
    assert kv(lib, d=80) == HEADDIM
    assert kv(lib, dtype=7) == DTYPE
    assert kv(lib, H=0) == SHAPE
    assert kv(lib, num_pages=0) == SHAPE
    assert kv(lib, page=0) == ARG
    assert kv(lib, splits=65) == ARG
    assert kv(lib, splits=-1) == ARG
    assert kv(lib, wl=-2) == ARG
    assert kv(lib, cap=-0.5) == ARG
    assert kv(lib, B=70000) == SHAPE
    assert kv(lib, mb=1 << 24, page=256) == SHAPE
    assert kv(lib, bt=None) == NULL
    assert kv(lib, sl=None) == NULL
    assert kv(lib, kc=P + 2) == ARG
    assert kv(lib, sl=P + 2) == ARG
    assert kv(lib, B=0, q=None) == OK
    need = lib.fa_kvcache_workspace_size(4, 2, 128, 16, 256, 4)
    assert need > 0
    assert kv(lib, splits=4, ws=None, ws_bytes=0) == WORKSPACE
    assert kv(lib, splits=4, ws=P, ws_bytes=need - 1) == WORKSPACE
    assert kv(lib, splits=4, ws=P + 4, ws_bytes=need) == WORKSPACE
    assert kv(lib, splits=4, ws=P, ws_bytes=need) in (OK, DEVICE)
    assert kv(lib, splits=1, ws=None) in (OK, DEVICE)


def test_split_count_resolution(lib):
    ns = lib.fa_kvcache_num_splits
    assert ns(64, 32, 128, 128, 256, 0) == 16      # 32K max length -> 2048-key splits
    assert ns(64, 32, 128, 128, 256, 5) == 5       # explicit
    assert ns(1, 8, 128, 16, 256, 0) == 16         # small batch: fill the GPU, >= 256 keys a split
    assert ns(1, 1, 128, 1, 256, 0) == 1           # one page: nothing to split
    assert ns(1024, 32, 128, 4, 256, 0) == 1       # short sequences, many heads
    assert ns(4, 2, 128, 16, 256, 65) == -1
    assert ns(4, 2, 96, 16, 256, 0) == -1
    for args in [(64, 32, 128, 128, 256), (3, 5, 64, 7, 16), (1, 1, 128, 2000, 16)]:
        assert 1 <= ns(*args, 0) <= 64


def test_grouped_query_split_count(lib):
    """The grouped-query query reports the count the grouped kernel launches:
    aimed at its CTAs (one per group of query heads), never above the
    one-head count; explicit counts, one-head caches and pages that are not
    multiples of 64 (no grouped kernel) keep the one-head answer."""
    ng, ns = lib.fa_kvcache_num_splits_gqa, lib.fa_kvcache_num_splits
    assert ns(64, 32, 128, 128, 256, 0) == 16
    assert ng(64, 32, 8, 128, 128, 256, 0) == 4     # groups of 4: 4 * 2048 keys a split
    assert ng(64, 32, 32, 128, 128, 256, 0) == 16   # H_kv == H: the one-head count
    assert ng(64, 32, 8, 128, 128, 256, 7) == 7     # explicit
    assert ng(64, 32, 8, 128, 2048, 16, 0) == ns(64, 32, 128, 2048, 16, 0)  # 16-token pages
    assert ng(64, 32, 5, 128, 128, 256, 0) == -1    # H not a multiple of H_kv
    for B, H, Hk, mb, page in [(1, 32, 8, 128, 256), (3, 16, 1, 40, 64), (64, 32, 4, 128, 256)]:
        s = ng(B, H, Hk, 128, mb, page, 0)
        assert 1 <= s <= ns(B, H, 128, mb, page, 0)


def test_workspace_size(lib):
    ws = lib.fa_kvcache_workspace_size
    assert ws(64, 32, 128, 128, 256, 1) == 0
    rows = 16 * 64 * 32
    o_bytes = (rows * 128 * 4 + 255) // 256 * 256
    assert ws(64, 32, 128, 128, 256, 16) == o_bytes + rows * 4
    assert ws(64, 32, 128, 128, 256, 0) == ws(64, 32, 128, 128, 256, 16)
    assert ws(4, 2, 96, 16, 256, 4) == 0          # invalid head dim


def test_gqa_validation(lib):
    def g(H=8, H_kv=2, **kw):
        a = dict(q=P, k=P, v=P, out=P, lse=P, B=1, Nq=128, Nk=128, d=128, dtype=1, scale=0.1, causal=0, wl=-1,
                 wr=-1, slopes=None, cap=0.0)
        a.update(kw)
        return lib.fa_fwd_gqa(a["q"], a["k"], a["v"], a["out"], a["lse"], a["B"], H, H_kv, a["Nq"], a["Nk"],
                              a["d"], a["dtype"], a["scale"], a["causal"], a["wl"], a["wr"], a["slopes"], a["cap"],
                              None)
    assert g(H_kv=3) == SHAPE        # 8 % 3 != 0
    assert g(H_kv=0) == SHAPE
    assert g(H_kv=16) == SHAPE       # more K/V heads than query heads
    assert g(d=80) == HEADDIM
    assert g(k=None) == NULL
    assert g(H_kv=1) in (OK, DEVICE)
    assert g(H_kv=8) in (OK, DEVICE)

    def gk(H=8, H_kv=2, **kw):
        a = dict(q=P, kc=P, vc=P, bt=P, sl=P, out=P, lse=P, B=4, d=128, num_pages=64, page=256, mb=16, dtype=1,
                 scale=0.1, wl=-1, slopes=None, cap=0.0, splits=1, ws=None, ws_bytes=0)
        a.update(kw)
        return lib.fa_fwd_kvcache_gqa(a["q"], a["kc"], a["vc"], a["bt"], a["sl"], a["out"], a["lse"], a["B"], H,
                                      H_kv, a["d"], a["num_pages"], a["page"], a["mb"], a["dtype"], a["scale"],
                                      a["wl"], a["slopes"], a["cap"], a["splits"], a["ws"], a["ws_bytes"], None)
    assert gk(H_kv=5) == SHAPE
    assert gk(H_kv=0) == SHAPE
    assert gk(bt=None) == NULL
    assert gk(splits=4, ws=None) == WORKSPACE
    assert gk(H_kv=4) in (OK, DEVICE)


def test_append_validation(lib):
    def ap(**kw):
        a = dict(kn=P, vn=P, kc=P, vc=P, bt=P, sl=P, B=4, n=1, Hkv=2, d=128, num_pages=64, page=256, mb=16,
                 dtype=1)
        a.update(kw)
        return lib.fa_kvcache_append(a["kn"], a["vn"], a["kc"], a["vc"], a["bt"], a["sl"], a["B"], a["n"],
                                     a["Hkv"], a["d"], a["num_pages"], a["page"], a["mb"], a["dtype"], None)
    assert ap(d=96) == HEADDIM
    assert ap(dtype=3) == DTYPE
    assert ap(B=-1) == SHAPE
    assert ap(n=-1) == SHAPE
    assert ap(Hkv=0) == SHAPE
    assert ap(num_pages=0) == SHAPE
    assert ap(page=0) == ARG
    assert ap(B=70000) == SHAPE
    assert ap(kn=None) == NULL
    assert ap(sl=None) == NULL
    assert ap(kc=P + 8) == ARG
    assert ap(bt=P + 2) == ARG
    assert ap(n=0, kn=None) == OK       # nothing to append
    assert ap() in (OK, DEVICE)


def test_qkvpacked_validation(lib):
    def pk(qkv=P, out=P, lse=P, B=1, H=2, N=128, d=128, dtype=1, cap=0.0, wl=-1):
        return lib.fa_fwd_qkvpacked(qkv, out, lse, B, H, N, d, dtype, 0.1, 1, wl, -1, None, cap, None)
    assert pk(d=96) == HEADDIM
    assert pk(dtype=4) == DTYPE
    assert pk(N=-1) == SHAPE
    assert pk(qkv=None) == NULL
    assert pk(lse=None) == NULL
    assert pk(cap=-1.0) == ARG
    assert pk(B=0, qkv=None) == OK
    assert pk() in (OK, DEVICE)

    def vpk(qkv=P, cu=P, B=2, total=300, mx=200):
        return lib.fa_fwd_varlen_qkvpacked(qkv, P, P, cu, B, 2, mx, total, 128, 1, 0.1, 1, -1, -1, None, 0.0, None)
    assert vpk(cu=None) == NULL
    assert vpk(total=-5) == SHAPE
    assert vpk(total=0) == OK
    assert vpk() in (OK, DEVICE)


def test_bwd_validation(lib):
    def bw(**kw):
        a = dict(q=P, k=P, v=P, out=P, lse=P, dout=P, dq=P, dk=P, dv=P, B=2, H=8, H_kv=2, Nq=100, Nk=200, d=128,
                 dtype=1, scale=0.1, causal=1, wl=-1, wr=-1, slopes=None, cap=0.0, det=0, ws=P,
                 ws_bytes=lib.fa_bwd_workspace_size(2, 8, 100, 128))
        a.update(kw)
        return lib.fa_bwd(a["q"], a["k"], a["v"], a["out"], a["lse"], a["dout"], a["dq"], a["dk"], a["dv"], a["B"],
                          a["H"], a["H_kv"], a["Nq"], a["Nk"], a["d"], a["dtype"], a["scale"], a["causal"], a["wl"],
                          a["wr"], a["slopes"], a["cap"], a["det"], a["ws"], a["ws_bytes"], None)
    assert bw() == DEVICE
    assert bw(det=1) == DEVICE
    assert bw(det=2) == ARG
    assert bw(H_kv=3) == SHAPE
    assert bw(H_kv=16) == SHAPE
    # jobs of the persistent kernels must number below 2^31: ceil(Nk / 128) B H_kv
    # (and ceil(Nq / 128) B H in the deterministic mode)
    assert bw(B=1024, Nk=1 << 28) == SHAPE        # 2^21 * 1024 * 2 = 2^32 key-block jobs
    big = lib.fa_bwd_workspace_size(40000, 8, 100, 128)
    assert bw(B=40000, H_kv=2, ws_bytes=big) == DEVICE              # B * H_kv = 80000: fine
    assert bw(B=40000, H_kv=2, det=1, ws_bytes=big) == DEVICE       # B * H = 320000: fine
    assert bw(B=1024, Nq=1 << 28, det=1) == SHAPE    # 2^21 * 1024 * 8 = 2^34 query-tile jobs
    assert bw(d=96) == HEADDIM
    assert bw(dtype=7) == DTYPE
    assert bw(scale=float("nan")) == ARG
    assert bw(cap=-1.0) == ARG
    assert bw(wl=-2) == ARG
    assert bw(causal=2) == ARG
    assert bw(dout=None) == NULL
    assert bw(dk=None) == NULL
    assert bw(dq=P + 8) == ARG                   # not 16-byte aligned
    assert bw(ws=None) == WORKSPACE
    assert bw(ws_bytes=lib.fa_bwd_workspace_size(2, 8, 100, 128) - 1) == WORKSPACE
    assert bw(B=0) == OK
    assert bw(Nq=0, ws=None, ws_bytes=0) == DEVICE   # zero dk, dv: no workspace needed
    # fp32 dq accumulator rows (256-byte rounded) + D rows + 256 bytes (the job counter)
    assert lib.fa_bwd_workspace_size(2, 8, 100, 128) == (2 * 8 * 100 * 128 * 4 + 255) // 256 * 256 + \
        (2 * 8 * 100 * 4 + 255) // 256 * 256 + 256
    assert lib.fa_bwd_workspace_size(-1, 8, 100, 128) == 0


def test_bwd_varlen_validation(lib):
    def bv(**kw):
        a = dict(q=P, k=P, v=P, out=P, lse=P, dout=P, dq=P, dk=P, dv=P, cq=P, ck=P, B=3, H=4, H_kv=2, mq=300,
                 mk=300, tq=500, tk=600, d=128, dtype=1, scale=0.1, causal=1, wl=-1, wr=-1, slopes=None, cap=0.0,
                 det=0, ws=P, ws_bytes=lib.fa_bwd_workspace_size(1, 4, 500, 128))
        a.update(kw)
        return lib.fa_bwd_varlen(a["q"], a["k"], a["v"], a["out"], a["lse"], a["dout"], a["dq"], a["dk"], a["dv"],
                                 a["cq"], a["ck"], a["B"], a["H"], a["H_kv"], a["mq"], a["mk"], a["tq"], a["tk"],
                                 a["d"], a["dtype"], a["scale"], a["causal"], a["wl"], a["wr"], a["slopes"],
                                 a["cap"], a["det"], a["ws"], a["ws_bytes"], None)
    assert bv() == DEVICE
    assert bv(H_kv=3) == SHAPE
    assert bv(B=20000) in (OK, DEVICE)          # no grid limit on B * H (persistent kernels)
    assert bv(tq=-1) == SHAPE
    assert bv(d=80) == HEADDIM
    assert bv(cq=None) == NULL
    assert bv(cq=P + 2) == ARG                   # int32 array not 4-byte aligned
    assert bv(det=3) == ARG
    assert bv(ws=None) == WORKSPACE
    assert bv(tq=0, tk=0) == OK


def test_bwd_qkvpacked_validation(lib):
    ws = lib.fa_bwd_workspace_size(2, 4, 100, 128)
    f = lambda **kw: lib.fa_bwd_qkvpacked(kw.get("qkv", P), P, P, P, kw.get("dqkv", P), 2, 4, 100,
                                          kw.get("d", 128), 1, 0.1, 1, -1, -1, None, 0.0, kw.get("det", 0),
                                          kw.get("ws", P), ws, None)
    assert f() == DEVICE
    assert f(d=48) == HEADDIM
    assert f(dqkv=None) == NULL
    assert f(det=5) == ARG
    assert f(ws=None) == WORKSPACE
    g = lambda **kw: lib.fa_bwd_varlen_qkvpacked(P, P, P, P, P, kw.get("cu", P), 3, 4, 100, 250, 128, 1, 0.1, 1,
                                                 -1, -1, None, 0.0, 0, P, lib.fa_bwd_workspace_size(1, 4, 250, 128),
                                                 None)
    assert g() == DEVICE
    assert g(cu=None) == NULL


def test_header_is_plain_c_and_every_entry_links(lib, tmp_path):
    """The boundary needs no C++ and no torch: a C99 program that takes the
    address of every function the header declares compiles with -Werror and
    links against the library."""
    import shutil
    import subprocess
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    names = declared_functions()
    src = tmp_path / "abi_user.c"
    src.write_text('#include "fa.h"\n#include <stdio.h>\nint main(void) {\n  void (*fns[])(void) = {\n' +
                   ",\n".join("    (void (*)(void))%s" % n for n in names) +
                   '\n  };\n  printf("%d\\n", (int)(sizeof(fns) / sizeof(fns[0])));\n  return 0;\n}\n')
    libdir = os.path.dirname(lib._name)
    cuda_inc = os.path.join(os.environ.get("CUDA_HOME", "/usr/local/cuda"), "include")
    out = tmp_path / "abi_user"
    r = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(ROOT, "include"), "-I", cuda_inc,
                        str(src), "-L", libdir, "-lfa_b200", "-o", str(out)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
