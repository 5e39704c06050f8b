"""Pins for the fp64 oracle, against facts fixed by the mathematics and the pages.

None of these tests re-types the oracle's formula and compares: each one
checks an invariant, a closed form, a special case that reduces to something
simpler, or a brute-force enumeration on a tiny input, chosen so that a
plausible slip in the oracle (a dropped scale, a wrong sign, a top-left
instead of bottom-right mask, an off-by-one window, a transposed operand, a
wrong page index, a wrong merge weight) fails at least one of them.
"""
import math

import numpy as np
import pytest
import torch

import oracle

TOL = 1e-12


def rnd(shape, seed, sigma=1.0):
    g = np.random.default_rng(seed)
    return g.standard_normal(shape) * sigma


# ---------------------------------------------------------------- storage widening

def test_widen_fp16_every_bit_pattern():
    bits = np.arange(65536, dtype=np.uint16)
    got = oracle.widen(bits, oracle.F16)
    want = bits.view(np.float16).astype(np.float64)
    same = (got == want) | (np.isnan(got) & np.isnan(want))
    assert same.all()


def test_widen_bf16_every_bit_pattern():
    bits = np.arange(65536, dtype=np.uint16)
    got = oracle.widen(bits, oracle.BF16)
    want = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    same = (got == want) | (np.isnan(got) & np.isnan(want))
    assert same.all()


# ---------------------------------------------------------------- invariants named by the spec

MASKS = [
    dict(causal=False),
    dict(causal=True),
    dict(causal=True, window_left=3, window_right=0),
    dict(causal=False, window_left=2, window_right=1),
]


@pytest.mark.parametrize("Nq,Nk", [(7, 7), (5, 11), (11, 5)])
@pytest.mark.parametrize("mask", MASKS)
def test_probability_rows_sum_to_one(Nq, Nk, mask):
    B, H, d = 2, 3, 8
    q, k, v = rnd((B, Nq, H, d), 1), rnd((B, Nk, H, d), 2), rnd((B, Nk, H, d), 3)
    o, lse, p = oracle.attn_fwd(q, k, v, 0.4, alibi_slopes=[0.5, 0.1, 0.0], softcap=3.0,
                                return_probs=True, **mask)
    sums = p.sum(axis=-1)
    nonempty = np.isfinite(lse)
    assert np.allclose(sums[nonempty], 1.0, atol=TOL, rtol=0)
    assert np.all(sums[~nonempty] == 0.0)
    assert (p >= 0).all()
    # the same fact seen through O: with V = 1 every non-empty row of O is 1
    o1, _ = oracle.attn_fwd(q, k, np.ones_like(v), 0.4, alibi_slopes=[0.5, 0.1, 0.0], softcap=3.0,
                            **mask)
    ne = np.transpose(nonempty, (0, 2, 1))  # [B, Nq, H]
    assert np.allclose(o1[ne], 1.0, atol=TOL, rtol=0)
    assert np.all(o1[~ne] == 0.0)


def test_single_key_returns_v():
    B, H, Nq, d = 2, 3, 9, 16
    q, k, v = rnd((B, Nq, H, d), 4), rnd((B, 1, H, d), 5), rnd((B, 1, H, d), 6)
    o, lse = oracle.attn_fwd(q, k, v, 0.25)
    assert np.allclose(o, np.broadcast_to(v, o.shape), atol=TOL, rtol=0)
    # with one key the LSE is that key's scaled score
    s = 0.25 * np.einsum("bihc,bhc->bhi", q, k[:, 0])
    assert np.allclose(lse, s, atol=TOL, rtol=0)


@pytest.mark.parametrize("Nk", [1, 6, 33])
def test_zero_query_gives_column_mean_and_ln_n(Nk):
    B, H, Nq, d = 2, 2, 5, 8
    q = np.zeros((B, Nq, H, d))
    k, v = rnd((B, Nk, H, d), 7), rnd((B, Nk, H, d), 8)
    o, lse = oracle.attn_fwd(q, k, v, 1.0)
    mean = v.mean(axis=1)  # [B, H, d]
    assert np.allclose(o, mean[:, None], atol=TOL, rtol=0)
    assert np.allclose(lse, math.log(Nk), atol=TOL, rtol=0)


def test_joint_permutation_of_keys_and_values():
    B, H, Nq, Nk, d = 2, 3, 6, 13, 8
    q, k, v = rnd((B, Nq, H, d), 9), rnd((B, Nk, H, d), 10), rnd((B, Nk, H, d), 11)
    perm = np.random.default_rng(12).permutation(Nk)
    o1, l1 = oracle.attn_fwd(q, k, v, 0.3, softcap=2.0)
    o2, l2 = oracle.attn_fwd(q, k[:, perm], v[:, perm], 0.3, softcap=2.0)
    assert np.allclose(o1, o2, atol=TOL, rtol=0)
    assert np.allclose(l1, l2, atol=TOL, rtol=0)
    # but the permutation must move V with K: permuting V alone changes O
    o3, _ = oracle.attn_fwd(q, k, v[:, perm], 0.3, softcap=2.0)
    assert np.abs(o3 - o1).max() > 1e-3


def brute_force(q, k, v, scale, causal=False, wl=-1, wr=-1, slopes=None, softcap=0.0):
    """Enumerates every (b, i, h) and every key with Python floats."""
    B, Nq, H, d = q.shape
    Nk = k.shape[1]
    o = np.zeros((B, Nq, H, d))
    lse = np.zeros((B, H, Nq))
    for b in range(B):
        for h in range(H):
            for i in range(Nq):
                pos = i + Nk - Nq          # bottom-right: last query row meets last key
                terms = []
                for j in range(Nk):
                    if causal and j > pos:
                        continue
                    if wl >= 0 and j < pos - wl:
                        continue
                    if wr >= 0 and j > pos + wr:
                        continue
                    x = scale * sum(float(q[b, i, h, c]) * float(k[b, j, h, c]) for c in range(d))
                    if softcap > 0:
                        x = softcap * math.tanh(x / softcap)
                    if slopes is not None:
                        x -= slopes[h] * abs(pos - j)
                    terms.append((j, x))
                if not terms:
                    lse[b, h, i] = -math.inf
                    continue
                mx = max(x for _, x in terms)
                z = sum(math.exp(x - mx) for _, x in terms)
                for j, x in terms:
                    o[b, i, h] += math.exp(x - mx) / z * v[b, j, h]
                lse[b, h, i] = mx + math.log(z)
    return o, lse


@pytest.mark.parametrize("Nq,Nk", [(4, 9), (9, 9), (9, 4), (1, 7)])
@pytest.mark.parametrize("opts", [
    dict(causal=True),
    dict(causal=True, wl=2, wr=0),
    dict(causal=False, wl=1, wr=2),
    dict(causal=True, slopes=[0.7, 0.05]),
    dict(causal=False, softcap=1.5),
    dict(causal=True, wl=3, wr=0, slopes=[0.3, 1.1], softcap=2.5),
])
def test_matches_brute_force_with_bottom_right_alignment(Nq, Nk, opts):
    B, H, d = 2, 2, 5
    q, k, v = rnd((B, Nq, H, d), 13, 1.5), rnd((B, Nk, H, d), 14, 1.5), rnd((B, Nk, H, d), 15)
    want_o, want_l = brute_force(q, k, v, 0.6, **opts)
    o, lse = oracle.attn_fwd(q, k, v, 0.6, causal=opts.get("causal", False),
                             window_left=opts.get("wl", -1), window_right=opts.get("wr", -1),
                             alibi_slopes=opts.get("slopes"), softcap=opts.get("softcap", 0.0))
    assert np.allclose(o, want_o, atol=1e-11, rtol=0)
    fin = np.isfinite(want_l)
    assert np.array_equal(fin, np.isfinite(lse))
    assert np.allclose(lse[fin], want_l[fin], atol=1e-11, rtol=0)


def test_unbounded_window_is_full_attention():
    B, H, Nq, Nk, d = 1, 2, 10, 14, 8
    q, k, v = rnd((B, Nq, H, d), 16), rnd((B, Nk, H, d), 17), rnd((B, Nk, H, d), 18)
    for causal in (False, True):
        o1, l1 = oracle.attn_fwd(q, k, v, 0.3, causal=causal)
        o2, l2 = oracle.attn_fwd(q, k, v, 0.3, causal=causal, window_left=10**9, window_right=10**9)
        assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


def test_huge_softcap_and_zero_slopes_are_plain_attention():
    B, H, Nq, Nk, d = 2, 3, 8, 8, 8
    q, k, v = rnd((B, Nq, H, d), 19), rnd((B, Nk, H, d), 20), rnd((B, Nk, H, d), 21)
    o0, l0 = oracle.attn_fwd(q, k, v, 0.3, causal=True)
    o1, l1 = oracle.attn_fwd(q, k, v, 0.3, causal=True, softcap=1e30)
    o2, l2 = oracle.attn_fwd(q, k, v, 0.3, causal=True, alibi_slopes=[0.0, 0.0, 0.0])
    for o, l in ((o1, l1), (o2, l2)):
        assert np.allclose(o, o0, atol=TOL, rtol=0) and np.allclose(l, l0, atol=TOL, rtol=0)


# ---------------------------------------------------------------- closed forms

def visible_count(Nq, Nk, i, causal, wl, wr):
    """Number of keys row i sees, from interval arithmetic (no enumeration)."""
    pos = i + Nk - Nq
    lo = 0 if wl < 0 else max(0, pos - wl)
    hi = Nk - 1
    if causal:
        hi = min(hi, pos)
    if wr >= 0:
        hi = min(hi, pos + wr)
    return max(0, hi - lo + 1), lo, hi


@pytest.mark.parametrize("Nq,Nk", [(16, 16), (6, 20), (20, 6)])
@pytest.mark.parametrize("causal,wl,wr", [(True, -1, -1), (True, 4, 0), (False, 3, 2), (False, 0, 0),
                                          (False, -1, 5)])
def test_zero_query_counts_visible_keys(Nq, Nk, causal, wl, wr):
    """With Q = 0 every visible score is 0, so LSE_i = ln(count_i) and O_i is
    the mean of the visible V rows; this fixes the mask of every row."""
    B, H, d = 1, 2, 4
    q = np.zeros((B, Nq, H, d))
    k, v = rnd((B, Nk, H, d), 22), rnd((B, Nk, H, d), 23)
    o, lse = oracle.attn_fwd(q, k, v, 1.0, causal=causal, window_left=wl, window_right=wr)
    for i in range(Nq):
        n, lo, hi = visible_count(Nq, Nk, i, causal, wl, wr)
        if n == 0:
            assert np.all(lse[:, :, i] == -np.inf) and np.all(o[:, i] == 0)
        else:
            assert np.allclose(lse[:, :, i], math.log(n), atol=TOL, rtol=0)
            assert np.allclose(o[:, i], v[:, lo:hi + 1].mean(axis=1), atol=TOL, rtol=0)


@pytest.mark.parametrize("Nq,Nk", [(8, 8), (3, 8), (8, 3)])
def test_one_hot_probe_pins_each_key(Nq, Nk):
    """K row t is lam * e0 and all others are 0; Q = e0. Then row i puts
    (almost) all weight on key t when t is visible, and else spreads it evenly
    over its visible keys (all other scores are 0)."""
    B, H, d, lam = 1, 1, 4, 200.0
    for causal, wl, wr in [(True, -1, -1), (True, 2, 0), (False, 1, 1)]:
        for t in range(Nk):
            q = np.zeros((B, Nq, H, d))
            q[..., 0] = 1.0
            k = np.zeros((B, Nk, H, d))
            k[0, t, 0, 0] = lam
            v = rnd((B, Nk, H, d), 24 + t)
            o, lse = oracle.attn_fwd(q, k, v, 1.0, causal=causal, window_left=wl, window_right=wr)
            for i in range(Nq):
                n, lo, hi = visible_count(Nq, Nk, i, causal, wl, wr)
                if n == 0:
                    assert lse[0, 0, i] == -np.inf
                elif lo <= t <= hi:
                    assert np.allclose(o[0, i, 0], v[0, t, 0], atol=1e-60 + 1e-80, rtol=1e-12)
                    assert abs(lse[0, 0, i] - lam) < 1e-12 * lam
                else:
                    assert np.allclose(o[0, i, 0], v[0, lo:hi + 1, 0].mean(axis=0), atol=TOL)


@pytest.mark.parametrize("slope", [0.0, 0.03, 0.5, 2.0])
def test_alibi_is_a_geometric_series(slope):
    """Q = 0, causal, Nq = Nk: row i has scores -slope*(i - j), j <= i, so with
    r = exp(-slope) the LSE is ln((1 - r^(i+1)) / (1 - r)) (or ln(i+1) for
    r = 1) and the weight on key j is r^(i-j) / sum."""
    B, H, N, d = 1, 1, 12, 4
    q = np.zeros((B, N, H, d))
    k = rnd((B, N, H, d), 40)
    v = np.zeros((B, N, H, d))
    v[0, :, 0, 0] = np.arange(N)          # O_i[0] is then the mean key index under P
    o, lse = oracle.attn_fwd(q, k, v, 1.0, causal=True, alibi_slopes=[slope])
    r = math.exp(-slope)
    for i in range(N):
        z = (i + 1.0) if slope == 0 else (1 - r ** (i + 1)) / (1 - r)
        assert abs(lse[0, 0, i] - math.log(z)) < 1e-12
        mean_j = sum(j * r ** (i - j) for j in range(i + 1)) / z
        assert abs(o[0, i, 0, 0] - mean_j) < 1e-12


@pytest.mark.parametrize("cap", [0.5, 2.0, 50.0])
def test_softcap_two_key_closed_form(cap):
    """Two keys with raw scaled scores a and b: softcap maps them to
    c*tanh(a/c), c*tanh(b/c); the weight of key 0 is the logistic of their
    difference. scale = 0.5 is applied before the cap."""
    q = np.zeros((1, 1, 1, 2))
    q[0, 0, 0] = [1.0, 0.0]
    k = np.zeros((1, 2, 1, 2))
    k[0, 0, 0, 0], k[0, 1, 0, 0] = 6.0, -2.0          # raw dots 6, -2 -> scaled 3, -1
    v = np.zeros((1, 2, 1, 2))
    v[0, 0, 0, 0] = 1.0                               # O[0] = weight of key 0
    o, lse = oracle.attn_fwd(q, k, v, 0.5, softcap=cap)
    a, b = cap * math.tanh(3.0 / cap), cap * math.tanh(-1.0 / cap)
    w0 = 1.0 / (1.0 + math.exp(b - a))
    assert abs(o[0, 0, 0, 0] - w0) < 1e-14
    assert abs(lse[0, 0, 0] - (a + math.log1p(math.exp(b - a)))) < 1e-14


def test_fully_masked_rows_are_empty():
    B, H, Nq, Nk, d = 1, 2, 9, 4, 8
    q, k, v = rnd((B, Nq, H, d), 25), rnd((B, Nk, H, d), 26), rnd((B, Nk, H, d), 27)
    o, lse = oracle.attn_fwd(q, k, v, 0.3, causal=True)
    # bottom-right alignment: rows 0..Nq-Nk-1 sit before the first key
    assert np.all(lse[:, :, :Nq - Nk] == -np.inf)
    assert np.all(o[:, :Nq - Nk] == 0.0)
    assert np.all(np.isfinite(lse[:, :, Nq - Nk:]))


def test_row_subset_matches_full():
    B, H, Nq, Nk, d = 2, 2, 17, 23, 8
    q, k, v = rnd((B, Nq, H, d), 28), rnd((B, Nk, H, d), 29), rnd((B, Nk, H, d), 30)
    o, lse = oracle.attn_fwd(q, k, v, 0.3, causal=True, window_left=5)
    rows = [0, 3, 16, 8]
    os_, ls = oracle.attn_fwd(q, k, v, 0.3, causal=True, window_left=5, rows=rows)
    assert np.array_equal(os_, o[:, rows]) and np.array_equal(ls, lse[:, :, rows])


def test_float64_library_softmax_on_tiny_shapes():
    """torch's float64 softmax (a library routine) over an explicitly masked
    score matrix agrees with the oracle."""
    B, H, Nq, Nk, d = 2, 2, 6, 10, 8
    q, k, v = rnd((B, Nq, H, d), 31), rnd((B, Nk, H, d), 32), rnd((B, Nk, H, d), 33)
    tq, tk, tv = (torch.from_numpy(x) for x in (q, k, v))
    s = torch.einsum("bihc,bjhc->bhij", tq, tk) * 0.35
    i = torch.arange(Nq)[:, None] + (Nk - Nq)
    j = torch.arange(Nk)[None, :]
    s = s.masked_fill(j > i, float("-inf"))
    p = torch.softmax(s, dim=-1)
    want = torch.einsum("bhij,bjhc->bihc", p, tv).numpy()
    o, lse = oracle.attn_fwd(q, k, v, 0.35, causal=True)
    assert np.allclose(o, want, atol=TOL, rtol=0)
    assert np.allclose(lse, torch.logsumexp(s, dim=-1).numpy(), atol=TOL, rtol=0)


def test_half_precision_storage_is_widened_exactly():
    B, H, Nq, Nk, d = 1, 2, 5, 7, 8
    for dt in (torch.float16, torch.bfloat16):
        q = torch.randn(B, Nq, H, d).to(dt)
        k = torch.randn(B, Nk, H, d).to(dt)
        v = torch.randn(B, Nk, H, d).to(dt)
        o1, l1 = oracle.attn_fwd(q, k, v, 0.3, causal=True)
        o2, l2 = oracle.attn_fwd(q.double(), k.double(), v.double(), 0.3, causal=True)
        assert np.array_equal(o1, o2) and np.array_equal(l1, l2)


# ---------------------------------------------------------------- paged decode

def contiguous_from_pages(w_k, w_v, table, lens, page):
    """Builds per-sequence contiguous K/V [B, Lmax, H, d] by walking pages."""
    B = table.shape[0]
    Lmax = int(max(lens))
    H, d = w_k.shape[2], w_k.shape[3]
    k = np.zeros((B, Lmax, H, d))
    v = np.zeros((B, Lmax, H, d))
    for b in range(B):
        for t in range(int(lens[b])):
            pg = table[b, t // page]
            k[b, t] = w_k[pg, t % page]
            v[b, t] = w_v[pg, t % page]
    return k, v


def decode_case(seed, B=3, H=2, d=8, page=4, max_blocks=5, lens=(7, 20, 1)):
    g = np.random.default_rng(seed)
    num_pages = B * max_blocks
    kc = g.standard_normal((num_pages, page, H, d))
    vc = g.standard_normal((num_pages, page, H, d))
    table = g.permutation(num_pages).reshape(B, max_blocks).astype(np.int32)
    q = g.standard_normal((B, 1, H, d))
    return q, kc, vc, table, np.array(lens, dtype=np.int32)


def test_identity_block_table_equals_contiguous_cache():
    B, H, d, page, mb = 2, 2, 8, 4, 5
    g = np.random.default_rng(50)
    k = g.standard_normal((B, mb * page, H, d))
    v = g.standard_normal((B, mb * page, H, d))
    q = g.standard_normal((B, 1, H, d))
    lens = np.array([13, 20], dtype=np.int32)
    table = np.arange(B * mb, dtype=np.int32).reshape(B, mb)      # identity
    kc = k.reshape(B * mb, page, H, d)
    vc = v.reshape(B * mb, page, H, d)
    o, lse = oracle.attn_decode_paged(q, kc, vc, table, lens, 0.3)
    for b in range(B):
        L = int(lens[b])
        want_o, want_l = oracle.attn_fwd(q[b:b + 1], k[b:b + 1, :L], v[b:b + 1, :L], 0.3, causal=True)
        assert np.allclose(o[b], want_o[0], atol=TOL, rtol=0)
        assert np.allclose(lse[b], want_l[0], atol=TOL, rtol=0)


@pytest.mark.parametrize("opts", [dict(), dict(window_left=5), dict(alibi_slopes=[0.2, 0.6], softcap=2.0)])
def test_permuted_block_table_is_a_reindexing(opts):
    q, kc, vc, table, lens = decode_case(51)
    o, lse = oracle.attn_decode_paged(q, kc, vc, table, lens, 0.3, **opts)
    k, v = contiguous_from_pages(kc, vc, table, lens, 4)
    for b in range(len(lens)):
        L = int(lens[b])
        wo, wl = brute_force(q[b:b + 1], k[b:b + 1, :L], v[b:b + 1, :L], 0.3, causal=True,
                             wl=opts.get("window_left", -1), slopes=opts.get("alibi_slopes"),
                             softcap=opts.get("softcap", 0.0))
        assert np.allclose(o[b], wo[0], atol=1e-11, rtol=0)
        assert np.allclose(lse[b], wl[0], atol=1e-11, rtol=0)


def test_decode_query_sees_all_cached_keys():
    """The decode example of the causal-alignment change: one query against
    N+1 keys attends to every key, i.e. equals non-causal attention."""
    q, kc, vc, table, lens = decode_case(52, lens=(9, 17, 4))
    o, lse = oracle.attn_decode_paged(q, kc, vc, table, lens, 0.3)
    k, v = contiguous_from_pages(kc, vc, table, lens, 4)
    for b in range(3):
        L = int(lens[b])
        wo, wl = oracle.attn_fwd(q[b:b + 1], k[b:b + 1, :L], v[b:b + 1, :L], 0.3, causal=False)
        assert np.allclose(o[b], wo[0], atol=TOL, rtol=0) and np.allclose(lse[b], wl[0], atol=TOL)


def test_empty_sequence_is_empty():
    q, kc, vc, table, lens = decode_case(53, lens=(0, 5, 0))
    o, lse = oracle.attn_decode_paged(q, kc, vc, table, lens, 0.3)
    assert np.all(o[0] == 0) and np.all(lse[0] == -np.inf) and np.all(lse[2] == -np.inf)
    assert np.all(np.isfinite(lse[1]))


@pytest.mark.parametrize("S", [2, 3, 4, 5, 8, 16])
@pytest.mark.parametrize("opts", [dict(), dict(window_left=6), dict(alibi_slopes=[0.2, 0.6], softcap=2.0)])
def test_any_split_count_matches_one_split(S, opts):
    q, kc, vc, table, lens = decode_case(54, lens=(7, 20, 1))
    o1, l1 = oracle.attn_decode_paged(q, kc, vc, table, lens, 0.3, **opts)
    op, lp = oracle.attn_decode_paged(q, kc, vc, table, lens, 0.3, num_splits=S, **opts)
    o, lse = oracle.combine_splits(op, lp)
    assert np.allclose(o, o1[:, 0], atol=TOL, rtol=0)
    assert np.allclose(lse, l1[:, :, 0], atol=TOL, rtol=0)
    # the partials cover disjoint key ranges: their exp(lse) add up to exp(lse)
    total = np.exp(lp).sum(axis=0)
    assert np.allclose(total, np.exp(l1[:, :, 0]), rtol=1e-12, atol=0)


def test_combine_of_all_empty_splits_is_empty():
    op = np.zeros((3, 2, 4))
    lp = np.full((3, 2), -np.inf)
    lp[1, 1] = 0.5
    op[1, 1] = [1, 2, 3, 4]
    o, lse = oracle.combine_splits(op, lp)
    assert lse[0] == -np.inf and np.all(o[0] == 0)
    assert abs(lse[1] - 0.5) < TOL and np.allclose(o[1], [1, 2, 3, 4], atol=TOL)


def test_decode_rejects_bad_block_table():
    q, kc, vc, table, lens = decode_case(55)
    bad = table.copy()
    bad[1, 0] = kc.shape[0]            # page index past the pool
    with pytest.raises(ValueError):
        oracle.attn_decode_paged(q, kc, vc, bad, lens, 0.3)


# ------------------------------------------------------------ variable length

def varlen_case(lens_q, lens_k, seed, H=2, d=8):
    cq = np.concatenate([[0], np.cumsum(lens_q)]).astype(np.int32)
    ck = np.concatenate([[0], np.cumsum(lens_k)]).astype(np.int32)
    q = rnd((int(cq[-1]), H, d), seed)
    k = rnd((int(ck[-1]), H, d), seed + 1)
    v = rnd((int(ck[-1]), H, d), seed + 2)
    return q, k, v, cq, ck


@pytest.mark.parametrize("opts", [
    dict(causal=True),
    dict(),
    dict(causal=True, window_left=2, window_right=0),
    dict(alibi_slopes=[0.25, 0.7], softcap=3.0, causal=True),
])
def test_varlen_matches_brute_force_per_sequence(opts):
    # ragged lengths, Nq < Nk, Nq > Nk, a sequence without keys and one
    # without queries: each sequence is its own bottom-right aligned problem
    lens_q, lens_k = [3, 5, 0, 4, 2], [6, 2, 3, 4, 0]
    q, k, v, cq, ck = varlen_case(lens_q, lens_k, 11)
    o, lse = oracle.attn_fwd_varlen(q, k, v, cq, ck, 0.4, **opts)
    bf = dict(causal=opts.get("causal", False), wl=opts.get("window_left", -1), wr=opts.get("window_right", -1),
              slopes=opts.get("alibi_slopes"), softcap=opts.get("softcap", 0.0))
    for b in range(len(lens_q)):
        q0, q1, k0, k1 = cq[b], cq[b + 1], ck[b], ck[b + 1]
        if q1 == q0:
            continue
        ob, lb = brute_force(q[q0:q1][None], k[k0:k1][None], v[k0:k1][None], 0.4, **bf)
        np.testing.assert_allclose(o[q0:q1], ob[0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[:, q0:q1], lb[0], rtol=0, atol=1e-12)


def test_varlen_equal_lengths_is_the_batched_problem():
    B, N, H, d = 3, 7, 2, 8
    q, k, v = rnd((B, N, H, d), 21), rnd((B, N + 2, H, d), 22), rnd((B, N + 2, H, d), 23)
    o, lse = oracle.attn_fwd(q, k, v, 0.3, causal=True)
    cq = np.arange(B + 1, dtype=np.int32) * N
    ck = np.arange(B + 1, dtype=np.int32) * (N + 2)
    ov, lv = oracle.attn_fwd_varlen(q.reshape(B * N, H, d), k.reshape(B * (N + 2), H, d),
                                    v.reshape(B * (N + 2), H, d), cq, ck, 0.3, causal=True)
    assert np.array_equal(ov, o.reshape(B * N, H, d))
    assert np.array_equal(lv, lse.transpose(1, 0, 2).reshape(H, B * N))


def test_varlen_sequences_do_not_see_each_other():
    q, k, v, cq, ck = varlen_case([4, 3], [5, 6], 31)
    o1, l1 = oracle.attn_fwd_varlen(q, k, v, cq, ck, 0.5)
    k2, v2 = k.copy(), v.copy()
    k2[ck[1]:] += 1.0
    v2[ck[1]:] -= 2.0
    o2, l2 = oracle.attn_fwd_varlen(q, k2, v2, cq, ck, 0.5)
    assert np.array_equal(o1[:cq[1]], o2[:cq[1]]) and np.array_equal(l1[:, :cq[1]], l2[:, :cq[1]])
    assert not np.allclose(o1[cq[1]:], o2[cq[1]:])


def test_varlen_rows_outside_every_sequence_are_nan():
    q, k, v, cq, ck = varlen_case([2, 3], [2, 3], 41)
    q = np.concatenate([q, rnd((2,) + q.shape[1:], 42)])  # two trailing rows no sequence owns
    o, lse = oracle.attn_fwd_varlen(q, k, v, cq, ck, 0.5)
    assert np.isnan(o[-2:]).all() and np.isnan(lse[:, -2:]).all()
    assert not np.isnan(o[:-2]).any()


# ------------------------------------------------------------ grouped-query heads and cache append

@pytest.mark.parametrize("H,H_kv", [(4, 2), (6, 3), (4, 1), (3, 3)])
def test_gqa_query_head_reads_kv_head_h_over_group(H, H_kv):
    # V of K/V head j is the constant j: every output of query head h is
    # exactly its K/V head index, whatever the attention weights
    B, Nq, Nk, d = 2, 5, 7, 4
    q, k = rnd((B, Nq, H, d), 51), rnd((B, Nk, H_kv, d), 52)
    v = np.broadcast_to(np.arange(H_kv, dtype=np.float64)[None, None, :, None], (B, Nk, H_kv, d)).copy()
    o, lse = oracle.attn_fwd_gqa(q, k, v, 0.7, causal=True)
    for h in range(H):
        np.testing.assert_allclose(o[:, :, h], h // (H // H_kv), rtol=0, atol=1e-12)
    # and the scores of head h are those of K head h // group: same LSE as
    # plain attention against that head
    for h in range(H):
        _, l1 = oracle.attn_fwd(q[:, :, h:h + 1], k[:, :, h // (H // H_kv):h // (H // H_kv) + 1], v[:, :, :1], 0.7,
                                causal=True)
        np.testing.assert_allclose(lse[:, h], l1[:, 0], rtol=0, atol=1e-12)


def test_gqa_decode_reads_cache_head_h_over_group():
    H, H_kv, d, page, mb = 6, 2, 4, 4, 3
    q, w_k, w_v, table, lens = decode_case(61, B=2, H=H, d=d, page=page, max_blocks=mb, lens=(9, 5))
    kc = rnd((2 * mb, page, H_kv, d), 62)
    vc = np.broadcast_to(np.arange(H_kv, dtype=np.float64)[None, None, :, None], kc.shape).copy()
    o, lse = oracle.attn_decode_paged_gqa(q, kc, vc, table, lens, 0.5)
    for h in range(H):
        np.testing.assert_allclose(o[:, 0, h], h // (H // H_kv), rtol=0, atol=1e-12)


def test_append_writes_tokens_where_the_table_says():
    B, n_new, H, d, page, mb = 3, 5, 2, 4, 4, 4
    rng = np.random.default_rng(71)
    table = rng.permutation(B * mb).reshape(B, mb).astype(np.int32)
    lens = np.array([0, 6, 13], dtype=np.int32)     # the last one runs past the table (16 slots)
    kc = rng.standard_normal((B * mb, page, H, d))
    vc = rng.standard_normal((B * mb, page, H, d))
    kn = rng.standard_normal((B, n_new, H, d))
    vn = rng.standard_normal((B, n_new, H, d))
    k2, v2 = oracle.kvcache_append(kn, vn, kc, vc, table, lens)
    for b in range(B):
        for t in range(mb * page):
            pg, row = table[b, t // page], t % page
            i = t - lens[b]
            if 0 <= i < n_new:
                assert np.array_equal(k2[pg, row], kn[b, i]) and np.array_equal(v2[pg, row], vn[b, i])
            else:
                assert np.array_equal(k2[pg, row], kc[pg, row]) and np.array_equal(v2[pg, row], vc[pg, row])


def test_qkvpacked_slots_are_q_k_v():
    # distinct q, k, v packed along axis 2 must give exactly the separate
    # call; swapping any two slots changes the result
    B, N, H, d = 2, 6, 2, 4
    q, k, v = rnd((B, N, H, d), 81), rnd((B, N, H, d), 82), rnd((B, N, H, d), 83)
    o, lse = oracle.attn_fwd(q, k, v, 0.5, causal=True)
    op, lp = oracle.attn_fwd_qkvpacked(np.stack([q, k, v], axis=2), 0.5, causal=True)
    assert np.array_equal(o, op) and np.array_equal(lse, lp)
    ow, _ = oracle.attn_fwd_qkvpacked(np.stack([k, q, v], axis=2), 0.5, causal=True)
    assert not np.allclose(ow, o)


# ---------------------------------------------------------------- backward

def _loss(q, k, v, dout, scale, **opts):
    o, _ = oracle.attn_fwd_gqa(q, k, v, scale, **opts)
    return float(np.sum(dout * o))


def _finite_difference(x, f, eps=1e-6):
    g = np.zeros_like(x)
    for idx in np.ndindex(x.shape):
        old = x[idx]
        x[idx] = old + eps
        fp = f()
        x[idx] = old - eps
        fm = f()
        x[idx] = old
        g[idx] = (fp - fm) / (2 * eps)
    return g


@pytest.mark.parametrize("H_kv", [2, 1])
@pytest.mark.parametrize("opts", [
    {},
    {"causal": True},
    {"causal": True, "window_left": 2, "window_right": 0},
    {"window_left": 1, "window_right": 2},
    {"causal": True, "alibi_slopes": [0.5, 0.125], "softcap": 1.5},
    {"alibi_slopes": [0.25, 1.0], "softcap": 0.7},
], ids=lambda o: "-".join(sorted(o)) or "plain")
def test_bwd_matches_finite_differences_of_the_forward(opts, H_kv):
    """Each gradient entry against a central difference of L = sum(dout * O)
    taken through the forward oracle alone (fp64 inputs): a wrong sign, a
    transposed product, a dropped softmax-Jacobian term, a missing softcap
    factor or a group sum over the wrong heads all fail here."""
    B, H, Nq, Nk, d, scale = 1, 2, 5, 7, 4, 0.7
    q, k, v = rnd((B, Nq, H, d), 61), rnd((B, Nk, H_kv, d), 62), rnd((B, Nk, H_kv, d), 63)
    dout = rnd((B, Nq, H, d), 64)
    dq, dk, dv = oracle.attn_bwd(q, k, v, dout, scale, **opts)
    f = lambda: _loss(q, k, v, dout, scale, **opts)
    for got, x, name in ((dq, q, "dq"), (dk, k, "dk"), (dv, v, "dv")):
        want = _finite_difference(x, f)
        assert np.abs(got - want).max() < 1e-7, name


def test_bwd_single_key_closed_form():
    """One key: every row's softmax is the constant 1, so O_i = v_0 whatever
    q and k are: dq = dk = 0 and dv = sum_i dout_i."""
    B, H, Nq, d = 2, 3, 6, 5
    q, k, v = rnd((B, Nq, H, d), 71), rnd((B, 1, H, d), 72), rnd((B, 1, H, d), 73)
    dout = rnd((B, Nq, H, d), 74)
    dq, dk, dv = oracle.attn_bwd(q, k, v, dout, 0.9)
    assert np.abs(dq).max() < TOL and np.abs(dk).max() < TOL
    assert np.abs(dv[:, 0] - dout.sum(axis=1)).max() < 1e-12


def test_bwd_zero_query_closed_form():
    """q = 0 and no mask: P is uniform 1/Nk. Then dv_j = mean-free sum of
    dout over rows / Nk, dk = 0 (it is scale * dS^T q), and dq_i = (scale/Nk)
    sum_j (dout_i . v_j - mean_k dout_i . v_k) k_j."""
    B, H, Nq, Nk, d, scale = 1, 2, 4, 6, 3, 0.8
    q = np.zeros((B, Nq, H, d))
    k, v, dout = rnd((B, Nk, H, d), 81), rnd((B, Nk, H, d), 82), rnd((B, Nq, H, d), 83)
    dq, dk, dv = oracle.attn_bwd(q, k, v, dout, scale)
    assert np.abs(dk).max() < TOL
    for h in range(H):
        assert np.abs(dv[0, :, h] - dout[0, :, h].sum(axis=0) / Nk).max() < 1e-12
        a = dout[0, :, h] @ v[0, :, h].T                       # [Nq, Nk]
        want = scale / Nk * ((a - a.mean(axis=1, keepdims=True)) @ k[0, :, h])
        assert np.abs(dq[0, :, h] - want).max() < 1e-12


def test_bwd_rows_without_keys_carry_no_gradient():
    """Causal with Nq > Nk: the first Nq - Nk rows see no key; their dq is 0
    and they add nothing to dk, dv."""
    B, H, Nq, Nk, d = 1, 1, 6, 3, 4
    q, k, v, dout = rnd((B, Nq, H, d), 91), rnd((B, Nk, H, d), 92), rnd((B, Nk, H, d), 93), rnd((B, Nq, H, d), 94)
    dq, dk, dv = oracle.attn_bwd(q, k, v, dout, 0.5, causal=True)
    assert np.all(dq[:, :Nq - Nk] == 0.0)
    dout2 = dout.copy()
    dout2[:, :Nq - Nk] = 123.0
    _, dk2, dv2 = oracle.attn_bwd(q, k, v, dout2, 0.5, causal=True)
    assert np.abs(dk2 - dk).max() < TOL and np.abs(dv2 - dv).max() < TOL


# ---------------------------------------------------------------- 8-bit inputs

@pytest.mark.parametrize("code,tdtype", [(oracle.E4M3, torch.float8_e4m3fn), (oracle.E5M2, torch.float8_e5m2)],
                         ids=["e4m3", "e5m2"])
def test_widen_fp8_every_bit_pattern(code, tdtype):
    """Every 8-bit pattern against torch's own float8 conversion (an
    independent implementation of the same formats)."""
    bits = np.arange(256, dtype=np.uint8)
    got = oracle.widen(bits, code)
    want = torch.from_numpy(bits).view(tdtype).to(torch.float64).numpy()
    assert np.array_equal(got, want, equal_nan=True)


@pytest.mark.parametrize("tdtype", [torch.float8_e4m3fn, torch.float8_e5m2], ids=["e4m3", "e5m2"])
@pytest.mark.parametrize("opts", [dict(causal=True), dict(causal=False, window_left=3, window_right=1),
                                  dict(causal=True, alibi_slopes=[0.25, 0.5], softcap=2.0)])
def test_fp8_attention_is_attention_of_the_dequantised_inputs(tdtype, opts):
    B, H, Nq, Nk, d = 1, 2, 6, 9, 16
    g = torch.Generator().manual_seed(41)
    q8, k8, v8 = (torch.randn(B, n, H, d, generator=g).mul(8.0).to(tdtype) for n in (Nq, Nk, Nk))
    dq, dk, dv, scale = 0.02, 0.05, 0.3, 0.25
    o, lse = oracle.attn_fwd_fp8(q8, k8, v8, scale, dq, dk, dv, **opts)
    deq = lambda t, s: t.to(torch.float64).numpy() * s
    o_ref, l_ref = oracle.attn_fwd(deq(q8, dq), deq(k8, dk), deq(v8, dv), scale, **opts)
    assert np.abs(o - o_ref).max() < 1e-12 and np.abs(lse - l_ref).max() < 1e-12


def test_fp8_oracle_rejects_mixed_storage():
    x = torch.zeros(1, 2, 1, 16).to(torch.float8_e4m3fn)
    with pytest.raises(ValueError):
        oracle.attn_fwd_fp8(x, x.to(torch.float32).to(torch.float8_e5m2), x, 0.1)
