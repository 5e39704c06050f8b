"""The pages' worked examples (tests/golden/pages_examples.txt) against the oracle."""
import math
import os

import numpy as np
import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def examples(kind):
    out = []
    with open(os.path.join(HERE, "golden", "pages_examples.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            name, *fields = line.split()
            if name == kind:
                out.append({k: int(v) for k, v in (x.split("=") for x in fields)})
    assert out, kind
    return out


@pytest.mark.parametrize("ex", examples("decode_alignment"), ids=lambda e: "N%d" % e["N"])
def test_decode_query_attends_to_all_keys(ex):
    """Causal attention of 1 query over N+1 keys: with Q = 0 every visible key
    scores 0, so LSE = ln(number of visible keys)."""
    N, H, d = ex["N"], 1, 4
    q = np.zeros((1, 1, H, d))
    k = np.random.default_rng(N).standard_normal((1, N + 1, H, d))
    v = np.random.default_rng(N + 1).standard_normal((1, N + 1, H, d))
    o, lse = oracle.attn_fwd(q, k, v, 1.0, causal=True)
    assert abs(lse[0, 0, 0] - math.log(ex["visible"])) < 1e-12
    assert np.allclose(o[0, 0, 0], v[0, :, 0].mean(axis=0), atol=1e-12)


@pytest.mark.parametrize("ex", examples("split_kv_halves"))
def test_split_kv_halves_merge_to_the_whole(ex):
    L, S, size = ex["keys"], ex["splits"], ex["split_size"]
    H, d, page = 1, 4, 250
    g = np.random.default_rng(7)
    nblk = L // page
    kc = g.standard_normal((nblk, page, H, d))
    vc = g.standard_normal((nblk, page, H, d))
    table = np.arange(nblk, dtype=np.int32)[None]
    lens = np.array([L], dtype=np.int32)
    # with Q = 0 each partial's LSE is ln(its key count): both halves hold 1000
    q0 = np.zeros((1, 1, H, d))
    _, lp = oracle.attn_decode_paged(q0, kc, vc, table, lens, 1.0, num_splits=S)
    assert np.allclose(lp[:, 0, 0], math.log(size), atol=1e-12)
    q = g.standard_normal((1, 1, H, d))
    o1, l1 = oracle.attn_decode_paged(q, kc, vc, table, lens, 0.5)
    op, lp = oracle.attn_decode_paged(q, kc, vc, table, lens, 0.5, num_splits=S)
    o, lse = oracle.combine_splits(op, lp)
    assert np.allclose(o, o1[:, 0], atol=1e-12) and np.allclose(lse, l1[:, :, 0], atol=1e-12)
