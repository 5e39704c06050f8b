"""The algorithmic work bench.py credits (CPU): visible query/key pairs of
the forward workloads against closed forms and against the oracle's own
probabilities (a pair is visible exactly when its probability is nonzero
for a query that sees any key), and the decode byte count."""
import numpy as np
import pytest
import torch

import bench
import oracle
from exact_io_aware_79_b200 import workloads as W


def test_causal_square_counts_the_lower_triangle():
    w = W.CAUSAL_2K
    assert bench.unmasked_pairs(w) == w.Nq * (w.Nq + 1) // 2
    assert bench.fwd_flops(w) == 4.0 * w.d * w.B * w.H * w.Nq * (w.Nq + 1) // 2


def test_window_16k_closed_form():
    w = W.WINDOW_16K                     # causal, window_left 4096: row i sees min(i, 4096) + 1 keys
    wl = w.window_left
    assert bench.unmasked_pairs(w) == (wl + 1) * (wl + 2) // 2 - (wl + 1) + (w.Nq - wl) * (wl + 1)


def test_rectangular_causal_is_bottom_right():
    w = W.CAUSAL_Q4K_K16K                # query i sees keys 0 .. i + Nk - Nq
    off = w.Nk - w.Nq
    assert bench.unmasked_pairs(w) == sum(i + off + 1 for i in range(w.Nq))


@pytest.mark.parametrize("opts", [dict(causal=True), dict(causal=True, window_left=3, window_right=0),
                                  dict(causal=False, window_left=2, window_right=1), dict(causal=False)])
@pytest.mark.parametrize("Nq,Nk", [(7, 7), (5, 11), (9, 4)])
def test_pair_count_matches_the_oracle_probabilities(Nq, Nk, opts):
    w = W.FwdWorkload("t", 1, 1, Nq, Nk, 8, torch.float16, **opts)
    g = np.random.default_rng(Nq * 100 + Nk)
    q, k, v = (g.standard_normal((1, n, 1, 8)) * 0.1 for n in (Nq, Nk, Nk))
    _, _, p = oracle.attn_fwd(q, k, v, 0.5, opts.get("causal", False), opts.get("window_left", -1),
                              opts.get("window_right", -1), return_probs=True)
    assert bench.unmasked_pairs(w) == int(np.count_nonzero(p))


def test_varlen_causal_pairs():
    lens = [1, 5, 128]
    assert bench.varlen_flops(W.VARLEN, lens) == 4.0 * W.VARLEN.d * W.VARLEN.H * (1 + 15 + 128 * 129 // 2)


def test_decode_bytes_are_k_and_v_of_every_cached_token():
    w = W.DECODE_GQA
    L = torch.tensor([100, 2000, 1], dtype=torch.int32)
    assert bench.decode_kv_bytes(w, L) == 2 * 2 * w.kv_heads * w.d * 2101
    ww = W.DecodeWorkload("w", 3, 8, 64, torch.bfloat16, 256, 1, 10, window_left=99)
    assert bench.decode_kv_bytes(ww, L) == 2 * 2 * 8 * 64 * (100 + 100 + 1)   # each row sees at most 100 keys
