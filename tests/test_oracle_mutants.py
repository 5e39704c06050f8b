"""Planted mistakes: each plausible slip in the oracle must fail a pin.

Every case below copies attn_oracle.c, plants one mistake by replacing one
exact snippet, compiles the copy with gcc and reruns a battery of pin checks
from test_oracle_pins against it. The unmodified source must pass the whole
battery and every mutant must fail at least one check. Mistakes are planted
in the oracle only, on the CPU.
"""
import os
import subprocess
import tempfile

import numpy as np
import pytest

import oracle
from oracle import build as obuild
from tests import test_oracle_pins as pins

MUTANTS = {
    "dropped_scale": ("double sj = r->scale * dot;", "double sj = dot;"),
    "alibi_sign": ("sj += -r->slope * fabs", "sj += r->slope * fabs"),
    "top_left_causal": (".pos = i + delta,", ".pos = i,"),
    "causal_off_by_one": ("if (causal && j > pos)", "if (causal && j >= pos)"),
    "window_off_by_one": ("if (wl >= 0 && j < pos - wl)", "if (wl >= 0 && j <= pos - wl)"),
    "softcap_before_scale": ("sj = r->softcap * tanh(sj / r->softcap);",
                             "sj = r->scale * r->softcap * tanh(dot / r->softcap);"),
    "lse_without_max": ("*lse = m + log(sum);", "*lse = log(sum);"),
    "no_normalisation": ("e[j] /= sum;", "e[j] /= 1.0;"),
    "v_used_as_k": ("load_elem(r->k, r->k_off[j] + c, r->dtype)", "load_elem(r->v, r->v_off[j] + c, r->dtype)"),
    "wrong_page_row": ("long pg = block_table[(long)b * max_blocks + t / page_size];",
                       "long pg = block_table[(long)((b + 1) % B) * max_blocks + t / page_size];"),
    "merge_weight": ("double w = exp(lse_part[(long)sp * n + r] - total);",
                     "double w = exp(lse_part[(long)sp * n + r] - m);"),
    "split_drops_a_key": ("long b = a + chunk;", "long b = a + chunk - 1;"),
    "fp16_exponent_bias": ("mag = ldexp((double)(1024 + frac), expo - 25);",
                           "mag = ldexp((double)(1024 + frac), expo - 24);"),
    "e4m3_exponent_bias": ("mag = ldexp((double)(8 + frac), expo - 10);",
                           "mag = ldexp((double)(8 + frac), expo - 9);"),
    "e5m2_subnormal_scale": ("mag = ldexp((double)frac, -16);", "mag = ldexp((double)frac, -15);"),
}


def battery():
    """Pin checks run against a (possibly broken) oracle build."""
    yield lambda: pins.test_widen_fp16_every_bit_pattern()
    yield lambda: pins.test_widen_bf16_every_bit_pattern()
    for mask in pins.MASKS:
        yield lambda mask=mask: pins.test_probability_rows_sum_to_one(5, 11, mask)
    yield lambda: pins.test_single_key_returns_v()
    yield lambda: pins.test_zero_query_gives_column_mean_and_ln_n(6)
    yield lambda: pins.test_joint_permutation_of_keys_and_values()
    for opts in [dict(causal=True), dict(causal=True, wl=2, wr=0), dict(causal=False, wl=1, wr=2),
                 dict(causal=True, slopes=[0.7, 0.05]), dict(causal=False, softcap=1.5)]:
        yield lambda opts=opts: pins.test_matches_brute_force_with_bottom_right_alignment(4, 9, opts)
    yield lambda: pins.test_zero_query_counts_visible_keys(6, 20, True, 4, 0)
    yield lambda: pins.test_one_hot_probe_pins_each_key(3, 8)
    yield lambda: pins.test_alibi_is_a_geometric_series(0.5)
    yield lambda: pins.test_softcap_two_key_closed_form(2.0)
    yield lambda: pins.test_permuted_block_table_is_a_reindexing({})
    yield lambda: pins.test_any_split_count_matches_one_split(3, {})
    yield lambda: pins.test_half_precision_storage_is_widened_exactly()
    yield lambda: pins.test_widen_fp8_every_bit_pattern(oracle.E4M3, pins.torch.float8_e4m3fn)
    yield lambda: pins.test_widen_fp8_every_bit_pattern(oracle.E5M2, pins.torch.float8_e5m2)


def run_battery():
    failures = 0
    for check in battery():
        try:
            check()
        except (AssertionError, ValueError):
            failures += 1
    return failures


def compile_variant(src_text, workdir, name):
    src = os.path.join(workdir, name + ".c")
    lib = os.path.join(workdir, "lib" + name + ".so")
    with open(src, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", lib, src, "-lm"],
                   check=True)
    return lib


@pytest.fixture(scope="module")
def source():
    with open(obuild.SRC) as f:
        text = f.read()
    yield text
    oracle.load_library()  # rebind the real oracle for the tests that follow


def test_unmodified_oracle_passes_battery(source):
    with tempfile.TemporaryDirectory() as wd:
        oracle.load_library(compile_variant(source, wd, "clean"))
        assert run_battery() == 0


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(source, name):
    old, new = MUTANTS[name]
    assert source.count(old) == 1, "snippet for %s not found exactly once" % name
    with tempfile.TemporaryDirectory() as wd:
        oracle.load_library(compile_variant(source.replace(old, new), wd, name))
        with np.errstate(all="ignore"):
            caught = run_battery()
    oracle.load_library()
    assert caught > 0, "mutant %s passed every pin" % name


# ---------------------------------------------------------------- backward

BWD_MUTANTS = {
    "softmax_jacobian_dropped": ("dz = p * (dp - np.sum(p * dp, axis=1, keepdims=True))", "dz = p * dp"),
    "softcap_factor_dropped": ("dz = dz * (1.0 - t * t)", "dz = dz"),
    "dk_from_dout": ("dk[b, :, h] = scale * (dz.T @ qh)", "dk[b, :, h] = scale * (dz.T @ doh)"),
    "dq_missing_scale": ("dq[b, :, h] = scale * (dz @ kh)", "dq[b, :, h] = dz @ kh"),
    "dp_with_k": ("dp = doh @ vh.T", "dp = doh @ kh.T"),
    "dv_not_transposed": ("dv[b, :, h] = p.T @ doh", "dv[b, :, h] = (p @ doh.T[:, : p.shape[1]].T)"),
    "group_sum_wrong_order": ("dk = dk.reshape(B, Nk, H_kv, G, d).sum(axis=3)",
                              "dk = dk.reshape(B, Nk, G, H_kv, d).sum(axis=2)"),
}


def _grouped_finite_difference_check():
    """Finite differences with four query heads over two K/V heads (groups
    of two), so a group sum over the wrong heads shows."""
    B, H, H_kv, Nq, Nk, d, scale = 1, 4, 2, 4, 5, 3, 0.6
    q, k, v = pins.rnd((B, Nq, H, d), 101), pins.rnd((B, Nk, H_kv, d), 102), pins.rnd((B, Nk, H_kv, d), 103)
    dout = pins.rnd((B, Nq, H, d), 104)
    dq, dk, dv = oracle.attn_bwd(q, k, v, dout, scale, causal=True)
    f = lambda: pins._loss(q, k, v, dout, scale, causal=True)
    for got, x in ((dq, q), (dk, k), (dv, v)):
        assert np.abs(got - pins._finite_difference(x, f)).max() < 1e-7


def bwd_battery():
    for opts in ({}, {"causal": True, "window_left": 2, "window_right": 0},
                 {"causal": True, "alibi_slopes": [0.5, 0.125], "softcap": 1.5}):
        for H_kv in (2, 1):
            yield lambda opts=opts, H_kv=H_kv: pins.test_bwd_matches_finite_differences_of_the_forward(opts, H_kv)
    yield pins.test_bwd_single_key_closed_form
    yield pins.test_bwd_zero_query_closed_form
    yield pins.test_bwd_rows_without_keys_carry_no_gradient
    yield _grouped_finite_difference_check


def _bwd_mutant(snippet, replacement):
    import inspect
    src = inspect.getsource(oracle.attn_bwd)
    assert src.count(snippet) == 1, snippet
    ns = dict(vars(oracle))
    exec(compile(src.replace(snippet, replacement), "<mutant>", "exec"), ns)
    return ns["attn_bwd"]


def _bwd_failures(fn, monkeypatch):
    monkeypatch.setattr(oracle, "attn_bwd", fn)
    failed = 0
    for check in bwd_battery():
        try:
            check()
        except Exception:
            failed += 1
    return failed


def test_unmodified_backward_oracle_passes_the_battery(monkeypatch):
    assert _bwd_failures(oracle.attn_bwd, monkeypatch) == 0


@pytest.mark.parametrize("name", sorted(BWD_MUTANTS))
def test_each_backward_mutant_fails_a_pin(name, monkeypatch):
    snippet, replacement = BWD_MUTANTS[name]
    assert _bwd_failures(_bwd_mutant(snippet, replacement), monkeypatch) > 0, name
