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
