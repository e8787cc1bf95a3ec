"""Plant plausible mistakes in copies of the C oracle and check that the pins
of tests/test_oracle.py catch every one of them.

Each mutant is the oracle source with one textual change, compiled into a
temporary library that is swapped in for the duration of the check. CPU
only; the committed oracle is never modified.
"""
import os
import subprocess

import pytest

import oracle
import tests.test_oracle as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "hils_oracle.c")

BIAS = "(double)p->bias[((int64_t)b * p->Hkv + g) * p->nC + c];"
MUTANTS = {
    "drop_bias": (BIAS, "0.0 * " + BIAS),
    "bias_scaled_by_sqrt_d": (BIAS, BIAS[:-1] + " / sqrt((double)p->d);"),
    "window_off_by_one": ("floordiv(i - p->W + 1, S)", "floordiv(i - p->W, S)"),
    "no_head_normalisation": ("double v = shat[hh * nc + c] - lse[hh];",
                              "double v = shat[hh * nc + c];"),
    "sum_over_heads": ("if (v > a) a = v;",
                       "a = (a == -INFINITY ? 0.0 : a) + exp(v);"),
    "ties_to_higher_index": ("return (u->c < v->c) ? -1 : (u->c > v->c);",
                             "return (u->c > v->c) ? -1 : (u->c < v->c);"),
    "window_mass_left_out": ("terms[nsel] = log_zswa;",
                             "terms[nsel] = -INFINITY;"),
    "no_intra_chunk_normalisation": (
        "e[t] = e[t] - log_zc + shat[hh * nc + c] - log_zhat;",
        "e[t] = e[t] + shat[hh * nc + c] - log_zhat;"),
    "logit_scale_1_over_d": ("return acc / sqrt((double)p->d);\n}",
                             "return acc / (double)p->d;\n}"),
    "value_row_shifted": ("p->kv_rows + tj[t]) * d;",
                          "p->kv_rows + (tj[t] > 0 ? tj[t] - 1 : 0)) * d;"),
    "scoring_ignores_qcal_query": ("const void *qb = p->Qs ? p->Qs : p->Q;",
                                   "const void *qb = p->Q;"),
    "one_chunk_short": ("int nsel = (int)(nc < K ? nc : K);",
                        "int nsel = (int)(nc < K ? nc : K - (K > 1));"),
    "gap_wrong_pair": ("cs[K - 1].a - cs[K].a", "cs[0].a - cs[K].a"),
}

PIN_TESTS = [
    lambda: pins.test_golden_toy_window_chunks(),
    lambda: pins.test_golden_gqa_group_rule(),
    *[(lambda c=c: pins.test_brute_matches_oracle(c)) for c in pins.CASES],
    lambda: pins.test_exact_scores_equal_naive_bsa([0, 1, 0, 1]),
    lambda: pins.test_reduces_to_full_causal("exact_scores"),
    lambda: pins.test_reduces_to_full_causal("exact_structure"),
    lambda: pins.test_constant_values_give_constant_output(),
    lambda: pins.test_tie_rule_lower_index(),
    lambda: pins.test_planted_bias_forces_selection(),
]


def _compile(src_text, out):
    c = out + ".c"
    with open(c, "w") as f:
        f.write(src_text)
    subprocess.run(["gcc", "-O1", "-std=c11", "-fopenmp", "-fPIC", "-shared",
                    c, "-o", out, "-lm"], check=True)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(old) >= 1, f"mutation anchor for {name} not found"
    lib_path = str(tmp_path / f"mut_{name}.so")
    _compile(text.replace(old, new, 1), lib_path)
    saved = oracle._load()
    oracle._lib = oracle.load_library(lib_path)
    caught = []
    try:
        for k, t in enumerate(PIN_TESTS):
            try:
                t()
            except (AssertionError, RuntimeError):
                caught.append(k)
    finally:
        oracle._lib = saved
    assert caught, f"no pin caught the planted mistake {name!r}"
