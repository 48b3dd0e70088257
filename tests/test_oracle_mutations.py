"""Planted mistakes in the oracle must be caught by the pins.

Each case rewrites one line of a private copy of the oracle's C source (a
dropped term, a wrong sign, an off-by-one index, a transposed stride), builds
it on the CPU into a temporary library, routes the oracle through it and
checks that at least one pin of `test_oracle_pins` fails.
"""
import os
import subprocess

import pytest

import oracle
import test_oracle_pins as pins
import test_rounding_bound as rb

SRC = os.path.join(os.path.dirname(oracle.__file__), "condensate_oracle.c")

MUTATIONS = {
    "order_sign": ("if (a->t > b->t) return -1;", "if (a->t < b->t) return -1;"),
    "tie_to_higher_index": ("if (a->j < b->j) return -1;\n  if (a->j > b->j) return 1;",
                            "if (a->j < b->j) return 1;\n  if (a->j > b->j) return -1;"),
    "candidate_overlaps_window": ("int64_t hi = i - W; /* last candidate position */",
                                  "int64_t hi = i - W + 1;"),
    "window_one_short": ("  int64_t lo = i - W + 1;\n  if (lo < 0) lo = 0;\n  int64_t n = 0;",
                         "  int64_t lo = i - W + 2;\n  if (lo < 0) lo = 0;\n  int64_t n = 0;"),
    "anchor_dropped": ("if (lo > 0) C[n++] = 0;", "if (lo > 0 && 0) C[n++] = 0;"),
    "scale_dropped": ("void oracle_attend(const double* t, const float* V, int d, const int64_t* C,\n"
                      "                   int64_t nC, double* o) {\n  double scale = 1.0 / sqrt((double)d);",
                      "void oracle_attend(const double* t, const float* V, int d, const int64_t* C,\n"
                      "                   int64_t nC, double* o) {\n  double scale = 1.0;"),
    "softmax_sign": ("double w = exp(t[C[r]] * scale - mx);", "double w = exp(mx - t[C[r]] * scale);"),
    "key_stride_transposed": ("const float* kj = K + j * (int64_t)d;\n    double acc",
                              "const float* kj = K + j;\n    double acc"),
    "value_row_index": ("const float* vj = V + C[r] * (int64_t)d;",
                        "const float* vj = V + r * (int64_t)d;"),
    "normalisation_dropped": ("for (int l = 0; l < d; ++l) o[l] /= den;", ""),
    "all_candidates_one_short": ("int64_t m = k < ncand ? k : ncand;",
                                 "int64_t m = k < ncand ? k : ncand - 1;"),
    "bound_unit_roundoff_too_small": ("double u = ldexp(1.0, -23);",
                                      "double u = ldexp(1.0, -30);"),
    "bound_unselected_term_dropped": ("diag[DG_BOUND] = gam * (amax_sel + amax_unsel);",
                                      "diag[DG_BOUND] = gam * amax_sel;"),
    "bound_ten_times_too_large": ("diag[DG_BOUND] = gam * (amax_sel + amax_unsel);",
                                  "diag[DG_BOUND] = 10.0 * gam * (amax_sel + amax_unsel);"),
    "lse_max_dropped": ("if (diag) diag[DG_LSE] = mx + log(den);",
                        "if (diag) diag[DG_LSE] = log(den);"),
    "score_term_dropped": ("for (int l = 0; l < d; ++l) acc += (double)q[l] * (double)kj[l];",
                           "for (int l = 1; l < d; ++l) acc += (double)q[l] * (double)kj[l];"),
}

PIN_TESTS = [
    lambda: [pins.test_topk_matches_brute_force_enumeration(W, k)
             for W in (1, 2, 3) for k in (0, 2, 4)],
    pins.test_set_size_finite_support,
    lambda: [pins.test_equals_full_attention_when_set_covers_all(W, k)
             for W, k in [(1, 10_000), (10_000, 0)]],
    pins.test_two_term_closed_form,
    pins.test_uniform_scores_closed_forms,
    pins.test_planted_needles_are_selected,
    pins.test_lemma_excluded_scores_below_threshold,
    lambda: [rb.test_oracle_bound_covers_every_order(d, adv)
             for d in (64, 128) for adv in (False, True)],
    rb.test_oracle_bound_on_workload_rows,
]


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, name
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                    "-o", str(so), str(mutated), "-lm"], check=True)
    caught = []
    with oracle.using_library(str(so)):
        for t in PIN_TESTS:
            try:
                t()
            except (AssertionError, ValueError):
                caught.append(t)
    assert caught, f"mutation {name} escaped every pin"
