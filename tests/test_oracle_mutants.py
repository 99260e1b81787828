"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a copy of ``oracle/attn_oracle.c`` (a dropped term, a
wrong sign, a wrong index or a transposed operand), builds it on the CPU, and runs the
battery of pins from ``test_oracle`` against it.  Every mutant must fail at least one.
"""
import os
import subprocess

import pytest

import oracle
from tests import test_oracle as pins
from tests import test_oracle_decode as dpins
from tests import test_oracle_fp8 as fpins

SRC = os.path.join(os.path.dirname(oracle.__file__), "attn_oracle.c")

MUTANTS = {
    "scale dropped from the scores": ("s[j] = P->scale * acc;", "s[j] = acc;"),
    "causal mask off by one": ("return causal ? i + 1 : n;", "return causal ? i + 2 : n;"),
    "GQA head mapping interleaved": ("const int g = (int)(((int64_t)h * P->hkv) / P->hq);\n    const double *qi = P->q + (row",
                                     "const int g = h % P->hkv;\n    const double *qi = P->q + (row"),
    "max dropped from LSE": ("return m + log(l);", "return log(l);"),
    "softmax not normalised": ("p[j] /= l;", "p[j] /= 1.0;"),
    "wrong sign in dS": ("ds[j] = p[j] * (dp - Di);", "ds[j] = p[j] * (dp + Di);"),
    "D from the wrong vector": ("acc += doi[c] * oi[c];", "acc += doi[c] * doi[c];"),
    "dK missing the scale": ("dkj[c] = P->scale * acck", "dkj[c] = acck"),
    "dV with Q in place of dO": ("av[c] += p[j] * doi[c];", "av[c] += p[j] * qi[c];"),
    "dQ with V in place of K": ("const double *kj = P->k + ((t0 + j) * P->hkv + g) * d;\n            for (int c = 0; c < d; ++c) dqi[c]",
                                "const double *kj = P->v + ((t0 + j) * P->hkv + g) * d;\n            for (int c = 0; c < d; ++c) dqi[c]"),
    "given LSE ignored": ("if (lse_in) lse[(int64_t)h * T + t] = lse_in[(int64_t)h * T + t];",
                          "if (lse_in) lse[(int64_t)h * T + t] = lse[(int64_t)h * T + t];"),
    "given O ignored for D": ("dd[(int64_t)h * T + t] = dsum;", "(void)dsum;"),
    "score mask boundary off by one": ("if (j >= vis) { s[j] = -INFINITY; continue; }", "if (j > vis) { s[j] = -INFINITY; continue; }"),
    "fp8 row sum from the rounded weights": ("                    l += pj;\n",
                                            "                    l += W->round_p ? oracle_round_e4m3(pj) : pj;\n"),
    "fp8 weights not rounded": ("const double pv = W->round_p ? oracle_round_e4m3(pj) : pj;", "const double pv = pj;"),
    "decode causal mask aligned top-left": ("const int v = lk - lq + i + 1;", "const int v = i + 1;"),
    "decode LSE stored to the sequence's first row": ("P->lse[(int64_t)h * W->tq + row] = lse;",
                                                      "P->lse[(int64_t)h * W->tq + q0] = lse;"),
    "decode keys addressed by the query offsets": ("score_row(P, row, k0, lk, vis, h, s);",
                                                   "score_row(P, row, q0, lk, vis, h, s);"),
    "value row from the wrong key": ("const double *vj = P->v + ((key0 + j) * P->hkv + g) * d;\n        for (int c = 0; c < d; ++c) oi[c]",
                                     "const double *vj = P->v + ((key0 + (n - 1 - j)) * P->hkv + g) * d;\n        for (int c = 0; c < d; ++c) oi[c]"),
}


def _battery():
    """True when every pin passes."""
    checks = [
        lambda: pins.test_forward_matches_brute_force([3, 7, 1], 4, 2, 2, True),
        lambda: pins.test_forward_matches_brute_force([8], 2, 2, 4, False),
        lambda: pins.test_matches_torch_sdpa_and_autograd(20, 6, 3, 5, True),
        lambda: pins.test_matches_torch_sdpa_and_autograd(9, 2, 2, 8, False),
        lambda: pins.test_gradients_match_finite_differences(True),
        lambda: pins.test_worked_example_online_merge(),
        lambda: pins.test_zero_queries_give_uniform_average(True),
        lambda: pins.test_gradient_invariants(False),
        lambda: pins.test_given_lse_shift_scales_gradients_exactly(),
        lambda: pins.test_given_o_changes_dq_by_closed_form(),
        lambda: dpins.test_cross_matches_brute_force(([1, 3], [2, 6]), True),
        lambda: dpins.test_cross_matches_brute_force(([2, 3], [7, 3]), False),
        lambda: dpins.test_cross_zero_queries_average_the_visible_values(),
        lambda: fpins.test_two_key_example_rounds_the_weights_but_not_the_sum(),
        lambda: fpins.test_unrounded_steps_equal_the_exact_forward(True, 30.0),
        lambda: fpins.test_rounded_weights_leave_the_lse_exact(True),
    ]
    for c in checks:
        try:
            c()
        except AssertionError:
            return False
    return True


def test_unmutated_oracle_passes_battery():
    assert _battery()


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name!r} not found exactly once"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
                           "-o", str(lib), str(mutated), "-lm"])
    with oracle.using_library(str(lib)):
        assert not _battery(), f"mutant {name!r} passed every pin"
