"""Plant plausible mistakes in a copy of the oracle and check the pins catch each.

Each mutant is a one-line textual edit of dla_oracle.c compiled into a
temporary library (CPU only); the pins of test_oracle_pins must reject it.
"""
import os
import subprocess
import tempfile

import pytest

from oracle import oracle as O
from tests import test_oracle_info as info_pins
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(O.__file__), "dla_oracle.c")

MUTANTS = {
    "ward_factor_dropped": ("double f = (na * nb) / (na + nb);", "double f = 1.0;"),
    "ward_on_sums_not_means": ("double diff = a->z[i] / na - b->z[i] / nb;",
                               "double diff = a->z[i] - b->z[i];"),
    "single_score_boundary": ("int join = hd->t > 0 && rt < J->tau && hd->prev_r < J->tau;",
                              "int join = hd->t > 0 && rt < J->tau;"),
    "non_strict_threshold": ("int join = hd->t > 0 && rt < J->tau && hd->prev_r < J->tau;",
                             "int join = hd->t > 0 && rt <= J->tau && hd->prev_r <= J->tau;"),
    "rightmost_tie": ("          if (l < bl) {", "          if (l <= bl) {"),
    "capacity_off_by_one": ("      if (!unbounded && hd->nsealed == C) {",
                            "      if (!unbounded && hd->nsealed == C - 1) {"),
    "phi_is_plain_elu": ("return x > 0.0 ? x + 1.0 : exp(x);", "return x > 0.0 ? x : exp(x) - 1.0;"),
    "transposed_state": ("acc = acc + st[i]->S[(size_t)r * dk + c] * p[c];",
                         "acc = acc + st[i]->S[(size_t)c * dk + r] * p[c];"),
    "logit_scale_1_over_d": ("a[i] = dot / sqrt((double)dk);", "a[i] = dot / (double)dk;"),
    "cos_sign_flipped": ("return 1.0 - dot / (sqrt(na) * sqrt(nb));",
                         "return 1.0 + dot / (sqrt(na) * sqrt(nb));"),
    "merge_keeps_right_ts": ("  left->n = left->n + right->n;",
                             "  left->n = left->n + right->n;\n  left->ts = right->ts;"),
    "readout_before_write": ("    for (int c = 0; c < dk; c++) hd->open.z[c] = hd->open.z[c] + u[c];\n    hd->open.n = hd->open.n + 1;\n    int m = 0;",
                             "    int m = 0;"),
    "margin_gap_over_second": ("else if (bl > 0.0 && (second - bl) / bl < min_gap) min_gap = (second - bl) / bl;\n        if (J->force_count)\n          best = forced_pair(J, r, &fk, hd->t, best, bl, C - 1, crit_ward",
                               "else if (bl > 0.0 && (second - bl) / second < min_gap) min_gap = (second - bl) / second;\n        if (J->force_count)\n          best = forced_pair(J, r, &fk, hd->t, best, bl, C - 1, crit_ward"),
    "margin_ties_not_counted": ("        if (second == bl) ties += 1.0;\n        else if (bl > 0.0 && (second - bl) / bl < min_gap) min_gap = (second - bl) / bl;\n        if (J->force_count)\n          best = forced_pair(J, r, &fk, hd->t, best, bl, C - 1, crit_ward",
                                "        if (second == bl) ties += 0.0;\n        else if (bl > 0.0 && (second - bl) / bl < min_gap) min_gap = (second - bl) / bl;\n        if (J->force_count)\n          best = forced_pair(J, r, &fk, hd->t, best, bl, C - 1, crit_ward"),
    "margin_includes_first_token": ("    if (hd->t > 0) {\n      double mrg = fabs(rt - J->tau);",
                                    "    {\n      double mrg = fabs(rt - J->tau);"),
    "forced_index_ignored": ("  if (e > *ex) *ex = e;\n  return i;", "  if (e > *ex) *ex = e;\n  return best;"),
    "forced_excess_over_second": ("double e = l == bl ? 0.0 : (bl > 0.0 ? (l - bl) / bl : INFINITY);",
                                  "double e = l == bl ? 0.0 : (bl > 0.0 ? (l - bl) / l : INFINITY);"),
    "forced_leftover_ignored": ("  if (fk != J->force_count[r]) ex = INFINITY;\n", ""),
    "unbounded_still_merges": ("      if (!unbounded && hd->nsealed == C) {", "      if (hd->nsealed == C) {"),
    "fenwick_no_carry": ("while (hd->nsealed >= 2 && hd->sealed[hd->nsealed - 1].n == hd->sealed[hd->nsealed - 2].n) {",
                         "while (0) {"),
}


# Plausible mistakes in the information policy, caught by its own pins.
INFO_MUTANTS = {
    "info_no_rmsnorm": ("double rs = sqrt(ss / cnt + OR_INFO_EPS), rS = sqrt(sS / cnt + OR_INFO_EPS);",
                        "double rs = 1.0, rS = 1.0;"),
    "info_denominator_not_normalised": ("return sqrt(diff) / (sqrt(norm) + OR_INFO_EPS);",
                                        "return sqrt(diff) / (sqrt(sS) + OR_INFO_EPS);"),
    "info_transposed_token_state": ("double ns = (vv[a] * u[c]) / rs,",
                                    "double ns = (vv[c] * u[a]) / rs,"),
    "info_non_strict_join": ("join = it < J->tau;", "join = it <= J->tau;"),
    "info_density_left_only": ("return (a->info + b->info) / ((double)a->n + (double)b->n);",
                               "return a->info / ((double)a->n + (double)b->n);"),
    "info_density_mean_of_means": ("return (a->info + b->info) / ((double)a->n + (double)b->n);",
                                   "return a->info / (double)a->n + b->info / (double)b->n;"),
    "info_rightmost_tie": ("double l = density(&hd->sealed[i], &hd->sealed[i + 1]);\n          if (l < bl) {",
                           "double l = density(&hd->sealed[i], &hd->sealed[i + 1]);\n          if (l <= bl) {"),
    "info_margin_ties_not_counted": ("        if (second == bl) ties += 1.0;\n        else if (bl > 0.0 && (second - bl) / bl < min_gap) min_gap = (second - bl) / bl;\n        if (J->force_count)\n          best = forced_pair(J, r, &fk, hd->t, best, bl, C - 1, crit_density",
                                     "        if (second == bl) ties += 0.0;\n        else if (bl > 0.0 && (second - bl) / bl < min_gap) min_gap = (second - bl) / bl;\n        if (J->force_count)\n          best = forced_pair(J, r, &fk, hd->t, best, bl, C - 1, crit_density"),
    "info_forced_uses_ward": ("best = forced_pair(J, r, &fk, hd->t, best, bl, C - 1, crit_density,",
                              "best = forced_pair(J, r, &fk, hd->t, best, bl, C - 1, crit_ward,"),
    "info_sum_not_carried": ("  left->info = left->info + right->info;\n", ""),
}


def build_mutant(name):
    old, new = {**MUTANTS, **INFO_MUTANTS}[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor for {name} not found"
    src = src.replace(old, new, 1)
    d = tempfile.mkdtemp(prefix="oracle_mut_")
    c = os.path.join(d, "m.c")
    so = os.path.join(d, "m.so")
    open(c, "w").write(src)
    subprocess.run(["gcc", "-O1", "-ffp-contract=off", "-fPIC", "-shared", "-pthread",
                    "-o", so, c, "-lm"], check=True)
    return O.load_library(so)


def all_pins(lib):
    pins.check_hand_trace(lib)
    pins.check_margins_hand(lib)
    for seed in range(3):
        for C in (3, 5):
            pins.check_forced_mode(seed, C, 0.5, lib)
    for seed in range(6):
        for C in (2, 3, 5):
            for tau in (0.3, 0.5, 1.0):
                pins.check_against_bruteforce(seed, C, tau, lib)
    pins.check_single_state(lib)
    pins.check_all_singletons(lib)
    pins.check_fenwick(lib)
    for seed in range(3):
        pins.check_unbounded(seed, 0.5, lib)


def test_real_oracle_passes_pins():
    all_pins(None)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name):
    lib = build_mutant(name)
    with pytest.raises(AssertionError):
        all_pins(lib)


def test_real_oracle_passes_info_pins():
    info_pins.all_info_pins(None)


@pytest.mark.parametrize("name", sorted(INFO_MUTANTS))
def test_info_mutant_is_caught(name):
    lib = build_mutant(name)
    with pytest.raises(AssertionError):
        info_pins.all_info_pins(lib)
