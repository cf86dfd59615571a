"""The oracle's pins catch plausible mistakes (no GPU).

Each mutation below plants one small error in a copy of oracle/psispec_oracle.c (a swapped
operand, a wrong sign or index, a dropped update, a changed comparison), builds it under a
temporary directory, and reruns the pin suites against it with ORACLE_LIB. Every mutant must
fail at least one pin; the unmodified source passes them (the other test files).
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "psispec_oracle.c")

PINS = ("test_oracle_pins.py", "test_oracle_lossless.py")
TREE_BUILD = ("test_oracle_tree_build.py",)
BANDS = ("test_oracle_bands.py",)

MUTATIONS = {
    "accept_operands_swapped": ("if (u * q[x] < p[x]) continue;", "if (u * p[x] < q[x]) continue;"),
    "accept_not_strict": ("if (u * q[x] < p[x]) continue;", "if (u * q[x] <= p[x]) continue;"),
    "residual_sign": ("res[v] = p[v] > q[v] ? p[v] - q[v] : 0.0;", "res[v] = q[v] > p[v] ? q[v] - p[v] : 0.0;"),
    "residual_not_clipped": ("res[v] = p[v] > q[v] ? p[v] - q[v] : 0.0;", "res[v] = p[v];"),
    "cdf_not_strict": ("if (C > target) {", "if (C >= target) {"),
    "bonus_wrong_row": ("oracle_row_dist_k(tgt + (size_t)K * V, V, T, tp, tk, p, &bp)",
                        "oracle_row_dist_k(tgt + (size_t)(K - 1) * V, V, T, tp, tk, p, &bp)"),
    "resid_uniform_index": ("u_resid[(size_t)b * (K + 1) + i], &b2);", "u_resid[(size_t)b * (K + 1) + i + 1], &b2);"),
    "temperature_multiplied": ("out[v] = exp((l[v] - m) / T);", "out[v] = exp((l[v] - m) * T);"),
    "topp_drops_ties": ("out[v] = (l[v] >= tau) ? out[v] / S_kept : 0.0;", "out[v] = (l[v] > tau) ? out[v] / S_kept : 0.0;"),
    "topp_not_renormalised": ("out[v] = (l[v] >= tau) ? out[v] / S_kept : 0.0;", "out[v] = (l[v] >= tau) ? out[v] / S : 0.0;"),
    "greedy_highest_index": ("if (l[v] > m) { m = l[v]; amax = v; }", "if (l[v] >= m) { m = l[v]; amax = v; }"),
    "tree_no_removal": ("qt[t] = 0.0;", "(void)t;"),
    "tree_no_residual_update": ("for (int v = 0; v < V; ++v) r[v] = res[v] / Z;", "(void)Z;"),
    "tree_wrong_uniform": ("double u = u_accept[n0 + c];", "double u = u_accept[n0 + cur];"),
    "topk_off_by_one": ("tau = vals[top_k - 1];", "tau = vals[top_k];"),
    "topk_topp_over_whole_row": ("const double floor_v = tau, total = S_kept;",
                                 "const double floor_v = tau, total = S;"),
    # the further tree rules and the candidate trie (pinned in test_oracle_tree_build.py)
    "det_no_renormalise": ("for (int v = 0; v < V; ++v) r[v] /= Zr;", "(void)Zr;", TREE_BUILD),
    "det_no_removal": ("          r[t] = 0.0;\n", "          (void)t;\n", TREE_BUILD),
    "det_accept_not_by_r": ("if (ud < r[t]) { next = c; break; }", "if (ud < 0.5) { next = c; break; }", TREE_BUILD),
    "wr_removes_token": ("if (rule == ORACLE_TREE_SAMPLED_WOR) {", "if (rule != ORACLE_TREE_DETERMINISTIC) {",
                         TREE_BUILD),
    "build_ties_to_deeper": ("(sa == sb && da < db)", "(sa == sb && da > db)", TREE_BUILD),
    "build_logit_sum_not_accumulated": ("lsum[nn] = lsum[pa] + draft[(size_t)d * V + tokens[nn]];",
                                        "lsum[nn] = draft[(size_t)d * V + tokens[nn]];", TREE_BUILD),
    "build_ties_rank_reversed": ("(cmp == 0 && f_rank[e] < f_rank[bi])", "(cmp == 0 && f_rank[e] > f_rank[bi])",
                                 TREE_BUILD),
    "build_candidate_ties_high_index": ("if (best < 0 || qi[v] > qi[best]) best = v;",
                                        "if (best < 0 || qi[v] >= qi[best]) best = v;", TREE_BUILD),
    "build_score_sum": ("score[nn] = score[pa] * q[(size_t)d * V + tokens[nn]];",
                        "score[nn] = score[pa] + q[(size_t)d * V + tokens[nn]];", TREE_BUILD),
    # the exception bands (pinned in test_oracle_bands.py): a wrong band would exempt requests
    # from the parity comparison, or leave near-ties unreported
    "cdf_band_zero": ("*band = dmin(fabs(before / Z - u), fabs(C / Z - u));", "*band = 0.0;", BANDS),
    "cdf_band_unscaled": ("*band = dmin(fabs(before / Z - u), fabs(C / Z - u));",
                          "*band = dmin(fabs(before - u), fabs(C - u));", BANDS),
    "cdf_band_upper_edge_only": ("*band = dmin(fabs(before / Z - u), fabs(C / Z - u));", "*band = fabs(C / Z - u);",
                                 BANDS),
    "topp_band_dropped": ("*band = dmin(fabs(tail / total - top_p), fabs(above / total - top_p));",
                          "*band = INFINITY;", BANDS),
    "topp_band_zero": ("*band = dmin(fabs(tail / total - top_p), fabs(above / total - top_p));", "*band = 0.0;",
                       BANDS),
    "topp_band_one_tail": ("*band = dmin(fabs(tail / total - top_p), fabs(above / total - top_p));",
                           "*band = fabs(tail / total - top_p);", BANDS),
    "ratio_band_dropped": ("if (q[x] > 0.0) note_band(&path_band, &path_kind, fabs(u - p[x] / q[x]), ORACLE_BAND_E1);",
                           "(void)u;", BANDS),
    "ratio_band_inverted": ("fabs(u - p[x] / q[x])", "fabs(u - q[x] / p[x])", BANDS),
    "resid_band_dropped": ("u_resid[(size_t)b * (K + 1) + i], &b2);\n      note_band(&path_band, &path_kind, b2, "
                           "ORACLE_BAND_E2);", "u_resid[(size_t)b * (K + 1) + i], &b2);", BANDS),
    "bonus_band_dropped": ("        note_band(&path_band, &path_kind, bp, ORACLE_BAND_E3);\n"
                           "        note_band(&path_band, &path_kind, b2, ORACLE_BAND_E2);",
                           "        note_band(&path_band, &path_kind, bp, ORACLE_BAND_E3);", BANDS),
    "band_past_rejection": ("      if (i > j) continue; /* past the first rejection: probabilities only */\n"
                            "      double u = u_accept[(size_t)b * K + i];\n"
                            "      note_band(&path_band, &path_kind, dmin(bp, bq), ORACLE_BAND_E3);\n"
                            "      if (q[x] > 0.0) note_band(&path_band, &path_kind, fabs(u - p[x] / q[x]), "
                            "ORACLE_BAND_E1);\n",
                            "      double u = u_accept[(size_t)b * K + i];\n"
                            "      note_band(&path_band, &path_kind, dmin(bp, bq), ORACLE_BAND_E3);\n"
                            "      if (q[x] > 0.0) note_band(&path_band, &path_kind, fabs(u - p[x] / q[x]), "
                            "ORACLE_BAND_E1);\n"
                            "      if (i > j) continue;\n", BANDS),
    "linear_topp_band_mislabelled": ("note_band(&path_band, &path_kind, dmin(bp, bq), ORACLE_BAND_E3);",
                                     "note_band(&path_band, &path_kind, dmin(bp, bq), ORACLE_BAND_E1);", BANDS),
    "sample_band_without_draw": ("note_band(&bi, &kind, b2, ORACLE_BAND_E2);", "(void)b2;", BANDS),
    "sample_band_without_topp": ("note_band(&bi, &kind, b3, ORACLE_BAND_E3);", "(void)b3;", BANDS),
    "tree_ratio_band_dropped": ("if (qt[t] > 0.0) note_band(&path_band, &path_kind, fabs(u - r[t] / qt[t]), "
                                "ORACLE_BAND_E1);", "(void)u;", BANDS),
    "tree_det_band_dropped": ("note_band(&path_band, &path_kind, fabs(ud - r[t]), ORACLE_BAND_E1);", "(void)ud;",
                              BANDS),
    "tree_draw_band_dropped": ("u_resid[n0 + cur], &b2);\n      note_band(&path_band, &path_kind, b2, ORACLE_BAND_E2);",
                               "u_resid[n0 + cur], &b2);", BANDS),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTATIONS[name][:2]
    files = MUTATIONS[name][2] if len(MUTATIONS[name]) > 2 else PINS
    src = open(SRC).read()
    assert src.count(old) == 1, name
    mut = tmp_path / "mutant.c"
    mut.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-shared", "-fPIC", "-I", os.path.dirname(SRC),
                           "-o", str(lib), str(mut), "-lm"])
    env = dict(os.environ, ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider"] +
                       [os.path.join(ROOT, "tests", f) for f in files],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, "mutation %s survived the pins" % name
