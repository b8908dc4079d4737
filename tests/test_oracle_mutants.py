"""The oracle's pins must reject broken copies of the oracle.

Each case below compiles kvc_oracle.c with one plausible slip planted in it (on the CPU,
into a temporary directory) and requires that at least one pin in test_oracle_pins.py
fails against that copy.  This shows the pins constrain the oracle rather than merely
agree with it.
"""
import os
import subprocess

import pytest

import test_oracle_pins as pins
from oracle import oracle as O

SRC = os.path.join(os.path.dirname(O.__file__), "kvc_oracle.c")

# (name, exact source text, replacement)
MUTANTS = [
    ("scale 1/D instead of 1/sqrt(D)", "1.0 / sqrt((double)D)", "1.0 / (double)D"),
    ("no logit scale", "row[j] = x * inv_sqrt_d;", "row[j] = x;"),
    ("mask drops the diagonal", "for (int j = 0; j <= t; ++j) {\n                double x",
     "for (int j = 0; j < t; ++j) {\n                double x"),
    ("query positions shifted", "const int t = N - w + i;", "const int t = N - w + i - 1;"),
    ("GQA mapping interleaved", "const int g = h * G + gg;", "const int g = gg * J->Hkv + h;"),
    ("no max shift", "l += exp(row[j] - m);", "l += exp(row[j]);"),
    ("unnormalised", "s[j] += exp(row[j] - m) / l;", "s[j] += exp(row[j] - m);"),
    ("ties to the higher index", "return (a->j > b->j) - (a->j < b->j);",
     "return (a->j < b->j) - (a->j > b->j);"),
    ("ascending selection", "if (a->v > b->v) return -1;\n    if (a->v < b->v) return 1;",
     "if (a->v > b->v) return 1;\n    if (a->v < b->v) return -1;"),
    ("pool radius P instead of (P-1)/2", "const int r = (P - 1) / 2;", "const int r = P / 2 + 1;"),
    ("pool not clipped at hi", "int t1 = j + r > hi - 1 ? hi - 1 : j + r;",
     "int t1 = j + r > N - 1 ? N - 1 : j + r;"),
    ("window not kept", "for (int j = N - w; j < N; ++j) kept[n++] = j;",
     "for (int j = N - w; j < N - 1; ++j) kept[n++] = j;\n        kept[n++] = c[k_sel].j;"),
    ("layers not summed", "for (int layer = 0; layer < L; ++layer)\n        for (int b = 0; b < B; ++b)",
     "for (int layer = L - 1; layer < L; ++layer)\n        for (int b = 0; b < B; ++b)"),
    ("entropy logit scale 1/D", "1.0 / sqrt((double)J->D)", "1.0 / (double)J->D"),
    ("entropy in bits", "if (p > 0.0) H -= p * log(p);", "if (p > 0.0) H -= p * log2(p);"),
    ("entropy row's keys one short", "for (int j = 0; j <= last; ++j) {\n        double acc",
     "for (int j = 0; j < last; ++j) {\n        double acc"),
    ("sample variance", "cand_var[row] = var / n_c;", "cand_var[row] = var / (n_c - 1);"),
    ("csm: dot product instead of cosine", "? key_dot(k, dtype, a, b, D) / (na * nb) : 0.0",
     "? key_dot(k, dtype, a, b, D) : 0.0"),
    ("csm: partition A odd", "for (int a = c0; a < c1; a += 2) {\n            const double na",
     "for (int a = c0 + 1; a < c1; a += 2) {\n            const double na"),
    ("csm: match ties to the higher position", "if (best[a] < 0 || s > sim[a])", "if (best[a] < 0 || s >= sim[a])"),
    ("csm: merge count rounds up", "const long m = (long)floor(r * (double)n_c);", "const long m = (long)ceil(r * (double)n_c);"),
    ("csm: unweighted mean", "acc_k[d] += (double)deg[a] * widen(k, dtype, (size_t)a * D + d);",
     "acc_k[d] += (double)deg[j] * widen(k, dtype, (size_t)a * D + d);"),
    ("csm: degrees not accumulated", "                    n += deg[a];\n", ""),
    ("decode: log2 of the degree", "x[t] = dot / sqrt_d + (deg ? log((double)deg[kv_row0 + t]) : 0.0);",
     "x[t] = dot / sqrt_d + (deg ? log2((double)deg[kv_row0 + t]) : 0.0);"),
    ("decode: degree term subtracted", "x[t] = dot / sqrt_d + (deg ? log((double)deg[kv_row0 + t]) : 0.0);",
     "x[t] = dot / sqrt_d - (deg ? log((double)deg[kv_row0 + t]) : 0.0);"),
    ("decode: degree ignored", "x[t] = dot / sqrt_d + (deg ? log((double)deg[kv_row0 + t]) : 0.0);",
     "x[t] = dot / sqrt_d;"),
    ("decode: no logit scale", "x[t] = dot / sqrt_d + (deg ?", "x[t] = dot + (deg ?"),
    ("decode: GQA interleaved", "const int kvh = g / G;", "const int kvh = g % Hkv;"),
    ("kept mass over the candidates only", "for (int j = 0; j < N; ++j) total += s[j];",
     "for (int j = S; j < N - w; ++j) total += s[j];"),
]

PIN_TESTS = [
    lambda: [pins.test_all_equal_logits_closed_form(*a) for a in [(17, 3, 2), (40, 8, 4), (5, 5, 1)]],
    pins.test_two_key_logistic_pins_scale,
    pins.test_causal_mask_boundary,
    pins.test_dominant_key_and_no_overflow,
    pins.test_gqa_mapping_contiguous_groups,
    lambda: pins.test_mass_invariant(__import__("torch").float32),
    pins.test_matches_library_softmax,
    pins.test_layers_and_heads_are_sums,
    lambda: [pins.test_pool_delta_gives_clipped_plateau(P) for P in (1, 3, 7)],
    pins.test_pool_ramp_and_no_leak_from_outside,
    pins.test_pool_matches_sliding_window_library,
    pins.test_select_brute_force_with_ties,
    pins.test_select_matches_library_sort_and_invariants,
    pins.test_select_all_equal_takes_lowest_indices,
    lambda: [pins.test_entropy_equal_logits_is_log_of_visible_count(*a) for a in [(17, 3, 2), (40, 8, 4)]],
    pins.test_entropy_two_keys_is_binary_entropy,
    pins.test_entropy_dominant_key_is_zero_and_matches_library,
    pins.test_row_stats_against_definitions,
    pins.test_csm_merge_count,
    lambda: [pins.test_csm_matches_brute_force(*a) for a in [(23, 1, 3, 4, 0.5), (40, 0, 0, 6, 0.3), (31, 2, 5, 8, 0.45),
                                                             (12, 1, 1, 2, 0.5)]],
    pins.test_csm_invariants_and_closed_forms,
    pins.test_csm_bf16_output_rounding,
    pins.test_csm_ties_go_to_lower_position,
    lambda: [pins.test_centroid_attention_unit_degrees_is_library_attention(*a)
             for a in [(1, 4, 1, 1, 37, __import__("torch").float64), (2, 8, 2, 3, 70, __import__("torch").float32)]],
    pins.test_centroid_attention_degree_is_replication,
    pins.test_centroid_attention_closed_forms,
    pins.test_centroid_attention_gqa_groups,
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_reject_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for '{name}' not unique"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", str(so), str(path),
                           "-lm", "-lpthread"])
    failures = 0
    with O.using_library(str(so)):
        for pin in PIN_TESTS:
            try:
                pin()
            except (AssertionError, ValueError):
                failures += 1
    assert failures > 0, f"no pin caught the mutant '{name}'"
