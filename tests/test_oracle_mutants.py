"""Plant plausible mistakes in copies of the oracle source (CPU only) and check
that the pins reject every one of them.  The product code is never touched:
each mutant is a temporary build of a patched copy of oracle/lb_oracle.c."""
import os
import subprocess

import pytest

import oracle
import pins
from oracle import build as obuild

MUTANTS = {
    "gate_drops_bias": ("acc += (double)bias[e];", "acc += 0.0;"),
    "gate_transposed_weight": ("orc_bf16(ht[c]) * orc_bf16(we[c])",
                               "orc_bf16(ht[c]) * orc_bf16(w[(int64_t)c * E + e % H])"),
    "gate_tie_to_higher_id": ("row[e] > row[best]", "row[e] >= row[best]"),
    "gate_float_accumulate": ("double acc = 0.0;", "float acc = 0.0f;"),
    "count_wrong_source_rank": ("int g = (int)(t / Tg);", "int g = (int)(t % G);"),
    "count_skips_duplicate_check": ("if (ids[t * k + jj] == e)", "if (0)"),
    "plan_phase1_tie_to_higher_id": ("c > cnt[(int64_t)g * E + best]", "c >= cnt[(int64_t)g * E + best]"),
    "plan_phase1_imports_unrequested": ("if (c <= 0)\n                    continue;", "if (c < 0)\n                    continue;"),
    "plan_no_halving": ("int64_t d = gap > 0 ? (gap >> 1) : 0;", "int64_t d = gap > 0 ? gap : 0;"),
    "plan_argmax_tie_to_higher_rank": ("if (load[r] > load[u])", "if (load[r] >= load[u])"),
    "plan_locality_dropped": ("int64_t c = cnt[(int64_t)cv * E + ce];", "int64_t c = 0;"),
    "plan_colouring_not_disjoint": ("while (busy[(int64_t)ou[i] * (maxe + 1) + c] || busy[(int64_t)ov[i] * (maxe + 1) + c])",
                                    "while (busy[(int64_t)ou[i] * (maxe + 1) + c])"),
    "split_no_halving": ("int64_t delta = (gap < 0 ? -gap : gap) >> 1;", "int64_t delta = (gap < 0 ? -gap : gap);"),
    "split_no_reverse_move": ("int64_t limit = gap > 0 ? (int64_t)mass[i] : (int64_t)(tok[i] - mass[i]);",
                              "int64_t limit = gap > 0 ? (int64_t)mass[i] : 0;"),
    "split_wrong_sign": ("loads[v] += sd;", "loads[v] -= sd;"),
    "split_partition_remainder_last": ("(j < R[e] % mcount ? 1 : 0)", "(j >= mcount - R[e] % mcount ? 1 : 0)"),
    "split_fixed_counts_replicated": ("if (rep_cnt[e] == 0)\n                x += R[e];", "x += R[e];"),
    "assign_home_and_replica_swapped": ("d = (q - off < mass[i]) ? home : edge_v[i];",
                                        "d = (q - off < mass[i]) ? edge_v[i] : home;"),
    "assign_unstable_order": ("perm[fill[key]++] = (int32_t)f;",
                              "{ int64_t at = fill[key]++; perm[(int64_t)offs[key + 1] - 1 - (at - offs[key])] = (int32_t)f; }"),
    "assign_remote_ignores_locality": ("if (holds[(int64_t)s * E + e]) {\n            d = s;",
                                       "if (0) {\n            d = s;"),
    "swaps_drops_gamma": ("const double prod = gamma * (double)dsq;", "const double prod = 0.0 * (double)dsq;"),
    "swaps_squared_term_sign": ("const double delta = (double)(loads[u] - mx) + prod;",
                                "const double delta = (double)(loads[u] - mx) - prod;"),
    "swaps_tie_to_last_pair": ("if (best_a < 0 || ratio > best_ratio)", "if (best_a < 0 || ratio >= best_ratio)"),
    "swaps_expert_moves_twice": ("moved[a] = moved[b] = 1;", "(void)moved;"),
    "swaps_link_budget_unspent": ("res_link[u * G + v] -= cost;\n        res_link[v * G + u] -= cost;", ";"),
    "swaps_tau_strict": ("if ((double)(loads[u] - loads[v]) <= tau) break;",
                         "if ((double)(loads[u] - loads[v]) < tau) break;"),
    "swaps_frontier_tie_to_higher_rank": ("if (loads[r] > loads[u]) u = r;", "if (loads[r] >= loads[u]) u = r;"),
    "swaps_ignores_untouched_ranks": ("if (rest > mx) mx = rest;", ";"),
    "variant_no_reverse_allows_reverse": ("(variant == ORC_SV_NO_REVERSE ? 0 : (int64_t)(tok[i] - mass[i]))",
                                          "(int64_t)(tok[i] - mass[i])"),
    "variant_jacobi_not_damped": ("(gap < 0 ? -gap : gap) >> (variant == ORC_SV_JACOBI ? 2 : 1)",
                                  "(gap < 0 ? -gap : gap) >> 1"),
    "variant_jacobi_no_snapshot": ("for (int i = 0; i < G; ++i) snap[i] = loads[i];",
                                   "for (int i = 0; i < G && p == 1; ++i) snap[i] = loads[i];"),
    "variant_hash_remainder_shifted": ("int64_t share = q + (j + 1 < rem ? 1 : 0);", "int64_t share = q + (j < rem ? 1 : 0);"),
    "variant_water_leftover_last": ("for (int h = 0; h < n && used < R; ++h)", "for (int h = n - 1; h >= 0 && used < R; --h)"),
    "variant_proportional_equal_weights": ("wt[h] = M - B[h] + 1;", "wt[h] = 1;"),
    "variant_fp32_truncates": ("float delta = (gap < 0.0f ? -gap : gap) * 0.5f;",
                               "float delta = floorf((gap < 0.0f ? -gap : gap) * 0.5f);"),
    "variant_q1120_no_fraction": ("const int f = 20 - s;", "const int f = 0 * s;"),
    "optimum_ignores_fixed": ("orc_flow_add(&f, n_edges + r, snk, z - fixed[r]);",
                              "orc_flow_add(&f, n_edges + r, snk, z);"),
}


def _build_mutant(tmp_path, name, old, new):
    src = open(obuild.SRC).read()
    assert src.count(old) == 1, f"{name}: pattern must occur exactly once"
    path = os.path.join(tmp_path, f"{name}.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    out = os.path.join(tmp_path, f"lib{name}.so")
    obuild.build(force=True, src=path, out=out)
    return oracle.Oracle(out)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    o = _build_mutant(str(tmp_path), name, old, new)
    failures = []
    for check in pins.ALL_CHECKS:
        try:
            check(o)
        except Exception as e:  # an assertion, a bad-data error or a crash of the check
            failures.append((check.__name__, type(e).__name__))
    assert failures, f"no pin caught mutant {name}"
