"""Plant plausible mistakes in copies of the oracle source (CPU only) and check
that the pins reject every one of them.  The product code is never touched:
each mutant is a temporary build of a patched copy of oracle/lb_oracle.c.

A mutant is (function, text, replacement[, occurrence]): the replacement is
made inside the body of the named oracle function only, at the given
occurrence of the text there (the first by default), so the oracle's wording
never has to bend to keep a pattern unique in the whole file."""
import os
import re

import pytest

import oracle
import pins
from oracle import build as obuild

MUTANTS = {
    "gate_drops_bias": ("orc_gate", "acc += (double)bias[e];", "acc += 0.0;"),
    "gate_transposed_weight": ("orc_gate", "orc_bf16(ht[c]) * orc_bf16(we[c])",
                               "orc_bf16(ht[c]) * orc_bf16(w[(int64_t)c * E + e % H])"),
    "gate_tie_to_higher_id": ("orc_gate", "row[e] > row[best]", "row[e] >= row[best]"),
    "gate_float_accumulate": ("orc_gate", "double acc = 0.0;", "float acc = 0.0f;"),
    "count_wrong_source_rank": ("orc_count", "int g = (int)(t / Tg);", "int g = (int)(t % G);"),
    "count_skips_duplicate_check": ("orc_count", "if (ids[t * k + jj] == e)", "if (0)"),
    "plan_phase1_tie_to_higher_id": ("orc_plan", "c > cnt[(int64_t)g * E + best]", "c >= cnt[(int64_t)g * E + best]"),
    "plan_phase1_imports_unrequested": ("orc_plan", "if (c <= 0)\n                    continue;", "if (c < 0)\n                    continue;"),
    "plan_no_halving": ("orc_plan", "int64_t d = gap > 0 ? (gap >> 1) : 0;", "int64_t d = gap > 0 ? gap : 0;"),
    "plan_argmax_tie_to_higher_rank": ("orc_plan", "if (load[r] > load[u])", "if (load[r] >= load[u])"),
    "plan_locality_dropped": ("orc_plan", "int64_t c = cnt[(int64_t)cv * E + ce];", "int64_t c = 0;"),
    "plan_colouring_not_disjoint": ("orc_plan", "while (busy[(int64_t)ou[i] * (maxe + 1) + c] || busy[(int64_t)ov[i] * (maxe + 1) + c])",
                                    "while (busy[(int64_t)ou[i] * (maxe + 1) + c])"),
    "split_no_halving": ("orc_split", "int64_t delta = (gap < 0 ? -gap : gap) >> 1;", "int64_t delta = (gap < 0 ? -gap : gap);"),
    "split_no_reverse_move": ("orc_split", "int64_t limit = gap > 0 ? (int64_t)mass[i] : (int64_t)(tok[i] - mass[i]);",
                              "int64_t limit = gap > 0 ? (int64_t)mass[i] : 0;"),
    "split_wrong_sign": ("orc_split", "loads[v] += sd;", "loads[v] -= sd;"),
    "split_partition_remainder_last": ("orc_split_start", "(j < R[e] % mcount ? 1 : 0)", "(j >= mcount - R[e] % mcount ? 1 : 0)"),
    "split_fixed_counts_replicated": ("orc_split_start", "if (rep_cnt[e] == 0)\n                x += R[e];", "x += R[e];"),
    "assign_home_and_replica_swapped": ("orc_assign", "d = (q - off < mass[i]) ? home : edge_v[i];",
                                        "d = (q - off < mass[i]) ? edge_v[i] : home;"),
    "assign_unstable_order": ("orc_assign", "perm[fill[key]++] = (int32_t)f;",
                              "{ int64_t at = fill[key]++; perm[(int64_t)offs[key + 1] - 1 - (at - offs[key])] = (int32_t)f; }"),
    "assign_remote_ignores_locality": ("orc_assign", "if (holds[(int64_t)s * E + e]) {\n            d = s;",
                                       "if (0) {\n            d = s;"),
    "swaps_drops_gamma": ("orc_plan_swaps", "const double prod = gamma * (double)dsq;", "const double prod = 0.0 * (double)dsq;"),
    "swaps_squared_term_sign": ("orc_plan_swaps", "const double delta = (double)(loads[u] - mx) + prod;",
                                "const double delta = (double)(loads[u] - mx) - prod;"),
    "swaps_tie_to_last_pair": ("orc_plan_swaps", "if (best_a < 0 || ratio > best_ratio)", "if (best_a < 0 || ratio >= best_ratio)"),
    "swaps_expert_moves_twice": ("orc_plan_swaps", "moved[a] = moved[b] = 1;", "(void)moved;"),
    "swaps_link_budget_unspent": ("orc_plan_swaps", "res_link[u * G + v] -= cost;\n        res_link[v * G + u] -= cost;", ";"),
    "swaps_tau_strict": ("orc_plan_swaps", "if ((double)(loads[u] - loads[v]) <= tau) break;",
                         "if ((double)(loads[u] - loads[v]) < tau) break;"),
    "swaps_frontier_tie_to_higher_rank": ("orc_plan_swaps", "if (loads[r] > loads[u]) u = r;", "if (loads[r] >= loads[u]) u = r;"),
    "swaps_ignores_untouched_ranks": ("orc_plan_swaps", "if (rest > mx) mx = rest;", ";"),
    "variant_no_reverse_allows_reverse": ("orc_split_variant", "(variant == ORC_SV_NO_REVERSE ? 0 : (int64_t)(tok[i] - mass[i]))",
                                          "(int64_t)(tok[i] - mass[i])"),
    "variant_jacobi_not_damped": ("orc_split_variant", "(gap < 0 ? -gap : gap) >> (variant == ORC_SV_JACOBI ? 2 : 1)",
                                  "(gap < 0 ? -gap : gap) >> 1"),
    "variant_jacobi_no_snapshot": ("orc_split_variant", "for (int i = 0; i < G; ++i) snap[i] = loads[i];",
                                   "for (int i = 0; i < G && p == 1; ++i) snap[i] = loads[i];"),
    "variant_hash_remainder_shifted": ("orc_split_variant", "int64_t share = q + (j + 1 < rem ? 1 : 0);", "int64_t share = q + (j < rem ? 1 : 0);"),
    "variant_water_leftover_last": ("orc_water_fill", "for (int h = 0; h < n && used < R; ++h)", "for (int h = n - 1; h >= 0 && used < R; --h)"),
    "variant_proportional_equal_weights": ("orc_split_variant", "wt[h] = M - B[h] + 1;", "wt[h] = 1;"),
    "variant_fp32_truncates": ("orc_split_variant", "float delta = (gap < 0.0f ? -gap : gap) * 0.5f;",
                               "float delta = floorf((gap < 0.0f ? -gap : gap) * 0.5f);"),
    "variant_q1120_no_fraction": ("orc_split_variant", "const int f = 20 - s;", "const int f = 0 * s;"),
    "optimum_ignores_fixed": ("orc_split_optimum", "orc_flow_add(&f, n_edges + r, snk, z - fixed[r]);",
                              "orc_flow_add(&f, n_edges + r, snk, z);"),
}


def function_span(src, fn):
    """[start, end) of the body (braces included) of C function `fn`: its
    definition starts a line with a return type and the name, and its body
    is the brace-balanced block after the parameter list."""
    m = re.search(r"^(?:static\s+)?[a-z_0-9]+\s+\**" + re.escape(fn) + r"\(", src, re.M)
    assert m, f"function {fn} not found"
    i, depth = src.index("(", m.start()), 0
    while True:
        depth += {"(": 1, ")": -1}.get(src[i], 0)
        if depth == 0:
            break
        i += 1
    i = src.index("{", i)
    j, depth = i, 0
    while True:
        depth += {"{": 1, "}": -1}.get(src[j], 0)
        if depth == 0:
            return i, j + 1
        j += 1


def patch(src, fn, old, new, occurrence=0):
    a, b = function_span(src, fn)
    body = src[a:b]
    at = -1
    for _ in range(occurrence + 1):
        at = body.find(old, at + 1)
        assert at >= 0, f"{fn}: occurrence {occurrence} of the pattern not found"
    return src[:a] + body[:at] + new + body[at + len(old):] + src[b:]


def _build_mutant(tmp_path, name, spec):
    src = open(obuild.SRC).read()
    path = os.path.join(tmp_path, f"{name}.c")
    with open(path, "w") as f:
        f.write(patch(src, *spec))
    out = os.path.join(tmp_path, f"lib{name}.so")
    obuild.build(force=True, src=path, out=out)
    return oracle.Oracle(out)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    o = _build_mutant(str(tmp_path), name, MUTANTS[name])
    failures = []
    for check in pins.ALL_CHECKS:
        try:
            check(o)
        except Exception as e:  # an assertion, a bad-data error or a crash of the check
            failures.append((check.__name__, type(e).__name__))
    assert failures, f"no pin caught mutant {name}"


def test_patch_is_scoped_to_the_function():
    """The same text in two functions: only the named function's copy changes."""
    src = "int orc_a(int x)\n{\n    return x + 1;\n}\nstatic int orc_b(int x)\n{\n    if (x) { x += 1; }\n    return x + 1;\n}\n"
    out = patch(src, "orc_b", "x + 1", "x - 1")
    assert out.count("x + 1") == 1 and "orc_b(int x)\n{\n    if (x) { x += 1; }\n    return x - 1;" in out
    assert patch(src, "orc_b", "x +", "x *", occurrence=1).count("x * 1") == 1
