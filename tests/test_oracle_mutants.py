"""Mutation test of the oracle's pins.

Each mutant plants one plausible mistake in a copy of oracle/oracle.c (a
dropped term, a swapped index, a wrong tie-break, a transposed operand), built
in a temporary directory; the pin suites are then run against it and must
fail.  A mutant that survives means some part of the oracle is not pinned."""
import os
import subprocess
import sys

import pytest

from conftest import ROOT

SRC = os.path.join(ROOT, "oracle", "oracle.c")
PINS = ["tests/test_oracle_pins.py", "tests/test_oracle_brute.py", "tests/test_oracle_prereduce.py",
        "tests/test_oracle_replicas.py", "tests/test_oracle_replicas_capped.py", "tests/test_oracle_shuffle_balanced.py", "tests/test_oracle_ema.py", "tests/test_oracle_capped.py",
        "tests/test_ep_cpu.py::test_routes_hand_worked", "tests/test_ep_cpu.py::test_route_definition",
        "tests/test_ep_cpu.py::test_exchange_rows_from_route_tables",
        "tests/test_oracle_property.py"]

MUTANTS = {
    "counts_drop_diagonal": ("                for (int a = 0; a < k; ++a)\n                    for (int b = 0; b < k; ++b)\n"
                             "                        Cl[(size_t)d[a] * E + d[b]] += 1;",
                             "                for (int a = 0; a < k; ++a)\n                    for (int b = 0; b < k; ++b)\n"
                             "                        if (a != b) Cl[(size_t)d[a] * E + d[b]] += 1;"),
    "ochiai_sum_not_product": ("double den = (double)Cl[(size_t)i * E + i] * (double)Cl[(size_t)j * E + j];",
                               "double den = (double)Cl[(size_t)i * E + i] + (double)Cl[(size_t)j * E + j];"),
    "transitions_transposed": ("Ml[(size_t)a[x] * E + b[y]] += 1;", "Ml[(size_t)b[y] * E + a[x]] += 1;"),
    "uniform_off_by_one": ("for (int e = 0; e < E; ++e) expert_to_rank[e] = e / per;",
                           "for (int e = 0; e < E; ++e) expert_to_rank[e] = ((e + 1) / per) % G;"),
    "rows_source_major": ("    if (a->dst != b->dst) return a->dst < b->dst ? -1 : 1;\n"
                          "    if (a->src != b->src) return a->src < b->src ? -1 : 1;",
                          "    if (a->src != b->src) return a->src < b->src ? -1 : 1;\n"
                          "    if (a->dst != b->dst) return a->dst < b->dst ? -1 : 1;"),
    "V_counts_source_node": ("if (node_hit[q] && q != s / rpn) V += 1;", "if (node_hit[q]) V += 1;"),
    "local_counts_remote": ("if (r == s) local += 1;", "if (r != s) local += 1;"),
    "jmask_reversed": ("jm |= (uint8_t)(1u << j);", "jm |= (uint8_t)(1u << (k - 1 - j));"),
    "combine_drops_last_pick": ("            for (int j = 0; j < k; ++j) {\n                size_t row",
                                "            for (int j = 0; j < k - 1; ++j) {\n                size_t row"),
    "shuffle_ties_highest_rank": ("if (r == 0 || s > best_s) { best = r; best_s = s; }",
                                  "if (r == 0 || s >= best_s) { best = r; best_s = s; }"),
    "correlated_seed_lowest_load": ("C[(size_t)pool[x] * E + pool[x]] > C[(size_t)pool[best] * E + pool[best]]",
                                    "C[(size_t)pool[x] * E + pool[x]] < C[(size_t)pool[best] * E + pool[best]]"),
    "rank_score_transposed": ("if (next_expert_to_rank[f] == r) s += trans[(size_t)e * E + f];",
                              "if (next_expert_to_rank[f] == r) s += trans[(size_t)f * E + e];"),
    "capacity_ties_highest_device": ("if (device_load[g] < device_load[best]) best = g;",
                                     "if (device_load[g] <= device_load[best]) best = g;"),
    "reduce_ignores_scale": ("acc += (double)send_w[i * k + j] * (double)scale[e] * x;",
                             "acc += (double)send_w[i * k + j] * x;"),
    "row_sum_counts_repeats": ("if (!seen) acc += load_elem(y, is_bf16, (size_t)r * d + c);",
                               "acc += load_elem(y, is_bf16, (size_t)r * d + c);"),
    "replica_pick_ignores_source_node": ("int allowed = any_ns ? (r / rpn == ns) : ((best_set >> (r / rpn)) & 1);",
                                         "int allowed = ((best_set >> (r / rpn)) & 1) || r / rpn == ns;"),
    "replica_pick_ignores_used_ranks": ("if (pick < 0) pick = used_pick >= 0 ? used_pick : low;",
                                        "if (pick < 0) pick = low;"),
    "replica_set_ties_largest": ("if (size < best_size) { best_size = size; best_set = set; }",
                                 "if (size <= best_size) { best_size = size; best_set = set; }"),
    "replica_room_ties_highest_rank": ("if (room[r] > 0 && (br < 0 || room[r] > room[br])) br = r;",
                                       "if (room[r] > 0 && (br < 0 || room[r] >= room[br])) br = r;"),
    "balanced_ties_highest_token": ("if (a->t != b->t) return a->t < b->t ? -1 : 1;",
                                    "if (a->t != b->t) return a->t > b->t ? -1 : 1;"),
    "balanced_ties_highest_rank": ("if (a->r != b->r) return a->r < b->r ? -1 : 1;",
                                   "if (a->r != b->r) return a->r > b->r ? -1 : 1;"),
    "balanced_capacity_off_by_one": ("if (target[p->t] < 0 && held[p->r] < capacity) {",
                                     "if (target[p->t] < 0 && held[p->r] <= capacity) {"),
    "balanced_score_ascending": ("if (a->s != b->s) return a->s > b->s ? -1 : 1;",
                                 "if (a->s != b->s) return a->s < b->s ? -1 : 1;"),
    "ema_weights_swapped": ("double a = alpha * x;\n            double b = (1.0 - alpha) * ema_in[c];",
                            "double a = (1.0 - alpha) * x;\n            double b = alpha * ema_in[c];"),
    "ema_first_batch_zero": ("            ema_out[c] = x;\n        }", "            ema_out[c] = 0.0 * x;\n        }"),
    "capped_forced_pick_heaviest": ("if (pick < 0 || C[(size_t)pool[x] * E + pool[x]] < C[(size_t)pool[pick] * E + pool[pick]])",
                                    "if (pick < 0 || C[(size_t)pool[x] * E + pool[x]] > C[(size_t)pool[pick] * E + pool[pick]])"),
    "capped_cap_ignored": ("if (cap >= 0.0 && (double)(load + nx) > cap) continue;", "(void)nx;"),
    "capped_closes_late": ("if (load[r] < cap) open_ranks |= (uint64_t)1 << r;",
                           "if (load[r] <= cap) open_ranks |= (uint64_t)1 << r;"),
    "capped_forced_pick_closed_only": ("#define USABLE(j, r) (!any_open[j] || ((open_ranks >> (r)) & 1))",
                                       "#define USABLE(j, r) (((open_ranks >> (r)) & 1))"),
    "capped_cap_rounded_up": ("const double c = floor((1.0 + eps) * (double)((int64_t)T * k) / (double)G);",
                              "const double c = ceil((1.0 + eps) * (double)((int64_t)T * k) / (double)G);"),
    "capped_load_drops_last_pick": ("for (int j = 0; j < k; ++j) load[pick_rank[(size_t)t * k + j]] += 1;",
                                    "for (int j = 0; j + 1 < k; ++j) load[pick_rank[(size_t)t * k + j]] += 1;"),
    "rank_loads_off_diagonal": ("load[expert_to_rank[e]] += coact[(size_t)e * E + e];",
                                "load[expert_to_rank[e]] += coact[(size_t)e * E + (e + 1) % E];"),
    "exchange_counts_own_device": ("            if (s / Gl == r / Gl) continue;\n            sent[s / Gl]",
                                   "            sent[s / Gl]"),
    "ep_routes_counts_transposed": ("run += counts_all[s * G + r];", "run += counts_all[r * G + s];"),
    "ep_routes_sender_base": ("const int64_t first_global = off[r * G + s] - off[(r / Gl) * Gl * G];",
                              "const int64_t first_global = off[r * G + s] - off[me * Gl * G];"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation site not found exactly once"
    mutant = tmp_path / "oracle_mutant.c"
    mutant.write_text(src.replace(old, new))
    lib = tmp_path / "liboracle_mutant.so"
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-std=c11", "-fPIC", "-shared", str(mutant),
                           "-o", str(lib), "-lm"])
    env = dict(os.environ, ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider"] + PINS,
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, "mutant %s survived the pins:\n%s" % (name, r.stdout[-2000:])
