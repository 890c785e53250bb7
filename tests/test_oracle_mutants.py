"""Plant one mistake at a time in a copy of the oracle source (on the CPU) and
check that at least one pin in test_oracle_pins fails for each.  Every planted
mistake keeps all memory accesses in bounds."""
import os
import shutil
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "moe_oracle.c")

MUTANTS = {
    "tie_keeps_higher_id": ("l[e] > l[best]", "l[e] >= l[best]"),
    "softmax_not_normalised": ("(float)(ex[j] / z)", "(float)(ex[j])"),
    "gate_and_up_swapped": ("g[c] = g[c] / (1.0 + exp(-g[c])) * u[c];", "g[c] = u[c] / (1.0 + exp(-u[c])) * g[c];"),
    "down_weight_transposed": ("(size_t)c * H + h", "(size_t)h * I + c"),
    "gate_weight_transposed": ("orc_load(w_gate[e], wdt, (size_t)h * I + c)", "orc_load(w_gate[e], wdt, (size_t)c * H + h)"),
    "rows_in_reverse_token_order": ("for (int t = 0; t < T; ++t) {\n    for (int j = 0; j < k; ++j) {\n      int s = t * k + j, e = ids[s];",
                                    "for (int t = T - 1; t >= 0; --t) {\n    for (int j = 0; j < k; ++j) {\n      int s = t * k + j, e = ids[s];"),
    "offsets_not_accumulated": ("expert_offsets[e + 1] = expert_offsets[e] + expert_counts[e];",
                                "expert_offsets[e + 1] = expert_counts[e];"),
    "rank_offsets_not_accumulated": ("rank_offsets[r + 1] = rank_offsets[r] + rank_counts[r];",
                                     "rank_offsets[r + 1] = rank_counts[r];"),
    "round_robin_placement": ("for (int e = r * EL; e < (r + 1) * EL; ++e)", "for (int e = r; e < E; e += R)"),
    "src_rank_round_robin": ("(int)(((int64_t)t * R) / T)", "(t % R)"),
    "combine_ignores_weight": ("out[h] += wj * y_disp", "out[h] += y_disp"),
    "router_weight_transposed": ("orc_load(w, wdt, (size_t)e * H + h)", "orc_load(w, wdt, (size_t)h * E + e)"),
    "router_drops_bias": ("      if (bias) acc += bias[e];\n", "\n"),
    "eplb_extra_replica_to_lightest": ("if (load[e] * (int64_t)n[best] > load[best] * (int64_t)n[e]) best = e;",
                                       "if (load[e] * (int64_t)n[best] < load[best] * (int64_t)n[e]) best = e;"),
    "eplb_share_ignores_remainder": ("share[m] = load[e] / n[e] + (j < load[e] % n[e] ? 1 : 0);",
                                     "share[m] = load[e] / n[e];"),
    "eplb_places_on_heaviest_rank": ("(r_best < 0 || rank_load[r] < rank_load[r_best])",
                                     "(r_best < 0 || rank_load[r] > rank_load[r_best])"),
    "eplb_remap_first_replica_only": ("out = replicas[replica_offsets[e] + t % n];", "out = replicas[replica_offsets[e]];"),
    "partials_round_robin_owner": ("e / EL != r) continue;", "e % R != r) continue;"),
    "partials_drop_weight": ("out[h] += affinity * y_disp", "out[h] += y_disp"),
    "reduce_skips_last_rank": ("for (int r = 0; r < R; ++r) acc += part", "for (int r = 0; r < R - 1; ++r) acc += part"),
    "ep_no_shared_delivery": ("          send_counts[d] += 1;\n          break;", "          send_counts[d] += 1;"),
    "ep_rows_in_reverse_token_order": ("    for (int t = 0; t < T; ++t) {\n      int n = 0;",
                                       "    for (int t = T - 1; t >= 0; --t) {\n      int n = 0;"),
    "ep_local_id_not_offset": ("row_ids[(size_t)row * k + n] = e - d * EL;", "row_ids[(size_t)row * k + n] = e;"),
    "combine_drops_last_choice": ("for (int j = 0; j < k; ++j) {\n      int row = slot_to_row", "for (int j = 0; j < k - 1; ++j) {\n      int row = slot_to_row"),
}

PINS = [
    pins.test_worked_example_route_and_dispatch,
    pins.test_worked_example_results_return_in_original_order,
    pins.test_top2_weights_and_combine,
    pins.test_imbalance_example,
    pins.test_masked_sum_ep8,
    pins.test_route_ties_lower_id_first_and_signed_zero,
    lambda: pins.test_route_matches_lexsort(37, 8, 2),
    lambda: pins.test_dispatch_index_invariants(127, 8, 2, 4),
    pins.test_src_rank_matches_toy_layer_statement,
    pins.test_swiglu_closed_forms,
    lambda: pins.test_round_trip_equals_dense_masked_moe(16, 32, 64, 8, 2, 4),
    pins.test_identity_experts_reproduce_input,
    pins.test_router_logits_hand_example,
    pins.test_router_logits_one_hot_rows_select_columns,
    pins.test_router_logits_bias_only_and_bf16_widening,
    pins.test_eplb_hand_example_one_hot_expert,
    pins.test_eplb_equal_loads_without_extra_slots_alternate_ranks,
    pins.test_eplb_remainders_go_to_the_first_replicas,
    lambda: pins.test_eplb_plan_invariants(20, 4, 6, 3),
    lambda: pins.test_rank_partials_equal_dense_masked_moe_per_rank(9, 16, 24, 8, 3, 4),
    pins.test_ep_plan_worked_example_top1,
    pins.test_ep_plan_top2_shares_input_delivery,
    lambda: pins.test_ep_round_trip_equals_single_gpu_round_trip((9, 3, 6), 16, 8, 6, 3, 3, 1.5),
]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("gcc missing")
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    path = tmp_path / "mut.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "libmut.so"
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", str(so), str(path), "-lm"])
    caught = []
    with oracle._substitute_library(str(so)):
        for pin in PINS:
            try:
                pin()
            except Exception:  # a failed assertion, or a wrong value that breaks the check itself
                caught.append(getattr(pin, "__name__", "pin"))
    assert caught, f"mutant {name} passed every pin"
