"""The pins have teeth: each plausible mistake planted in a copy of the oracle
(on the CPU, rebuilt with the same compiler flags) makes at least one pin fail."""
import ctypes
import os

import pytest

import oracle
from tests import test_oracle_pins as pins

MUTANTS = [
    # (name, original text, planted mistake, pins expected to catch it)
    ("no_renormalisation", "for (int64_t i = 0; i < n; ++i) p[i] = p[i] / z;",
     "for (int64_t i = 0; i < n; ++i) p[i] = p[i];",
     [pins.test_gate_weights_sum_to_one_and_order, pins.test_two_way_gate_is_logistic_of_gap]),
    ("ties_to_higher_index", "scores[j] == scores[e] && j < e", "scores[j] == scores[e] && j > e",
     [pins.test_topk_matches_library_sort_with_many_ties, pins.test_tie_break_duplicate_router_columns]),
    ("ascending_rank", "if (scores[j] > scores[e]) r += 1;", "if (scores[j] < scores[e]) r += 1;",
     [pins.test_worked_router_example]),
    ("ties_not_ranked", "else if (scores[j] == scores[e] && j < e) r += 1;", "else if (0) r += 1;",
     [pins.test_topk_matches_library_sort_with_many_ties, pins.test_tie_break_duplicate_router_columns]),
    ("softmax_over_all_experts", "for (int64_t e = 0; e < N; ++e) v[e] = -INFINITY;",
     "for (int64_t e = 0; e < N; ++e) v[e] = scores[e];",
     [pins.test_gate_weights_sum_to_one_and_order, pins.test_gate_weights_equal_masked_full_softmax]),
    ("combine_drops_last_slot", "for (int64_t j = 0; j < K; ++j)\n        for (int64_t c = 0; c < D; ++c) y[c]",
     "for (int64_t j = 0; j < K - 1; ++j)\n        for (int64_t c = 0; c < D; ++c) y[c]",
     [pins.test_sparse_layer_equals_dense_masked_gate]),
    ("gate_up_swapped", "hid[n] = orc_silu(g) * u;", "hid[n] = orc_silu(u) * g;",
     [pins.test_one_expert_top1_is_dense_ffn]),
    ("down_weight_transposed", "orc_get(W2e, dtype, c * H + n)", "orc_get(W2e, dtype, n * D + c)",
     [pins.test_one_expert_top1_is_dense_ffn]),
    ("router_weight_transposed", "orc_get(Wg, w_dtype, i * N + e)", "orc_get(Wg, w_dtype, e * D + i)",
     [pins.test_router_scores_match_library_matmul]),
    ("router_bias_dropped", "if (bg) s += (double)bg[e];", "(void)bg;",
     [pins.test_router_scores_match_library_matmul]),
    ("gelu_tanh_form", "0.5 * v * (1.0 + erf(v / sqrt(2.0)))",
     "0.5 * v * (1.0 + tanh(sqrt(2.0 / 3.141592653589793) * (v + 0.044715 * v * v * v)))",
     [pins.test_activation_closed_forms]),
    ("expert_bias_dropped", "if (b1e) a += (double)b1e[n];", "(void)b1e;",
     [pins.test_one_expert_top1_is_dense_ffn]),
    ("sample_variance", "var /= (double)n;", "var /= (double)(n - 1);",
     [pins.test_cv_squared_closed_forms]),
    ("switch_f_over_T", "(counts[e] / (double)(T * K))", "(counts[e] / (double)T)",
     [pins.test_aux_stats_uniform_and_empty, pins.test_aux_stats_invariants_and_library_checks]),
    ("p_mean_not_normalised", "p_mean[e] += p[e] / z;", "p_mean[e] += p[e];",
     [pins.test_aux_stats_invariants_and_library_checks]),
    ("expert_params_one_matrix", "return 2 * D * H + (has_bias ? H + D : 0);", "return D * H + (has_bias ? H + D : 0);",
     [pins.test_gpt2_moe_parameter_totals]),
    ("softmax_shift_flipped", "p[i] = v[i] == -INFINITY ? 0.0 : exp(v[i] - M);",
     "p[i] = v[i] == -INFINITY ? 0.0 : exp(M - v[i]);",
     [pins.test_gate_weights_sum_to_one_and_order, pins.test_two_way_gate_is_logistic_of_gap]),
    ("down_bias_dropped", "if (b2e) a += (double)b2e[c];", "(void)b2e;",
     [pins.test_one_expert_top1_is_dense_ffn]),
    ("silu_sign_flipped", "return g / (1.0 + exp(-g));", "return g / (1.0 + exp(g));",
     [pins.test_activation_closed_forms, pins.test_one_expert_top1_is_dense_ffn]),
    ("combine_unweighted", "y[c] = y[c] + w[j] * E[j * D + c];", "y[c] = y[c] + E[j * D + c];",
     [pins.test_sparse_layer_equals_dense_masked_gate]),
    ("simple_loss_missing_N", "return (double)N * sum;", "return sum;",
     [pins.test_balance_loss_extremes, pins.test_aux_stats_uniform_and_empty]),
    ("switch_loss_missing_N", "scalars[0] = (double)N * fP;", "scalars[0] = fP;",
     [pins.test_aux_stats_uniform_and_empty, pins.test_aux_stats_invariants_and_library_checks]),
    ("cv2_mean_not_squared", "return var / (mean * mean);", "return var / mean;",
     [pins.test_cv_squared_closed_forms]),
    ("importance_counts_tokens", "importance[sel[t * K + j]] += w[t * K + j];", "importance[sel[t * K + j]] += 1.0;",
     [pins.test_aux_stats_invariants_and_library_checks]),
    ("shared_expert_dropped", "            orc_add_shared(D, sh, y_out + t * D);", "            (void)sh;",
     [pins.test_one_expert_with_shared_expert_is_two_dense_ffns,
      pins.test_shared_expert_alone_when_routed_experts_are_zero]),
    ("shared_expert_replaces_routed", "for (int64_t c = 0; c < D; ++c) y[c] = y[c] + s[c];",
     "for (int64_t c = 0; c < D; ++c) y[c] = s[c];",
     [pins.test_one_expert_with_shared_expert_is_two_dense_ffns]),
    ("selection_bias_ignored", "s[e] + (bsel ? (double)bsel[e] : 0.0);", "s[e];",
     [pins.test_selection_bias_changes_the_kept_set_not_the_weights]),
    ("selection_bias_in_weights", "        orc_gate_weights(N, K, s, sel, w);\n        for (int64_t j = 0; j < K; ++j) {",
     "        orc_gate_weights(N, K, tmp, sel, w);\n        for (int64_t j = 0; j < K; ++j) {",
     [pins.test_selection_bias_changes_the_kept_set_not_the_weights]),
    ("capacity_floor", "return (int64_t)ceil(cf * (double)T * (double)K / (double)N);",
     "return (int64_t)floor(cf * (double)T * (double)K / (double)N);",
     [pins.test_capacity_closed_forms]),
    ("capacity_off_by_one", "if (load[e] < C) {\n                load[e] += 1;\n                keep",
     "if (load[e] <= C) {\n                load[e] += 1;\n                keep",
     [pins.test_capacity_keeps_the_first_C_of_each_expert_in_row_order]),
    ("dropped_slot_still_added", "if ((keep && !keep[t * K + j]) || e < 0) {", "if (0) {",
     [pins.test_capacity_layer_is_the_masked_dense_gate]),
    ("reroute_to_worst", "if (best < 0 || vt[e] > vt[best]) best = e;", "if (best < 0 || vt[e] < vt[best]) best = e;",
     [pins.test_reroute_worked_examples, pins.test_reroute_equals_deferred_acceptance]),
    ("reroute_takes_held_expert", "if (held[e] || load[e] >= C) continue;", "if (load[e] >= C) continue;",
     [pins.test_reroute_worked_examples, pins.test_reroute_equals_deferred_acceptance]),
    ("reroute_ignores_capacity", "if (held[e] || load[e] >= C) continue;", "if (held[e]) continue;",
     [pins.test_reroute_worked_examples, pins.test_reroute_equals_deferred_acceptance]),
    ("reroute_ties_to_higher_index", "if (best < 0 || vt[e] > vt[best]) best = e;",
     "if (best < 0 || vt[e] >= vt[best]) best = e;",
     [pins.test_reroute_worked_examples, pins.test_reroute_equals_deferred_acceptance]),
    ("reroute_evaluates_selected_expert", "const int32_t e = assign ? assign[t * K + j] : sel[j];",
     "const int32_t e = assign ? (assign[t * K + j] < 0 ? -1 : sel[j]) : sel[j];",
     [pins.test_reroute_layer_against_single_expert_layers]),
    ("gelu_grad_missing_density", "+ v * exp(-0.5 * v * v) / sqrt(2.0 * 3.14159265358979323846);", ";",
     [pins.test_activation_derivatives_closed_forms, pins.test_backward_one_expert_top1_is_dense_ffn_autograd]),
    ("swiglu_grad_gate_up_swapped", "double dg = dh[n] * pre[H + n] * orc_silu_grad(pre[n]);",
     "double dg = dh[n] * pre[n] * orc_silu_grad(pre[H + n]);",
     [pins.test_backward_one_expert_top1_is_dense_ffn_autograd]),
    ("expert_grad_unscaled", "for (int64_t c = 0; c < D; ++c) go[c] = w[t * K + j] * dyr[c];",
     "for (int64_t c = 0; c < D; ++c) go[c] = dyr[c];",
     [pins.test_backward_matches_central_differences]),
    ("softmax_grad_not_centred", "ds[sel[t * K + j]] += w[t * K + j] * (dw[j] - wdw);",
     "ds[sel[t * K + j]] += w[t * K + j] * dw[j];",
     [pins.test_backward_matches_central_differences]),
    ("switch_grad_sign", "ds[e] += alpha_switch * ((double)N / (double)T) * p[e] * (f[e] - fp);",
     "ds[e] -= alpha_switch * ((double)N / (double)T) * p[e] * (f[e] - fp);",
     [pins.test_backward_matches_central_differences]),
    ("p_mean_not_averaged", "for (int64_t e = 0; e < N; ++e) p_mean[e] /= (double)T;",
     "for (int64_t e = 0; e < N; ++e) p_mean[e] /= 1.0;",
     [pins.test_aux_stats_invariants_and_library_checks]),
]


def _call(pin, golden_dir):
    import inspect
    params = inspect.signature(pin).parameters
    if "golden_dir" in params:
        pin(golden_dir)
        return
    marks = getattr(pin, "pytestmark", [])
    cases = [m for m in marks if m.name == "parametrize"]
    if cases:
        names = [n.strip() for n in cases[0].args[0].split(",")]
        for vals in cases[0].args[1]:
            vals = vals if isinstance(vals, tuple) else (vals,)
            pin(**dict(zip(names, vals)))
    else:
        pin()


@pytest.mark.parametrize("name,old,new,catchers", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_planted_mistake_is_caught(name, old, new, catchers, tmp_path, golden_dir, monkeypatch):
    src = open(oracle._SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    mutated = tmp_path / "moe_oracle_mutant.c"
    mutated.write_text(src.replace(old, new))
    so = oracle.compile_source(str(mutated), str(tmp_path / "liboracle_mutant.so"))
    monkeypatch.setattr(oracle, "_lib", oracle.configure(ctypes.CDLL(so)))
    caught = 0
    for pin in catchers:
        try:
            _call(pin, golden_dir)
        except AssertionError:
            caught += 1
    assert caught > 0, f"no pin caught the planted mistake {name}"


def test_unmutated_copy_passes_the_same_pins(tmp_path, golden_dir, monkeypatch):
    so = oracle.compile_source(oracle._SRC, str(tmp_path / "liboracle_copy.so"))
    monkeypatch.setattr(oracle, "_lib", oracle.configure(ctypes.CDLL(so)))
    for _, _, _, catchers in MUTANTS:
        for pin in catchers:
            _call(pin, golden_dir)
