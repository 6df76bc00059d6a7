"""The pins catch plausible mistakes: each case plants one mistake in a temporary
copy of the oracle's C source (on the CPU), builds it, points the oracle module at
it and checks that the named pin tests now fail. CPU only.
"""
import os
import subprocess

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "spa_oracle.c")


def dense_causal_at_p_one():
    pins.test_top_p_one_equals_dense_causal_attention(70, 16)

# (name, text to replace, replacement, pins that must fail)
MUTATIONS = [
    ("dropped_half_in_variance_term", "log1p(0.5 * scale * scale * quad)",
     "log1p(scale * scale * quad)",
     [pins.test_score_hand_worked_examples, pins.test_score_error_is_third_order_in_query_norm]),
    ("dropped_scale_squared", "log1p(0.5 * scale * scale * quad)", "log1p(0.5 * quad)",
     [pins.test_score_error_is_third_order_in_query_norm]),
    ("std_instead_of_variance", "lrow[j] = scale * dot", "quad = sqrt(quad); lrow[j] = scale * dot",
     [pins.test_score_error_is_third_order_in_query_norm]),
    ("dropped_block_count", " + log((double)nj);", ";",
     [pins.test_score_exact_when_block_keys_identical, pins.test_score_hand_worked_examples]),
    ("sample_variance", "vr[c] = s / n;", "vr[c] = s / (n > 1 ? n - 1 : 1);",
     [pins.test_stats_match_numpy_mean_and_population_variance, pins.test_stats_two_key_closed_form]),
    ("mean_divides_by_block", "mu[c] = s / n;", "mu[c] = s / block;",
     [pins.test_stats_match_numpy_mean_and_population_variance]),
    ("sum_pooled_query", "qbar[c] = s / nr;", "qbar[c] = s;",
     [pins.test_score_hand_worked_examples]),
    ("wrong_gqa_group_in_scores", "g = h / G;\n            const int r0", "g = h % Hkv;\n            const int r0",
     [pins.test_score_gqa_head_reads_its_group]),
    ("strict_causal_mask", "if (!(u <= pos && kept[u / block]))", "if (!(u < pos && kept[u / block]))",
     [pins.test_attention_hand_worked_example, pins.test_attention_constant_keys_average_allowed_values]),
    ("dropped_softmax_scale", "z[u] = scale * s;", "z[u] = s;",
     [dense_causal_at_p_one]),
    ("ties_prefer_larger_index", "return (x->j > y->j) - (x->j < y->j);",
     "return (x->j < y->j) - (x->j > y->j);",
     [pins.test_top_p_hand_worked_examples, pins.test_top_p_equal_scores_prefer_smaller_index]),
    ("crossing_block_dropped", "cum += exp((double)cand[k].key - mx);\n                ++nk;",
     "cum += exp((double)cand[k].key - mx);\n                if (cum / total < top_p) ++nk;",
     [pins.test_top_p_hand_worked_examples]),
    ("local_window_too_wide", "(j > jmax - n_local)", "(j >= jmax - n_local)",
     [pins.test_top_p_hand_worked_examples]),
    ("rla_sums_kept_blocks", "if (kept[u / block]) continue;", "if (!kept[u / block]) continue;",
     [pins.test_rla_hand_worked_examples, pins.test_rla_is_zero_when_every_causal_block_is_kept,
      pins.test_rla_global_minus_kept_equals_residual]),
    ("rla_strict_causal", "for (int u = 0; u <= pos; ++u) {\n                if (kept",
     "for (int u = 0; u < pos; ++u) {\n                if (kept",
     [pins.test_rla_hand_worked_examples, pins.test_rla_global_minus_kept_equals_residual]),
    ("rla_linear_kernel_feature_map", "a += phq[c] * exp(elem(k, is_bf16, (kvbase + u) * d + c));",
     "a += log(phq[c]) * elem(k, is_bf16, (kvbase + u) * d + c);",
     [pins.test_rla_hand_worked_examples, pins.test_rla_query_shift_scales_output,
      pins.test_rla_unit_features_sum_residual_values]),
    ("rla_states_transposed", "w[(size_t)e * d + c] += ve * exp(", "w[(size_t)c * d + e] += ve * exp(",
     [pins.test_rla_block_states_contract_to_residual_output]),
    ("rla_magnitude_without_abs", "m[c] += a * fabs(vu);", "m[c] += a * vu;",
     [pins.test_rla_hand_worked_examples]),
    ("quant_round_half_away", "double q1 = nearbyint(ldexp(xm[c], -k1));",
     "double q1 = round(ldexp(xm[c], -k1));",
     [pins.test_quantized_stats_hand_worked_group]),
    ("quant_scale_one_step_coarse", "const int k1 = qexp(am, 7.0), k2 = qexp(av, 15.0);",
     "const int k1 = qexp(am, 7.0) + 1, k2 = qexp(av, 15.0);",
     [pins.test_quantized_stats_hand_worked_group, pins.test_quantized_stats_error_and_scale_bounds,
      pins.test_quantized_stats_on_the_grid_round_trip_exactly]),
    ("quant_variance_signed_range", "qexp(av, 15.0)", "qexp(av, 7.0)",
     [pins.test_quantized_stats_hand_worked_group, pins.test_quantized_stats_error_and_scale_bounds]),
    ("fp4_ties_away_from_zero", "if (di < db || (di == db && (i & 1) == 0)) best = i;",
     "if (di <= db) best = i;",
     [pins.test_fp4_stats_hand_worked_group, pins.test_fp4_codes_are_the_nearest_e2m1_values]),
    ("fp4_ties_toward_zero", "if (di < db || (di == db && (i & 1) == 0)) best = i;",
     "if (di < db) best = i;",
     [pins.test_fp4_stats_hand_worked_group, pins.test_fp4_codes_are_the_nearest_e2m1_values]),
    ("fp4_sign_dropped", "return (uint8_t)(best | (signbit(y) ? 8 : 0));", "return (uint8_t)best;",
     [pins.test_fp4_stats_hand_worked_group, pins.test_fp4_error_and_scale_bounds,
      pins.test_fp4_on_the_grid_round_trip_exactly]),
    ("fp4_scale_clips_like_a_floor_exponent", "const int k1 = qexp(am, 6.0), k2 = qexp(av, 6.0);",
     "const int k1 = qexp(am, 4.0), k2 = qexp(av, 6.0);",
     [pins.test_fp4_stats_hand_worked_group, pins.test_fp4_error_and_scale_bounds,
      pins.test_fp4_on_the_grid_round_trip_exactly]),
    ("fp4_variance_with_the_mean_scale", "cv[base + c] = e2m1_code(ldexp(xv[c], -k2));",
     "cv[base + c] = e2m1_code(ldexp(xv[c], -k1));",
     [pins.test_fp4_stats_hand_worked_group, pins.test_fp4_error_and_scale_bounds]),
    ("fp4_table_three_as_two_and_a_half", "{0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0}",
     "{0.0, 0.5, 1.0, 1.5, 2.0, 2.5, 4.0, 6.0}",
     [pins.test_fp4_codes_decode_to_the_e2m1_values, pins.test_fp4_codes_are_the_nearest_e2m1_values]),
    ("fp4_dequantised_without_sign", "const double m = kE2M1[cm[x] & 7] * ((cm[x] & 8) ? -1.0 : 1.0);",
     "const double m = kE2M1[cm[x] & 7];",
     [pins.test_fp4_codes_decode_to_the_e2m1_values, pins.test_fp4_on_the_grid_round_trip_exactly]),
    ("early_stop_on_reserved_blocks", "if (!reserved && R < tau) {", "if (R < tau) {",
     [pins.test_early_stop_limits_of_tau]),
    ("early_stop_drops_the_stopping_block", "done = n + 1;", "done = n;",
     [pins.test_early_stop_constant_keys_closed_form, pins.test_early_stop_limits_of_tau]),
    ("early_stop_ratio_before_accumulating",
     "acc[r] += gsum;\n                    const double ratio = acc[r] > 0.0 ? gsum / acc[r] : 0.0;",
     "const double ratio = acc[r] > 0.0 ? gsum / acc[r] : 0.0;\n                    acc[r] += gsum;",
     [pins.test_early_stop_ratio_is_gain_over_accumulated_mass,
      pins.test_early_stop_constant_keys_closed_form]),
    ("segperm_ascending_importance", "if (x->score > y->score) return -1;\n    if (x->score < y->score) return 1;",
     "if (x->score < y->score) return -1;\n    if (x->score > y->score) return 1;",
     [pins.test_segperm_hand_worked_permutation,
      pins.test_segperm_importance_sums_to_one_and_sorts_each_segment]),
    ("segperm_pooled_over_the_first_block", "const int r0 = (nq - 1) * block, nr = L - r0;",
     "const int r0 = 0, nr = block < L ? block : L;",
     [pins.test_segperm_hand_worked_permutation,
      pins.test_segperm_importance_at_vanishing_scale_is_uniform_causal,
      pins.test_segperm_importance_reads_only_its_groups_last_block]),
    ("segperm_logit_proxy", "acc[u] += z[u] / den;", "acc[u] += log(z[u]);",
     [pins.test_segperm_hand_worked_permutation,
      pins.test_segperm_importance_sums_to_one_and_sorts_each_segment]),
    ("segperm_unnormalised_rows", "acc[u] += z[u] / den;", "acc[u] += z[u];",
     [pins.test_segperm_hand_worked_permutation,
      pins.test_segperm_importance_sums_to_one_and_sorts_each_segment]),
    ("segperm_rows_see_later_keys", "const int n_seen = t + 1;", "const int n_seen = L;",
     [pins.test_segperm_hand_worked_permutation,
      pins.test_segperm_importance_at_vanishing_scale_is_uniform_causal]),
    ("segperm_dropped_scale", "z[u] = s * scale;    /* the attention's logit */", "z[u] = s;",
     [pins.test_segperm_importance_at_vanishing_scale_is_uniform_causal]),
    ("segperm_heads_of_another_group", "(((size_t)b * Hq + g * G + hh) * L + t) * d",
     "(((size_t)b * Hq + hh) * L + t) * d",
     [pins.test_segperm_importance_reads_only_its_groups_last_block]),
    ("segperm_earlier_keys_by_original_block", "kept[inv[u] / block]", "kept[u / block]",
     [pins.test_segperm_attention_in_the_permuted_layout]),
    ("ascending_sort", "if (x->key > y->key) return -1;\n    if (x->key < y->key) return 1;",
     "if (x->key < y->key) return -1;\n    if (x->key > y->key) return 1;",
     [pins.test_top_p_hand_worked_examples, pins.test_top_p_tiny_p_keeps_top_one]),
]


@pytest.fixture(scope="module")
def workdir(tmp_path_factory):
    return tmp_path_factory.mktemp("oracle_mutants")


@pytest.mark.parametrize("name,old,new,must_fail", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_planted_mistake(name, old, new, must_fail, workdir):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    mutant_c = os.path.join(workdir, f"{name}.c")
    mutant_so = os.path.join(workdir, f"{name}.so")
    with open(mutant_c, "w") as f:
        f.write(src.replace(old, new))
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
                    "-w", mutant_c, "-o", mutant_so, "-lm"], check=True)
    oracle.use_library(mutant_so)
    try:
        caught = []
        for test in must_fail:
            try:
                test()
            except (AssertionError, RuntimeError):
                caught.append(test.__name__)
        assert caught, f"no pin caught mutation {name}"
        assert len(caught) == len(must_fail), f"{name}: only {caught} failed"
    finally:
        oracle.use_library(None)
