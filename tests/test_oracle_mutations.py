"""Plant plausible mistakes in the oracle (CPU only) and check that the pins fail.

Each mutant replaces one oracle function with a subtly wrong version; at least
one pin in ``test_oracle_pins`` must then raise. This shows the pins are
sensitive to the mistakes they are meant to catch.
"""
import math

import numpy as np
import pytest
from scipy.special import erf

import oracle
import oracle.moe_oracle as om
import test_oracle_pins as pins

_orig = {n: getattr(om, n) for n in ("select_topk", "dispatch", "gelu_erf", "gini_exact",
                                      "capacity", "load_stats", "expert_ffn", "selection_scores",
                                      "moe_layer_forward", "bias_update", "expert_offsets",
                                      "combine")}


def _topk_high_index_ties(logits, bias, K, noise=None):
    s = om.selection_scores(logits, bias, noise)
    order = np.argsort(-s.astype(np.float64)[:, ::-1], axis=1, kind="stable")
    idx = (s.shape[1] - 1 - order[:, :K]).astype(np.int32)
    ss = np.take_along_axis(s, idx, 1).astype(np.float64)
    z = np.exp(ss - ss[:, :1])
    return idx, z / z.sum(1, keepdims=True), s


def _topk_no_renorm(logits, bias, K, noise=None):
    idx, _, s = _orig["select_topk"](logits, bias, K, noise)
    s64 = s.astype(np.float64)
    p = np.exp(s64 - s64.max(1, keepdims=True))
    p /= p.sum(1, keepdims=True)
    return idx, np.take_along_axis(p, idx, 1), s


def _scores_ignore_bias(logits, bias, noise=None):
    return _orig["selection_scores"](logits, None, noise)


def _scores_fp64(logits, bias, noise=None):
    b = 0.0 if bias is None else np.asarray(bias, np.float64)[None, :]
    g = 0.0 if noise is None else np.asarray(noise, np.float64)
    return np.asarray(logits, np.float64) + b + g


def _scores_ignore_noise(logits, bias, noise=None):
    return _orig["selection_scores"](logits, bias, None)


def _topk_weights_from_clean_scores(logits, bias, K, noise=None):
    idx, _, s = _orig["select_topk"](logits, bias, K, noise)
    clean = _orig["selection_scores"](logits, bias, None).astype(np.float64)
    sel = np.take_along_axis(clean, idx, 1)
    z = np.exp(sel - sel.max(1, keepdims=True))
    return idx, z / z.sum(1, keepdims=True), s


def _dispatch_descending(idx, E):
    counts, off, perm, inv = _orig["dispatch"](idx, E)
    for e in range(E):
        perm[off[e]:off[e + 1]] = perm[off[e]:off[e + 1]][::-1]
    inv[perm] = np.arange(perm.size, dtype=np.int32)
    return counts, off, perm, inv


def _gelu_tanh(z):
    z = np.asarray(z, np.float64)
    return 0.5 * z * (1 + np.tanh(math.sqrt(2 / math.pi) * (z + 0.044715 * z ** 3)))


def _gelu_wrong_scale(z):
    z = np.asarray(z, np.float64)
    return 0.5 * z * (1 + erf(z))


def _gini_zero_based(counts):
    c = np.sort(np.asarray(counts, np.int64))
    n, S = c.size, int(c.sum())
    if S == 0:
        return 0.0
    return float(2 * int(np.sum(np.arange(n) * c)) - (n + 1) * S) / float(n * S)


def _capacity_ceil(T, K, E, cf_num=5, cf_den=4):
    return -((-T * K * cf_num) // (E * cf_den))


def _ffn_no_gelu(rows, w1, w2):
    rows = np.asarray(rows, np.float64)
    return (rows @ np.asarray(w1, np.float64).T) @ np.asarray(w2, np.float64).T


def _ffn_transposed_second(rows, w1, w2):
    rows = np.asarray(rows, np.float64)
    h = om.gelu_erf(rows @ np.asarray(w1, np.float64).T)
    w2 = np.asarray(w2, np.float64)
    if w2.shape[0] == w2.shape[1]:
        return h @ w2
    return h @ w2.T * 1.0001


def _layer_no_shared(x, w_router, bias, w1, w2, ws1, ws2, K, tokens=None, noise=None,
                     logits=None):
    return _orig["moe_layer_forward"](x, w_router, bias, w1, w2, None, None, K, tokens, noise,
                                      logits)


def _layer_ignores_given_logits(x, w_router, bias, w1, w2, ws1, ws2, K, tokens=None, noise=None,
                                logits=None):
    return _orig["moe_layer_forward"](x, w_router, bias, w1, w2, ws1, ws2, K, tokens, noise)


def _stats_overflow_counts_experts(counts, T, K, cf_num=5, cf_den=4):
    st = _orig["load_stats"](counts, T, K, cf_num, cf_den)
    st["overflow"] = st["num_stragglers"]
    return st


def _bias_sign_flipped(bias, counts, T, K, gamma, cf_num=5, cf_den=4):
    return _orig["bias_update"](bias, counts, T, K, -gamma, cf_num, cf_den)


def _bias_overload_at_capacity(bias, counts, T, K, gamma, cf_num=5, cf_den=4):
    b = np.asarray(bias, np.float32).copy()
    c = np.asarray(counts, np.int64)
    cap = om.capacity(T, K, c.size, cf_num, cf_den)
    g = np.float32(gamma)
    b[c >= cap] -= g
    b[c == 0] += g
    return b


def _bias_idle_untouched(bias, counts, T, K, gamma, cf_num=5, cf_den=4):
    b = np.asarray(bias, np.float32).copy()
    c = np.asarray(counts, np.int64)
    b[c > om.capacity(T, K, c.size, cf_num, cf_den)] -= np.float32(gamma)
    return b


def _offsets_inclusive(counts):
    c = np.asarray(counts, np.int64)
    return np.concatenate([np.cumsum(c), [c.sum()]]).astype(np.int32)


def _combine_unweighted(y_rows, w, inv, y_shared=None):
    return _orig["combine"](y_rows, np.ones_like(np.asarray(w, np.float64)), inv, y_shared)


def _stats_skew_without_epsilon(counts, T, K, cf_num=5, cf_den=4):
    st = _orig["load_stats"](counts, T, K, cf_num, cf_den)
    mn = int(np.min(counts))
    st["skew_ratio"] = float(np.max(counts)) / mn if mn else math.inf
    return st


def _stats_max_over_mean_of_min(counts, T, K, cf_num=5, cf_den=4):
    st = _orig["load_stats"](counts, T, K, cf_num, cf_den)
    c = np.asarray(counts, np.int64)
    st["max_over_mean"] = float(c.min()) * c.size / (T * K) if T * K else 0.0
    return st


MUTANTS = {
    "ties_to_higher_index": ("select_topk", _topk_high_index_ties),
    "weights_not_renormalised": ("select_topk", _topk_no_renorm),
    "bias_ignored": ("selection_scores", _scores_ignore_bias),
    "decision_in_fp64": ("selection_scores", _scores_fp64),
    "dispatch_descending_tokens": ("dispatch", _dispatch_descending),
    "gelu_tanh_approximation": ("gelu_erf", _gelu_tanh),
    "gelu_missing_sqrt2": ("gelu_erf", _gelu_wrong_scale),
    "gini_zero_based_rank": ("gini_exact", _gini_zero_based),
    "capacity_rounded_up": ("capacity", _capacity_ceil),
    "ffn_without_gelu": ("expert_ffn", _ffn_no_gelu),
    "ffn_second_linear_transposed": ("expert_ffn", _ffn_transposed_second),
    "shared_expert_dropped": ("moe_layer_forward", _layer_no_shared),
    "given_logits_ignored": ("moe_layer_forward", _layer_ignores_given_logits),
    "overflow_counts_experts": ("load_stats", _stats_overflow_counts_experts),
    "gumbel_noise_ignored": ("selection_scores", _scores_ignore_noise),
    "noisy_weights_from_clean_scores": ("select_topk", _topk_weights_from_clean_scores),
    "bias_update_sign_flipped": ("bias_update", _bias_sign_flipped),
    "bias_update_overload_at_capacity": ("bias_update", _bias_overload_at_capacity),
    "bias_update_idle_untouched": ("bias_update", _bias_idle_untouched),
    "offsets_inclusive": ("expert_offsets", _offsets_inclusive),
    "combine_unweighted": ("combine", _combine_unweighted),
    "skew_without_epsilon": ("load_stats", _stats_skew_without_epsilon),
    "max_over_mean_of_min": ("load_stats", _stats_max_over_mean_of_min),
}

PIN_TESTS = [
    lambda: [pins.test_topk_matches_brute_force_enumeration(s) for s in range(6)],
    pins.test_selection_is_decided_in_fp32,
    pins.test_negative_and_positive_zero_tie_to_lower_index,
    pins.test_K_equals_E_gives_full_softmax,
    pins.test_weights_sum_to_one_and_ratio_is_exp_gap,
    pins.test_router_matches_page_pipeline_in_torch_fp64,
    lambda: pins.test_dispatch_invariants_and_brute_force(37, 8, 2),
    pins.test_gelu_closed_forms_and_torch,
    pins.test_E1_K1_reduces_to_dense_ffn,
    lambda: pins.test_identical_experts_give_single_ffn_for_any_routing(2),
    pins.test_K1_is_an_identity_scatter_of_the_chosen_expert,
    pins.test_layer_sum_over_k_matches_explicit_per_token_loop,
    pins.test_given_logits_decide_the_routing,
    pins.test_gini_golden_cases,
    pins.test_gini_matches_mean_absolute_difference_form,
    pins.test_load_stats_golden_cases,
    pins.test_capacity_integer_form_equals_page_float_form,
    pins.test_gumbel_max_picks_each_expert_with_its_softmax_probability,
    pins.test_noisy_weights_are_the_softmax_of_the_noisy_scores,
    pins.test_combine_worked_example,
    pins.test_max_over_mean_closed_forms,
    pins.test_stagewise_grouped_ffn_and_combine_equal_layer_definition,
    pins.test_bias_update_moves_only_overloaded_and_idle_experts,
    pins.test_bias_update_is_a_fixed_point_for_an_even_load,
    pins.test_repeated_bias_updates_even_out_a_skewed_router,
]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, monkeypatch):
    fn_name, mutant = MUTANTS[name]
    monkeypatch.setattr(om, fn_name, mutant)
    monkeypatch.setattr(oracle, fn_name, mutant)
    failures = 0
    for t in PIN_TESTS:
        try:
            t()
        except (AssertionError, ValueError, IndexError):
            failures += 1
    assert failures >= 1, f"no pin caught mutant {name}"


def test_unmutated_oracle_passes_every_pin():
    for t in PIN_TESTS:
        t()
