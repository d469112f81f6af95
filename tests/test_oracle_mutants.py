"""Plant plausible mistakes in the CPU oracle and check that the pins catch each one.

Every mutant replaces one oracle function for the duration of a test; the pin
suite in ``test_oracle_pins`` must then fail somewhere.  Nothing here runs on
a GPU.
"""
import numpy as np
import pytest

import oracle.moe_oracle as M
import tests.test_oracle_pins as P

_orig = {name: getattr(M, name) for name in
         ("silu", "softmax_affinity", "sigmoid_affinity", "select_top_k", "gate_values",
          "swiglu_ffn", "affinity_logits", "expert_permutation", "moe_forward", "bias_update")}


def _silu_wrong_sign(a):
    return a / (1.0 + np.exp(a))


def _softmax_no_shift_renorm_topk(z):
    s = _orig["softmax_affinity"](z)
    return s / s.max(axis=1, keepdims=True)


def _top_k_ties_to_higher_index(key, K):
    N = key.shape[1]
    order = np.argsort(-key[:, ::-1], axis=1, kind="stable")
    return (N - 1 - order[:, :K]).astype(np.int64)


def _top_k_ascending(key, K):
    return _orig["select_top_k"](key, K)[:, ::-1].copy()


def _gates_renormalised_softmax(s, idx, gate_kind):
    g = np.take_along_axis(s, idx, axis=1)
    return g / g.sum(axis=1, keepdims=True)


def _gates_sigmoid_not_renormalised(s, idx, gate_kind):
    return np.take_along_axis(s, idx, axis=1)


def _ffn_transposed_down(u, w_gate, w_up, w_down):
    wg, wu, wd = M.f64(w_gate), M.f64(w_up), M.f64(w_down)
    mid = M.silu(u @ wg.T) * (u @ wu.T)
    wdt = wd.reshape(wd.shape[1], wd.shape[0])   # wrong: reinterprets [d, I] as [I, d]
    return mid @ wdt


def _ffn_gate_up_swapped(u, w_gate, w_up, w_down):
    return _orig["swiglu_ffn"](u, w_up, w_gate, w_down)


def _logits_bias_dropped(u, e, logit_bias=None):
    return _orig["affinity_logits"](u, e, None)


def _permutation_descending(idx, N):
    p = _orig["expert_permutation"](idx, N)
    src = p.src.copy()
    for i in range(N):
        a, b = p.offsets[i], p.offsets[i + 1]
        src[a:b] = src[a:b][::-1]
    p.src = src
    return p


def _forward_drops_residual(u, router_w, K, experts, shared=None, **kw):
    kw["flags"] = kw.get("flags", 0) | M.FLAG_NO_RESIDUAL
    return _orig["moe_forward"](u, router_w, K, experts, shared, **kw)


def _forward_drops_shared(u, router_w, K, experts, shared=None, **kw):
    return _orig["moe_forward"](u, router_w, K, experts, None, **kw)


def _bias_update_wrong_sign(bias, counts, gamma):
    return _orig["bias_update"](bias, counts, -gamma)


MUTANTS = {
    "silu_wrong_sign": ("silu", _silu_wrong_sign),
    "softmax_wrong_normaliser": ("softmax_affinity", _softmax_no_shift_renorm_topk),
    "ties_to_higher_index": ("select_top_k", _top_k_ties_to_higher_index),
    "selection_ascending": ("select_top_k", _top_k_ascending),
    "softmax_gates_renormalised": ("gate_values", _gates_renormalised_softmax),
    "sigmoid_gates_not_renormalised": ("gate_values", _gates_sigmoid_not_renormalised),
    "w_down_transposed": ("swiglu_ffn", _ffn_transposed_down),
    "gate_and_up_swapped": ("swiglu_ffn", _ffn_gate_up_swapped),
    "logit_bias_dropped": ("affinity_logits", _logits_bias_dropped),
    "permutation_not_stable": ("expert_permutation", _permutation_descending),
    "residual_dropped": ("moe_forward", _forward_drops_residual),
    "shared_dropped": ("moe_forward", _forward_drops_shared),
    "bias_update_wrong_sign": ("bias_update", _bias_update_wrong_sign),
}

PINS = [
    lambda: [P.test_closed_form_tiny_layer(c) for c in
             ("softmax", "softmax_logit_bias", "sigmoid", "sigmoid_select_bias")],
    P.test_closed_form_components_by_flag,
    P.test_softmax_matches_library_and_sums_to_one,
    P.test_sigmoid_and_silu_match_library,
    P.test_ffn_one_hot_weights_place_the_product_in_the_right_component,
    lambda: P.test_top_k_equals_brute_force_with_forced_ties(0),
    P.test_selection_bias_moves_selection_but_not_gates,
    P.test_softmax_gates_are_not_renormalised,
    lambda: P.test_fine_grained_split_identity("softmax", 2),
    P.test_dense_counterpart_when_all_experts_active,
    lambda: P.test_gshard_reduction_matches_brute_force(0),
    lambda: P.test_permutation_matches_sorted_pairs(7, 3),
    P.test_bias_update_hand_example,
    P.test_bias_update_balances_a_skewed_router,
]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, monkeypatch):
    fn_name, mutant = MUTANTS[name]
    monkeypatch.setattr(M, fn_name, mutant)
    # the package namespace re-exports the functions the tests call
    import oracle
    if hasattr(oracle, fn_name):
        monkeypatch.setattr(oracle, fn_name, mutant)
    caught = 0
    for pin in PINS:
        try:
            pin()
        except Exception:  # an assertion or a shape error both count as caught
            caught += 1
    assert caught > 0, f"no pin caught the mutant {name}"


def test_pins_pass_without_mutant():
    for pin in PINS:
        pin()
