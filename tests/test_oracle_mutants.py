"""Plant plausible mistakes in the CPU oracle and check that the pins catch each one.

Every mutant replaces one oracle function for the duration of a test; the pin
suite in ``test_oracle_pins`` must then fail somewhere.  Nothing here runs on
a GPU.
"""
import numpy as np
import pytest

import oracle.moe_oracle as M
import tests.test_oracle_node_limited as PN
import tests.test_oracle_pins as P

_orig = {name: getattr(M, name) for name in
         ("silu", "softmax_affinity", "sigmoid_affinity", "select_top_k", "gate_values",
          "swiglu_ffn", "affinity_logits", "expert_permutation", "moe_forward", "bias_update",
          "select_top_k_node_limited")}


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


def _node_limited(score_fn=None, interleaved=False, ascending=False, extra=0):
    def f(key, K, n_nodes, lim):
        T, N = key.shape
        per = N // n_nodes
        node_of = np.arange(N) % n_nodes if interleaved else np.arange(N) // per
        score = np.stack([(score_fn or np.max)(key[:, node_of == g], axis=1) for g in range(n_nodes)], axis=1)
        nodes = np.argsort(score if ascending else -score, axis=1, kind="stable")[:, :min(n_nodes, lim + extra)]
        allowed = np.zeros((T, N), dtype=bool)
        for t in range(T):
            allowed[t] = np.isin(node_of, nodes[t])
        return M.select_top_k(np.where(allowed, key, -np.inf), K)
    return f


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
    "node_score_is_sum_of_keys": ("select_top_k_node_limited", _node_limited(score_fn=np.sum)),
    "experts_interleaved_over_nodes": ("select_top_k_node_limited", _node_limited(interleaved=True)),
    "worst_nodes_chosen": ("select_top_k_node_limited", _node_limited(ascending=True)),
    "one_node_too_many": ("select_top_k_node_limited", _node_limited(extra=1)),
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
    PN.test_hand_example,
    lambda: PN.test_matches_the_walk_down_the_experts(2),
    PN.test_properties,
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


# --- the FP8 quantization oracle ------------------------------------------

import oracle.fp8 as F8  # noqa: E402
import tests.test_oracle_fp8 as P8  # noqa: E402

_orig8 = {name: getattr(F8, name) for name in
          ("e4m3_decode", "e4m3_encode", "scale_exponent", "quantize_rows", "qdq_rows", "qdq_blocks",
           "swiglu_ffn_fp8", "quantize_cols")}


def _encode_truncating(v):
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    code = np.searchsorted(F8._POS_VALUES, a, side="right") - 1   # largest value <= a
    return np.where(np.signbit(v), code | 0x80, code).astype(np.uint8)


def _encode_ties_away(v):
    v = np.asarray(v, dtype=np.float64)
    nudged = np.nextafter(np.abs(v), np.inf)                       # a tie now rounds up
    return _orig8["e4m3_encode"](np.where(np.signbit(v), -nudged, nudged).clip(-448, 448))


def _decode_wrong_bias(codes):
    return _orig8["e4m3_decode"](codes) / 2.0


def _scale_exponent_off_at_powers(amax):
    a = np.asarray(amax, dtype=np.float64)
    out = np.empty(a.shape, dtype=np.int64)
    for i, x in np.ndenumerate(a):
        out[i] = -127 if x == 0 else min(max(int(np.frexp(x / 448.0)[1]), -127), 127)
    return out


def _rows_in_column_groups(x):
    return F8.quantize_groups(x, F8.GROUP, 1)


def _qdq_rows_in_column_groups(x):
    return F8.dequantize_groups(*F8.quantize_groups(x, F8.GROUP, 1), F8.GROUP, 1)


def _qdq_weights_row_wise(w):
    w = M.f64(w)
    if w.ndim == 3:
        return np.stack([_qdq_weights_row_wise(m) for m in w])
    return F8.dequantize_groups(*F8.quantize_groups(w, 1, F8.GROUP), 1, F8.GROUP)


def _ffn_h_not_quantized(u, w_gate, w_up, w_down):
    uq = F8.qdq_rows(u)
    h = M.silu(uq @ F8.qdq_blocks(w_gate).T) * (uq @ F8.qdq_blocks(w_up).T)
    return h @ F8.qdq_blocks(w_down).T


def _ffn_u_not_quantized(u, w_gate, w_up, w_down):
    u = M.f64(u)
    h = F8.qdq_rows(M.silu(u @ F8.qdq_blocks(w_gate).T) * (u @ F8.qdq_blocks(w_up).T))
    return h @ F8.qdq_blocks(w_down).T


MUTANTS_FP8 = {
    "e4m3_truncating": ("e4m3_encode", _encode_truncating),
    "e4m3_ties_away_from_zero": ("e4m3_encode", _encode_ties_away),
    "e4m3_wrong_exponent_bias": ("e4m3_decode", _decode_wrong_bias),
    "scale_exponent_off_by_one_at_powers": ("scale_exponent", _scale_exponent_off_at_powers),
    "activation_groups_128x1": ("quantize_rows", _rows_in_column_groups),
    "activation_qdq_128x1": ("qdq_rows", _qdq_rows_in_column_groups),
    "weights_grouped_row_wise": ("qdq_blocks", _qdq_weights_row_wise),
    "h_not_quantized": ("swiglu_ffn_fp8", _ffn_h_not_quantized),
    "input_rows_not_quantized": ("swiglu_ffn_fp8", _ffn_u_not_quantized),
    "backward_groups_1x128": ("quantize_cols", lambda x: F8.quantize_groups(x, 1, F8.GROUP)),
}

PINS_FP8 = [getattr(P8, n) for n in dir(P8) if n.startswith("test_")]


@pytest.mark.parametrize("name", sorted(MUTANTS_FP8))
def test_fp8_pins_catch_mutant(name, monkeypatch):
    fn_name, mutant = MUTANTS_FP8[name]
    monkeypatch.setattr(F8, fn_name, mutant)
    caught = 0
    for pin in PINS_FP8:
        try:
            pin()
        except Exception:
            caught += 1
    assert caught > 0, f"no FP8 pin caught the mutant {name}"


def test_fp8_pins_pass_without_mutant():
    for pin in PINS_FP8:
        pin()


# --- the backward oracle ----------------------------------------------------

import oracle.moe_backward as MBW  # noqa: E402
import tests.test_oracle_backward as PB  # noqa: E402

_origb = {name: getattr(MBW, name) for name in ("silu_grad", "swiglu_ffn_backward", "gate_logit_backward")}


def _silu_grad_sigma_only(a):
    return 1.0 / (1.0 + np.exp(-a))


def _ffn_backward_drops_up_path(u, w_gate, w_up, w_down, dy):
    du, dwg, dwu, dwd = _origb["swiglu_ffn_backward"](u, w_gate, w_up, w_down, dy)
    wg, wu, wd = M.f64(w_gate), M.f64(w_up), M.f64(w_down)
    a = u @ wg.T
    db = (dy @ wd) * M.silu(a)
    return du - db @ wu, dwg, dwu, dwd


def _ffn_backward_gate_up_weight_grads_swapped(u, w_gate, w_up, w_down, dy):
    du, dwg, dwu, dwd = _origb["swiglu_ffn_backward"](u, w_gate, w_up, w_down, dy)
    return du, dwu, dwg, dwd


def _softmax_backward_not_centred(s, idx, gate, dg, gate_kind):
    if gate_kind != M.GATE_SOFTMAX:
        return _origb["gate_logit_backward"](s, idx, gate, dg, gate_kind)
    T, N = s.shape
    ds = np.zeros((T, N))
    np.add.at(ds, (np.repeat(np.arange(T), idx.shape[1]), idx.ravel()), dg.ravel())
    return s * ds


def _sigmoid_backward_not_normalised(s, idx, gate, dg, gate_kind):
    if gate_kind != M.GATE_SIGMOID:
        return _origb["gate_logit_backward"](s, idx, gate, dg, gate_kind)
    s_sel = np.take_along_axis(s, idx, axis=1)
    dz = np.zeros_like(s)
    np.put_along_axis(dz, idx, dg * s_sel * (1.0 - s_sel), axis=1)
    return dz


def _logit_backward_wrong_sign(s, idx, gate, dg, gate_kind):
    return -_origb["gate_logit_backward"](s, idx, gate, dg, gate_kind)


def _ffn_backward_down_grad_without_silu(u, w_gate, w_up, w_down, dy):
    du, dwg, dwu, _ = _origb["swiglu_ffn_backward"](u, w_gate, w_up, w_down, dy)
    a, b = u @ M.f64(w_gate).T, u @ M.f64(w_up).T
    return du, dwg, dwu, dy.T @ (a * b)


def _ffn_backward_drops_gate_path(u, w_gate, w_up, w_down, dy):
    du, dwg, dwu, dwd = _origb["swiglu_ffn_backward"](u, w_gate, w_up, w_down, dy)
    wg, wu, wd = M.f64(w_gate), M.f64(w_up), M.f64(w_down)
    a, b = u @ wg.T, u @ wu.T
    da = (dy @ wd) * b * _origb["silu_grad"](a)
    return du - da @ wg, dwg, dwu, dwd


def _ffn_backward_weight_grads_transposed_inputs(u, w_gate, w_up, w_down, dy):
    """dW_gate from the rows of dy instead of u (the two operands of the outer product mixed up)."""
    du, dwg, dwu, dwd = _origb["swiglu_ffn_backward"](u, w_gate, w_up, w_down, dy)
    wg, wu, wd = M.f64(w_gate), M.f64(w_up), M.f64(w_down)
    a, b = u @ wg.T, u @ wu.T
    da = (dy @ wd) * b * _origb["silu_grad"](a)
    return du, da.T @ dy, dwu, dwd


MUTANTS_BWD = {
    "silu_grad_sigma_only": ("silu_grad", _silu_grad_sigma_only),
    "ffn_backward_drops_up_path": ("swiglu_ffn_backward", _ffn_backward_drops_up_path),
    "gate_up_weight_grads_swapped": ("swiglu_ffn_backward", _ffn_backward_gate_up_weight_grads_swapped),
    "softmax_backward_not_centred": ("gate_logit_backward", _softmax_backward_not_centred),
    "sigmoid_backward_not_normalised": ("gate_logit_backward", _sigmoid_backward_not_normalised),
    "logit_backward_wrong_sign": ("gate_logit_backward", _logit_backward_wrong_sign),
    "down_grad_without_silu": ("swiglu_ffn_backward", _ffn_backward_down_grad_without_silu),
    "ffn_backward_drops_gate_path": ("swiglu_ffn_backward", _ffn_backward_drops_gate_path),
    "gate_weight_grad_from_dy": ("swiglu_ffn_backward", _ffn_backward_weight_grads_transposed_inputs),
}

PINS_BWD = [
    lambda: [PB.test_gradients_match_central_differences(k, s) for k, s in
             ((M.GATE_SOFTMAX, 1), (M.GATE_SIGMOID, 2))],
    lambda: [PB.test_single_elements_match_central_differences(k) for k in (M.GATE_SOFTMAX, M.GATE_SIGMOID)],
    PB.test_softmax_logit_gradients_sum_to_zero,
]


@pytest.mark.parametrize("name", sorted(MUTANTS_BWD))
def test_backward_pins_catch_mutant(name, monkeypatch):
    fn_name, mutant = MUTANTS_BWD[name]
    monkeypatch.setattr(MBW, fn_name, mutant)
    caught = 0
    for pin in PINS_BWD:
        try:
            pin()
        except Exception:
            caught += 1
    assert caught > 0, f"no backward pin caught the mutant {name}"


def test_backward_pins_pass_without_mutant():
    for pin in PINS_BWD:
        pin()
