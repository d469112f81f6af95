"""Pins of the backward oracle (``oracle/moe_backward.py``) to the pinned forward oracle.

The loss L = sum(dh * h) has dL/dh = dh, so every gradient the backward
returns must equal the central finite difference of the forward oracle along
any direction (float64: step 1e-5, agreement to ~1e-8 relative), as long as
the perturbation does not change which experts are chosen (checked).  Plus
invariants: softmax logit gradients sum to zero over the experts; a uniform
shift of the selection bias changes nothing; the gradients are linear in dh.
"""
import numpy as np
import pytest

import oracle.moe_backward as MB
import oracle.moe_oracle as M

EPS = 1e-5
RTOL = 1e-6


def _layer(gate_kind, seed, T=12, d=32, N=6, I=16, K=2, Ks=2, Is=8):
    rng = np.random.default_rng(seed)
    p = {
        "u": rng.standard_normal((T, d)),
        "router_w": rng.standard_normal((N, d)) * 0.3,
        "logit_bias": rng.standard_normal(N) * 0.5,
        "w_gate": rng.standard_normal((N, I, d)) * 0.2,
        "w_up": rng.standard_normal((N, I, d)) * 0.2,
        "w_down": rng.standard_normal((N, d, I)) * 0.2,
        "ws_gate": rng.standard_normal((Ks, Is, d)) * 0.2,
        "ws_up": rng.standard_normal((Ks, Is, d)) * 0.2,
        "ws_down": rng.standard_normal((Ks, d, Is)) * 0.2,
    }
    sb = rng.uniform(-0.1, 0.1, N) if gate_kind == M.GATE_SIGMOID else None
    dh = rng.standard_normal((T, d))
    return p, sb, dh, K


def _forward(p, K, gate_kind, sb):
    h, r = M.moe_forward(p["u"], p["router_w"], K, (p["w_gate"], p["w_up"], p["w_down"]),
                         (p["ws_gate"], p["ws_up"], p["ws_down"]), gate_kind=gate_kind,
                         logit_bias=p["logit_bias"], select_bias=sb)
    return h, r.idx


def _grads(p, K, gate_kind, sb, dh):
    g = MB.moe_backward(p["u"], p["router_w"], K, (p["w_gate"], p["w_up"], p["w_down"]),
                        (p["ws_gate"], p["ws_up"], p["ws_down"]), dh, gate_kind=gate_kind,
                        logit_bias=p["logit_bias"], select_bias=sb)
    return {"u": g.du, "router_w": g.d_router, "logit_bias": g.d_logit_bias, "w_gate": g.d_w_gate,
            "w_up": g.d_w_up, "w_down": g.d_w_down, "ws_gate": g.d_ws_gate, "ws_up": g.d_ws_up,
            "ws_down": g.d_ws_down}


def _directional_fd(p, name, v, K, gate_kind, sb, dh):
    idx0 = _forward(p, K, gate_kind, sb)[1]
    vals = []
    for sign in (1, -1):
        q = dict(p)
        q[name] = p[name] + sign * EPS * v
        h, idx = _forward(q, K, gate_kind, sb)
        assert np.array_equal(idx, idx0), "the perturbation changed the choice of experts"
        vals.append((dh * h).sum())
    return (vals[0] - vals[1]) / (2 * EPS)


@pytest.mark.parametrize("gate_kind,seed", [(M.GATE_SOFTMAX, 1), (M.GATE_SIGMOID, 2), (M.GATE_SOFTMAX, 3)])
def test_gradients_match_central_differences(gate_kind, seed):
    p, sb, dh, K = _layer(gate_kind, seed)
    g = _grads(p, K, gate_kind, sb, dh)
    rng = np.random.default_rng(100 + seed)
    for name in p:
        for _ in range(2):
            v = rng.standard_normal(p[name].shape)
            fd = _directional_fd(p, name, v, K, gate_kind, sb, dh)
            an = (g[name] * v).sum()
            assert abs(fd - an) <= RTOL * max(1.0, abs(an)), (name, fd, an)


@pytest.mark.parametrize("gate_kind", [M.GATE_SOFTMAX, M.GATE_SIGMOID])
def test_single_elements_match_central_differences(gate_kind):
    """One-hot directions: catches a gradient that is right in sum but in the wrong place."""
    p, sb, dh, K = _layer(gate_kind, 4)
    g = _grads(p, K, gate_kind, sb, dh)
    rng = np.random.default_rng(5)
    for name in p:
        for _ in range(4):
            at = tuple(int(rng.integers(0, n)) for n in p[name].shape)
            v = np.zeros(p[name].shape)
            v[at] = 1.0
            fd = _directional_fd(p, name, v, K, gate_kind, sb, dh)
            assert abs(fd - g[name][at]) <= RTOL * max(1.0, abs(fd)), (name, at, fd, g[name][at])


def test_all_experts_active():
    """K = mN: every gate is live; the softmax gates sum to 1, so a uniform logit shift is inert."""
    p, sb, dh, K = _layer(M.GATE_SOFTMAX, 6, N=4, K=4)
    g = _grads(p, K, M.GATE_SOFTMAX, sb, dh)
    rng = np.random.default_rng(7)
    for name in ("router_w", "logit_bias", "w_down", "u"):
        v = rng.standard_normal(p[name].shape)
        fd = _directional_fd(p, name, v, K, M.GATE_SOFTMAX, sb, dh)
        assert abs(fd - (g[name] * v).sum()) <= RTOL * max(1.0, abs(fd))
    assert abs(g["logit_bias"].sum()) < 1e-12


def test_softmax_logit_gradients_sum_to_zero():
    p, sb, dh, K = _layer(M.GATE_SOFTMAX, 8)
    g = _grads(p, K, M.GATE_SOFTMAX, sb, dh)
    assert abs(g["logit_bias"].sum()) < 1e-12
    assert np.allclose(g["router_w"].sum(axis=0), 0.0, atol=1e-12)


def test_uniform_selection_bias_shift_changes_nothing():
    p, sb, dh, K = _layer(M.GATE_SIGMOID, 9)
    a = _grads(p, K, M.GATE_SIGMOID, sb, dh)
    b = _grads(p, K, M.GATE_SIGMOID, sb + 0.37, dh)
    for k in a:
        assert np.array_equal(a[k], b[k]), k


def test_gradients_are_linear_in_dh_and_zero_for_zero_dh():
    p, sb, dh, K = _layer(M.GATE_SIGMOID, 10)
    dh2 = np.random.default_rng(11).standard_normal(dh.shape)
    a, b = _grads(p, K, M.GATE_SIGMOID, sb, dh), _grads(p, K, M.GATE_SIGMOID, sb, dh2)
    c = _grads(p, K, M.GATE_SIGMOID, sb, dh + 2 * dh2)
    z = _grads(p, K, M.GATE_SIGMOID, sb, np.zeros_like(dh))
    for k in a:
        assert np.allclose(c[k], a[k] + 2 * b[k], rtol=1e-12, atol=1e-12), k
        assert not np.any(z[k]), k


def test_residual_only_layer_passes_dh_through():
    """With every expert weight zero the output is h = u: du = dh and every other gradient
    except the experts' own is zero."""
    p, sb, dh, K = _layer(M.GATE_SOFTMAX, 12)
    for k in ("w_gate", "w_up", "w_down", "ws_gate", "ws_up", "ws_down"):
        p[k] = np.zeros_like(p[k])
    g = _grads(p, K, M.GATE_SOFTMAX, sb, dh)
    assert np.array_equal(g["u"], dh)
    assert not np.any(g["router_w"]) and not np.any(g["logit_bias"])
