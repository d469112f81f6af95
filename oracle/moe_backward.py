"""CPU oracle of the DeepSeekMoE layer's backward pass.  TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` may import this
module.  The GPU path never calls it and shares no code with it.

What it computes
----------------
The pages train the layer (DeepSeek-V3 technical report summary, section
3.2.1 "DualPipe and Computation-Communication Overlap", names the MLP's
backward-for-input and backward-for-weights as separate pieces of a training
step) but print no backward formula.  The backward is the gradient of the
forward of ``moe_oracle`` (steps 1-7 there) with respect to its inputs and
parameters, for an upstream gradient dh = dL/dh of the output.  Readings:

B1  the top-K choice is piecewise constant in its inputs, so the gradient
    flows through the gate values of the chosen experts and not through the
    choice itself; the V3 selection bias b only moves the choice and gets no
    gradient.
B2  the logit bias c is differentiated like a parameter (dc = sum over tokens
    of dz); the router weights e get dE = dz^T u.
B3  float64 throughout, on the bf16 values of the inputs.

Per expert FFN(u) = W_down m, m = SiLU(a) * b, a = W_gate u, b = W_up u, for
one token's row and its gate g (1 for a shared expert), the chain rule gives,
with dy = g dh:
    dW_down += dy m^T,   dm = W_down^T dy,
    db = dm * SiLU(a),   da = dm * b * SiLU'(a),
    SiLU'(a) = sigma(a) (1 + a (1 - sigma(a))),
    dW_gate += da u^T,   dW_up += db u^T,   du += W_gate^T da + W_up^T db,
and dg = dh . FFN(u) for a routed expert.  The residual adds dh to du.
Gates to logits:
    softmax (g = s_i of the chosen i):  ds_i = sum of dg over the slots that
        chose i (0 elsewhere); dz = s * (ds - sum_j s_j ds_j) over all mN.
    sigmoid (g_k = s_k / S, S = sum of the chosen s):  ds_k = (dg_k -
        sum_l g_l dg_l) / S on the chosen experts; dz = ds * s (1 - s).
    du += dz E.

Parity pins (``tests/test_oracle_backward.py``): central finite differences
of the pinned forward oracle along random directions, for every input and
parameter, in both gate modes; invariants (softmax logit gradients sum to
zero per token; the selection bias has no influence on the gradient other
than through the choice).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import numpy as np

from . import moe_oracle as M


@dataclass
class LayerGrads:
    du: np.ndarray            # [T, d]
    d_router: np.ndarray      # [N, d]
    d_logit_bias: Optional[np.ndarray]   # [N] or None
    d_w_gate: np.ndarray      # [N, I, d]
    d_w_up: np.ndarray        # [N, I, d]
    d_w_down: np.ndarray      # [N, d, I]
    d_ws_gate: Optional[np.ndarray]      # [Ks, Is, d]
    d_ws_up: Optional[np.ndarray]
    d_ws_down: Optional[np.ndarray]      # [Ks, d, Is]


def silu_grad(a: np.ndarray) -> np.ndarray:
    """d/da of a * sigma(a) = sigma(a) (1 + a (1 - sigma(a)))."""
    sg = 1.0 / (1.0 + np.exp(-a))
    return sg * (1.0 + a * (1.0 - sg))


def swiglu_ffn_backward(u, w_gate, w_up, w_down, dy):
    """Gradients of y = W_down (SiLU(W_gate u) * W_up u) for rows u [n, d] and dy [n, d]
    -> (du [n, d], dW_gate [I, d], dW_up [I, d], dW_down [d, I])."""
    wg, wu, wd = M.f64(w_gate), M.f64(w_up), M.f64(w_down)
    a = u @ wg.T
    b = u @ wu.T
    m = M.silu(a) * b
    dwd = dy.T @ m
    dm = dy @ wd
    db = dm * M.silu(a)
    da = dm * b * silu_grad(a)
    return da @ wg + db @ wu, da.T @ u, db.T @ u, dwd


def gate_logit_backward(s: np.ndarray, idx: np.ndarray, gate: np.ndarray, dg: np.ndarray,
                        gate_kind: str) -> np.ndarray:
    """dL/dz [T, N] from dL/dg [T, K] (reading B1: the choice idx is held fixed)."""
    T, N = s.shape
    if gate_kind == M.GATE_SOFTMAX:
        ds = np.zeros((T, N))
        np.add.at(ds, (np.repeat(np.arange(T), idx.shape[1]), idx.ravel()), dg.ravel())
        return s * (ds - (s * ds).sum(axis=1, keepdims=True))
    if gate_kind == M.GATE_SIGMOID:
        s_sel = np.take_along_axis(s, idx, axis=1)
        S = s_sel.sum(axis=1, keepdims=True)
        ds_sel = (dg - (gate * dg).sum(axis=1, keepdims=True)) / S
        dz = np.zeros((T, N))
        np.put_along_axis(dz, idx, ds_sel * s_sel * (1.0 - s_sel), axis=1)
        return dz
    raise ValueError(gate_kind)


def moe_backward(u, router_w, K: int, experts, shared=None, dh=None, *,
                 gate_kind: str = M.GATE_SOFTMAX, logit_bias=None, select_bias=None) -> LayerGrads:
    """All gradients of the layer output h (``moe_oracle.moe_forward``) for the upstream gradient dh."""
    u = M.f64(u)
    dh = M.f64(dh)
    T, d = u.shape
    e = M.f64(router_w)
    N = e.shape[0]
    w_gate, w_up, w_down = (M.f64(w) for w in experts)
    r = M.route(u, e, K, gate_kind, logit_bias, select_bias)

    du = dh.copy()                                     # the residual
    dwg, dwu, dwd = np.zeros_like(w_gate), np.zeros_like(w_up), np.zeros_like(w_down)
    dg = np.zeros((T, K))
    for ex in np.unique(r.idx):                        # each routed expert on the tokens that chose it
        rows, slots = np.nonzero(r.idx == ex)
        ur = u[rows]
        y = M.swiglu_ffn(ur, w_gate[ex], w_up[ex], w_down[ex])
        dg[rows, slots] = (dh[rows] * y).sum(axis=1)
        g = r.gate[rows, slots][:, None]
        dur, gwg, gwu, gwd = swiglu_ffn_backward(ur, w_gate[ex], w_up[ex], w_down[ex], g * dh[rows])
        np.add.at(du, rows, dur)
        dwg[ex] += gwg
        dwu[ex] += gwu
        dwd[ex] += gwd

    ds_g = ds_u = ds_d = None
    if shared is not None:
        sg, su, sd = (M.f64(w) for w in shared)
        ds_g, ds_u, ds_d = np.zeros_like(sg), np.zeros_like(su), np.zeros_like(sd)
        for j in range(sg.shape[0]):                   # gate 1 for every token
            dur, ds_g[j], ds_u[j], ds_d[j] = swiglu_ffn_backward(u, sg[j], su[j], sd[j], dh)
            du += dur

    dz = gate_logit_backward(r.s, r.idx, r.gate, dg, gate_kind)
    du += dz @ e
    return LayerGrads(du=du, d_router=dz.T @ u,
                      d_logit_bias=None if logit_bias is None else dz.sum(axis=0),
                      d_w_gate=dwg, d_w_up=dwu, d_w_down=dwd,
                      d_ws_gate=ds_g, d_ws_up=ds_u, d_ws_down=ds_d)
