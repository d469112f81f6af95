"""Parity of the layer's backward for the input and the router (moe_backward)
with the oracle's backward (oracle.moe_backward, pinned by central finite
differences of the forward oracle).

Comparison rules (the tolerances are written in the asserts below):
* dgate, dL/dg per (token, slot): max |gpu - oracle| <= 2e-2 * RMS(oracle),
  RMS(gpu - oracle) <= 1e-2 * RMS(oracle).  The GPU rounds dm = W_down^T dh to
  bf16 between two GEMMs (2^-9 relative) and sums dm . m in fp32.
* dx with the residual: the forward's output rule (max error <= 2e-2 * RMS).
* dx without the residual (the NO_RESIDUAL flag; the oracle's du minus dh),
  and the routed part alone (NO_RESIDUAL | NO_SHARED): the forward's term rule,
  max error <= 5e-2 * RMS: dm, da and db are rounded to bf16 between the GEMMs
  (2^-9 relative each, through sums of I and d terms) and each of the K rows
  before the k-ordered sum, as in the forward.
* d_router = dz^T u and d_logit_bias = sum_t dz: the term rule.
* the expert weights' gradients, per tensor: RMS(gpu - oracle) <= 1e-2 *
  RMS(oracle) and max |gpu - oracle| <= 2e-2 * max |oracle|.  Each element is a
  sum over an expert's rows of products of bf16-rounded operands (g dh, m, da,
  db; u is exact), so its error is up to about 2^-8 of the sum of the terms'
  magnitudes; the largest elements (sums of mostly same-signed terms, up to
  ~30x the tensor's RMS) keep that relative error, which a bound relative to
  the RMS would not admit.  Against an oracle that rounds the same operands to
  bf16 the GPU agrees to ~1e-5 of the RMS.
Tokens at a near-tie of the selection (the forward tests' exemption) would
route differently on the two sides and change dE; the seeded shapes have none,
which the tests assert.  Inside a token's K experts two nearly equal keys may
come out in either order, which moves their dgate between the two slots: the
oracle's dgate is computed for the GPU's own slot order, after checking that
each token's set of experts is the oracle's.
"""
import numpy as np
import pytest
import torch

import oracle as O
import oracle.moe_backward as OB
import workloads as W
from fine_grained_shared_b200 import moe as B
from tests import harness as H

pytestmark = pytest.mark.gpu

LS = W.LayerShape
SHAPES = {
    "softmax_logit_bias": LS("bwd_soft", T=300, d=256, N=16, I=128, K=4, Ks=1, Is=128, sigma=0.05, bias="normal",
                             seed=91),
    "sigmoid": LS("bwd_sig", T=333, d=384, N=40, I=128, K=8, Ks=2, Is=128, gate="sigmoid", sigma=0.03,
                  bias="uniform", seed=92),
    # no shared experts, d and I not multiples of 64 (ragged k-blocks in every GEMM)
    "ragged_no_shared": LS("bwd_rag", T=257, d=208, N=13, I=48, K=3, Ks=0, Is=0, sigma=0.05, seed=93),
    # the forward of a decode-sized batch runs the decode FFN; the backward runs the grouped GEMMs
    "decode": LS("bwd_dec", T=40, d=256, N=24, I=128, K=6, Ks=2, Is=64, sigma=0.03, bias="zipf", seed=94),
}


def _rows(t):
    return t.float().cpu().numpy().astype(np.float64)


def _compare(got, want, what, tol):
    rms = float(np.sqrt(np.mean(want ** 2)))
    err = float(np.max(np.abs(got - want)))
    rms_err = float(np.sqrt(np.mean((got - want) ** 2)))
    assert np.isfinite(got).all(), f"{what}: non-finite"
    assert err <= tol * rms, f"{what}: max|diff| {err:.3e} > {tol} * rms {rms:.3e}"
    assert rms_err <= 1e-2 * rms, f"{what}: rms diff {rms_err:.3e} > 1e-2 * rms {rms:.3e}"
    return err / rms, rms_err / rms


def _compare_wgrad(got, want, what):
    rms = float(np.sqrt(np.mean(want ** 2)))
    top = float(np.max(np.abs(want)))
    err = float(np.max(np.abs(got - want)))
    rms_err = float(np.sqrt(np.mean((got - want) ** 2)))
    assert np.isfinite(got).all(), f"{what}: non-finite"
    assert err <= 2e-2 * top, f"{what}: max|diff| {err:.3e} > 2e-2 * max|oracle| {top:.3e}"
    assert rms_err <= 1e-2 * rms, f"{what}: rms diff {rms_err:.3e} > 1e-2 * rms {rms:.3e}"


def _oracle_dgate(shape, host, dh, idx, rows=None, experts=None):
    """dL/dg = dh . FFN_e(u) per (token, slot) for the experts idx [n, K], from the oracle's FFN."""
    u = O.f64(host["x"]) if rows is None else O.f64(host["x"])[rows]
    dh = O.f64(dh) if rows is None else O.f64(dh)[rows]
    experts = experts if experts is not None else H.oracle_experts(shape, host)
    fn = experts if callable(experts) else (lambda e: (experts[0][e], experts[1][e], experts[2][e]))
    dg = np.zeros(idx.shape)
    for ex in np.unique(idx):
        r, k = np.nonzero(idx == ex)
        y = O.swiglu_ffn(u[r], *fn(int(ex)))
        dg[r, k] = (dh[r] * y).sum(axis=1)
    return dg


def _same_expert_sets(gpu_idx, ref_idx):
    np.testing.assert_array_equal(np.sort(gpu_idx, axis=1), np.sort(ref_idx, axis=1))


def _run(shape, dev, flags, dh, router_grad=True, weight_grads=False):
    layer = H.make_layer(shape, dev, flags=flags)
    H.run(layer, dev["x"], shape.K)
    res = layer.backward(dev["x"], shape.K, dh, router_grad=router_grad, weight_grads=weight_grads)
    assert layer.status() == B.MOE_OK, B.status_string(layer.status())
    idx = layer.routing(shape.T, shape.K)[0].cpu().numpy()
    layer.close()
    return res + (idx,)


@pytest.mark.parametrize("name", sorted(SHAPES))
def test_backward_matches_the_oracle(name):
    shape = SHAPES[name]
    host, dev = H.device_inputs(shape)
    dh_host = W.output_gradient(shape)
    dh = dh_host.to("cuda")
    route = H.oracle_routing(shape, host)
    assert (route.gap < H.GAP_EXEMPT).sum() == 0
    grads = OB.moe_backward(host["x"], host["router"], shape.K, (host["w_gate"], host["w_up"], host["w_down"]),
                            H.oracle_shared(shape, host), dh=dh_host, gate_kind=shape.gate,
                            logit_bias=host["logit_bias"], select_bias=host["select_bias"])
    dx, dgate, d_router, d_bias, wg, idx = _run(shape, dev, 0, dh, weight_grads=True)
    _same_expert_sets(idx, route.idx)
    for key, want in (("w_gate", grads.d_w_gate), ("w_up", grads.d_w_up), ("w_down", grads.d_w_down),
                      ("ws_gate", grads.d_ws_gate), ("ws_up", grads.d_ws_up), ("ws_down", grads.d_ws_down)):
        if want is None:
            assert key not in wg
            continue
        _compare_wgrad(wg[key].cpu().numpy().astype(np.float64), want, f"{name} d{key}")
    _compare(_rows(dgate), _oracle_dgate(shape, host, dh_host, idx), f"{name} dgate", 2e-2)
    _compare(_rows(dx), grads.du, f"{name} dx", 2e-2)
    _compare(d_router.cpu().numpy().astype(np.float64), grads.d_router, f"{name} d_router", 5e-2)
    if host["logit_bias"] is not None:
        _compare(d_bias.cpu().numpy().astype(np.float64), grads.d_logit_bias, f"{name} d_logit_bias", 5e-2)
    else:
        assert d_bias is None
    # without the residual: every other term at the term rule
    dx_nr = _run(shape, dev, B.MOE_FLAG_NO_RESIDUAL, dh, router_grad=False)[0]
    du_nr = grads.du - O.f64(dh_host)
    _compare(_rows(dx_nr), du_nr, f"{name} dx without the residual", 5e-2)
    if shape.Ks:
        # the routed experts and the router alone
        dx_r = _run(shape, dev, B.MOE_FLAG_NO_RESIDUAL | B.MOE_FLAG_NO_SHARED, dh, router_grad=False)[0]
        sg, su, sd = (O.f64(w) for w in H.oracle_shared(shape, host))
        shared_du = sum(OB.swiglu_ffn_backward(O.f64(host["x"]), sg[j], su[j], sd[j], O.f64(dh_host))[0]
                        for j in range(shape.Ks))
        _compare(_rows(dx_r), du_nr - shared_du, f"{name} routed and router terms of dx", 5e-2)


def test_weight_gradients_ignore_an_earlier_forwards_rows():
    """A forward of all-NaN tokens (every key ranks last, so every token takes experts 0..K-1) and its
    backward leave NaN in X_perm's and g dh's rows of those experts' segments.  A later clean forward
    routes about T*K/mN rows to each expert, so those rows are now the padding past each expert's count
    inside the weight-gradient GEMMs' last 64-row K block; the clean backward's weight gradients must
    still be finite and match the oracle."""
    shape = SHAPES["softmax_logit_bias"]
    host, dev = H.device_inputs(shape)
    dh_host = W.output_gradient(shape)
    dh = dh_host.to("cuda")
    layer = H.make_layer(shape, dev)
    bad = torch.full_like(dev["x"], float("nan"))
    layer.forward(bad, shape.K)
    layer.backward(bad, shape.K, dh, weight_grads=True)
    assert layer.status() == B.MOE_OK
    H.run(layer, dev["x"], shape.K)
    wg = layer.backward(dev["x"], shape.K, dh, weight_grads=True)[4]
    assert layer.status() == B.MOE_OK
    counts = np.bincount(layer.routing(shape.T, shape.K)[0].cpu().numpy().ravel(), minlength=shape.N)
    assert (counts[:shape.K] % 64 != 0).all()        # each stale segment has padding rows in a K block
    layer.close()
    grads = OB.moe_backward(host["x"], host["router"], shape.K, (host["w_gate"], host["w_up"], host["w_down"]),
                            H.oracle_shared(shape, host), dh=dh_host, gate_kind=shape.gate,
                            logit_bias=host["logit_bias"], select_bias=host["select_bias"])
    for key, want in (("w_gate", grads.d_w_gate), ("w_up", grads.d_w_up), ("w_down", grads.d_w_down),
                      ("ws_gate", grads.d_ws_gate), ("ws_up", grads.d_ws_up), ("ws_down", grads.d_ws_down)):
        _compare_wgrad(wg[key].cpu().numpy().astype(np.float64), want, f"after a NaN forward: d{key}")


def test_backward_is_deterministic():
    shape = SHAPES["sigmoid"]
    host, dev = H.device_inputs(shape)
    dh = W.output_gradient(shape).to("cuda")
    layer = H.make_layer(shape, dev)
    outs = []
    for _ in range(2):
        H.run(layer, dev["x"], shape.K)
        outs.append([t.clone() for t in layer.backward(dev["x"], shape.K, dh, router_grad=True) if t is not None])
    for a, b in zip(*outs):
        assert torch.equal(a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32),
                           b.view(torch.int16) if b.dtype == torch.bfloat16 else b.view(torch.int32))


def test_backward_wait_timeout_is_reported():
    """The test-only flag makes CTA 0 of the backward's recompute wait 20 ms on a barrier nothing
    arrives on: the backward reports MOE_ERR_TIMEOUT, and a new handle's backward is correct."""
    shape = SHAPES["softmax_logit_bias"]
    host, dev = H.device_inputs(shape)
    dh = W.output_gradient(shape).to("cuda")
    bad = H.make_layer(shape, dev, flags=B.MOE_FLAG_DEBUG_WAIT_TIMEOUT)
    bad.forward(dev["x"], shape.K)
    assert bad.status() == B.MOE_ERR_TIMEOUT        # the forward's GEMM took the flag too
    bad.backward(dev["x"], shape.K, dh)
    assert bad.status() == B.MOE_ERR_TIMEOUT
    assert bad.status() == B.MOE_OK
    bad.close()
    good = H.make_layer(shape, dev)
    H.run(good, dev["x"], shape.K)
    dx = good.backward(dev["x"], shape.K, dh)[0]
    assert good.status() == B.MOE_OK
    want = H.make_layer(shape, dev)
    H.run(want, dev["x"], shape.K)
    assert torch.equal(dx.view(torch.int16), want.backward(dev["x"], shape.K, dh)[0].view(torch.int16))


def test_backward_checks_its_forward():
    shape = SHAPES["softmax_logit_bias"]
    host, dev = H.device_inputs(shape)
    dh = W.output_gradient(shape).to("cuda")
    layer = H.make_layer(shape, dev)
    with pytest.raises(B.MoEError) as e:
        layer.backward(dev["x"], shape.K, dh)                   # no forward yet
    assert e.value.status == B.MOE_ERR_INVALID_ARG
    H.run(layer, dev["x"], shape.K)
    with pytest.raises(B.MoEError):
        layer.backward(dev["x"][:100], shape.K, dh[:100])       # not the forward's T
    with pytest.raises(B.MoEError):
        layer.backward(dev["x"], shape.K - 1, dh)               # not the forward's K
    with pytest.raises(B.MoEError):
        layer.backward(dev["x"], shape.K, dh, dx=dh)             # dx over dh
    layer.backward(dev["x"], shape.K, dh)
    assert layer.status() == B.MOE_OK


@pytest.mark.parametrize("name", ["16b_prefill", "2b", "v3"])
def test_backward_full_size_every_tile(name):
    """A full-size layer's backward on a token set with a row in every GEMM tile: dx and dgate of
    those tokens (tokens are independent in both, so the oracle runs on them alone).  The 2B layer
    has an odd number of routed experts (63) and a logit bias; V3 the sigmoid gate with a selection
    bias over 256 experts."""
    shape = W.CONFIGS[name]
    host, dev = H.device_inputs(shape)
    dh_host = W.output_gradient(shape)
    dh = dh_host.to("cuda")
    ref = H.oracle_routing(shape, host)
    rows, covered, total = H.stratified_rows(shape, ref)
    assert covered == total
    layer = H.make_layer(shape, dev)
    H.run(layer, dev["x"], shape.K)
    dx, dgate, _, _ = layer.backward(dev["x"], shape.K, dh)
    assert layer.status() == B.MOE_OK
    gpu_idx = layer.routing(shape.T, shape.K)[0].cpu().numpy()
    layer.close()
    rows = rows[ref.gap[rows] >= H.GAP_EXEMPT]
    sub = O.route(host["x"][rows], host["router"], shape.K, shape.gate, host["logit_bias"], host["select_bias"])
    _same_expert_sets(gpu_idx[rows], sub.idx)
    u = O.f64(host["x"])[rows]
    dhr = O.f64(dh_host)[rows]
    experts = H.oracle_experts(shape, host, prefetch=np.unique(sub.idx))
    fn = experts if callable(experts) else (lambda e: (experts[0][e], experts[1][e], experts[2][e]))
    du = dhr.copy()
    if shape.Ks:
        sg, su, sd = (O.f64(w) for w in H.oracle_shared(shape, host))
        for j in range(shape.Ks):
            du += OB.swiglu_ffn_backward(u, sg[j], su[j], sd[j], dhr)[0]
    dg = np.zeros(sub.idx.shape)
    for ex in np.unique(sub.idx):
        r, k = np.nonzero(sub.idx == ex)
        wg, wu, wd = fn(int(ex))
        dg[r, k] = (dhr[r] * O.swiglu_ffn(u[r], wg, wu, wd)).sum(axis=1)
        np.add.at(du, r, OB.swiglu_ffn_backward(u[r], wg, wu, wd, sub.gate[r, k][:, None] * dhr[r])[0])
    dz = OB.gate_logit_backward(sub.s, sub.idx, sub.gate, dg, shape.gate)
    du += dz @ O.f64(host["router"])
    dg_gpu_order = _oracle_dgate(shape, host, dh_host, gpu_idx[rows], rows, experts)
    e1 = _compare(_rows(dgate)[rows], dg_gpu_order, f"{name} dgate", 2e-2)
    e2 = _compare(_rows(dx)[rows], du, f"{name} dx", 2e-2)
    print(f"{name} backward: {rows.size} rows; dgate max/rms err {e1}, dx {e2}")
