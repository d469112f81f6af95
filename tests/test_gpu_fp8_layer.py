"""Parity of the FP8 layer forward (moe_forward_fp8) with the FP8 oracle.

The oracle (oracle.fp8.moe_forward_fp8) routes in high precision like the
plain layer, quantizes x and H 1 x 128 and the expert weights 128 x 128 to
E4M3 with power-of-two scales, and accumulates in float64.  The GPU path is
given the weights as the library's block quantizer writes them (its codes and
scale bytes are bit-exact against the oracle's, tests/test_gpu_fp8.py); the
oracle quantizes its own copy from the bf16 weights.

Rules: routing as the bf16 path (bit-exact indices, gates to 1e-5); outputs
within the bf16 path's tolerances of the FP8 oracle.  Those hold although H is
rounded to E4M3 on both sides from values that differ in the last bits (fp32
here, float64 in the oracle): an H code on a rounding midpoint may land on the
neighbouring code, a change of one E4M3 step (1/16 of the value's binade) in
one element of the down projection's input, far below the tolerances.
"""
import numpy as np
import pytest
import torch

import oracle.fp8 as F8
import workloads as W
from fine_grained_shared_b200 import moe as B
from tests import harness as H

pytestmark = pytest.mark.gpu

LS = W.LayerShape
SHAPES = {
    "small": LS("fp8_small", T=300, d=256, N=16, I=256, K=4, Ks=1, Is=128, sigma=0.05, seed=61),
    "sigmoid": LS("fp8_sigmoid", T=333, d=384, N=40, I=128, K=8, Ks=2, Is=128, gate="sigmoid", sigma=0.03,
                  bias="uniform", seed=62),
    "no_shared": LS("fp8_no_shared", T=200, d=128, N=12, I=384, K=3, Ks=0, Is=0, sigma=0.05, bias="normal",
                    seed=63),
    "decode": LS("fp8_decode", T=20, d=512, N=24, I=256, K=6, Ks=2, Is=128, sigma=0.03, bias="zipf", seed=64),
    # decode batches run the FP8 decode FFN: two token blocks of routed rows without shared experts, and
    # two shared token blocks
    "decode_t64_sigmoid": LS("fp8_decode_t64", T=64, d=384, N=20, I=256, K=4, Ks=0, Is=0, gate="sigmoid",
                             sigma=0.03, bias="uniform", seed=65),
    "decode_t40": LS("fp8_decode_t40", T=40, d=256, N=12, I=384, K=2, Ks=2, Is=128, sigma=0.05, seed=66),
}

FLAGS_ROUTED = B.MOE_FLAG_NO_RESIDUAL | B.MOE_FLAG_NO_SHARED
FLAGS_SHARED = B.MOE_FLAG_NO_RESIDUAL | B.MOE_FLAG_NO_ROUTED


def _fp8_weights(dev, shape):
    ex = tuple(B.quantize_fp8_blocks(dev[k]) for k in ("w_gate", "w_up", "w_down"))
    sh = tuple(B.quantize_fp8_blocks(dev[k]) for k in ("ws_gate", "ws_up", "ws_down")) if shape.Ks else None
    return ex, sh


def _layer(shape, dev, flags=0):
    layer = H.make_layer(shape, dev, flags=flags | B.MOE_FLAG_FP8)
    layer.set_weights_fp8(*_fp8_weights(dev, shape))
    return layer


def _check(shape, host, dev, rows, ref):
    experts = H.oracle_experts(shape, host, prefetch=np.unique(ref.idx[rows]) if "w_gate" not in host else None)
    shared = H.oracle_shared(shape, host)
    cases = [(0, "output"), (FLAGS_ROUTED, "routed term")]
    if shape.Ks:
        cases.append((FLAGS_SHARED, "shared term"))
    res = {}
    for flags, what in cases:
        layer = _layer(shape, dev, flags)
        out = layer.forward_fp8(dev["x"], shape.K)
        st = layer.status()
        assert st == B.MOE_OK, B.status_string(st)
        if flags == 0:
            res["exempt"] = H.check_routing(shape, layer, ref)[0]
        layer.close()
        want, _ = F8.moe_forward_fp8(host["x"], host["router"], shape.K, experts, shared, gate_kind=shape.gate,
                                     logit_bias=host["logit_bias"], select_bias=host["select_bias"], flags=flags,
                                     rows=rows, routing=ref)
        got = out.float().cpu().numpy()[rows].astype(np.float64)
        res[what] = H.compare_output(got, want, f"{shape.name} fp8 {what}", term=flags != 0)
    return res


@pytest.mark.parametrize("name", sorted(SHAPES))
def test_fp8_layer_small_shapes_every_token(name):
    shape = SHAPES[name]
    host, dev = H.device_inputs(shape)
    ref = H.oracle_routing(shape, host)
    rows = np.nonzero(ref.gap >= H.GAP_EXEMPT)[0]
    _check(shape, host, dev, rows, ref)


def test_fp8_layer_16b_prefill_every_tile():
    """The 16B prefill layer on a token set with a compared row in every GEMM tile."""
    shape = W.CONFIGS["16b_prefill"]
    host, dev = H.device_inputs(shape)
    ref = H.oracle_routing(shape, host)
    rows, covered, total = H.stratified_rows(shape, ref)
    assert covered == total
    res = _check(shape, host, dev, rows, ref)
    print(f"16b_prefill fp8: compared rows {rows.size}, "
          + ", ".join(f"{k}: max err {v[0]:.2e} rms err {v[2]:.2e} rms {v[1]:.2e}"
                      for k, v in res.items() if k != "exempt"))


def test_fp8_layer_16b_decode_every_token():
    """The 16B decode layer (T = 32, the FP8 decode FFN) on every token."""
    shape = W.CONFIGS["16b_decode"]
    host, dev = H.device_inputs(shape)
    ref = H.oracle_routing(shape, host)
    rows = np.nonzero(ref.gap >= H.GAP_EXEMPT)[0]
    res = _check(shape, host, dev, rows, ref)
    print(f"16b_decode fp8: compared rows {rows.size}, "
          + ", ".join(f"{k}: max err {v[0]:.2e} rms err {v[2]:.2e} rms {v[1]:.2e}"
                      for k, v in res.items() if k != "exempt"))


def test_fp8_decode_ffn_is_deterministic():
    shape = SHAPES["decode"]
    host, dev = H.device_inputs(shape)
    layer = _layer(shape, dev)
    outs = [layer.forward_fp8(dev["x"], shape.K).clone() for _ in range(3)]
    assert all(torch.equal(outs[0].view(torch.int16), o.view(torch.int16)) for o in outs[1:])
    assert layer.status() == B.MOE_OK


@pytest.mark.parametrize("name", ["small", "decode_t40"])
def test_fp8_device_wait_timeout_is_reported_and_the_context_stays_usable(name):
    """A bounded wait that runs out in the FP8 gate/up GEMM (prefill) or the FP8 decode FFN: the call
    reports MOE_ERR_TIMEOUT and a later forward gives the same bits as one taken before it."""
    shape = SHAPES[name]
    host, dev = H.device_inputs(shape)
    good = _layer(shape, dev)
    before = good.forward_fp8(dev["x"], shape.K).clone()
    assert good.status() == B.MOE_OK
    bad = _layer(shape, dev, B.MOE_FLAG_DEBUG_WAIT_TIMEOUT)
    for _ in range(2):
        bad.forward_fp8(dev["x"], shape.K)
        assert bad.status() == B.MOE_ERR_TIMEOUT
        assert bad.status() == B.MOE_OK
    bad.close()
    after = good.forward_fp8(dev["x"], shape.K)
    assert good.status() == B.MOE_OK
    assert torch.equal(before.view(torch.int16), after.view(torch.int16))


def test_fp8_layer_is_deterministic_and_close_to_the_bf16_layer():
    shape = SHAPES["small"]
    host, dev = H.device_inputs(shape)
    layer = _layer(shape, dev)
    a = layer.forward_fp8(dev["x"], shape.K).clone()
    b = layer.forward_fp8(dev["x"], shape.K).clone()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    bf = layer.forward(dev["x"], shape.K).float()
    # the FP8 layer differs from the bf16 one by a few per cent of the FFN terms only
    ffn = (bf - dev["x"].float())
    diff = (a.float() - bf)
    assert float(diff.pow(2).mean().sqrt()) < 0.15 * float(ffn.pow(2).mean().sqrt())
    assert layer.status() == B.MOE_OK


def test_fp8_forward_needs_an_fp8_handle():
    shape = SHAPES["small"]
    host, dev = H.device_inputs(shape)
    plain = H.make_layer(shape, dev)
    plain.set_weights_fp8(*_fp8_weights(dev, shape))
    st, _ = plain.forward_fp8(dev["x"], shape.K, check=False)
    assert st == B.MOE_ERR_UNSUPPORTED
