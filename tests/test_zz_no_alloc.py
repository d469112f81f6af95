"""The allocation-free routing entry point against the normal one.

moe_route_noalloc exists for callers that cannot call cudaMalloc (a runtime
that plans all device memory up front, a framework whose allocator must own
every allocation, a loop that cannot take cudaMalloc's implicit device
synchronisation).  It keeps its scratch in a fixed device array inside the
library.  This file runs last (pytest collects it after the others) and
passes both alone in a fresh process and after the rest of the suite.
"""
import ctypes

import numpy as np
import pytest
import torch

import workloads as W
from fine_grained_shared_b200 import moe as B
from tests import harness as H

pytestmark = pytest.mark.gpu

LS = W.LayerShape
CASES = {
    "tiny": W.CONFIGS["tiny"],
    "sigmoid_ragged": LS("sigmoid_ragged", T=333, d=192, N=40, I=96, K=8, Ks=1, Is=64, gate="sigmoid",
                         sigma=0.03, bias="uniform", seed=16),
    # the scratch's largest layout: 256 experts (a 256-row TMA box, the 4-stage ring, the widest
    # block histogram), K = 8, sigmoid gate with a selection bias, a ragged last token block
    "n256_sigmoid": LS("n256_sigmoid", T=1000, d=512, N=256, I=64, K=8, Ks=1, Is=64, gate="sigmoid",
                       sigma=0.006, bias="uniform", seed=31),
    # batches of at most 256 tokens, where moe_forward routes on the CUDA cores instead
    "decode_t32": LS("decode_t32", T=32, d=2048, N=64, I=64, K=6, Ks=2, Is=64, sigma=0.02, bias="zipf", seed=32),
    "one_token": LS("one_token", T=1, d=256, N=16, I=64, K=4, Ks=1, Is=64, sigma=0.02, seed=33),
}


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("name", sorted(CASES))
def test_noalloc_routing_matches_moe_forward_twice_in_a_row(name):
    shape = CASES[name]
    host, dev = H.device_inputs(shape)
    layer = H.make_layer(shape, dev)
    H.run(layer, dev["x"], shape.K)
    ref_idx, ref_gate, ref_counts, ref_offsets, _ = (t.cpu().numpy() for t in layer.routing(shape.T, shape.K))
    layer.close()
    oracle = H.oracle_routing(shape, host)
    ok = oracle.gap >= H.GAP_EXEMPT          # tokens without a near-tie at the selection boundary
    same_kernel = shape.T > 256              # moe_forward runs the same router kernel on these

    T, K, N = shape.T, shape.K, shape.N
    gate_kind = B.MOE_GATE_SIGMOID_BIASED if shape.gate == "sigmoid" else B.MOE_GATE_SOFTMAX
    router = B.moe_router(dev["router"].data_ptr(),
                          dev["logit_bias"].data_ptr() if dev["logit_bias"] is not None else None,
                          dev["select_bias"].data_ptr() if dev["select_bias"] is not None else None)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call in range(2):
        idx = torch.full((T, K), -1, dtype=torch.int32, device="cuda")
        gate = torch.full((T, K), -1.0, dtype=torch.float32, device="cuda")
        counts = torch.full((N,), -1, dtype=torch.int32, device="cuda")
        offsets = torch.full((N + 1,), -1, dtype=torch.int32, device="cuda")
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        st = B.moe_route_noalloc(_ptr(dev["x"]), T, shape.d, router, N, gate_kind, K, _ptr(idx), _ptr(gate),
                                 _ptr(counts), _ptr(offsets), _ptr(err), stream)
        assert st == B.MOE_OK, B.status_string(st)
        torch.cuda.synchronize()
        assert int(err.item()) == 0, f"call {call}: device error bits {int(err.item()):#x}"
        idx, gate, counts, offsets = (t.cpu().numpy() for t in (idx, gate, counts, offsets))
        msg = f"{name}, call {call}"
        # against the existing entry point
        if same_kernel:
            np.testing.assert_array_equal(idx, ref_idx, err_msg=msg)
            np.testing.assert_array_equal(counts, ref_counts, err_msg=msg)
            np.testing.assert_array_equal(offsets, ref_offsets, err_msg=msg)
        else:
            np.testing.assert_array_equal(idx[ok], ref_idx[ok], err_msg=msg)
        np.testing.assert_allclose(gate[ok], ref_gate[ok], rtol=0, atol=H.GATE_TOL, err_msg=msg)
        # against the oracle, under the near-tie rule of the parity tests
        np.testing.assert_array_equal(idx[ok], oracle.idx[ok], err_msg=msg)
        np.testing.assert_allclose(gate[ok], oracle.gate[ok], rtol=0, atol=H.GATE_TOL, err_msg=msg)
        assert ((idx >= 0) & (idx < N)).all(), msg
        assert all(len(set(r)) == K for r in idx.tolist()), msg
        np.testing.assert_array_equal(counts, np.bincount(idx.ravel(), minlength=N), err_msg=msg)
        np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(counts)]), err_msg=msg)


def test_noalloc_rejects_bad_arguments_before_any_launch():
    x = torch.zeros((8, 256), dtype=torch.bfloat16, device="cuda")
    router = B.moe_router(torch.zeros((16, 256), dtype=torch.bfloat16, device="cuda").data_ptr(), None, None)
    out = torch.zeros(16, dtype=torch.int32, device="cuda")
    args = (_ptr(out), _ptr(out), _ptr(out), _ptr(out))
    assert B.moe_route_noalloc(_ptr(x), 65537, 256, router, 16, B.MOE_GATE_SOFTMAX, 4, *args, _ptr(out),
                               None) == B.MOE_ERR_SHAPE
    assert B.moe_route_noalloc(_ptr(x), 8, 256, router, 16, B.MOE_GATE_SOFTMAX, 4, *args, None,
                               None) == B.MOE_ERR_INVALID_ARG
    assert B.moe_route_noalloc(_ptr(x), 8, 256, router, 16, B.MOE_GATE_SOFTMAX, 4, *args,
                               ctypes.c_void_p(out.data_ptr() + 2), None) == B.MOE_ERR_ALIGNMENT
    torch.cuda.synchronize()
