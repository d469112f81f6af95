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


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr())


@pytest.mark.parametrize("name", ["tiny", "sigmoid_ragged"])
def test_noalloc_routing_matches_moe_forward_twice_in_a_row(name):
    shape = W.CONFIGS["tiny"] if name == "tiny" else W.LayerShape(
        "sigmoid_ragged", T=333, d=192, N=40, I=96, K=8, Ks=1, Is=64, gate="sigmoid", sigma=0.03,
        bias="uniform", seed=16)
    host, dev = H.device_inputs(shape)
    layer = H.make_layer(shape, dev)
    H.run(layer, dev["x"], shape.K)
    ref_idx, ref_gate, ref_counts, ref_offsets, _ = (t.cpu() for t in layer.routing(shape.T, shape.K))
    layer.close()

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
        np.testing.assert_array_equal(idx.cpu().numpy(), ref_idx.numpy(), err_msg=f"call {call}")
        np.testing.assert_allclose(gate.cpu().numpy(), ref_gate.numpy(), rtol=0, atol=H.GATE_TOL,
                                   err_msg=f"call {call}")
        np.testing.assert_array_equal(counts.cpu().numpy(), ref_counts.numpy(), err_msg=f"call {call}")
        np.testing.assert_array_equal(offsets.cpu().numpy(), ref_offsets.numpy(), err_msg=f"call {call}")


def test_noalloc_rejects_batches_beyond_its_scratch():
    x = torch.zeros((8, 256), dtype=torch.bfloat16, device="cuda")
    router = B.moe_router(torch.zeros((16, 256), dtype=torch.bfloat16, device="cuda").data_ptr(), None, None)
    out = torch.zeros(1, dtype=torch.int32, device="cuda")
    st = B.moe_route_noalloc(_ptr(x), 65537, 256, router, 16, B.MOE_GATE_SOFTMAX, 4, _ptr(out), _ptr(out),
                             _ptr(out), _ptr(out), None, None)
    assert st == B.MOE_ERR_SHAPE
