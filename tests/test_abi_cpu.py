"""The C ABI without a GPU: the library loads, exports every entry point the
header declares, and rejects bad configurations before any CUDA call."""
import ctypes
import os
import re

import pytest
import torch

from fine_grained_shared_b200 import moe as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = []
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            text = open(os.path.join(ROOT, "include", f)).read()
            names += re.findall(r"^\s*(?:moe_status|const char\*)\s+(moe_\w+)\s*\(", text, re.M)
    return names


def test_library_exports_every_declared_entry_point():
    lib = B.lib()
    names = _declared()
    assert "moe_forward" in names and "moe_create" in names and len(names) >= 8
    for n in names:
        assert hasattr(lib, n), n


def _cfg(**kw):
    base = dict(d_model=256, n_routed=16, d_ff=128, n_shared=1, d_ff_shared=128, max_tokens=512, max_k=4,
                gate=B.MOE_GATE_SOFTMAX, flags=0, route_nodes=0, route_max_nodes=0)
    base.update(kw)
    return B.moe_config(**base)


@pytest.mark.parametrize("kw,status", [
    ({}, B.MOE_OK),
    ({"d_model": 200}, B.MOE_ERR_ALIGNMENT),
    ({"d_ff": 72}, B.MOE_ERR_ALIGNMENT),
    ({"d_ff_shared": 24}, B.MOE_ERR_ALIGNMENT),
    ({"n_routed": 257, "max_k": 4}, B.MOE_ERR_UNSUPPORTED),
    ({"max_k": 9, "n_routed": 64}, B.MOE_ERR_UNSUPPORTED),
    ({"max_k": 17}, B.MOE_ERR_UNSUPPORTED),
    ({"max_k": 8, "n_routed": 4}, B.MOE_ERR_INVALID_ARG),
    ({"max_tokens": 0}, B.MOE_ERR_SHAPE),
    ({"max_tokens": (1 << 20) + 1}, B.MOE_ERR_SHAPE),
    ({"n_shared": -1}, B.MOE_ERR_SHAPE),
    ({"d_model": 0}, B.MOE_ERR_SHAPE),
    ({"gate": 7}, B.MOE_ERR_INVALID_ARG),
    ({"flags": 0x40}, B.MOE_ERR_INVALID_ARG),
    ({"n_shared": 0, "d_ff_shared": 0}, B.MOE_OK),
    # node-limited routing: nodes divide mN, 1 <= M <= nodes <= 16, K fits in M nodes' experts
    ({"route_nodes": 4, "route_max_nodes": 2}, B.MOE_OK),
    ({"route_nodes": 3, "route_max_nodes": 2}, B.MOE_ERR_INVALID_ARG),
    ({"route_nodes": 4, "route_max_nodes": 5}, B.MOE_ERR_INVALID_ARG),
    ({"route_nodes": 4, "route_max_nodes": 0}, B.MOE_ERR_INVALID_ARG),
    ({"route_nodes": 16, "route_max_nodes": 1, "max_k": 2}, B.MOE_ERR_INVALID_ARG),
    ({"route_nodes": 32, "route_max_nodes": 1, "n_routed": 64}, B.MOE_ERR_INVALID_ARG),
    ({"route_nodes": 0, "route_max_nodes": 2}, B.MOE_ERR_INVALID_ARG),
    # the FP8 workspace wants 128-column groups
    ({"flags": 0x8}, B.MOE_OK),
    ({"flags": 0x8, "d_ff": 208}, B.MOE_ERR_ALIGNMENT),
    ({"flags": 0x8, "d_ff_shared": 144}, B.MOE_ERR_ALIGNMENT),
    ({"flags": 0x8, "d_model": 272}, B.MOE_ERR_ALIGNMENT),
    ({"flags": 0x8, "d_model": 8320}, B.MOE_ERR_SHAPE),
])
def test_config_validation(kw, status):
    st, nbytes = B.moe_workspace_bytes(_cfg(**kw))
    assert st == status, B.status_string(st)
    if status == B.MOE_OK:
        assert nbytes > 0
    else:
        st2, h = B.moe_create(_cfg(**kw), 0)
        assert st2 == status and not h.value


def test_workspace_grows_with_the_layer():
    _, plain = B.moe_workspace_bytes(_cfg())
    _, fp8 = B.moe_workspace_bytes(_cfg(flags=0x8))
    assert fp8 > plain
    _, small = B.moe_workspace_bytes(_cfg())
    _, big = B.moe_workspace_bytes(_cfg(max_tokens=4096))
    _, wider = B.moe_workspace_bytes(_cfg(d_model=512))
    assert big > small and wider > small


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-device path")
def test_create_without_a_gpu_fails_cleanly():
    st, h = B.moe_create(_cfg(), 0)
    assert st == B.MOE_ERR_CUDA and not h.value


def test_null_handles():
    lib = B.lib()
    assert lib.moe_destroy(None) == B.MOE_OK
    assert lib.moe_status_query(None) == B.MOE_ERR_INVALID_ARG
    r, e = B.moe_router(), B.moe_experts()
    assert lib.moe_forward(None, None, 1, ctypes.byref(r), ctypes.byref(e), None, 1, None, None) == \
        B.MOE_ERR_INVALID_ARG
    assert lib.moe_get_routing(None, None, None, None, None, None, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_update_bias(None, None, 0.001, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_set_timing(None, 1) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_forward_host(None, None, 1, ctypes.byref(r), ctypes.byref(e), None, 1, None, None) == \
        B.MOE_ERR_INVALID_ARG
    assert lib.moe_kernel_times(None, None, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_forward_fp8(None, None, 1, ctypes.byref(r), None, None, 1, None, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_backward(None, None, 1, ctypes.byref(r), ctypes.byref(e), None, 1, None, None, None, None, None,
                            None, None) == B.MOE_ERR_INVALID_ARG
    # the expert-parallel calls
    assert lib.moe_ep_workspace(None, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_set_peers(None, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_ipc_handle(None, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_open_peers(None, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_route(None, None, 1, ctypes.byref(r), 1, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_dispatch(None, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_experts(None, ctypes.byref(e), None, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_experts_fp8(None, None, None, None) == B.MOE_ERR_INVALID_ARG
    assert lib.moe_ep_combine(None, None, None) == B.MOE_ERR_INVALID_ARG


def test_fp8_quantize_arguments_are_checked_before_any_cuda_call():
    """Fake, never dereferenced device addresses: every case returns before a launch."""
    lib = B.lib()
    a, b, c = 0x10000, 0x20000, 0x30000
    rows = lib.moe_quantize_fp8_rows
    assert rows(None, 4, 128, b, c, None) == B.MOE_ERR_INVALID_ARG
    assert rows(a, 4, 128, b, None, None) == B.MOE_ERR_INVALID_ARG
    assert rows(a, -1, 128, b, c, None) == B.MOE_ERR_SHAPE
    assert rows(a, 4, 0, b, c, None) == B.MOE_ERR_SHAPE
    assert rows(a, 4, 120, b, c, None) == B.MOE_ERR_ALIGNMENT
    assert rows(a + 8, 4, 128, b, c, None) == B.MOE_ERR_ALIGNMENT
    assert rows(a, 4, 128, b + 4, c, None) == B.MOE_ERR_ALIGNMENT
    assert rows(a, 0, 128, b, c, None) == B.MOE_OK
    blocks = lib.moe_quantize_fp8_blocks
    assert blocks(a, 2, 128, 128, None, c, None) == B.MOE_ERR_INVALID_ARG
    assert blocks(a, 70000, 128, 128, b, c, None) == B.MOE_ERR_SHAPE
    assert blocks(a, 2, -5, 128, b, c, None) == B.MOE_ERR_SHAPE
    assert blocks(a, 2, 128, 136, b, c, None) == B.MOE_ERR_ALIGNMENT
    assert blocks(a, 0, 128, 128, b, c, None) == B.MOE_OK
    assert blocks(a, 3, 0, 128, b, c, None) == B.MOE_OK


def test_noalloc_routing_arguments_are_checked_before_any_cuda_call():
    """Fake, never dereferenced device addresses: every case returns before a CUDA call."""
    lib = B.lib()
    x, w, o, e = 0x10000, 0x20000, 0x30000, 0x40000
    r = B.moe_router(w, None, None)
    rs = B.moe_router(w, None, 0x50000)            # a selection bias, which only the sigmoid gate takes
    f = lib.moe_route_noalloc
    soft, sig = B.MOE_GATE_SOFTMAX, B.MOE_GATE_SIGMOID_BIASED
    call = lambda T=8, d=256, rt=r, N=16, g=soft, K=4, err=e, xp=x: f(xp, T, d, ctypes.byref(rt), N, g, K,
                                                                      o, o, o, o, err, None)
    assert call(T=65537) == B.MOE_ERR_SHAPE           # beyond the static scratch
    assert call(T=-1) == B.MOE_ERR_SHAPE
    assert call(N=257, K=4) == B.MOE_ERR_UNSUPPORTED
    assert call(K=9, N=64) == B.MOE_ERR_UNSUPPORTED
    assert call(K=0) == B.MOE_ERR_INVALID_ARG
    assert call(g=5) == B.MOE_ERR_INVALID_ARG
    assert call(d=200) == B.MOE_ERR_ALIGNMENT
    assert call(err=None) == B.MOE_ERR_INVALID_ARG     # a timeout must have somewhere to be reported
    assert call(err=e + 2) == B.MOE_ERR_ALIGNMENT
    assert call(xp=None) == B.MOE_ERR_INVALID_ARG
    assert call(xp=x + 8) == B.MOE_ERR_ALIGNMENT
    assert call(rt=rs, g=soft) == B.MOE_ERR_INVALID_ARG
    assert call(T=0) == B.MOE_OK                       # nothing to route


def test_status_strings():
    for v, name in [(0, "MOE_OK"), (1, "MOE_ERR_INVALID_ARG"), (7, "MOE_ERR_TIMEOUT"), (99, "MOE_ERR_UNKNOWN")]:
        assert B.status_string(v) == name


def test_header_compiles_as_plain_c_and_links(tmp_path):
    """A C99 program includes the header, links the library and calls the two
    entry points that need no GPU."""
    import shutil
    import subprocess
    cc = shutil.which("gcc") or shutil.which("cc")
    if cc is None:
        pytest.skip("no C compiler")
    src = tmp_path / "abi.c"
    src.write_text(r'''
#include <stdio.h>
#include <string.h>
#include "fgs_moe.h"
int main(void) {
  moe_config c;
  uint64_t bytes = 0;
  memset(&c, 0, sizeof c);
  c.d_model = 2048; c.n_routed = 64; c.d_ff = 1408; c.n_shared = 2; c.d_ff_shared = 1408;
  c.max_tokens = 16384; c.max_k = 6; c.gate = MOE_GATE_SOFTMAX; c.flags = 0;
  if (moe_workspace_bytes(&c, &bytes) != MOE_OK || bytes == 0) return 1;
  if (strcmp(moe_status_string(MOE_ERR_SHAPE), "MOE_ERR_SHAPE") != 0) return 2;
  printf("%llu\n", (unsigned long long)bytes);
  return 0;
}
''')
    lib_dir = os.path.dirname(B.LIB_PATH)
    exe = tmp_path / "abi"
    r = subprocess.run([cc, "-std=c99", "-Wall", "-Werror", str(src), "-I", os.path.join(ROOT, "include"),
                        "-L", lib_dir, "-lfgs_moe", "-Wl,-rpath," + lib_dir, "-o", str(exe)],
                       capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, (r.returncode, r.stderr)
    cfg = B.moe_config(d_model=2048, n_routed=64, d_ff=1408, n_shared=2, d_ff_shared=1408, max_tokens=16384,
                       max_k=6, gate=B.MOE_GATE_SOFTMAX, flags=0)
    want = ctypes.c_uint64()
    assert B.lib().moe_workspace_bytes(ctypes.byref(cfg), ctypes.byref(want)) == B.MOE_OK
    assert int(r.stdout.strip()) == want.value
