"""ctypes binding of the C ABI in ``include/fgs_moe.h`` (argument marshalling only).

Every step of the layer runs in ``libfgs_moe.so``; this module only turns
torch tensors into pointers and sizes.  There is no fallback: if the library
is missing the import of :func:`lib` raises.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_int, c_int32, c_int64, c_uint32, c_uint64, c_void_p

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libfgs_moe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_SHAPE = 2
MOE_ERR_ALIGNMENT = 3
MOE_ERR_UNSUPPORTED = 4
MOE_ERR_NOMEM = 5
MOE_ERR_CUDA = 6
MOE_ERR_TIMEOUT = 7

MOE_GATE_SOFTMAX = 0
MOE_GATE_SIGMOID_BIASED = 1

MOE_FLAG_NO_RESIDUAL = 0x1
MOE_FLAG_NO_SHARED = 0x2
MOE_FLAG_NO_ROUTED = 0x4
MOE_FLAG_FP8 = 0x8
MOE_FLAG_DEBUG_WAIT_TIMEOUT = 0x100

KERNEL_NAMES = ("router", "permute", "gate_up", "down", "combine")


class moe_config(ctypes.Structure):
    _fields_ = [("d_model", c_int32), ("n_routed", c_int32), ("d_ff", c_int32),
                ("n_shared", c_int32), ("d_ff_shared", c_int32), ("max_tokens", c_int32),
                ("max_k", c_int32), ("gate", c_int32), ("flags", c_uint32),
                ("route_nodes", c_int32), ("route_max_nodes", c_int32), ("ep_ranks", c_int32),
                ("ep_rank", c_int32)]


class moe_router(ctypes.Structure):
    _fields_ = [("weight", c_void_p), ("logit_bias", c_void_p), ("select_bias", c_void_p)]


class moe_experts(ctypes.Structure):
    _fields_ = [("w_gate", c_void_p), ("w_up", c_void_p), ("w_down", c_void_p)]


class moe_shared(ctypes.Structure):
    _fields_ = [("w_gate", c_void_p), ("w_up", c_void_p), ("w_down", c_void_p)]


class moe_weight_grads(ctypes.Structure):
    _fields_ = [("w_gate", c_void_p), ("w_up", c_void_p), ("w_down", c_void_p),
                ("ws_gate", c_void_p), ("ws_up", c_void_p), ("ws_down", c_void_p)]


class moe_experts_fp8(ctypes.Structure):
    _fields_ = [("w_gate", c_void_p), ("w_up", c_void_p), ("w_down", c_void_p),
                ("s_gate", c_void_p), ("s_up", c_void_p), ("s_down", c_void_p)]


moe_handle = c_void_p

_lib = None


class MoEError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {status_string(status)} ({status})")
        self.status = status


def lib() -> ctypes.CDLL:
    """Load ``libfgs_moe.so`` (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with fine_grained_shared_b200.csrc.build.build()")
    L = ctypes.CDLL(LIB_PATH)
    L.moe_workspace_bytes.argtypes = [POINTER(moe_config), POINTER(c_uint64)]
    L.moe_create.argtypes = [POINTER(moe_config), c_int, POINTER(moe_handle)]
    L.moe_forward.argtypes = [moe_handle, c_void_p, c_int64, POINTER(moe_router), POINTER(moe_experts),
                              POINTER(moe_shared), c_int32, c_void_p, c_void_p]
    L.moe_forward_host.argtypes = L.moe_forward.argtypes
    L.moe_forward_fp8.argtypes = [moe_handle, c_void_p, c_int64, POINTER(moe_router), POINTER(moe_experts_fp8),
                                  POINTER(moe_experts_fp8), c_int32, c_void_p, c_void_p]
    L.moe_get_routing.argtypes = [moe_handle, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]
    L.moe_status_query.argtypes = [moe_handle]
    L.moe_destroy.argtypes = [moe_handle]
    L.moe_set_timing.argtypes = [moe_handle, ctypes.c_uint32]
    L.moe_kernel_times.argtypes = [moe_handle, c_void_p, c_void_p]
    L.moe_route_noalloc.argtypes = [c_void_p, c_int64, c_int32, POINTER(moe_router), c_int32, c_int32, c_int32,
                                    c_void_p, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]
    L.moe_update_bias.argtypes = [moe_handle, c_void_p, ctypes.c_float, c_void_p]
    L.moe_quantize_fp8_rows.argtypes = [c_void_p, c_int64, c_int32, c_void_p, c_void_p, c_void_p]
    L.moe_quantize_fp8_blocks.argtypes = [c_void_p, c_int32, c_int32, c_int32, c_void_p, c_void_p, c_void_p]
    L.moe_backward.argtypes = [moe_handle, c_void_p, c_int64, POINTER(moe_router), POINTER(moe_experts),
                               POINTER(moe_shared), c_int32, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p,
                               POINTER(moe_weight_grads), c_void_p]
    L.moe_ep_workspace.argtypes = [moe_handle, POINTER(c_void_p)]
    L.moe_ep_set_peers.argtypes = [moe_handle, POINTER(c_void_p)]
    L.moe_ep_ipc_handle.argtypes = [moe_handle, c_void_p]
    L.moe_ep_open_peers.argtypes = [moe_handle, c_void_p]
    L.moe_ep_route.argtypes = [moe_handle, c_void_p, c_int64, POINTER(moe_router), c_int32, c_void_p]
    L.moe_ep_dispatch.argtypes = [moe_handle, c_void_p]
    L.moe_ep_experts.argtypes = [moe_handle, POINTER(moe_experts), POINTER(moe_shared), c_void_p]
    L.moe_ep_experts_fp8.argtypes = [moe_handle, POINTER(moe_experts_fp8), POINTER(moe_experts_fp8), c_void_p]
    L.moe_ep_combine.argtypes = [moe_handle, c_void_p, c_void_p]
    L.moe_ep_plan.argtypes = [c_void_p, c_int32, c_int32, c_int32, c_void_p, c_void_p, c_void_p, c_void_p, c_void_p]
    L.moe_status_string.argtypes = [c_int]
    L.moe_status_string.restype = c_char_p
    for name in ("moe_workspace_bytes", "moe_create", "moe_forward", "moe_forward_host", "moe_forward_fp8",
                 "moe_get_routing",
                 "moe_status_query", "moe_destroy", "moe_set_timing", "moe_kernel_times", "moe_route_noalloc",
                 "moe_update_bias", "moe_quantize_fp8_rows", "moe_quantize_fp8_blocks", "moe_backward",
                 "moe_ep_workspace",
                 "moe_ep_set_peers", "moe_ep_ipc_handle", "moe_ep_open_peers", "moe_ep_route", "moe_ep_dispatch",
                 "moe_ep_experts", "moe_ep_experts_fp8", "moe_ep_combine", "moe_ep_plan"):
        getattr(L, name).restype = c_int
    _lib = L
    return L


def status_string(s: int) -> str:
    return lib().moe_status_string(int(s)).decode()


# --- the C entry points under their own names ------------------------------

def moe_workspace_bytes(cfg: moe_config):
    n = c_uint64(0)
    st = lib().moe_workspace_bytes(ctypes.byref(cfg), ctypes.byref(n))
    return st, n.value


def moe_create(cfg: moe_config, device: int = 0):
    h = moe_handle()
    st = lib().moe_create(ctypes.byref(cfg), int(device), ctypes.byref(h))
    return st, h


def moe_forward(h, x, T, router, experts, shared, K, out, stream):
    return lib().moe_forward(h, x, int(T), ctypes.byref(router), ctypes.byref(experts),
                             ctypes.byref(shared) if shared is not None else None, int(K), out, stream)


def moe_forward_host(h, x_host, T, router, experts, shared, K, out_host, stream):
    return lib().moe_forward_host(h, x_host, int(T), ctypes.byref(router), ctypes.byref(experts),
                                  ctypes.byref(shared) if shared is not None else None, int(K),
                                  out_host, stream)


def moe_forward_fp8(h, x, T, router, experts, shared, K, out, stream):
    """The layer forward with FP8 expert GEMMs (handle created with MOE_FLAG_FP8); see the header."""
    return lib().moe_forward_fp8(h, x, int(T), ctypes.byref(router), ctypes.byref(experts),
                                 ctypes.byref(shared) if shared is not None else None, int(K), out, stream)


def moe_get_routing(h, idx, gate, counts, offsets, src, stream):
    return lib().moe_get_routing(h, idx, gate, counts, offsets, src, stream)


def moe_status_query(h):
    return lib().moe_status_query(h)


def moe_destroy(h):
    return lib().moe_destroy(h)


def moe_route_noalloc(x, T, d_model, router, n_routed, gate, K, idx, gate_out, counts, offsets, err, stream):
    """Routing with the library's fixed device scratch (no allocation); see the header."""
    return lib().moe_route_noalloc(x, int(T), int(d_model), ctypes.byref(router), int(n_routed), int(gate),
                                   int(K), idx, gate_out, counts, offsets, err, stream)


def moe_update_bias(h, bias, gamma, stream):
    """One auxiliary-loss-free update of float32 [mN] device biases from the last forward's loads."""
    return lib().moe_update_bias(h, bias, float(gamma), stream)


def moe_set_timing(h, kernel_mask):
    """kernel_mask: bit k times kernel KERNEL_NAMES[k]; 0 turns timing off."""
    return lib().moe_set_timing(h, int(kernel_mask))


def moe_kernel_times(h):
    total = (ctypes.c_float * len(KERNEL_NAMES))()
    count = (c_int32 * len(KERNEL_NAMES))()
    st = lib().moe_kernel_times(h, total, count)
    return st, {n: (float(total[i]), int(count[i])) for i, n in enumerate(KERNEL_NAMES)}


def moe_quantize_fp8_rows(x, rows, cols, q, scale, stream):
    """E4M3 codes and UE8M0 scales of 1 x 128 row groups; see the header."""
    return lib().moe_quantize_fp8_rows(x, int(rows), int(cols), q, scale, stream)


def moe_quantize_fp8_blocks(w, batch, rows, cols, q, scale, stream):
    """E4M3 codes and UE8M0 scales of 128 x 128 blocks of `batch` matrices; see the header."""
    return lib().moe_quantize_fp8_blocks(w, int(batch), int(rows), int(cols), q, scale, stream)


def moe_backward(h, x, T, router, experts, shared, K, dh, dx, d_router, d_logit_bias, dgate, wgrad, stream):
    """The backward of the last moe_forward (input, router and, with wgrad, expert weights); see the header."""
    return lib().moe_backward(h, x, int(T), ctypes.byref(router), ctypes.byref(experts),
                              ctypes.byref(shared) if shared is not None else None, int(K), dh, dx, d_router,
                              d_logit_bias, dgate, ctypes.byref(wgrad) if wgrad is not None else None, stream)


def moe_ep_workspace(h):
    p = c_void_p()
    st = lib().moe_ep_workspace(h, ctypes.byref(p))
    return st, p.value


def moe_ep_set_peers(h, workspaces):
    arr = (c_void_p * len(workspaces))(*workspaces)
    return lib().moe_ep_set_peers(h, arr)


def moe_ep_ipc_handle(h):
    buf = ctypes.create_string_buffer(64)
    st = lib().moe_ep_ipc_handle(h, buf)
    return st, buf.raw


def moe_ep_open_peers(h, handles):
    """handles: one 64-byte IPC handle per rank, in rank order."""
    blob = ctypes.create_string_buffer(b"".join(handles), 64 * len(handles))
    return lib().moe_ep_open_peers(h, blob)


def moe_ep_route(h, x, T, router, K, stream):
    return lib().moe_ep_route(h, x, int(T), ctypes.byref(router), int(K), stream)


def moe_ep_dispatch(h, stream):
    return lib().moe_ep_dispatch(h, stream)


def moe_ep_experts(h, experts, shared, stream):
    return lib().moe_ep_experts(h, ctypes.byref(experts), ctypes.byref(shared) if shared is not None else None,
                                stream)


def moe_ep_experts_fp8(h, experts, shared, stream):
    return lib().moe_ep_experts_fp8(h, ctypes.byref(experts), ctypes.byref(shared) if shared is not None else None,
                                    stream)


def moe_ep_combine(h, out, stream):
    return lib().moe_ep_combine(h, out, stream)


def moe_ep_plan(counts_all, G, n_routed, rank):
    """Host computation of the dispatch plan (no GPU): counts_all int32 [G, mN] (a C-contiguous
    numpy array) -> (status, base [mN], counts_local, row_start, mtile_start, mtile128_start
    [mN / G + 1] each)."""
    import numpy as np
    counts_all = np.ascontiguousarray(counts_all, dtype=np.int32)
    per = max(1, n_routed // max(G, 1))
    base = np.zeros(max(n_routed, 1), np.int32)
    tabs = [np.zeros(per + 1, np.int32) for _ in range(4)]
    st = lib().moe_ep_plan(counts_all.ctypes.data_as(c_void_p), int(G), int(n_routed), int(rank),
                           base.ctypes.data_as(c_void_p), *(t.ctypes.data_as(c_void_p) for t in tabs))
    return (st, base, *tabs)


# --- torch convenience wrapper (pointers and sizes only) --------------------

def _ptr(t):
    return None if t is None else c_void_p(t.data_ptr())


def _stream_ptr(stream):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return c_void_p(s.cuda_stream)


class MoELayer:
    """A handle plus the layer's weights as torch CUDA tensors.

    ``router`` bf16 [mN, d]; ``logit_bias`` / ``select_bias`` float32 [mN] or
    None; ``experts`` = (W_gate [mN,I,d], W_up [mN,I,d], W_down [mN,d,I]);
    ``shared`` = (W_gate [Ks,Is,d], W_up [Ks,Is,d], W_down [Ks,d,Is]) or None.
    """

    def __init__(self, *, d_model, n_routed, d_ff, n_shared, d_ff_shared, max_tokens, max_k,
                 gate="softmax", flags=0, device=0, node_limit=None, ep_ranks=0, ep_rank=0):
        nodes, max_nodes = node_limit if node_limit is not None else (0, 0)
        self.cfg = moe_config(d_model, n_routed, d_ff, n_shared, d_ff_shared if n_shared else 0,
                              max_tokens, max_k,
                              MOE_GATE_SIGMOID_BIASED if gate == "sigmoid" else MOE_GATE_SOFTMAX, flags,
                              nodes, max_nodes, ep_ranks, ep_rank)
        st, self.h = moe_create(self.cfg, device)
        if st != MOE_OK:
            raise MoEError(st, "moe_create")
        self.device = device

    def close(self):
        if self.h:
            moe_destroy(self.h)
            self.h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def set_weights(self, router, experts, shared=None, logit_bias=None, select_bias=None):
        self._keep = (router, experts, shared, logit_bias, select_bias)
        self.router = moe_router(router.data_ptr(), _ptr(logit_bias), _ptr(select_bias))
        self.experts = moe_experts(*(w.data_ptr() for w in experts))
        self.shared = moe_shared(*(w.data_ptr() for w in shared)) if shared is not None else None

    def forward(self, x, K, out=None, stream=None, check=True):
        import torch
        T = x.shape[0]
        if out is None:
            out = torch.empty_like(x)
        st = moe_forward(self.h, _ptr(x), T, self.router, self.experts, self.shared, K, _ptr(out),
                         _stream_ptr(stream))
        if check and st != MOE_OK:
            raise MoEError(st, "moe_forward")
        return out if check else (st, out)

    def backward(self, x, K, dh, dx=None, router_grad=False, weight_grads=False, stream=None):
        """Gradients of the last ``forward(x, K)`` for the upstream gradient dh (bf16 [T, d]):
        returns (dx bf16 [T, d], dgate float32 [T, K], d_router float32 [mN, d] or None,
        d_logit_bias float32 [mN] or None), and with ``weight_grads`` a fifth item: a dict of
        float32 gradients "w_gate", "w_up", "w_down" (and "ws_*" with shared experts) in the
        weights' layouts.  ``router_grad`` asks for d_router (and d_logit_bias when the layer has
        a logit bias)."""
        import torch
        T = x.shape[0]
        dev = x.device
        if dx is None:
            dx = torch.empty_like(x)
        dgate = torch.empty((T, K), dtype=torch.float32, device=dev)
        d_router = torch.empty((self.cfg.n_routed, self.cfg.d_model), dtype=torch.float32, device=dev) \
            if router_grad else None
        d_bias = torch.empty(self.cfg.n_routed, dtype=torch.float32, device=dev) \
            if router_grad and self.router.logit_bias else None
        wg, wgrad = None, None
        if weight_grads:
            c = self.cfg
            N, I, d, Ks, Is = c.n_routed, c.d_ff, c.d_model, c.n_shared, c.d_ff_shared
            f32 = dict(dtype=torch.float32, device=dev)
            wg = {"w_gate": torch.empty((N, I, d), **f32), "w_up": torch.empty((N, I, d), **f32),
                  "w_down": torch.empty((N, d, I), **f32)}
            if Ks:
                wg.update(ws_gate=torch.empty((Ks, Is, d), **f32), ws_up=torch.empty((Ks, Is, d), **f32),
                          ws_down=torch.empty((Ks, d, Is), **f32))
            wgrad = moe_weight_grads(*(wg[k].data_ptr() if k in wg else None
                                       for k in ("w_gate", "w_up", "w_down", "ws_gate", "ws_up", "ws_down")))
        st = moe_backward(self.h, _ptr(x), T, self.router, self.experts, self.shared, K, _ptr(dh), _ptr(dx),
                          _ptr(d_router), _ptr(d_bias), _ptr(dgate), wgrad, _stream_ptr(stream))
        if st != MOE_OK:
            raise MoEError(st, "moe_backward")
        return (dx, dgate, d_router, d_bias) + ((wg,) if weight_grads else ())

    def set_weights_fp8(self, experts_fp8, shared_fp8=None):
        """FP8 expert weights for forward_fp8: (codes, scales) pairs as quantize_fp8_blocks returns
        them, for (W_gate, W_up, W_down) of the routed experts and (when K_s > 0) of the shared ones."""
        def pack(ws):
            (g, sg), (u, su), (dn, sd) = ws
            return moe_experts_fp8(g.data_ptr(), u.data_ptr(), dn.data_ptr(), sg.data_ptr(), su.data_ptr(),
                                   sd.data_ptr())
        self._keep_fp8 = (experts_fp8, shared_fp8)
        self.experts_fp8 = pack(experts_fp8)
        self.shared_fp8 = pack(shared_fp8) if shared_fp8 is not None else None

    def forward_fp8(self, x, K, out=None, stream=None, check=True):
        import torch
        T = x.shape[0]
        if out is None:
            out = torch.empty_like(x)
        st = moe_forward_fp8(self.h, _ptr(x), T, self.router, self.experts_fp8, self.shared_fp8, K, _ptr(out),
                             _stream_ptr(stream))
        if check and st != MOE_OK:
            raise MoEError(st, "moe_forward_fp8")
        return out if check else (st, out)

    def forward_host(self, x_host, K, out_host, stream=None):
        st = moe_forward_host(self.h, c_void_p(x_host.data_ptr()), x_host.shape[0], self.router,
                              self.experts, self.shared, K, c_void_p(out_host.data_ptr()),
                              _stream_ptr(stream))
        if st != MOE_OK:
            raise MoEError(st, "moe_forward_host")
        return out_host

    def update_bias(self, bias, gamma, stream=None):
        """bias: float32 [mN] CUDA tensor (normally the router's select_bias), updated in place
        from the last forward's per-expert loads."""
        st = moe_update_bias(self.h, _ptr(bias), gamma, _stream_ptr(stream))
        if st != MOE_OK:
            raise MoEError(st, "moe_update_bias")
        return bias

    def routing(self, T, K, stream=None):
        import torch
        dev = torch.device("cuda", self.device)
        N = self.cfg.n_routed
        idx = torch.empty((T, K), dtype=torch.int32, device=dev)
        gate = torch.empty((T, K), dtype=torch.float32, device=dev)
        counts = torch.empty(N, dtype=torch.int32, device=dev)
        offsets = torch.empty(N + 1, dtype=torch.int32, device=dev)
        src = torch.empty(T * K, dtype=torch.int32, device=dev)
        st = moe_get_routing(self.h, _ptr(idx), _ptr(gate), _ptr(counts), _ptr(offsets), _ptr(src),
                             _stream_ptr(stream))
        if st != MOE_OK:
            raise MoEError(st, "moe_get_routing")
        return idx, gate, counts, offsets, src

    def status(self):
        return moe_status_query(self.h)

    def set_timing(self, enable=True, kernels=None):
        """Per-kernel CUDA-event timing: of every kernel, or of the named ones (KERNEL_NAMES)."""
        if not enable:
            mask = 0
        elif kernels is None:
            mask = (1 << len(KERNEL_NAMES)) - 1
        else:
            mask = sum(1 << KERNEL_NAMES.index(k) for k in kernels)
        st = moe_set_timing(self.h, mask)
        if st != MOE_OK:
            raise MoEError(st, "moe_set_timing")

    def kernel_times(self):
        st, t = moe_kernel_times(self.h)
        if st != MOE_OK:
            raise MoEError(st, "moe_kernel_times")
        return t


class ExpertParallelLayer(MoELayer):
    """Rank ``ep_rank`` of a layer whose mN routed experts are split over ``ep_ranks`` ranks: it
    holds experts [ep_rank * mN / G, (ep_rank + 1) * mN / G) (``set_weights`` takes those, stacked)
    and all shared experts, and runs the layer for its own tokens.

    A forward is four calls with a barrier across the ranks between them, ordered on the stream
    (see the header): ``forward`` takes that barrier as a callable (``nccl_barrier``);
    ``forward_emulated`` runs the ranks of one process in lockstep on one stream, whose order is
    the barrier.  Peers: ``connect_emulated`` (handles of one process) or ``connect_ipc`` (one
    process per rank)."""

    def __init__(self, *, ep_ranks, ep_rank, **kw):
        super().__init__(ep_ranks=ep_ranks, ep_rank=ep_rank, **kw)
        self.ep_ranks, self.ep_rank = ep_ranks, ep_rank

    def _check(self, st, what):
        if st != MOE_OK:
            raise MoEError(st, what)

    def workspace(self):
        st, p = moe_ep_workspace(self.h)
        self._check(st, "moe_ep_workspace")
        return p

    def set_peers(self, workspaces):
        self._check(moe_ep_set_peers(self.h, workspaces), "moe_ep_set_peers")

    def ipc_handle(self):
        st, hnd = moe_ep_ipc_handle(self.h)
        self._check(st, "moe_ep_ipc_handle")
        return hnd

    def open_peers(self, handles):
        self._check(moe_ep_open_peers(self.h, handles), "moe_ep_open_peers")

    def route(self, x, K, stream=None):
        self._x = x
        self._check(moe_ep_route(self.h, _ptr(x) if x.numel() else None, x.shape[0], self.router, K,
                                 _stream_ptr(stream)), "moe_ep_route")

    def dispatch(self, stream=None):
        self._check(moe_ep_dispatch(self.h, _stream_ptr(stream)), "moe_ep_dispatch")

    def experts_step(self, stream=None):
        if self.cfg.flags & MOE_FLAG_FP8:   # the dispatch sent FP8 rows: the FP8 expert GEMMs
            self._check(moe_ep_experts_fp8(self.h, self.experts_fp8, self.shared_fp8, _stream_ptr(stream)),
                        "moe_ep_experts_fp8")
        else:
            self._check(moe_ep_experts(self.h, self.experts, self.shared, _stream_ptr(stream)), "moe_ep_experts")

    def combine(self, out=None, stream=None):
        import torch
        if out is None:
            out = torch.empty_like(self._x)
        self._check(moe_ep_combine(self.h, _ptr(out) if out.numel() else None, _stream_ptr(stream)),
                    "moe_ep_combine")
        return out

    def forward(self, x, K, barrier, out=None, stream=None):
        """This rank's part of one forward; ``barrier()`` must order every rank's work on the stream."""
        self.route(x, K, stream)
        barrier()
        self.dispatch(stream)
        barrier()
        self.experts_step(stream)
        barrier()
        return self.combine(out, stream)


def connect_emulated(layers):
    """Expert-parallel layers of one process (one GPU, or GPUs with peer access): each learns the
    others' workspaces."""
    ws = [layer.workspace() for layer in layers]
    for layer in layers:
        layer.set_peers(ws)


def connect_ipc(layer, group=None):
    """One process per rank: exchange the workspaces' IPC handles over torch.distributed and open them."""
    import torch.distributed as dist
    handles = [None] * layer.ep_ranks
    dist.all_gather_object(handles, layer.ipc_handle(), group=group)
    layer.open_peers(handles)


def nccl_barrier(device, group=None):
    """A barrier across the ranks ordered on the current stream: a one-element all-reduce."""
    import torch
    import torch.distributed as dist
    flag = torch.zeros(1, dtype=torch.int32, device=device)

    def barrier():
        dist.all_reduce(flag, group=group)
    return barrier


def forward_emulated(layers, xs, K, outs=None, stream=None):
    """The G ranks' forwards in lockstep on one stream (each step of every rank before the next
    step of any): the stream order takes the place of the barriers."""
    for layer, x in zip(layers, xs):
        layer.route(x, K, stream)
    for layer in layers:
        layer.dispatch(stream)
    for layer in layers:
        layer.experts_step(stream)
    return [layer.combine(None if outs is None else outs[r], stream) for r, layer in enumerate(layers)]


def quantize_fp8_rows(x, stream=None):
    """bf16 CUDA tensor [rows, cols] -> (codes uint8 [rows, cols], scales uint8 [rows, ceil(cols/128)])."""
    import torch
    rows, cols = x.shape
    q = torch.empty((rows, cols), dtype=torch.uint8, device=x.device)
    sc = torch.empty((rows, -(-cols // 128)), dtype=torch.uint8, device=x.device)
    st = moe_quantize_fp8_rows(_ptr(x), rows, cols, _ptr(q), _ptr(sc), _stream_ptr(stream))
    if st != MOE_OK:
        raise MoEError(st, "moe_quantize_fp8_rows")
    return q, sc


def quantize_fp8_blocks(w, stream=None):
    """bf16 CUDA tensor [batch, rows, cols] (or [rows, cols]) -> (codes uint8, scales uint8
    [batch, ceil(rows/128), ceil(cols/128)])."""
    import torch
    w3 = w if w.dim() == 3 else w.unsqueeze(0)
    b, rows, cols = w3.shape
    q = torch.empty((b, rows, cols), dtype=torch.uint8, device=w.device)
    sc = torch.empty((b, -(-rows // 128), -(-cols // 128)), dtype=torch.uint8, device=w.device)
    st = moe_quantize_fp8_blocks(_ptr(w3), b, rows, cols, _ptr(q), _ptr(sc), _stream_ptr(stream))
    if st != MOE_OK:
        raise MoEError(st, "moe_quantize_fp8_blocks")
    return (q, sc) if w.dim() == 3 else (q[0], sc[0])
