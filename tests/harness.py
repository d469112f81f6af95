"""Shared helpers of the parity tests: upload seeded inputs, run the C ABI,
run the oracle on the same inputs and compare under the stated rules.

Comparison rules
----------------
* expert indices and per-expert token counts: bit-exact, except for tokens
  whose oracle selection keys at positions K and K+1 differ by less than
  1e-6 (a near-tie that float32 rounding may legitimately flip); those
  tokens and the experts at their selection boundary are excluded and
  counted;
* the permutation (src): bit-exact against the oracle's stable counting
  sort of the GPU's own expert indices;
* gates: within 1e-5 absolute;
* the layer output: max |gpu - oracle| <= 2e-2 * RMS(oracle) over the
  compared tokens;
* the routed and the shared terms alone (residual and the other term left
  out): max |gpu - oracle| <= 5e-2 * RMS(oracle term).  Each term is itself
  rounded to bf16 on output (half an ulp, 2^-9 relative, at the largest
  value ~5 RMS: ~1% of RMS), its g-scaled expert rows are rounded to bf16
  before the k-ordered sum (up to K roundings of 2^-9 each, ~sqrt(K) * 1%)
  and so is the SwiGLU intermediate H (2^-9 relative through the down
  projection, ~1%): about 4-5% of RMS in the worst case;
* every compared tensor: RMS(gpu - oracle) <= 1e-2 * RMS(oracle), which a
  dropped or mis-scaled term would exceed by far.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import torch

import oracle as O
import workloads as W
from fine_grained_shared_b200 import moe as B

GAP_EXEMPT = 1e-6
OUT_TOL = 2e-2
TERM_TOL = 5e-2
RMS_TOL = 1e-2
GATE_TOL = 1e-5


def device_inputs(shape: W.LayerShape, host: dict | None = None, dev="cuda"):
    """The layer's inputs on the GPU.  Routed experts are generated one at a
    time (in parallel on the host) and copied into stacked device tensors."""
    host = host if host is not None else W.layer_inputs(shape, with_experts=shape.N * shape.I * shape.d < 2**28)
    out = {k: (v.to(dev) if v is not None else None) for k, v in host.items()
           if k in ("x", "router", "logit_bias", "select_bias", "ws_gate", "ws_up", "ws_down")}
    if "w_gate" in host:
        out["w_gate"], out["w_up"], out["w_down"] = (host["w_gate"].to(dev), host["w_up"].to(dev),
                                                     host["w_down"].to(dev))
    else:
        N, I, d = shape.N, shape.I, shape.d
        wg = torch.empty((N, I, d), dtype=torch.bfloat16, device=dev)
        wu = torch.empty((N, I, d), dtype=torch.bfloat16, device=dev)
        wd = torch.empty((N, d, I), dtype=torch.bfloat16, device=dev)
        workers = min(32, os.cpu_count() or 1)
        with ThreadPoolExecutor(max_workers=workers) as ex:
            for e, (g, u, dn) in enumerate(ex.map(lambda e: W.expert_weights(shape, e), range(N))):
                wg[e].copy_(g)
                wu[e].copy_(u)
                wd[e].copy_(dn)
        out["w_gate"], out["w_up"], out["w_down"] = wg, wu, wd
    return host, out


def make_layer(shape: W.LayerShape, dev_in: dict, flags: int = 0, max_tokens=None, device=0):
    layer = B.MoELayer(d_model=shape.d, n_routed=shape.N, d_ff=shape.I, n_shared=shape.Ks,
                       d_ff_shared=shape.Is, max_tokens=max_tokens or shape.T, max_k=shape.K,
                       gate=shape.gate, flags=flags, device=device)
    shared = (dev_in["ws_gate"], dev_in["ws_up"], dev_in["ws_down"]) if shape.Ks else None
    layer.set_weights(dev_in["router"], (dev_in["w_gate"], dev_in["w_up"], dev_in["w_down"]), shared,
                      logit_bias=dev_in["logit_bias"], select_bias=dev_in["select_bias"])
    return layer


def run(layer, x, K):
    out = layer.forward(x, K)
    st = layer.status()
    assert st == B.MOE_OK, B.status_string(st)
    return out


def oracle_experts(shape: W.LayerShape, host: dict, prefetch=None):
    """The routed experts' weights for the oracle, from the seeded generator:
    the stacked host tensors when the layer is small, else a callable that
    generates (and keeps) each expert on first use.  ``prefetch`` lists experts
    to generate up front, in parallel on the host's cores."""
    if "w_gate" in host:
        return (host["w_gate"], host["w_up"], host["w_down"])
    cache = {}
    if prefetch is not None:
        ids = sorted({int(e) for e in prefetch})
        workers = min(32, os.cpu_count() or 1)
        with ThreadPoolExecutor(max_workers=workers) as ex:
            for e, w in zip(ids, ex.map(lambda e: W.expert_weights(shape, e), ids)):
                cache[e] = w

    def fn(e):
        if e not in cache:
            cache[e] = W.expert_weights(shape, e)
        return cache[e]
    return fn


def stratified_rows(shape: W.LayerShape, ref: O.Routing, tile_rows: int = 128, seed: int = 0):
    """Tokens that put at least one compared row in every GEMM tile of the layer.

    The expert GEMMs run over 128-row m-tiles of each expert's segment of the
    expert-ordered rows (the routed tiles) and over 128-token blocks of x (the
    shared experts' tiles).  For every (expert, m-tile) this picks one token
    whose row lands in that tile -- a seeded random one, its last row for the
    expert's ragged tail -- and one token of every 128-token block of x, plus
    the first and the last token.  Tokens with a near-tie at the selection
    boundary are passed over (another token of the tile stands in).  The tiles
    come from the oracle's own counting sort of its selection, which the GPU's
    permutation must equal bit for bit on every other token.

    Returns (sorted token ids, tiles covered, tiles in all)."""
    rng = np.random.default_rng(seed)
    ok = ref.gap >= GAP_EXEMPT
    perm = O.expert_permutation(ref.idx, shape.N)
    chosen = set()
    covered = total = 0

    def pick(cands):
        cands = [int(t) for t in cands if ok[t]]
        if not cands:
            return False
        chosen.add(cands[int(rng.integers(len(cands)))])
        return True

    for e in range(shape.N):
        lo, hi = int(perm.offsets[e]), int(perm.offsets[e + 1])
        for m0 in range(0, hi - lo, tile_rows):
            total += 1
            rows = perm.src[lo + m0: min(hi, lo + m0 + tile_rows)]
            if ok[rows[-1]] and m0 + tile_rows >= hi - lo:   # the ragged tail's last row
                chosen.add(int(rows[-1]))
                covered += 1
            elif pick(rows):
                covered += 1
    for b0 in range(0, shape.T, tile_rows):
        total += 1
        covered += pick(range(b0, min(shape.T, b0 + tile_rows)))
    for t in (0, shape.T - 1):
        if ok[t]:
            chosen.add(t)
    return np.array(sorted(chosen), dtype=np.int64), covered, total


def oracle_shared(shape, host):
    return (host["ws_gate"], host["ws_up"], host["ws_down"]) if shape.Ks else None


def oracle_routing(shape, host):
    return O.route(host["x"], host["router"], shape.K, shape.gate, host["logit_bias"], host["select_bias"])


def check_routing(shape, layer, ref: O.Routing):
    """Bit-exact idx / counts / src (with the near-tie exemption), gates to 1e-5."""
    T, K, N = shape.T, shape.K, shape.N
    idx, gate, counts, offsets, src = (t.cpu().numpy() for t in layer.routing(T, K))
    exempt = ref.gap < GAP_EXEMPT
    ok = ~exempt
    bad = np.nonzero((idx[ok] != ref.idx[ok]).any(axis=1))[0]
    assert bad.size == 0, (f"{bad.size} tokens with a different selection; first token "
                           f"{np.nonzero(ok)[0][bad[0]]}: gpu {idx[ok][bad[0]]} oracle {ref.idx[ok][bad[0]]} "
                           f"gap {ref.gap[ok][bad[0]]:.3e}")
    # exempted tokens must still pick K distinct experts that the oracle's
    # keys rank within the near-tie
    for t in np.nonzero(exempt)[0]:
        assert len(set(idx[t].tolist())) == K
        kth = np.sort(ref.key[t])[::-1][K - 1]
        assert (ref.key[t][idx[t]] >= kth - 2 * GAP_EXEMPT).all()
    np.testing.assert_allclose(gate[ok], ref.gate[ok], rtol=0, atol=GATE_TOL)
    ref_counts = np.bincount(ref.idx.ravel(), minlength=N)
    boundary = np.zeros(N, dtype=bool)
    for t in np.nonzero(exempt)[0]:
        boundary[idx[t]] = True
        boundary[ref.idx[t]] = True
    np.testing.assert_array_equal(counts[~boundary], ref_counts[~boundary])
    # the permutation of the GPU's own selection is exact
    perm = O.expert_permutation(idx.astype(np.int64), N)
    np.testing.assert_array_equal(counts, perm.counts)
    np.testing.assert_array_equal(offsets, perm.offsets)
    np.testing.assert_array_equal(src, perm.src)
    return int(exempt.sum()), idx


def compare_output(gpu_rows: np.ndarray, ref_rows: np.ndarray, what: str, term: bool = False):
    rms = float(np.sqrt(np.mean(ref_rows ** 2)))
    err = float(np.max(np.abs(gpu_rows - ref_rows)))
    rms_err = float(np.sqrt(np.mean((gpu_rows - ref_rows) ** 2)))
    tol = TERM_TOL if term else OUT_TOL
    assert np.isfinite(gpu_rows).all(), f"{what}: non-finite GPU output"
    assert err <= tol * rms, f"{what}: max|diff| {err:.3e} > {tol} * rms {rms:.3e}"
    assert rms_err <= RMS_TOL * rms, f"{what}: rms(diff) {rms_err:.3e} > {RMS_TOL} * rms {rms:.3e}"
    return err, rms, rms_err
