"""Parity of the sm_100a path (through the C ABI) with the CPU oracle.

Small shapes are compared on every token; the five layer shapes at full size
are compared on their whole routing and on a seeded sample of tokens (tokens
are independent, so a sampled row of the oracle equals that row of the full
layer).  Rules in ``tests/harness.py``.
"""
import ctypes
import numpy as np
import pytest
import torch

import oracle as O
import workloads as W
from fine_grained_shared_b200 import moe as B

from tests import harness as H

pytestmark = pytest.mark.gpu

LS = W.LayerShape
SMALL = {
    "tiny": W.CONFIGS["tiny"],
    "ragged": LS("ragged", T=300, d=208, N=13, I=48, K=3, Ks=2, Is=80, sigma=0.05, bias="normal", seed=11),
    "k1": LS("k1", T=257, d=128, N=8, I=64, K=1, Ks=1, Is=64, sigma=0.05, seed=12),
    "k_equals_n": LS("k_equals_n", T=130, d=64, N=8, I=32, K=8, Ks=1, Is=32, sigma=0.05, seed=13),
    "no_shared": LS("no_shared", T=200, d=256, N=16, I=128, K=4, Ks=0, Is=0, seed=14),
    "one_token": LS("one_token", T=1, d=256, N=16, I=128, K=4, Ks=1, Is=128, seed=15),
    "sigmoid": LS("sigmoid", T=333, d=192, N=40, I=96, K=8, Ks=1, Is=64, gate="sigmoid", sigma=0.03,
                  bias="uniform", seed=16),
    "n256": LS("n256", T=512, d=128, N=256, I=64, K=8, Ks=3, Is=64, sigma=0.05, seed=17),
    "wide_k_dim": LS("wide_k_dim", T=160, d=1104, N=12, I=272, K=2, Ks=1, Is=176, sigma=0.02, seed=18),
    # batches of at most 256 tokens take the CUDA-core router
    "small_sigmoid": LS("small_sigmoid", T=100, d=256, N=40, I=64, K=8, Ks=1, Is=64, gate="sigmoid", sigma=0.03,
                        bias="uniform", seed=19),
    "small_softmax_n256": LS("small_softmax_n256", T=48, d=512, N=256, I=64, K=6, Ks=2, Is=64, sigma=0.03,
                             bias="normal", seed=20),
    # T <= 32: 32-row gate/up and down tiles; T <= 64: 32-row down tiles (the
    # zipf bias piles most tokens onto the first experts, so whole tiles fill)
    "decode_t32": LS("decode_t32", T=32, d=208, N=24, I=160, K=4, Ks=2, Is=96, sigma=0.03, bias="zipf",
                     seed=24),
    "decode_t64": LS("decode_t64", T=64, d=320, N=16, I=144, K=6, Ks=1, Is=80, sigma=0.03, bias="zipf",
                     seed=25),
    "decode_t7_sigmoid": LS("decode_t7_sigmoid", T=7, d=256, N=20, I=96, K=3, Ks=1, Is=64, gate="sigmoid",
                            sigma=0.03, bias="uniform", seed=26),
    # the smallest sizes the ABI accepts: one 16-column k-block, K = N, a single m- and n-tile
    "minimal": LS("minimal", T=5, d=16, N=4, I=16, K=4, Ks=1, Is=16, sigma=0.3, seed=27),
    # batches of at most 64 tokens run the weight-streaming decode GEMMs; these cut tiles between
    # CTAs (stream-K): 18 k-blocks of d against ~5 per CTA, two 32-token blocks (the second ragged),
    # ragged weight blocks (I = 272, d = 1104) and a shared intermediate of 2.75 k-blocks
    "decode_split": LS("decode_split", T=40, d=1104, N=12, I=272, K=2, Ks=1, Is=176, sigma=0.02, seed=29),
    "decode_n256_sigmoid": LS("decode_n256_sigmoid", T=64, d=512, N=256, I=192, K=8, Ks=2, Is=128,
                              gate="sigmoid", sigma=0.02, bias="uniform", seed=30),
}

FLAGS_ROUTED = B.MOE_FLAG_NO_RESIDUAL | B.MOE_FLAG_NO_SHARED
FLAGS_SHARED = B.MOE_FLAG_NO_RESIDUAL | B.MOE_FLAG_NO_ROUTED


def _gpu_rows(out, rows):
    return out.float().cpu().numpy()[rows].astype(np.float64)


def _check_layer(shape, host, dev, rows, routing=None):
    """Whole output and the routed / shared terms alone, on ``rows``."""
    ref_routing_rows = routing.idx[rows] if routing is not None else None
    experts = H.oracle_experts(shape, host, prefetch=None if ref_routing_rows is None
                               else np.unique(ref_routing_rows))
    shared = H.oracle_shared(shape, host)
    ref_routing = routing if routing is not None else H.oracle_routing(shape, host)
    cases = [(0, "output")]
    cases.append((FLAGS_ROUTED, "routed term"))
    if shape.Ks:
        cases.append((FLAGS_SHARED, "shared term"))
    results = {}
    for flags, what in cases:
        layer = H.make_layer(shape, dev, flags=flags)
        out = H.run(layer, dev["x"], shape.K)
        if flags == 0:
            exempt, gpu_idx = H.check_routing(shape, layer, ref_routing)
            results["exempt"] = exempt
        layer.close()
        ref, _ = O.moe_forward(host["x"], host["router"], shape.K, experts, shared, gate_kind=shape.gate,
                               logit_bias=host["logit_bias"], select_bias=host["select_bias"], flags=flags,
                               rows=rows, routing=ref_routing)
        results[what] = H.compare_output(_gpu_rows(out, rows), ref, f"{shape.name} {what}", term=flags != 0)
    return results


@pytest.mark.parametrize("name", sorted(SMALL))
def test_small_shapes_every_token(name):
    shape = SMALL[name]
    host, dev = H.device_inputs(shape)
    ref = H.oracle_routing(shape, host)
    rows = np.nonzero(ref.gap >= H.GAP_EXEMPT)[0]   # near-tied tokens compared by routing rules only
    _check_layer(shape, host, dev, rows, ref)


@pytest.mark.parametrize("name", ["2b", "16b_prefill", "16b_decode", "v3"])
def test_full_size_layers(name):
    """The whole routing on every token, and the output on a token set that
    puts a compared row in every (expert, 128-row m-tile) GEMM tile and in
    every 128-token tile of the shared experts."""
    shape = W.CONFIGS[name]
    host, dev = H.device_inputs(shape)
    ref = H.oracle_routing(shape, host)
    rows, covered, total = H.stratified_rows(shape, ref)
    assert covered == total, f"{total - covered} of {total} GEMM tiles have no comparable token"
    if shape.T <= 512:          # a decode batch: every token
        rows = np.nonzero(ref.gap >= H.GAP_EXEMPT)[0]
    res = _check_layer(shape, host, dev, rows, ref)
    print(f"{name}: exempt tokens {res['exempt']}, compared rows {rows.size}, tiles covered {covered}/{total}, "
          + ", ".join(f"{k}: max err {v[0]:.2e} rms err {v[2]:.2e} rms {v[1]:.2e}"
                      for k, v in res.items() if k != "exempt"))


def _custom_layer(shape, router=None, logit_bias=None):
    host = W.layer_inputs(shape)
    if router is not None:
        host["router"] = router
    if logit_bias is not None:
        host["logit_bias"] = logit_bias
    return H.device_inputs(shape, host)


@pytest.mark.parametrize("T", [384, 200])  # tensor-core router, CUDA-core router
def test_exact_ties_go_to_the_lower_expert_index(T):
    """Integer-valued tokens and affinity vectors: every logit is an integer
    of magnitude <= 256, exact in float32 whatever the summation order, so
    ties are exact on both sides and must go to the lower expert index on
    every token (no near-tie exemption)."""
    shape = LS("ties", T=T, d=128, N=12, I=64, K=3, Ks=1, Is=64, sigma=0.05, seed=21)
    g = torch.Generator().manual_seed(21)
    x = torch.randint(-2, 3, (shape.T, shape.d), generator=g).to(torch.bfloat16)
    r = torch.randint(-1, 2, (shape.N, shape.d), generator=g).to(torch.bfloat16)
    r[1] = r[0]
    r[2] = r[0]          # experts 0, 1, 2 always tie
    r[7] = r[5]
    r[9] = r[5]          # experts 5, 7, 9 always tie
    host = W.layer_inputs(shape)
    host["x"], host["router"] = x, r
    host, dev = H.device_inputs(shape, host)
    ref = H.oracle_routing(shape, host)
    assert (ref.gap == 0).sum() > T // 8         # many tokens tie at the selection boundary
    layer = H.make_layer(shape, dev)
    out = H.run(layer, dev["x"], shape.K)
    idx = layer.routing(shape.T, shape.K)[0].cpu().numpy()
    np.testing.assert_array_equal(idx, ref.idx)
    has = lambda e: (idx == e).any(axis=1)
    assert (~has(1) | has(0)).all() and (~has(2) | (has(0) & has(1))).all()
    assert (~has(7) | has(5)).all() and (~has(9) | (has(5) & has(7))).all()
    h, _ = O.moe_forward(host["x"], host["router"], shape.K, H.oracle_experts(shape, host),
                         H.oracle_shared(shape, host), routing=ref)
    H.compare_output(_gpu_rows(out, slice(None)), h, "ties output")


def test_duplicated_expert_rows_tie_exactly():
    """Random-valued affinity vectors with duplicated rows: the tensor cores
    give the copies bit-identical logits, so the copies tie exactly and the
    lower index must win on every token (no near-tie exemption)."""
    shape = LS("ties_rand", T=2048, d=512, N=12, I=64, K=3, Ks=1, Is=64, sigma=0.05, seed=21)
    host = W.layer_inputs(shape)
    r = host["router"].clone()
    r[1] = r[0]
    r[2] = r[0]
    r[7] = r[5]
    r[9] = r[5]
    host["router"] = r
    host, dev = H.device_inputs(shape, host)
    ref = H.oracle_routing(shape, host)
    assert (ref.gap == 0).sum() > 200
    layer = H.make_layer(shape, dev)
    H.run(layer, dev["x"], shape.K)
    idx = layer.routing(shape.T, shape.K)[0].cpu().numpy()
    np.testing.assert_array_equal(idx, ref.idx)


@pytest.mark.parametrize("T", [300, 100])  # tensor-core router, CUDA-core router
def test_non_finite_tokens_still_route_to_valid_experts(T):
    """A token whose row holds a NaN (or an infinity) has NaN affinities.  Its
    K slots must still name K distinct experts in [0, mN) (a NaN key ranks
    below every number, ties to the lower index), the counts must add up to
    T*K, and every other token must be unaffected."""
    shape = LS("nan_rows", T=T, d=256, N=24, I=64, K=4, Ks=1, Is=64, sigma=0.05, seed=28)
    host = W.layer_inputs(shape)
    bad = [0, 5, T // 2, T - 1]
    x = host["x"].clone()
    x[bad[0], 3] = float("nan")
    x[bad[1], :] = float("nan")
    x[bad[2], 7] = float("inf")
    x[bad[3], 0] = float("-inf")
    host_bad = dict(host, x=x)
    _, dev = H.device_inputs(shape, host_bad)
    layer = H.make_layer(shape, dev)
    out = H.run(layer, dev["x"], shape.K)
    idx, gate, counts, offsets, src = (t.cpu().numpy() for t in layer.routing(shape.T, shape.K))
    assert ((idx >= 0) & (idx < shape.N)).all()
    assert all(len(set(r)) == shape.K for r in idx.tolist())
    assert counts.sum() == T * shape.K
    np.testing.assert_array_equal(counts, np.bincount(idx.ravel(), minlength=shape.N))
    good = np.setdiff1d(np.arange(T), bad)
    ref = H.oracle_routing(shape, host)           # the finite tokens' routing does not depend on the others
    ok = good[ref.gap[good] >= H.GAP_EXEMPT]
    np.testing.assert_array_equal(idx[ok], ref.idx[ok])
    np.testing.assert_allclose(gate[ok], ref.gate[ok], rtol=0, atol=H.GATE_TOL)
    h, _ = O.moe_forward(host["x"], host["router"], shape.K, H.oracle_experts(shape, host),
                         H.oracle_shared(shape, host), routing=ref, rows=ok)
    H.compare_output(_gpu_rows(out, ok), h, "finite tokens beside non-finite ones")


def _node_limited_gaps(key, K, nodes, M):
    """Per token: the gap between the M-th and (M+1)-th node scores (a node's largest key) and
    between the K-th and (K+1)-th keys among the chosen nodes' experts (+inf where there is none);
    a gap under the near-tie threshold may flip in float32."""
    T, N = key.shape
    per = N // nodes
    ns = np.sort(key.reshape(T, nodes, per).max(axis=2), axis=1)[:, ::-1]
    node_gap = ns[:, M - 1] - ns[:, M] if M < nodes else np.full(T, np.inf)
    chosen = np.argsort(-key.reshape(T, nodes, per).max(axis=2), axis=1, kind="stable")[:, :M]
    allowed = np.zeros((T, nodes), dtype=bool)
    np.put_along_axis(allowed, chosen, True, axis=1)
    masked = np.where(np.repeat(allowed, per, axis=1), key, -np.inf)
    srt = -np.sort(-masked, axis=1)
    k_gap = srt[:, K - 1] - srt[:, K] if K < M * per else np.full(T, np.inf)
    return np.minimum(node_gap, k_gap)


@pytest.mark.parametrize("case", ["tc_softmax", "small_sigmoid", "v3_like", "decode_softmax"])
def test_node_limited_routing_matches_the_oracle(case):
    """Node-limited routing (DeepSeek-V3 report summary, section 2): each token's K experts come
    from at most M nodes, those holding its largest keys; bit-exact against the oracle's
    select_top_k_node_limited except at near-ties, and the layer's output as the oracle's."""
    spec = {"tc_softmax": (LS("nl_soft", T=300, d=256, N=64, I=64, K=6, Ks=1, Is=64, sigma=0.05, seed=71), 8, 3),
            "small_sigmoid": (LS("nl_sig", T=100, d=256, N=64, I=64, K=6, Ks=1, Is=64, gate="sigmoid",
                                 sigma=0.03, bias="uniform", seed=72), 4, 2),
            "v3_like": (LS("nl_v3", T=1000, d=512, N=256, I=64, K=8, Ks=1, Is=64, gate="sigmoid", sigma=0.006,
                           bias="uniform", seed=73), 8, 4),
            # a decode batch: one router CTA per token, the tables built by the permutation
            "decode_softmax": (LS("nl_dec", T=48, d=512, N=64, I=64, K=6, Ks=1, Is=64, sigma=0.05, seed=74), 8, 3)}[case]
    shape, nodes, M = spec
    host, dev = H.device_inputs(shape)
    layer = B.MoELayer(d_model=shape.d, n_routed=shape.N, d_ff=shape.I, n_shared=shape.Ks, d_ff_shared=shape.Is,
                       max_tokens=shape.T, max_k=shape.K, gate=shape.gate, node_limit=(nodes, M))
    layer.set_weights(dev["router"], (dev["w_gate"], dev["w_up"], dev["w_down"]),
                      (dev["ws_gate"], dev["ws_up"], dev["ws_down"]), logit_bias=dev["logit_bias"],
                      select_bias=dev["select_bias"])
    out = H.run(layer, dev["x"], shape.K)
    idx, gate, counts, offsets, src = (t.cpu().numpy() for t in layer.routing(shape.T, shape.K))
    ref = O.route(host["x"], host["router"], shape.K, shape.gate, host["logit_bias"], host["select_bias"],
                  node_limit=(nodes, M))
    ok = _node_limited_gaps(ref.key, shape.K, nodes, M) >= H.GAP_EXEMPT
    assert ok.sum() > 0.9 * shape.T
    np.testing.assert_array_equal(idx[ok], ref.idx[ok])
    np.testing.assert_allclose(gate[ok], ref.gate[ok], rtol=0, atol=H.GATE_TOL)
    per = shape.N // nodes
    assert all(len(set(r)) == shape.K and len({e // per for e in r}) <= M for r in idx.tolist())
    perm = O.expert_permutation(idx.astype(np.int64), shape.N)
    np.testing.assert_array_equal(counts, perm.counts)
    np.testing.assert_array_equal(src, perm.src)
    rows = np.nonzero(ok)[0]
    h, _ = O.moe_forward(host["x"], host["router"], shape.K, H.oracle_experts(shape, host),
                         H.oracle_shared(shape, host), gate_kind=shape.gate, logit_bias=host["logit_bias"],
                         select_bias=host["select_bias"], routing=ref, rows=rows)
    H.compare_output(_gpu_rows(out, rows), h, f"{case} output")
    # without the limit the same inputs route differently on some tokens (the limit is live)
    free = O.route(host["x"], host["router"], shape.K, shape.gate, host["logit_bias"], host["select_bias"])
    assert (free.idx != ref.idx).any()


def test_zero_router_sends_every_token_to_the_first_experts():
    shape = LS("zero_router", T=700, d=128, N=16, I=64, K=4, Ks=1, Is=64, sigma=0.05, seed=22)
    host, dev = _custom_layer(shape, router=torch.zeros((16, 128), dtype=torch.bfloat16))
    layer = H.make_layer(shape, dev)
    out = H.run(layer, dev["x"], shape.K)
    idx, gate, counts, offsets, src = (t.cpu().numpy() for t in layer.routing(shape.T, shape.K))
    assert (idx == np.arange(4)[None, :]).all()
    np.testing.assert_allclose(gate, 1.0 / 16, rtol=1e-6)
    assert counts.tolist() == [700] * 4 + [0] * 12
    ref = H.oracle_routing(shape, host)
    h, _ = O.moe_forward(host["x"], host["router"], shape.K, H.oracle_experts(shape, host),
                         H.oracle_shared(shape, host), routing=ref)
    H.compare_output(_gpu_rows(out, slice(None)), h, "zero router output")


def test_one_expert_takes_every_token():
    shape = LS("skew", T=1000, d=256, N=32, I=128, K=2, Ks=1, Is=128, sigma=0.02, bias="normal", seed=23)
    lb = torch.zeros(32)
    lb[5] = 4.0          # expert 5 leads every token; the others keep real score gaps
    host, dev = _custom_layer(shape, logit_bias=lb)
    ref = H.oracle_routing(shape, host)
    layer = H.make_layer(shape, dev)
    out = H.run(layer, dev["x"], shape.K)
    H.check_routing(shape, layer, ref)
    counts = layer.routing(shape.T, shape.K)[2].cpu().numpy()
    assert counts[5] == 1000
    h, _ = O.moe_forward(host["x"], host["router"], shape.K, H.oracle_experts(shape, host),
                         H.oracle_shared(shape, host), routing=ref, logit_bias=host["logit_bias"])
    rows = np.nonzero(ref.gap >= H.GAP_EXEMPT)[0]
    H.compare_output(_gpu_rows(out, rows), h[rows], "skewed output")


def test_runs_are_bitwise_deterministic():
    shape = W.CONFIGS["tiny"].with_(T=512)
    host, dev = H.device_inputs(shape)
    layer = H.make_layer(shape, dev)
    a = H.run(layer, dev["x"], shape.K).clone()
    b = H.run(layer, dev["x"], shape.K).clone()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("name", ["decode_t32", "16b_decode"])
def test_small_batch_forwards_back_to_back(name):
    """Twenty forwards queued without a synchronize in between give the same bits as one."""
    shape = SMALL[name] if name in SMALL else W.CONFIGS[name]
    host, dev = H.device_inputs(shape)
    layer = H.make_layer(shape, dev)
    ref = H.run(layer, dev["x"], shape.K).clone()
    out = torch.empty_like(ref)
    for _ in range(20):
        layer.forward(dev["x"], shape.K, out)
    assert layer.status() == B.MOE_OK
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))


def test_smaller_batches_reuse_one_handle():
    shape = SMALL["ragged"]
    host, dev = H.device_inputs(shape)
    layer = H.make_layer(shape, dev)
    full = H.run(layer, dev["x"], shape.K).float().cpu()
    for T in (1, 77, 128, 129, 300):
        x = dev["x"][:T].contiguous()
        part = H.run(layer, x, shape.K).float().cpu()
        # tokens are independent: a prefix batch gives the prefix rows (up to summation order)
        assert torch.allclose(part, full[:T], atol=1e-2, rtol=0)
    # K below max_k
    out = H.run(layer, dev["x"], 2)
    ref = O.route(host["x"], host["router"], 2, "softmax", host["logit_bias"])
    h, _ = O.moe_forward(host["x"], host["router"], 2, H.oracle_experts(shape, host),
                         H.oracle_shared(shape, host), routing=ref)
    rows = np.nonzero(ref.gap >= H.GAP_EXEMPT)[0]
    H.compare_output(_gpu_rows(out, rows), h[rows], "K=2 on a K=3 handle")


@pytest.mark.parametrize("T", [512, 4096, 9000])  # one chunk; 2 chunks; 4 uneven chunks
def test_host_buffer_entry_point_matches_device_entry_point(T):
    """The host-buffer forward (copies pipelined with token chunks for large T)
    gives the device forward's bits: tokens are independent."""
    shape = W.CONFIGS["tiny"].with_(T=T)
    host, dev = H.device_inputs(shape)
    layer = H.make_layer(shape, dev)
    dev_out = H.run(layer, dev["x"], shape.K).cpu()
    x_pinned = host["x"].pin_memory()
    out_pinned = torch.empty_like(x_pinned).pin_memory()
    layer.forward_host(x_pinned, shape.K, out_pinned)
    assert torch.equal(out_pinned.view(torch.int16), dev_out.view(torch.int16))


def test_empty_batch_is_a_no_op():
    shape = W.CONFIGS["tiny"]
    host, dev = H.device_inputs(shape)
    layer = H.make_layer(shape, dev)
    x = torch.empty((0, shape.d), dtype=torch.bfloat16, device="cuda")
    st, _ = layer.forward(x, shape.K, out=torch.empty_like(x), check=False)
    assert st == B.MOE_OK


def test_bad_arguments_are_rejected_before_launch():
    shape = W.CONFIGS["tiny"]
    host, dev = H.device_inputs(shape)
    layer = H.make_layer(shape, dev)
    x = dev["x"]
    out = torch.empty_like(x)
    assert layer.forward(x, 0, out, check=False)[0] == B.MOE_ERR_INVALID_ARG
    assert layer.forward(x, shape.K + 1, out, check=False)[0] == B.MOE_ERR_INVALID_ARG
    big = torch.zeros((shape.T + 1, shape.d), dtype=torch.bfloat16, device="cuda")
    assert layer.forward(big, shape.K, torch.empty_like(big), check=False)[0] == B.MOE_ERR_SHAPE
    assert layer.forward(x, shape.K, x, check=False)[0] == B.MOE_ERR_INVALID_ARG       # out aliases x
    buf = torch.zeros(shape.T * shape.d + 8, dtype=torch.bfloat16, device="cuda")
    mis = buf[1:1 + shape.T * shape.d].view(shape.T, shape.d)                           # 2-byte offset
    assert layer.forward(mis, shape.K, out, check=False)[0] == B.MOE_ERR_ALIGNMENT
    saved = layer.shared
    layer.shared = None
    assert layer.forward(x, shape.K, out, check=False)[0] == B.MOE_ERR_INVALID_ARG     # Ks > 0 needs shared
    layer.shared = saved
    layer.router.select_bias = dev["x"].data_ptr()                                      # sigmoid-only input
    assert layer.forward(x, shape.K, out, check=False)[0] == B.MOE_ERR_INVALID_ARG
    layer.router.select_bias = None
    assert layer.status() == B.MOE_OK
    H.run(layer, x, shape.K)


@pytest.mark.parametrize("tokens", [None, 32], ids=["grouped_gemms", "decode_ffn"])
def test_device_wait_timeout_is_reported_and_the_context_stays_usable(tokens):
    """A bounded wait that runs out (a barrier nothing arrives on) in the grouped GEMMs of a prefill batch,
    or in the decode FFN of a batch of 32 tokens: the call reports MOE_ERR_TIMEOUT, every other CTA stops
    within its own limit, and the next forward on the same handle and on a new one is correct."""
    shape = W.CONFIGS["tiny"]
    host, dev = H.device_inputs(shape)
    x = dev["x"] if tokens is None else dev["x"][:tokens]
    bad = H.make_layer(shape, dev, flags=B.MOE_FLAG_DEBUG_WAIT_TIMEOUT)
    for _ in range(2):                       # the handle's counters are left usable after the error
        bad.forward(x, shape.K)
        assert bad.status() == B.MOE_ERR_TIMEOUT
        assert bad.status() == B.MOE_OK      # the error word is cleared once reported
    bad.close()
    good = H.make_layer(shape, dev)
    ref = H.oracle_routing(shape, host)
    h, _ = O.moe_forward(host["x"], host["router"], shape.K, H.oracle_experts(shape, host),
                         H.oracle_shared(shape, host), routing=ref)
    rows = np.nonzero(ref.gap >= H.GAP_EXEMPT)[0]
    if tokens is not None:
        rows = rows[rows < tokens]
    out = H.run(good, x, shape.K)
    H.compare_output(_gpu_rows(out, rows), h[rows], "after a timeout")


# ---------------------------------------------------------------------------
# auxiliary-loss-free bias update
# ---------------------------------------------------------------------------

def test_bias_update_matches_the_oracle_bit_for_bit():
    shape = SMALL["sigmoid"]
    host, dev = H.device_inputs(shape)
    layer = H.make_layer(shape, dev)
    bias = dev["select_bias"].clone()
    with pytest.raises(B.MoEError):
        layer.update_bias(bias, 0.01)          # no forward yet: no loads to balance
    H.run(layer, dev["x"], shape.K)
    _, _, counts, _, _ = layer.routing(shape.T, shape.K)
    counts = counts.cpu().numpy()
    for gamma in (0.01, 1e-3):
        before = bias.cpu().numpy()
        layer.update_bias(bias, gamma)
        torch.cuda.synchronize()
        want = O.bias_update(before, counts, gamma)
        np.testing.assert_array_equal(bias.cpu().numpy(), want)
    with pytest.raises(B.MoEError):
        layer.update_bias(bias, float("nan"))
    raw = torch.zeros(4 * shape.N + 4, dtype=torch.uint8, device="cuda")
    assert B.moe_update_bias(layer.h, ctypes.c_void_p(raw.data_ptr() + 2), 0.1, None) == B.MOE_ERR_INVALID_ARG


def test_bias_update_balances_a_skewed_layer_on_the_gpu():
    """Forward, update, repeat: the routed load evens out (the reason for the update)."""
    shape = LS("skewed", T=2048, d=256, N=16, I=64, K=2, Ks=1, Is=64, gate="sigmoid", sigma=0.05,
               bias="uniform", seed=41)
    host = W.layer_inputs(shape)
    mean_dir = host["x"].float().mean(dim=0)
    mean_dir = mean_dir / mean_dir.norm()
    router = host["router"].float()
    router[0] += 0.6 * mean_dir
    router[1] += 0.4 * mean_dir
    host["router"] = router.to(torch.bfloat16)
    host["x"] = (host["x"].float() + 3.0 * mean_dir).to(torch.bfloat16)
    _, dev = H.device_inputs(shape, host)
    layer = H.make_layer(shape, dev)
    bias = torch.zeros(shape.N, dtype=torch.float32, device="cuda")
    layer.set_weights(dev["router"], (dev["w_gate"], dev["w_up"], dev["w_down"]),
                      (dev["ws_gate"], dev["ws_up"], dev["ws_down"]), select_bias=bias)

    def max_violation():
        H.run(layer, dev["x"], shape.K)
        c = layer.routing(shape.T, shape.K)[2].cpu().numpy()
        return (c.max() - c.mean()) / c.mean()

    v0 = max_violation()
    for _ in range(150):
        max_violation()
        layer.update_bias(bias, 0.002)
    v1 = max_violation()
    assert v0 > 1.0, v0
    assert v1 < 0.3 * v0, (v0, v1)


# ---------------------------------------------------------------------------
# seeded random shapes: every size the ABI accepts at small scale
# ---------------------------------------------------------------------------

def _random_shape(seed: int) -> W.LayerShape:
    rng = np.random.default_rng(1000 + seed)
    N = int(rng.choice([1, 2, 3, 5, 8, 13, 24, 40, 64, 100]))
    K = int(rng.integers(1, min(8, N) + 1))
    Ks = int(rng.integers(0, 3))
    gate = "sigmoid" if rng.random() < 0.4 else "softmax"
    bias = ("uniform" if rng.random() < 0.7 else "none") if gate == "sigmoid" else \
        str(rng.choice(["none", "normal", "zipf"]))
    return LS(f"random{seed}", T=int(rng.integers(1, 700)), d=16 * int(rng.integers(1, 33)),
              N=N, I=16 * int(rng.integers(1, 21)), K=K, Ks=Ks, Is=16 * int(rng.integers(1, 17)) if Ks else 0,
              gate=gate, sigma=0.02, bias=bias, seed=5000 + seed)


@pytest.mark.parametrize("seed", range(12))
def test_random_shapes_every_token(seed):
    shape = _random_shape(seed)
    host, dev = H.device_inputs(shape)
    ref = H.oracle_routing(shape, host)
    rows = np.nonzero(ref.gap >= H.GAP_EXEMPT)[0]
    _check_layer(shape, host, dev, rows, ref)


def test_timing_records_only_the_kernels_asked_for():
    shape = SMALL["tiny"]
    host, dev = H.device_inputs(shape)
    layer = H.make_layer(shape, dev)
    layer.set_timing(True, kernels=["gate_up"])
    for _ in range(3):
        H.run(layer, dev["x"], shape.K)
    t = layer.kernel_times()
    assert t["gate_up"][1] == 3 and t["gate_up"][0] > 0
    assert all(n == 0 for k, (_, n) in t.items() if k != "gate_up")
    layer.set_timing(True)
    H.run(layer, dev["x"], shape.K)
    assert all(n == 1 for _, n in layer.kernel_times().values())
    # a decode-sized batch: routing and permutation in one launch (timed as the router), both expert
    # GEMMs in another (timed as gate_up)
    small = dev["x"][:40].contiguous()
    H.run(layer, small, shape.K)
    t = layer.kernel_times()
    assert t["permute"][1] == 0 and t["down"][1] == 0
    assert all(n == 1 for k, (_, n) in t.items() if k not in ("permute", "down"))
    layer.set_timing(False)
    H.run(layer, dev["x"], shape.K)
    assert all(n == 0 for _, n in layer.kernel_times().values())
    assert B.moe_set_timing(layer.h, 1 << len(B.KERNEL_NAMES)) == B.MOE_ERR_INVALID_ARG

