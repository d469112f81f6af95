"""Pins of the CPU oracle to things other than itself (no GPU needed).

Each test checks the oracle against a closed form, an invariant, a special
case that reduces to a textbook or library routine, or brute force on tiny
inputs, chosen so that a dropped term, a wrong sign, a wrong index or a
transposed operand anywhere in the oracle fails at least one of them.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import scipy.special
import torch

import oracle as O
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, rng, scale=1.0):
    return rng.standard_normal(shape) * scale


def _silu(a):  # textbook SiLU, scalar
    return a / (1.0 + math.exp(-a))


# ---------------------------------------------------------------------------
# closed form on a hand-built layer
# ---------------------------------------------------------------------------

def _tiny():
    with open(os.path.join(GOLDEN, "tiny_layer.json")) as f:
        g = json.load(f)
    arr = {k: np.array(v, dtype=np.float64) for k, v in g.items()
           if k in ("u", "router", "w_gate", "w_up", "w_down", "ws_gate", "ws_up",
                    "ws_down", "logit_bias_case", "select_bias_case")}
    return g, arr


def _tiny_ffn(i, u0, u1):
    if i == 0:
        v = _silu(u0) * u1
        return (v, 0.0)
    if i == 1:
        v = 2.0 * _silu(u1) * (u0 + u1)
        return (0.0, v)
    v = _silu(u0 + u1) * u0
    return (0.5 * v, -1.0 * v)


def _tiny_expected(u, gate_kind, logit_bias=None, select_bias=None, K=2):
    out = []
    for (u0, u1) in u:
        z = [0.0, u0, u1]
        if logit_bias is not None:
            z = [z[i] + logit_bias[i] for i in range(3)]
        if gate_kind == "softmax":
            den = sum(math.exp(v) for v in z)
            s = [math.exp(v) / den for v in z]
            key = s
        else:
            s = [1.0 / (1.0 + math.exp(-v)) for v in z]
            key = [s[i] + (select_bias[i] if select_bias is not None else 0.0) for i in range(3)]
        sel = sorted(range(3), key=lambda i: (-key[i], i))[:K]
        g = [s[i] for i in sel]
        if gate_kind == "sigmoid":
            tot = sum(g)
            g = [v / tot for v in g]
        sh = _silu(-u0) * u0
        h = [u0 + sh, u1 + sh]
        for gk, i in zip(g, sel):
            f = _tiny_ffn(i, u0, u1)
            h[0] += gk * f[0]
            h[1] += gk * f[1]
        out.append((h, sel, g))
    return out


@pytest.mark.parametrize("case", ["softmax", "softmax_logit_bias", "sigmoid", "sigmoid_select_bias"])
def test_closed_form_tiny_layer(case):
    g, a = _tiny()
    gate = "sigmoid" if case.startswith("sigmoid") else "softmax"
    lb = a["logit_bias_case"] if case == "softmax_logit_bias" else None
    sb = a["select_bias_case"] if case == "sigmoid_select_bias" else None
    h, r = O.moe_forward(a["u"], a["router"], g["K"], (a["w_gate"], a["w_up"], a["w_down"]),
                         (a["ws_gate"], a["ws_up"], a["ws_down"]), gate_kind=gate,
                         logit_bias=lb, select_bias=sb)
    exp = _tiny_expected(g["u"], gate, lb, sb)
    for t, (he, sel, ge) in enumerate(exp):
        assert list(r.idx[t]) == sel, (t, r.idx[t], sel)
        np.testing.assert_allclose(r.gate[t], ge, rtol=1e-13, atol=0)
        np.testing.assert_allclose(h[t], he, rtol=1e-12, atol=1e-14)
    # token 2 has all logits equal: lower indices win the tie
    if case in ("softmax", "sigmoid"):
        assert list(r.idx[2]) == [0, 1]


def test_closed_form_components_by_flag():
    g, a = _tiny()
    ex = (a["w_gate"], a["w_up"], a["w_down"])
    sh = (a["ws_gate"], a["ws_up"], a["ws_down"])
    full, _ = O.moe_forward(a["u"], a["router"], 2, ex, sh)
    parts = [O.moe_forward(a["u"], a["router"], 2, ex, sh, flags=f)[0]
             for f in (O.FLAG_NO_SHARED | O.FLAG_NO_ROUTED,
                       O.FLAG_NO_RESIDUAL | O.FLAG_NO_ROUTED,
                       O.FLAG_NO_RESIDUAL | O.FLAG_NO_SHARED)]
    np.testing.assert_array_equal(parts[0], a["u"])               # residual only
    for t, (u0, u1) in enumerate(g["u"]):                          # shared only
        v = _silu(-u0) * u0
        np.testing.assert_allclose(parts[1][t], [v, v], rtol=1e-13)
    np.testing.assert_allclose(parts[0] + parts[1] + parts[2], full, rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------------------
# library routines and textbook special cases
# ---------------------------------------------------------------------------

def test_softmax_matches_library_and_sums_to_one():
    rng = np.random.default_rng(1)
    z = _rand((50, 64), rng, 3.0)
    s = O.softmax_affinity(z)
    np.testing.assert_allclose(s, scipy.special.softmax(z, axis=1), rtol=1e-13)
    np.testing.assert_allclose(s.sum(axis=1), 1.0, rtol=0, atol=1e-14)


def test_sigmoid_and_silu_match_library():
    rng = np.random.default_rng(2)
    z = _rand((1000,), rng, 5.0)
    np.testing.assert_allclose(O.sigmoid_affinity(z), scipy.special.expit(z), rtol=1e-14)
    ref = torch.nn.functional.silu(torch.from_numpy(z)).numpy()
    np.testing.assert_allclose(O.silu(z), ref, rtol=1e-14, atol=1e-300)


def test_affinity_logits_are_dot_products_with_expert_rows():
    rng = np.random.default_rng(3)
    u, e = _rand((4, 5), rng), _rand((3, 5), rng)
    z = O.affinity_logits(u, e, logit_bias=np.array([0.0, 10.0, -1.0]))
    for t in range(4):
        for i in range(3):
            dot = math.fsum(u[t, j] * e[i, j] for j in range(5))
            assert z[t, i] == pytest.approx(dot + [0.0, 10.0, -1.0][i], rel=1e-14, abs=1e-14)


def test_ffn_one_hot_weights_place_the_product_in_the_right_component():
    # W_gate picks u[a], W_up picks u[b], W_down has one nonzero at [p, q]:
    # FFN(u) = w * SiLU(u[a]) * u[b] in component p, zero elsewhere.
    d, I = 4, 3
    a_, b_, p, q, w = 1, 3, 0, 2, -1.5
    wg = np.zeros((I, d)); wg[q, a_] = 1.0
    wu = np.zeros((I, d)); wu[q, b_] = 1.0
    wd = np.zeros((d, I)); wd[p, q] = w
    u = np.array([[0.3, -0.7, 2.0, 1.25]])
    y = O.swiglu_ffn(u, wg, wu, wd)[0]
    expect = np.zeros(d)
    expect[p] = w * _silu(u[0, a_]) * u[0, b_]
    np.testing.assert_allclose(y, expect, rtol=1e-14, atol=0)


# ---------------------------------------------------------------------------
# selection: brute force over every K-subset
# ---------------------------------------------------------------------------

def _brute_top_k(key, K):
    n = len(key)
    valid = []
    for S in itertools.combinations(range(n), K):
        rest = [key[i] for i in range(n) if i not in S]
        if not rest or min(key[i] for i in S) >= max(rest):
            valid.append(S)
    best = min(valid)  # lexicographically smallest index set among valid ones = ties to lower index
    return sorted(best, key=lambda i: (-key[i], i))


@pytest.mark.parametrize("seed", range(6))
def test_top_k_equals_brute_force_with_forced_ties(seed):
    rng = np.random.default_rng(seed)
    for N in (2, 5, 8):
        for K in range(1, min(N, 4) + 1):
            # keys from a small set of values, so ties are common
            key = rng.integers(0, 4, size=(20, N)).astype(np.float64) / 3.0
            idx = O.select_top_k(key, K)
            for t in range(key.shape[0]):
                assert list(idx[t]) == _brute_top_k(list(key[t]), K)


def test_selection_bias_moves_selection_but_not_gates():
    rng = np.random.default_rng(4)
    u, e = _rand((30, 16), rng), _rand((8, 16), rng, 0.3)
    b = np.zeros(8); b[5] = 10.0                # forces expert 5 into every selection
    r = O.route(u, e, 3, O.GATE_SIGMOID, select_bias=b)
    assert (r.idx[:, 0] == 5).all()
    s = scipy.special.expit(u @ e.T)
    for t in range(30):
        sel = r.idx[t]
        np.testing.assert_allclose(r.gate[t], s[t, sel] / s[t, sel].sum(), rtol=1e-13)
    np.testing.assert_allclose(r.gate.sum(axis=1), 1.0, atol=1e-14)
    # a bias equal for every expert changes nothing
    r0 = O.route(u, e, 3, O.GATE_SIGMOID)
    r1 = O.route(u, e, 3, O.GATE_SIGMOID, select_bias=np.full(8, 0.25))
    np.testing.assert_array_equal(r0.idx, r1.idx)
    np.testing.assert_allclose(r0.gate, r1.gate, rtol=1e-15)


def test_softmax_gates_are_not_renormalised():
    rng = np.random.default_rng(5)
    u, e = _rand((40, 8), rng), _rand((6, 8), rng)
    r = O.route(u, e, 2, O.GATE_SOFTMAX)
    full = scipy.special.softmax(u @ e.T, axis=1)
    np.testing.assert_allclose(r.gate, np.take_along_axis(full, r.idx, 1), rtol=1e-13)
    assert (r.gate.sum(axis=1) < 1.0).all()


# ---------------------------------------------------------------------------
# identities of the method
# ---------------------------------------------------------------------------

def _rand_layer(rng, T, d, N, I, Ks, Is, scale=0.3):
    u = _rand((T, d), rng)
    e = _rand((N, d), rng, scale)
    ex = (_rand((N, I, d), rng, scale), _rand((N, I, d), rng, scale), _rand((N, d, I), rng, scale))
    sh = None
    if Ks:
        sh = (_rand((Ks, Is, d), rng, scale), _rand((Ks, Is, d), rng, scale),
              _rand((Ks, d, Is), rng, scale))
    return u, e, ex, sh


@pytest.mark.parametrize("gate_kind", [O.GATE_SOFTMAX, O.GATE_SIGMOID])
@pytest.mark.parametrize("m", [2, 3])
def test_fine_grained_split_identity(gate_kind, m):
    """Segmenting every expert into m experts of intermediate I/m, replicating
    its affinity vector m times, scaling each segment's W_down by m and
    activating mK experts reproduces the unsplit top-K layer (the
    computation-preserving segmentation of DeepSeekMoE, Abstract and blog
    section 'Fine-Grained Expert Segmentation (Section 3.1)')."""
    rng = np.random.default_rng(10 + m)
    T, d, N, I, K = 24, 12, 5, 6, 2
    u, e, (wg, wu, wd), sh = _rand_layer(rng, T, d, N, I, 1, 4)
    sb = rng.uniform(-0.1, 0.1, N) if gate_kind == O.GATE_SIGMOID else None
    h, r = O.moe_forward(u, e, K, (wg, wu, wd), sh, gate_kind=gate_kind, select_bias=sb)
    assert (r.gap > 1e-9).all()
    seg = I // m
    e2 = np.repeat(e, m, axis=0)
    wg2 = wg.reshape(N * m, seg, d)
    wu2 = wu.reshape(N * m, seg, d)
    wd2 = np.stack([m * wd[i][:, j * seg:(j + 1) * seg] for i in range(N) for j in range(m)])
    sb2 = np.repeat(sb, m) if sb is not None else None
    h2, r2 = O.moe_forward(u, e2, m * K, (wg2, wu2, wd2), sh, gate_kind=gate_kind, select_bias=sb2)
    np.testing.assert_allclose(h2, h, rtol=1e-11, atol=1e-12)
    # the selected segments are exactly the segments of the selected experts
    np.testing.assert_array_equal(np.sort(r2.idx // m, axis=1), np.sort(np.repeat(r.idx, m, axis=1), axis=1))


def test_single_expert_split_reproduces_unsplit_expert():
    rng = np.random.default_rng(20)
    d, I, m = 10, 12, 4
    u = _rand((7, d), rng)
    wg, wu, wd = _rand((I, d), rng), _rand((I, d), rng), _rand((d, I), rng)
    whole = O.swiglu_ffn(u, wg, wu, wd)
    parts = sum(O.swiglu_ffn(u, wg[j::m], wu[j::m], wd[:, j::m]) for j in range(m))
    np.testing.assert_allclose(parts, whole, rtol=1e-12, atol=1e-13)


def test_dense_counterpart_when_all_experts_active():
    """mK = mN with equal affinities: every s = 1/N and the routed part equals
    a dense SwiGLU of intermediate N*I scaled by 1/N (the dense counterpart of
    DeepSeekMoE's Abstract)."""
    rng = np.random.default_rng(21)
    T, d, N, I = 9, 8, 4, 5
    u, _, (wg, wu, wd), sh = _rand_layer(rng, T, d, N, I, 2, 3)
    e = np.tile(_rand((1, d), rng), (N, 1))       # all affinity vectors equal
    h, r = O.moe_forward(u, e, N, (wg, wu, wd), sh)
    np.testing.assert_allclose(r.gate, 1.0 / N, rtol=1e-14)
    dense = O.swiglu_ffn(u, wg.reshape(N * I, d), wu.reshape(N * I, d),
                         np.concatenate(list(wd), axis=1))
    shared = O.swiglu_ffn(u, sh[0].reshape(-1, d), sh[1].reshape(-1, d),
                          np.concatenate(list(sh[2]), axis=1))
    np.testing.assert_allclose(h, u + shared + dense / N, rtol=1e-12, atol=1e-13)


def test_shared_experts_equal_one_concatenated_expert():
    rng = np.random.default_rng(22)
    d, Ks, Is = 6, 3, 4
    u = _rand((5, d), rng)
    wg, wu, wd = _rand((Ks, Is, d), rng), _rand((Ks, Is, d), rng), _rand((Ks, d, Is), rng)
    zero_router = np.zeros((2, d))
    zero_experts = (np.zeros((2, 1, d)), np.zeros((2, 1, d)), np.zeros((2, d, 1)))
    h, _ = O.moe_forward(u, zero_router, 1, zero_experts, (wg, wu, wd),
                         flags=O.FLAG_NO_RESIDUAL | O.FLAG_NO_ROUTED)
    cat = O.swiglu_ffn(u, wg.reshape(Ks * Is, d), wu.reshape(Ks * Is, d),
                       np.concatenate(list(wd), axis=1))
    np.testing.assert_allclose(h, cat, rtol=1e-12, atol=1e-13)


def _brute_gshard_layer(u, e, ex, K):
    """Independent pure-Python top-K MoE: every expert on every token, then a
    mask from brute-force selection (m = 1, K_s = 0 -- GShard's top-K)."""
    wg, wu, wd = ex
    T, d = len(u), len(u[0])
    N, I = len(wg), len(wg[0])
    out = []
    for t in range(T):
        z = [sum(u[t][j] * e[i][j] for j in range(d)) for i in range(N)]
        mx = max(z)
        den = sum(math.exp(v - mx) for v in z)
        s = [math.exp(v - mx) / den for v in z]
        sel = _brute_top_k(s, K)
        h = list(u[t])
        for i in range(N):
            mid = [_silu(sum(wg[i][c][j] * u[t][j] for j in range(d)))
                   * sum(wu[i][c][j] * u[t][j] for j in range(d)) for c in range(I)]
            y = [sum(wd[i][r][c] * mid[c] for c in range(I)) for r in range(d)]
            gate = s[i] if i in sel else 0.0
            h = [h[r] + gate * y[r] for r in range(d)]
        out.append(h)
    return np.array(out)


@pytest.mark.parametrize("seed", range(3))
def test_gshard_reduction_matches_brute_force(seed):
    rng = np.random.default_rng(30 + seed)
    T, d, N, I, K = 6, 5, 5, 3, 2
    u, e, ex, _ = _rand_layer(rng, T, d, N, I, 0, 0, scale=0.6)
    h, _ = O.moe_forward(u, e, K, ex, None)
    ref = _brute_gshard_layer(u.tolist(), e.tolist(), tuple(w.tolist() for w in ex), K)
    np.testing.assert_allclose(h, ref, rtol=1e-11, atol=1e-12)


def test_routed_part_is_linear_in_w_down():
    rng = np.random.default_rng(40)
    u, e, (wg, wu, wd), sh = _rand_layer(rng, 10, 8, 6, 4, 1, 4)
    f = O.FLAG_NO_RESIDUAL | O.FLAG_NO_SHARED
    h1, _ = O.moe_forward(u, e, 3, (wg, wu, wd), sh, flags=f)
    h2, _ = O.moe_forward(u, e, 3, (wg, wu, -2.5 * wd), sh, flags=f)
    np.testing.assert_allclose(h2, -2.5 * h1, rtol=1e-13, atol=1e-15)


def test_tokens_are_independent():
    rng = np.random.default_rng(41)
    u, e, ex, sh = _rand_layer(rng, 16, 8, 6, 4, 2, 3)
    h, _ = O.moe_forward(u, e, 2, ex, sh)
    rows = np.array([11, 2, 7])
    hs, _ = O.moe_forward(u, e, 2, ex, sh, rows=rows)
    np.testing.assert_allclose(hs, h[rows], rtol=1e-14, atol=0)
    perm = rng.permutation(16)
    hp, _ = O.moe_forward(u[perm], e, 2, ex, sh)
    np.testing.assert_allclose(hp, h[perm], rtol=1e-14, atol=0)


# ---------------------------------------------------------------------------
# permutation: invariants and brute force
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("N,K", [(4, 1), (7, 3), (16, 4)])
def test_permutation_matches_sorted_pairs(N, K):
    rng = np.random.default_rng(50 + N)
    T = 37
    idx = np.stack([rng.choice(N, K, replace=False) for _ in range(T)])
    p = O.expert_permutation(idx, N)
    pairs = sorted((int(idx[t, k]), t) for t in range(T) for k in range(K))
    assert list(p.src) == [t for _, t in pairs]
    assert p.counts.sum() == T * K and p.offsets[-1] == T * K
    for i in range(N):
        assert p.counts[i] == sum(1 for e, _ in pairs if e == i)
        assert p.offsets[i] == sum(1 for e, _ in pairs if e < i)
    for t in range(T):
        for k in range(K):
            s = p.slot[t, k]
            assert p.src[s] == t and p.offsets[idx[t, k]] <= s < p.offsets[idx[t, k] + 1]
    assert sorted(p.slot.ravel().tolist()) == list(range(T * K))


# ---------------------------------------------------------------------------
# shapes printed on the pages
# ---------------------------------------------------------------------------

def test_workload_shapes_match_the_pages():
    with open(os.path.join(GOLDEN, "page_shapes.json")) as f:
        g = json.load(f)
    c2, c3, c4, c5 = (W.CONFIGS[k] for k in ("2b", "16b_prefill", "16b_decode", "v3"))
    s2b = g["deepseekmoe_2b"]
    assert (c2.N, c2.Ks, c2.K) == (s2b["n_routed"], s2b["n_shared"], s2b["k_routed"])
    s16 = g["deepseekmoe_16b"]
    for c in (c3, c4):
        assert (c.d, c.N, c.Ks, c.K) == (s16["d_model"], s16["n_routed"], s16["n_shared"], s16["k_routed"])
    sv3 = g["deepseek_v3"]
    assert (c5.N, c5.K, c5.gate) == (sv3["n_routed"], sv3["k_routed"], "sigmoid")
    # the chosen intermediate sizes keep the expert parameters just under the printed totals
    p2b = s2b["layers"] * (c2.N + c2.Ks) * 3 * c2.d * c2.I
    assert 0.85 * s2b["total_params"] <= p2b <= 1.0 * s2b["total_params"]
    p16 = s16["moe_layers"] * (c3.N + c3.Ks) * 3 * c3.d * c3.I
    assert 0.85 * s16["total_params"] <= p16 <= 1.0 * s16["total_params"]


# ---------------------------------------------------------------------------
# auxiliary-loss-free bias update (DeepSeek-V3 summary, section 2)
# ---------------------------------------------------------------------------

def test_bias_update_hand_example():
    # loads 5, 1, 3, 3 (mean 3): the overloaded expert drops, the underloaded rises, the rest stay
    b = np.array([0.25, -0.5, 0.125, 0.0], dtype=np.float32)
    got = O.bias_update(b, [5, 1, 3, 3], 0.0625)
    assert got.dtype == np.float32
    np.testing.assert_array_equal(got, np.array([0.1875, -0.4375, 0.125, 0.0], dtype=np.float32))


def test_bias_update_compares_against_a_fractional_mean_exactly():
    # loads 2 and 1: mean 1.5 lies between them; equal loads leave every bias alone
    np.testing.assert_array_equal(O.bias_update(np.zeros(2, np.float32), [2, 1], 1.0), [-1.0, 1.0])
    np.testing.assert_array_equal(O.bias_update(np.full(6, 0.3, np.float32), [7] * 6, 0.5),
                                  np.full(6, 0.3, np.float32))


def test_bias_update_balances_a_skewed_router():
    """Routing with the updated biases spreads the load: the property the update exists for."""
    rng = np.random.default_rng(31)
    T, d, N, K = 512, 32, 8, 2
    u = rng.standard_normal((T, d))
    e = rng.standard_normal((N, d)) * 0.05
    e[0] += 0.8 * u.mean(axis=0) / np.linalg.norm(u.mean(axis=0))  # experts 0 and 1 favoured
    e[1] += 0.6 * u.mean(axis=0) / np.linalg.norm(u.mean(axis=0))
    u += u.mean(axis=0)

    def max_violation(b):
        r = O.route(u, e, K, "sigmoid", select_bias=b)
        load = np.bincount(r.idx.ravel(), minlength=N)
        return (load.max() - load.mean()) / load.mean(), load

    b = np.zeros(N, np.float32)
    v0, load0 = max_violation(b)
    for _ in range(300):
        _, load = max_violation(b)
        b = O.bias_update(b, load, 0.002)
    v1, _ = max_violation(b)
    assert v0 > 1.0, v0            # the skew is real
    assert v1 < 0.2 * v0, (v0, v1)
    assert b[0] < 0 and b[1] < 0   # the favoured experts were pushed down
