"""Pins of the node-limited top-K (``oracle.select_top_k_node_limited``).

A hand-worked example that separates the reading taken (a node ranks by its
best expert's key) from a sum-of-keys score; the special case of M = all
nodes (plain top-K, itself pinned by brute force); an independent pure-Python
statement of the same rule as a walk down the experts; and the properties the
restriction must have.
"""
import numpy as np
import pytest

import oracle as O
import oracle.moe_oracle as M


def test_hand_example():
    # 8 experts on 4 nodes: node 0 = {0, 1}, node 1 = {2, 3}, node 2 = {4, 5}, node 3 = {6, 7}
    key = np.array([
        # A: node maxima 0.10, 0.30, 0.25, 0.03 -> nodes 1, 2 -> experts 2 (0.30), 4 (0.25), 5 (0.24)
        [0.10, 0.05, 0.30, 0.02, 0.25, 0.24, 0.01, 0.03],
        # C: plain top-3 = 0, 2, 4 spans three nodes; node maxima 0.20, 0.19, 0.18, 0.04 -> nodes 0, 1
        #    -> experts 0 (0.20), 2 (0.19), 3 (0.02).  (A sum-of-keys node score would pick node 2,
        #    0.18 + 0.17 = 0.35, and give 0, 4, 5.)
        [0.20, 0.01, 0.19, 0.02, 0.18, 0.17, 0.03, 0.04],
    ])
    got = M.select_top_k_node_limited(key, 3, 4, 2)
    assert got.tolist() == [[2, 4, 5], [0, 2, 3]]
    # D: M = 1, nodes 0 and 1 tie at 0.3 -> the lower node, 0 -> experts 0 (0.3), 1 (0.0)
    tie = np.array([[0.3, 0.0, 0.0, 0.3, 0.1, 0.0, 0.0, 0.0]])
    assert M.select_top_k_node_limited(tie, 2, 4, 1).tolist() == [[0, 1]]


def test_all_nodes_allowed_is_plain_top_k():
    rng = np.random.default_rng(1)
    key = np.round(rng.random((200, 24)), 2)          # coarse grid: many ties
    for nodes in (1, 2, 3, 4, 6, 8, 12, 24):
        for K in (1, 3, 8):
            assert np.array_equal(M.select_top_k_node_limited(key, K, nodes, nodes), M.select_top_k(key, K))


def _walk(key_row, K, nodes, limit):
    """The rule as the pages put it: go down the experts by affinity, collecting the nodes
    that hold them until `limit` nodes are found; then the best K experts on those nodes."""
    N = len(key_row)
    per = N // nodes
    order = sorted(range(N), key=lambda i: (-key_row[i], i))
    chosen = []
    for i in order:
        if i // per not in chosen:
            chosen.append(i // per)
        if len(chosen) == limit:
            break
    allowed = [i for i in order if i // per in chosen]
    return allowed[:K]


@pytest.mark.parametrize("seed", [2, 3])
def test_matches_the_walk_down_the_experts(seed):
    rng = np.random.default_rng(seed)
    for N, nodes, limit, K in [(16, 4, 2, 4), (64, 8, 4, 6), (256, 8, 4, 8), (12, 6, 1, 2), (20, 5, 3, 7)]:
        key = np.round(rng.random((60, N)), 2)
        got = M.select_top_k_node_limited(key, K, nodes, limit)
        want = np.array([_walk(list(row), K, nodes, limit) for row in key])
        assert np.array_equal(got, want), (N, nodes, limit, K)


def test_properties():
    rng = np.random.default_rng(4)
    N, nodes, limit, K = 64, 8, 3, 8
    key = rng.random((500, N))
    got = M.select_top_k_node_limited(key, K, nodes, limit)
    plain = M.select_top_k(key, K)
    per = N // nodes
    for t in range(len(key)):
        assert len(set(got[t] // per)) <= limit
        assert got[t][0] == plain[t][0]                         # the best expert always goes
        assert np.all(np.diff(key[t, got[t]]) <= 0)              # ordered by key, descending
        if len(set(plain[t] // per)) <= limit:                   # nothing to restrict
            assert np.array_equal(got[t], plain[t])
        else:
            assert key[t, got[t]].sum() < key[t, plain[t]].sum()


def test_route_and_layer_take_the_node_limit():
    rng = np.random.default_rng(5)
    T, d, N, I, K = 40, 32, 16, 8, 4
    u = rng.standard_normal((T, d))
    e = rng.standard_normal((N, d))
    for gate in (O.GATE_SOFTMAX, O.GATE_SIGMOID):
        r = O.route(u, e, K, gate, node_limit=(4, 2))
        assert np.array_equal(r.idx, M.select_top_k_node_limited(r.key, K, 4, 2))
        assert np.array_equal(r.gate, M.gate_values(r.s, r.idx, gate))
    ex = tuple(rng.standard_normal(s) * 0.1 for s in ((N, I, d), (N, I, d), (N, d, I)))
    h, r = O.moe_forward(u, e, K, ex, node_limit=(4, 1))
    h2, _ = O.moe_forward(u, e, K, ex, routing=r)
    assert np.array_equal(h, h2) and np.all((r.idx // 4 == r.idx[:, :1] // 4))


def test_invalid_limits_are_rejected():
    key = np.zeros((1, 8))
    for args in ((3, 3, 2), (2, 4, 0), (2, 4, 5), (5, 4, 2)):   # 8 % 3, M = 0, M > nodes, K > M * per
        with pytest.raises(ValueError):
            M.select_top_k_node_limited(key, *args)
