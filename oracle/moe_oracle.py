"""CPU oracle of the DeepSeekMoE layer forward.  TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py`` (its
``cpu_baseline`` leg and its ``--impl reference`` arm) may import this module.
The GPU product path never calls it and shares no code with it.

It is a plain, slow restatement of what one DeepSeekMoE layer computes, in
float64 on the bf16 input values, one step at a time in the order the method
states them.  numpy's matmul, exp, argsort and bincount serve as library
steps; nothing is blocked, fused or reordered beyond that.

What the layer computes
-----------------------
DeepSeekMoE (arXiv 2401.06066), Abstract: the experts are finely segmented
into mN experts of which mK are activated per token, and K_s experts are
isolated as shared experts.  The blog summary of the same paper (sections
"Fine-Grained Expert Segmentation (Section 3.1)", "Shared Expert Isolation
(Section 3.2)" and "DeepSeekMoE 2B Model Example") adds that the shared
experts are always active for every token while the routed ones are chosen
per token.  The DeepSeek-V3 technical report summary (section 2,
"Auxiliary-Loss-Free Load Balancing") adds per-expert biases that steer
which experts are chosen; it also states that no token is dropped.

The pages print no formula.  The readings taken here (each listed in the
design notes) are the standard ones for this layer:

1. affinity logits   z_{t,i} = u_t . e_i (+ c_i, an optional logit bias)
2. affinity          s_{t,i} = softmax_i(z_{t,i}) over all mN experts, or
                     s_{t,i} = sigmoid(z_{t,i}) (the V3 variant)
3. selection key     k_{t,i} = s_{t,i} (+ b_i, the V3 selection bias)
4. selection         the mK experts with the largest key, ordered by key
                     descending, ties to the lower expert index
5. gate              g = s of the selected expert (softmax; no
                     renormalisation) or s / sum of the selected s (sigmoid)
6. expert FFN        FFN_i(u) = W_down,i (SiLU(W_gate,i u) * (W_up,i u)),
                     SiLU(a) = a / (1 + exp(-a))
7. output            h_t = u_t + sum_j FFN^shared_j(u_t)
                           + sum_k g_{t,k} FFN_{sel_k}(u_t)   (k ascending)

No capacity factor, no token dropping.

Parity pins: every function here is checked, in ``tests/test_oracle_*.py``,
against closed forms, invariants, special cases that reduce to a textbook or
library routine, and brute force on tiny inputs.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable, Optional, Sequence

import numpy as np

GATE_SOFTMAX = "softmax"
GATE_SIGMOID = "sigmoid"

FLAG_NO_RESIDUAL = 1
FLAG_NO_SHARED = 2
FLAG_NO_ROUTED = 4


def f64(a) -> np.ndarray:
    """Any bf16/float tensor or array as a float64 numpy array (exact for bf16)."""
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor
        a = a.detach().to("cpu").float().numpy()
    return np.asarray(a, dtype=np.float64)


# ---------------------------------------------------------------------------
# steps 1-5: routing
# ---------------------------------------------------------------------------

def affinity_logits(u: np.ndarray, e: np.ndarray, logit_bias=None) -> np.ndarray:
    """z[t, i] = u_t . e_i (+ c_i).  u: [T, d], e: [N, d] -> z: [T, N].

    The token-to-expert affinity is a dot product of the token's hidden state
    with the expert's affinity vector (the routing scores of the DeepSeekMoE
    blog summary, "Experiment 1").  ``logit_bias`` c adds a per-expert constant
    to every logit, which shifts both selection and gate values.
    """
    z = u @ e.T
    if logit_bias is not None:
        z = z + f64(logit_bias)[None, :]
    return z


def softmax_affinity(z: np.ndarray) -> np.ndarray:
    """s[t, i] = exp(z[t,i]) / sum_j exp(z[t,j]) over all mN routed experts."""
    m = z.max(axis=1, keepdims=True)
    ez = np.exp(z - m)
    return ez / ez.sum(axis=1, keepdims=True)


def sigmoid_affinity(z: np.ndarray) -> np.ndarray:
    """s[t, i] = 1 / (1 + exp(-z[t, i])) (DeepSeek-V3 variant)."""
    return 1.0 / (1.0 + np.exp(-z))


def select_top_k(key: np.ndarray, K: int) -> np.ndarray:
    """The K experts with the largest key per token -> idx [T, K].

    Ordered by key descending; equal keys are ordered by ascending expert
    index (a stable sort of -key keeps equal keys in index order).  Every
    token gets exactly K experts: there is no capacity limit and no token is
    dropped (DeepSeek-V3 technical report summary, section 2).
    """
    order = np.argsort(-key, axis=1, kind="stable")
    return order[:, :K].astype(np.int64)


def select_top_k_node_limited(key: np.ndarray, K: int, n_nodes: int, M: int) -> np.ndarray:
    """Top-K restricted to at most M of the n_nodes nodes -> idx [T, K].

    DeepSeek-V3 technical report summary, section 2 ("DeepSeekMoE"): routing
    is node-limited, each token going to at most M nodes, chosen among the
    nodes that hold its highest-affinity routed experts.  The pages give no
    formula; the reading taken: the mN experts sit on the nodes in equal
    contiguous ranges (expert i on node i // (mN / n_nodes)); a node ranks by
    the largest key among its experts (equivalently: walk the experts by key,
    descending, collecting their nodes until M are found), ties to the lower
    node index; the token's K experts are then the top K of the chosen nodes'
    experts, ordered and tie-broken as in ``select_top_k``.
    """
    T, N = key.shape
    if N % n_nodes or not 1 <= M <= n_nodes or K > M * (N // n_nodes):
        raise ValueError("node-limited routing needs mN % nodes == 0, 1 <= M <= nodes, K <= M * mN / nodes")
    per = N // n_nodes
    node_score = key.reshape(T, n_nodes, per).max(axis=2)
    nodes = np.argsort(-node_score, axis=1, kind="stable")[:, :M]          # ties -> lower node
    allowed = np.zeros((T, n_nodes), dtype=bool)
    np.put_along_axis(allowed, nodes, True, axis=1)
    masked = np.where(np.repeat(allowed, per, axis=1), key, -np.inf)
    return select_top_k(masked, K)


def gate_values(s: np.ndarray, idx: np.ndarray, gate_kind: str) -> np.ndarray:
    """g[t, k]: the affinity of the k-th selected expert (softmax), or that
    affinity divided by the sum over the selected experts (sigmoid)."""
    g = np.take_along_axis(s, idx, axis=1)
    if gate_kind == GATE_SIGMOID:
        g = g / g.sum(axis=1, keepdims=True)
    return g


@dataclass
class Routing:
    z: np.ndarray        # [T, N] logits (bias included)
    s: np.ndarray        # [T, N] affinities
    key: np.ndarray      # [T, N] selection keys
    idx: np.ndarray      # [T, K] selected experts
    gate: np.ndarray     # [T, K] gate values
    gap: np.ndarray      # [T] key(K-th) - key((K+1)-th); +inf when K == N


def route(u, router_w, K: int, gate_kind: str = GATE_SOFTMAX,
          logit_bias=None, select_bias=None, node_limit=None) -> Routing:
    """Steps 1-5 for every token of u.  ``node_limit`` = (nodes, M) restricts
    each token's experts to at most M nodes (``select_top_k_node_limited``);
    ``gap`` is then left at +inf."""
    u, e = f64(u), f64(router_w)
    z = affinity_logits(u, e, logit_bias)
    if gate_kind == GATE_SOFTMAX:
        s = softmax_affinity(z)
        key = s
    elif gate_kind == GATE_SIGMOID:
        s = sigmoid_affinity(z)
        key = s if select_bias is None else s + f64(select_bias)[None, :]
    else:
        raise ValueError(gate_kind)
    idx = select_top_k(key, K) if node_limit is None else select_top_k_node_limited(key, K, *node_limit)
    gate = gate_values(s, idx, gate_kind)
    N = key.shape[1]
    if K < N and node_limit is None:
        srt = -np.sort(-key, axis=1)
        gap = srt[:, K - 1] - srt[:, K]
    else:
        gap = np.full(key.shape[0], np.inf)
    return Routing(z=z, s=s, key=key, idx=idx, gate=gate, gap=gap)


# ---------------------------------------------------------------------------
# step 3 of the data path: token permutation by expert
# ---------------------------------------------------------------------------

@dataclass
class Permutation:
    counts: np.ndarray   # [N]   tokens routed to each expert
    offsets: np.ndarray  # [N+1] exclusive prefix sum of counts
    src: np.ndarray      # [T*K] token ids, expert-contiguous, ascending within an expert
    slot: np.ndarray     # [T, K] position of (t, k) in src


def expert_permutation(idx: np.ndarray, N: int) -> Permutation:
    """Group the (token, slot) pairs by expert with a stable counting sort.

    The expert-parallel dispatch of the DeepSeek-V3 report (section 3.2.1)
    sends each token to the experts that were chosen for it; on one GPU the
    same grouping is an expert-contiguous list of token ids.  Within one
    expert the tokens appear in ascending token order.
    """
    T, K = idx.shape
    counts = np.bincount(idx.ravel(), minlength=N).astype(np.int64)
    offsets = np.zeros(N + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(counts)
    fill = offsets[:-1].copy()
    src = np.empty(T * K, dtype=np.int64)
    slot = np.empty((T, K), dtype=np.int64)
    for t in range(T):           # ascending token order -> stable
        for k in range(K):
            e = idx[t, k]
            src[fill[e]] = t
            slot[t, k] = fill[e]
            fill[e] += 1
    return Permutation(counts=counts, offsets=offsets, src=src, slot=slot)


# ---------------------------------------------------------------------------
# steps 6-7: expert FFNs and the output
# ---------------------------------------------------------------------------

def silu(a: np.ndarray) -> np.ndarray:
    """SiLU(a) = a * sigmoid(a) = a / (1 + exp(-a))."""
    return a / (1.0 + np.exp(-a))


def swiglu_ffn(u: np.ndarray, w_gate, w_up, w_down) -> np.ndarray:
    """FFN(u) = W_down (SiLU(W_gate u) * (W_up u)) for the rows of u.

    u: [n, d]; w_gate, w_up: [I, d]; w_down: [d, I] (the [out, in] layout of
    a linear layer) -> [n, d].
    """
    wg, wu, wd = f64(w_gate), f64(w_up), f64(w_down)
    a = u @ wg.T                 # [n, I]
    b = u @ wu.T                 # [n, I]
    hmid = silu(a) * b           # [n, I]
    return hmid @ wd.T           # [n, d]


ExpertFn = Callable[[int], Sequence]


def _as_expert_fn(w_gate, w_up, w_down) -> ExpertFn:
    return lambda e: (w_gate[e], w_up[e], w_down[e])


def moe_forward(u, router_w, K: int, experts, shared=None, *,
                gate_kind: str = GATE_SOFTMAX, logit_bias=None, select_bias=None,
                flags: int = 0, rows: Optional[np.ndarray] = None,
                routing: Optional[Routing] = None, ffn: Optional[Callable] = None,
                node_limit=None):
    """h_t for the tokens ``rows`` (all tokens when None) -> (h [n, d], Routing).

    ``experts`` is either a tuple (W_gate [N,I,d], W_up [N,I,d], W_down [N,d,I])
    or a callable e -> (W_gate_e, W_up_e, W_down_e).  ``shared`` is a tuple of
    stacked shared-expert weights ([Ks,Is,d], [Ks,Is,d], [Ks,d,Is]) or None.
    ``flags`` leaves out terms of the sum (residual, shared, routed) so that
    each term can be checked on its own.  Tokens are independent, so the
    output of a subset of rows equals those rows of the full output.
    ``ffn`` replaces ``swiglu_ffn`` for every expert (the FP8 variant);
    ``node_limit`` = (nodes, M) is passed to ``route``.
    """
    u_all = f64(u)
    if rows is None:
        rows = np.arange(u_all.shape[0])
    rows = np.asarray(rows, dtype=np.int64)
    ur = u_all[rows]
    if routing is None:
        routing = route(ur, router_w, K, gate_kind, logit_bias, select_bias, node_limit)
        idx, gate = routing.idx, routing.gate
    else:
        idx, gate = routing.idx[rows], routing.gate[rows]
    expert_fn = experts if callable(experts) else _as_expert_fn(*experts)
    if ffn is None:
        ffn = swiglu_ffn

    n, d = ur.shape
    h = np.zeros((n, d), dtype=np.float64)
    if not flags & FLAG_NO_RESIDUAL:
        h += ur
    if shared is not None and not flags & FLAG_NO_SHARED:
        ws_gate, ws_up, ws_down = shared
        for j in range(len(ws_gate)):          # every shared expert, gate 1
            h += ffn(ur, ws_gate[j], ws_up[j], ws_down[j])
    if not flags & FLAG_NO_ROUTED:
        y = np.zeros((n, K, d), dtype=np.float64)
        for e in np.unique(idx):               # FFN_e on the tokens that chose e
            r, k = np.nonzero(idx == e)
            wg, wu, wd = expert_fn(int(e))
            y[r, k] = gate[r, k][:, None] * ffn(ur[r], wg, wu, wd)
        for k in range(K):                     # gate-weighted sum, k ascending
            h += y[:, k]
    return h, routing


def bias_update(bias, counts, gamma: float) -> np.ndarray:
    """One auxiliary-loss-free balancing step of the per-expert selection biases.

    DeepSeek-V3 technical report summary, section 2 "Auxiliary-Loss-Free Load
    Balancing": after each training step every expert's bias moves according
    to whether the expert was overloaded or underloaded.  The pages give no
    formula; the reading taken is the plainest one: with load_i the number of
    (token, slot) pairs routed to expert i in the step and mean = sum(load)/mN,
    b_i <- b_i + gamma * sign(mean - load_i) -- an overloaded expert's bias
    drops by gamma, an underloaded one's rises by gamma, an expert exactly at
    the mean keeps its bias.  The comparison is made on integers
    (load_i * mN against sum(load)), so no rounding decides a sign.  The
    biases are float32 (they are a float32 input of the layer); the float64
    sum of two float32 values rounded once to float32 is the float32 sum.
    """
    counts = np.asarray(counts, dtype=np.int64)
    N = counts.size
    total = int(counts.sum())
    sign = np.sign(total - counts * N).astype(np.float64)  # sign(mean - load) with mean = total / N
    b = np.asarray(bias, dtype=np.float32).astype(np.float64)
    return (b + np.float64(np.float32(gamma)) * sign).astype(np.float32)
