"""The expert-parallel dispatch plan on the CPU.

``moe_ep_plan`` is the host twin of the plan the dispatch kernel computes
(the same functions of the library's ep_plan.h).  Its rows must be those of the
oracle's stable counting sort (``oracle.expert_permutation``) of the
concatenated batch [rank 0's tokens, rank 1's tokens, ...], restricted to each
rank's experts and laid out with every expert's segment padded to a multiple
of 256 rows (the layout the grouped GEMMs read).  The last test restates the
dispatch and the combine on two gloo ranks: each rank sends its rows to the
owners' buffers at the planned rows and reads them back at the same rows.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle as O
from fine_grained_shared_b200 import moe as B

ALIGN = 256


def _routing(rng, T, K, N):
    """T tokens' K distinct experts each (the order of a token's slots is random too)."""
    if T == 0:
        return np.zeros((0, K), np.int64)
    return np.argsort(rng.random((T, N)), axis=1)[:, :K].astype(np.int64)


def _counts(idx, N):
    return np.bincount(idx.ravel(), minlength=N).astype(np.int32)


def _expected(idx_list, N, G):
    """Per rank r and (t, k): (owner, row) in the owner's buffer; per owner its tables."""
    idx_all = np.concatenate(idx_list) if idx_list else np.zeros((0, 1), np.int64)
    perm = O.expert_permutation(idx_all, N)
    per = N // G
    start = np.zeros(N, np.int64)   # first row of each expert in its owner's buffer
    tables = []
    for q in range(G):
        rs, mt, m1 = [0], [0], [0]
        for e in range(q * per, (q + 1) * per):
            start[e] = rs[-1]
            c = int(perm.counts[e])
            rs.append(rs[-1] + -(-c // ALIGN) * ALIGN)
            mt.append(mt[-1] + -(-c // ALIGN))
            m1.append(m1[-1] + -(-c // 128))
        counts = np.append(perm.counts[q * per:(q + 1) * per], 0)
        tables.append((counts, np.array(rs), np.array(mt), np.array(m1)))
    dest, t0 = [], 0
    for idx in idx_list:
        T, K = idx.shape
        rows = np.empty((T, K), np.int64)
        for t in range(T):
            for k in range(K):
                e = idx[t, k]
                rows[t, k] = start[e] + perm.slot[t0 + t, k] - perm.offsets[e]
        dest.append((idx // per, rows))
        t0 += T
    return dest, tables


def _planned_rows(plan_base, idx, N):
    """A rank's rows from its plan: base[e] + the pair's rank among this rank's pairs of e."""
    own = O.expert_permutation(idx, N)
    return plan_base[idx] + own.slot - own.offsets[idx]


@pytest.mark.parametrize("G,N,K,Ts", [
    (2, 16, 4, [300, 333]),
    (4, 64, 6, [257, 0, 1, 129]),
    (8, 256, 8, [40, 3, 0, 77, 5, 120, 1, 64]),
    (2, 2, 2, [7, 9]),                       # one expert per rank, K = N
])
def test_plan_matches_the_counting_sort_of_the_concatenated_batch(G, N, K, Ts):
    rng = np.random.default_rng(1000 * G + N)
    idx_list = [_routing(rng, T, K, N) for T in Ts]
    counts_all = np.stack([_counts(i, N) for i in idx_list])
    dest, tables = _expected(idx_list, N, G)
    per = N // G
    for r in range(G):
        st, base, cnt, rs, mt, m1 = B.moe_ep_plan(counts_all, G, N, r)
        assert st == B.MOE_OK
        q, rows = dest[r]
        np.testing.assert_array_equal(_planned_rows(base, idx_list[r], N), rows)
        np.testing.assert_array_equal(idx_list[r] // per, q)
        for got, want in zip((cnt, rs, mt, m1), tables[r]):
            np.testing.assert_array_equal(got, want)
    # every owner's rows: each expert's segment filled exactly once, nothing outside it
    for q in range(G):
        cnt, rs = tables[q][0], tables[q][1]
        taken = np.concatenate([dest[r][1][dest[r][0] == q] for r in range(G)])
        assert np.unique(taken).size == taken.size
        want = np.concatenate([np.arange(rs[l], rs[l] + cnt[l]) for l in range(per)])
        np.testing.assert_array_equal(np.sort(taken), want)


@settings(max_examples=60, deadline=None)
@given(st.integers(min_value=0, max_value=3), st.integers(min_value=1, max_value=8), st.data())
def test_plan_on_random_splits(log_g, per_rank, data):
    """Any G in {2, 4, 8} (and 1 expert per rank and up), K up to 8, ragged batches including empty
    ranks: the plan still places every rank's rows at the concatenated batch's counting-sort rows."""
    G = 2 ** max(1, log_g)
    N = G * per_rank
    K = data.draw(st.integers(min_value=1, max_value=min(8, N)))
    Ts = data.draw(st.lists(st.integers(min_value=0, max_value=300), min_size=G, max_size=G))
    rng = np.random.default_rng(data.draw(st.integers(min_value=0, max_value=2**31)))
    idx_list = [_routing(rng, T, K, N) for T in Ts]
    counts_all = np.stack([_counts(i, N) for i in idx_list])
    dest, tables = _expected(idx_list, N, G)
    for r in range(G):
        st_, base, cnt, rs, mt, m1 = B.moe_ep_plan(counts_all, G, N, r)
        assert st_ == B.MOE_OK
        np.testing.assert_array_equal(_planned_rows(base, idx_list[r], N), dest[r][1])
        for got, want in zip((cnt, rs, mt, m1), tables[r]):
            np.testing.assert_array_equal(got, want)


def test_plan_rejects_bad_arguments():
    c = np.ones((2, 4), np.int32)
    assert B.moe_ep_plan(c, 1, 4, 0)[0] == B.MOE_ERR_INVALID_ARG       # one rank is no split
    assert B.moe_ep_plan(c, 3, 4, 0)[0] == B.MOE_ERR_INVALID_ARG       # 3 does not divide 4
    assert B.moe_ep_plan(c, 2, 4, 2)[0] == B.MOE_ERR_INVALID_ARG       # no rank 2
    assert B.moe_ep_plan(c, 33, 66, 0)[0] == B.MOE_ERR_INVALID_ARG     # more than 32 ranks
    bad = c.copy()
    bad[1, 2] = -1
    assert B.moe_ep_plan(bad, 2, 4, 0)[0] == B.MOE_ERR_INVALID_ARG


def test_config_checks_of_an_expert_parallel_handle():
    """The checks run before any device call, so they answer without a GPU."""
    def create(**kw):
        args = dict(d_model=64, n_routed=8, d_ff=64, n_shared=0, d_ff_shared=0, max_tokens=16, max_k=2,
                    gate=0, flags=0, route_nodes=0, route_max_nodes=0, ep_ranks=2, ep_rank=0)
        args.update(kw)
        return B.moe_workspace_bytes(B.moe_config(**args))[0]
    assert create() == B.MOE_OK
    assert create(ep_ranks=3) == B.MOE_ERR_INVALID_ARG            # 3 does not divide 8
    assert create(ep_rank=2) == B.MOE_ERR_INVALID_ARG
    assert create(ep_ranks=0, ep_rank=1) == B.MOE_ERR_INVALID_ARG
    assert create(ep_ranks=64, n_routed=64) == B.MOE_ERR_INVALID_ARG
    assert create(flags=B.MOE_FLAG_FP8, d_model=128, d_ff=128) == B.MOE_OK         # FP8 dispatch
    assert create(flags=B.MOE_FLAG_FP8, d_model=64, d_ff=128) == B.MOE_ERR_ALIGNMENT   # the FP8 rule holds
    # the row buffers of a rank hold every rank's rows: 4 x 4096 x 2 rows (+ 255 per local expert)
    # against 4096 x 2 (+ 255 per expert)
    one = B.moe_workspace_bytes(B.moe_config(64, 8, 64, 0, 0, 4096, 2, 0, 0, 0, 0, 0, 0))[1]
    four = B.moe_workspace_bytes(B.moe_config(64, 8, 64, 0, 0, 4096, 2, 0, 0, 0, 0, 4, 1))[1]
    rows_one, rows_four = 4096 * 2 + 8 * 255, 4 * 4096 * 2 + 2 * 255
    assert four - one >= (rows_four - rows_one) * (64 + 64 + 64) * 2     # X_perm, H and Y rows, bf16


# ---------------------------------------------------------------------------
# the exchange on two gloo ranks
# ---------------------------------------------------------------------------

def _free_port() -> int:
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _exchange_rank(rank, world, port, N, K, results):
    import torch.distributed as dist
    os.environ.update({"MASTER_ADDR": "127.0.0.1", "MASTER_PORT": str(port)})
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        T = 150 + 61 * rank
        idx = _routing(np.random.default_rng(77 + rank), T, K, N)
        # the counts every plan reads, and the token count that makes global token ids
        counts = torch.from_numpy(_counts(idx, N))
        gathered = [torch.zeros_like(counts) for _ in range(world)]
        dist.all_gather(gathered, counts)
        counts_all = torch.stack(gathered).numpy()
        Ts = [None] * world
        dist.all_gather_object(Ts, T)
        t_off = int(np.sum(Ts[:rank]))
        st, base, cnt, rs, _, _ = B.moe_ep_plan(counts_all, world, N, rank)
        assert st == B.MOE_OK
        per = N // world
        rows = _planned_rows(base, idx, N)
        owner = idx // per
        # dispatch: each row (here: its global token id and slot) to its owner's buffer at the planned row
        outbox = [[(int(rows[t, k]), t_off + t, k) for t in range(T) for k in range(K) if owner[t, k] == q]
                  for q in range(world)]
        inboxes = [None] * world
        dist.all_gather_object(inboxes, outbox)
        size = int(rs[-1])
        buf = np.full((size, 2), -1, np.int64)
        for src in range(world):
            for row, tok, k in inboxes[src][rank]:
                assert buf[row, 0] == -1, "two rows stored to one place"
                buf[row] = (tok, k)
        # the owner's rows of each expert: the concatenated batch's tokens of that expert, ascending
        all_idx = [None] * world
        dist.all_gather_object(all_idx, idx)
        perm = O.expert_permutation(np.concatenate(all_idx), N)
        for l in range(per):
            e = rank * per + l
            seg = buf[rs[l]:rs[l] + cnt[l], 0]
            np.testing.assert_array_equal(seg, perm.src[perm.offsets[e]:perm.offsets[e + 1]])
            assert (buf[rs[l] + cnt[l]:rs[l + 1]] == -1).all()
        # combine: every source reads its (t, k) rows back from the owners at the same rows
        buffers = [None] * world
        dist.all_gather_object(buffers, buf)
        back = np.array([[buffers[owner[t, k]][rows[t, k]] for k in range(K)] for t in range(T)])
        np.testing.assert_array_equal(back[:, :, 0], t_off + np.arange(T)[:, None].repeat(K, 1))
        np.testing.assert_array_equal(back[:, :, 1], np.arange(K)[None, :].repeat(T, 0))
        results[rank] = True
    finally:
        dist.destroy_process_group()


def test_dispatch_and_combine_on_two_gloo_ranks():
    world, port = 2, _free_port()
    results = mp.Manager().dict()
    mp.start_processes(_exchange_rank, args=(world, port, 16, 4, results), nprocs=world, start_method="spawn",
                       join=True)
    assert dict(results) == {0: True, 1: True}
