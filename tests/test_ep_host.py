"""Expert parallelism, host side (no GPU): the plan every rank computes from
the all-gathered counts, and the two all-to-all exchanges over gloo ranks.

The plan is pinned to the oracle: G ranks must keep, for each expert, exactly
the assignments that the oracle's capacity dispatch keeps on the concatenated
batch (rank 0's tokens first)."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle as O
from sparse_mixture_experts_22_b200 import ep


def _routing(T, E, k, seed):
    z = np.random.default_rng(seed).standard_normal((T, E))
    z[:, 0] += 1.0   # skew towards expert 0 so that capacities bind
    idx, _ = O.topk(O.make_cfg(T, 4, 4, E, k), z)
    return idx


@pytest.mark.parametrize("G,cf", [(2, (1, 1)), (2, (5, 4)), (4, (1, 2)), (4, None), (1, (3, 2))])
def test_plan_keeps_what_the_concatenated_queue_keeps(G, cf):
    E, k, T_loc = 8, 2, 37
    idxs = [_routing(T_loc, E, k, 100 + r) for r in range(G)]
    counts = np.stack([np.bincount(i.ravel(), minlength=E) for i in idxs])
    plan = ep.make_plan(counts, G * T_loc, k, E, cf, pad=16)
    # the oracle on the concatenated batch
    allidx = np.concatenate(idxs)
    cfg = O.make_cfg(G * T_loc, 4, 4, E, k, cf=cf)
    C = O.capacity(cfg)
    assert plan.C == C
    routed, kept, rank, keep = O.dispatch(cfg, allidx, C)
    for r in range(G):
        kr = keep[r * T_loc:(r + 1) * T_loc]
        ir = idxs[r]
        for e in range(E):
            assert plan.kept[r, e] == int(kr[ir == e].sum()), (r, e)
    np.testing.assert_array_equal(plan.kept.sum(0), kept)
    np.testing.assert_array_equal(plan.counts.sum(0), routed)


def test_plan_layout():
    counts = np.array([[5, 0, 9, 3], [4, 7, 0, 1]])
    plan = ep.make_plan(counts, 20, 2, 4, (1, 1), pad=16)
    assert plan.C == 10
    np.testing.assert_array_equal(plan.cap, [[10, 10, 10, 10], [5, 10, 1, 7]])
    np.testing.assert_array_equal(plan.kept, [[5, 0, 9, 3], [4, 7, 0, 1]])
    np.testing.assert_array_equal(plan.seg % 16, 0)
    # rank 0 owns experts 0, 1 and rank 1 experts 2, 3
    np.testing.assert_array_equal(plan.send, [[16, 32], [32, 16]])
    rows, off, wi = plan.groups(1)
    np.testing.assert_array_equal(rows, [9, 3, 0, 1])
    np.testing.assert_array_equal(off, [0, 16, 32, 32])
    np.testing.assert_array_equal(wi, [0, 1, 0, 1])
    assert plan.recv_rows(1).sum() == 48


def test_peer_rows_land_where_the_exchange_puts_them():
    """Every source's segments, placed at peer_row_starts in each owner's
    buffer, rebuild exactly what the all-to-all concatenation (sources in
    order, each source's split for the owner) receives."""
    counts = np.array([[5, 0, 9, 3, 1, 7], [4, 7, 0, 1, 2, 2], [0, 3, 3, 8, 6, 1]])
    G, E = counts.shape
    plan = ep.make_plan(counts, 30, 2, E, (1, 1), pad=16)
    sends = [_send_buffer(plan, r).numpy() for r in range(G)]
    for q in range(G):
        # the all-to-all: source s's split for q, sources in order
        own = np.concatenate([np.zeros((G, 1)), np.cumsum(plan.send, axis=1)], axis=1).astype(int)
        a2a = np.concatenate([sends[s][own[s, q]:own[s, q + 1]] for s in range(G)])
        # the peer stores: source s writes its segment of expert e (owner q)
        # at peer_row_starts(s)[q] + (its x_perm slot - its first slot for q)
        buf = np.full((int(plan.recv_rows(q).sum()), 4), -7.0, np.float32)
        for s in range(G):
            seg_start = np.concatenate([[0], np.cumsum(plan.seg[s])]).astype(int)
            first = seg_start[q * plan.E_loc]
            for e in range(q * plan.E_loc, (q + 1) * plan.E_loc):
                rows = sends[s][seg_start[e]:seg_start[e] + plan.kept[s, e]]
                at = ep.peer_row_starts(plan, s)[q] + seg_start[e] - first
                buf[at:at + len(rows)] = rows
        kept_rows = a2a[:, 3] == 1
        assert len(buf) == len(a2a)
        np.testing.assert_array_equal(buf[kept_rows], a2a[kept_rows])


# ---------------------------------------------------------------- gloo exchange

WORLD = 2
COUNTS = np.array([[5, 0, 9, 3], [4, 7, 0, 1]])


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _send_buffer(plan, rank):
    """Rows tagged (source, expert, row in segment, 1); padding rows -1."""
    rows = []
    for e in range(plan.E):
        for i in range(int(plan.seg[rank, e])):
            rows.append([rank, e, i, 1] if i < plan.kept[rank, e] else [-1, -1, -1, -1])
    return torch.tensor(rows, dtype=torch.float32).reshape(-1, 4)


def _rank(rank, port, out):
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    sys.path.insert(0, root)
    import torch.distributed as dist
    from sparse_mixture_experts_22_b200 import ep as EP

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=WORLD)
    try:
        counts = EP.all_gather_counts(torch.tensor(COUNTS[rank], dtype=torch.int32), WORLD)
        plan = EP.make_plan(counts, 20, 2, 4, (1, 1), pad=16)
        send = _send_buffer(plan, rank)
        recv = EP.exchange_rows(send, plan, rank)
        back = EP.exchange_back(recv * 2.0, plan, rank)
        out[rank] = (counts, recv.numpy(), back.numpy(), send.numpy())
    finally:
        dist.destroy_process_group()


def test_exchanges_over_gloo_ranks():
    port = _free_port()
    ctx = mp.get_context("spawn")
    manager = ctx.Manager()
    out = manager.dict()
    procs = [ctx.Process(target=_rank, args=(r, port, out)) for r in range(WORLD)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    plan = ep.make_plan(COUNTS, 20, 2, 4, (1, 1), pad=16)
    for rank in range(WORLD):
        counts, recv, back, send = out[rank]
        np.testing.assert_array_equal(counts, COUNTS)
        # every (source, local expert) group holds that source's rows of the expert
        rows, off, wi = plan.groups(rank)
        g = 0
        for src in range(WORLD):
            for el in range(plan.E_loc):
                e = rank * plan.E_loc + el
                blk = recv[off[g]:off[g] + rows[g]]
                np.testing.assert_array_equal(blk[:, 0], src)
                np.testing.assert_array_equal(blk[:, 1], e)
                np.testing.assert_array_equal(blk[:, 2], np.arange(rows[g]))
                g += 1
        # the returned rows land where the sent rows were
        np.testing.assert_array_equal(back, send * 2.0)
        # the peer-memory dispatch writes source src's rows where the
        # all-to-all put them: its first group starts at peer_row_starts
        for src in range(WORLD):
            assert ep.peer_row_starts(plan, src)[rank] == off[src * plan.E_loc]


def test_plan_rejects_experts_not_divisible_by_ranks():
    with pytest.raises(ValueError):
        ep.make_plan(np.zeros((3, 8), np.int64), 30, 2, 8, (1, 1), pad=16)


def test_capacity_is_the_integer_ceiling():
    # 2048 tokens, top-2, cf 1.25, 8 experts -> 640; no limit -> every token
    assert ep.capacity(2048, 2, 8, (5, 4)) == 640
    assert ep.capacity(4096, 6, 160, (3, 2)) == 231
    assert ep.capacity(100, 2, 8, None) == 100
    assert ep.capacity(7, 1, 3, (1, 1)) == 3


def test_plan_with_no_tokens_sends_nothing():
    plan = ep.make_plan(np.zeros((2, 4), np.int64), 0, 2, 4, (1, 1), pad=16)
    assert plan.send.sum() == 0 and plan.kept.sum() == 0
    np.testing.assert_array_equal(ep.peer_row_starts(plan, 1), [0, 0])
