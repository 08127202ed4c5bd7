"""Expert-parallel plan across ranks, on CPU: sep_ep_plan (host-only C) against
the oracle.

Owner o's pool must be exactly owner o's segment of the single-GPU layout of
all ranks' tokens concatenated in rank order (rows of an expert ordered by
source rank, token, slot).  So for every rank, every assignment's local row
plus the plan's shift must land on the row the oracle gives that assignment
in the concatenated layout, minus the owner's segment start; the owner sizes,
block offsets and counts must be the segment's.  Checked in one process for
many rank counts, and across two gloo processes that exchange their counts
with an all-gather, as real ranks do.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import combine_route_layout_02_b200 as sep
import oracle


def _routing(rank_seed, T, k, E, masked=0.2):
    rng = np.random.default_rng(rank_seed)
    idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
    idx[rng.random((T, k)) < masked] = -1
    return idx


def _check_rank(rank, idx_r, delta, Ts, lay_all, E, R, B):
    """Every valid assignment of this rank lands on its concatenated-layout row."""
    lay_r = oracle.layout(idx_r, E, R, B)
    t0 = int(sum(Ts[:rank]))
    T, k = idx_r.shape
    for t in range(T):
        for j in range(k):
            local = lay_r.src_pool_row[t, j]
            want = lay_all.src_pool_row[t0 + t, j]
            assert (local < 0) == (want < 0)
            if local < 0:
                continue
            e = idx_r[t, j]
            o = e // (E // R)
            assert local + delta[e] == want - lay_all.owner_pool_row_offset[o], (rank, t, j)


def _check_owner(rank, plan, lay_all, E, R, B):
    El = E // R
    seg = lay_all.owner_pool_row_offset
    np.testing.assert_array_equal(plan["owner_rows"], np.diff(seg))
    boff = lay_all.expert_pool_block_offset[rank * El: (rank + 1) * El + 1] - seg[rank] // B
    np.testing.assert_array_equal(plan["owner_block_offset"], boff)
    np.testing.assert_array_equal(plan["owner_expert_counts"], lay_all.expert_counts[rank * El: (rank + 1) * El])


@pytest.mark.parametrize("R,E,B,k,Ts", [(2, 8, 16, 2, [40, 57]), (4, 16, 8, 3, [0, 33, 1, 70]),
                                        (8, 64, 32, 8, [20] * 8), (1, 4, 4, 2, [9]), (3, 3, 1, 1, [5, 0, 6])])
def test_plan_matches_the_concatenated_layout(R, E, B, k, Ts):
    idx = [_routing(100 * R + r, Ts[r], k, E) for r in range(R)]
    lay_all = oracle.layout(np.concatenate(idx) if sum(Ts) else np.zeros((0, k), np.int32), E, R, B)
    counts = np.stack([oracle.layout(idx[r], E, R, B).expert_counts for r in range(R)]).astype(np.int32)
    for r in range(R):
        plan = sep.sep_ep_plan(counts, r, B)
        _check_rank(r, idx[r], plan["delta"], Ts, lay_all, E, R, B)
        _check_owner(r, plan, lay_all, E, R, B)


def test_plan_rejects_bad_input():
    counts = np.ones((2, 8), np.int32)
    with pytest.raises(sep.SepError):
        sep.sep_ep_plan(counts, 2, 16)                   # rank outside the group
    with pytest.raises(sep.SepError):
        sep.sep_ep_plan(np.ones((3, 8), np.int32), 0, 16)   # E not divisible by R
    bad = counts.copy()
    bad[1, 3] = -1
    with pytest.raises(sep.SepError):
        sep.sep_ep_plan(bad, 0, 16)
    with pytest.raises(sep.SepError):
        sep.sep_ep_plan(np.full((2, 8), 2 ** 30, np.int32), 0, 16)   # pool rows past 2^31


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out, E, B, k, Ts):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        idx = _routing(7 + rank, Ts[rank], k, E)
        mine = torch.from_numpy(oracle.layout(idx, E, world, B).expert_counts.astype(np.int32))
        gathered = [torch.zeros_like(mine) for _ in range(world)]
        dist.all_gather(gathered, mine)                  # the counts exchange
        plan = sep.sep_ep_plan(torch.stack(gathered).numpy(), rank, B)
        out[rank] = (idx, plan)
    finally:
        dist.destroy_process_group()


def test_two_ranks_exchange_counts_and_agree_on_the_plan():
    world, E, B, k, Ts = 2, 16, 16, 4, [61, 38]
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out, E, B, k, Ts), nprocs=world, join=True)
        res = dict(out)
    lay_all = oracle.layout(np.concatenate([res[r][0] for r in range(world)]), E, world, B)
    for r in range(world):
        idx, plan = res[r]
        _check_rank(r, idx, plan["delta"], Ts, lay_all, E, world, B)
        _check_owner(r, plan, lay_all, E, world, B)
        np.testing.assert_array_equal(plan["owner_rows"], res[0][1]["owner_rows"])   # every rank sees the same sizes


def test_group_pool_capacity_holds_the_worst_routing():
    """EPGroup sizes every owner's pool for the worst case: every assignment of
    every rank on one owner, spread so each of its experts wastes BLOCK_M - 1
    padding rows.  The plan's owner sizes must never exceed it."""
    from combine_route_layout_02_b200.ep import _pool_rows_cap
    rng = np.random.default_rng(11)
    for _ in range(200):
        R = int(rng.choice([1, 2, 4, 8]))
        El = int(rng.integers(1, 9))
        E, B, k = R * El, int(rng.choice([1, 16, 128])), int(rng.integers(1, 9))
        max_tokens = int(rng.integers(1, 200))
        cap = _pool_rows_cap(R, max_tokens, k, El, B)
        counts = np.zeros((R, E), np.int32)
        for r in range(R):                               # all of rank r's assignments, on owner 0's experts
            n = max_tokens * k
            split = rng.multinomial(n, np.ones(El) / El)
            counts[r, :El] = split
        plan = sep.sep_ep_plan(counts, 0, B)
        assert plan["owner_rows"].max() <= cap
        assert cap % B == 0
