"""Expert parallelism across ranks, emulated on one GPU.

R ranks' tokens, routings and pools live on one GPU; each rank lays out its
own routing, the ranks' expert counts are gathered and planned
(sep_ep_plan), then every rank dispatches into every owner's pool through the
array of owner pointers and combines from the owners' expert outputs
(identity experts).  The kernels are those a multi-GPU group runs with peer
pointers; none of them waits on another, so running the ranks one after the
other on one GPU is safe.  The oracle is the single-GPU layout of all ranks'
tokens concatenated in rank order: owner o's pool must equal owner o's segment
of it bit for bit (payload and receive maps, with -1 on padding), and each
rank's combine must equal its slice of the concatenated combine bit for bit.
"""
import numpy as np
import pytest
import torch

import combine_route_layout_02_b200 as sep
import oracle
import workloads as W
from gpu_harness import POISON_BF16, bf16_bits, poisoned_bf16

pytestmark = pytest.mark.gpu

GUARD = 3                                                # poisoned rows past every pool


def _routing(seed, T, k, E, masked):
    rng = np.random.default_rng(seed)
    idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
    if masked:
        idx[rng.random((T, k)) < masked] = -1
    return idx


def _run(R, E, B, k, H, Ts, seed, masked=0.0, short_owner=None):
    idx = [_routing(seed + r, Ts[r], k, E, masked) for r in range(R)]
    xs = [W.random_x(Ts[r], H, seed=seed + 50 + r) for r in range(R)]
    ws = [W.random_weights(Ts[r], k, seed=seed + 90 + r) for r in range(R)]
    handles = [sep.sep_layout(torch.from_numpy(idx[r]).cuda(), E, R, B, flags=sep.SEP_LAYOUT_SYNC_COUNTS)
               for r in range(R)]
    try:
        counts = np.stack([h.view("expert_counts").cpu().numpy() for h in handles]).astype(np.int32)
        plans = [sep.sep_ep_plan(counts, r, B) for r in range(R)]
        rows = [int(v) for v in plans[0]["owner_rows"]]
        given = list(rows)
        if short_owner is not None:
            given[short_owner] = max(rows[short_owner] - B, 0)
        pools = [poisoned_bf16(rows[o] + GUARD, H) for o in range(R)]
        maps = [[torch.full((rows[o] + GUARD,), -7, dtype=torch.int32, device="cuda") for o in range(R)]
                for _ in range(3)]
        deltas = [torch.from_numpy(p["delta"]).cuda() for p in plans]
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        for o in range(R):                               # owners mark their padding
            sep.sep_ep_mark_padding(torch.from_numpy(plans[o]["owner_block_offset"]).cuda(),
                                    torch.from_numpy(plans[o]["owner_expert_counts"]).cuda(), B, given[o],
                                    maps[0][o], maps[1][o], maps[2][o])
        for r in range(R):
            sep.sep_ep_dispatch(handles[r], xs[r].cuda(), r, deltas[r], pools, given, err,
                                recv_token=maps[0], recv_rank=maps[1], recv_slot=maps[2])
        outs = [poisoned_bf16(Ts[r], H) for r in range(R)]
        for r in range(R):                               # identity experts: y = the received rows
            sep.sep_ep_combine(handles[r], pools, given, deltas[r], ws[r].cuda(), outs[r], err)
        torch.cuda.synchronize()
        return idx, xs, ws, rows, pools, maps, outs, int(err.item())
    finally:
        for h in handles:
            sep.sep_handle_free(h)


def _oracle(idx, xs, ws, E, R, B, k):
    Ts = [len(i) for i in idx]
    cat = np.concatenate(idx) if sum(Ts) else np.zeros((0, k), np.int32)
    lay = oracle.layout(cat, E, R, B)
    pool = oracle.dispatch_bf16(torch.cat(xs), lay)
    out = oracle.combine(pool, torch.cat(ws).numpy(), lay)
    return lay, pool, out, np.concatenate([[0], np.cumsum(Ts)])


@pytest.mark.parametrize("R,E,B,k,H,Ts,masked", [
    (4, 16, 16, 4, 264, [100, 0, 37, 211], 0.2),
    (8, 64, 32, 8, 512, [64] * 8, 0.0),
    (2, 8, 128, 2, 3072, [1000, 1000], 0.0),
    (3, 6, 8, 3, 24, [5, 1, 9], 0.5),
    (2, 8, 16, 2, 65536, [20, 13], 0.1),
    (4, 32, 16, 12, 136, [50, 20, 0, 33], 0.1),   # k > 8: the combine's batched-pointer path
])
def test_ep_dispatch_and_combine_match_the_concatenated_oracle(R, E, B, k, H, Ts, masked):
    idx, xs, ws, rows, pools, maps, outs, err = _run(R, E, B, k, H, Ts, seed=R * 1000 + H, masked=masked)
    assert err == 0
    lay, pool, out, cum = _oracle(idx, xs, ws, E, R, B, k)
    off = lay.owner_pool_row_offset
    for o in range(R):
        seg = slice(off[o], off[o + 1])
        assert rows[o] == off[o + 1] - off[o]
        tok = lay.pool_recv_token[seg]
        valid = tok >= 0
        got = bf16_bits(pools[o])
        np.testing.assert_array_equal(got[:rows[o]][valid], pool[seg][valid])
        assert (got[:rows[o]][~valid] == POISON_BF16).all(), "a padding row was written"
        assert (got[rows[o]:] == POISON_BF16).all(), "a row past the pool was written"
        src_rank = np.searchsorted(cum, tok, side="right") - 1
        want_rank = np.where(valid, src_rank, -1)
        want_tok = np.where(valid, tok - cum[np.clip(src_rank, 0, R - 1)], -1)
        want_slot = np.where(valid, lay.pool_recv_slot[seg], -1)
        for m, want in zip(maps, (want_tok, want_rank, want_slot)):
            got_m = m[o].cpu().numpy()
            np.testing.assert_array_equal(got_m[:rows[o]], want)
            assert (got_m[rows[o]:] == -7).all()
    for r in range(R):
        np.testing.assert_array_equal(bf16_bits(outs[r])[:len(idx[r])], out[cum[r]:cum[r + 1]])


def test_ep_rows_outside_a_short_pool_are_refused_on_the_device():
    """An owner whose pool is declared one tile short: rows past it are not
    written (the guard rows keep their poison) and the error word is set."""
    R, E, B, k, H, Ts = 2, 8, 16, 4, 64, [300, 300]
    idx, xs, ws, rows, pools, maps, outs, err = _run(R, E, B, k, H, Ts, seed=5, short_owner=0)
    assert err == 1
    short = max(rows[0] - B, 0)
    assert (bf16_bits(pools[0])[short:] == POISON_BF16).all()


@pytest.mark.parametrize("scale", ["ue8m0", "f32", "f32_pow2"])
def test_ep_fp8_dispatch_matches_the_concatenated_oracle(scale):
    """The FP8 payload across ranks: codes and scales in every owner's pool equal
    the single-GPU FP8 dispatch of the concatenated tokens, bit for bit."""
    R, E, B, k, H, Ts = 4, 16, 16, 4, 384, [100, 0, 37, 211]
    G = H // 128
    idx = [_routing(900 + r, Ts[r], k, E, 0.2) for r in range(R)]
    xs = [W.random_x(Ts[r], H, seed=950 + r) for r in range(R)]
    handles = [sep.sep_layout(torch.from_numpy(idx[r]).cuda(), E, R, B, flags=sep.SEP_LAYOUT_SYNC_COUNTS)
               for r in range(R)]
    try:
        counts = np.stack([h.view("expert_counts").cpu().numpy() for h in handles]).astype(np.int32)
        plans = [sep.sep_ep_plan(counts, r, B) for r in range(R)]
        rows = [int(v) for v in plans[0]["owner_rows"]]
        pools = [torch.full((rows[o] + GUARD, H), 0xA5, dtype=torch.uint8, device="cuda") for o in range(R)]
        if scale == "ue8m0":
            scales = [torch.full((rows[o] + GUARD, G), 0xA5, dtype=torch.uint8, device="cuda") for o in range(R)]
        else:
            scales = [torch.full((rows[o] + GUARD, G), 0x7FC00ABC, dtype=torch.int32, device="cuda").view(torch.float32)
                      for o in range(R)]
        tok = [torch.full((rows[o] + GUARD,), -7, dtype=torch.int32, device="cuda") for o in range(R)]
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        for r in range(R):
            sep.sep_ep_dispatch_fp8(handles[r], xs[r].cuda(), r, torch.from_numpy(plans[r]["delta"]).cuda(), pools,
                                    scales, rows, err, scale=scale, recv_token=tok)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        lay = oracle.layout(np.concatenate(idx), E, R, B)
        codes, scl = oracle.dispatch_fp8(torch.cat(xs), lay, scale)
        off = lay.owner_pool_row_offset
        for o in range(R):
            seg = slice(off[o], off[o + 1])
            valid = lay.pool_recv_token[seg] >= 0
            got = pools[o].cpu().numpy()
            np.testing.assert_array_equal(got[:rows[o]][valid], codes[seg][valid])
            assert (got[:rows[o]][~valid] == 0xA5).all() and (got[rows[o]:] == 0xA5).all()
            gs = scales[o].cpu().numpy()
            if scale == "ue8m0":
                np.testing.assert_array_equal(gs[:rows[o]][valid], scl[seg][valid])
            else:
                np.testing.assert_array_equal(gs[:rows[o]][valid].view(np.uint32), scl[seg][valid].view(np.uint32))
    finally:
        for h in handles:
            sep.sep_handle_free(h)
