"""Expert parallelism with the plan on the GPU and per-tile publication.

R ranks emulated on one GPU, one after another (no kernel of one rank waits on
another rank's kernel while both could be running: every owner's consumer is
launched only after the dispatches it needs have been enqueued before it on
the same stream).  Checked against the oracle of all ranks' tokens
concatenated in rank order (StreamEP README, "Streaming dispatch in one
paragraph": arrivals are counted per tile on the receiver and the tile's
dispatch_seq is released at system scope once it is complete):

* sep_ep_plan_device equals the host sep_ep_plan on every output, and its
  expert_rows / expert_tile_offset equal the oracle's per-expert counts and
  the owners' tile offsets;
* after every rank's publishing dispatch, each owner tile's flag holds the
  step's sequence number, each owner's consumer copies every tile (status
  [0, 0]) and the copy equals the oracle pool segment bit for bit, the
  arrival counters are back to zero, and a second step reuses them;
* with one rank's dispatch withheld, each owner's consumer gives up within its
  limit (SEP_ERR_TIMEOUT) and reports exactly the tiles that needed that
  rank's rows, and the GPU stays usable.
"""
import numpy as np
import pytest
import torch

import combine_route_layout_02_b200 as sep
import oracle
import workloads as W
from gpu_harness import POISON_BF16, bf16_bits, poisoned_bf16

pytestmark = pytest.mark.gpu


def _routing(seed, T, k, E, masked):
    rng = np.random.default_rng(seed)
    idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
    if masked:
        idx[rng.random((T, k)) < masked] = -1
    return idx


@pytest.mark.parametrize("R,E,B", [(1, 8, 16), (2, 16, 4), (4, 64, 32), (8, 1024, 128), (8, 128, 1), (3, 9, 7)])
def test_device_plan_equals_the_host_plan(R, E, B):
    rng = np.random.default_rng(R * 31 + E)
    counts = rng.integers(0, 300, size=(R, E)).astype(np.int32)
    counts[:, ::5] = 0
    dev = torch.from_numpy(counts).cuda()
    El = E // R
    for rank in range(R):
        host = sep.sep_ep_plan(counts, rank, B)
        got = sep.sep_ep_plan_device(dev, rank, B)
        torch.cuda.synchronize()
        assert int(got["error"].item()) == 0
        for name in ("delta", "owner_rows", "owner_block_offset", "owner_expert_counts"):
            np.testing.assert_array_equal(got[name].cpu().numpy(), host[name], err_msg=name)
        N = counts.sum(0)
        np.testing.assert_array_equal(got["expert_rows"].cpu().numpy(), N)
        tiles = -(-N // B)
        for o in range(R):                                  # owner-local exclusive prefix of tiles
            seg = tiles[o * El:(o + 1) * El]
            np.testing.assert_array_equal(got["expert_tile_offset"].cpu().numpy()[o * El:(o + 1) * El],
                                          np.concatenate([[0], np.cumsum(seg)[:-1]]))


def test_device_plan_flags_a_negative_count():
    counts = torch.tensor([[3, -1], [2, 2]], dtype=torch.int32, device="cuda")
    got = sep.sep_ep_plan_device(counts, 0, 4)
    torch.cuda.synchronize()
    assert int(got["error"].item()) == 1


class _Group:
    """R ranks' layouts, pools, maps and signal arrays on one GPU."""

    def __init__(self, R, E, B, k, H, Ts, seed, masked=0.0, payload="bf16", scale="none"):
        self.R, self.E, self.B, self.k, self.H = R, E, B, k, H
        self.payload, self.scale = payload, scale
        self.idx = [_routing(seed + r, Ts[r], k, E, masked) for r in range(R)]
        self.xs = [W.random_x(Ts[r], H, seed=seed + 50 + r) for r in range(R)]
        self.handles = [sep.sep_layout(torch.from_numpy(self.idx[r]).cuda(), E, R, B) for r in range(R)]
        counts = torch.stack([h.view("expert_counts") for h in self.handles]).to(torch.int32).contiguous()
        self.plans = [sep.sep_ep_plan_device(counts, r, B) for r in range(R)]
        self.rows = [int(v) for v in self.plans[0]["owner_rows"].cpu()]
        cap = [max(n, B) for n in self.rows]
        self.cap = cap
        if payload == "bf16":
            self.pools = [poisoned_bf16(cap[o], H) for o in range(R)]
            self.scales = None
        else:
            self.pools = [torch.full((cap[o], H), 0xA5, dtype=torch.uint8, device="cuda") for o in range(R)]
            G = H // 128
            dt = torch.uint8 if scale == "ue8m0" else torch.float32
            self.scales = [torch.zeros(cap[o], G, dtype=dt, device="cuda") for o in range(R)]
        self.maps = [[torch.full((cap[o],), -7, dtype=torch.int32, device="cuda") for o in range(R)]
                     for _ in range(3)]
        nt = [-(-c // B) for c in cap]
        self.tile_ready = [torch.zeros(nt[o], dtype=torch.int32, device="cuda") for o in range(R)]
        self.arrival = [torch.zeros(nt[o], dtype=torch.int32, device="cuda") for o in range(R)]
        self.err = torch.zeros(1, dtype=torch.int32, device="cuda")
        for o in range(R):
            sep.sep_ep_mark_padding(self.plans[o]["owner_block_offset"], self.plans[o]["owner_expert_counts"], B,
                                    cap[o], self.maps[0][o], self.maps[1][o], self.maps[2][o])

    def dispatch(self, r, seq):
        sep.sep_ep_dispatch_publish(self.handles[r], self.xs[r].cuda(), r, self.plans[r], self.pools, self.cap,
                                    self.tile_ready, self.arrival, seq, self.err, payload=self.payload,
                                    scale=self.scale, scales=self.scales, recv_token=self.maps[0],
                                    recv_rank=self.maps[1], recv_slot=self.maps[2])

    def consume(self, o, seq, timeout_ns=0):
        dst = torch.zeros_like(self.pools[o])
        status = torch.full((2,), 9, dtype=torch.int32, device="cuda")
        sep.sep_ep_consume_tiles(self.plans[o]["owner_block_offset"], self.pools[o], self.maps[0][o],
                                 self.tile_ready[o], self.arrival[o], seq, dst, status, self.B, num_ctas=8,
                                 timeout_ns=timeout_ns)
        return dst, status

    def oracle(self):
        cat = np.concatenate(self.idx)
        lay = oracle.layout(cat, self.E, self.R, self.B)
        return lay, np.concatenate([[0], np.cumsum([len(i) for i in self.idx])])

    def close(self):
        for h in self.handles:
            sep.sep_handle_free(h)


@pytest.mark.parametrize("R,E,B,k,H,Ts,masked,payload,scale", [
    (4, 16, 16, 4, 264, [100, 0, 37, 211], 0.2, "bf16", "none"),
    (8, 64, 32, 8, 512, [64] * 8, 0.0, "bf16", "none"),
    (2, 8, 128, 2, 3072, [1000, 1000], 0.0, "bf16", "none"),
    (3, 6, 8, 3, 384, [5, 1, 9], 0.5, "fp8", "ue8m0"),
    (4, 32, 64, 8, 7168, [64, 64, 64, 64], 0.0, "fp8", "f32"),
])
def test_published_tiles_are_consumed_and_equal_the_oracle(R, E, B, k, H, Ts, masked, payload, scale):
    g = _Group(R, E, B, k, H, Ts, seed=R * 100 + H, masked=masked, payload=payload, scale=scale)
    try:
        lay, cum = g.oracle()
        off = lay.owner_pool_row_offset
        cat_x = torch.cat(g.xs)
        if payload == "bf16":
            want_pool = oracle.dispatch_bf16(cat_x, lay)
        else:
            want_pool, want_sc = oracle.dispatch_fp8(cat_x, lay, scale)
        for step, seq in enumerate((1, 2)):
            for r in range(R):
                g.dispatch(r, seq)
            for o in range(R):
                dst, status = g.consume(o, seq)
                torch.cuda.synchronize()
                assert status.cpu().tolist() == [0, 0], f"owner {o} step {step}"
                assert int(g.err.item()) == 0
                nt = (off[o + 1] - off[o]) // g.B
                tr = g.tile_ready[o].cpu().numpy()
                assert (tr[:nt] == seq).all() and (tr[nt:] == 0).all()
                assert (g.arrival[o].cpu().numpy() == 0).all(), "consumed tiles' counters are zeroed"
                seg = slice(off[o], off[o + 1])
                valid = lay.pool_recv_token[seg] >= 0
                P = off[o + 1] - off[o]
                if payload == "bf16":
                    got = bf16_bits(dst)[:P]
                    np.testing.assert_array_equal(got[valid], want_pool[seg][valid])
                    assert (got[~valid] == 0).all(), "a padding row was copied"
                    np.testing.assert_array_equal(bf16_bits(g.pools[o])[:P][valid], want_pool[seg][valid])
                else:
                    got = dst.cpu().numpy()[:P]
                    np.testing.assert_array_equal(got[valid], want_pool[seg][valid])
                    sc = g.scales[o].cpu().numpy()[:P]
                    if scale == "ue8m0":
                        np.testing.assert_array_equal(sc[valid], want_sc[seg][valid])
                    else:
                        np.testing.assert_array_equal(sc[valid].view(np.uint32), want_sc[seg][valid].view(np.uint32))
    finally:
        g.close()


def test_a_withheld_rank_times_out_with_the_exact_tiles_missing():
    R, E, B, k, H, Ts = 3, 12, 8, 3, 128, [60, 50, 70]
    g = _Group(R, E, B, k, H, Ts, seed=11)
    try:
        lay, cum = g.oracle()
        off = lay.owner_pool_row_offset
        withheld = 1
        for r in range(R):
            if r != withheld:
                g.dispatch(r, 3)
        for o in range(R):
            dst, status = g.consume(o, 3, timeout_ns=20_000_000)
            torch.cuda.synchronize()
            seg_tok = lay.pool_recv_token[off[o]:off[o + 1]]
            src_rank = np.searchsorted(cum, seg_tok, side="right") - 1
            needs = (seg_tok >= 0) & (src_rank == withheld)
            missing = int(needs.reshape(-1, B).any(axis=1).sum())
            want = [sep.SEP_ERR_TIMEOUT, missing] if missing else [0, 0]
            assert status.cpu().tolist() == want, f"owner {o}"
        # the GPU is still usable: a plain layout afterwards works
        h = sep.sep_layout(torch.from_numpy(g.idx[0]).cuda(), E, R, B, flags=sep.SEP_LAYOUT_SYNC_COUNTS)
        sep.sep_handle_free(h)
    finally:
        g.close()
