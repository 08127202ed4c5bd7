"""Expert parallelism across processes, through the EPGroup host side.

Two processes share the one GPU (each a rank; gloo carries the counts
all-gather and the barriers), hand each other their pools by CUDA IPC and run
three steps: identity experts (the combine reads the received rows),
experts that double their input (written into the shared y buffers), and an
FP8 dispatch (codes and UE8M0 scales into the shared pools).  The EP
kernels never wait on another process's kernel — every barrier follows a
device synchronisation — so two ranks on one GPU are safe.  The oracle is the
single-GPU layout, dispatch and combine of both ranks' tokens concatenated in
rank order, compared bit for bit: each owner's received rows and maps, and
each rank's combined output.
"""
import os
import socket

import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu

E, K, B, H = 16, 4, 16, 256
TS = [150, 97]


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _inputs(rank):
    rng = np.random.default_rng(500 + rank)
    idx = rng.integers(0, E, size=(TS[rank], K)).astype(np.int32)
    idx[rng.random((TS[rank], K)) < 0.15] = -1
    return idx, W.random_x(TS[rank], H, seed=600 + rank), W.random_weights(TS[rank], K, seed=700 + rank)


def _worker(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    import combine_route_layout_02_b200 as sep
    from combine_route_layout_02_b200.ep import EPGroup
    from gpu_harness import bf16_bits
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        idx, x, w = _inputs(rank)
        g = EPGroup(E, K, B, H, max_tokens=max(TS))
        try:
            res = {}
            pool, tok, src, slot = g.dispatch(x.cuda(), torch.from_numpy(idx).cuda())
            res["pool"] = bf16_bits(pool)
            res["maps"] = (tok.cpu().numpy(), src.cpu().numpy(), slot.cpu().numpy())
            y1 = torch.empty(TS[rank], H, dtype=torch.bfloat16, device="cuda")
            g.combine(w.cuda(), y1, y_is_pool=True)
            res["out_identity"] = bf16_bits(y1)
            g.dispatch(x.cuda(), torch.from_numpy(idx).cuda())      # a second step on the same buffers
            P = g.rows[rank]
            g.expert_output().copy_(g.pools[rank][:P] * 2)         # experts: doubling, exact in bf16
            y2 = torch.empty_like(y1)
            g.combine(w.cuda(), y2)
            res["out_double"] = bf16_bits(y2)
            (codes, scales), _, _, _ = g.dispatch(x.cuda(), torch.from_numpy(idx).cuda(), payload="fp8",
                                                  scale="ue8m0")
            res["codes"] = codes.cpu().numpy()
            res["scales"] = scales.cpu().numpy()
            out[rank] = res
        finally:
            g.close()
    finally:
        dist.destroy_process_group()


def test_two_processes_dispatch_and_combine_through_ipc_pools():
    import torch.multiprocessing as mp
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    ins = [_inputs(r) for r in range(world)]
    idx = np.concatenate([i[0] for i in ins])
    lay = oracle.layout(idx, E, world, B)
    pool = oracle.dispatch_bf16(torch.cat([i[1] for i in ins]), lay)
    w = torch.cat([i[2] for i in ins]).numpy()
    want1 = oracle.combine(pool, w, lay)
    doubled = oracle.f32_to_bf16(oracle.bf16_to_f32(pool) * 2).reshape(pool.shape)
    want2 = oracle.combine(doubled, w, lay)
    cum = np.concatenate([[0], np.cumsum(TS)])
    off = lay.owner_pool_row_offset
    for o in range(world):
        seg = slice(off[o], off[o + 1])
        t = lay.pool_recv_token[seg]
        valid = t >= 0
        got = res[o]["pool"]
        assert got.shape[0] == off[o + 1] - off[o]
        np.testing.assert_array_equal(got[valid], pool[seg][valid])
        src = np.searchsorted(cum, t, side="right") - 1
        tok, rk, sl = res[o]["maps"]
        np.testing.assert_array_equal(tok, np.where(valid, t - cum[np.clip(src, 0, world - 1)], -1))
        np.testing.assert_array_equal(rk, np.where(valid, src, -1))
        np.testing.assert_array_equal(sl, np.where(valid, lay.pool_recv_slot[seg], -1))
    for r in range(world):
        np.testing.assert_array_equal(res[r]["out_identity"], want1[cum[r]:cum[r + 1]])
        np.testing.assert_array_equal(res[r]["out_double"], want2[cum[r]:cum[r + 1]])
    codes, scl = oracle.dispatch_fp8(torch.cat([i[1] for i in ins]), lay, "ue8m0")
    for o in range(world):
        seg = slice(off[o], off[o + 1])
        valid = lay.pool_recv_token[seg] >= 0
        np.testing.assert_array_equal(res[o]["codes"][valid], codes[seg][valid])
        np.testing.assert_array_equal(res[o]["scales"][valid], scl[seg][valid])


def _worker_signals(rank, world, port, out):
    import datetime
    import torch.distributed as dist
    from combine_route_layout_02_b200.ep import EPGroup
    from gpu_harness import bf16_bits
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        idx, x, w = _inputs(rank)
        g = EPGroup(E, K, B, H, max_tokens=max(TS), signals=True)
        try:
            res = {"status": [], "out": []}
            for _ in range(2):                           # two steps: the arrival counters are reused
                pool, tok, src, slot = g.dispatch(x.cuda(), torch.from_numpy(idx).cuda())
                P = int(g.plan["owner_rows"][rank].item())
                res["P"] = P
                res["pool"] = bf16_bits(pool[:P])
                res["maps"] = (tok[:P].cpu().numpy(), src[:P].cpu().numpy(), slot[:P].cpu().numpy())
                res["status"].append(g.consume().cpu().tolist())   # identity experts: the published tiles
                y = torch.empty(TS[rank], H, dtype=torch.bfloat16, device="cuda")
                g.combine(w.cuda(), y)
                res["out"].append(bf16_bits(y))
            (codes, scales), _, _, _ = g.dispatch(x.cuda(), torch.from_numpy(idx).cuda(), payload="fp8",
                                                  scale="ue8m0")
            P = int(g.plan["owner_rows"][rank].item())
            res["codes"] = codes[:P].cpu().numpy()
            res["scales"] = scales[:P].cpu().numpy()
            res["flags"] = g.tile_ready[rank][:P // B].cpu().numpy()
            res["seq"] = g.seq
            out[rank] = res
        finally:
            g.close()
    finally:
        dist.destroy_process_group()


def test_two_processes_with_the_device_plan_and_published_tiles():
    """The same group with signals=True: the counts gathered and planned on the
    GPU, every owner tile published at system scope in the owner's memory,
    and each owner's consumer copying the published tiles into its y buffer
    (identity experts) before the combine; the barriers stay, so no kernel
    waits on the other process's kernels."""
    import torch.multiprocessing as mp
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker_signals, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    ins = [_inputs(r) for r in range(world)]
    idx = np.concatenate([i[0] for i in ins])
    lay = oracle.layout(idx, E, world, B)
    pool = oracle.dispatch_bf16(torch.cat([i[1] for i in ins]), lay)
    want = oracle.combine(pool, torch.cat([i[2] for i in ins]).numpy(), lay)
    cum = np.concatenate([[0], np.cumsum(TS)])
    off = lay.owner_pool_row_offset
    codes, scl = oracle.dispatch_fp8(torch.cat([i[1] for i in ins]), lay, "ue8m0")
    for o in range(world):
        seg = slice(off[o], off[o + 1])
        t = lay.pool_recv_token[seg]
        valid = t >= 0
        assert res[o]["P"] == off[o + 1] - off[o]
        np.testing.assert_array_equal(res[o]["pool"][valid], pool[seg][valid])
        src = np.searchsorted(cum, t, side="right") - 1
        tok, rk, sl = res[o]["maps"]
        np.testing.assert_array_equal(tok, np.where(valid, t - cum[np.clip(src, 0, world - 1)], -1))
        np.testing.assert_array_equal(rk, np.where(valid, src, -1))
        np.testing.assert_array_equal(sl, np.where(valid, lay.pool_recv_slot[seg], -1))
        assert res[o]["status"] == [[0, 0], [0, 0]]
        np.testing.assert_array_equal(res[o]["codes"][valid], codes[seg][valid])
        np.testing.assert_array_equal(res[o]["scales"][valid], scl[seg][valid])
        assert (res[o]["flags"] == res[o]["seq"]).all()
    for r in range(world):
        for got in res[r]["out"]:
            np.testing.assert_array_equal(got, want[cum[r]:cum[r + 1]])
