"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Layout, maps, counts, bf16 payload, FP8 codes and scales are compared bit for
bit; combine within |d| <= 1e-3 + 1e-2*|oracle| and, since the kernel uses the
oracle's exact fp32 operation order, also bit for bit.  Cases cover the five
workloads (small sizes that span several chunks and tiles with ragged tails,
and the full sizes in the benchmark's launch configuration), the extreme
routings the DeepEP dispatch/combine blog lists ("Correctness validation
should cover extreme routing"), and the degenerate sizes.
"""
import numpy as np
import pytest
import torch

import combine_route_layout_02_b200 as sep
import oracle
import workloads as W
from gpu_harness import (POISON_BF16, POISON_F32_BITS, POISON_U8, bf16_bits, check_combine, check_layout,
                         poisoned_bf16, run_bf16_path, run_fp8_path, u16_to_bf16_tensor)

pytestmark = pytest.mark.gpu


def _inputs(w, T=None, H=None):
    w = W.scaled(w, T) if T is not None else w
    if H is not None:
        from dataclasses import replace
        w = replace(w, H=H)
    return w, W.make_inputs(w)


# ------------------------------------------------------------- workloads

@pytest.mark.parametrize("name,T,H", [("tiny", None, None), ("train8k", 1000, None),
                                      ("streaming", 3001, 512), ("train8k", 5000, 3072)])
def test_bf16_workloads(name, T, H):
    w, d = _inputs(W.WORKLOADS[name], T, H)
    run_bf16_path(d["topk_idx"], d["x"], d["topk_weight"], w.E, w.R, w.B)


@pytest.mark.parametrize("name,T,scale", [("decode", None, "ue8m0"), ("decode", None, "f32"),
                                          ("decode", 100, "f32_pow2"), ("prefill_skew", 700, "f32")])
def test_fp8_workloads(name, T, scale):
    w, d = _inputs(W.WORKLOADS[name], T)
    run_fp8_path(d["topk_idx"], d["x"], w.E, w.R, w.B, scale)


def test_fp8_dispatch_then_bf16_combine_recovers_x():
    """FP8 dispatch + BF16 combine (blog checklist item 8): combine of the
    dequantised rows (identity experts) is sum_j w_j * dequant(q(x_t))."""
    w, d = _inputs(W.WORKLOADS["decode"], 64)
    lay, recv, scales = run_fp8_path(d["topk_idx"], d["x"], w.E, w.R, w.B, "ue8m0")
    codes, sc = oracle.dispatch_fp8(d["x"], lay, "ue8m0")
    y32 = oracle.dequant_rows(codes, sc, "ue8m0")
    y = torch.from_numpy(y32).to(torch.bfloat16)           # expert output: bf16 of the dequantised rows
    h = sep.sep_layout(d["topk_idx"].cuda(), w.E, w.R, w.B, flags=sep.SEP_LAYOUT_SYNC_COUNTS)
    try:
        out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
        sep.sep_combine(h, y.cuda(), d["topk_weight"].cuda(), out)
        want = oracle.combine(y, d["topk_weight"].numpy(), lay)
        check_combine(bf16_bits(out), want)
        xf = d["x"].float().numpy()
        got = out.float().cpu().numpy()
        # e4m3 keeps 3 mantissa bits (relative error <= 2^-4), then bf16 rounding twice
        assert (np.abs(got - xf) <= (2 ** -4 + 2 ** -7) * np.abs(xf) + 1e-3).all()
    finally:
        sep.sep_handle_free(h)


# ---------------------------------------------------------- edge routings

@pytest.mark.parametrize("kind", ["one_expert", "owner_empty", "same_owner", "masked", "skew", "uniform"])
@pytest.mark.parametrize("T,k,E,R,B", [(300, 4, 16, 4, 16), (1030, 8, 64, 8, 128), (77, 2, 8, 2, 3)])
def test_extreme_routings(kind, T, k, E, R, B):
    idx = W.edge_routing(kind, T, k, E, R, seed=T + k + E)
    x = W.random_x(T, 64, seed=5)
    wt = W.random_weights(T, k, seed=6)
    lay = run_bf16_path(idx, x, wt, E, R, B, flags=sep.SEP_LAYOUT_SYNC_COUNTS | sep.SEP_LAYOUT_TOKEN_IN_OWNER)
    if kind == "owner_empty":
        assert lay.owner_counts[0] == 0
    if kind == "one_expert":
        assert lay.expert_counts[E - 1] == T * k


@pytest.mark.parametrize("k", [1, 2, 3, 8, 32])
def test_top_k_range(k):
    T, E = 257, 64
    idx = W.edge_routing("uniform", T, k, E, 4, seed=k)
    run_bf16_path(idx, W.random_x(T, 40, seed=k), W.random_weights(T, k, seed=k), E, 4, 16)


@pytest.mark.parametrize("B", [1, 5, 16, 64, 1024])
def test_block_m_range(B):
    T, k, E = 200, 4, 32
    idx = W.edge_routing("masked", T, k, E, 4, seed=B)
    run_bf16_path(idx, W.random_x(T, 16, seed=B), W.random_weights(T, k, seed=B), E, 4, B)


@pytest.mark.parametrize("E,R", [(1, 1), (3, 3), (1024, 8), (1024, 1024)])
def test_expert_count_range(E, R):
    T, k = 400, min(4, E)
    idx = W.edge_routing("uniform", T, k, E, R, seed=E)
    run_bf16_path(idx, W.random_x(T, 8, seed=E), W.random_weights(T, k, seed=E), E, R, 8)


@pytest.mark.parametrize("H", [8, 24, 264, 4104, 16384, 65536])
def test_hidden_sizes_bf16(H):
    T, k, E = 97, 3, 12
    idx = W.edge_routing("uniform", T, k, E, 3, seed=H)
    run_bf16_path(idx, W.random_x(T, H, seed=H), W.random_weights(T, k, seed=H), E, 3, 16)


@pytest.mark.parametrize("H", [128, 384, 640, 16384, 65536])
@pytest.mark.parametrize("scale", ["f32", "ue8m0", "f32_pow2"])
def test_hidden_sizes_fp8(H, scale):
    T, k, E = 61, 4, 16
    idx = W.edge_routing("masked", T, k, E, 4, seed=H)
    run_fp8_path(idx, W.random_x(T, H, seed=H + 1), E, 4, 32, scale)


@pytest.mark.parametrize("scale", ["f32", "ue8m0", "f32_pow2"])
def test_fp8_special_magnitudes(scale):
    """Zero groups, huge and tiny (subnormal bf16) values, exact ties, signed zeros."""
    T, H, k, E = 8, 1024, 2, 4
    x = W.random_x(T, H, seed=3).float()
    x[0] = 0.0
    x[1, :128] = -0.0
    x[2] *= 1e36
    x[3] *= 1e-38
    x[4, :128] = 2.0 ** -133                      # smallest bf16 subnormal
    x[5, 0] = 448.0
    x[5, 1:128] = torch.tensor([17.0, 17.5, 2.5, -64.0] * 32)[:127] / 64.0 * 7.0 / 7.0
    x[6, 128:256] = 3.0e38
    x = x.to(torch.bfloat16)
    idx = W.edge_routing("uniform", T, k, E, 2, seed=9)
    run_fp8_path(idx, x, E, 2, 4, scale)


def test_int64_indices_and_token_in_owner():
    w, d = _inputs(W.WORKLOADS["decode"], 200)
    run_bf16_path(d["topk_idx"].to(torch.int64), d["x"], d["topk_weight"], w.E, w.R, w.B,
                  flags=sep.SEP_LAYOUT_SYNC_COUNTS | sep.SEP_LAYOUT_TOKEN_IN_OWNER, idx_dtype=torch.int64)


def test_unsynced_layout_uses_worst_case_capacity():
    w, d = _inputs(W.WORKLOADS["train8k"], 333)
    run_bf16_path(d["topk_idx"], d["x"], d["topk_weight"], w.E, w.R, w.B, flags=0)


def test_zero_tokens():
    idx = torch.zeros(0, 4, dtype=torch.int32)
    h = sep.sep_layout(idx.cuda(), 16, 4, 16, flags=sep.SEP_LAYOUT_SYNC_COUNTS)
    try:
        info = h.info()
        assert info.num_pool_rows == 0 and info.num_tiles == 0
        assert (h.view("expert_counts") == 0).all()
        recv = poisoned_bf16(1, 64)
        sep.sep_dispatch(h, torch.zeros(0, 64, dtype=torch.bfloat16, device="cuda"), recv)
        out = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
        sep.sep_combine(h, recv, torch.zeros(0, 4, device="cuda"), out)
        torch.cuda.synchronize()
        assert (bf16_bits(recv) == POISON_BF16).all()
    finally:
        sep.sep_handle_free(h)


def test_combine_k1_unit_weight_is_exact_gather_and_masked_tokens_are_zero():
    T, E = 500, 16
    idx = W.edge_routing("uniform", T, 1, E, 4, seed=1)
    idx[::7] = -1                                  # some tokens with no assignment at all
    x = W.random_x(T, 256, seed=2)
    lay = run_bf16_path(idx, x, torch.ones(T, 1), E, 4, 16)
    h = sep.sep_layout(idx.cuda(), E, 4, 16, flags=sep.SEP_LAYOUT_SYNC_COUNTS)
    try:
        recv = poisoned_bf16(h.info().num_pool_rows, 256)
        sep.sep_dispatch(h, x.cuda(), recv)
        out = torch.empty(T, 256, dtype=torch.bfloat16, device="cuda")
        sep.sep_combine(h, recv, torch.ones(T, 1, device="cuda"), out)
        got = bf16_bits(out)
        xb = oracle.as_u16(x)
        keep = np.ones(T, bool)
        keep[::7] = False
        np.testing.assert_array_equal(got[keep], xb[keep])
        assert (got[~keep] == 0).all()
    finally:
        sep.sep_handle_free(h)
    assert lay.expert_counts.sum() == keep.sum()


# ---------------------------------------------------- handle and errors

def test_bad_expert_id_is_reported_and_skipped():
    T, k, E = 64, 2, 8
    idx = W.edge_routing("uniform", T, k, E, 2, seed=4)
    idx[5, 1] = E + 3
    idx[9, 0] = 1 << 20
    lay = oracle.layout(idx.numpy(), E, 2, 16)
    assert lay.status == oracle.BAD_EXPERT_ID
    h = sep.sep_layout(idx.cuda(), E, 2, 16)
    try:
        with pytest.raises(sep.SepError) as ei:
            sep.sep_handle_sync(h)
        assert ei.value.status == sep.SEP_ERR_BAD_EXPERT_ID
        check_layout(h, lay)                         # bad entries are skipped exactly like the oracle
        # a correct routing laid out into the same handle clears the error
        sep.sep_layout(W.edge_routing("uniform", T, k, E, 2, seed=5).cuda(), E, 2, 16, handle=h)
        sep.sep_handle_sync(h)
    finally:
        sep.sep_handle_free(h)


def test_handle_reuse_and_epoch_guard():
    E, R, B, k = 32, 4, 16, 4
    h = sep.sep_handle_create(1000, k, E, R, B)
    try:
        for seed, T in [(1, 1000), (2, 10), (3, 517)]:
            idx = W.edge_routing("uniform", T, k, E, R, seed=seed)
            sep.sep_layout(idx.cuda(), E, R, B, handle=h)
            check_layout(h, oracle.layout(idx.numpy(), E, R, B))
        epoch = h.epoch
        x = W.random_x(517, 32, seed=1).cuda()
        recv = poisoned_bf16(h.info().max_pool_rows, 32)
        sep.sep_dispatch(h, x, recv)
        sep.sep_layout(W.edge_routing("uniform", 517, k, E, R, seed=9).cuda(), E, R, B, handle=h)
        out = torch.empty(517, 32, dtype=torch.bfloat16, device="cuda")
        with pytest.raises(sep.SepError) as ei:            # the handle now holds another routing
            sep.sep_combine(h, recv, torch.ones(517, k, device="cuda"), out, layout_epoch=epoch)
        assert ei.value.status == sep.SEP_ERR_HANDLE_MISMATCH
        with pytest.raises(sep.SepError) as ei:            # too many tokens for the handle
            sep.sep_layout(W.edge_routing("uniform", 1001, k, E, R, seed=9).cuda(), E, R, B, handle=h)
        assert ei.value.status == sep.SEP_ERR_HANDLE_MISMATCH
        with pytest.raises(sep.SepError) as ei:            # other shape
            sep.sep_layout(W.edge_routing("uniform", 10, k, E, R, seed=9).cuda(), E, R, 32, handle=h)
        assert ei.value.status == sep.SEP_ERR_HANDLE_MISMATCH
    finally:
        sep.sep_handle_free(h)


def test_capacity_and_argument_errors():
    w, d = _inputs(W.WORKLOADS["tiny"])
    h = sep.sep_layout(d["topk_idx"].cuda(), w.E, w.R, w.B)
    try:
        info = h.info()
        x = d["x"].cuda()
        with pytest.raises(sep.SepError) as ei:            # worst case not covered before a sync
            sep.sep_dispatch(h, x, poisoned_bf16(info.max_pool_rows - 1, w.H))
        assert ei.value.status == sep.SEP_ERR_CAPACITY
        sep.sep_handle_sync(h)
        P = h.info().num_pool_rows
        sep.sep_dispatch(h, x, poisoned_bf16(P, w.H))       # exact size is enough after a sync
        with pytest.raises(sep.SepError) as ei:
            sep.sep_dispatch(h, x, poisoned_bf16(P - 1, w.H))
        assert ei.value.status == sep.SEP_ERR_CAPACITY
        with pytest.raises(sep.SepError) as ei:            # misaligned x
            sep.sep_dispatch(h, x.view(-1)[1:1 + w.T * (w.H - 8)].view(w.T, w.H - 8), poisoned_bf16(P, w.H - 8))
        assert ei.value.status == sep.SEP_ERR_INVALID_ARG
        tr = torch.zeros(info.max_tiles, dtype=torch.int32, device="cuda")
        sep.sep_dispatch(h, x, poisoned_bf16(P, w.H), tile_ready=tr, dispatch_seq=3)
        with pytest.raises(sep.SepError) as ei:            # dispatch_seq must advance
            sep.sep_dispatch(h, x, poisoned_bf16(P, w.H), tile_ready=tr, dispatch_seq=3)
        assert ei.value.status == sep.SEP_ERR_INVALID_ARG
        with pytest.raises(sep.SepError) as ei:            # tile_ready too short
            sep.sep_dispatch(h, x, poisoned_bf16(P, w.H), tile_ready=tr[:1], dispatch_seq=4)
        assert ei.value.status == sep.SEP_ERR_CAPACITY
        with pytest.raises(sep.SepError) as ei:            # FP8 needs H % 128 == 0 and a scale kind
            sep.sep_dispatch(h, x, torch.empty(P, w.H, dtype=torch.uint8, device="cuda"), payload="fp8",
                             scale="none")
        assert ei.value.status == sep.SEP_ERR_INVALID_ARG
        torch.cuda.synchronize()
    finally:
        sep.sep_handle_free(h)


# ------------------------------------------------------------ streaming

def _streaming_round(h, lay, x, recv, tile_ready, seq, dst, status, consumer_first=True):
    main = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    ready = torch.cuda.Event()
    ready.record(main)                              # the layout is complete on `main`
    side.wait_event(ready)
    if consumer_first:
        sep.sep_consume_tiles(h, recv, tile_ready, seq, dst, status, num_ctas=16, stream=side)
        sep.sep_dispatch(h, x, recv, tile_ready=tile_ready, dispatch_seq=seq, stream=main)
    else:
        sep.sep_dispatch(h, x, recv, tile_ready=tile_ready, dispatch_seq=seq, stream=main)
        sep.sep_consume_tiles(h, recv, tile_ready, seq, dst, status, num_ctas=16, stream=side)
    main.wait_stream(side)
    torch.cuda.synchronize()


def test_streaming_tile_ready_and_consumer():
    w, d = _inputs(W.WORKLOADS["streaming"], 8192, 512)
    lay = oracle.layout(d["topk_idx"].numpy(), w.E, w.R, w.B)
    h = sep.sep_layout(d["topk_idx"].cuda(), w.E, w.R, w.B)
    try:
        info = h.info()
        rows, NT = info.max_pool_rows, lay.num_tiles
        x = d["x"].cuda()
        want = oracle.dispatch_bf16(d["x"], lay)
        valid = lay.pool_recv_token >= 0
        tile_ready = torch.zeros(info.max_tiles, dtype=torch.int32, device="cuda")
        status = torch.zeros(2, dtype=torch.int32, device="cuda")
        for seq, first in [(1, True), (2, False), (7, True)]:
            recv = poisoned_bf16(rows, w.H)
            dst = poisoned_bf16(rows, w.H)
            _streaming_round(h, lay, x, recv, tile_ready, seq, dst, status, consumer_first=first)
            assert status.cpu().tolist() == [0, 0]
            tr = tile_ready.cpu().numpy()
            assert (tr[:NT] == seq).all() and (tr[NT:] == 0).all()
            # every tile received the same whole number of arrivals per valid row
            # (one per warp that wrote a piece of the row)
            cnt = h.view("pool_arrival_count")[:NT].cpu().numpy()
            assert (cnt % lay.pool_arrival_target == 0).all()
            assert len(np.unique(cnt // lay.pool_arrival_target)) == 1 and cnt[0] >= lay.pool_arrival_target[0]
            got = bf16_bits(dst)[:lay.num_pool_rows]
            np.testing.assert_array_equal(got[valid], want[valid])
            assert (got[~valid] == POISON_BF16).all()
            np.testing.assert_array_equal(bf16_bits(recv)[:lay.num_pool_rows][valid], want[valid])
        out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
        sep.sep_combine(h, recv, d["topk_weight"].cuda(), out)
        check_combine(bf16_bits(out), oracle.combine(want, d["topk_weight"].numpy(), lay))
    finally:
        sep.sep_handle_free(h)


def test_handle_free_between_consumer_and_dispatch_does_not_wait_for_the_device():
    """A handle is freed on the host after a consumer was launched and before
    the dispatch it waits for.  The free must not wait for the device: if it
    did, the host would sit in it until the consumer's bounded wait gave up,
    and the consumer would report SEP_ERR_TIMEOUT instead of copying every
    tile."""
    w, d = _inputs(W.WORKLOADS["streaming"], 2048, 512)
    lay = oracle.layout(d["topk_idx"].numpy(), w.E, w.R, w.B)
    idx = d["topk_idx"].cuda()
    other = sep.sep_layout(idx, w.E, w.R, w.B)
    h = sep.sep_layout(idx, w.E, w.R, w.B)
    freed = False
    try:
        info = h.info()
        rows = info.max_pool_rows
        x = d["x"].cuda()
        recv = poisoned_bf16(rows, w.H)
        dst = poisoned_bf16(rows, w.H)
        tile_ready = torch.zeros(info.max_tiles, dtype=torch.int32, device="cuda")
        status = torch.zeros(2, dtype=torch.int32, device="cuda")
        main = torch.cuda.current_stream()
        side = torch.cuda.Stream()
        torch.cuda.synchronize()
        side.wait_stream(main)
        sep.sep_consume_tiles(h, recv, tile_ready, 5, dst, status, num_ctas=16, stream=side)
        sep.sep_handle_free(other)                     # between the consumer and its producer
        freed = True
        sep.sep_dispatch(h, x, recv, tile_ready=tile_ready, dispatch_seq=5, stream=main)
        main.wait_stream(side)
        torch.cuda.synchronize()
        assert status.cpu().tolist() == [0, 0]
        want = oracle.dispatch_bf16(d["x"], lay)
        valid = lay.pool_recv_token >= 0
        np.testing.assert_array_equal(bf16_bits(dst)[:lay.num_pool_rows][valid], want[valid])
    finally:
        if not freed:
            sep.sep_handle_free(other)
        sep.sep_handle_free(h)


def test_streaming_fp8_publishes_every_tile():
    w, d = _inputs(W.WORKLOADS["decode"], 256)
    lay = oracle.layout(d["topk_idx"].numpy(), w.E, w.R, w.B)
    h = sep.sep_layout(d["topk_idx"].cuda(), w.E, w.R, w.B, flags=sep.SEP_LAYOUT_SYNC_COUNTS)
    try:
        P, NT = lay.num_pool_rows, lay.num_tiles
        recv = torch.full((P, w.H), 0, dtype=torch.uint8, device="cuda")
        scales = torch.zeros(P, w.H // 128, dtype=torch.uint8, device="cuda")
        tile_ready = torch.zeros(NT, dtype=torch.int32, device="cuda")
        dst = torch.zeros_like(recv)
        status = torch.zeros(2, dtype=torch.int32, device="cuda")
        x = d["x"].cuda()             # before the consumer: a pageable copy would wait for it
        side = torch.cuda.Stream()
        ev = torch.cuda.Event()
        ev.record()
        side.wait_event(ev)
        sep.sep_consume_tiles(h, recv, tile_ready, 11, dst, status, num_ctas=8, stream=side)
        sep.sep_dispatch(h, x, recv, payload="fp8", scale="ue8m0", recv_scales=scales,
                         tile_ready=tile_ready, dispatch_seq=11)
        torch.cuda.synchronize()
        assert status.cpu().tolist() == [0, 0]
        assert (tile_ready.cpu() == 11).all()
        codes, _ = oracle.dispatch_fp8(d["x"], lay, "ue8m0")
        valid = lay.pool_recv_token >= 0
        np.testing.assert_array_equal(dst.cpu().numpy()[valid], codes[valid])
    finally:
        sep.sep_handle_free(h)


def test_consumer_wait_times_out_cleanly():
    """A flag nothing sets: every wait gives up after the limit, the kernel
    reports SEP_ERR_TIMEOUT and the context stays usable."""
    w, d = _inputs(W.WORKLOADS["tiny"])
    h = sep.sep_layout(d["topk_idx"].cuda(), w.E, w.R, w.B, flags=sep.SEP_LAYOUT_SYNC_COUNTS)
    try:
        info = h.info()
        recv = poisoned_bf16(info.num_pool_rows, w.H)
        dst = poisoned_bf16(info.num_pool_rows, w.H)
        tile_ready = torch.zeros(info.num_tiles, dtype=torch.int32, device="cuda")
        status = torch.zeros(2, dtype=torch.int32, device="cuda")
        sep.sep_consume_tiles(h, recv, tile_ready, 5, dst, status, num_ctas=4, timeout_ns=20_000_000)
        torch.cuda.synchronize()
        st = status.cpu().tolist()
        assert st[0] == sep.SEP_ERR_TIMEOUT and st[1] == info.num_tiles
        assert (bf16_bits(dst) == POISON_BF16).all()
        # the context still works
        sep.sep_dispatch(h, d["x"].cuda(), recv)
        torch.cuda.synchronize()
    finally:
        sep.sep_handle_free(h)


# ---------------------------------------- full sizes, bench launch config

@pytest.mark.slow
def test_full_train8k_bench_configuration():
    """T=8192, H=3072, E=128 in 8 owners, top-8, BLOCK_M=128: unsynced layout
    and worst-case buffers as the benchmark runs them; every output compared."""
    w = W.WORKLOADS["train8k"]
    d = W.make_inputs(w)
    run_bf16_path(d["topk_idx"], d["x"], d["topk_weight"], w.E, w.R, w.B, flags=0)


@pytest.mark.slow
def test_full_prefill_skew_bench_configuration():
    """T=16384, H=7168, E=256 in 8 owners, Zipf(1.2)-skewed top-8, BLOCK_M=128,
    FP8 with fp32 scales, in the benchmark's launch configuration (unsynced
    layout, worst-case buffers): every valid row's codes and scales, and every
    token's combine output, compared with the oracle."""
    w = W.WORKLOADS["prefill_skew"]
    d = W.make_inputs(w)
    lay = oracle.layout(d["topk_idx"].numpy(), w.E, w.R, w.B)
    h = sep.sep_layout(d["topk_idx"].cuda(), w.E, w.R, w.B, flags=0)
    try:
        check_layout(h, lay)
        info = h.info()
        rows, G, P = info.max_pool_rows, w.H // 128, lay.num_pool_rows
        recv = torch.full((rows, w.H), POISON_U8, dtype=torch.uint8, device="cuda")
        scales = torch.full((rows, G), POISON_F32_BITS, dtype=torch.int32, device="cuda").view(torch.float32)
        sep.sep_dispatch(h, d["x"].cuda(), recv, payload="fp8", scale="f32", recv_scales=scales)
        valid = lay.pool_recv_token >= 0
        codes_gpu = recv[:P].cpu().numpy()
        scales_gpu = scales[:P].cpu().numpy()
        del recv, scales
        want_codes, want_scales = oracle.dispatch_fp8(d["x"], lay, "f32")
        np.testing.assert_array_equal(codes_gpu[valid], want_codes[valid])
        np.testing.assert_array_equal(scales_gpu[valid].view(np.uint32), want_scales[valid].view(np.uint32))
        assert (codes_gpu[~valid] == POISON_U8).all(), "a padding row was written"
        del codes_gpu, scales_gpu, want_codes, want_scales
        # combine over a seeded bf16 pool (rows repeat a 61-row table), every token
        table = W.random_x(61, w.H, seed=77)
        y = table[torch.arange(rows) % 61].contiguous()
        out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
        sep.sep_combine(h, y.cuda(), d["topk_weight"].cuda(), out)
        want = oracle.combine(y, d["topk_weight"].numpy(), lay)
        check_combine(bf16_bits(out), want)
    finally:
        sep.sep_handle_free(h)


@pytest.mark.slow
def test_full_streaming_bench_configuration():
    w = W.WORKLOADS["streaming"]
    d = W.make_inputs(w)
    lay = oracle.layout(d["topk_idx"].numpy(), w.E, w.R, w.B)
    h = sep.sep_layout(d["topk_idx"].cuda(), w.E, w.R, w.B)
    try:
        check_layout(h, lay)
        info = h.info()
        recv = poisoned_bf16(info.max_pool_rows, w.H)
        dst = poisoned_bf16(info.max_pool_rows, w.H)
        tile_ready = torch.zeros(info.max_tiles, dtype=torch.int32, device="cuda")
        status = torch.zeros(2, dtype=torch.int32, device="cuda")
        _streaming_round(h, lay, d["x"].cuda(), recv, tile_ready, 1, dst, status)
        assert status.cpu().tolist() == [0, 0]
        want = oracle.dispatch_bf16(d["x"], lay)
        valid = lay.pool_recv_token >= 0
        P = lay.num_pool_rows
        np.testing.assert_array_equal(bf16_bits(recv)[:P][valid], want[valid])
        np.testing.assert_array_equal(bf16_bits(dst)[:P][valid], want[valid])
        out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
        sep.sep_combine(h, recv, d["topk_weight"].cuda(), out)
        check_combine(bf16_bits(out), oracle.combine(want, d["topk_weight"].numpy(), lay))
    finally:
        sep.sep_handle_free(h)


_FRESH_PROCESS_STREAMING = r"""
import sys, torch
sys.path.insert(0, sys.argv[1])
import combine_route_layout_02_b200 as sep
import workloads as W
w = W.scaled(W.WORKLOADS["decode"], 256)
d = W.make_inputs(w)
idx, x = d["topk_idx"].cuda(), d["x"].cuda()
h = sep.sep_layout(idx, w.E, w.R, w.B, flags=sep.SEP_LAYOUT_SYNC_COUNTS)
info = h.info()
P, NT = info.num_pool_rows, info.num_tiles
recv = torch.zeros(P, w.H, dtype=torch.uint8, device="cuda")
scales = torch.zeros(P, w.H // 128, dtype=torch.float32, device="cuda")
tile_ready = torch.zeros(NT, dtype=torch.int32, device="cuda")
dst = torch.zeros_like(recv)
status = torch.zeros(2, dtype=torch.int32, device="cuda")
side = torch.cuda.Stream()
side.wait_stream(torch.cuda.current_stream())
sep.sep_consume_tiles(h, recv, tile_ready, 1, dst, status, num_ctas=8, stream=side)
sep.sep_dispatch(h, x, recv, payload="fp8", scale="f32_pow2", recv_scales=scales,
                 tile_ready=tile_ready, dispatch_seq=1)
torch.cuda.synchronize()
ok = status.cpu().tolist() == [0, 0] and bool((tile_ready == 1).all()) and bool(torch.equal(dst, recv))
sep.sep_handle_free(h)
print("STATUS", status.cpu().tolist(), "OK" if ok else "BAD")
sys.exit(0 if ok else 1)
"""


def test_streaming_first_launch_in_a_fresh_process():
    """Consumer launched first, then a dispatch kernel this process has never
    run: the library must already have loaded it (a lazy load on first launch
    would wait for the spinning consumer)."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, "-c", _FRESH_PROCESS_STREAMING, root], capture_output=True,
                       text=True, timeout=300)
    assert r.returncode == 0 and "OK" in r.stdout, r.stdout + r.stderr


# ------------------------------------------------------ borrowed receive

def test_borrowed_view_rows_equal_the_copied_pool():
    """PR #769's borrowed receive: the view (x, row map) read by an indexed
    consumer gives exactly the rows a copying dispatch writes."""
    w, d = _inputs(W.WORKLOADS["train8k"], 2000)
    lay = oracle.layout(d["topk_idx"].numpy(), w.E, w.R, w.B)
    want = oracle.dispatch_bf16(d["x"], lay)
    valid = lay.pool_recv_token >= 0
    h = sep.sep_layout(d["topk_idx"].cuda(), w.E, w.R, w.B, flags=sep.SEP_LAYOUT_SYNC_COUNTS)
    try:
        x = d["x"].cuda()
        P = h.info().num_pool_rows
        # copy path: dispatch, then the consumer reads the pool in place
        recv = poisoned_bf16(P, w.H)
        sep.sep_dispatch(h, x, recv)
        dst_copy = poisoned_bf16(P, w.H)
        sep.sep_gather_rows(sep.pool_view(h, recv), dst_copy)
        # borrowed path: no copy, the consumer gathers from x through the row map
        view = sep.sep_dispatch_borrow(h, x)
        assert view.num_rows == P and view.indexed == 1 and view.row_bytes == 2 * w.H
        rows = torch.as_tensor(sep.sep._DeviceArray(view.row_indices, (P,), "<i4"), device="cuda").clone()
        np.testing.assert_array_equal(rows.cpu().numpy(), lay.pool_recv_token)
        dst = poisoned_bf16(P, w.H)
        sep.sep_gather_rows(view, dst)
        sep.sep_view_release(h, [torch.cuda.current_stream()])
        torch.cuda.synchronize()
        for got in (bf16_bits(dst), bf16_bits(dst_copy)):
            np.testing.assert_array_equal(got[valid], want[valid])
            assert (got[~valid] == POISON_BF16).all()
    finally:
        sep.sep_handle_free(h)


def test_borrowed_view_is_rejected_up_front_and_leases_the_handle():
    w, d = _inputs(W.WORKLOADS["tiny"])
    x = d["x"].cuda()
    h = sep.sep_layout(d["topk_idx"].cuda(), w.E, w.R, w.B)
    try:
        with pytest.raises(sep.SepError) as ei:              # needs CPU counts
            sep.sep_dispatch_borrow(h, x)
        assert ei.value.status == sep.SEP_ERR_INVALID_ARG
        sep.sep_handle_sync(h)
        lib = sep.library()
        view = sep.RecvView()
        import ctypes
        st = lib.sep_dispatch_borrow(h.ptr, ctypes.c_void_p(x.data_ptr()), w.H, sep.sep.SEP_PAYLOAD_FP8_E4M3,
                                     ctypes.byref(view))
        assert st == sep.SEP_ERR_INVALID_ARG                   # FP8 cannot be borrowed
        view = sep.sep_dispatch_borrow(h, x)
        recv = poisoned_bf16(h.info().num_pool_rows, w.H)
        out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
        for call in (lambda: sep.sep_layout(d["topk_idx"].cuda(), w.E, w.R, w.B, handle=h),
                     lambda: sep.sep_dispatch(h, x, recv),
                     lambda: sep.sep_dispatch_borrow(h, x),
                     lambda: sep.sep_combine(h, recv, d["topk_weight"].cuda(), out)):
            with pytest.raises(sep.SepError) as ei:
                call()
            assert ei.value.status == sep.SEP_ERR_HANDLE_MISMATCH
        lib.sep_handle_free(h.ptr)                              # refused while the view is active
        assert "borrowed view" in lib.sep_last_error().decode()
        sep.sep_view_release(h, [])
        with pytest.raises(sep.SepError):                       # nothing left to release
            sep.sep_view_release(h, [])
        sep.sep_dispatch(h, x, recv)                            # usable again
        torch.cuda.synchronize()
    finally:
        sep.sep_handle_free(h)


def test_borrowed_view_delayed_cross_stream_reader():
    """The consumer runs late on another stream; after the release, the next
    layout into the handle (a different routing) waits for it, so the consumer
    still reads the old row map."""
    w, d = _inputs(W.WORKLOADS["train8k"], 1500)
    lay = oracle.layout(d["topk_idx"].numpy(), w.E, w.R, w.B)
    want = oracle.dispatch_bf16(d["x"], lay)
    valid = lay.pool_recv_token >= 0
    other = W.edge_routing("uniform", 1500, w.k, w.E, w.R, seed=3)
    h = sep.sep_layout(d["topk_idx"].cuda(), w.E, w.R, w.B, flags=sep.SEP_LAYOUT_SYNC_COUNTS)
    try:
        x = d["x"].cuda()
        P = h.info().num_pool_rows
        dst = poisoned_bf16(h.info().max_pool_rows, w.H)
        idx2 = other.cuda()
        torch.cuda.synchronize()
        side = torch.cuda.Stream()
        view = sep.sep_dispatch_borrow(h, x)
        with torch.cuda.stream(side):
            torch.cuda._sleep(20_000_000)                       # a late reader (bounded spin, ~10 ms)
        sep.sep_gather_rows(view, dst, stream=side)
        sep.sep_view_release(h, [side])
        sep.sep_layout(idx2, w.E, w.R, w.B, handle=h)           # must wait for the reader
        torch.cuda.synchronize()
        np.testing.assert_array_equal(bf16_bits(dst)[:P][valid], want[valid])
        check_layout(h, oracle.layout(other.numpy(), w.E, w.R, w.B))
    finally:
        sep.sep_handle_free(h)


@pytest.mark.parametrize("max_ctas", [1, 3, 37])
def test_cta_budget_keeps_every_result(max_ctas):
    """With a CTA budget the dispatch and combine grids walk all their work
    items with fewer CTAs: pool rows (bf16 and FP8), codes, scales and the
    combine equal the oracle bit for bit."""
    w, d = _inputs(W.WORKLOADS["train8k"], 700)
    lay = oracle.layout(d["topk_idx"].numpy(), w.E, w.R, w.B)
    h = sep.sep_layout(d["topk_idx"].cuda(), w.E, w.R, w.B, flags=sep.SEP_LAYOUT_SYNC_COUNTS)
    try:
        sep.sep_handle_set_max_ctas(h, max_ctas)
        P = lay.num_pool_rows
        valid = lay.pool_recv_token >= 0
        recv = poisoned_bf16(P, w.H)
        sep.sep_dispatch(h, d["x"].cuda(), recv)
        want = oracle.dispatch_bf16(d["x"], lay)
        got = bf16_bits(recv)
        np.testing.assert_array_equal(got[valid], want[valid])
        assert (got[~valid] == POISON_BF16).all()
        out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
        sep.sep_combine(h, recv, d["topk_weight"].cuda(), out)
        check_combine(bf16_bits(out), oracle.combine(want, d["topk_weight"].numpy(), lay))
        codes = torch.full((P, w.H), POISON_U8, dtype=torch.uint8, device="cuda")
        scales = torch.zeros(P, w.H // 128, dtype=torch.uint8, device="cuda")
        sep.sep_dispatch(h, d["x"].cuda(), codes, payload="fp8", scale="ue8m0", recv_scales=scales)
        want_c, want_s = oracle.dispatch_fp8(d["x"], lay, "ue8m0")
        np.testing.assert_array_equal(codes.cpu().numpy()[valid], want_c[valid])
        np.testing.assert_array_equal(scales.cpu().numpy()[valid], want_s[valid])
    finally:
        sep.sep_handle_free(h)


@pytest.mark.parametrize("kind,T,k,H,max_ctas", [
    ("uniform", 1000, 8, 3072, 37),
    ("masked", 777, 4, 264, 5),         # a ragged 528-byte row; masked assignments
    ("skew", 300, 8, 7168, 2),
    ("one_expert", 129, 2, 8, 1),       # 16-byte rows, duplicate experts, one CTA
    ("uniform", 64, 8, 16384, 100),     # long rows split over several warps
    ("uniform", 257, 32, 64, 3),        # k = 32
])
def test_budget_grids_match_the_oracle(kind, T, k, H, max_ctas):
    """A CTA budget below the default grid launches at most max_ctas CTAs of
    32 warps that walk every item: pool rows, the combine and the unit-weight
    combine of the backward equal the oracle bit for bit, and padding rows
    stay unwritten."""
    E, R, B = 64, 8, 16
    idx = W.edge_routing(kind, T, k, E, R, seed=T + k)
    x = W.random_x(T, H, seed=T)
    wt = W.random_weights(T, k, seed=k)
    lay = oracle.layout(idx.numpy(), E, R, B)
    h = sep.sep_layout(idx.cuda(), E, R, B, flags=sep.SEP_LAYOUT_SYNC_COUNTS)
    try:
        sep.sep_handle_set_max_ctas(h, max_ctas)
        P = lay.num_pool_rows
        valid = lay.pool_recv_token >= 0
        recv = poisoned_bf16(P + 2, H)
        sep.sep_dispatch(h, x.cuda(), recv)
        want = oracle.dispatch_bf16(x, lay)
        got = bf16_bits(recv)
        np.testing.assert_array_equal(got[:P][valid], want[valid])
        assert (got[:P][~valid] == POISON_BF16).all(), "a padding row was written"
        assert (got[P:] == POISON_BF16).all(), "a row past the pool was written"
        out = poisoned_bf16(T, H)
        sep.sep_combine(h, recv, wt.cuda(), out)
        check_combine(bf16_bits(out), oracle.combine(want, wt.numpy(), lay))
        grad_x = poisoned_bf16(T, H)
        sep.sep_combine_grads(h, recv, grad_x)
        np.testing.assert_array_equal(bf16_bits(grad_x), oracle.combine_grads(want, lay))
        sep.sep_handle_sync(h)
    finally:
        sep.sep_handle_free(h)


def test_cta_budget_with_publication_and_an_empty_routing():
    """Under a CTA budget the publishing dispatch still publishes every tile
    once its rows have landed (the reference consumer, launched first on
    another stream, copies them all), and a routing of no tokens launches
    nothing."""
    w, d = _inputs(W.WORKLOADS["streaming"], 4096, 512)
    lay = oracle.layout(d["topk_idx"].numpy(), w.E, w.R, w.B)
    h = sep.sep_layout(d["topk_idx"].cuda(), w.E, w.R, w.B)
    try:
        sep.sep_handle_set_max_ctas(h, 6)
        info = h.info()
        rows, NT = info.max_pool_rows, lay.num_tiles
        want = oracle.dispatch_bf16(d["x"], lay)
        valid = lay.pool_recv_token >= 0
        tile_ready = torch.zeros(info.max_tiles, dtype=torch.int32, device="cuda")
        status = torch.zeros(2, dtype=torch.int32, device="cuda")
        recv, dst = poisoned_bf16(rows, w.H), poisoned_bf16(rows, w.H)
        _streaming_round(h, lay, d["x"].cuda(), recv, tile_ready, 5, dst, status, consumer_first=True)
        assert status.cpu().tolist() == [0, 0]
        assert (tile_ready.cpu().numpy()[:NT] == 5).all()
        got = bf16_bits(dst)[:lay.num_pool_rows]
        np.testing.assert_array_equal(got[valid], want[valid])
        assert (got[~valid] == POISON_BF16).all()
    finally:
        sep.sep_handle_free(h)
    h = sep.sep_layout(torch.zeros(0, 4, dtype=torch.int32, device="cuda"), 16, 4, 16, flags=sep.SEP_LAYOUT_SYNC_COUNTS)
    try:
        sep.sep_handle_set_max_ctas(h, 1)
        recv = poisoned_bf16(1, 64)
        n0 = sep.sep_launch_count()
        sep.sep_dispatch(h, torch.zeros(0, 64, dtype=torch.bfloat16, device="cuda"), recv)
        sep.sep_combine(h, recv, torch.zeros(0, 4, device="cuda"), torch.empty(0, 64, dtype=torch.bfloat16,
                                                                                device="cuda"))
        assert sep.sep_launch_count() == n0
        torch.cuda.synchronize()
        assert (bf16_bits(recv) == POISON_BF16).all()
    finally:
        sep.sep_handle_free(h)
