"""sep_layout_dispatch: the layout and the dispatch of one routing in one call.

The call must compute exactly what sep_layout followed by sep_dispatch
computes ("DeepEP MoE dispatch/combine" blog, "一轮 DeepEP 数据流": count by
expert, lay out, move the hidden states; the low-latency article's dispatch
takes x and topk_idx together).  With SEP_LAYOUT_ONE_LAUNCH small routings
run as one cooperative launch (layout CTAs beside dispatch CTAs that wait for
them); larger ones, and every routing by default, as the two kernels.  Every case is compared with the oracle: the layout arrays and the
pool rows (bf16 bits, or FP8 codes and scales) bit for bit, padding rows
untouched, and which path ran is read from sep_launch_count.
"""
import numpy as np
import pytest
import torch

import combine_route_layout_02_b200 as sep
import oracle
import workloads as W
from gpu_harness import (POISON_BF16, POISON_F32_BITS, POISON_U8, bf16_bits, check_combine, check_layout,
                         poisoned_bf16)

pytestmark = pytest.mark.gpu


def _pool(rows, H, payload, scale):
    if payload == "bf16":
        return poisoned_bf16(rows, H), None
    recv = torch.full((rows, H), POISON_U8, dtype=torch.uint8, device="cuda")
    if scale == "ue8m0":
        sc = torch.full((rows, H // 128), POISON_U8, dtype=torch.uint8, device="cuda")
    else:
        sc = torch.full((rows, H // 128), POISON_F32_BITS, dtype=torch.int32, device="cuda").view(torch.float32)
    return recv, sc


def _check_pool(lay, x, recv, sc, payload, scale):
    P = lay.num_pool_rows
    valid = lay.pool_recv_token >= 0
    if payload == "bf16":
        got = bf16_bits(recv)
        want = oracle.dispatch_bf16(x, lay)
        np.testing.assert_array_equal(got[:P][valid], want[valid])
        assert (got[:P][~valid] == POISON_BF16).all(), "a padding row was written"
        assert (got[P:] == POISON_BF16).all(), "a row past the pool was written"
        return
    codes = recv.cpu().numpy()
    scales = sc.cpu().numpy()
    want_c, want_s = oracle.dispatch_fp8(x, lay, scale)
    np.testing.assert_array_equal(codes[:P][valid], want_c[valid])
    if scale == "ue8m0":
        np.testing.assert_array_equal(scales[:P][valid], want_s[valid])
    else:
        np.testing.assert_array_equal(scales[:P][valid].view(np.uint32), want_s[valid].view(np.uint32))
    assert (codes[:P][~valid] == POISON_U8).all(), "a padding row was written"
    assert (codes[P:] == POISON_U8).all()


ONE = sep.SEP_LAYOUT_ONE_LAUNCH


def _run(idx, x, E, R, B, payload="bf16", scale="none", handle=None, idx_dtype=torch.int32, flags=ONE):
    T, k = idx.shape
    H = x.shape[1]
    worst = oracle.capacity_rows(T * k, E, B)
    worst = -(-worst // B) * B
    recv, sc = _pool(max(worst, 1), H, payload, scale)
    idx_d, x_d = idx.to(idx_dtype).cuda(), x.cuda()
    torch.cuda.synchronize()
    n0 = sep.sep_launch_count()
    h = sep.sep_layout_dispatch(idx_d, x_d, recv, E, R, B, payload=payload, scale=scale, recv_scales=sc,
                                handle=handle, flags=flags)
    launches = sep.sep_launch_count() - n0
    torch.cuda.synchronize()
    lay = oracle.layout(idx.numpy(), E, R, B)
    try:
        sep.sep_handle_sync(h)
        check_layout(h, lay)
        _check_pool(lay, x, recv, sc, payload, scale)
    except BaseException:
        if handle is None:
            sep.sep_handle_free(h)
        raise
    return h, lay, launches, recv


@pytest.mark.parametrize("name,T,H,payload,scale", [
    ("decode", None, None, "fp8", "ue8m0"),
    ("decode", None, None, "fp8", "f32"),
    ("decode", 64, 1024, "fp8", "f32_pow2"),
    ("decode", 100, 384, "fp8", "f32"),           # 384 channels: one 512-channel step, ragged
    ("tiny", None, None, "bf16", "none"),
    ("tiny", 77, 264, "bf16", "none"),            # 33 vectors a row: a ragged 32-vector step
    ("decode", 256, 7168, "bf16", "none"),
])
def test_small_routings_run_as_one_launch(name, T, H, payload, scale):
    from dataclasses import replace
    w = W.WORKLOADS[name]
    w = W.scaled(w, T) if T else w
    if H:
        w = replace(w, H=H)
    d = W.make_inputs(w)
    h, lay, launches, recv = _run(d["topk_idx"], d["x"], w.E, w.R, w.B, payload, scale)
    try:
        assert launches == 1, f"{launches} launches: the small routing did not run as one launch"
        if payload == "bf16":                       # the handle serves the combine as usual
            out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
            sep.sep_combine(h, recv, d["topk_weight"].cuda(), out)
            want = oracle.combine(oracle.dispatch_bf16(d["x"], lay), d["topk_weight"].numpy(), lay)
            check_combine(bf16_bits(out), want)
    finally:
        sep.sep_handle_free(h)


@pytest.mark.parametrize("kind", ["masked", "one_expert", "skew", "uniform"])
def test_edge_routings_int64_ids(kind):
    idx = W.edge_routing(kind, 333, 6, 48, 4, seed=71)
    x = W.random_x(333, 640, seed=72)
    h, lay, launches, _ = _run(idx, x, 48, 4, 8, "fp8", "ue8m0", idx_dtype=torch.int64)
    sep.sep_handle_free(h)
    assert launches == 1


def test_duplicate_experts_and_many_experts():
    rng = np.random.default_rng(73)
    idx = rng.integers(0, 1024, size=(200, 4))
    idx[::3, 1] = idx[::3, 0]                       # an expert twice in one top-k
    idx[5] = -1
    x = W.random_x(200, 512, seed=74)
    h, lay, launches, _ = _run(torch.from_numpy(idx), x, 1024, 8, 16, "bf16", "none")
    sep.sep_handle_free(h)
    assert launches == 1


@pytest.mark.parametrize("name,payload,scale", [("decode", "fp8", "ue8m0"), ("tiny", "bf16", "none")])
def test_two_launches_by_default(name, payload, scale):
    w = W.WORKLOADS[name]
    d = W.make_inputs(w)
    h, lay, launches, _ = _run(d["topk_idx"], d["x"], w.E, w.R, w.B, payload, scale, flags=0)
    sep.sep_handle_free(h)
    assert launches == 2


def test_the_one_launch_flag_is_refused_by_sep_layout():
    idx = torch.zeros(4, 2, dtype=torch.int32, device="cuda")
    with pytest.raises(sep.SepError, match="SEP_ERR_INVALID_ARG"):
        sep.sep_layout(idx, 8, 2, 16, flags=sep.SEP_LAYOUT_ONE_LAUNCH)


def test_large_routing_falls_back_to_two_launches():
    w = W.WORKLOADS["train8k"]
    d = W.make_inputs(w)
    h, lay, launches, _ = _run(d["topk_idx"], d["x"], w.E, w.R, w.B)
    sep.sep_handle_free(h)
    assert launches == 2


def test_zero_tokens():
    h, lay, launches, _ = _run(torch.zeros(0, 4, dtype=torch.int64), torch.zeros(0, 256, dtype=torch.bfloat16),
                               8, 2, 16)
    assert h.info().num_pool_rows == 0
    sep.sep_handle_free(h)


def test_handle_reuse_mixed_with_the_separate_calls():
    """One handle through fused calls, a separate sep_layout + sep_dispatch, and
    fused calls again: the never-reset counters stay on their windows."""
    w = W.WORKLOADS["decode"]
    h = sep.sep_handle_create(w.T, w.k, w.E, w.R, w.B)
    try:
        for rep in range(5):
            from dataclasses import replace
            d = W.make_inputs(replace(w, seed=w.seed + 31 * rep))
            if rep == 2:
                lay = oracle.layout(d["topk_idx"].numpy(), w.E, w.R, w.B)
                rows = h.info().max_pool_rows
                recv, sc = _pool(rows, w.H, "fp8", "ue8m0")
                sep.sep_layout(d["topk_idx"].cuda(), w.E, w.R, w.B, handle=h)
                sep.sep_dispatch(h, d["x"].cuda(), recv, payload="fp8", scale="ue8m0", recv_scales=sc)
                sep.sep_handle_sync(h)
                check_layout(h, lay)
                _check_pool(lay, d["x"], recv, sc, "fp8", "ue8m0")
                continue
            _, _, launches, _ = _run(d["topk_idx"], d["x"], w.E, w.R, w.B, "fp8", "ue8m0", handle=h)
            assert launches == 1
    finally:
        sep.sep_handle_free(h)


def test_capacity_checked_against_the_worst_case_before_anything_changes():
    w = W.WORKLOADS["decode"]
    d = W.make_inputs(w)
    h = sep.sep_handle_create(w.T, w.k, w.E, w.R, w.B)
    try:
        epoch = h.epoch
        worst = h.info().max_pool_rows
        recv, sc = _pool(worst - 1, w.H, "fp8", "ue8m0")
        with pytest.raises(sep.SepError, match="SEP_ERR_CAPACITY"):
            sep.sep_layout_dispatch(d["topk_idx"].cuda(), d["x"].cuda(), recv, w.E, w.R, w.B, payload="fp8",
                                    scale="ue8m0", recv_scales=sc, handle=h)
        assert h.epoch == epoch
    finally:
        sep.sep_handle_free(h)


@pytest.mark.parametrize("name,payload,scale", [("decode", "fp8", "ue8m0"), ("tiny", "bf16", "none")])
def test_one_launch_step_replays_from_a_cuda_graph(name, payload, scale):
    """Captured once, replayed with new routings and activations: the layout's
    and the dispatch wait's counters move by a fixed window per launch, so
    replays (which repeat the captured epoch) still synchronise."""
    from dataclasses import replace
    w = W.WORKLOADS[name]
    d0 = W.make_inputs(w)
    idx, x, wt = d0["topk_idx"].cuda(), d0["x"].cuda(), d0["topk_weight"].cuda()
    h = sep.sep_handle_create(w.T, w.k, w.E, w.R, w.B)
    try:
        rows = h.info().max_pool_rows
        recv, sc = _pool(rows, w.H, payload, scale)
        y = W.random_x(rows, w.H, seed=5).cuda()
        out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())

        def step():
            sep.sep_layout_dispatch(idx, x, recv, w.E, w.R, w.B, payload=payload, scale=scale, recv_scales=sc,
                                    handle=h, flags=ONE)
            sep.sep_combine(h, y, wt, out)

        with torch.cuda.stream(s):
            step()
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            step()
        for rep in range(4):
            d = W.make_inputs(replace(w, seed=w.seed + 13 * (rep + 1)))
            idx.copy_(d["topk_idx"])
            x.copy_(d["x"])
            wt.copy_(d["topk_weight"])
            fresh, fresh_sc = _pool(rows, w.H, payload, scale)   # a new routing's padding rows may have been
            recv.copy_(fresh)                                  # valid rows of the previous one
            if sc is not None:
                sc.copy_(fresh_sc)
            torch.cuda.synchronize()
            g.replay()
            torch.cuda.synchronize()
            lay = oracle.layout(d["topk_idx"].numpy(), w.E, w.R, w.B)
            check_layout(h, lay)
            _check_pool(lay, d["x"], recv, sc, payload, scale)
            check_combine(bf16_bits(out), oracle.combine(y.cpu(), d["topk_weight"].numpy(), lay))
        del g
    finally:
        sep.sep_handle_free(h)


@pytest.mark.parametrize("flags", [sep.SEP_LAYOUT_SYNC_COUNTS | sep.SEP_LAYOUT_TOKEN_IN_OWNER,
                                   sep.SEP_LAYOUT_SYNC_COUNTS | sep.SEP_LAYOUT_TOKEN_IN_OWNER | ONE])
def test_layout_flags_pass_through(flags):
    """SEP_LAYOUT_SYNC_COUNTS makes the exact pool size known on return and
    SEP_LAYOUT_TOKEN_IN_OWNER fills is_token_in_rank and the per-owner token
    counts, as with sep_layout."""
    w = W.WORKLOADS["decode"]
    d = W.make_inputs(w)
    lay = oracle.layout(d["topk_idx"].numpy(), w.E, w.R, w.B)
    h = sep.sep_handle_create(w.T, w.k, w.E, w.R, w.B, flags=sep.SEP_LAYOUT_TOKEN_IN_OWNER)
    try:
        rows = h.info().max_pool_rows
        recv, sc = _pool(rows, w.H, "fp8", "ue8m0")
        sep.sep_layout_dispatch(d["topk_idx"].cuda(), d["x"].cuda(), recv, w.E, w.R, w.B, payload="fp8",
                                scale="ue8m0", recv_scales=sc, handle=h, flags=flags)
        info = h.info()
        assert info.num_pool_rows == lay.num_pool_rows and info.num_tiles == lay.num_tiles
        check_layout(h, lay, token_in_owner=True)
        _check_pool(lay, d["x"], recv, sc, "fp8", "ue8m0")
    finally:
        sep.sep_handle_free(h)


@pytest.mark.parametrize("payload,scale", [("bf16", "none"), ("fp8", "ue8m0")])
def test_cta_budget_on_the_two_launches(payload, scale):
    """A CTA budget on the handle bounds the dispatch launch of
    sep_layout_dispatch: the same two launches and the same pool."""
    w = W.scaled(W.WORKLOADS["train8k"], 900)
    d = W.make_inputs(w)
    h = sep.sep_handle_create(w.T, w.k, w.E, w.R, w.B)
    try:
        sep.sep_handle_set_max_ctas(h, 5)
        _, lay, launches, recv = _run(d["topk_idx"], d["x"], w.E, w.R, w.B, payload, scale, handle=h, flags=0)
        assert launches == 2
        if payload == "bf16":
            out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
            sep.sep_combine(h, recv, d["topk_weight"].cuda(), out)
            want = oracle.combine(oracle.dispatch_bf16(d["x"], lay), d["topk_weight"].numpy(), lay)
            check_combine(bf16_bits(out), want)
    finally:
        sep.sep_handle_free(h)
