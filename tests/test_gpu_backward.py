"""GPU parity of the backward pair and the per-token combine gate.

dispatch_grads (the backward of combine) and combine_grads (the backward of
dispatch) against the oracle's definitions (StreamEP README, "What's in the
box"): grad_y and grad_x bit for bit, since the kernels use the definitions'
fp32 operations in the same order; grad_w within a bound derived from its fp32
summation (the products of two bf16 values are exact in fp32, so only the
H - 1 additions round: a lane adds ceil(H/256)*8 products in sequence, the warp
adds 32 lane sums in a 5-level tree, and the oracle's fp64 sum is exact to far
below that, so |gpu - oracle| <= (ceil(H/256)*8 + 6) * 2^-24 * sum_h |g_h y_h|).

The gate (StreamEP README, opening section: y_done_per_token) is exercised in
the streaming pipeline it exists for: a streaming dispatch, the reference
consumer standing in for identity experts that stamps each token once its rows
are written, and the gated combine on a third stream; plus a partial gate and a
gate that nothing sets (bounded waits that give up, the context still usable).
"""
import numpy as np
import pytest
import torch

import combine_route_layout_02_b200 as sep
import oracle
import workloads as W
from gpu_harness import POISON_BF16, bf16_bits, check_combine, poisoned_bf16, u16_to_bf16_tensor

pytestmark = pytest.mark.gpu


def _inputs(w, T=None, H=None):
    w = W.scaled(w, T) if T is not None else w
    if H is not None:
        from dataclasses import replace
        w = replace(w, H=H)
    return w, W.make_inputs(w)


def _grad_w_bound(g_bits, y_bits, lay):
    """Per-assignment bound on |gpu - oracle| for grad_w (see the module docstring)."""
    H = g_bits.shape[1]
    n_seq = -(-H // 256) * 8 + 6
    g = oracle.bf16_to_f32(g_bits).astype(np.float64)
    y = oracle.bf16_to_f32(y_bits).astype(np.float64)
    rows = lay.src_pool_row
    ok = rows >= 0
    absdot = np.zeros(rows.shape)
    for j in range(rows.shape[1]):
        r = np.where(ok[:, j], rows[:, j], 0)
        absdot[:, j] = np.where(ok[:, j], np.abs(g * y[r]).sum(1), 0.0)
    return n_seq * 2.0 ** -24 * absdot


def _check_backward(idx, E, R, B, H, seed, with_grad_w=True):
    T, k = idx.shape
    lay = oracle.layout(idx.numpy(), E, R, B)
    g = W.random_x(T, H, seed=seed)
    w = W.random_weights(T, k, seed=seed + 1)
    P = max(lay.num_pool_rows, 1)
    y = W.random_x(P, H, seed=seed + 2)
    h = sep.sep_layout(idx.cuda(), E, R, B, flags=sep.SEP_LAYOUT_SYNC_COUNTS)
    try:
        rows = h.info().num_pool_rows
        grad_y = poisoned_bf16(rows + 3, H)
        grad_w = torch.full((max(T, 1), k), float("nan"), device="cuda") if with_grad_w else None
        y_dev = y.cuda() if with_grad_w else None
        sep.sep_dispatch_grads(h, g.cuda(), w.cuda(), grad_y, y_pool=y_dev, grad_w=grad_w)
        grad_x = poisoned_bf16(T, H)
        sep.sep_combine_grads(h, grad_y, grad_x)
        torch.cuda.synchronize()
        want_y, want_w = oracle.dispatch_grads(oracle.as_u16(g), w.numpy(), lay,
                                               y_pool=oracle.as_u16(y) if with_grad_w else None)
        valid = lay.pool_recv_token >= 0
        got_y = bf16_bits(grad_y)
        np.testing.assert_array_equal(got_y[:lay.num_pool_rows][valid], want_y[valid])
        assert (got_y[:lay.num_pool_rows][~valid] == POISON_BF16).all(), "a padding row was written"
        assert (got_y[lay.num_pool_rows:] == POISON_BF16).all(), "a row past the pool was written"
        if with_grad_w:
            got_w = grad_w.cpu().numpy().astype(np.float64)[:T]
            bound = _grad_w_bound(oracle.as_u16(g), oracle.as_u16(y), lay)
            err = np.abs(got_w - want_w)
            assert (err <= bound + 1e-30).all(), f"grad_w off by {err.max()} (bound {bound.max()})"
            assert (got_w[lay.src_pool_row < 0] == 0).all()
        # combine_grads of the kernel's own grad_y against the oracle on the same input
        want_x = oracle.combine_grads(want_y, lay)
        np.testing.assert_array_equal(bf16_bits(grad_x)[:T], want_x)
    finally:
        sep.sep_handle_free(h)


@pytest.mark.parametrize("name,T,H", [("tiny", None, None), ("decode", None, None), ("train8k", 1000, None),
                                      ("streaming", 3001, 512), ("prefill_skew", 700, 1024)])
def test_backward_pair_workloads(name, T, H):
    w, d = _inputs(W.WORKLOADS[name], T, H)
    _check_backward(d["topk_idx"], w.E, w.R, w.B, w.H, seed=50 + (T or 0))


@pytest.mark.parametrize("kind", ["one_expert", "owner_empty", "same_owner", "masked", "skew"])
def test_backward_pair_extreme_routings(kind):
    idx = W.edge_routing(kind, 777, 4, 16, 4, seed=61)
    _check_backward(idx, 16, 4, 32, 264, seed=62)          # H = 264: a ragged last 16-byte column block


@pytest.mark.parametrize("T,k,H", [(1, 1, 8), (5, 3, 24), (300, 9, 136), (64, 32, 64), (40, 4, 65536)])
def test_backward_pair_shapes(T, k, H):
    g = torch.Generator().manual_seed(T * 100 + k)
    idx = torch.randint(-1, 40, (T, k), generator=g, dtype=torch.int32)
    _check_backward(idx, 40, 4, 16, H, seed=70 + T)


def test_dispatch_grads_without_grad_w_splits_rows():
    # few tokens and a long row: the row is split over several warps
    w, d = _inputs(W.WORKLOADS["decode"], 37)
    _check_backward(d["topk_idx"], w.E, w.R, w.B, w.H, seed=80, with_grad_w=False)


def test_backward_pair_zero_tokens():
    idx = torch.zeros(0, 4, dtype=torch.int32)
    h = sep.sep_layout(idx.cuda(), 8, 2, 16, flags=sep.SEP_LAYOUT_SYNC_COUNTS)
    try:
        e = torch.empty(0, 64, dtype=torch.bfloat16, device="cuda")
        sep.sep_dispatch_grads(h, e, torch.empty(0, 4, device="cuda"), poisoned_bf16(1, 64))
        sep.sep_combine_grads(h, poisoned_bf16(1, 64), e)
        torch.cuda.synchronize()
    finally:
        sep.sep_handle_free(h)


def test_backward_rejects_a_stale_epoch_and_missing_y():
    w, d = _inputs(W.WORKLOADS["tiny"])
    h = sep.sep_layout(d["topk_idx"].cuda(), w.E, w.R, w.B, flags=sep.SEP_LAYOUT_SYNC_COUNTS)
    try:
        rows = h.info().num_pool_rows
        g = d["x"].cuda()
        wt = d["topk_weight"].cuda()
        gy = poisoned_bf16(rows, w.H)
        with pytest.raises(sep.SepError) as e:
            sep.sep_dispatch_grads(h, g, wt, gy, layout_epoch=h.epoch + 1)
        assert e.value.status == sep.SEP_ERR_HANDLE_MISMATCH
        lib = sep.library()
        st = lib.sep_dispatch_grads(h.ptr, h.epoch, g.data_ptr(), w.H, wt.data_ptr(), None, 0, gy.data_ptr(),
                                    rows, torch.empty(w.T, w.k, device="cuda").data_ptr(), None)
        assert st == sep.SEP_ERR_INVALID_ARG
        with pytest.raises(sep.SepError) as e:
            sep.sep_combine_grads(h, gy[: rows - 1], g)
        assert e.value.status == sep.SEP_ERR_CAPACITY
    finally:
        sep.sep_handle_free(h)


@pytest.mark.slow
def test_backward_pair_full_size_train8k():
    """The full train8k shape (T=8192, H=3072, E=128, k=8), every element."""
    w, d = _inputs(W.WORKLOADS["train8k"])
    _check_backward(d["topk_idx"], w.E, w.R, w.B, w.H, seed=90)


# ------------------------------------------------------------------ gate

def _gated_round(h, lay, x, recv, y_pool, tile_ready, seq, weights, out, y_done, st_c, st_g):
    """Streaming dispatch -> stamping consumer (identity experts) -> gated combine."""
    main = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    third = torch.cuda.Stream()
    ready = torch.cuda.Event()
    ready.record(main)
    side.wait_event(ready)
    third.wait_event(ready)
    sep.sep_consume_tiles_stamp(h, recv, tile_ready, seq, y_pool, st_c, y_done, seq, num_ctas=16, stream=side)
    sep.sep_combine_gated(h, y_pool, weights, out, y_done, seq, st_g, num_ctas=32, stream=third)
    sep.sep_dispatch(h, x, recv, tile_ready=tile_ready, dispatch_seq=seq, stream=main)
    main.wait_stream(side)
    main.wait_stream(third)
    torch.cuda.synchronize()


@pytest.mark.parametrize("name,T,H", [("streaming", 4096, 512), ("train8k", 2000, None), ("tiny", None, None)])
def test_gated_combine_in_the_streaming_pipeline(name, T, H):
    w, d = _inputs(W.WORKLOADS[name], T, H)
    lay = oracle.layout(d["topk_idx"].numpy(), w.E, w.R, w.B)
    h = sep.sep_layout(d["topk_idx"].cuda(), w.E, w.R, w.B)
    try:
        info = h.info()
        rows = info.max_pool_rows
        x = d["x"].cuda()
        weights = d["topk_weight"].cuda()
        tile_ready = torch.zeros(info.max_tiles, dtype=torch.int32, device="cuda")
        y_done = torch.zeros(w.T, dtype=torch.int32, device="cuda")
        st_c = torch.zeros(2, dtype=torch.int32, device="cuda")
        st_g = torch.zeros(2, dtype=torch.int32, device="cuda")
        want_pool = oracle.dispatch_bf16(d["x"], lay)
        want = oracle.combine(want_pool, d["topk_weight"].numpy(), lay)
        for seq in (1, 2, 9):
            recv = poisoned_bf16(rows, w.H)
            y_pool = poisoned_bf16(rows, w.H)
            out = poisoned_bf16(w.T, w.H)
            _gated_round(h, lay, x, recv, y_pool, tile_ready, seq, weights, out, y_done, st_c, st_g)
            assert st_c.cpu().tolist() == [0, 0] and st_g.cpu().tolist() == [0, 0]
            has_row = (lay.src_pool_row >= 0).any(1)
            yd = y_done.cpu().numpy()
            assert (yd[has_row] == seq).all()          # every token with a row was stamped
            check_combine(bf16_bits(out), want)
    finally:
        sep.sep_handle_free(h)


def test_gated_combine_partial_gate_and_timeout():
    """Only even tokens are marked done: those are reduced exactly, the odd
    ones give up after the limit (status = TIMEOUT, count = odd tokens) and keep
    their poison; the context stays usable."""
    w, d = _inputs(W.WORKLOADS["tiny"])
    lay = oracle.layout(d["topk_idx"].numpy(), w.E, w.R, w.B)
    h = sep.sep_layout(d["topk_idx"].cuda(), w.E, w.R, w.B, flags=sep.SEP_LAYOUT_SYNC_COUNTS)
    try:
        P = lay.num_pool_rows
        y = W.random_x(P, w.H, seed=5)
        y_done = torch.zeros(w.T, dtype=torch.int32)
        y_done[0::2] = 4
        y_done = y_done.cuda()
        out = poisoned_bf16(w.T, w.H)
        st = torch.zeros(2, dtype=torch.int32, device="cuda")
        sep.sep_combine_gated(h, y.cuda(), d["topk_weight"].cuda(), out, y_done, 4, st, num_ctas=4,
                              timeout_ns=20_000_000)
        torch.cuda.synchronize()
        assert st.cpu().tolist() == [sep.SEP_ERR_TIMEOUT, w.T // 2]
        want = oracle.combine(oracle.as_u16(y), d["topk_weight"].numpy(), lay)
        got = bf16_bits(out)
        np.testing.assert_array_equal(got[0::2], want[0::2])
        assert (got[1::2] == POISON_BF16).all()
        # the context still works, and a later done_seq wraps correctly
        out2 = poisoned_bf16(w.T, w.H)
        y_done.fill_(4)
        sep.sep_combine_gated(h, y.cuda(), d["topk_weight"].cuda(), out2, y_done, 3, st, num_ctas=4)
        torch.cuda.synchronize()
        assert st.cpu().tolist() == [0, 0]
        np.testing.assert_array_equal(bf16_bits(out2), want)
    finally:
        sep.sep_handle_free(h)
