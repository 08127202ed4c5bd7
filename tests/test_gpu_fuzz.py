"""Randomised shapes through the whole path, each checked against the oracle.

Forty seeded configurations draw the token count (zero included), top-k,
expert count, owners, BLOCK_M, hidden size, index width, masking rate, payload
and scale format, whether the layout is synced, and whether the handle is
reused from a larger routing; each runs layout -> dispatch -> combine, and the
bf16 ones also the backward pair and the scatter combine.  Layout, payload,
codes, scales, combine, grad_y and grad_x are compared bit for bit; grad_w and
the scatter within the bounds their own tests derive.
"""
import numpy as np
import pytest
import torch

import combine_route_layout_02_b200 as sep
import oracle
import workloads as W
from gpu_harness import check_combine, run_bf16_path, run_fp8_path
from test_gpu_backward import _check_backward
from test_gpu_scatter import _check_scatter

pytestmark = pytest.mark.gpu


def _config(seed):
    rng = np.random.default_rng(90_000 + seed)
    R = int(rng.choice([1, 2, 3, 4, 8]))
    E = R * int(rng.integers(1, 33))
    k = int(rng.integers(1, 13))
    T = int(rng.choice([0, 1, int(rng.integers(2, 700))], p=[0.05, 0.05, 0.9]))
    B = int(rng.choice([1, 3, 16, 64, 128, 256]))
    fp8 = bool(rng.random() < 0.35)
    H = 128 * int(rng.integers(1, 9)) if fp8 else 8 * int(rng.integers(1, 130))
    scale = str(rng.choice(["f32", "ue8m0", "f32_pow2"]))
    masked = float(rng.choice([0.0, 0.1, 0.5]))
    idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
    idx[rng.random((T, k)) < masked] = -1
    idx64 = bool(rng.random() < 0.2)
    synced = bool(rng.random() < 0.7)
    return dict(R=R, E=E, k=k, T=T, B=B, fp8=fp8, H=H, scale=scale, idx=torch.from_numpy(idx), idx64=idx64,
                synced=synced, seed=seed)


@pytest.mark.parametrize("seed", range(40))
def test_random_configuration(seed):
    c = _config(seed)
    T, H, k = c["T"], c["H"], c["k"]
    x = W.random_x(T, H, seed=seed)
    w = W.random_weights(T, k, seed=seed + 1) if T else torch.zeros(0, k)
    flags = sep.SEP_LAYOUT_SYNC_COUNTS if c["synced"] else 0
    if c["fp8"]:
        if T == 0:
            return
        run_fp8_path(c["idx"], x, c["E"], c["R"], c["B"], c["scale"], flags=flags)
        return
    run_bf16_path(c["idx"], x, w, c["E"], c["R"], c["B"], flags=flags,
                  idx_dtype=torch.int64 if c["idx64"] else torch.int32)
    if T:
        _check_backward(c["idx"], c["E"], c["R"], c["B"], H, seed=seed + 7)
        _check_scatter(c["idx"], w, c["E"], c["R"], c["B"], H, seed=seed + 9, sync=c["synced"])


def test_handle_reuse_across_random_routings():
    """One handle, sized once, laid out again and again with smaller routings
    of varying shape: every layout and combine is exact."""
    rng = np.random.default_rng(4242)
    E, R, B, k, H = 48, 4, 32, 6, 136
    h = sep.sep_handle_create(900, k, E, R, B)
    try:
        for i in range(12):
            T = int(rng.integers(0, 901))
            idx = rng.integers(-1, E, size=(T, k)).astype(np.int32)
            lay = oracle.layout(idx, E, R, B)
            sep.sep_layout(torch.from_numpy(idx).cuda(), E, R, B, handle=h)
            rows = h.info().max_pool_rows
            x = W.random_x(T, H, seed=i)
            recv = torch.empty(rows, H, dtype=torch.bfloat16, device="cuda")
            sep.sep_dispatch(h, x.cuda(), recv)
            wt = W.random_weights(T, k, seed=100 + i) if T else torch.zeros(0, k)
            out = torch.empty(max(T, 1), H, dtype=torch.bfloat16, device="cuda")
            sep.sep_combine(h, recv, wt.cuda(), out)
            torch.cuda.synchronize()
            np.testing.assert_array_equal(h.view("src_pool_row").cpu().numpy(), lay.src_pool_row)
            if T:
                want = oracle.combine(oracle.dispatch_bf16(x, lay), wt.numpy(), lay)
                got = out[:T].cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
                np.testing.assert_array_equal(got, want)
                check_combine(got, want)
    finally:
        sep.sep_handle_free(h)
