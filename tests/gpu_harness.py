"""Helpers for the GPU parity tests: run the CUDA path through the C ABI and
compare it with the CPU oracle on the same seeded inputs.

Expected values always come from ``oracle``; inputs come from ``workloads``
(or are built here from seeded generators); nothing the GPU produced is fed
to the oracle.
"""
from __future__ import annotations

import numpy as np
import torch

import combine_route_layout_02_b200 as sep
import oracle

POISON_BF16 = 0x7FC1          # a NaN bit pattern: rows that must stay unwritten keep it
POISON_U8 = 0xA5
POISON_F32_BITS = 0x7FC00ABC

# combine tolerance: |gpu - oracle| <= ATOL + RTOL * |oracle|
ATOL, RTOL = 1e-3, 1e-2


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def u16_to_bf16_tensor(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def poisoned_bf16(rows: int, H: int) -> torch.Tensor:
    return torch.full((max(rows, 1), H), POISON_BF16, dtype=torch.int16, device="cuda").view(torch.bfloat16)


def check_layout(h: sep.Handle, lay: oracle.Layout, token_in_owner: bool = False) -> None:
    """Every layout array of the handle equals the oracle's, bit for bit."""
    P, NT = lay.num_pool_rows, lay.num_tiles
    eq = np.testing.assert_array_equal
    eq(h.view("expert_counts").cpu().numpy(), lay.expert_counts)
    eq(h.view("owner_counts").cpu().numpy(), lay.owner_counts)
    eq(h.view("expert_pool_block_offset").cpu().numpy(), lay.expert_pool_block_offset)
    eq(h.view("owner_pool_row_offset").cpu().numpy(), lay.owner_pool_row_offset)
    eq(h.view("tile_expert")[:NT].cpu().numpy(), lay.tile_expert)
    eq(h.view("pool_arrival_target")[:NT].cpu().numpy(), lay.pool_arrival_target)
    eq(h.view("src_pool_row").cpu().numpy(), lay.src_pool_row)
    eq(h.view("pool_recv_token")[:P].cpu().numpy(), lay.pool_recv_token)
    eq(h.view("pool_recv_slot")[:P].cpu().numpy(), lay.pool_recv_slot)
    eq(h.view("device_sizes").cpu().numpy(), [P, NT])
    if token_in_owner:
        eq(h.view("is_token_in_rank").cpu().numpy(), lay.is_token_in_rank)
        eq(h.view("owner_token_counts").cpu().numpy(), lay.owner_token_counts)


def check_combine(got_bits: np.ndarray, want_bits: np.ndarray, exact: bool = True) -> None:
    got = oracle.bf16_to_f32(got_bits).astype(np.float64)
    want = oracle.bf16_to_f32(want_bits).astype(np.float64)
    err = np.abs(got - want)
    bad = err > ATOL + RTOL * np.abs(want)
    assert not bad.any(), f"{bad.sum()} combine outputs out of tolerance; max err {err.max()}"
    if exact:
        np.testing.assert_array_equal(got_bits, want_bits)


def run_bf16_path(idx: torch.Tensor, x: torch.Tensor, w: torch.Tensor, E: int, R: int, B: int,
                  flags: int = sep.SEP_LAYOUT_SYNC_COUNTS, idx_dtype=torch.int32,
                  y: torch.Tensor | None = None):
    """Layout + bf16 dispatch + combine on the GPU, each step checked against the oracle.

    y: optional bf16 pool for combine (defaults to the dispatched rows,
    i.e. identity experts).  Returns the handle's oracle layout."""
    T, k = idx.shape
    H = x.shape[1]
    lay = oracle.layout(idx.numpy(), E, R, B)
    h = sep.sep_layout(idx.to(idx_dtype).cuda(), E, R, B, flags=flags)
    try:
        info = h.info()
        if flags & sep.SEP_LAYOUT_SYNC_COUNTS:
            assert info.num_pool_rows == lay.num_pool_rows and info.num_tiles == lay.num_tiles
        check_layout(h, lay, token_in_owner=bool(flags & sep.SEP_LAYOUT_TOKEN_IN_OWNER))
        rows = info.num_pool_rows if info.num_pool_rows >= 0 else info.max_pool_rows
        recv = poisoned_bf16(rows, H)
        sep.sep_dispatch(h, x.cuda(), recv)
        got = bf16_bits(recv)
        want = oracle.dispatch_bf16(x, lay)
        P = lay.num_pool_rows
        valid = lay.pool_recv_token >= 0
        np.testing.assert_array_equal(got[:P][valid], want[valid])
        assert (got[:P][~valid] == POISON_BF16).all(), "a padding row was written"
        assert (got[P:] == POISON_BF16).all(), "a row past the pool was written"
        out = torch.empty(T, H, dtype=torch.bfloat16, device="cuda")
        if y is None:
            sep.sep_combine(h, recv, w.cuda(), out)
            want_out = oracle.combine(want, w.numpy(), lay)
        else:
            sep.sep_combine(h, y.cuda(), w.cuda(), out)
            want_out = oracle.combine(y, w.numpy(), lay)
        check_combine(bf16_bits(out), want_out)
        return lay
    finally:
        sep.sep_handle_free(h)


def run_fp8_path(idx: torch.Tensor, x: torch.Tensor, E: int, R: int, B: int, scale: str,
                 flags: int = sep.SEP_LAYOUT_SYNC_COUNTS):
    """Layout + FP8 dispatch on the GPU; codes and scales must equal the oracle's."""
    T, k = idx.shape
    H = x.shape[1]
    G = H // 128
    lay = oracle.layout(idx.numpy(), E, R, B)
    h = sep.sep_layout(idx.cuda(), E, R, B, flags=flags)
    try:
        check_layout(h, lay)
        info = h.info()
        rows = info.num_pool_rows if info.num_pool_rows >= 0 else info.max_pool_rows
        recv = torch.full((rows, H), POISON_U8, dtype=torch.uint8, device="cuda")
        if scale == "ue8m0":
            scales = torch.full((rows, G), POISON_U8, dtype=torch.uint8, device="cuda")
        else:
            scales = torch.full((rows, G), POISON_F32_BITS, dtype=torch.int32, device="cuda").view(torch.float32)
        sep.sep_dispatch(h, x.cuda(), recv, payload="fp8", scale=scale, recv_scales=scales)
        codes = recv.cpu().numpy()
        sc = scales.cpu().numpy()
        want_codes, want_scales = oracle.dispatch_fp8(x, lay, scale)
        P = lay.num_pool_rows
        valid = lay.pool_recv_token >= 0
        np.testing.assert_array_equal(codes[:P][valid], want_codes[valid])
        if scale == "ue8m0":
            np.testing.assert_array_equal(sc[:P][valid], want_scales[valid])
        else:
            np.testing.assert_array_equal(sc[:P][valid].view(np.uint32), want_scales[valid].view(np.uint32))
        assert (codes[:P][~valid] == POISON_U8).all(), "a padding row was written"
        assert (codes[P:] == POISON_U8).all()
        return lay, recv, scales
    finally:
        sep.sep_handle_free(h)
