"""sep_layout_noalloc: the routing layout for callers that cannot allocate.

Some callers must not call cudaMalloc on this path: a serving runtime that has
already given all of HBM to its own memory pool, code where an allocation
would synchronise the device, and deployments that need a fixed memory
footprint known at start-up.  For them the library offers one entry point that
allocates nothing: its working memory is a file-scope device array (256 KB +
256 B) and every output array belongs to the caller.

The GPU test calls it through the C ABI twice in a row on different routings
and shapes, so the second call runs on the first call's leftovers in the shared
working array, and compares every output with what sep_layout (the handle-based
entry point) produces: the layout is integer data, so they must be equal bit
for bit.  This file is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import combine_route_layout_02_b200 as sep
import workloads as W


def _outputs(T, k, E, R, B):
    Na = T * k
    worst = (Na + min(E, Na) * (B - 1) + B - 1) // B * B
    i32 = dict(dtype=torch.int32, device="cuda")
    return {
        "expert_counts": torch.full((E,), -9, **i32),
        "owner_counts": torch.full((R,), -9, **i32),
        "expert_pool_block_offset": torch.full((E + 1,), -9, **i32),
        "owner_pool_row_offset": torch.full((R + 1,), -9, **i32),
        "tile_expert": torch.full((max(worst // B, 1),), -9, **i32),
        "pool_arrival_target": torch.full((max(worst // B, 1),), -9, **i32),
        "src_pool_row": torch.full((max(T, 1), k), -9, **i32),
        "pool_recv_token": torch.full((max(worst, 1),), -9, **i32),
        "pool_recv_slot": torch.full((max(worst, 1),), -9, **i32),
        "sizes": torch.full((2,), -9, dtype=torch.int64, device="cuda"),
        "status": torch.full((2,), 7, **i32),
    }


def _compare_with_handle(idx, E, R, B, out):
    h = sep.sep_layout(idx, E, R, B, flags=sep.SEP_LAYOUT_SYNC_COUNTS)
    try:
        info = h.info()
        P, NT = info.num_pool_rows, info.num_tiles
        np.testing.assert_array_equal(out["sizes"].cpu().numpy(), [P, NT])
        for name in ("expert_counts", "owner_counts", "expert_pool_block_offset", "owner_pool_row_offset",
                     "src_pool_row"):
            np.testing.assert_array_equal(out[name].cpu().numpy(), h.view(name).cpu().numpy(), err_msg=name)
        for name in ("tile_expert", "pool_arrival_target"):
            np.testing.assert_array_equal(out[name][:NT].cpu().numpy(), h.view(name)[:NT].cpu().numpy(),
                                          err_msg=name)
        for name in ("pool_recv_token", "pool_recv_slot"):
            np.testing.assert_array_equal(out[name][:P].cpu().numpy(), h.view(name)[:P].cpu().numpy(),
                                          err_msg=name)
    finally:
        sep.sep_handle_free(h)


@pytest.mark.gpu
def test_noalloc_layout_equals_sep_layout_on_two_calls_in_a_row():
    w1 = W.WORKLOADS["train8k"]
    w2 = W.WORKLOADS["decode"]
    cases = [(W.make_inputs(w1, with_x=False)["topk_idx"], w1.E, w1.R, w1.B),
             (W.make_inputs(w2, with_x=False)["topk_idx"], w2.E, w2.R, w2.B)]
    for idx_cpu, E, R, B in cases:                      # two calls in a row, different shapes
        idx = idx_cpu.cuda()
        T, k = idx.shape
        out = _outputs(T, k, E, R, B)
        sep.sep_layout_noalloc(idx, E, R, B, out)
        torch.cuda.synchronize()
        assert out["status"].cpu().tolist() == [0, 0]
        _compare_with_handle(idx, E, R, B, out)


def test_noalloc_rejects_sizes_beyond_its_limits():
    # host-side checks, before any CUDA call
    lib = sep.library()
    la = sep.sep.LayoutArrays()
    for name, _ in sep.sep.LayoutArrays._fields_[:11]:
        setattr(la, name, 16)                           # non-null, aligned placeholders; never dereferenced
    la.max_pool_rows = 1 << 40
    la.max_tiles = 1 << 40
    too_many_experts = lib.sep_layout_noalloc(ctypes.c_void_p(16), 4, 8, 2, 512, 8, 16, ctypes.byref(la), None)
    assert too_many_experts == sep.SEP_ERR_INVALID_ARG
    assert "256" in lib.sep_last_error().decode()
    too_many_tokens = lib.sep_layout_noalloc(ctypes.c_void_p(16), 4, (1 << 21) // 8 + 1, 8, 128, 8, 128,
                                             ctypes.byref(la), None)
    assert too_many_tokens == sep.SEP_ERR_INVALID_ARG
    assert "2097152" in lib.sep_last_error().decode()
    la.max_pool_rows = 10
    small = lib.sep_layout_noalloc(ctypes.c_void_p(16), 4, 100, 2, 8, 2, 16, ctypes.byref(la), None)
    assert small == sep.SEP_ERR_CAPACITY


@pytest.mark.gpu
@pytest.mark.parametrize("T,k,E,R,B,masked", [(0, 4, 8, 2, 16, 0.0), (1, 1, 1, 1, 1, 0.0), (333, 3, 12, 4, 5, 0.3),
                                               (2048, 8, 256, 32, 64, 0.1), (9000, 6, 96, 8, 128, 0.0)])
def test_noalloc_layout_equals_the_oracle(T, k, E, R, B, masked):
    """Shapes up to the limits (E = 256), a ragged BLOCK_M, masked entries and an
    empty routing, each against the oracle directly."""
    import oracle
    rng = np.random.default_rng(T * 7 + E)
    idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
    idx[rng.random((T, k)) < masked] = -1
    lay = oracle.layout(idx, E, R, B)
    out = _outputs(T, k, E, R, B)
    sep.sep_layout_noalloc(torch.from_numpy(idx).cuda(), E, R, B, out)
    torch.cuda.synchronize()
    assert out["status"].cpu().tolist() == [0, 0]
    P, NT = lay.num_pool_rows, lay.num_tiles
    np.testing.assert_array_equal(out["sizes"].cpu().numpy(), [P, NT])
    np.testing.assert_array_equal(out["expert_counts"].cpu().numpy(), lay.expert_counts)
    np.testing.assert_array_equal(out["owner_counts"].cpu().numpy(), lay.owner_counts)
    np.testing.assert_array_equal(out["expert_pool_block_offset"].cpu().numpy(), lay.expert_pool_block_offset)
    np.testing.assert_array_equal(out["owner_pool_row_offset"].cpu().numpy(), lay.owner_pool_row_offset)
    np.testing.assert_array_equal(out["tile_expert"][:NT].cpu().numpy(), lay.tile_expert)
    np.testing.assert_array_equal(out["pool_arrival_target"][:NT].cpu().numpy(), lay.pool_arrival_target)
    if T:
        np.testing.assert_array_equal(out["src_pool_row"].cpu().numpy(), lay.src_pool_row)
    np.testing.assert_array_equal(out["pool_recv_token"][:P].cpu().numpy(), lay.pool_recv_token)
    np.testing.assert_array_equal(out["pool_recv_slot"][:P].cpu().numpy(), lay.pool_recv_slot)


def test_noalloc_wrapper_rejects_short_or_mistyped_arrays():
    """The C ABI receives only pointers, so the binding checks every output
    array's type and length before the call (CPU tensors: nothing reaches the
    library)."""
    T, k, E, R, B = 16, 2, 8, 2, 4
    idx = torch.zeros(T, k, dtype=torch.int32)
    good = {
        "expert_counts": torch.zeros(E, dtype=torch.int32), "owner_counts": torch.zeros(R, dtype=torch.int32),
        "expert_pool_block_offset": torch.zeros(E + 1, dtype=torch.int32),
        "owner_pool_row_offset": torch.zeros(R + 1, dtype=torch.int32),
        "tile_expert": torch.zeros(64, dtype=torch.int32), "pool_arrival_target": torch.zeros(64, dtype=torch.int32),
        "src_pool_row": torch.zeros(T, k, dtype=torch.int32), "pool_recv_token": torch.zeros(256, dtype=torch.int32),
        "pool_recv_slot": torch.zeros(256, dtype=torch.int32), "sizes": torch.zeros(2, dtype=torch.int64),
        "status": torch.zeros(2, dtype=torch.int32),
    }
    for name, bad in [("expert_counts", torch.zeros(E - 1, dtype=torch.int32)),
                      ("expert_pool_block_offset", torch.zeros(E, dtype=torch.int32)),
                      ("owner_pool_row_offset", torch.zeros(R, dtype=torch.int32)),
                      ("src_pool_row", torch.zeros(T * k - 1, dtype=torch.int32)),
                      ("sizes", torch.zeros(2, dtype=torch.int32)),
                      ("status", torch.zeros(1, dtype=torch.int32)),
                      ("owner_counts", torch.zeros(R, dtype=torch.int64))]:
        with pytest.raises(ValueError, match=name):
            sep.sep_layout_noalloc(idx, E, R, B, {**good, name: bad})
    missing = dict(good)
    del missing["pool_recv_slot"]
    with pytest.raises(ValueError, match="pool_recv_slot"):
        sep.sep_layout_noalloc(idx, E, R, B, missing)
    with pytest.raises(ValueError, match="device"):               # well-formed, but host memory
        sep.sep_layout_noalloc(idx, E, R, B, good)


@pytest.mark.gpu
def test_noalloc_reports_an_expert_id_out_of_range():
    """An id equal to num_experts is skipped before any memory access and
    reported in status[0]; every output equals the oracle's layout of the same
    routing with that entry masked."""
    import oracle
    T, k, E, R, B = 300, 4, 16, 4, 8
    rng = np.random.default_rng(5)
    idx = rng.integers(0, E, size=(T, k)).astype(np.int32)
    idx[17, 2] = E
    idx[250, 0] = E
    masked = idx.copy()
    masked[masked >= E] = -1
    lay = oracle.layout(masked, E, R, B)
    out = _outputs(T, k, E, R, B)
    sep.sep_layout_noalloc(torch.from_numpy(idx).cuda(), E, R, B, out)
    torch.cuda.synchronize()
    assert out["status"].cpu().tolist() == [1, 0]
    P, NT = lay.num_pool_rows, lay.num_tiles
    np.testing.assert_array_equal(out["sizes"].cpu().numpy(), [P, NT])
    np.testing.assert_array_equal(out["expert_counts"].cpu().numpy(), lay.expert_counts)
    np.testing.assert_array_equal(out["src_pool_row"].cpu().numpy(), lay.src_pool_row)
    np.testing.assert_array_equal(out["pool_recv_token"][:P].cpu().numpy(), lay.pool_recv_token)
    np.testing.assert_array_equal(out["pool_recv_slot"][:P].cpu().numpy(), lay.pool_recv_slot)
    np.testing.assert_array_equal(out["tile_expert"][:NT].cpu().numpy(), lay.tile_expert)
    np.testing.assert_array_equal(out["expert_pool_block_offset"].cpu().numpy(), lay.expert_pool_block_offset)
