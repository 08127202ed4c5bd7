"""GPU check of the atomic-scatter combine against the oracle's combine.

The scatter adds each token's k weighted rows in bf16, in arrival order
(StreamEP README, "What's in the box": kernel_y's bf16 atomic scatter), so it is
neither bit-exact nor deterministic.  Its bound follows from the arithmetic:
each term w*y is rounded to bf16 (relative error <= 2^-8, the unit roundoff of
an 8-bit significand), each of the k - 1 additions rounds a partial sum whose
magnitude is at most S = sum_j |w_j y_j|, and the oracle's own result carries
one bf16 rounding; so |scatter - oracle| <= (2k + 1) * 2^-8 * S, with 2% slack
for second-order terms.
"""
import numpy as np
import pytest
import torch

import combine_route_layout_02_b200 as sep
import oracle
import workloads as W
from gpu_harness import bf16_bits, poisoned_bf16

pytestmark = pytest.mark.gpu


def _bound(y_bits, w, lay):
    y = oracle.bf16_to_f32(y_bits).astype(np.float64)
    rows = lay.src_pool_row
    S = np.zeros((lay.T, y.shape[1]))
    for j in range(lay.k):
        ok = rows[:, j] >= 0
        S[ok] += np.abs(w[ok, j, None].astype(np.float64) * y[rows[ok, j]])
    return (2 * lay.k + 1) * 2.0 ** -8 * S * 1.02


def _check_scatter(idx, w, E, R, B, H, seed, sync=True):
    T, k = idx.shape
    lay = oracle.layout(idx.numpy(), E, R, B)
    y = W.random_x(max(lay.num_pool_rows, 1), H, seed=seed)
    h = sep.sep_layout(idx.cuda(), E, R, B, flags=sep.SEP_LAYOUT_SYNC_COUNTS if sync else 0)
    try:
        rows = h.info().max_pool_rows if not sync else lay.num_pool_rows
        y_dev = poisoned_bf16(max(rows, 1), H)        # rows past P stay poison: never read
        y_dev[: lay.num_pool_rows] = y.cuda()[: lay.num_pool_rows]
        out = poisoned_bf16(T, H)
        sep.sep_combine_scatter(h, y_dev, w.cuda(), out)
        torch.cuda.synchronize()
        got = oracle.bf16_to_f32(bf16_bits(out)).astype(np.float64)
        want = oracle.bf16_to_f32(oracle.combine(oracle.as_u16(y), w.numpy(), lay)).astype(np.float64)
        err = np.abs(got - want)
        bound = _bound(oracle.as_u16(y), w.numpy(), lay)
        assert np.isfinite(got).all()
        assert (err <= bound).all(), f"max err {err.max()}, worst excess {(err - bound).max()}"
        return err.max()
    finally:
        sep.sep_handle_free(h)


@pytest.mark.parametrize("name,T,H", [("tiny", None, None), ("train8k", 1000, None), ("streaming", 3001, 512),
                                      ("decode", None, None)])
def test_scatter_combine_workloads(name, T, H):
    w = W.WORKLOADS[name]
    w = W.scaled(w, T) if T else w
    if H:
        from dataclasses import replace
        w = replace(w, H=H)
    d = W.make_inputs(w, with_x=False)
    _check_scatter(d["topk_idx"], d["topk_weight"], w.E, w.R, w.B, w.H, seed=300 + (T or 0))


@pytest.mark.parametrize("kind", ["one_expert", "masked", "skew"])
def test_scatter_combine_extreme_routings(kind):
    idx = W.edge_routing(kind, 555, 4, 16, 4, seed=31)
    wts = W.random_weights(555, 4, seed=32)
    _check_scatter(idx, wts, 16, 4, 32, 264, seed=33)


def test_scatter_combine_on_an_unsynced_layout():
    """The grid covers the worst-case pool; rows past the device-side P are
    skipped (they are poison here and would show up as NaN)."""
    w = W.scaled(W.WORKLOADS["train8k"], 700)
    d = W.make_inputs(w, with_x=False)
    _check_scatter(d["topk_idx"], d["topk_weight"], w.E, w.R, w.B, w.H, seed=34, sync=False)


def test_scatter_combine_largest_hidden():
    """H = 65536, the largest the ABI accepts: 8192 16-byte vectors per row."""
    idx = W.edge_routing("uniform", 40, 4, 16, 4, seed=34)
    wts = W.random_weights(40, 4, seed=35)
    _check_scatter(idx, wts, 16, 4, 32, 65536, seed=36)
