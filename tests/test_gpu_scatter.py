"""GPU check of the atomic-scatter combine against the oracle's combine.

The scatter adds each token's k weighted rows in bf16, in arrival order
(StreamEP README, "What's in the box": kernel_y's bf16 atomic scatter), so it is
neither bit-exact nor deterministic.  Its bound follows from the arithmetic:
each term w*y is rounded to bf16 (relative error <= 2^-8, the unit roundoff of
an 8-bit significand), each of the k - 1 additions rounds a partial sum whose
magnitude is at most S = sum_j |w_j y_j|, and the oracle's own result carries
one bf16 rounding; so |scatter - oracle| <= (2k + 1) * 2^-8 * S, with 2% slack
for second-order terms.

That worst case is loose: the roundings rarely line up.  A second, empirical
ceiling catches a regression well inside it.  A CPU simulation of the same
arithmetic (N(0,1) rows, renormalised weights, products and partial sums
rounded to bf16, the k terms added in a random order) puts the 99.9th
percentile of |scatter - oracle| / (2^-8 * S) at 2.0 to 2.3 for k <= 8 and its
mean at 0.31 to 0.34; the tests require the 99.9th percentile to stay at or
below 3 and the mean at or below 0.6, and print what they observe.
"""
import numpy as np
import pytest
import torch

import combine_route_layout_02_b200 as sep
import oracle
import workloads as W
from gpu_harness import bf16_bits, poisoned_bf16

pytestmark = pytest.mark.gpu


P999_CEILING, MEAN_CEILING = 3.0, 0.6       # in units of 2^-8 * S (see above)


def _abs_sum(y_bits, w, lay):
    """S = sum_j |w_j y_j| per output element."""
    y = oracle.bf16_to_f32(y_bits).astype(np.float64)
    rows = lay.src_pool_row
    S = np.zeros((lay.T, y.shape[1]))
    for j in range(lay.k):
        ok = rows[:, j] >= 0
        S[ok] += np.abs(w[ok, j, None].astype(np.float64) * y[rows[ok, j]])
    return S


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
        S = _abs_sum(oracle.as_u16(y), w.numpy(), lay)
        bound = (2 * lay.k + 1) * 2.0 ** -8 * S * 1.02
        assert np.isfinite(got).all()
        assert (err <= bound).all(), f"max err {err.max()}, worst excess {(err - bound).max()}"
        nz = S > 0
        assert (err[~nz] == 0).all()                    # tokens with nothing to add stay exactly zero
        if nz.any():
            ratio = err[nz] / (2.0 ** -8 * S[nz])
            p999, mean = float(np.quantile(ratio, 0.999)), float(ratio.mean())
            print(f"scatter error / (2^-8 S): p99.9 {p999:.3f}, mean {mean:.3f}, max {ratio.max():.3f} "
                  f"(worst-case bound {2 * lay.k + 1})")
            assert p999 <= P999_CEILING, f"99.9th percentile {p999:.3f} above {P999_CEILING}"
            assert mean <= MEAN_CEILING, f"mean {mean:.3f} above {MEAN_CEILING}"
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
