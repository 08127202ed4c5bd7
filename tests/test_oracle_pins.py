"""Pins for the CPU oracle: checks against things other than the oracle itself.

* hand-worked golden examples (tests/golden/, each with its citation);
* brute-force enumeration from the definitions on tiny routings;
* invariants the pages state: counts sum to the number of valid assignments
  (N_valid,send = N_valid,recv = N_t*k, DeepEP dispatch/combine blog,
  "Correctness validation should cover extreme routing"), the pool map is a
  bijection onto valid rows, padding rows are never referenced (StreamEP
  README, "Streaming dispatch in one paragraph"), combine of an identity
  expert returns sum_j w_j x_t (blog, "When router weights are applied");
* library routines the oracle must agree with: torch's bf16 rounding and its
  float8_e4m3fn conversion (inside the non-saturating range);
* an exhaustive nearest-code search over all 256 e4m3 codes;
* mutation checks: planted mistakes in a copy of oracle.c must each fail a pin.

All of these run on the CPU.
"""
import ctypes
import json
import os
import subprocess

import numpy as np
import pytest
import torch

import oracle
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _f32_to_bf16_bits(v):
    return torch.tensor(np.asarray(v, np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


# ------------------------------------------------------------ brute force

def brute_layout(idx, E, R, B):
    """Layout straight from the definitions, by enumeration (O(N^2))."""
    idx = np.asarray(idx, np.int64)
    T, k = idx.shape
    valid = [(t, j, int(idx[t, j])) for t in range(T) for j in range(k) if 0 <= idx[t, j] < E]
    n = [sum(1 for v in valid if v[2] == e) for e in range(E)]
    tiles = [-(-n[e] // B) for e in range(E)]
    start_tile = [sum(tiles[:e]) for e in range(E)]
    src = -np.ones((T, k), np.int64)
    for (t, j, e) in valid:
        rank = sum(1 for (t2, j2, e2) in valid if e2 == e and (t2, j2) < (t, j))
        src[t, j] = start_tile[e] * B + rank
    P = sum(tiles) * B
    tok = -np.ones(P, np.int64)
    slot = -np.ones(P, np.int64)
    for (t, j, e) in valid:
        tok[src[t, j]] = t
        slot[src[t, j]] = j
    tile_expert, target = [], []
    for e in range(E):
        for i in range(tiles[e]):
            tile_expert.append(e)
            target.append(min(B, n[e] - i * B))
    E_loc = E // R
    owner_counts = [sum(n[r * E_loc:(r + 1) * E_loc]) for r in range(R)]
    in_rank = np.zeros((T, R), np.int64)
    for (t, j, e) in valid:
        in_rank[t, e // E_loc] = 1
    return dict(expert_counts=n, src_pool_row=src, pool_recv_token=tok, pool_recv_slot=slot,
                tile_expert=tile_expert, pool_arrival_target=target, num_pool_rows=P,
                owner_counts=owner_counts, is_token_in_rank=in_rank,
                owner_token_counts=in_rank.sum(0),
                expert_pool_block_offset=[0] + list(np.cumsum(tiles)),
                owner_pool_row_offset=[start_tile[r * E_loc] * B if r < R else sum(tiles) * B
                                       for r in range(R)] + [sum(tiles) * B])


def e4m3_value_table():
    """All 256 e4m3 codes decoded from the format definition (NaN for S.1111.111)."""
    vals = np.zeros(256)
    for c in range(256):
        s, e, m = c >> 7, (c >> 3) & 15, c & 7
        if e == 15 and m == 7:
            v = np.nan
        elif e == 0:
            v = m * 2.0 ** -9
        else:
            v = (1 + m / 8) * 2.0 ** (e - 7)
        vals[c] = -v if s else v
    return vals


_TABLE = e4m3_value_table()


def brute_e4m3(values):
    """Nearest finite code by exhaustive search, ties to the even mantissa,
    magnitudes beyond 448 saturate; the sign of zero is kept."""
    v = np.asarray(values, np.float64)
    codes = np.zeros(v.shape, np.uint8)
    pos = np.array([c for c in range(128) if c != 0x7f])
    posv = _TABLE[pos]
    for i, x in enumerate(v.reshape(-1)):
        a = min(abs(x), 448.0)
        d = np.abs(posv - a)
        best = np.flatnonzero(d == d.min())
        if len(best) > 1:
            best = [b for b in best if (pos[b] & 1) == 0]
        c = int(pos[best[0]])
        if np.signbit(x):
            c |= 0x80
        codes.reshape(-1)[i] = c
    return codes


# ------------------------------------------------------------ layout pins

def check_layout_against(lay, ref):
    np.testing.assert_array_equal(lay.expert_counts, ref["expert_counts"])
    np.testing.assert_array_equal(lay.src_pool_row, ref["src_pool_row"])
    np.testing.assert_array_equal(lay.pool_recv_token, ref["pool_recv_token"])
    np.testing.assert_array_equal(lay.pool_recv_slot, ref["pool_recv_slot"])
    np.testing.assert_array_equal(lay.tile_expert, ref["tile_expert"])
    np.testing.assert_array_equal(lay.pool_arrival_target, ref["pool_arrival_target"])
    np.testing.assert_array_equal(lay.owner_counts, ref["owner_counts"])
    np.testing.assert_array_equal(lay.owner_token_counts, ref["owner_token_counts"])
    np.testing.assert_array_equal(lay.is_token_in_rank, ref["is_token_in_rank"])
    np.testing.assert_array_equal(lay.expert_pool_block_offset, ref["expert_pool_block_offset"])
    np.testing.assert_array_equal(lay.owner_pool_row_offset, ref["owner_pool_row_offset"])
    assert lay.num_pool_rows == ref["num_pool_rows"]


def test_layout_golden_worked_example():
    g = _golden("layout_worked_example.json")
    lay = oracle.layout(np.array(g["topk_idx"]), g["E"], g["R"], g["B"])
    assert lay.status == oracle.OK
    check_layout_against(lay, g)
    assert lay.num_tiles == g["num_tiles"]


def _random_tiny_routings(n_cases, seed):
    rng = np.random.default_rng(seed)
    for _ in range(n_cases):
        T = int(rng.integers(0, 12))
        k = int(rng.integers(1, 5))
        R = int(rng.integers(1, 4))
        E = R * int(rng.integers(1, 4))
        B = int(rng.integers(1, 5))
        idx = rng.integers(-1, E, size=(T, k))
        yield idx, E, R, B


def test_layout_bruteforce_tiny():
    for idx, E, R, B in _random_tiny_routings(200, 7):
        lay = oracle.layout(idx, E, R, B)
        assert lay.status == oracle.OK
        check_layout_against(lay, brute_layout(idx, E, R, B))


def test_layout_bad_expert_id_reported_and_skipped():
    idx = np.array([[0, 5], [1, 2]])
    lay = oracle.layout(idx, 4, 2, 2)
    assert lay.status == oracle.BAD_EXPERT_ID
    assert lay.src_pool_row[0, 1] == -1
    assert lay.expert_counts.sum() == 3


@pytest.mark.parametrize("name", ["tiny", "decode", "train8k", "prefill_skew"])
def test_layout_invariants_on_workloads(name):
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, with_x=False)
    idx = inp["topk_idx"].numpy()
    lay = oracle.layout(idx, w.E, w.R, w.B)
    Na = w.T * w.k
    # N_valid,send = N_valid,recv = N_t * k
    assert lay.expert_counts.sum() == Na
    assert lay.pool_arrival_target.sum() == Na
    assert lay.pool_arrival_target.min() >= 1 and lay.pool_arrival_target.max() <= w.B
    assert lay.num_pool_rows == lay.num_tiles * w.B
    # bijection between valid (t, j) and valid pool rows
    rows = lay.src_pool_row.reshape(-1)
    assert (rows >= 0).all() and len(np.unique(rows)) == Na
    valid = lay.pool_recv_token >= 0
    assert valid.sum() == Na
    t_of = np.repeat(np.arange(w.T), w.k)
    j_of = np.tile(np.arange(w.k), w.T)
    np.testing.assert_array_equal(lay.pool_recv_token[rows], t_of)
    np.testing.assert_array_equal(lay.pool_recv_slot[rows], j_of)
    # padding rows are never referenced by the source->slot map
    assert not np.isin(np.flatnonzero(~valid), rows).any()
    # each row lies in the block of its own expert, and rows are (t, j)-sorted per expert
    off = lay.expert_pool_block_offset
    e_of = idx.reshape(-1)
    assert ((rows >= off[e_of] * w.B) & (rows < off[e_of + 1] * w.B)).all()
    for e in range(w.E):
        seg = lay.pool_recv_token[off[e] * w.B: off[e] * w.B + lay.expert_counts[e]] * w.k + \
            lay.pool_recv_slot[off[e] * w.B: off[e] * w.B + lay.expert_counts[e]]
        assert (np.diff(seg) > 0).all()
    # each owner's block is the contiguous run of its experts' blocks
    E_loc = w.E // w.R
    for r in range(w.R):
        assert lay.owner_pool_row_offset[r] == off[r * E_loc] * w.B
        assert lay.owner_counts[r] == lay.expert_counts[r * E_loc:(r + 1) * E_loc].sum()


def test_skewed_workload_is_skewed():
    w = W.WORKLOADS["prefill_skew"]
    lay = oracle.layout(W.make_inputs(W.scaled(w, 2048), with_x=False)["topk_idx"].numpy(), w.E, w.R, w.B)
    assert lay.owner_counts[0] > 2 * lay.owner_counts[-1]


# ---------------------------------------------------------- dispatch pins

def test_dispatch_bf16_rows_equal_source_tokens():
    w = W.WORKLOADS["tiny"]
    inp = W.make_inputs(w)
    lay = oracle.layout(inp["topk_idx"].numpy(), w.E, w.R, w.B)
    recv = oracle.dispatch_bf16(inp["x"], lay, fill=0xFFFF)
    xu = oracle.as_u16(inp["x"])
    rows = lay.src_pool_row.reshape(-1)
    np.testing.assert_array_equal(recv[rows], np.repeat(xu, w.k, axis=0))
    pad = lay.pool_recv_token < 0
    assert (recv[pad] == 0xFFFF).all()


# ------------------------------------------------------------- fp8 pins

def _fp8_dispatch_case(seed=21, T=24, k=4, E=6, R=2, B=4, H=384):
    """A routing with masked entries and duplicate experts inside a token's top-k."""
    rng = np.random.default_rng(seed)
    idx = rng.integers(-1, E, size=(T, k))
    idx[0] = [2, 2, -1, 2][:k]                   # the same expert three times, one masked entry
    idx[1] = -1                                  # a token with no assignment
    lay = oracle.layout(idx, E, R, B)
    x = W.random_x(T, H, seed=seed + 1)
    x[3, :128] = 0                               # an all-zero group
    x[5] *= 300.0                                # groups that saturate
    return lay, x


@pytest.mark.parametrize("scale", ["f32", "ue8m0", "f32_pow2"])
def test_dispatch_fp8_rows_equal_quantised_source_tokens(scale):
    """FP8 dispatch places each token's codes and per-group scales, quantised once,
    into every pool row of that token (low-latency kernels article, "FP8 and
    Quantization Support": the scales travel with the payload rows).  Each valid
    row is checked against the separately pinned single-row quantiser of its
    source token; padding rows stay untouched."""
    lay, x = _fp8_dispatch_case()
    xu = oracle.as_u16(x)
    codes, scales = oracle.dispatch_fp8(x, lay, scale)
    P = lay.num_pool_rows
    assert codes.shape == (P, x.shape[1]) and scales.shape == (P, x.shape[1] // 128)
    assert (lay.src_pool_row < 0).any() and len(set(lay.src_pool_row[0][lay.src_pool_row[0] >= 0])) == 3
    for row in range(P):
        t = lay.pool_recv_token[row]
        if t < 0:
            assert (codes[row] == 0).all() and (scales[row] == 0).all()
            continue
        want_c, want_s = oracle.quant_row(xu[t], scale)
        np.testing.assert_array_equal(codes[row], want_c)
        np.testing.assert_array_equal(scales[row], want_s)
    # every valid (t, j) reaches a row holding token t's quantisation
    for t in range(lay.T):
        for j in range(lay.k):
            r = lay.src_pool_row[t, j]
            if r >= 0:
                np.testing.assert_array_equal(codes[r], oracle.quant_row(xu[t], scale)[0])


def test_dequant_rows_follow_the_format_and_the_group_scales():
    """decode(code) times its own 128-channel group's scale, from the e4m3 value
    table of the format definition and the scale encodings (fp32 value or UE8M0
    byte b meaning 2^(b-127))."""
    rng = np.random.default_rng(31)
    rows, H = 5, 512
    codes = rng.integers(0, 256, size=(rows, H)).astype(np.uint8)
    codes[codes == 0x7f] = 0x7e
    codes[codes == 0xff] = 0xfe
    su = rng.integers(100, 150, size=(rows, H // 128)).astype(np.uint8)
    sf = rng.uniform(0.01, 3.0, size=(rows, H // 128)).astype(np.float32)
    tab = _TABLE[codes.astype(np.int64)]
    got_u = oracle.dequant_rows(codes, su, "ue8m0")
    want_u = (tab * np.repeat(2.0 ** (su.astype(np.float64) - 127), 128, axis=1)).astype(np.float32)
    np.testing.assert_array_equal(got_u, want_u)
    got_f = oracle.dequant_rows(codes, sf, "f32")
    want_f = (tab.astype(np.float32) * np.repeat(sf, 128, axis=1)).astype(np.float32)
    np.testing.assert_array_equal(got_f, want_f)



def test_e4m3_decode_matches_format_and_torch():
    g = _golden("e4m3_codes.json")
    dec = oracle.e4m3_decode(np.arange(256))
    for c, v in g["codes"].items():
        assert dec[int(c, 16)] == v and np.signbit(dec[int(c, 16)]) == np.signbit(v)
    for c in g["nan_codes"]:
        assert np.isnan(dec[int(c, 16)])
    finite = ~np.isnan(_TABLE)
    np.testing.assert_array_equal(dec[finite], _TABLE[finite].astype(np.float32))
    via_torch = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).to(torch.float32).numpy()
    np.testing.assert_array_equal(dec[finite], via_torch[finite])


def test_e4m3_encode_exhaustive_bf16():
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = oracle.bf16_to_f32(bits)
    vals = vals[np.isfinite(vals)]
    got = oracle.e4m3_encode(vals)
    np.testing.assert_array_equal(got, brute_e4m3(vals))


def test_e4m3_encode_random_fp32_vs_bruteforce_and_torch():
    rng = np.random.default_rng(3)
    mags = 2.0 ** rng.uniform(-14, 10, size=20000)
    v = (mags * rng.choice([-1.0, 1.0], size=mags.size)).astype(np.float32)
    got = oracle.e4m3_encode(v)
    np.testing.assert_array_equal(got, brute_e4m3(v))
    inr = np.abs(v) < 464.0              # torch does not saturate past 464
    ref = torch.tensor(v[inr]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    np.testing.assert_array_equal(got[inr], ref)


def test_ue8m0_exponent_definition():
    rng = np.random.default_rng(5)
    amaxes = list((2.0 ** rng.uniform(-120, 120, size=3000)).astype(np.float32))
    amaxes += [np.float32(448.0 * 2.0 ** m) for m in range(-100, 100)]       # exact boundaries
    amaxes += [np.nextafter(np.float32(448.0 * 2.0 ** m), np.float32(np.inf)) for m in range(-50, 50)]
    for a in amaxes:
        E = oracle.ue8m0_exponent(a)
        assert 448.0 * 2.0 ** E >= a
        assert E == -127 or 448.0 * 2.0 ** (E - 1) < a
    assert oracle.ue8m0_exponent(0.0) == 0
    assert oracle.ue8m0_exponent(448.0) == 0
    assert oracle.ue8m0_exponent(7.0) == -6


@pytest.mark.parametrize("scale", ["f32", "ue8m0", "f32_pow2"])
def test_quant_golden_worked_example(scale):
    g = _golden("fp8_worked_example.json")
    x = np.zeros(g["H"], np.float32)
    for i, v in g["nonzero_x"].items():
        x[int(i)] = v
    codes, scales = oracle.quant_row(_f32_to_bf16_bits(x), scale)
    exp = g[scale]
    np.testing.assert_array_equal(scales, np.array(exp["scales"], scales.dtype))
    want = np.zeros(g["H"], np.uint8)
    for i, c in exp["nonzero_codes"].items():
        want[int(i)] = int(c, 16)
    np.testing.assert_array_equal(codes, want)


@pytest.mark.parametrize("scale", ["f32", "ue8m0", "f32_pow2"])
def test_quant_random_rows_properties(scale):
    H = 1024
    x = W.random_x(6, H, seed=11)
    x[2, :128] = 0                         # an all-zero group
    x[3] *= 1e-3
    for t in range(x.shape[0]):
        xu = oracle.as_u16(x[t:t + 1])[0]
        xf = oracle.bf16_to_f32(xu).reshape(-1, 128)
        codes, scales = oracle.quant_row(xu, scale)
        amax = np.abs(xf).max(axis=1)
        if scale == "f32":
            s = np.where(amax == 0, np.float32(1), amax / np.float32(448)).astype(np.float32)
            np.testing.assert_array_equal(scales, s)
        else:
            E = np.array([oracle.ue8m0_exponent(a) for a in amax])
            assert all((448.0 * 2.0 ** e >= a) and (a == 0 or 448.0 * 2.0 ** (e - 1) < a)
                       for e, a in zip(E, amax))
            s = (2.0 ** E).astype(np.float32)
            if scale == "ue8m0":
                np.testing.assert_array_equal(scales, (E + 127).astype(np.uint8))
            else:
                np.testing.assert_array_equal(scales, s)
        q = (xf / s[:, None]).astype(np.float32)
        np.testing.assert_array_equal(codes, brute_e4m3(q.reshape(-1)))
        # dequantised values are within half an e4m3 step (relative 2^-4) of x, or 2^-10 * s absolute
        deq = oracle.dequant_rows(codes[None, :], scales[None, :], scale)[0].reshape(-1, 128)
        tol = np.maximum(np.abs(xf) * 2.0 ** -4, 2.0 ** -10 * s[:, None]) * 1.0000001
        assert (np.abs(deq - xf) <= tol).all()


# ---------------------------------------------------------- combine pins

def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(9)
    v = (rng.standard_normal(50000) * 2.0 ** rng.uniform(-30, 30, 50000)).astype(np.float32)
    ties = oracle.bf16_to_f32(rng.integers(0, 1 << 16, 2000).astype(np.uint16))
    ties = ties[np.isfinite(ties)]
    tie_vals = (ties.view(np.uint32) | 0x8000).view(np.float32)            # exact halfway points
    v = np.concatenate([v, tie_vals[np.isfinite(tie_vals)]])
    np.testing.assert_array_equal(oracle.f32_to_bf16(v), _f32_to_bf16_bits(v))


def test_combine_golden_worked_example():
    g = _golden("combine_worked_example.json")
    lay = oracle.layout(np.array(g["topk_idx"]), g["E"], g["R"], g["B"])
    np.testing.assert_array_equal(lay.src_pool_row, g["src_pool_row"])
    y = _f32_to_bf16_bits(np.array(g["y_pool"], np.float32))
    out = oracle.combine(y, np.array(g["topk_weight"], np.float32), lay)
    np.testing.assert_array_equal(oracle.bf16_to_f32(out), np.array(g["out"], np.float32))


def test_combine_within_fp32_error_of_exact_sum():
    w = W.WORKLOADS["tiny"]
    inp = W.make_inputs(w)
    lay = oracle.layout(inp["topk_idx"].numpy(), w.E, w.R, w.B)
    y = W.random_x(lay.num_pool_rows, w.H, seed=21)
    wt = inp["topk_weight"].numpy()
    out = oracle.bf16_to_f32(oracle.combine(y, wt, lay)).astype(np.float64)
    yf = oracle.bf16_to_f32(oracle.as_u16(y)).astype(np.float64)
    rows = lay.src_pool_row
    terms = wt.astype(np.float64)[:, :, None] * yf[rows]                  # [T, k, H]
    exact = terms.sum(1)
    bound = 2.0 ** -8 * np.abs(exact) + (w.k + 1) * 2.0 ** -24 * np.abs(terms).sum(1) * 1.01
    assert (np.abs(out - exact) <= bound + 1e-30).all()


def test_combine_identity_experts():
    w = W.WORKLOADS["tiny"]
    inp = W.make_inputs(w)
    lay = oracle.layout(inp["topk_idx"].numpy(), w.E, w.R, w.B)
    recv = oracle.dispatch_bf16(inp["x"], lay)
    out = oracle.bf16_to_f32(oracle.combine(recv, inp["topk_weight"].numpy(), lay))
    xf = inp["x"].float().numpy()
    # sum_j w_j x_t with sum_j w_j = 1 (to fp32 rounding)
    assert np.allclose(out, xf, rtol=2 ** -7, atol=0)
    # k = 1, weight 1: combine is an exact gather
    lay1 = oracle.layout(inp["topk_idx"].numpy()[:, :1], w.E, w.R, w.B)
    recv1 = oracle.dispatch_bf16(inp["x"], lay1)
    out1 = oracle.combine(recv1, np.ones((w.T, 1), np.float32), lay1)
    np.testing.assert_array_equal(out1, oracle.as_u16(inp["x"]))


def test_combine_skips_masked_assignments():
    idx = np.array([[0, -1], [-1, -1]])
    lay = oracle.layout(idx, 2, 1, 2)
    y = _f32_to_bf16_bits(np.array([[3.0, 4.0], [9.0, 9.0]], np.float32))
    out = oracle.bf16_to_f32(oracle.combine(y, np.array([[0.5, 100.0], [7.0, 7.0]], np.float32), lay))
    np.testing.assert_array_equal(out, [[1.5, 2.0], [0.0, 0.0]])


# ------------------------------------------------------- mutation checks

def _pins_fail(L) -> bool:
    """Run a compact set of the pins above against an oracle library; True if one fails."""
    try:
        g = _golden("layout_worked_example.json")
        lay = oracle.layout(np.array(g["topk_idx"]), g["E"], g["R"], g["B"], L=L)
        check_layout_against(lay, g)
        for idx, E, R, B in _random_tiny_routings(40, 8):
            check_layout_against(oracle.layout(idx, E, R, B, L=L), brute_layout(idx, E, R, B))
        x = W.random_x(3, 256, seed=4)
        lay = oracle.layout(np.array([[0, 1], [1, 1], [0, -1]]), 2, 1, 2, L=L)
        recv = oracle.dispatch_bf16(x, lay, L=L)
        np.testing.assert_array_equal(recv[lay.src_pool_row[:, 0]], oracle.as_u16(x))
        for scale in ("f32", "ue8m0"):
            gq = _golden("fp8_worked_example.json")
            xx = np.zeros(gq["H"], np.float32)
            for i, v in gq["nonzero_x"].items():
                xx[int(i)] = v
            codes, scales = oracle.quant_row(_f32_to_bf16_bits(xx), scale, L=L)
            np.testing.assert_array_equal(scales, np.array(gq[scale]["scales"], scales.dtype))
            want = np.zeros(gq["H"], np.uint8)
            for i, c in gq[scale]["nonzero_codes"].items():
                want[int(i)] = int(c, 16)
            np.testing.assert_array_equal(codes, want)
        lay8, x8 = _fp8_dispatch_case()
        x8u = oracle.as_u16(x8)
        for scale in ("f32", "ue8m0"):
            codes, scales = oracle.dispatch_fp8(x8, lay8, scale, L=L)
            for row in range(lay8.num_pool_rows):
                t = lay8.pool_recv_token[row]
                if t >= 0:
                    want_c, want_s = oracle.quant_row(x8u[t], scale)
                    np.testing.assert_array_equal(codes[row], want_c)
                    np.testing.assert_array_equal(scales[row], want_s)
            deq = oracle.dequant_rows(codes, scales, scale, L=L)
            sc = scales.astype(np.float64) if scale == "f32" else 2.0 ** (scales.astype(np.float64) - 127)
            want = (_TABLE[codes.astype(np.int64)] * np.repeat(sc, 128, axis=1)).astype(np.float32)
            np.testing.assert_array_equal(deq, want)
        for a in [448.0, 896.0, 7.0, 1e-3]:
            E = oracle.ue8m0_exponent(a, L=L)
            assert 448.0 * 2.0 ** E >= a and 448.0 * 2.0 ** (E - 1) < a
        gc = _golden("combine_worked_example.json")
        lay = oracle.layout(np.array(gc["topk_idx"]), gc["E"], gc["R"], gc["B"], L=L)
        y = _f32_to_bf16_bits(np.array(gc["y_pool"], np.float32))
        out = oracle.combine(y, np.array(gc["topk_weight"], np.float32), lay, L=L)
        np.testing.assert_array_equal(oracle.bf16_to_f32(out), np.array(gc["out"], np.float32))
    except AssertionError:
        return True
    return False


MUTANTS = [
    ("if (e < 0)\n            continue;\n        if (e >= E) {\n            bad = 1;",
     "if (e <= 0)\n            continue;\n        if (e >= E) {\n            bad = 1;"),        # drops expert 0
    ("(expert_counts[e] + B - 1) / B", "expert_counts[e] / B"),                             # floor, not ceil
    ("pool_recv_token[row] = (int32_t)(a / k);", "pool_recv_token[row] = (int32_t)(a % k);"),  # t/j swapped
    ("pool_arrival_target[i] = left < B ? left : B;", "pool_arrival_target[i] = B;"),
    ("e / E_loc == r", "e % R == r"),                                                     # wrong owner map
    ("src_pool_row[a] = -1;\n            continue;", "src_pool_row[a] = 0;\n            continue;"),
    ("recv[(int64_t)row * H + h] = x[t * H + h];", "recv[(int64_t)row * H + h] = x[t * H + (H - 1 - h)];"),
    ("return (fmod(f, 2.0) == 0.0) ? f : f + 1.0;", "return f + 1.0;"),                    # ties away
    ("((e + 7) << 3)", "((e + 8) << 3)"),                                                 # wrong bias
    ("amax / 448.0f", "amax / 256.0f"),
    ("while (ldexp(448.0, e - 1) >= a)", "while (ldexp(448.0, e - 1) > a)"),               # boundary
    ("scales_u8[g] = (uint8_t)(E + 127);", "scales_u8[g] = (uint8_t)(E + 128);"),
    ("acc = acc + prod;", "acc = prod;"),                                                 # dropped term
    ("float prod = topk_weight[t * k + j] *", "float prod = topk_weight[t * k + (k - 1 - j)] *"),  # wrong operand
    ("if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u)))",
     "if (lower >= 0x8000u)"),                                                            # ties away in bf16
    # FP8 dispatch: scales placed at the token's index instead of the pool row's
    ("memcpy(recv_scales_u8 + (int64_t)row * G, su_tmp, (size_t)G);",
     "memcpy(recv_scales_u8 + (int64_t)t * G, su_tmp, (size_t)G);"),
    ("memcpy(recv_scales_f32 + (int64_t)row * G, sf_tmp, (size_t)G * sizeof(float));",
     "memcpy(recv_scales_f32 + (int64_t)t * G, sf_tmp, (size_t)G * sizeof(float));"),
    # FP8 dispatch: codes written only for the first top-k slot
    ("memcpy(recv + (int64_t)row * H, codes_tmp, (size_t)H);",
     "if (j == 0) memcpy(recv + (int64_t)row * H, codes_tmp, (size_t)H);"),
    # FP8 dispatch: a group's scale taken from the wrong group
    ("memcpy(recv_scales_f32 + (int64_t)row * G, sf_tmp, (size_t)G * sizeof(float));",
     "memcpy(recv_scales_f32 + (int64_t)row * G, sf_tmp + 1, (size_t)(G - 1) * sizeof(float));"),
    # dequantisation: wrong 128-channel group, wrong UE8M0 bias
    ("scales_f32[r * G + h / 128];", "scales_f32[r * G + h / 256];"),
    ("(int)scales_u8[r * G + h / 128] - 127)", "(int)scales_u8[r * G + h / 128] - 128)"),
]


@pytest.mark.parametrize("i", range(len(MUTANTS)))
def test_planted_oracle_mistake_fails_a_pin(i, tmp_path):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "oracle.c")).read()
    old, new = MUTANTS[i]
    assert src.count(old) == 1, f"mutation pattern not unique: {old!r}"
    mutated = src.replace(old, new)
    c = tmp_path / "m.c"
    so = tmp_path / f"m{i}.so"
    c.write_text(mutated)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared",
                           "-o", str(so), str(c), "-lm"])
    assert _pins_fail(oracle.load(str(so))), f"mutant {i} passed every pin: {new!r}"


def test_unmutated_oracle_passes_the_compact_pins():
    assert not _pins_fail(None)


# --------------------------------------------------------- backward pins

def _bwd_case(seed, T=40, k=4, E=8, R=2, B=4, H=48):
    rng = np.random.default_rng(seed)
    idx = rng.integers(-1, E, size=(T, k))
    lay = oracle.layout(idx, E, R, B)
    w = rng.uniform(0.05, 1.0, size=(T, k)).astype(np.float32)
    g = oracle.as_u16(W.random_x(T, H, seed=seed + 1))
    y = oracle.as_u16(W.random_x(max(lay.num_pool_rows, 1), H, seed=seed + 2))
    return lay, w, g, y


def test_backward_golden_worked_example():
    g = _golden("backward_worked_example.json")
    lay = oracle.layout(np.array(g["topk_idx"]), g["E"], g["R"], g["B"])
    gy, gw = oracle.dispatch_grads(_f32_to_bf16_bits(np.array(g["grad_out"], np.float32)),
                                   np.array(g["topk_weight"], np.float32), lay,
                                   y_pool=_f32_to_bf16_bits(np.array(g["y_pool"], np.float32)))
    np.testing.assert_array_equal(oracle.bf16_to_f32(gy), np.array(g["grad_y"], np.float32))
    np.testing.assert_array_equal(gw, np.array(g["grad_w"]))
    gx = oracle.combine_grads(gy, lay)
    np.testing.assert_array_equal(oracle.bf16_to_f32(gx), np.array(g["grad_x"], np.float32))


def test_dispatch_grads_with_unit_weights_is_a_permutation():
    lay, _, g, y = _bwd_case(3, k=1)
    gy, _ = oracle.dispatch_grads(g, np.ones((lay.T, 1), np.float32), lay)
    rows = lay.src_pool_row[:, 0]
    ok = rows >= 0
    np.testing.assert_array_equal(gy[rows[ok]], g[ok])


def test_combine_grads_of_a_dispatch_counts_assignments():
    """combine_grads(dispatch(x))[t] = n_t * x[t], n_t the token's valid
    assignments (exact in bf16 for n_t a power of two)."""
    rng = np.random.default_rng(4)
    T, k, E = 64, 4, 8
    idx = rng.integers(0, E, size=(T, k))
    idx[::3, 1:] = -1                                    # n_t = 1 on every third token, else 4
    lay = oracle.layout(idx, E, 2, 4)
    x = W.random_x(T, 32, seed=5)
    gx = oracle.bf16_to_f32(oracle.combine_grads(oracle.dispatch_bf16(x, lay), lay))
    n = (idx >= 0).sum(1)[:, None].astype(np.float32)
    np.testing.assert_array_equal(gx, x.float().numpy() * n)


def test_backward_adjoint_identities():
    """<grad_y, y> = <g, combine(y, w)> and sum w * grad_w = the same number;
    <combine_grads(r), x> = <r, dispatch(x)> -- each to within the bf16 and
    fp32 rounding the definitions allow."""
    for seed in range(5):
        lay, w, g, y = _bwd_case(10 + seed)
        gy, gw = oracle.dispatch_grads(g, w, lay, y_pool=y)
        gf = oracle.bf16_to_f32(g).astype(np.float64)
        yf = oracle.bf16_to_f32(y).astype(np.float64)
        rows = lay.src_pool_row
        ok = rows >= 0
        # <g, combine(y, w)> in fp64 from the pinned forward definition's terms
        terms = np.where(ok[:, :, None], w.astype(np.float64)[:, :, None] * yf[np.where(ok, rows, 0)], 0.0)
        lhs = float((gf * terms.sum(1)).sum())
        valid_rows = lay.pool_recv_token >= 0
        rhs = float((oracle.bf16_to_f32(gy).astype(np.float64)[valid_rows] * yf[valid_rows]).sum())
        mag = float(np.abs(gf[:, None, :] * terms).sum())
        assert abs(lhs - rhs) <= 2.0 ** -8 * mag + 1e-9
        assert abs(float((w.astype(np.float64) * gw).sum()) - lhs) <= 1e-12 * mag + 1e-9
        # dispatch / combine_grads adjoint
        x = W.random_x(lay.T, y.shape[1], seed=seed)
        r = oracle.as_u16(W.random_x(max(lay.num_pool_rows, 1), y.shape[1], seed=seed + 7))
        d = oracle.bf16_to_f32(oracle.dispatch_bf16(x, lay)).astype(np.float64)
        rf = oracle.bf16_to_f32(r).astype(np.float64)
        lhs2 = float((oracle.bf16_to_f32(oracle.combine_grads(r, lay)).astype(np.float64)
                      * x.float().numpy()).sum())
        rhs2 = float((rf[valid_rows] * d[valid_rows]).sum())
        mag2 = float(np.abs(rf[valid_rows] * d[valid_rows]).sum())
        assert abs(lhs2 - rhs2) <= 2.0 ** -8 * mag2 * (lay.k + 1) + 1e-9


BACKWARD_MUTANTS = [
    ("float prod = w * g;", "float prod = g;"),                                     # weight dropped
    ("float w = topk_weight[t * k + j];", "float w = topk_weight[t * k + (k - 1 - j)];"),
    ("dot += (double)g * (double)oracle_bf16_to_f32(y_pool[(int64_t)row * H + h]);",
     "dot += (double)g * (double)oracle_bf16_to_f32(y_pool[(int64_t)row * H + (H - 1 - h)]);"),
    ("acc = acc + oracle_bf16_to_f32(grad_recv[(int64_t)row * H + h]);",
     "acc = oracle_bf16_to_f32(grad_recv[(int64_t)row * H + h]);"),
]


@pytest.mark.parametrize("i", range(len(BACKWARD_MUTANTS)))
def test_planted_backward_mistake_fails_a_pin(i, tmp_path):
    src = open(os.path.join(os.path.dirname(oracle.__file__), "oracle.c")).read()
    old, new = BACKWARD_MUTANTS[i]
    assert src.count(old) == 1, old
    c = tmp_path / "m.c"
    so = tmp_path / f"mb{i}.so"
    c.write_text(src.replace(old, new))
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fPIC", "-shared",
                           "-o", str(so), str(c), "-lm"])
    L = oracle.load(str(so))
    L.oracle_dispatch_grads.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int] + \
        [ctypes.c_void_p] * 5
    L.oracle_combine_grads.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                                       ctypes.c_void_p, ctypes.c_void_p]
    g = _golden("backward_worked_example.json")
    caught = False
    try:
        lay = oracle.layout(np.array(g["topk_idx"]), g["E"], g["R"], g["B"], L=L)
        gy, gw = oracle.dispatch_grads(_f32_to_bf16_bits(np.array(g["grad_out"], np.float32)),
                                       np.array(g["topk_weight"], np.float32), lay,
                                       y_pool=_f32_to_bf16_bits(np.array(g["y_pool"], np.float32)), L=L)
        np.testing.assert_array_equal(oracle.bf16_to_f32(gy), np.array(g["grad_y"], np.float32))
        np.testing.assert_array_equal(gw, np.array(g["grad_w"]))
        gx = oracle.combine_grads(gy, lay, L=L)
        np.testing.assert_array_equal(oracle.bf16_to_f32(gx), np.array(g["grad_x"], np.float32))
    except AssertionError:
        caught = True
    assert caught, f"backward mutant {i} passed the golden pin"
