"""CPU oracle for MoE dispatch + combine.  TEST INFRASTRUCTURE ONLY.

A thin numpy/ctypes wrapper over ``oracle.c``: plain, slow, single-threaded
C that defines what the dispatch/combine path computes.  Only ``tests/``,
``__graft_entry__.smoke()`` and the benchmark's CPU baseline (and its
``--impl reference`` arm) may import it.  The product library never does and
shares no code with it.

Every function cites the passage it follows in ``oracle.c``'s header.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

SCALE_F32, SCALE_UE8M0, SCALE_F32_POW2 = 1, 2, 3
SCALE_KINDS = {"f32": SCALE_F32, "ue8m0": SCALE_UE8M0, "f32_pow2": SCALE_F32_POW2}
OK, BAD_EXPERT_ID, CAPACITY, INVALID = 0, 1, 2, 3


def build(force: bool = False) -> str:
    """Compile oracle.c with gcc (no fast-math, no FP contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def load(path: str):
    """Load an oracle shared object (the default one, or a test-built variant)."""
    L = ctypes.CDLL(path)
    P = ctypes.c_void_p
    i64, i32 = ctypes.c_int64, ctypes.c_int
    L.oracle_layout.argtypes = [P, i64, i32, i32, i32, i32] + [P] * 11 + [i64, P, P]
    L.oracle_layout.restype = i32
    L.oracle_dispatch_bf16.argtypes = [P, i64, i64, i32, P, P]
    L.oracle_dispatch_fp8.argtypes = [P, i64, i64, i32, P, i32, P, P, P, P, P, P]
    L.oracle_quant_row.argtypes = [P, i64, i32, P, P, P]
    L.oracle_dequant_rows.argtypes = [P, i64, i64, i32, P, P, P]
    L.oracle_combine.argtypes = [P, i64, i64, i32, P, P, P]
    L.oracle_dispatch_grads.argtypes = [P, i64, i64, i32, P, P, P, P, P]
    L.oracle_combine_grads.argtypes = [P, i64, i64, i32, P, P]
    L.oracle_e4m3_encode.argtypes = [ctypes.c_float]
    L.oracle_e4m3_encode.restype = ctypes.c_uint8
    L.oracle_e4m3_decode.argtypes = [ctypes.c_uint8]
    L.oracle_e4m3_decode.restype = ctypes.c_float
    L.oracle_ue8m0_exponent.argtypes = [ctypes.c_float]
    L.oracle_ue8m0_exponent.restype = i32
    L.oracle_f32_to_bf16.argtypes = [ctypes.c_float]
    L.oracle_f32_to_bf16.restype = ctypes.c_uint16
    return L


def lib(L=None):
    global _lib
    if L is not None:
        return L
    if _lib is None:
        _lib = load(build())
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def as_u16(x) -> np.ndarray:
    """bf16 data (torch tensor or uint16 array) as a contiguous uint16 numpy array."""
    if hasattr(x, "view") and hasattr(x, "dtype") and "bfloat16" in str(x.dtype):
        import torch
        return x.contiguous().view(torch.int16).numpy().view(np.uint16)
    a = np.ascontiguousarray(x)
    assert a.dtype == np.uint16
    return a


@dataclass
class Layout:
    T: int
    k: int
    E: int
    R: int
    B: int
    status: int
    expert_counts: np.ndarray
    owner_counts: np.ndarray
    owner_token_counts: np.ndarray
    is_token_in_rank: np.ndarray
    expert_pool_block_offset: np.ndarray
    owner_pool_row_offset: np.ndarray
    tile_expert: np.ndarray
    pool_arrival_target: np.ndarray
    src_pool_row: np.ndarray
    pool_recv_token: np.ndarray
    pool_recv_slot: np.ndarray
    num_pool_rows: int
    num_tiles: int


def capacity_rows(n_assign: int, E: int, B: int) -> int:
    """Rows that hold any routing of n_assign assignments: each used expert
    wastes at most B-1 padding rows."""
    return n_assign + min(E, n_assign) * (B - 1)


def layout(topk_idx, E: int, R: int, B: int, L=None) -> Layout:
    """Counts, pool layout, tile tables and stable slot maps (oracle.c: oracle_layout)."""
    idx = np.ascontiguousarray(np.asarray(topk_idx), dtype=np.int64)
    T, k = idx.shape
    cap = capacity_rows(T * k, E, B)
    nt_cap = max(1, -(-cap // B))
    i32 = np.int32
    out = dict(
        expert_counts=np.zeros(E, i32), owner_counts=np.zeros(R, i32),
        owner_token_counts=np.zeros(R, i32), is_token_in_rank=np.zeros((T, R), np.uint8),
        expert_pool_block_offset=np.zeros(E + 1, i32), owner_pool_row_offset=np.zeros(R + 1, i32),
        tile_expert=np.full(nt_cap, -7, i32), pool_arrival_target=np.full(nt_cap, -7, i32),
        src_pool_row=np.full((T, k), -7, i32), pool_recv_token=np.full(max(cap, 1), -7, i32),
        pool_recv_slot=np.full(max(cap, 1), -7, i32))
    P = ctypes.c_int64(0)
    NT = ctypes.c_int64(0)
    st = lib(L).oracle_layout(
        _p(idx), T, k, E, R, B, _p(out["expert_counts"]), _p(out["owner_counts"]),
        _p(out["owner_token_counts"]), _p(out["is_token_in_rank"]),
        _p(out["expert_pool_block_offset"]), _p(out["owner_pool_row_offset"]),
        _p(out["tile_expert"]), _p(out["pool_arrival_target"]), _p(out["src_pool_row"]),
        _p(out["pool_recv_token"]), _p(out["pool_recv_slot"]), cap,
        ctypes.byref(P), ctypes.byref(NT))
    if st == INVALID:
        raise ValueError("oracle_layout: invalid arguments")
    p, nt = P.value, NT.value
    out["tile_expert"] = out["tile_expert"][:nt]
    out["pool_arrival_target"] = out["pool_arrival_target"][:nt]
    out["pool_recv_token"] = out["pool_recv_token"][:p]
    out["pool_recv_slot"] = out["pool_recv_slot"][:p]
    return Layout(T=T, k=k, E=E, R=R, B=B, status=st, num_pool_rows=p, num_tiles=nt, **out)


def dispatch_bf16(x, lay: Layout, rows: int | None = None, fill: int = 0, L=None) -> np.ndarray:
    """recv_x [rows, H] uint16 (bf16 bits); padding rows keep ``fill`` (oracle_dispatch_bf16)."""
    xu = as_u16(x)
    T, H = xu.shape
    rows = lay.num_pool_rows if rows is None else rows
    recv = np.full((max(rows, 1), H), fill, np.uint16)
    lib(L).oracle_dispatch_bf16(_p(xu), T, H, lay.k, _p(lay.src_pool_row), _p(recv))
    return recv[:rows]


def quant_row(xrow, scale: str, L=None):
    """One token row -> (codes uint8 [H], scales [H/128]) (oracle_quant_row)."""
    xu = np.ascontiguousarray(as_u16(xrow).reshape(-1))
    H = xu.shape[0]
    codes = np.zeros(H, np.uint8)
    sf = np.zeros(H // 128, np.float32)
    su = np.zeros(H // 128, np.uint8)
    lib(L).oracle_quant_row(_p(xu), H, SCALE_KINDS[scale], _p(codes), _p(sf), _p(su))
    return codes, (su if scale == "ue8m0" else sf)


def dispatch_fp8(x, lay: Layout, scale: str, rows: int | None = None, L=None):
    """(codes uint8 [rows, H], scales [rows, H/128]) (oracle_dispatch_fp8)."""
    xu = as_u16(x)
    T, H = xu.shape
    G = H // 128
    rows = lay.num_pool_rows if rows is None else rows
    n = max(rows, 1)
    recv = np.zeros((n, H), np.uint8)
    sf = np.zeros((n, G), np.float32)
    su = np.zeros((n, G), np.uint8)
    ct = np.zeros(H, np.uint8)
    sft = np.zeros(G, np.float32)
    sut = np.zeros(G, np.uint8)
    lib(L).oracle_dispatch_fp8(_p(xu), T, H, lay.k, _p(lay.src_pool_row), SCALE_KINDS[scale],
                              _p(recv), _p(sf), _p(su), _p(ct), _p(sft), _p(sut))
    return recv[:rows], (su if scale == "ue8m0" else sf)[:rows]


def dequant_rows(codes: np.ndarray, scales: np.ndarray, scale: str, L=None) -> np.ndarray:
    """fp32 [rows, H] = decode(code) * scale (oracle_dequant_rows)."""
    codes = np.ascontiguousarray(codes, dtype=np.uint8)
    rows, H = codes.shape
    out = np.zeros((max(rows, 1), H), np.float32)
    sf = np.ascontiguousarray(scales, dtype=np.float32) if scale != "ue8m0" else np.zeros(1, np.float32)
    su = np.ascontiguousarray(scales, dtype=np.uint8) if scale == "ue8m0" else np.zeros(1, np.uint8)
    lib(L).oracle_dequant_rows(_p(codes), rows, H, SCALE_KINDS[scale], _p(sf), _p(su), _p(out))
    return out[:rows]


def combine(y_pool, topk_weight, lay: Layout, L=None) -> np.ndarray:
    """out [T, H] uint16 (bf16 bits) (oracle_combine)."""
    yu = as_u16(y_pool)
    H = yu.shape[1]
    w = np.ascontiguousarray(np.asarray(topk_weight), dtype=np.float32)
    out = np.zeros((max(lay.T, 1), H), np.uint16)
    lib(L).oracle_combine(_p(yu), lay.T, H, lay.k, _p(lay.src_pool_row), _p(w), _p(out))
    return out[:lay.T]


def e4m3_encode(v, L=None) -> np.ndarray:
    v = np.ascontiguousarray(np.asarray(v, dtype=np.float32)).reshape(-1)
    f = lib(L).oracle_e4m3_encode
    return np.array([f(float(a)) for a in v], dtype=np.uint8)


def e4m3_decode(c, L=None) -> np.ndarray:
    c = np.asarray(c, dtype=np.uint8).reshape(-1)
    f = lib(L).oracle_e4m3_decode
    return np.array([f(int(a)) for a in c], dtype=np.float32)


def ue8m0_exponent(amax: float, L=None) -> int:
    return int(lib(L).oracle_ue8m0_exponent(float(amax)))


def f32_to_bf16(v, L=None) -> np.ndarray:
    v = np.asarray(v, dtype=np.float32).reshape(-1)
    f = lib(L).oracle_f32_to_bf16
    return np.array([f(float(a)) for a in v], dtype=np.uint16)


def bf16_to_f32(u: np.ndarray) -> np.ndarray:
    return (np.asarray(u, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def dispatch_grads(grad_out, topk_weight, lay: Layout, y_pool=None, rows: int | None = None, fill: int = 0, L=None):
    """(grad_y uint16 [rows, H], grad_w float64 [T, k] or None) (oracle_dispatch_grads)."""
    g = as_u16(grad_out)
    T, H = g.shape
    rows = lay.num_pool_rows if rows is None else rows
    gy = np.full((max(rows, 1), H), fill, np.uint16)
    w = np.ascontiguousarray(np.asarray(topk_weight), dtype=np.float32)
    if y_pool is not None:
        yu = as_u16(y_pool)
        gw = np.zeros((max(T, 1), lay.k), np.float64)
        lib(L).oracle_dispatch_grads(_p(g), T, H, lay.k, _p(lay.src_pool_row), _p(w), _p(yu), _p(gy), _p(gw))
        return gy[:rows], gw[:T]
    lib(L).oracle_dispatch_grads(_p(g), T, H, lay.k, _p(lay.src_pool_row), _p(w), None, _p(gy), None)
    return gy[:rows], None


def combine_grads(grad_recv, lay: Layout, L=None) -> np.ndarray:
    """grad_x uint16 [T, H] (oracle_combine_grads)."""
    g = as_u16(grad_recv)
    H = g.shape[1]
    out = np.zeros((max(lay.T, 1), H), np.uint16)
    lib(L).oracle_combine_grads(_p(g), lay.T, H, lay.k, _p(lay.src_pool_row), _p(out))
    return out[:lay.T]
