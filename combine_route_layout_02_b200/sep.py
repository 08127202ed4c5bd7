"""Thin ctypes binding of the sep C ABI (include/sep.h).

Argument marshalling only: every step of layout, dispatch and combine runs in
the CUDA kernels of ``libsep.so``.  PyTorch supplies device memory and streams.
Each function has the name of the C entry point it calls.  There is no CPU
path: if the library cannot be loaded, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os
import re
from dataclasses import dataclass

import torch

from . import build as _build

SEP_OK, SEP_ERR_INVALID_ARG, SEP_ERR_CAPACITY, SEP_ERR_BAD_EXPERT_ID = 0, 1, 2, 3
SEP_ERR_HANDLE_MISMATCH, SEP_ERR_TIMEOUT, SEP_ERR_CUDA = 4, 5, 6
SEP_PAYLOAD_BF16, SEP_PAYLOAD_FP8_E4M3 = 0, 1
SEP_SCALE_NONE, SEP_SCALE_F32, SEP_SCALE_UE8M0, SEP_SCALE_F32_POW2 = 0, 1, 2, 3
SEP_LAYOUT_SYNC_COUNTS, SEP_LAYOUT_TOKEN_IN_OWNER, SEP_LAYOUT_ONE_LAUNCH = 0x1, 0x2, 0x4

PAYLOADS = {"bf16": SEP_PAYLOAD_BF16, "fp8": SEP_PAYLOAD_FP8_E4M3}
SCALES = {"none": SEP_SCALE_NONE, "f32": SEP_SCALE_F32, "ue8m0": SEP_SCALE_UE8M0,
          "f32_pow2": SEP_SCALE_F32_POW2}

_P = ctypes.c_void_p
_i32, _i64, _u32, _u64 = ctypes.c_int, ctypes.c_int64, ctypes.c_uint32, ctypes.c_uint64


class LayoutInfo(ctypes.Structure):
    """Mirror of sep_layout_info."""
    _fields_ = [
        ("num_tokens", _i64), ("top_k", ctypes.c_int32), ("num_experts", ctypes.c_int32),
        ("num_owners", ctypes.c_int32), ("block_m", ctypes.c_int32), ("max_tokens", _i64),
        ("max_pool_rows", _i64), ("max_tiles", _i64), ("num_pool_rows", _i64), ("num_tiles", _i64),
        ("epoch", _u32), ("flags", _u32),
        ("expert_counts", _P), ("owner_counts", _P), ("owner_token_counts", _P),
        ("is_token_in_rank", _P), ("expert_pool_block_offset", _P), ("owner_pool_row_offset", _P),
        ("tile_expert", _P), ("pool_arrival_target", _P), ("pool_arrival_count", _P),
        ("src_pool_row", _P), ("pool_recv_token", _P), ("pool_recv_slot", _P), ("device_sizes", _P),
    ]


class LayoutArrays(ctypes.Structure):
    """Mirror of sep_layout_arrays (caller-owned outputs of sep_layout_noalloc)."""
    _fields_ = [
        ("expert_counts", _P), ("owner_counts", _P), ("expert_pool_block_offset", _P),
        ("owner_pool_row_offset", _P), ("tile_expert", _P), ("pool_arrival_target", _P),
        ("src_pool_row", _P), ("pool_recv_token", _P), ("pool_recv_slot", _P), ("sizes", _P),
        ("status", _P), ("max_pool_rows", _i64), ("max_tiles", _i64),
    ]


class RecvView(ctypes.Structure):
    """Mirror of sep_recv_view."""
    _fields_ = [("slab", _P), ("row_indices", _P), ("num_rows", _i64), ("row_bytes", _i64),
                ("indexed", ctypes.c_int32), ("epoch", _u32)]


# (name, restype, argtypes) of every entry point declared in include/sep.h
_SIGNATURES = [
    ("sep_layout", _i32, [_P, _i32, _i64, _i32, _i32, _i32, _i32, _u32, _P, ctypes.POINTER(_P)]),
    ("sep_handle_create", _i32, [_i64, _i32, _i32, _i32, _i32, _u32, _P, ctypes.POINTER(_P)]),
    ("sep_handle_info", _i32, [_P, ctypes.POINTER(LayoutInfo)]),
    ("sep_handle_sync", _i32, [_P, _P]),
    ("sep_handle_set_max_ctas", _i32, [_P, _i32]),
    ("sep_dispatch", _i32, [_P, _P, _i64, _i32, _i32, _P, _P, _i64, _P, _i64, _u32, _P]),
    ("sep_combine", _i32, [_P, _u32, _P, _i64, _i64, _P, _P, _P]),
    ("sep_consume_tiles", _i32, [_P, _P, _i64, _i64, _P, _i64, _u32, _P, _i32, _u64, _P, _P]),
    ("sep_handle_free", None, [_P]),
    ("sep_last_error", ctypes.c_char_p, []),
    ("sep_status_string", ctypes.c_char_p, [_i32]),
    ("sep_abi_version", _i32, []),
    ("sep_launch_count", _u64, []),
    ("sep_dispatch_borrow", _i32, [_P, _P, _i64, _i32, ctypes.POINTER(RecvView)]),
    ("sep_view_release", _i32, [_P, ctypes.POINTER(_P), _i32]),
    ("sep_gather_rows", _i32, [ctypes.POINTER(RecvView), _P, _i64, _P]),
    ("sep_layout_dispatch", _i32, [_P, _i32, _i64, _i32, _i32, _i32, _i32, _u32, _P, _i64, _i32, _i32, _P, _P, _i64,
                                   _P, ctypes.POINTER(_P)]),
    ("sep_layout_noalloc", _i32, [_P, _i32, _i64, _i32, _i32, _i32, _i32, ctypes.POINTER(LayoutArrays), _P]),
    ("sep_consume_tiles_stamp", _i32, [_P, _P, _i64, _i64, _P, _i64, _u32, _P, _i32, _u64, _P, _P, _i64, _u32,
                                       _P]),
    ("sep_combine_gated", _i32, [_P, _u32, _P, _i64, _i64, _P, _P, _P, _i64, _u32, _i32, _u64, _P, _P]),
    ("sep_dispatch_grads", _i32, [_P, _u32, _P, _i64, _P, _P, _i64, _P, _i64, _P, _P]),
    ("sep_combine_grads", _i32, [_P, _u32, _P, _i64, _i64, _P, _P]),
    ("sep_combine_scatter", _i32, [_P, _u32, _P, _i64, _i64, _P, _P, _P]),
    ("sep_ep_plan", _i32, [_P, _i32, _i32, _i32, _i32, _P, _P, _P, _P]),
    ("sep_ep_dispatch", _i32, [_P, _u32, _P, _i64, _i32, _P, _P, _P, _P, _P, _P, _P, _P]),
    ("sep_ep_mark_padding", _i32, [_i32, _i32, _P, _P, _i64, _P, _P, _P, _P]),
    ("sep_ep_dispatch_fp8", _i32, [_P, _u32, _P, _i64, _i32, _i32, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    ("sep_ep_combine", _i32, [_P, _u32, _P, _P, _i64, _P, _P, _P, _P, _P]),
    ("sep_ep_plan_device", _i32, [_P, _i32, _i32, _i32, _i32, _P, _P, _P, _P, _P, _P, _P, _P]),
    ("sep_ep_dispatch_publish", _i32, [_P, _u32, _P, _i64, _i32, _i32, _i32, _P, _P, _P, _P, _P, _P, _P, _P, _P,
                                       _P, _P, _u32, _P, _P]),
    ("sep_ep_consume_tiles", _i32, [_i32, _i32, _P, _P, _P, _i64, _i64, _P, _P, _u32, _P, _i32, _u64, _P, _P]),
    ("sep_ep_buffer_alloc", _i32, [_i64, ctypes.POINTER(_P), _P]),
    ("sep_ep_buffer_open", _i32, [_P, ctypes.POINTER(_P)]),
    ("sep_ep_buffer_close", _i32, [_P, _i32]),
]


def _load() -> ctypes.CDLL:
    path = _build.build()          # compiles only when missing or older than its sources
    lib = ctypes.CDLL(path)
    for name, res, args in _SIGNATURES:
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def library() -> ctypes.CDLL:
    return _lib


def library_path() -> str:
    return _build.LIB


def declared_entry_points(header: str | None = None) -> list[str]:
    """Entry-point names declared in include/sep.h."""
    header = header or os.path.join(_build.INCLUDE, "sep.h")
    text = open(header).read()
    return sorted(set(re.findall(r"^SEP_API\s+[^;(]*?\b(sep_\w+)\s*\(", text, flags=re.M)))


class SepError(RuntimeError):
    def __init__(self, status: int, where: str):
        msg = _lib.sep_last_error().decode(errors="replace")
        name = _lib.sep_status_string(status).decode()
        super().__init__(f"{where}: {name}: {msg}")
        self.status = status


def _check(status: int, where: str) -> None:
    if status != SEP_OK:
        raise SepError(status, where)


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _ptr(t) -> ctypes.c_void_p:
    if t is None:
        return ctypes.c_void_p(None)
    if not t.is_cuda:
        raise ValueError("sep takes device tensors")
    if not t.is_contiguous():
        raise ValueError("sep takes contiguous tensors")
    return ctypes.c_void_p(t.data_ptr())


class _DeviceArray:
    """A raw device array seen by torch through __cuda_array_interface__."""

    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (ptr, False), "version": 3, "strides": None}


@dataclass
class Handle:
    """Owns one sep_handle*; free it with sep_handle_free (or close())."""
    ptr: ctypes.c_void_p

    def info(self) -> LayoutInfo:
        info = LayoutInfo()
        _check(_lib.sep_handle_info(self.ptr, ctypes.byref(info)), "sep_handle_info")
        return info

    @property
    def epoch(self) -> int:
        return self.info().epoch

    def view(self, name: str) -> torch.Tensor:
        """Copy of one of the handle's device arrays (current layout only)."""
        info = self.info()
        T, k, E, R = info.num_tokens, info.top_k, info.num_experts, info.num_owners
        shapes = {
            "expert_counts": ((E,), "<i4"), "owner_counts": ((R,), "<i4"),
            "owner_token_counts": ((R,), "<i4"), "is_token_in_rank": ((T, R), "|u1"),
            "expert_pool_block_offset": ((E + 1,), "<i4"), "owner_pool_row_offset": ((R + 1,), "<i4"),
            "tile_expert": ((info.max_tiles,), "<i4"), "pool_arrival_target": ((info.max_tiles,), "<i4"),
            "pool_arrival_count": ((info.max_tiles,), "<i4"), "src_pool_row": ((T, k), "<i4"),
            "pool_recv_token": ((info.max_pool_rows,), "<i4"),
            "pool_recv_slot": ((info.max_pool_rows,), "<i4"), "device_sizes": ((2,), "<i8"),
        }
        shape, typestr = shapes[name]
        ptr = getattr(info, name)
        if ptr is None or 0 in shape:
            dt = {"<i4": torch.int32, "|u1": torch.uint8, "<i8": torch.int64}[typestr]
            return torch.zeros(shape, dtype=dt, device="cuda")
        t = torch.as_tensor(_DeviceArray(ptr, shape, typestr), device="cuda")
        return t.clone()

    def close(self) -> None:
        if self.ptr:
            _lib.sep_handle_free(self.ptr)
            self.ptr = ctypes.c_void_p(None)


def sep_handle_create(max_tokens: int, top_k: int, num_experts: int, num_owners: int, block_m: int,
                      flags: int = 0, stream=None) -> Handle:
    out = ctypes.c_void_p(None)
    _check(_lib.sep_handle_create(max_tokens, top_k, num_experts, num_owners, block_m, flags,
                                  _stream(stream), ctypes.byref(out)), "sep_handle_create")
    return Handle(out)


def sep_layout(topk_idx: torch.Tensor, num_experts: int, num_owners: int, block_m: int,
               flags: int = 0, handle: Handle | None = None, stream=None) -> Handle:
    """Lay out a routing; reuses ``handle`` when given (its previous layout is invalidated)."""
    if topk_idx.dtype not in (torch.int32, torch.int64) or topk_idx.dim() != 2:
        raise ValueError("topk_idx must be a [T, k] int32 or int64 tensor")
    T, k = topk_idx.shape
    h = handle.ptr if handle is not None else ctypes.c_void_p(None)
    _check(_lib.sep_layout(_ptr(topk_idx) if T else ctypes.c_void_p(None), topk_idx.element_size(),
                           T, k, num_experts, num_owners, block_m, flags, _stream(stream),
                           ctypes.byref(h)), "sep_layout")
    if handle is not None:
        handle.ptr = h
        return handle
    return Handle(h)


def sep_handle_sync(handle: Handle, stream=None) -> None:
    _check(_lib.sep_handle_sync(handle.ptr, _stream(stream)), "sep_handle_sync")


def sep_handle_set_max_ctas(handle: Handle, max_ctas: int) -> None:
    """CTA budget of the handle's dispatch and combine launches (0: unbounded)."""
    _check(_lib.sep_handle_set_max_ctas(handle.ptr, int(max_ctas)), "sep_handle_set_max_ctas")


def sep_dispatch(handle: Handle, x: torch.Tensor, recv_x: torch.Tensor, payload: str = "bf16",
                 scale: str = "none", recv_scales: torch.Tensor | None = None,
                 tile_ready: torch.Tensor | None = None, dispatch_seq: int = 0, stream=None) -> None:
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise ValueError("x must be a [T, H] bf16 tensor")
    _check(_lib.sep_dispatch(handle.ptr, _ptr(x), x.shape[1], PAYLOADS[payload], SCALES[scale],
                             _ptr(recv_x), _ptr(recv_scales), recv_x.shape[0], _ptr(tile_ready),
                             0 if tile_ready is None else tile_ready.numel(), dispatch_seq,
                             _stream(stream)), "sep_dispatch")


def sep_layout_dispatch(topk_idx: torch.Tensor, x: torch.Tensor, recv_x: torch.Tensor, num_experts: int,
                        num_owners: int, block_m: int, payload: str = "bf16", scale: str = "none",
                        recv_scales: torch.Tensor | None = None, flags: int = 0, handle: Handle | None = None,
                        stream=None) -> Handle:
    """Layout and dispatch of one routing in one call (flags SEP_LAYOUT_ONE_LAUNCH: one
    cooperative launch when the routing is small; by default the two kernels)."""
    if topk_idx.dtype not in (torch.int32, torch.int64) or topk_idx.dim() != 2:
        raise ValueError("topk_idx must be a [T, k] int32 or int64 tensor")
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise ValueError("x must be a [T, H] bf16 tensor")
    T, k = topk_idx.shape
    h = handle.ptr if handle is not None else ctypes.c_void_p(None)
    _check(_lib.sep_layout_dispatch(_ptr(topk_idx) if T else ctypes.c_void_p(None), topk_idx.element_size(),
                                    T, k, num_experts, num_owners, block_m, flags, _ptr(x), x.shape[1],
                                    PAYLOADS[payload], SCALES[scale], _ptr(recv_x), _ptr(recv_scales),
                                    recv_x.shape[0], _stream(stream), ctypes.byref(h)), "sep_layout_dispatch")
    if handle is not None:
        handle.ptr = h
        return handle
    return Handle(h)


def sep_combine(handle: Handle, y_pool: torch.Tensor, topk_weight: torch.Tensor, out: torch.Tensor,
                layout_epoch: int | None = None, stream=None) -> None:
    if y_pool.dtype != torch.bfloat16 or out.dtype != torch.bfloat16 or topk_weight.dtype != torch.float32:
        raise ValueError("y_pool/out must be bf16 and topk_weight fp32")
    epoch = handle.epoch if layout_epoch is None else layout_epoch
    _check(_lib.sep_combine(handle.ptr, epoch, _ptr(y_pool), y_pool.shape[1], y_pool.shape[0],
                            _ptr(topk_weight), _ptr(out), _stream(stream)), "sep_combine")


def sep_consume_tiles(handle: Handle, recv_x: torch.Tensor, tile_ready: torch.Tensor, dispatch_seq: int,
                      dst: torch.Tensor, status: torch.Tensor, num_ctas: int = 16, timeout_ns: int = 0,
                      stream=None) -> None:
    row_bytes = recv_x.shape[1] * recv_x.element_size()
    if dst.shape[0] < recv_x.shape[0] or dst.shape[1] * dst.element_size() != row_bytes:
        raise ValueError("dst must have recv_x's row size and at least its rows")
    if status.numel() < 2 or status.element_size() != 4:
        raise ValueError("status must hold two 32-bit words")
    _check(_lib.sep_consume_tiles(handle.ptr, _ptr(recv_x), row_bytes, recv_x.shape[0], _ptr(tile_ready),
                                  tile_ready.numel(), dispatch_seq, _ptr(dst), num_ctas, timeout_ns,
                                  _ptr(status), _stream(stream)), "sep_consume_tiles")


def sep_ep_plan(all_counts, rank: int, block_m: int) -> dict:
    """Host-only plan from every rank's expert counts (numpy int32 [R, E]):
    delta [E], owner_rows [R], owner_block_offset [E/R + 1], owner_expert_counts [E/R]."""
    import numpy as np
    counts = np.ascontiguousarray(np.asarray(all_counts, dtype=np.int32))
    R, E = counts.shape
    El = E // R if R > 0 and E % R == 0 else 1
    delta = np.zeros(E, np.int32)
    rows = np.zeros(R, np.int64)
    boff = np.zeros(El + 1, np.int32)
    ecnt = np.zeros(El, np.int32)
    _check(_lib.sep_ep_plan(counts.ctypes.data, R, E, block_m, rank, delta.ctypes.data, rows.ctypes.data,
                            boff.ctypes.data, ecnt.ctypes.data), "sep_ep_plan")
    return {"delta": delta, "owner_rows": rows, "owner_block_offset": boff, "owner_expert_counts": ecnt}


def _ptr_array(tensors):
    arr = (ctypes.c_void_p * len(tensors))()
    for i, t in enumerate(tensors):
        arr[i] = None if t is None else t.data_ptr()
    return arr


def sep_ep_dispatch(handle: Handle, x: torch.Tensor, rank: int, delta: torch.Tensor, pools, pool_rows,
                    error: torch.Tensor, recv_token=None, recv_rank=None, recv_slot=None,
                    layout_epoch: int | None = None, stream=None) -> None:
    """Rows of this rank's tokens into the owners' pools (lists of R device tensors)."""
    if x.dtype != torch.bfloat16 or delta.dtype != torch.int32:
        raise ValueError("x must be bf16 and delta int32")
    R = len(pools)
    rows = (ctypes.c_int64 * R)(*[int(r) for r in pool_rows])
    maps = [None if m is None else _ptr_array(m) for m in (recv_token, recv_rank, recv_slot)]
    epoch = handle.epoch if layout_epoch is None else layout_epoch
    _check(_lib.sep_ep_dispatch(handle.ptr, epoch, _ptr(x), x.shape[1], rank, _ptr(delta), _ptr_array(pools), rows,
                                maps[0], maps[1], maps[2], _ptr(error), _stream(stream)), "sep_ep_dispatch")


def sep_ep_dispatch_fp8(handle: Handle, x: torch.Tensor, rank: int, delta: torch.Tensor, pools, scales, pool_rows,
                        error: torch.Tensor, scale: str = "ue8m0", recv_token=None, recv_rank=None, recv_slot=None,
                        layout_epoch: int | None = None, stream=None) -> None:
    """FP8 rows (codes + per-128-channel scales) of this rank's tokens into the owners' pools."""
    if x.dtype != torch.bfloat16 or delta.dtype != torch.int32:
        raise ValueError("x must be bf16 and delta int32")
    R = len(pools)
    rows = (ctypes.c_int64 * R)(*[int(r) for r in pool_rows])
    maps = [None if m is None else _ptr_array(m) for m in (recv_token, recv_rank, recv_slot)]
    epoch = handle.epoch if layout_epoch is None else layout_epoch
    _check(_lib.sep_ep_dispatch_fp8(handle.ptr, epoch, _ptr(x), x.shape[1], rank, SCALES[scale], _ptr(delta),
                                    _ptr_array(pools), _ptr_array(scales), rows, maps[0], maps[1], maps[2],
                                    _ptr(error), _stream(stream)), "sep_ep_dispatch_fp8")


def sep_ep_plan_device(all_counts: torch.Tensor, rank: int, block_m: int, stream=None) -> dict:
    """sep_ep_plan on the GPU from device counts int32 [R, E]: device tensors delta [E],
    owner_rows [R] (int64), owner_block_offset [E/R + 1], owner_expert_counts [E/R],
    expert_rows [E], expert_tile_offset [E] and error [1]."""
    if all_counts.dtype != torch.int32 or all_counts.dim() != 2 or not all_counts.is_cuda:
        raise ValueError("all_counts must be a device int32 [R, E] tensor")
    counts = all_counts.contiguous()
    R, E = counts.shape
    El = E // R if R > 0 and E % R == 0 else 1
    dev = counts.device
    i32 = dict(dtype=torch.int32, device=dev)
    out = dict(delta=torch.zeros(E, **i32), owner_rows=torch.zeros(R, dtype=torch.int64, device=dev),
               owner_block_offset=torch.zeros(El + 1, **i32), owner_expert_counts=torch.zeros(El, **i32),
               expert_rows=torch.zeros(E, **i32), expert_tile_offset=torch.zeros(E, **i32),
               error=torch.zeros(1, **i32))
    _check(_lib.sep_ep_plan_device(_ptr(counts), R, E, block_m, rank, _ptr(out["delta"]), _ptr(out["owner_rows"]),
                                   _ptr(out["owner_block_offset"]), _ptr(out["owner_expert_counts"]),
                                   _ptr(out["expert_rows"]), _ptr(out["expert_tile_offset"]), _ptr(out["error"]),
                                   _stream(stream)), "sep_ep_plan_device")
    return out


def sep_ep_dispatch_publish(handle: Handle, x: torch.Tensor, rank: int, plan: dict, pools, pool_rows,
                            tile_ready, arrival_count, dispatch_seq: int, error: torch.Tensor, payload: str = "bf16",
                            scale: str = "none", scales=None, recv_token=None, recv_rank=None, recv_slot=None,
                            layout_epoch: int | None = None, stream=None) -> None:
    """This rank's rows into the owners' pools, each owner tile published (tile_ready
    = dispatch_seq) once complete.  plan: sep_ep_plan_device's tensors."""
    if x.dtype != torch.bfloat16:
        raise ValueError("x must be bf16")
    R = len(pools)
    B = handle.info().block_m
    for o in range(R):
        need = -(-int(pool_rows[o]) // B)
        if tile_ready[o].numel() < need or arrival_count[o].numel() < need or tile_ready[o].element_size() != 4 \
                or arrival_count[o].element_size() != 4:
            raise ValueError(f"tile_ready[{o}] / arrival_count[{o}] must hold {need} 32-bit entries")
    rows = (ctypes.c_int64 * R)(*[int(r) for r in pool_rows])
    maps = [None if m is None else _ptr_array(m) for m in (recv_token, recv_rank, recv_slot)]
    epoch = handle.epoch if layout_epoch is None else layout_epoch
    _check(_lib.sep_ep_dispatch_publish(handle.ptr, epoch, _ptr(x), x.shape[1], rank, PAYLOADS[payload],
                                        SCALES[scale], _ptr(plan["delta"]), _ptr_array(pools),
                                        None if scales is None else _ptr_array(scales), rows, maps[0], maps[1],
                                        maps[2], _ptr_array(tile_ready), _ptr_array(arrival_count),
                                        _ptr(plan["expert_rows"]), _ptr(plan["expert_tile_offset"]), dispatch_seq,
                                        _ptr(error), _stream(stream)), "sep_ep_dispatch_publish")


def sep_ep_consume_tiles(owner_block_offset: torch.Tensor, pool: torch.Tensor, recv_token: torch.Tensor,
                         tile_ready: torch.Tensor, arrival_count: torch.Tensor, dispatch_seq: int, dst: torch.Tensor,
                         status: torch.Tensor, block_m: int, num_ctas: int = 16, timeout_ns: int = 0,
                         stream=None) -> None:
    """Owner side: copy each published tile of pool into dst (valid rows only)."""
    rows = pool.shape[0]
    row_bytes = pool.shape[1] * pool.element_size()
    if dst.shape[0] < rows or dst.shape[1] * dst.element_size() != row_bytes or recv_token.numel() < rows:
        raise ValueError("dst and recv_token must cover the pool's rows")
    need = rows // block_m
    if tile_ready.numel() < need or arrival_count.numel() < need or status.numel() < 2:
        raise ValueError("tile_ready / arrival_count must cover the pool's tiles and status hold two words")
    _check(_lib.sep_ep_consume_tiles(owner_block_offset.numel() - 1, block_m, _ptr(owner_block_offset), _ptr(pool),
                                     _ptr(recv_token), row_bytes, rows, _ptr(tile_ready), _ptr(arrival_count),
                                     dispatch_seq, _ptr(dst), num_ctas, timeout_ns, _ptr(status), _stream(stream)),
           "sep_ep_consume_tiles")


def sep_ep_mark_padding(owner_block_offset: torch.Tensor, owner_expert_counts: torch.Tensor, block_m: int,
                        pool_rows: int, recv_token=None, recv_rank=None, recv_slot=None, stream=None) -> None:
    _check(_lib.sep_ep_mark_padding(owner_expert_counts.numel(), block_m, _ptr(owner_block_offset),
                                    _ptr(owner_expert_counts), int(pool_rows), _ptr(recv_token), _ptr(recv_rank),
                                    _ptr(recv_slot), _stream(stream)), "sep_ep_mark_padding")


def sep_ep_combine(handle: Handle, y_pools, pool_rows, delta: torch.Tensor, topk_weight: torch.Tensor,
                   out: torch.Tensor, error: torch.Tensor, layout_epoch: int | None = None, stream=None) -> None:
    """out[t] = bf16(sum_j w[t,j] * y_pools[owner][row(t,j)]) from the owners' expert outputs."""
    if out.dtype != torch.bfloat16 or topk_weight.dtype != torch.float32:
        raise ValueError("out must be bf16 and topk_weight fp32")
    R = len(y_pools)
    rows = (ctypes.c_int64 * R)(*[int(r) for r in pool_rows])
    epoch = handle.epoch if layout_epoch is None else layout_epoch
    _check(_lib.sep_ep_combine(handle.ptr, epoch, _ptr_array(y_pools), rows, out.shape[1], _ptr(delta),
                               _ptr(topk_weight), _ptr(out), _ptr(error), _stream(stream)), "sep_ep_combine")


IPC_HANDLE_BYTES = 64


class SharedBuffer:
    """A device buffer shared between the processes of a group (CUDA IPC): either
    allocated here (``opened`` False) or mapped from another process's handle."""

    def __init__(self, ptr: int, nbytes: int, handle: bytes, opened: bool):
        self.ptr, self.nbytes, self.handle, self.opened = ptr, nbytes, handle, opened

    def tensor(self, shape, dtype: torch.dtype) -> torch.Tensor:
        """A torch view of the buffer (no copy)."""
        typestr = {torch.bfloat16: "<V2", torch.int32: "<i4", torch.float32: "<f4", torch.uint8: "|u1"}[dtype]
        n = 1
        for d in shape:
            n *= d
        if n * torch.empty((), dtype=dtype).element_size() > self.nbytes:
            raise ValueError("view larger than the buffer")
        if dtype == torch.bfloat16:          # torch has no bf16 typestr: view int16 storage as bf16
            t = torch.as_tensor(_DeviceArray(self.ptr, shape, "<i2"), device="cuda")
            return t.view(torch.bfloat16)
        return torch.as_tensor(_DeviceArray(self.ptr, shape, typestr), device="cuda")

    def close(self) -> None:
        if self.ptr:
            _check(_lib.sep_ep_buffer_close(ctypes.c_void_p(self.ptr), 1 if self.opened else 0), "sep_ep_buffer_close")
            self.ptr = 0


def sep_ep_buffer_alloc(nbytes: int) -> SharedBuffer:
    ptr = ctypes.c_void_p()
    hd = ctypes.create_string_buffer(IPC_HANDLE_BYTES)
    _check(_lib.sep_ep_buffer_alloc(int(nbytes), ctypes.byref(ptr), hd), "sep_ep_buffer_alloc")
    return SharedBuffer(ptr.value, int(nbytes), hd.raw, False)


def sep_ep_buffer_open(handle: bytes, nbytes: int) -> SharedBuffer:
    if len(handle) != IPC_HANDLE_BYTES:
        raise ValueError("an IPC handle has 64 bytes")
    ptr = ctypes.c_void_p()
    _check(_lib.sep_ep_buffer_open(ctypes.create_string_buffer(handle, IPC_HANDLE_BYTES), ctypes.byref(ptr)),
           "sep_ep_buffer_open")
    return SharedBuffer(ptr.value, int(nbytes), handle, True)


def sep_combine_scatter(handle: Handle, y_pool: torch.Tensor, topk_weight: torch.Tensor, out: torch.Tensor,
                        layout_epoch: int | None = None, stream=None) -> None:
    """The combine by bf16 atomic scatter from the pool rows (not deterministic)."""
    if y_pool.dtype != torch.bfloat16 or out.dtype != torch.bfloat16 or topk_weight.dtype != torch.float32:
        raise ValueError("y_pool/out must be bf16 and topk_weight fp32")
    epoch = handle.epoch if layout_epoch is None else layout_epoch
    _check(_lib.sep_combine_scatter(handle.ptr, epoch, _ptr(y_pool), y_pool.shape[1], y_pool.shape[0],
                                    _ptr(topk_weight), _ptr(out), _stream(stream)), "sep_combine_scatter")


def sep_consume_tiles_stamp(handle: Handle, recv_x: torch.Tensor, tile_ready: torch.Tensor, dispatch_seq: int,
                            dst: torch.Tensor, status: torch.Tensor, y_done: torch.Tensor, done_seq: int,
                            num_ctas: int = 16, timeout_ns: int = 0, stream=None) -> None:
    row_bytes = recv_x.shape[1] * recv_x.element_size()
    if dst.shape[0] < recv_x.shape[0] or dst.shape[1] * dst.element_size() != row_bytes:
        raise ValueError("dst must have recv_x's row size and at least its rows")
    if status.numel() < 2 or status.element_size() != 4 or y_done.element_size() != 4:
        raise ValueError("status and y_done hold 32-bit words")
    _check(_lib.sep_consume_tiles_stamp(handle.ptr, _ptr(recv_x), row_bytes, recv_x.shape[0], _ptr(tile_ready),
                                        tile_ready.numel(), dispatch_seq, _ptr(dst), num_ctas, timeout_ns,
                                        _ptr(status), _ptr(y_done), y_done.numel(), done_seq, _stream(stream)),
           "sep_consume_tiles_stamp")


def sep_combine_gated(handle: Handle, y_pool: torch.Tensor, topk_weight: torch.Tensor, out: torch.Tensor,
                      y_done: torch.Tensor, done_seq: int, status: torch.Tensor, num_ctas: int = 64,
                      timeout_ns: int = 0, layout_epoch: int | None = None, stream=None) -> None:
    if y_pool.dtype != torch.bfloat16 or out.dtype != torch.bfloat16 or topk_weight.dtype != torch.float32:
        raise ValueError("y_pool/out must be bf16 and topk_weight fp32")
    if status.numel() < 2 or status.element_size() != 4 or y_done.element_size() != 4:
        raise ValueError("status and y_done hold 32-bit words")
    epoch = handle.epoch if layout_epoch is None else layout_epoch
    _check(_lib.sep_combine_gated(handle.ptr, epoch, _ptr(y_pool), y_pool.shape[1], y_pool.shape[0],
                                  _ptr(topk_weight), _ptr(out), _ptr(y_done), y_done.numel(), done_seq, num_ctas,
                                  timeout_ns, _ptr(status), _stream(stream)), "sep_combine_gated")


def sep_dispatch_grads(handle: Handle, grad_out: torch.Tensor, topk_weight: torch.Tensor, grad_y: torch.Tensor,
                       y_pool: torch.Tensor | None = None, grad_w: torch.Tensor | None = None,
                       layout_epoch: int | None = None, stream=None) -> None:
    """grad_y[row(t,j)] = bf16(w[t,j] * grad_out[t]); grad_w[t,j] = <grad_out[t], y_pool[row(t,j)]> if given."""
    if grad_out.dtype != torch.bfloat16 or grad_y.dtype != torch.bfloat16 or topk_weight.dtype != torch.float32:
        raise ValueError("grad_out/grad_y must be bf16 and topk_weight fp32")
    if grad_w is not None and (grad_w.dtype != torch.float32 or y_pool is None or y_pool.dtype != torch.bfloat16):
        raise ValueError("grad_w must be fp32 and needs a bf16 y_pool")
    epoch = handle.epoch if layout_epoch is None else layout_epoch
    _check(_lib.sep_dispatch_grads(handle.ptr, epoch, _ptr(grad_out), grad_out.shape[1], _ptr(topk_weight),
                                   _ptr(y_pool), 0 if y_pool is None else y_pool.shape[0], _ptr(grad_y),
                                   grad_y.shape[0], _ptr(grad_w), _stream(stream)), "sep_dispatch_grads")


def sep_combine_grads(handle: Handle, grad_recv: torch.Tensor, grad_x: torch.Tensor,
                      layout_epoch: int | None = None, stream=None) -> None:
    """grad_x[t] = bf16(sum over valid j of grad_recv[row(t,j)])."""
    if grad_recv.dtype != torch.bfloat16 or grad_x.dtype != torch.bfloat16:
        raise ValueError("grad_recv/grad_x must be bf16")
    epoch = handle.epoch if layout_epoch is None else layout_epoch
    _check(_lib.sep_combine_grads(handle.ptr, epoch, _ptr(grad_recv), grad_recv.shape[1], grad_recv.shape[0],
                                  _ptr(grad_x), _stream(stream)), "sep_combine_grads")


def sep_handle_free(handle: Handle) -> None:
    handle.close()


def alloc_pool(handle: Handle, hidden: int, payload: str = "bf16", scale: str = "none",
               rows: int | None = None):
    """Device buffers for a dispatch: recv_x [rows, H] and, for FP8, recv_scales [rows, H/128]."""
    info = handle.info()
    if rows is None:
        rows = info.num_pool_rows if info.num_pool_rows >= 0 else info.max_pool_rows
    rows = max(int(rows), 1)
    if payload == "bf16":
        return torch.empty(rows, hidden, dtype=torch.bfloat16, device="cuda"), None
    recv = torch.empty(rows, hidden, dtype=torch.uint8, device="cuda")
    sdt = torch.uint8 if scale == "ue8m0" else torch.float32
    return recv, torch.empty(rows, hidden // 128, dtype=sdt, device="cuda")


def sep_layout_noalloc(topk_idx: torch.Tensor, num_experts: int, num_owners: int, block_m: int,
                       arrays: dict, stream=None) -> None:
    """Layout into caller-owned device tensors without any allocation by the library.

    ``arrays`` maps the sep_layout_arrays field names to device tensors
    (int32, except ``sizes`` int64 [2] and ``status`` int32 [2]); the pool-row
    and tile capacities are taken from the tensors' lengths."""
    if topk_idx.dtype not in (torch.int32, torch.int64) or topk_idx.dim() != 2:
        raise ValueError("topk_idx must be a [T, k] int32 or int64 tensor")
    T, k = topk_idx.shape
    E, R = int(num_experts), int(num_owners)
    # the C ABI sees only pointers, so every array's type and length is checked
    # here: a short or mistyped array would be written past its end on the device
    least = {"expert_counts": E, "owner_counts": R, "expert_pool_block_offset": E + 1,
             "owner_pool_row_offset": R + 1, "src_pool_row": T * k, "sizes": 2, "status": 2}
    for name, _ in LayoutArrays._fields_[:11]:
        if name not in arrays or arrays[name] is None:
            raise ValueError(f"sep_layout_noalloc: arrays[{name!r}] is missing")
        a = arrays[name]
        want = torch.int64 if name == "sizes" else torch.int32
        if a.dtype != want:
            raise ValueError(f"sep_layout_noalloc: {name} must be {want} (got {a.dtype})")
        if name in least and a.numel() < least[name]:
            raise ValueError(f"sep_layout_noalloc: {name} must hold at least {least[name]} elements "
                             f"(got {a.numel()})")
    for name, _ in LayoutArrays._fields_[:11]:
        a = arrays[name]
        if not a.is_cuda or (T and topk_idx.is_cuda and a.device != topk_idx.device):
            raise ValueError(f"sep_layout_noalloc: {name} must be on the device of topk_idx")
    if T and (not topk_idx.is_cuda or topk_idx.device.index != torch.cuda.current_device()):
        raise ValueError("sep_layout_noalloc: topk_idx must be on the current CUDA device")
    la = LayoutArrays()
    for name, _ in LayoutArrays._fields_[:11]:
        setattr(la, name, _ptr(arrays[name]).value)
    la.max_pool_rows = min(arrays["pool_recv_token"].numel(), arrays["pool_recv_slot"].numel())
    la.max_tiles = min(arrays["tile_expert"].numel(), arrays["pool_arrival_target"].numel())
    _check(_lib.sep_layout_noalloc(_ptr(topk_idx) if T else ctypes.c_void_p(None), topk_idx.element_size(),
                                   T, k, num_experts, num_owners, block_m, ctypes.byref(la), _stream(stream)),
           "sep_layout_noalloc")


def sep_launch_count() -> int:
    """Kernels this process has launched through the library."""
    return int(_lib.sep_launch_count())


def sep_dispatch_borrow(handle: Handle, x: torch.Tensor) -> RecvView:
    """Borrowed receive: a view (x, row map) instead of a copied pool; leases the handle."""
    if x.dtype != torch.bfloat16 or x.dim() != 2:
        raise ValueError("x must be a [T, H] bf16 tensor")
    view = RecvView()
    _check(_lib.sep_dispatch_borrow(handle.ptr, _ptr(x), x.shape[1], SEP_PAYLOAD_BF16, ctypes.byref(view)),
           "sep_dispatch_borrow")
    view._keep = x                                   # the slab must outlive the view
    return view


def sep_view_release(handle: Handle, streams=()) -> None:
    arr = (_P * max(len(streams), 1))(*[_stream(st).value for st in streams])
    _check(_lib.sep_view_release(handle.ptr, arr, len(streams)), "sep_view_release")


def pool_view(handle: Handle, recv_x: torch.Tensor) -> RecvView:
    """A view of a copied pool (indexed = 0): the copy path's input to sep_gather_rows."""
    info = handle.info()
    if info.num_pool_rows < 0:
        raise ValueError("the layout must be synced to know the pool size")
    view = RecvView()
    view.slab = _ptr(recv_x).value
    view.row_indices = info.pool_recv_token
    view.num_rows = info.num_pool_rows
    view.row_bytes = recv_x.shape[1] * recv_x.element_size()
    view.indexed = 0
    view.epoch = info.epoch
    view._keep = recv_x
    return view


def sep_gather_rows(view: RecvView, dst: torch.Tensor, stream=None) -> None:
    if dst.shape[1] * dst.element_size() != view.row_bytes:
        raise ValueError("dst rows must have the view's row size")
    _check(_lib.sep_gather_rows(ctypes.byref(view), _ptr(dst), dst.shape[0], _stream(stream)), "sep_gather_rows")
