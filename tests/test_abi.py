"""The C-ABI library loads, exports every entry point include/sep.h declares, and
rejects invalid arguments on the host before touching CUDA (no GPU needed)."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

import combine_route_layout_02_b200 as sep
from combine_route_layout_02_b200 import build

HEADER = os.path.join(build.INCLUDE, "sep.h")


def test_library_is_built_for_sm100a_and_in_tree():
    path = sep.library_path()
    assert os.path.dirname(path) == os.path.dirname(os.path.abspath(sep.__file__))
    assert os.path.exists(path)
    assert "arch=compute_100a,code=sm_100a" in " ".join(build.ARCH)


def test_exports_match_header():
    declared = sep.declared_entry_points(HEADER)
    assert len(declared) == 34
    out = subprocess.run(["nm", "-D", "--defined-only", sep.library_path()], capture_output=True,
                         text=True, check=True).stdout
    exported = sorted(set(re.findall(r"\sT\s+(sep_\w+)$", out, flags=re.M)))
    assert exported == declared
    lib = sep.library()
    for name in declared:
        assert hasattr(lib, name)


def test_version_and_status_strings():
    lib = sep.library()
    assert lib.sep_abi_version() == 1
    names = [lib.sep_status_string(i).decode() for i in range(7)]
    assert names == ["SEP_OK", "SEP_ERR_INVALID_ARG", "SEP_ERR_CAPACITY", "SEP_ERR_BAD_EXPERT_ID",
                     "SEP_ERR_HANDLE_MISMATCH", "SEP_ERR_TIMEOUT", "SEP_ERR_CUDA"]


def _layout(lib, idx_bytes=4, T=4, k=2, E=8, R=2, B=16, flags=0, ptr=None, out=True):
    h = ctypes.c_void_p(None)
    return lib.sep_layout(ptr, idx_bytes, T, k, E, R, B, flags, None, ctypes.byref(h) if out else None)


@pytest.mark.parametrize("kw", [
    dict(idx_bytes=2), dict(k=0), dict(k=33), dict(E=0), dict(E=1025), dict(R=3), dict(R=0),
    dict(B=0), dict(B=1025), dict(T=-1), dict(flags=0x8), dict(T=1 << 29, k=8), dict(out=False),
])
def test_layout_rejects_invalid_arguments(kw):
    lib = sep.library()
    assert _layout(lib, **kw) == sep.SEP_ERR_INVALID_ARG
    assert lib.sep_last_error().decode() != ""


def test_layout_rejects_null_indices_for_nonempty_routing():
    lib = sep.library()
    assert _layout(lib, T=4, ptr=None) == sep.SEP_ERR_INVALID_ARG
    assert "topk_idx" in lib.sep_last_error().decode()


def test_calls_on_null_handle_are_rejected():
    lib = sep.library()
    assert lib.sep_dispatch(None, None, 8, 0, 0, None, None, 0, None, 0, 0, None) == sep.SEP_ERR_INVALID_ARG
    assert lib.sep_combine(None, 0, None, 8, 0, None, None, None) == sep.SEP_ERR_INVALID_ARG
    assert lib.sep_consume_tiles(None, None, 16, 0, None, 0, 1, None, 1, 0, None, None) == sep.SEP_ERR_INVALID_ARG
    assert lib.sep_consume_tiles_stamp(None, None, 16, 0, None, 0, 1, None, 1, 0, None, None, 0, 1,
                                       None) == sep.SEP_ERR_INVALID_ARG
    assert lib.sep_combine_gated(None, 0, None, 8, 0, None, None, None, 0, 1, 1, 0, None,
                                 None) == sep.SEP_ERR_INVALID_ARG
    assert lib.sep_dispatch_grads(None, 0, None, 8, None, None, 0, None, 0, None, None) == sep.SEP_ERR_INVALID_ARG
    assert lib.sep_combine_grads(None, 0, None, 8, 0, None, None) == sep.SEP_ERR_INVALID_ARG
    assert lib.sep_combine_scatter(None, 0, None, 8, 0, None, None, None) == sep.SEP_ERR_INVALID_ARG
    assert lib.sep_handle_sync(None, None) == sep.SEP_ERR_INVALID_ARG
    assert lib.sep_handle_info(None, None) == sep.SEP_ERR_INVALID_ARG
    lib.sep_handle_free(None)            # no-op


def test_handle_create_rejects_invalid_arguments():
    lib = sep.library()
    h = ctypes.c_void_p(None)
    assert lib.sep_handle_create(10, 0, 8, 2, 16, 0, None, ctypes.byref(h)) == sep.SEP_ERR_INVALID_ARG
    assert lib.sep_handle_create(10, 2, 8, 2, 16, 0, None, None) == sep.SEP_ERR_INVALID_ARG
    assert not h.value


def test_no_cpu_fallback_in_the_binding():
    # the binding has no host implementation of any step: its source never
    # imports the oracle or reaches for torch compute on the data path
    src = open(os.path.join(os.path.dirname(sep.__file__), "sep.py")).read()
    assert "oracle" not in src
    for op in ("index_select", ".scatter(", ".scatter_(", "scatter_add", "torch.sum", ".sum(", "torch.matmul",
               "torch.gather", ".gather("):
        assert op not in src


def test_launch_counter_starts_without_gpu_work():
    assert sep.sep_launch_count() >= 0


def test_expert_parallel_calls_reject_bad_arguments_before_any_cuda_call():
    lib = sep.library()
    assert lib.sep_ep_dispatch(None, 0, None, 8, 0, None, None, None, None, None, None, None, None) == \
        sep.SEP_ERR_INVALID_ARG
    assert lib.sep_ep_dispatch_fp8(None, 0, None, 128, 0, 2, None, None, None, None, None, None, None, None,
                                   None) == sep.SEP_ERR_INVALID_ARG
    assert lib.sep_ep_combine(None, 0, None, None, 8, None, None, None, None, None) == sep.SEP_ERR_INVALID_ARG
    assert lib.sep_ep_mark_padding(0, 16, None, None, 0, None, None, None, None) == sep.SEP_ERR_INVALID_ARG
    assert lib.sep_ep_mark_padding(4, 0, None, None, 0, None, None, None, None) == sep.SEP_ERR_INVALID_ARG
    assert lib.sep_ep_mark_padding(4, 16, None, None, 64, None, None, None, None) == sep.SEP_ERR_INVALID_ARG
    ptr = ctypes.c_void_p()
    assert lib.sep_ep_buffer_alloc(0, ctypes.byref(ptr), ctypes.create_string_buffer(64)) == sep.SEP_ERR_INVALID_ARG
    assert lib.sep_ep_buffer_alloc(64, None, None) == sep.SEP_ERR_INVALID_ARG
    assert lib.sep_ep_buffer_open(None, ctypes.byref(ptr)) == sep.SEP_ERR_INVALID_ARG
    assert lib.sep_ep_buffer_close(None, 1) == sep.SEP_OK


def test_host_tensors_are_refused_not_computed():
    """The binding has no CPU path: host tensors are refused with an error
    before the library is called, never laid out, dispatched or combined."""
    h = sep.Handle(ctypes.c_void_p(None))
    idx = torch.zeros(4, 2, dtype=torch.int32)
    x = torch.zeros(4, 16, dtype=torch.bfloat16)
    pool = torch.zeros(64, 16, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="device tensors"):
        sep.sep_layout(idx, 8, 2, 16)
    with pytest.raises(ValueError, match="device tensors"):
        sep.sep_dispatch(h, x, pool)
    with pytest.raises(ValueError, match="device tensors"):
        sep.sep_combine(h, pool, torch.zeros(4, 2), torch.zeros(4, 16, dtype=torch.bfloat16), layout_epoch=1)


def test_layout_dispatch_rejects_bad_arguments_before_any_cuda_call():
    """Every check of sep_layout_dispatch comes before the handle is created or
    changed: the capacity against the worst case for num_tokens (4 tokens x 2
    over 8 experts with BLOCK_M 16 need 8 + 8 * 15 = 128 rows), the payload,
    the hidden size and the alignment."""
    lib = sep.library()
    h = ctypes.c_void_p(None)

    def call(cap, payload=0, scale=0, hidden=16, x=16, recv=16, k=2):
        return lib.sep_layout_dispatch(ctypes.c_void_p(16), 4, 4, k, 8, 2, 16, 0, ctypes.c_void_p(x), hidden,
                                       payload, scale, ctypes.c_void_p(recv), None, cap, None, ctypes.byref(h))

    assert call(127) == sep.SEP_ERR_CAPACITY
    assert "128" in lib.sep_last_error().decode()
    assert call(1 << 20, payload=5) == sep.SEP_ERR_INVALID_ARG
    assert call(1 << 20, payload=1, scale=0) == sep.SEP_ERR_INVALID_ARG
    assert call(1 << 20, hidden=12) == sep.SEP_ERR_INVALID_ARG
    assert call(1 << 20, x=8) == sep.SEP_ERR_INVALID_ARG
    assert call(1 << 20, k=0) == sep.SEP_ERR_INVALID_ARG
    assert not h.value


def test_cta_budget_rejects_bad_arguments_before_any_cuda_call():
    lib = sep.library()
    assert lib.sep_handle_set_max_ctas(None, 4) == sep.SEP_ERR_INVALID_ARG
