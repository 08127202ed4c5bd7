"""Single-GPU MoE expert-parallel dispatch + combine for B200 (sm_100a).

The C ABI lives in ``include/sep.h`` and ``libsep.so`` (built from ``csrc/``);
``sep`` is its ctypes binding.  There is no CPU implementation: importing the
binding fails if the CUDA library cannot be loaded.
"""
from .sep import (  # noqa: F401
    Handle, LayoutArrays, LayoutInfo, RecvView, SepError, pool_view, sep_dispatch_borrow, sep_gather_rows,
    sep_view_release, alloc_pool, declared_entry_points, library, library_path,
    sep_combine, sep_consume_tiles, sep_dispatch, sep_handle_create, sep_handle_free,
    sep_handle_sync, sep_handle_set_max_ctas, sep_launch_count, sep_layout, sep_layout_dispatch, sep_layout_noalloc,
    sep_combine_gated, sep_combine_grads, sep_combine_scatter,
    sep_ep_combine, sep_ep_dispatch, sep_ep_dispatch_fp8, sep_ep_mark_padding, sep_ep_plan,
    sep_ep_plan_device, sep_ep_dispatch_publish, sep_ep_consume_tiles,
    SharedBuffer, sep_ep_buffer_alloc, sep_ep_buffer_open, sep_consume_tiles_stamp, sep_dispatch_grads,
    SEP_OK, SEP_ERR_INVALID_ARG, SEP_ERR_CAPACITY, SEP_ERR_BAD_EXPERT_ID, SEP_ERR_HANDLE_MISMATCH,
    SEP_ERR_TIMEOUT, SEP_ERR_CUDA, SEP_LAYOUT_SYNC_COUNTS, SEP_LAYOUT_TOKEN_IN_OWNER, SEP_LAYOUT_ONE_LAUNCH,
)
