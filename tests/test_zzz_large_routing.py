"""A routing too large for the single-launch layout.

Up to 2 097 152 assignments a routing has at most 128 CTA chunks, which always
fit on the GPU at once, so the layout is one cooperative launch.  Beyond that
the chunk count grows with the routing (one chunk per 16 384 assignments), and
once it exceeds what the GPU holds resident the layout runs as three launches
(count, scan, assign).  With 1024 experts (the most the ABI accepts, and the
largest per-CTA tables) and 16 777 216 assignments there are 1024 chunks, more
than one B200 holds resident; every layout array must still equal the
oracle's, bit for bit.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import combine_route_layout_02_b200 as sep
import oracle
from gpu_harness import check_layout

pytestmark = pytest.mark.gpu


def test_layout_of_a_routing_beyond_the_single_launch():
    T, k, E, R, B = 2_097_152, 8, 1024, 8, 128
    rng = np.random.default_rng(77)
    idx = rng.integers(-1, E, size=(T, k), dtype=np.int32)           # about 1 in 1025 masked
    lay = oracle.layout(idx, E, R, B)
    h = sep.sep_handle_create(T, k, E, R, B)
    try:
        before = sep.sep_launch_count()
        sep.sep_layout(torch.from_numpy(idx).cuda(), E, R, B, flags=sep.SEP_LAYOUT_SYNC_COUNTS, handle=h)
        launches = sep.sep_launch_count() - before
        check_layout(h, lay)
        assert launches == 3, f"expected the three-launch layout, saw {launches} launch(es)"
    finally:
        sep.sep_handle_free(h)
