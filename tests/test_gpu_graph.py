"""The forward step replayed from a CUDA graph.

layout -> dispatch -> combine is captured once on a stream and replayed with
new routings, activations and weights copied into the captured input buffers
between replays.  Nothing on the device may depend on host state that a replay
does not refresh: the single-launch layout's grid barrier advances its counter
by a fixed window per launch instead of by the host's epoch, so replays (which
repeat the captured epoch) still synchronise; a one-chunk layout (tiny) is an
ordinary dependent launch.  Every replay's layout arrays and output are checked
against the oracle bit for bit.
"""
import numpy as np
import pytest
import torch

import combine_route_layout_02_b200 as sep
import oracle
import workloads as W
from gpu_harness import bf16_bits, check_layout

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,T", [("tiny", None), ("train8k", 2000), ("decode", None),
                                    ("decode", 150),   # 1200 assignments: 10 narrow chunks
                                    ("decode", 400)])  # 3200 assignments: 25 narrow chunks
def test_forward_step_replays_from_a_cuda_graph(name, T):
    w = W.WORKLOADS[name]
    w = W.scaled(w, T) if T else w
    from dataclasses import replace
    w = replace(w, payload="bf16", scale="none")
    d0 = W.make_inputs(w)
    idx = d0["topk_idx"].cuda()
    x = d0["x"].cuda()
    wt = d0["topk_weight"].cuda()
    h = sep.sep_handle_create(w.T, w.k, w.E, w.R, w.B)
    try:
        rows = h.info().max_pool_rows
        recv = torch.zeros(rows, w.H, dtype=torch.bfloat16, device="cuda")
        out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device="cuda")
        s = torch.cuda.Stream()
        s.wait_stream(torch.cuda.current_stream())
        with torch.cuda.stream(s):                     # one eager pass first
            sep.sep_layout(idx, w.E, w.R, w.B, handle=h)
            sep.sep_dispatch(h, x, recv)
            sep.sep_combine(h, recv, wt, out)
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=s):
            sep.sep_layout(idx, w.E, w.R, w.B, handle=h)
            sep.sep_dispatch(h, x, recv)
            sep.sep_combine(h, recv, wt, out)
        for rep in range(4):
            d = W.make_inputs(replace(w, seed=w.seed + 17 * (rep + 1)))
            idx.copy_(d["topk_idx"])
            x.copy_(d["x"])
            wt.copy_(d["topk_weight"])
            torch.cuda.synchronize()
            g.replay()
            torch.cuda.synchronize()
            lay = oracle.layout(d["topk_idx"].numpy(), w.E, w.R, w.B)
            check_layout(h, lay)
            want = oracle.combine(oracle.dispatch_bf16(d["x"], lay), d["topk_weight"].numpy(), lay)
            np.testing.assert_array_equal(bf16_bits(out), want)
        del g
    finally:
        sep.sep_handle_free(h)
