"""The bf16 dispatch's two store paths against the oracle.

By default the bf16 dispatch stages each 2 KB step of a token row in shared
memory and hands the k pool-row stores to the bulk-copy unit; every other GPU
test runs that path.  SEP_DISPATCH_STAGED=0 (read once per process) selects
the stores from registers instead; this file runs both in child processes on
bf16 cases with ragged rows and unsynced layouts (and FP8 cases, whose
stores are from registers either way), bit for bit: pool rows,
codes and scales, padding rows untouched, and the combine of the dispatched
pool (StreamEP README, "Streaming dispatch in one paragraph": each landed
(token, k) pair lands in its pool slot; padding is never written)."""
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))

CHILD = r'''
import sys
sys.path.insert(0, {root!r}); sys.path.insert(0, {here!r})
from dataclasses import replace
import combine_route_layout_02_b200 as sep
import workloads as W
from gpu_harness import run_bf16_path, run_fp8_path
cases = [("tiny", None, None, 0), ("train8k", 1500, None, 0), ("decode", 200, 264, sep.SEP_LAYOUT_SYNC_COUNTS),
         ("streaming", 700, 4104, 0)]
for name, T, H, flags in cases:
    w = W.WORKLOADS[name]
    w = W.scaled(w, T) if T else w
    w = replace(w, H=H) if H else w
    d = W.make_inputs(w)
    run_bf16_path(d["topk_idx"], d["x"], d["topk_weight"], w.E, w.R, w.B, flags=flags)
for name, T, H, scale, flags in [("decode", None, None, "ue8m0", 0), ("prefill_skew", 300, 1408, "f32", 0),
                                 ("decode", 77, 640, "f32_pow2", sep.SEP_LAYOUT_SYNC_COUNTS)]:
    w = W.WORKLOADS[name]
    w = W.scaled(w, T) if T else w
    w = replace(w, H=H) if H else w
    d = W.make_inputs(w)
    run_fp8_path(d["topk_idx"], d["x"], w.E, w.R, w.B, scale, flags=flags)
print("dispatch ok")
'''


@pytest.mark.parametrize("staged", ["0", "1"])
def test_both_store_paths_equal_the_oracle(staged):
    root = os.path.dirname(HERE)
    env = dict(os.environ, SEP_DISPATCH_STAGED=staged)
    out = subprocess.run([sys.executable, "-c", CHILD.format(root=root, here=HERE)], env=env,
                         capture_output=True, text=True, timeout=600)
    assert out.returncode == 0, out.stderr[-3000:]
    assert "dispatch ok" in out.stdout
