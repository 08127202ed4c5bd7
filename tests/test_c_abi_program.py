"""The C ABI from a plain C program (tests/c/abi_step.c), no Python between.

The program is compiled with the system C compiler against include/sep.h,
libsep.so and the CUDA runtime on CPU (the build check), and on the GPU it
runs one layout -> dispatch -> combine step on inputs this test writes; its
maps, pool rows and combined output must equal the oracle's bit for bit.
"""
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

import combine_route_layout_02_b200 as sep
import oracle
import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CUDA = os.environ.get("CUDA_HOME", "/usr/local/cuda")


def _compile(out_dir):
    lib_dir = os.path.dirname(sep.library_path())
    exe = os.path.join(out_dir, "abi_step")
    cc = shutil.which("gcc") or shutil.which("cc")
    subprocess.check_call([cc, "-O2", "-std=c11", "-Wall", "-Werror", "-o", exe,
                           os.path.join(ROOT, "tests", "c", "abi_step.c"),
                           "-I", os.path.join(ROOT, "include"), "-I", os.path.join(CUDA, "include"),
                           "-L", lib_dir, "-lsep", f"-Wl,-rpath,{lib_dir}",
                           "-L", os.path.join(CUDA, "lib64"), "-lcudart", f"-Wl,-rpath,{os.path.join(CUDA, 'lib64')}"])
    return exe


def test_c_program_compiles_against_the_header(tmp_path):
    assert os.access(_compile(str(tmp_path)), os.X_OK)


@pytest.mark.gpu
@pytest.mark.parametrize("name,T", [("tiny", None), ("train8k", 1500)])
def test_c_program_step_matches_the_oracle(name, T, tmp_path):
    w = W.WORKLOADS[name]
    w = W.scaled(w, T) if T else w
    d = W.make_inputs(w)
    d["topk_idx"].numpy().astype(np.int32).tofile(tmp_path / "topk_idx.bin")
    oracle.as_u16(d["x"]).tofile(tmp_path / "x.bin")
    d["topk_weight"].numpy().astype(np.float32).tofile(tmp_path / "topk_weight.bin")
    exe = _compile(str(tmp_path))
    subprocess.check_call([exe, str(tmp_path), str(w.T), str(w.k), str(w.E), str(w.R), str(w.B), str(w.H)],
                          timeout=120)
    lay = oracle.layout(d["topk_idx"].numpy(), w.E, w.R, w.B)
    P, NT = map(int, (tmp_path / "sizes.txt").read_text().split())
    assert (P, NT) == (lay.num_pool_rows, lay.num_tiles)
    spr = np.fromfile(tmp_path / "src_pool_row.bin", dtype=np.int32).reshape(w.T, w.k)
    np.testing.assert_array_equal(spr, lay.src_pool_row)
    want_pool = oracle.dispatch_bf16(d["x"], lay)
    recv = np.fromfile(tmp_path / "recv.bin", dtype=np.uint16).reshape(P, w.H)
    valid = lay.pool_recv_token >= 0
    np.testing.assert_array_equal(recv[valid], want_pool[valid])
    out = np.fromfile(tmp_path / "out.bin", dtype=np.uint16).reshape(w.T, w.H)
    np.testing.assert_array_equal(out, oracle.combine(want_pool, d["topk_weight"].numpy(), lay))
