"""Multi-rank host logic of the benchmark, on CPU with gloo (world size 2).

The path shards by tokens: every rank runs layout -> dispatch -> combine on
its own token shard with no data-path collective; the only cross-rank steps
are the timing barrier and the max-over-ranks reduction of step times.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle
import workloads as W


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        r, w_, local = bench.dist_env()
        assert (r, w_, local) == (rank, world, rank)
        wl = bench.shard_workload(W.WORKLOADS["tiny"], rank)
        d = W.make_inputs(wl)
        # each rank's shard is laid out independently; counts sum to its own T*k
        lay = oracle.layout(d["topk_idx"].numpy(), wl.E, wl.R, wl.B)
        assert lay.expert_counts.sum() == wl.T * wl.k
        bench.barrier(world)
        step_ms = [1.0 + rank, 5.0 - rank]
        mx = bench.reduce_max(step_ms, world)
        out[rank] = (wl.seed, float(d["x"].float().sum()), mx)
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_tokens_and_reduce_max():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    (s0, x0, m0), (s1, x1, m1) = res[0], res[1]
    assert s0 == W.WORKLOADS["tiny"].seed and s1 != s0      # distinct shards
    assert x0 != x1
    assert m0 == m1 == [2.0, 5.0]                            # max over ranks, same on every rank


def test_single_rank_reduce_is_identity():
    assert bench.reduce_max([3.0, 4.0], 1) == [3.0, 4.0]


def test_algorithmic_bytes_of_the_train8k_workload():
    ab = bench.algorithmic_bytes(W.WORKLOADS["train8k"])
    T, H, Na = 8192, 3072, 65536
    assert ab["dispatch"] == T * H * 2 + Na * H * 2 + 4 * Na
    assert ab["combine"] == Na * H * 2 + T * H * 2 + 8 * Na
    assert ab["total"] == 2 * (T * H * 2 + Na * H * 2) + 28 * Na   # 906.0 MB of rows + 1.8 MB of maps


def test_parse_defaults_finish_quickly():
    a = bench.parse_args([])
    assert a.gpus == 1 and a.warmup >= 3 and a.workload == "train8k" and a.impl == "ours"
