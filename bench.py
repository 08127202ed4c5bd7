#!/usr/bin/env python
"""MoE dispatch + combine on B200: tokens/s and achieved HBM GB/s.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload train8k]
    python bench.py --impl reference ...      # the CPU oracle, timed on host cores

One step is the whole hot path over one batch: layout (count, scan, assign)
-> dispatch (permute into the expert-major pool; FP8 quantisation for the FP8
workloads; tile_ready publication plus a consumer on a second stream for the
streaming workload) -> combine (weighted top-k reduction back to token order),
with identity experts (combine reads the dispatched pool; FP8 workloads read a
seeded bf16 pool).  Inputs are resident in HBM before timing; the L2 is flushed
(a 2 x L2 write, then read back so no dirty line of the flush is written back
inside the step) before every timed step, outside the events.

After the timed steps, on the same data: the phase split (its own loop, with
events between the kernels), a loop without the L2 flush, the step replayed
from a CUDA graph, the end-to-end pipeline through the C ABI with host copies,
the CPU oracle (one core and every core), and the measurements chosen with
--extras (borrowed receive, backward pair, combine gate, scatter combine,
expert parallelism emulated on one GPU).

Multi-GPU (torchrun): every rank runs the same workload on its own token shard
(its own seed), with no collective on the data path (weak scaling); the step
time is the maximum over ranks.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import re
import json
import os
import statistics
import sys
import threading
import time
from dataclasses import replace

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

METRIC = "dispatch+combine tokens/s and achieved HBM GB/s (% of B200 peak), 1 GPU"
FALLBACK_HBM_GBS = 6650.0


# ------------------------------------------------------------------ helpers

def parse_args(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--workload", default="train8k", choices=sorted(W.WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-flush", action="store_true", help="skip the L2 flush (reported in config)")
    ap.add_argument("--e2e-steps", type=int, default=100)
    ap.add_argument("--cpu-budget", type=float, default=10.0, help="seconds of oracle work for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--consumer-ctas", type=int, default=64)
    ap.add_argument("--gate-ctas", type=int, default=0,
                    help="CTAs of the gated combine in the combine_gate measurement (0: one per SM)")
    ap.add_argument("--no-graph", action="store_true",
                    help="skip timing the step replayed from a CUDA graph (non-streaming workloads)")
    ap.add_argument("--extras", default="borrowed,backward,gate,scatter,ep,budget,overlap",
                    help="comma list of the measurements taken after the timed region")
    ap.add_argument("--profile-case", default=None,
                    choices=["layout", "layout_dispatch", "one_launch", "dispatch", "combine", "consumer", "gated",
                             "gather", "scatter", "backward", "ep", "ep_plain"],
                    help="run one kernel family a few times, its producers finished first (for ncu); no timing")
    ap.add_argument("--max-ctas", type=int, default=0,
                    help="with --profile-case: the handle's CTA budget (sep_handle_set_max_ctas; 0 = default grid)")
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the borrowed-receive, backward-pair, combine-gate and scatter-combine measurements")
    return ap.parse_args(argv)


def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return rank, world, local


def shard_workload(w: W.Workload, rank: int) -> W.Workload:
    """Each rank's token shard: same shapes, its own seed (rank 0 keeps the workload's seed)."""
    return replace(w, seed=w.seed + 100_000 * rank)


def algorithmic_bytes(w: W.Workload) -> dict:
    """Bytes the path must move at minimum; padding rows are never counted.

    dispatch: read x once (T*H*2) + write N_a payload rows (N_a*H*b_p) + scales
              (N_a*H/128*b_s) + read src_pool_row (4*N_a)
    combine:  read N_a rows of y (N_a*H*2) + write out (T*H*2) + read
              src_pool_row and topk_weight (8*N_a)
    layout:   read topk_idx (4*N_a) + write src_pool_row, pool_recv_token,
              pool_recv_slot (12*N_a)
    """
    Na, T, H = w.n_assign, w.T, w.H
    bp = 2 if w.payload == "bf16" else 1
    bs = {"none": 0, "f32": 4, "f32_pow2": 4, "ue8m0": 1}[w.scale]
    groups = H // 128 if w.payload == "fp8" else 0
    layout = 16 * Na
    dispatch = T * H * 2 + Na * H * bp + Na * groups * bs + 4 * Na
    combine = Na * H * 2 + T * H * 2 + 8 * Na
    consumer = 2 * Na * H * bp if w.streaming else 0
    return {"layout": layout, "dispatch": dispatch, "combine": combine,
            "total": layout + dispatch + combine, "consumer": consumer}


def load_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "source": "measured"}
    except Exception:
        return {"hbm_gbs": FALLBACK_HBM_GBS, "source": "fallback"}


KERNEL_PARAMS = {"layout": "LayoutParams", "dispatch": "DispatchParams", "combine": "CombineParams"}


def kernel_source_hash(kernel: str) -> str:
    """Hash of what decides a kernel's memory traffic: its source file (kernels
    and launch shape), its parameter struct and the shared row-split helper."""
    csrc = os.path.join(ROOT, "combine_route_layout_02_b200", "csrc")
    with open(os.path.join(csrc, "sep_internal.cuh")) as f:
        header = f.read()
    parts = [open(os.path.join(csrc, f"{kernel}.cu")).read()]
    for pattern in (r"struct %s \{.*?\n\};" % KERNEL_PARAMS[kernel], r"inline void split_rows\(.*?\n\}"):
        m = re.search(pattern, header, flags=re.S)
        parts.append(m.group(0) if m else "")
    return hashlib.sha256("\x00".join(parts).encode()).hexdigest()[:16]


def profiled_traffic(workload: str, kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(path) as f:
            table = json.load(f)
    except Exception:
        return None
    ent = table.get(workload, {}).get(kernel)
    if not ent or ent.get("source_hash") != kernel_source_hash(kernel):
        return None
    return ent.get("bytes_per_launch")


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = [("hw_slowdown", "nvmlClocksEventReasonHwSlowdown"),
               ("hw_thermal_slowdown", "nvmlClocksEventReasonHwThermalSlowdown"),
               ("sw_thermal_slowdown", "nvmlClocksEventReasonSwThermalSlowdown"),
               ("sw_power_cap", "nvmlClocksEventReasonSwPowerCap"),
               ("hw_power_brake", "nvmlClocksEventReasonHwPowerBrakeSlowdown")]

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self._stop = threading.Event()
        self._period = period_s
        self._ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            visible = os.environ.get("CUDA_VISIBLE_DEVICES")
            phys = device_index
            if visible:
                ids = [v for v in visible.split(",") if v.strip()]
                if device_index < len(ids) and ids[device_index].strip().isdigit():
                    phys = int(ids[device_index])
            self._nv = pynvml
            self._h = pynvml.nvmlDeviceGetHandleByIndex(phys)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            self._ok = False
        self._t = threading.Thread(target=self._run, daemon=True)

    def _run(self):
        nv = self._nv
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._h, nv.NVML_CLOCK_SM))
                bits = nv.nvmlDeviceGetCurrentClocksEventReasons(self._h)
                for name, const in self.REASONS:
                    if bits & getattr(nv, const, 0):
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self._period)

    def __enter__(self):
        if self._ok:
            self._t.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._ok:
            self._t.join()

    def summary(self) -> dict:
        if not self._ok or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": sorted(self.reasons),
                    "samples": len(self.samples), "source": "nvml unavailable" if not self._ok else "nvml"}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples), "source": "nvml"}


def reduce_max(values, world: int, device=None):
    """Element-wise max over ranks (timing only; not a data-path collective)."""
    if world <= 1:
        return list(values)
    import torch
    import torch.distributed as dist
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ------------------------------------------------------------ cpu oracle

def oracle_step(w: W.Workload, d: dict, y_pool=None):
    """One step of the plain oracle: layout -> dispatch -> combine."""
    import oracle
    lay = oracle.layout(d["topk_idx"].numpy(), w.E, w.R, w.B)
    if w.payload == "bf16":
        recv = oracle.dispatch_bf16(d["x"], lay)
        y = recv
    else:
        oracle.dispatch_fp8(d["x"], lay, w.scale)
        y = y_pool
    return oracle.combine(y, d["topk_weight"].numpy(), lay)


def oracle_y_pool(w: W.Workload, rows: int):
    import numpy as np
    import oracle
    table = oracle.as_u16(W.random_x(61, w.H, seed=w.seed + 7))
    return np.take(table, np.arange(max(rows, 1)) % 61, axis=0)


def sample_inputs(w: W.Workload, d: dict, T: int):
    ws = replace(w, T=T)
    return ws, {"x": d["x"][:T].contiguous(), "topk_idx": d["topk_idx"][:T].contiguous(),
                "topk_weight": d["topk_weight"][:T].contiguous()}


def _oracle_worker(job):
    """One host process: the unchanged oracle on its own token batch (a spawned
    process, so no CUDA state is inherited)."""
    name, T, seed, budget_s = job
    import oracle
    w = replace(W.WORKLOADS[name], T=T, seed=seed)
    d = W.make_inputs(w)
    y = oracle_y_pool(w, oracle.capacity_rows(w.n_assign, w.E, w.B)) if w.payload != "bf16" else None
    oracle_step(w, d, y)                                 # warm-up
    n, t0 = 0, time.perf_counter()
    while True:
        oracle_step(w, d, y)
        n += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            return n * T, el


def cpu_parallel(w: W.Workload, budget_s: float) -> dict:
    """The same oracle on every host core at once: one spawned process per core,
    each stepping its own batch of T/8 tokens (independent batches, as the
    ranks of the multi-GPU run); throughput summed over the processes."""
    import multiprocessing as mp
    from concurrent.futures import ProcessPoolExecutor
    cores = min(os.cpu_count() or 1, 64)
    T = max(1, w.T // 8)
    jobs = [(w.name, T, w.seed + 31 * (i + 1), budget_s) for i in range(cores)]
    # a worker that dies breaks the pool with an error instead of hanging it
    with ProcessPoolExecutor(cores, mp_context=mp.get_context("spawn")) as pool:
        res = list(pool.map(_oracle_worker, jobs, timeout=budget_s + 300))
    value = sum(tok / el for tok, el in res)
    return {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": f"{cores} processes, each {T}-token {w.name} batches (own seeds) for about "
                      f"{budget_s:.0f} s, single-threaded C oracle in each"}


def cpu_baseline(w: W.Workload, d: dict, budget_s: float) -> dict:
    """The oracle as it stands (single-threaded C), timed on a bounded sample:
    one core on full steps, and every core on independent batches; the line
    reports the faster, with both."""
    import oracle
    y = None
    if w.payload != "bf16":
        y = oracle_y_pool(w, oracle.capacity_rows(w.n_assign, w.E, w.B))
    t0 = time.perf_counter()
    oracle_step(w, d, y)
    first = time.perf_counter() - t0
    reps, total = 1, first
    while total + first <= budget_s:
        t0 = time.perf_counter()
        oracle_step(w, d, y)
        total += time.perf_counter() - t0
        reps += 1
    per = total / reps
    single = {"value": w.T / per, "unit": "tokens/s", "cores": 1, "kind": "oracle",
              "sample": f"full {w.name} step (T={w.T}) x {reps}, single-threaded C oracle, "
                        f"{per * 1e3:.1f} ms per step",
              "ms_per_step": per * 1e3}
    try:
        par = cpu_parallel(w, budget_s)
    except Exception as exc:                             # a host without spawn support: report one core
        par = {"error": str(exc)[:200]}
    best = par if par.get("value", 0) > single["value"] else single
    return {**{k: best[k] for k in ("value", "unit", "cores", "kind", "sample")},
            "single_core": single, "all_cores": par}


# ------------------------------------------------------------- our arm

def run_ours(args, rank: int, world: int, local: int) -> dict | None:
    import torch
    import combine_route_layout_02_b200 as sep

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = W.WORKLOADS[args.workload]
    wr = shard_workload(w, rank)
    d = W.make_inputs(wr)
    x = d["x"].to(dev)
    idx = d["topk_idx"].to(dev)
    wt = d["topk_weight"].to(dev)
    T, H = w.T, w.H

    h = sep.sep_handle_create(T, w.k, w.E, w.R, w.B)
    info = h.info()
    rows = info.max_pool_rows
    recv, scales = sep.alloc_pool(h, H, w.payload, w.scale, rows=rows)
    if w.payload == "bf16":
        y = recv
    else:
        import numpy as np
        table = W.random_x(61, H, seed=w.seed + 7).to(dev)
        y = table[torch.arange(rows, device=dev) % 61].contiguous()
    out = torch.empty(T, H, dtype=torch.bfloat16, device=dev)
    main = torch.cuda.current_stream()
    side = torch.cuda.Stream() if w.streaming else None
    tile_ready = torch.zeros(info.max_tiles, dtype=torch.int32, device=dev) if w.streaming else None
    dst = torch.empty_like(recv) if w.streaming else None
    status = torch.zeros(2, dtype=torch.int32, device=dev) if w.streaming else None
    seq = [0]
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_buf = None if args.no_flush else torch.empty(2 * l2 // 4, dtype=torch.int32, device=dev)

    class _Flush:
        """Write a 2 x L2 buffer, then read it back: afterwards the L2 holds
        only clean lines of that buffer, so no dirty line left by the flush is
        written back inside the next timed step."""

        def zero_(self):
            flush_buf.zero_()
            flush_buf.sum()

    flush = None if flush_buf is None else _Flush()
    n_sms = torch.cuda.get_device_properties(dev).multi_processor_count

    def step(ev=None, xs=x, idxs=idx, wts=wt, phases=False):
        # ev[0] / ev[3] bracket the step; ev[1] / ev[2] split it into phases only
        # when asked, since an event between two kernels keeps the second from
        # starting while the first drains (programmatic dependent launch)
        if ev is not None:
            ev[0].record(main)
        if not w.streaming and not phases:
            # layout and dispatch in one call (one launch when the routing is small)
            sep.sep_layout_dispatch(idxs, xs, recv, w.E, w.R, w.B, payload=w.payload, scale=w.scale,
                                    recv_scales=scales, handle=h)
            sep.sep_combine(h, y, wts, out)
            if ev is not None:
                ev[3].record(main)
            return
        sep.sep_layout(idxs, w.E, w.R, w.B, handle=h)
        epoch = h.epoch
        if ev is not None and phases:
            ev[1].record(main)
        if w.streaming:
            seq[0] += 1
            side.wait_stream(main)
            sep.sep_consume_tiles(h, recv, tile_ready, seq[0], dst, status, num_ctas=args.consumer_ctas,
                                  stream=side)
            sep.sep_dispatch(h, xs, recv, tile_ready=tile_ready, dispatch_seq=seq[0])
        else:
            sep.sep_dispatch(h, xs, recv, payload=w.payload, scale=w.scale, recv_scales=scales)
        if ev is not None and phases:
            ev[2].record(main)
        sep.sep_combine(h, y, wts, out, layout_epoch=epoch)
        if ev is not None:
            ev[3].record(main)
        if w.streaming:
            main.wait_stream(side)
            if ev is not None:
                ev[4].record(main)

    for _ in range(args.warmup):
        if flush is not None:
            flush.zero_()
        step()
    torch.cuda.synchronize()
    if w.streaming:
        assert status.cpu().tolist() == [0, 0], f"consumer status {status.cpu().tolist()}"

    nev = 5 if w.streaming else 4
    events = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(args.steps)]
    n_phase = min(args.steps, 200)
    phase_events = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(n_phase)]
    barrier(world)
    torch.cuda.synchronize()
    # the clock record spans the timed steps and the phase and warm loops after
    # them (the same kernels back to back), so it holds more than the one or two
    # samples a short timed region leaves
    sampler = ClockSampler(local)
    sampler.__enter__()
    launches_before = sep.sep_launch_count()
    for i in range(args.steps):
        if flush is not None:
            flush.zero_()
        step(events[i])
    torch.cuda.synchronize()
    launches = sep.sep_launch_count() - launches_before
    barrier(world)
    if w.streaming:
        assert status.cpu().tolist() == [0, 0], f"consumer status {status.cpu().tolist()}"

    # phase split, in a separate loop (its events cost the step its kernel overlap)
    for i in range(n_phase):
        if flush is not None:
            flush.zero_()
        step(phase_events[i], phases=True)
    torch.cuda.synchronize()
    barrier(world)
    if w.streaming:
        assert status.cpu().tolist() == [0, 0], f"consumer status {status.cpu().tolist()}"

    # the same step with the L2 left warm between steps (reported beside the flushed
    # number); at least 500 steps, which also gives the clock record tens of samples
    n_warm = max(min(args.steps, 2000), 500)
    warm_events = [[torch.cuda.Event(enable_timing=True) for _ in range(nev)] for _ in range(n_warm)]
    for i in range(n_warm):
        step(warm_events[i])
    torch.cuda.synchronize()
    sampler.__exit__(None, None, None)
    barrier(world)
    if w.streaming:
        assert status.cpu().tolist() == [0, 0], f"consumer status {status.cpu().tolist()}"

    # streaming: the publishing dispatch alone, with no consumer beside it
    disp_alone_ms = None
    if w.streaming:
        ev_a = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n_phase)]
        for i in range(n_phase):
            if flush is not None:
                flush.zero_()
            sep.sep_layout(idx, w.E, w.R, w.B, handle=h)
            seq[0] += 1
            ev_a[i][0].record(main)
            sep.sep_dispatch(h, x, recv, tile_ready=tile_ready, dispatch_seq=seq[0])
            ev_a[i][1].record(main)
        torch.cuda.synchronize()
        (disp_alone_ms,) = reduce_max([statistics.fmean(a.elapsed_time(b) for a, b in ev_a)], world, dev)

    graph_ms = replay_step_graph(args, w, step, main, flush, world, dev) if (not args.no_graph and not w.streaming) else None

    lay_ms = [e[0].elapsed_time(e[1]) for e in phase_events]
    dis_ms = [e[1].elapsed_time(e[2]) for e in phase_events]
    com_ms = [e[2].elapsed_time(e[3]) for e in phase_events]
    phased_ms = [e[0].elapsed_time(e[3]) for e in phase_events]
    # the step is layout -> dispatch (with the consumer running beside it on the
    # side stream) -> combine on the main stream; for the streaming workload the
    # time until the consumer has also finished is reported separately
    tot_ms = [e[0].elapsed_time(e[3]) for e in events]
    all_ms = [e[0].elapsed_time(e[nev - 1]) for e in events]
    mean = statistics.fmean
    warm_ms = [e[0].elapsed_time(e[3]) for e in warm_events]
    srt = sorted(tot_ms)
    local_vals = [mean(tot_ms), mean(lay_ms), mean(dis_ms), mean(com_ms), mean(all_ms), mean(phased_ms),
                  statistics.median(tot_ms), srt[min(len(srt) - 1, int(0.9 * len(srt)))], mean(warm_ms)]
    (step_ms, layout_ms, dispatch_ms, combine_ms, with_consumer_ms, phased_step_ms, median_ms, p90_ms,
     warm_step_ms) = reduce_max(local_vals, world, dev)

    # end to end through the C ABI: every step uploads its inputs from pinned
    # host memory and downloads its combined output.  Two buffer sets and two
    # handles pipeline the steps over three streams (upload of step i+1 and
    # download of step i-1 overlap the kernels of step i), as a caller feeding a
    # stream of batches would run them.  The streaming workload's consumer needs
    # its own side stream, so that workload runs its end-to-end steps one by one.
    x_h, idx_h, wt_h = d["x"].pin_memory(), d["topk_idx"].pin_memory(), d["topk_weight"].pin_memory()
    h2d = x_h.numel() * 2 + idx_h.numel() * idx_h.element_size() + wt_h.numel() * 4
    d2h = T * H * 2
    if w.streaming:
        out_h = torch.empty(T, H, dtype=torch.bfloat16).pin_memory()
        x_d, idx_d, wt_d = torch.empty_like(x), torch.empty_like(idx), torch.empty_like(wt)

        def e2e_step():
            x_d.copy_(x_h, non_blocking=True)
            idx_d.copy_(idx_h, non_blocking=True)
            wt_d.copy_(wt_h, non_blocking=True)
            step(None, x_d, idx_d, wt_d)
            out_h.copy_(out, non_blocking=True)

        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize()
        e2e_ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.e2e_steps)]
        barrier(world)
        for i in range(args.e2e_steps):
            e2e_ev[i][0].record(main)
            e2e_step()
            e2e_ev[i][1].record(main)
        torch.cuda.synchronize()
        barrier(world)
        e2e_local = mean([a.elapsed_time(b) for a, b in e2e_ev])
        copies_local = 0.0                               # not measured one step at a time
        e2e_mode = "one step at a time (the consumer occupies a side stream)"
    else:
        nb = 2
        handles = [h] + [sep.sep_handle_create(T, w.k, w.E, w.R, w.B) for _ in range(nb - 1)]
        sets = []
        for b in range(nb):
            rb, sb = (recv, scales) if b == 0 else sep.alloc_pool(handles[b], H, w.payload, w.scale, rows=rows)
            sets.append(dict(x=torch.empty_like(x), idx=torch.empty_like(idx), wt=torch.empty_like(wt),
                             out=torch.empty_like(out), recv=rb, scales=sb,
                             y=(rb if w.payload == "bf16" else y),
                             out_h=torch.empty(T, H, dtype=torch.bfloat16).pin_memory()))
        s_in, s_cmp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event() for _ in range(nb)]
        ev_cmp = [torch.cuda.Event() for _ in range(nb)]
        ev_out = [torch.cuda.Event() for _ in range(nb)]

        def e2e_step(i, kernels=True):
            b = i % nb
            S, hb = sets[b], handles[b]
            s_in.wait_event(ev_cmp[b])                   # step i-nb has finished with these inputs
            with torch.cuda.stream(s_in):
                S["x"].copy_(x_h, non_blocking=True)
                S["idx"].copy_(idx_h, non_blocking=True)
                S["wt"].copy_(wt_h, non_blocking=True)
            ev_in[b].record(s_in)
            s_cmp.wait_event(ev_in[b])
            s_cmp.wait_event(ev_out[b])                  # step i-nb's output has been downloaded
            if kernels:
                sep.sep_layout_dispatch(S["idx"], S["x"], S["recv"], w.E, w.R, w.B, payload=w.payload,
                                        scale=w.scale, recv_scales=S["scales"], handle=hb, stream=s_cmp)
                sep.sep_combine(hb, S["y"], S["wt"], S["out"], stream=s_cmp)
            ev_cmp[b].record(s_cmp)
            s_out.wait_event(ev_cmp[b])
            with torch.cuda.stream(s_out):
                S["out_h"].copy_(S["out"], non_blocking=True)
            ev_out[b].record(s_out)

        for i in range(4):
            e2e_step(i)
        torch.cuda.synchronize()
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        barrier(world)
        t0.record(s_in)
        for i in range(args.e2e_steps):
            e2e_step(i)
        t1.record(s_out)
        torch.cuda.synchronize()
        barrier(world)
        e2e_local = t0.elapsed_time(t1) / args.e2e_steps
        # the same pipeline with the kernels left out: the host-link floor of a step
        for i in range(4):
            e2e_step(i, kernels=False)
        torch.cuda.synchronize()
        t0.record(s_in)
        for i in range(args.e2e_steps):
            e2e_step(i, kernels=False)
        t1.record(s_out)
        torch.cuda.synchronize()
        copies_local = t0.elapsed_time(t1) / args.e2e_steps
        for hb in handles[1:]:
            sep.sep_handle_free(hb)
        e2e_mode = "pipelined: two buffer sets, uploads / kernels / downloads on three streams"
    (e2e_ms, copies_ms) = reduce_max([e2e_local, copies_local], world, dev)
    peaks = load_peaks()
    extras = set() if args.no_extras else set(args.extras.split(","))

    def want(name):
        return name in extras

    borrowed = (borrow_compare(args, w, h, x, idx, recv, dev)
                if (w.payload == "bf16" and not w.streaming and want("borrowed")) else None)
    backward = (backward_compare(w, h, idx, wt, y, None if flush is None else flush.zero_, peaks["hbm_gbs"])
                if w.payload == "bf16" and want("backward") else None)
    gate = gate_compare(args, w, h, x, idx, wt, recv, dev) if w.payload == "bf16" and want("gate") else None
    scatter = (scatter_compare(w, h, idx, wt, y, None if flush is None else flush.zero_, peaks["hbm_gbs"])
               if want("scatter") else None)
    ep = (ep_compare(w, dev, None if flush is None else flush.zero_, peaks["hbm_gbs"])
          if not w.streaming and want("ep") and w.T % w.R == 0 and (w.payload == "bf16" or w.T // w.R >= 128)
          else None)
    budget = (budget_compare(w, h, x, idx, recv, scales, y, wt, None if flush is None else flush.zero_, peaks["hbm_gbs"])
              if not w.streaming and want("budget") else None)
    overlap = (overlap_compare(w, h, x, idx, recv, y, wt, None if flush is None else flush.zero_)
               if w.payload == "bf16" and not w.streaming and want("overlap") else None)
    sep.sep_handle_free(h)

    ab = algorithmic_bytes(w)
    kern = {"dispatch": (dispatch_ms, ab["dispatch"]), "combine": (combine_ms, ab["combine"])}
    dom = max(kern, key=lambda k: kern[k][0])
    dom_ms, dom_bytes = kern[dom]
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9
    step_gbs = ab["total"] / (step_ms * 1e-3) / 1e9
    traffic = profiled_traffic(w.name, dom)

    res = {
        "metric": METRIC,
        "value": world * T / (step_ms * 1e-3),
        "unit": "tokens/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": step_ms,
        "step_ms_stats": {"mean": step_ms, "median": median_ms, "p90": p90_ms,
                          "l2_not_flushed_mean": warm_step_ms, "l2_not_flushed_steps": n_warm},
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.payload == "bf16" else "fp8-e4m3 dispatch, bf16 combine",
        "data": "synthetic",
        "config": {"workload": w.name, "T": T, "H": H, "E": w.E, "owners": w.R, "top_k": w.k,
                   "block_m": w.B, "payload": w.payload, "scale": w.scale,
                   "experts": "identity (combine reads the dispatched pool)" if w.payload == "bf16"
                   else "identity-shaped (combine reads a seeded bf16 pool)",
                   "streaming": w.streaming, "parallelism": f"{world} independent token shards",
                   "l2": "not flushed" if args.no_flush else f"flushed before every timed step ({2 * l2 >> 20} MB write then read back, outside the events)",
                   "sm_count": n_sms, "timing": "CUDA events per step on the launching stream, mean of steps, max over ranks"},
        "achieved_gbs": step_gbs,
        "pct_of_peak": 100.0 * step_gbs / peaks["hbm_gbs"],
        "phases_us": {"layout": layout_ms * 1e3, "dispatch": dispatch_ms * 1e3, "combine": combine_ms * 1e3,
                      "step_with_phase_events": phased_step_ms * 1e3, "steps": n_phase,
                      "note": "a separate loop with an event between phases (which stops each kernel from "
                              "starting while the previous drains); ms_per_step has events only around the step"},
        "phase_gbs": {"layout": ab["layout"] / (layout_ms * 1e-3) / 1e9,
                      "dispatch": ab["dispatch"] / (dispatch_ms * 1e-3) / 1e9,
                      "combine": ab["combine"] / (combine_ms * 1e-3) / 1e9},
        "algorithmic_bytes": ab,
        **({"consumer": {"until_consumer_done_us": with_consumer_ms * 1e3, "ctas": args.consumer_ctas,
                         "dispatch_alone_us": disp_alone_ms * 1e3,
                         "copy_bytes": ab["consumer"],
                         "note": "the reference consumer copies every ready tile on a second stream; it runs "
                                 "beside dispatch and combine and is not part of ms_per_step"}}
           if w.streaming else {}),
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": achieved, "peak": peaks["hbm_gbs"],
                     "peak_source": peaks["source"], "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
                     "traffic": traffic,
                     # the whole step's algorithmic bytes over its time: lines a kernel leaves dirty in L2
                     # are written back during the next one, so the step's figure is the one that
                     # charges every byte to the time it took
                     "step_frac": step_gbs / peaks["hbm_gbs"]},
        "e2e": {"value": world * T / (e2e_ms * 1e-3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms, "mode": e2e_mode,
                "copies_only_ms_per_step": copies_ms or None,
                "l2": "not flushed: every step uploads its inputs and the step's working set cycles the L2"},
        "gpu_launches": launches,
        **({"graph_replay": {"ms_per_step": graph_ms, "value": world * T / (graph_ms * 1e-3),
                             "note": "the same step captured once in a CUDA graph and replayed (one host launch "
                                     "per step); L2 flushed between replays"}} if graph_ms else {}),
        **({"borrowed_receive": borrowed} if borrowed else {}),
        **({"backward": backward} if backward else {}),
        **({"combine_gate": gate} if gate else {}),
        **({"combine_scatter": scatter} if scatter else {}),
        **({"ep_emulated": ep} if ep else {}),
        **({"sm_budget": budget} if budget else {}),
        **({"gemm_overlap": overlap} if overlap else {}),
        "clocks": sampler.summary(),
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(wr, d, args.cpu_budget)
    return res if rank == 0 else None


def replay_step_graph(args, w, step, main, flush, world, dev):
    """The same step captured once in a CUDA graph and replayed: one launch per
    step from the host, so for small workloads the time is the kernels' own
    rather than the host's launch rate.  Events bracket each replay on the
    launching stream; the L2 is flushed between replays as in the eager loop."""
    import torch
    cap = torch.cuda.Stream()
    cap.wait_stream(main)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=cap):
        step()
    torch.cuda.synchronize()
    for _ in range(args.warmup):
        if flush is not None:
            flush.zero_()
        g.replay()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    for i in range(args.steps):
        if flush is not None:
            flush.zero_()
        ev[i][0].record(main)
        g.replay()
        ev[i][1].record(main)
    torch.cuda.synchronize()
    barrier(world)
    (ms,) = reduce_max([statistics.fmean(a.elapsed_time(b) for a, b in ev)], world, dev)
    del g
    return ms


def _time_arm(fn, steps, flush=None, warmup=5):
    """Mean device time of fn() in microseconds, CUDA events around each call."""
    import torch
    main = torch.cuda.current_stream()
    for _ in range(warmup):
        fn()
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
    torch.cuda.synchronize()
    for i in range(steps):
        if flush is not None:
            flush()
        ev[i][0].record(main)
        fn()
        ev[i][1].record(main)
    torch.cuda.synchronize()
    return statistics.fmean(a.elapsed_time(b) for a, b in ev) * 1e3


def backward_compare(w, h, idx, wt, y, flush, peak_gbs, steps=100):
    """The backward pair on the same layout: dispatch_grads (grad_y and grad_w)
    and combine_grads, each timed alone with the L2 flushed before every call.

    dispatch_grads bytes: read grad_out (T*H*2) and y (N_a*H*2), write grad_y
    (N_a*H*2), read weights and row map, write grad_w (12*N_a).
    combine_grads bytes: read N_a rows (N_a*H*2), write grad_x (T*H*2), read
    the row map (4*N_a)."""
    import torch
    import combine_route_layout_02_b200 as sep
    Na, T, H = w.n_assign, w.T, w.H
    sep.sep_layout(idx, w.E, w.R, w.B, handle=h)
    g = W.random_x(T, H, seed=w.seed + 11).to(y.device)
    grad_y = torch.empty_like(y)
    grad_w = torch.empty(T, w.k, dtype=torch.float32, device=y.device)
    grad_x = torch.empty(T, H, dtype=torch.bfloat16, device=y.device)
    n0 = sep.sep_launch_count()
    sep.sep_dispatch_grads(h, g, wt, grad_y, y_pool=y, grad_w=grad_w)
    sep.sep_combine_grads(h, grad_y, grad_x)
    assert sep.sep_launch_count() - n0 == 2
    dg_us = _time_arm(lambda: sep.sep_dispatch_grads(h, g, wt, grad_y, y_pool=y, grad_w=grad_w), steps, flush)
    cg_us = _time_arm(lambda: sep.sep_combine_grads(h, grad_y, grad_x), steps, flush)
    dg_bytes = T * H * 2 + 2 * Na * H * 2 + 12 * Na
    cg_bytes = Na * H * 2 + T * H * 2 + 4 * Na
    res = {}
    for name, us, b in (("dispatch_grads", dg_us, dg_bytes), ("combine_grads", cg_us, cg_bytes)):
        gbs = b / (us * 1e-6) / 1e9
        res[name] = {"us": us, "algorithmic_bytes": b, "achieved_gbs": gbs, "frac": gbs / peak_gbs}
    res["note"] = ("each kernel timed alone on the bench workload's layout, L2 flushed before every call; "
                   "dispatch_grads computes grad_w too; frac is of the measured copy bandwidth")
    return res


def scatter_compare(w, h, idx, wt, y, flush, peak_gbs, steps=100):
    """The gather combine against the atomic-scatter combine on the same layout
    and pool, each timed alone with the L2 flushed before every call.  The
    scatter's time includes zeroing out (it reduces into it)."""
    import torch
    import combine_route_layout_02_b200 as sep
    sep.sep_layout(idx, w.E, w.R, w.B, handle=h)
    out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device=y.device)
    gather_us = _time_arm(lambda: sep.sep_combine(h, y, wt, out), steps, flush)
    scatter_us = _time_arm(lambda: sep.sep_combine_scatter(h, y, wt, out), steps, flush)
    b = algorithmic_bytes(w)["combine"]
    return {"gather_us": gather_us, "scatter_us": scatter_us,
            "scatter_gbs": b / (scatter_us * 1e-6) / 1e9, "scatter_frac": b / (scatter_us * 1e-6) / 1e9 / peak_gbs,
            "delta_pct": 100.0 * (scatter_us - gather_us) / gather_us,
            "note": "same combine bytes for both (the scatter also writes out's zeros first); "
                    "L2 flushed before every call"}


def budget_compare(w, h, x, idx, recv, scales, y, wt, flush, peak_gbs, steps=50):
    """The dispatch and the combine alone (L2 flushed before every call) with a
    CTA budget: how much of the copy bandwidth a fraction of the SMs reaches
    (the DeepEP vibeleaderboard entry, "Why it's ranked here": peak bandwidth
    with up to 4x fewer SMs).  0 is the default grid (one CTA per 8 items)."""
    import torch
    import combine_route_layout_02_b200 as sep
    out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device=x.device)
    sep.sep_layout(idx, w.E, w.R, w.B, handle=h)
    ab = algorithmic_bytes(w)
    sms = torch.cuda.get_device_properties(x.device).multi_processor_count
    res = []
    for ctas in (sms // 8, sms // 4, sms // 2, sms, 2 * sms, 0):
        sep.sep_handle_set_max_ctas(h, ctas)
        d_us = _time_arm(lambda: sep.sep_dispatch(h, x, recv, payload=w.payload, scale=w.scale, recv_scales=scales),
                         steps, flush)
        c_us = _time_arm(lambda: sep.sep_combine(h, y, wt, out), steps, flush)
        res.append({"max_ctas": ctas, "dispatch_us": d_us, "combine_us": c_us,
                    "dispatch_frac": ab["dispatch"] / (d_us * 1e-6) / 1e9 / peak_gbs,
                    "combine_frac": ab["combine"] / (c_us * 1e-6) / 1e9 / peak_gbs})
    sep.sep_handle_set_max_ctas(h, 0)
    return {"sms": sms, "budgets": res,
            "note": "each kernel alone on the bench workload's layout, L2 flushed before every call; max_ctas 0 is "
                    "the default grid; 8-warp CTAs, so max_ctas = SMs means about one CTA per SM"}



def overlap_compare(w, h, x, idx, recv, y, wt, flush, steps=30):
    """What the CTA budget is for: the dispatch and combine on one stream beside
    a dense bf16 GEMM on another (cuBLAS through torch, [T, H] x [H, 4096],
    standing in for an expert GEMM of another micro-batch).  Per budget: the
    GEMM alone, dispatch + combine alone, the two one after the other, and the
    two concurrently (fork on the main stream, join back; L2 flushed before
    each)."""
    import torch
    import combine_route_layout_02_b200 as sep
    dev = x.device
    main = torch.cuda.current_stream()
    side = torch.cuda.Stream()
    g = torch.Generator(device="cpu").manual_seed(5)
    a = torch.randn(w.T, w.H, generator=g).to(dev, torch.bfloat16)
    b = torch.randn(w.H, 4096, generator=g).to(dev, torch.bfloat16)
    c = torch.empty(w.T, 4096, dtype=torch.bfloat16, device=dev)
    out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device=dev)
    sep.sep_layout(idx, w.E, w.R, w.B, handle=h)

    def gemm():
        torch.matmul(a, b, out=c)

    def comm():
        sep.sep_dispatch(h, x, recv)
        sep.sep_combine(h, y, wt, out)

    def serial():
        gemm()
        comm()

    def concurrent():
        side.wait_stream(main)
        with torch.cuda.stream(side):
            gemm()
        comm()
        main.wait_stream(side)

    sms = torch.cuda.get_device_properties(dev).multi_processor_count
    gemm_us = _time_arm(gemm, steps, flush)
    res = []
    for ctas in (0, sms // 4, sms // 2, 3 * sms // 4):
        sep.sep_handle_set_max_ctas(h, ctas)
        comm_us = _time_arm(comm, steps, flush)
        serial_us = _time_arm(serial, steps, flush)
        conc_us = _time_arm(concurrent, steps, flush)
        res.append({"max_ctas": ctas, "comm_us": comm_us, "serial_us": serial_us, "concurrent_us": conc_us,
                    "saved_pct": 100.0 * (serial_us - conc_us) / serial_us})
    sep.sep_handle_set_max_ctas(h, 0)
    return {"gemm_us": gemm_us, "gemm_tflops": 2.0 * w.T * w.H * 4096 / (gemm_us * 1e-6) / 1e12, "budgets": res,
            "note": "bf16 GEMM [T,H]x[H,4096] on a side stream beside the budgeted dispatch + combine; max_ctas 0 is "
                    "the default grid; L2 flushed before every call"}


def ep_compare(w, dev, flush, peak_gbs, steps=100):
    """Expert parallelism across the workload's R owners as ranks, emulated on
    one GPU: the workload's T tokens split into R rank shards of T/R (own
    seeds), each rank laid out alone, the counts planned, then every rank's
    dispatch into the owners' pools and every rank's combine from them (the
    kernels a multi-GPU group runs with peer pointers), timed two ways: the
    ranks one after another on one stream, and each rank on its own stream
    with a join (the group's barrier) between the dispatches and the combines.
    Against the single-GPU dispatch + combine of the same tokens concatenated
    (same rows, same bytes).  Layouts and the plan are outside the timed
    region in all three."""
    import numpy as np
    import torch
    import combine_route_layout_02_b200 as sep
    R, Tr = w.R, w.T // w.R
    fp8 = w.payload != "bf16"
    shards = [W.make_inputs(replace(w, T=Tr, seed=w.seed + 7919 * (r + 1))) for r in range(R)]
    hs = [sep.sep_layout(sd["topk_idx"].to(dev), w.E, R, w.B, flags=sep.SEP_LAYOUT_SYNC_COUNTS) for sd in shards]
    counts = np.stack([h.view("expert_counts").cpu().numpy() for h in hs]).astype(np.int32)
    plans = [sep.sep_ep_plan(counts, r, w.B) for r in range(R)]
    rows = [int(v) for v in plans[0]["owner_rows"]]
    y_src = W.random_x(61, w.H, seed=w.seed + 7).to(dev) if fp8 else None

    def y_rows(n):
        """An FP8 workload's expert outputs: a seeded bf16 pool of n rows."""
        return y_src[torch.arange(max(n, 1), device=dev) % 61].contiguous()

    pools = [torch.empty(max(n, 1), w.H, dtype=torch.uint8 if fp8 else torch.bfloat16, device=dev) for n in rows]
    sdt = torch.uint8 if w.scale == "ue8m0" else torch.float32
    scale_pools = [torch.empty(max(n, 1), w.H // 128, dtype=sdt, device=dev) for n in rows] if fp8 else None
    y_pools = [y_rows(n) for n in rows] if fp8 else pools
    deltas = [torch.from_numpy(p["delta"]).to(dev) for p in plans]
    xs = [sd["x"].to(dev) for sd in shards]
    ws = [sd["topk_weight"].to(dev) for sd in shards]
    outs = [torch.empty(Tr, w.H, dtype=torch.bfloat16, device=dev) for _ in range(R)]
    err = torch.zeros(1, dtype=torch.int32, device=dev)

    def ep_dispatch(r, stream=None):
        if fp8:
            sep.sep_ep_dispatch_fp8(hs[r], xs[r], r, deltas[r], pools, scale_pools, rows, err, scale=w.scale,
                                    stream=stream)
        else:
            sep.sep_ep_dispatch(hs[r], xs[r], r, deltas[r], pools, rows, err, stream=stream)

    def ep_combine(r, stream=None):
        sep.sep_ep_combine(hs[r], y_pools, rows, deltas[r], ws[r], outs[r], err, stream=stream)

    def ep_step():
        for r in range(R):
            ep_dispatch(r)
        for r in range(R):
            ep_combine(r)

    streams = [torch.cuda.Stream(device=dev) for _ in range(R)]

    def join(main):
        for st in streams:                               # the group's barrier: every rank's kernels done
            main.wait_stream(st)
        for st in streams:
            st.wait_stream(main)

    def ep_concurrent_step():
        main = torch.cuda.current_stream()
        for st in streams:
            st.wait_stream(main)
        for r in range(R):
            ep_dispatch(r, streams[r])
        join(main)
        for r in range(R):
            ep_combine(r, streams[r])
        for st in streams:
            main.wait_stream(st)

    def ep_concurrent_phase(combine):
        main = torch.cuda.current_stream()
        for st in streams:
            st.wait_stream(main)
        for r in range(R):
            if combine:
                ep_combine(r, streams[r])
            else:
                ep_dispatch(r, streams[r])
        for st in streams:
            main.wait_stream(st)

    idx_cat = torch.cat([sd["topk_idx"] for sd in shards]).to(dev)
    x_cat = torch.cat([sd["x"] for sd in shards]).to(dev)
    w_cat = torch.cat([sd["topk_weight"] for sd in shards]).to(dev)
    h1 = sep.sep_layout(idx_cat, w.E, R, w.B, flags=sep.SEP_LAYOUT_SYNC_COUNTS)
    P1 = h1.info().num_pool_rows
    pool1, scales1 = sep.alloc_pool(h1, w.H, w.payload, w.scale, rows=max(P1, 1))
    y1 = y_rows(P1) if fp8 else pool1
    out1 = torch.empty(R * Tr, w.H, dtype=torch.bfloat16, device=dev)

    def single_dispatch():
        sep.sep_dispatch(h1, x_cat, pool1, payload=w.payload, scale=w.scale, recv_scales=scales1)

    def single_combine():
        sep.sep_combine(h1, y1, w_cat, out1)

    def single_step():
        single_dispatch()
        single_combine()

    def graph_of(fn):
        """fn captured once (side streams fork from and join back to the capture stream)."""
        cap = torch.cuda.Stream(device=dev)
        cap.wait_stream(torch.cuda.current_stream())
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=cap):
            fn()
        torch.cuda.synchronize()
        return g

    ep_us = _time_arm(ep_step, steps, flush)
    ep_conc_us = _time_arm(ep_concurrent_step, steps, flush)
    single_us = _time_arm(single_step, steps, flush)
    phase_us = [_time_arm(lambda c=c: ep_concurrent_phase(c), steps, flush) for c in (False, True)]
    single_phase_us = [_time_arm(single_dispatch, steps, flush), _time_arm(single_combine, steps, flush)]
    graphs = [graph_of(f) for f in (ep_step, ep_concurrent_step, single_step)]
    ep_g_us, ep_conc_g_us, single_g_us = (_time_arm(g.replay, steps, flush) for g in graphs)
    assert int(err.item()) == 0, "a row fell outside its owner's pool"
    del graphs
    for h in hs + [h1]:
        sep.sep_handle_free(h)
    b = algorithmic_bytes(replace(w, T=R * Tr))
    moved = b["dispatch"] + b["combine"]
    return {"ranks": R, "tokens_per_rank": Tr, "ep_us": ep_us, "ep_concurrent_us": ep_conc_us,
            "single_gpu_us": single_us,
            "ep_gbs": moved / (ep_us * 1e-6) / 1e9, "ep_frac": moved / (ep_us * 1e-6) / 1e9 / peak_gbs,
            "ep_concurrent_frac": moved / (ep_conc_us * 1e-6) / 1e9 / peak_gbs,
            "phases_us": {"ep_concurrent_dispatch": phase_us[0], "ep_concurrent_combine": phase_us[1],
                          "single_gpu_dispatch": single_phase_us[0], "single_gpu_combine": single_phase_us[1]},
            "graph_replay": {"ep_us": ep_g_us, "ep_concurrent_us": ep_conc_g_us, "single_gpu_us": single_g_us,
                             "ep_concurrent_frac": moved / (ep_conc_g_us * 1e-6) / 1e9 / peak_gbs,
                             "note": "each arm captured once in a CUDA graph and replayed: the same kernels "
                                     "without the host's per-launch cost (16 library calls per EP step)"},
            "note": "R ranks emulated on one GPU (2R launches: every rank's dispatch, then every rank's combine, "
                    "into / from the owners' pools); ep_us runs them one after another on one stream, "
                    "ep_concurrent_us runs each rank on its own stream with a join between the dispatches and "
                    "the combines (the group's barrier); single_gpu is the same tokens' dispatch + combine; "
                    "layouts outside the timed region; L2 flushed before every step"}


_gate_seq = [1 << 20]


def gate_compare(args, w, h, x, idx, wt, recv, dev, steps=50):
    """The per-token combine gate in the streaming pipeline: a streaming
    dispatch, the reference consumer standing in for identity experts (it
    copies each ready tile into y and stamps the tile's tokens), then combine.
    serial: combine starts after the consumer has finished.  gated: the gated
    combine runs on a third stream beside the consumer and starts on each token
    as soon as it is stamped.  Times from the layout's end to the last kernel's
    end; the consumer and both combines are the same in the two arms."""
    import torch
    import combine_route_layout_02_b200 as sep
    main = torch.cuda.current_stream()
    side, third = torch.cuda.Stream(), torch.cuda.Stream()
    info = h.info()
    tile_ready = torch.zeros(info.max_tiles, dtype=torch.int32, device=dev)
    y = torch.empty_like(recv)
    out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device=dev)
    y_done = torch.zeros(w.T, dtype=torch.int32, device=dev)
    st_c = torch.zeros(2, dtype=torch.int32, device=dev)
    st_g = torch.zeros(2, dtype=torch.int32, device=dev)
    seq = _gate_seq                                      # advances across calls: tile_ready may reuse an address
    ctas = args.consumer_ctas
    gctas = args.gate_ctas or torch.cuda.get_device_properties(dev).multi_processor_count

    def serial():
        seq[0] += 1
        side.wait_stream(main)
        sep.sep_consume_tiles(h, recv, tile_ready, seq[0], y, st_c, num_ctas=ctas, stream=side)
        sep.sep_dispatch(h, x, recv, tile_ready=tile_ready, dispatch_seq=seq[0])
        main.wait_stream(side)
        sep.sep_combine(h, y, wt, out)

    def gated():
        seq[0] += 1
        side.wait_stream(main)
        third.wait_stream(main)
        sep.sep_consume_tiles_stamp(h, recv, tile_ready, seq[0], y, st_c, y_done, seq[0], num_ctas=ctas,
                                    stream=side)
        sep.sep_combine_gated(h, y, wt, out, y_done, seq[0], st_g, num_ctas=gctas, stream=third)
        sep.sep_dispatch(h, x, recv, tile_ready=tile_ready, dispatch_seq=seq[0])
        main.wait_stream(side)
        main.wait_stream(third)

    sep.sep_layout(idx, w.E, w.R, w.B, handle=h)
    res = {}
    for name, fn in (("serial", serial), ("gated", gated)):
        res[name + "_us"] = _time_arm(fn, steps)
        assert st_c.cpu().tolist() == [0, 0] and st_g.cpu().tolist() == [0, 0], (name, st_c, st_g)
    res["delta_pct"] = 100.0 * (res["gated_us"] - res["serial_us"]) / res["serial_us"]
    res["gate_ctas"] = gctas
    res["note"] = (f"dispatch + reference consumer ({ctas} CTAs, identity experts) + combine after one layout, "
                   "L2 not flushed; the consumer stands in for the expert compute")
    return res


def borrow_compare(args, w, h, x, idx, recv, dev, steps=200):
    """PR #769's comparison on one GPU: dispatch plus an indexed consumer, with
    the rows copied into the pool (sep_dispatch, then the consumer reads the
    pool) against the borrowed receive (no copy; the consumer gathers from x
    through the row map).  Both arms start after the same synced layout; the
    consumer copies every valid row to a destination buffer."""
    import torch
    import combine_route_layout_02_b200 as sep
    main = torch.cuda.current_stream()
    sep.sep_layout(idx, w.E, w.R, w.B, flags=sep.SEP_LAYOUT_SYNC_COUNTS, handle=h)
    P = h.info().num_pool_rows
    dst = torch.empty(P, w.H, dtype=torch.bfloat16, device=dev)

    def copy_arm():
        sep.sep_dispatch(h, x, recv)
        sep.sep_gather_rows(sep.pool_view(h, recv), dst)

    def borrow_arm():
        view = sep.sep_dispatch_borrow(h, x)
        sep.sep_gather_rows(view, dst)
        sep.sep_view_release(h, [main])

    out = {}
    for name, fn in (("copy", copy_arm), ("borrowed", borrow_arm)):
        for _ in range(5):
            fn()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(steps)]
        torch.cuda.synchronize()
        for i in range(steps):
            ev[i][0].record(main)
            fn()
            ev[i][1].record(main)
        torch.cuda.synchronize()
        out[name] = statistics.fmean(a.elapsed_time(b) for a, b in ev) * 1e3
    return {"copy_path_us": out["copy"], "borrowed_path_us": out["borrowed"],
            "delta_pct": 100.0 * (out["borrowed"] - out["copy"]) / out["copy"],
            "note": "dispatch + the same indexed consumer after a synced layout, L2 not flushed between "
                    "steps; the pages' figure for this comparison is -13.1% at 8192 tokens/rank on 8xH200"}


# ------------------------------------------------------- reference arm

def _reference_worker(job):
    """One host process of the reference arm: the unchanged oracle stepping its
    own token batch `warmup` times untimed, then `steps` times timed."""
    name, T, seed, warmup, steps = job
    import oracle
    w = replace(W.WORKLOADS[name], T=T, seed=seed)
    y = oracle_y_pool(w, oracle.capacity_rows(w.n_assign, w.E, w.B)) if w.payload != "bf16" else None
    d = W.make_inputs(w)
    for _ in range(warmup):
        oracle_step(w, d, y)
    times = []
    for _ in range(steps):
        t0 = time.perf_counter()
        oracle_step(w, d, y)
        times.append(time.perf_counter() - t0)
    return times


def run_reference(args, rank: int) -> dict | None:
    """The CPU oracle as it stands, on the host cores: one spawned process per
    core (up to 64), each stepping its own batch of at most T/8 tokens of the
    workload (fewer if warm-up + timed steps would pass about two minutes),
    independently; throughput is summed over the processes."""
    if rank != 0:
        return None
    import multiprocessing as mp
    from concurrent.futures import ProcessPoolExecutor
    import oracle
    w = W.WORKLOADS[args.workload]
    cores = min(os.cpu_count() or 1, 64)
    ws, ds = sample_inputs(w, W.make_inputs(w), min(w.T, 256))
    y = oracle_y_pool(ws, oracle.capacity_rows(ws.n_assign, ws.E, ws.B)) if w.payload != "bf16" else None
    t0 = time.perf_counter()
    oracle_step(ws, ds, y)                               # one core, in this process, to size the sample
    per_tok = (time.perf_counter() - t0) / ws.T
    budget = 120.0 / max(1, args.steps + args.warmup)
    Ts = int(max(16, min(max(w.T // 8, 16), budget / max(per_tok, 1e-9))))
    jobs = [(w.name, Ts, w.seed + 31 * i, args.warmup, args.steps) for i in range(cores)]
    with ProcessPoolExecutor(cores, mp_context=mp.get_context("spawn")) as pool:
        res = list(pool.map(_reference_worker, jobs, timeout=900))
    per = [statistics.fmean(t) for t in res]
    value = sum(Ts / p for p in per)
    ms = statistics.fmean(per) * 1e3
    sample = (f"{cores} processes (one per host core), each stepping {Ts} tokens of {w.name} on its own seed, "
              f"single-threaded C oracle in each; tokens/s summed over the processes")
    return {
        "impl": "reference",
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16" if w.payload == "bf16" else "fp8-e4m3 dispatch, bf16 combine",
        "data": "synthetic",
        "config": {"workload": w.name, "T": w.T, "H": w.H, "E": w.E, "owners": w.R, "top_k": w.k,
                   "block_m": w.B, "payload": w.payload, "scale": w.scale, "sample_tokens_per_core": Ts},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": cores, "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }


def profile_case(args) -> int:
    """One kernel family of the path on the workload's inputs, launched `steps`
    times after `warmup` untimed launches, with every kernel it waits for
    finished before it starts (a profiler serialises kernels, so a consumer
    launched before its producer would only wait out its bound).  For ncu
    captures of one kernel (-k, -c); prints one line, no measurement."""
    import torch
    import combine_route_layout_02_b200 as sep
    w = W.WORKLOADS[args.workload]
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(0)
    d = W.make_inputs(w)
    x, idx, wt = d["x"].to(dev), d["topk_idx"].to(dev), d["topk_weight"].to(dev)
    h = sep.sep_layout(idx, w.E, w.R, w.B, flags=sep.SEP_LAYOUT_SYNC_COUNTS)
    sep.sep_handle_set_max_ctas(h, args.max_ctas)
    info = h.info()
    rows = info.max_pool_rows
    recv, scales = sep.alloc_pool(h, w.H, w.payload, w.scale, rows=rows)
    out = torch.empty(w.T, w.H, dtype=torch.bfloat16, device=dev)
    case = args.profile_case
    needs_y = case in ("combine", "scatter", "backward")     # an FP8 case's bf16 pool is large: only when read
    y = (recv if w.payload == "bf16" else
         W.random_x(61, w.H, seed=w.seed + 7).to(dev)[torch.arange(rows, device=dev) % 61].contiguous()
         if needs_y else None)
    n = args.warmup + args.steps
    status = torch.zeros(2, dtype=torch.int32, device=dev)
    if case in ("consumer", "gated"):
        tile_ready = torch.zeros(info.max_tiles, dtype=torch.int32, device=dev)
        dst = torch.empty_like(recv)
        y_done = torch.zeros(w.T, dtype=torch.int32, device=dev)
        st2 = torch.zeros(2, dtype=torch.int32, device=dev)
        for i in range(n):
            sep.sep_dispatch(h, x, recv, tile_ready=tile_ready, dispatch_seq=i + 1)
            torch.cuda.synchronize()                     # every tile is published before the consumer starts
            if case == "consumer":
                sep.sep_consume_tiles(h, recv, tile_ready, i + 1, dst, status, num_ctas=args.consumer_ctas)
            else:
                sep.sep_consume_tiles_stamp(h, recv, tile_ready, i + 1, dst, status, y_done, i + 1,
                                            num_ctas=args.consumer_ctas)
                torch.cuda.synchronize()                 # every token is stamped before the gated combine
                sep.sep_combine_gated(h, dst, wt, out, y_done, i + 1, st2,
                                      num_ctas=args.gate_ctas or torch.cuda.get_device_properties(dev)
                                      .multi_processor_count)
            torch.cuda.synchronize()
            assert status.cpu().tolist() == [0, 0] and st2.cpu().tolist() == [0, 0]
    elif case == "ep":
        R, Tr = w.R, w.T // w.R
        shards = [W.make_inputs(replace(w, T=Tr, seed=w.seed + 7919 * (r + 1))) for r in range(R)]
        hs = [sep.sep_layout(sd["topk_idx"].to(dev), w.E, R, w.B) for sd in shards]
        counts = torch.stack([hh.view("expert_counts") for hh in hs]).to(torch.int32).contiguous()
        plans = [sep.sep_ep_plan_device(counts, r, w.B) for r in range(R)]
        owner_rows = [int(v) for v in plans[0]["owner_rows"].cpu()]
        cap = [max(v, w.B) for v in owner_rows]
        pools = [torch.empty(c, w.H, dtype=torch.bfloat16, device=dev) for c in cap]
        maps = [torch.full((c,), -1, dtype=torch.int32, device=dev) for c in cap]
        ready = [torch.zeros(c // w.B, dtype=torch.int32, device=dev) for c in cap]
        arrival = [torch.zeros(c // w.B, dtype=torch.int32, device=dev) for c in cap]
        dsts = [torch.empty_like(pl) for pl in pools]
        err = torch.zeros(1, dtype=torch.int32, device=dev)
        xs = [sd["x"].to(dev) for sd in shards]
        ws = [sd["topk_weight"].to(dev) for sd in shards]
        outs = [torch.empty(Tr, w.H, dtype=torch.bfloat16, device=dev) for _ in range(R)]
        for o in range(R):
            sep.sep_ep_mark_padding(plans[o]["owner_block_offset"], plans[o]["owner_expert_counts"], w.B, cap[o],
                                    maps[o])
        for i in range(n):
            for r in range(R):
                sep.sep_ep_plan_device(counts, r, w.B)
                sep.sep_ep_dispatch_publish(hs[r], xs[r], r, plans[r], pools, cap, ready, arrival, i + 1, err,
                                            recv_token=maps)
            for o in range(R):                           # every tile already published
                sep.sep_ep_consume_tiles(plans[o]["owner_block_offset"], pools[o], maps[o], ready[o], arrival[o],
                                         i + 1, dsts[o], status, w.B, num_ctas=args.consumer_ctas)
            for r in range(R):
                sep.sep_ep_combine(hs[r], dsts, cap, plans[r]["delta"], ws[r], outs[r], err)
            torch.cuda.synchronize()
            assert status.cpu().tolist() == [0, 0] and int(err.item()) == 0
        for hh in hs:
            sep.sep_handle_free(hh)
    elif case == "ep_plain":
        # the expert-parallel dispatch without publication (bf16: staged bulk stores; FP8: codes and scales) and
        # the combine from the owners' pools (an FP8 workload's combine reads seeded bf16 expert outputs)
        import numpy as np
        R, Tr = w.R, w.T // w.R
        fp8 = w.payload != "bf16"
        shards = [W.make_inputs(replace(w, T=Tr, seed=w.seed + 7919 * (r + 1))) for r in range(R)]
        hs = [sep.sep_layout(sd["topk_idx"].to(dev), w.E, R, w.B, flags=sep.SEP_LAYOUT_SYNC_COUNTS) for sd in shards]
        counts = np.stack([hh.view("expert_counts").cpu().numpy() for hh in hs]).astype(np.int32)
        plans = [sep.sep_ep_plan(counts, r, w.B) for r in range(R)]
        prow = [max(int(v), 1) for v in plans[0]["owner_rows"]]
        pools = [torch.empty(n, w.H, dtype=torch.uint8 if fp8 else torch.bfloat16, device=dev) for n in prow]
        sdt = torch.uint8 if w.scale == "ue8m0" else torch.float32
        scale_pools = [torch.empty(n, w.H // 128, dtype=sdt, device=dev) for n in prow] if fp8 else None
        y_src = W.random_x(61, w.H, seed=w.seed + 7).to(dev) if fp8 else None
        y_pools = ([y_src[torch.arange(n, device=dev) % 61].contiguous() for n in prow] if fp8 else pools)
        deltas = [torch.from_numpy(pl["delta"]).to(dev) for pl in plans]
        xs = [sd["x"].to(dev) for sd in shards]
        ws = [sd["topk_weight"].to(dev) for sd in shards]
        outs = [torch.empty(Tr, w.H, dtype=torch.bfloat16, device=dev) for _ in range(R)]
        err = torch.zeros(1, dtype=torch.int32, device=dev)
        for _ in range(n):
            for r in range(R):
                if fp8:
                    sep.sep_ep_dispatch_fp8(hs[r], xs[r], r, deltas[r], pools, scale_pools, prow, err, scale=w.scale)
                else:
                    sep.sep_ep_dispatch(hs[r], xs[r], r, deltas[r], pools, prow, err)
            for r in range(R):
                sep.sep_ep_combine(hs[r], y_pools, prow, deltas[r], ws[r], outs[r], err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        for hh in hs:
            sep.sep_handle_free(hh)
    else:
        view_dst = torch.empty(info.num_pool_rows, w.H, dtype=torch.bfloat16, device=dev) if case == "gather" else None
        grad_y = torch.empty_like(recv) if case == "backward" and w.payload == "bf16" else None
        grad_w = torch.empty(w.T, w.k, dtype=torch.float32, device=dev)
        for _ in range(n):
            if case == "layout":
                sep.sep_layout(idx, w.E, w.R, w.B, handle=h)
            elif case in ("layout_dispatch", "one_launch"):
                sep.sep_layout_dispatch(idx, x, recv, w.E, w.R, w.B, payload=w.payload, scale=w.scale,
                                        recv_scales=scales, handle=h,
                                        flags=sep.SEP_LAYOUT_ONE_LAUNCH if case == "one_launch" else 0)
            elif case == "dispatch":
                sep.sep_dispatch(h, x, recv, payload=w.payload, scale=w.scale, recv_scales=scales)
            elif case == "combine":
                sep.sep_combine(h, y, wt, out)
            elif case == "scatter":
                sep.sep_combine_scatter(h, y, wt, out)
            elif case == "backward":
                sep.sep_dispatch_grads(h, out, wt, grad_y, y_pool=y, grad_w=grad_w)
                sep.sep_combine_grads(h, grad_y, out)
            elif case == "gather":
                sep.sep_gather_rows(sep.sep_dispatch_borrow(h, x), view_dst)
                sep.sep_view_release(h, [torch.cuda.current_stream()])
        torch.cuda.synchronize()
    sep.sep_handle_free(h)
    print(f"profile case {case} on {w.name}: {n} rounds done", flush=True)
    return 0


def main(argv=None) -> int:
    args = parse_args(argv)
    rank, world, local = dist_env()
    if args.profile_case is not None:
        return profile_case(args)
    if args.impl == "reference":
        res = run_reference(args, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return 0
    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    try:
        res = run_ours(args, rank, world, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    if res is not None:
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
