"""Expert parallelism across processes: the host side around the EP kernels.

One process per rank (normally one per GPU; several may share one GPU).  Rank
o owns experts [o*E/R, (o+1)*E/R).  Each step:

1. the rank lays out its own routing (``sep_layout`` with num_owners = R);
2. the ranks exchange their expert counts (an all-gather of E integers, the
   one collective of the path) and each computes its plan (``sep_ep_plan``);
3. each owner marks the padding rows of its pool; a barrier;
4. each rank writes its token rows straight into the owners' pools through
   their pointers (``sep_ep_dispatch``); a barrier;
5. the owners compute their experts' outputs into their shared y buffers;
   a barrier;
6. each rank reads its tokens' k output rows from the owners' y buffers and
   reduces them (``sep_ep_combine``); a barrier before the buffers are reused.

With ``signals=True`` the plan is computed on the GPU (``sep_ep_plan_device``)
from counts gathered device to device (through the host only when the
group's backend is gloo), so the host never waits for a count; every owner
tile is published once complete (``sep_ep_dispatch_publish``: per-tile
arrivals and a system-scope release of the step's sequence number in the
owner's memory), and the owner's reference consumer (``consume``) copies each
tile as it is published.  A step then holds two or three barriers instead
of four: the one after the combine goes (the next step's barrier before its
dispatches follows every rank's synchronised combine), and
``concurrent=True`` drops the one between the dispatches and the owners'
consumers, for groups whose ranks are on different GPUs (never for ranks
sharing a GPU, whose kernels are not guaranteed to run at the same time).

The dispatch may carry the bf16 rows or the FP8 e4m3 payload with its
per-128-channel scales.  The pools, y buffers, scales and receive maps are
allocated by the library and shared
by CUDA IPC (plain device memory mapped into every peer; no multicast).  The
barriers follow a device synchronisation, so no kernel ever waits on another
process's kernel.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.distributed as dist

from . import sep as _sep


def _pool_rows_cap(world: int, max_tokens: int, top_k: int, num_local_experts: int, block_m: int) -> int:
    """Rows of an owner's pool that hold any routing: every assignment of every
    rank on this owner, plus at most block_m - 1 padding rows per local expert."""
    n = world * max_tokens * top_k
    rows = n + min(num_local_experts, n) * (block_m - 1)
    return max((rows + block_m - 1) // block_m * block_m, block_m)


class EPGroup:
    """Dispatch and combine across the ranks of a torch.distributed group."""

    def __init__(self, num_experts: int, top_k: int, block_m: int, hidden: int, max_tokens: int, group=None,
                 signals: bool = False, concurrent: bool = False):
        self.group = group
        self.rank = dist.get_rank(group)
        self.world = dist.get_world_size(group)
        if num_experts % self.world != 0:
            raise ValueError("num_experts must be divisible by the number of ranks")
        self.E, self.k, self.B, self.H = num_experts, top_k, block_m, hidden
        self.E_loc = num_experts // self.world
        self.rows_cap = _pool_rows_cap(self.world, max_tokens, top_k, self.E_loc, block_m)
        self.tiles_cap = self.rows_cap // block_m
        self.signals, self.concurrent = signals, concurrent
        self.cpu_collectives = dist.get_backend(group) != "nccl"
        self.G = max(hidden // 128, 1)
        own = [_sep.sep_ep_buffer_alloc(self.rows_cap * hidden * 2),   # pool (bf16 rows, or e4m3 codes)
               _sep.sep_ep_buffer_alloc(self.rows_cap * hidden * 2),   # expert outputs y
               _sep.sep_ep_buffer_alloc(3 * self.rows_cap * 4),        # receive maps: token, rank, slot
               _sep.sep_ep_buffer_alloc(self.rows_cap * self.G * 4),   # FP8 scales (fp32 or u8)
               _sep.sep_ep_buffer_alloc(2 * self.tiles_cap * 4)]       # tile_ready, arrival counters
        handles = [None] * self.world
        dist.all_gather_object(handles, [b.handle for b in own], group=group)
        self.buffers = []                                # [rank] -> [pool, y, maps, scales]
        for r in range(self.world):
            if r == self.rank:
                self.buffers.append(own)
            else:
                self.buffers.append([_sep.sep_ep_buffer_open(h, b.nbytes) for h, b in zip(handles[r], own)])
        shape = (self.rows_cap, hidden)
        self.pools = [bufs[0].tensor(shape, torch.bfloat16) for bufs in self.buffers]
        self.ys = [bufs[1].tensor(shape, torch.bfloat16) for bufs in self.buffers]
        maps = [bufs[2].tensor((3, self.rows_cap), torch.int32) for bufs in self.buffers]
        self.codes = [bufs[0].tensor((self.rows_cap, hidden), torch.uint8) for bufs in self.buffers]
        self.scales_f32 = [bufs[3].tensor((self.rows_cap, self.G), torch.float32) for bufs in self.buffers]
        self.scales_u8 = [bufs[3].tensor((self.rows_cap, self.G), torch.uint8) for bufs in self.buffers]
        self.recv_token = [m[0] for m in maps]
        self.recv_rank = [m[1] for m in maps]
        self.recv_slot = [m[2] for m in maps]
        flags = [bufs[4].tensor((2, self.tiles_cap), torch.int32) for bufs in self.buffers]
        self.tile_ready = [f[0] for f in flags]
        self.arrival = [f[1] for f in flags]
        flags[self.rank].zero_()                         # counters start at zero; flags below any sequence
        self.seq = 0
        self.status = torch.zeros(2, dtype=torch.int32, device="cuda")
        self.handle = _sep.sep_handle_create(max_tokens, top_k, num_experts, self.world, block_m)
        self.error = torch.zeros(1, dtype=torch.int32, device="cuda")
        self.plan = None
        self._barrier()

    def _barrier(self):
        torch.cuda.synchronize()                         # this process's kernels are done first
        dist.barrier(group=self.group)

    def _all_counts(self) -> np.ndarray:
        mine = self.handle.view("expert_counts").to(torch.int32)
        if self.cpu_collectives:
            mine = mine.cpu()
        out = [torch.zeros_like(mine) for _ in range(self.world)]
        dist.all_gather(out, mine, group=self.group)
        return torch.stack(out).cpu().numpy()

    def _all_counts_device(self) -> torch.Tensor:
        mine = self.handle.view("expert_counts").to(torch.int32)
        if self.cpu_collectives:
            out = [torch.zeros(self.E, dtype=torch.int32) for _ in range(self.world)]
            dist.all_gather(out, mine.cpu(), group=self.group)
            return torch.stack(out).cuda()
        out = torch.empty(self.world, self.E, dtype=torch.int32, device="cuda")
        dist.all_gather_into_tensor(out, mine, group=self.group)
        return out

    def _dispatch_signals(self, x, topk_idx, payload, scale):
        """Steps 1-4 with the plan on the GPU and per-tile publication."""
        _sep.sep_layout(topk_idx, self.E, self.world, self.B, handle=self.handle)
        plan = _sep.sep_ep_plan_device(self._all_counts_device(), self.rank, self.B)
        self.plan, self.delta = plan, plan["delta"]
        self.rows = [self.rows_cap] * self.world         # capacities: the kernels refuse rows past them
        _sep.sep_ep_mark_padding(plan["owner_block_offset"], plan["owner_expert_counts"], self.B, self.rows_cap,
                                 self.recv_token[self.rank], self.recv_rank[self.rank], self.recv_slot[self.rank])
        # this owner's arrival counters start the step at zero even if the last
        # step's tiles were not all consumed (the consumer zeroes only what it copies)
        self.arrival[self.rank].zero_()
        self._barrier()                                  # every owner ready, the last step's readers done
        self.seq = (self.seq + 1) & 0x7FFFFFFF or 1
        maps = dict(recv_token=self.recv_token, recv_rank=self.recv_rank, recv_slot=self.recv_slot)
        if payload == "fp8":
            scales = self.scales_u8 if scale == "ue8m0" else self.scales_f32
            _sep.sep_ep_dispatch_publish(self.handle, x, self.rank, plan, self.codes, self.rows, self.tile_ready,
                                         self.arrival, self.seq, self.error, payload="fp8", scale=scale,
                                         scales=scales, **maps)
            received = (self.codes[self.rank], scales[self.rank])
        else:
            _sep.sep_ep_dispatch_publish(self.handle, x, self.rank, plan, self.pools, self.rows, self.tile_ready,
                                         self.arrival, self.seq, self.error, **maps)
            received = self.pools[self.rank]
        if not self.concurrent:
            self._barrier()                              # every row has landed
        return received, self.recv_token[self.rank], self.recv_rank[self.rank], self.recv_slot[self.rank]

    def consume(self, timeout_ns: int = 0) -> torch.Tensor:
        """Owner side, signals only: the reference consumer copies each tile of
        this owner's pool into its y buffer as soon as the tile is published
        (identity experts).  Returns the status words [code, tiles not copied]."""
        if not self.signals:
            raise RuntimeError("consume() needs an EPGroup made with signals=True")
        _sep.sep_ep_consume_tiles(self.plan["owner_block_offset"], self.pools[self.rank], self.recv_token[self.rank],
                                  self.tile_ready[self.rank], self.arrival[self.rank], self.seq,
                                  self.ys[self.rank], self.status, self.B, timeout_ns=timeout_ns)
        return self.status

    def dispatch(self, x: torch.Tensor, topk_idx: torch.Tensor, payload: str = "bf16", scale: str = "none"):
        """Steps 1-4; returns this owner's received rows (a view of its pool:
        bf16 [P_o, H], or with payload="fp8" the pair of e4m3 codes [P_o, H] as
        bytes and scales [P_o, H/128], fp32 or u8) and receive maps (token,
        rank, slot), each [P_o].  With signals=True the views cover the pool's
        whole capacity (the pool size stays on the GPU, in the plan's
        owner_rows) and rows past the pool keep -1 in the maps."""
        if self.signals:
            return self._dispatch_signals(x, topk_idx, payload, scale)
        _sep.sep_layout(topk_idx, self.E, self.world, self.B, handle=self.handle)
        plan = _sep.sep_ep_plan(self._all_counts(), self.rank, self.B)
        rows = [int(v) for v in plan["owner_rows"]]
        if max(rows) > self.rows_cap:
            raise RuntimeError(f"an owner needs {max(rows)} pool rows, the group holds {self.rows_cap}")
        self.plan = plan
        self.rows = rows
        self.delta = torch.from_numpy(plan["delta"]).cuda()
        _sep.sep_ep_mark_padding(torch.from_numpy(plan["owner_block_offset"]).cuda(),
                                 torch.from_numpy(plan["owner_expert_counts"]).cuda(), self.B, rows[self.rank],
                                 self.recv_token[self.rank], self.recv_rank[self.rank], self.recv_slot[self.rank])
        self._barrier()                                  # every owner ready, the last step's readers done
        maps = dict(recv_token=self.recv_token, recv_rank=self.recv_rank, recv_slot=self.recv_slot)
        P = rows[self.rank]
        if payload == "fp8":
            scales = self.scales_u8 if scale == "ue8m0" else self.scales_f32
            _sep.sep_ep_dispatch_fp8(self.handle, x, self.rank, self.delta, self.codes, scales, rows, self.error,
                                     scale=scale, **maps)
            self._barrier()                              # every row has landed
            received = (self.codes[self.rank][:P], scales[self.rank][:P])
        else:
            _sep.sep_ep_dispatch(self.handle, x, self.rank, self.delta, self.pools, rows, self.error, **maps)
            self._barrier()                              # every row has landed
            received = self.pools[self.rank][:P]
        return (received, self.recv_token[self.rank][:P], self.recv_rank[self.rank][:P],
                self.recv_slot[self.rank][:P])

    def expert_output(self) -> torch.Tensor:
        """This owner's y buffer [P_o, H], to be filled with its experts' outputs
        (row r of y is the output for row r of the received pool)."""
        return self.ys[self.rank][: self.rows[self.rank]]

    def combine(self, topk_weight: torch.Tensor, out: torch.Tensor, y_is_pool: bool = False) -> None:
        """Step 6: out[t] = bf16(sum_j w[t, j] * y_owner[row(t, j)]).  With
        y_is_pool the received rows themselves are the outputs (identity experts)."""
        self._barrier()                                  # every owner's outputs are written
        ys = self.pools if y_is_pool else self.ys
        if self.signals and int(self.plan["error"].item()) != 0:
            raise RuntimeError("the exchanged counts hold a negative count or exceed 32-bit pool rows")
        if self.signals and int(self.status[0].item()) != 0:
            raise RuntimeError(f"an owner's consumer reported {self.status.cpu().tolist()}")
        _sep.sep_ep_combine(self.handle, ys, self.rows, self.delta, topk_weight, out, self.error)
        if not self.signals:
            self._barrier()                              # before the next step reuses the buffers
        # with signals the next step's pre-dispatch barrier follows every rank's
        # synchronised combine before any pool, y buffer or counter is written again
        if int(self.error.item()) != 0:
            raise RuntimeError("a row fell outside its owner's pool")

    def close(self) -> None:
        self._barrier()
        for r, bufs in enumerate(self.buffers):
            if r != self.rank:
                for b in bufs:
                    b.close()
        self._barrier()                                  # every peer has unmapped this rank's buffers
        for b in self.buffers[self.rank]:
            b.close()
        _sep.sep_handle_free(self.handle)
