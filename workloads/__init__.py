"""Seeded synthetic inputs for MoE dispatch/combine.

This module only draws the inputs the method consumes: hidden states ``x``,
router logits, and the top-k routing (``topk_idx``, ``topk_weight``) a router
would hand to dispatch.  It holds none of the dispatch/combine arithmetic
(counting, layout, permutation, quantisation, weighted reduction); both the
CPU oracle and the CUDA path take its outputs as plain arrays.

Recipe (same for every workload):

* ``x`` ~ N(0, 1) drawn in fp32, rounded to bf16 (round-to-nearest-even).
* Router logits ~ N(0, 1) fp32 of shape ``[T, E]``.  For the skewed prefill
  workload ``log p_e`` with ``p_e`` proportional to ``(e+1)^-s`` (Zipf,
  expert 0 most popular) is added to every row first.
* ``topk_idx`` = the k experts with the largest logits, in descending logit
  order, ties broken towards the lower expert id (stable sort).
* ``topk_weight`` = softmax over all E of the (possibly skewed) logits,
  gathered at ``topk_idx`` and renormalised to sum to 1 per token.
* One ``torch.Generator`` on the CPU per workload, seeded ``1000 + index`` in
  the order of ``WORKLOADS`` below; ``x`` is drawn before the logits.

The five workloads follow the shapes named for this path: a tiny case, a
decode-like FP8 case, the 8192-token training case, a Zipf-skewed FP8 prefill
case and a streaming case with per-tile ready flags.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
from typing import Optional

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    T: int            # tokens
    H: int            # hidden size
    E: int            # experts
    R: int            # logical owners ("ranks"), E % R == 0
    k: int            # top-k
    B: int            # BLOCK_M: pool tile height in rows
    payload: str      # "bf16" | "fp8"
    scale: str        # "none" | "f32" | "ue8m0" | "f32_pow2"
    seed: int
    zipf_s: Optional[float] = None
    streaming: bool = False

    @property
    def n_assign(self) -> int:
        return self.T * self.k


WORKLOADS = {
    "tiny": Workload("tiny", T=128, H=256, E=8, R=2, k=2, B=16,
                     payload="bf16", scale="none", seed=1000),
    "decode": Workload("decode", T=256, H=7168, E=256, R=32, k=8, B=64,
                       payload="fp8", scale="ue8m0", seed=1001),
    "train8k": Workload("train8k", T=8192, H=3072, E=128, R=8, k=8, B=128,
                        payload="bf16", scale="none", seed=1002),
    "prefill_skew": Workload("prefill_skew", T=16384, H=7168, E=256, R=8, k=8, B=128,
                             payload="fp8", scale="f32", seed=1003, zipf_s=1.2),
    "streaming": Workload("streaming", T=32768, H=4096, E=64, R=8, k=4, B=128,
                          payload="bf16", scale="none", seed=1004, streaming=True),
}


def scaled(w: Workload, T: int) -> Workload:
    """The same workload with fewer tokens (same seed, shapes per token)."""
    return replace(w, T=T)


def draw_x(g: torch.Generator, T: int, H: int) -> torch.Tensor:
    """bf16 [T, H], N(0,1) drawn in fp32 then rounded to nearest even."""
    return torch.randn(T, H, generator=g, dtype=torch.float32).to(torch.bfloat16)


def draw_logits(g: torch.Generator, T: int, E: int, zipf_s: Optional[float]) -> torch.Tensor:
    logits = torch.randn(T, E, generator=g, dtype=torch.float32)
    if zipf_s is not None:
        ranks = torch.arange(1, E + 1, dtype=torch.float64)
        p = ranks.pow(-zipf_s)
        p = p / p.sum()
        logits = logits + p.log().to(torch.float32)[None, :]
    return logits


def route_topk(logits: torch.Tensor, k: int):
    """Top-k by descending logit (ties to the lower id), softmax weights renormalised."""
    order = torch.sort(logits, dim=-1, descending=True, stable=True).indices[:, :k]
    probs = torch.softmax(logits, dim=-1)
    w = probs.gather(1, order)
    w = w / w.sum(dim=-1, keepdim=True)
    return order.to(torch.int32).contiguous(), w.to(torch.float32).contiguous()


def make_inputs(w: Workload, with_x: bool = True) -> dict:
    """CPU tensors: x bf16 [T,H] (optional), topk_idx int32 [T,k], topk_weight f32 [T,k]."""
    g = torch.Generator().manual_seed(w.seed)
    out = {}
    if with_x:
        out["x"] = draw_x(g, w.T, w.H)
    else:
        # keep the logits stream identical whether or not x is materialised
        _skip_normals(g, w.T * w.H)
    logits = draw_logits(g, w.T, w.E, w.zipf_s)
    out["topk_idx"], out["topk_weight"] = route_topk(logits, w.k)
    return out


def _skip_normals(g: torch.Generator, n: int) -> None:
    chunk = 1 << 24
    while n > 0:
        m = min(n, chunk)
        torch.randn(m, generator=g, dtype=torch.float32)
        n -= m


def random_x(T: int, H: int, seed: int) -> torch.Tensor:
    g = torch.Generator().manual_seed(seed)
    return draw_x(g, T, H)


def random_weights(T: int, k: int, seed: int) -> torch.Tensor:
    """Positive weights renormalised per token (for hand-built routings)."""
    g = torch.Generator().manual_seed(seed)
    w = torch.rand(T, k, generator=g, dtype=torch.float32) + 0.05
    return (w / w.sum(dim=-1, keepdim=True)).contiguous()


def edge_routing(kind: str, T: int, k: int, E: int, R: int, seed: int) -> torch.Tensor:
    """Extreme routings for correctness tests (int32 [T,k]).

    kinds: ``one_expert`` (every assignment to expert E-1, duplicates within a
    token), ``owner_empty`` (owner 0 gets nothing), ``same_owner`` (a token's
    k experts all on one owner), ``masked`` (about a quarter of the entries
    are -1, i.e. no assignment), ``skew`` (nearly everything on expert 0),
    ``uniform`` (distinct experts drawn uniformly).
    """
    g = torch.Generator().manual_seed(seed)
    E_loc = E // R
    if kind == "one_expert":
        return torch.full((T, k), E - 1, dtype=torch.int32)
    if kind == "uniform" or kind == "masked":
        idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32)
        if kind == "masked":
            drop = torch.rand(T, k, generator=g) < 0.25
            idx[drop] = -1
        return idx.contiguous()
    if kind == "owner_empty":
        assert k <= E - E_loc
        idx = torch.stack([E_loc + torch.randperm(E - E_loc, generator=g)[:k] for _ in range(T)])
        return idx.to(torch.int32).contiguous()
    if kind == "same_owner":
        assert k <= E_loc
        owner = torch.randint(0, R, (T,), generator=g)
        rows = [owner[t].item() * E_loc + torch.randperm(E_loc, generator=g)[:k] for t in range(T)]
        return torch.stack(rows).to(torch.int32).contiguous()
    if kind == "skew":
        idx = torch.stack([torch.randperm(E, generator=g)[:k] for _ in range(T)]).to(torch.int32)
        hot = torch.rand(T, generator=g) < 0.9
        idx[hot, 0] = 0
        # keep experts distinct within a token after forcing slot 0 to expert 0
        for t in torch.nonzero(hot).flatten().tolist():
            row = idx[t]
            dup = (row[1:] == 0).nonzero().flatten()
            for d in dup.tolist():
                row[1 + d] = E - 1 if row[0] != E - 1 else E - 2
        return idx.contiguous()
    raise ValueError(f"unknown routing kind {kind!r}")


__all__ = ["Workload", "WORKLOADS", "scaled", "make_inputs", "edge_routing", "random_x",
           "random_weights", "route_topk", "draw_logits", "draw_x"]
