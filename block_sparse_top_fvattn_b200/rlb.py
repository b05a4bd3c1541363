"""Runtime load balancing of heads across ranks (FVAttn blog summary, section
"RLB：不搞全局重洗，只做P2P“微创手术”，修复临界路径").

One process per GPU. Each rank holds the full sequence of its local heads, [1, Hl, S, d], the
layout after the sequence-to-head all-to-all of sequence parallelism. With data-dependent
Top-p routing the ranks' loads differ; the slowest rank sets the step time. balanced_attention
repairs that at run time, once the layer's masks exist:

  1. route the local heads (fvattn_route);
  2. all-gather the per-head loads, ranks x Hl int64 (the only collective);
  3. plan the moves (fvattn_rlb_plan; a pure function, so every rank computes the same plan);
  4. send each moved head's Q, K and V point to point to its receiver, while the sender runs
     the attention of the heads it keeps (fvattn_select_heads, fvattn_sparse_attn);
  5. the receiver routes and attends the received heads and sends their outputs back.

A migrated head is computed exactly as at home (same kernels, same routing), so the outputs do
not depend on the plan. The per-rank compute is behind a small interface (`Kernels`) so that the
exchange can be exercised on CPU process groups; the default is this library's CUDA path.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional, Tuple

import numpy as np
import torch
import torch.distributed as dist

from . import (RouteConfig, alloc_csr, rlb_plan, route, route_finish, route_pool, select_heads, sparse_attn,
               workspace_bytes)


class Kernels:
    """Per-rank compute of balanced_attention: this library's CUDA path."""

    def __init__(self, cfg: RouteConfig):
        self.cfg = cfg

    def route(self, q: torch.Tensor, k: torch.Tensor):
        B, H, S, _ = q.shape
        return route(q, k, self.cfg, csr=alloc_csr(B, H, S, q.device, codes=self.cfg.frame_exact))

    # The router in two stages (fvattn_route_pool / fvattn_route_finish), for pooling the blocks
    # of each part of the sequence as it arrives.
    def begin_route(self, q: torch.Tensor):
        return torch.empty(workspace_bytes(q, self.cfg), dtype=torch.uint8, device=q.device)

    def pool_blocks(self, handle, q: torch.Tensor, k: torch.Tensor, block_begin: int, block_end: int) -> None:
        route_pool(q, k, self.cfg, block_begin, block_end, handle)

    def finish_route(self, handle, q: torch.Tensor):
        return route_finish(q, self.cfg, handle)

    @staticmethod
    def head_load(state) -> torch.Tensor:
        return state.head_load

    def attend(self, q, k, v, state, active: Optional[List[bool]], out: torch.Tensor) -> None:
        if active is not None:
            select_heads(state, torch.tensor(active, dtype=torch.uint8, device=q.device))
        sparse_attn(q, k, v, state, out=out)


@dataclasses.dataclass
class Plan:
    moves: List[Tuple[int, int, int]]      # (sender rank, sender's local head, receiver rank)
    loads: np.ndarray                      # [ranks, Hl] per-head loads
    rank_loads_before: List[int]
    rank_loads_after: List[int]

    @staticmethod
    def _imb(L) -> float:
        tot = sum(L)
        return max(L) * len(L) / tot if tot else 1.0

    @property
    def imbalance_before(self) -> float:
        return self._imb(self.rank_loads_before)

    @property
    def imbalance_after(self) -> float:
        return self._imb(self.rank_loads_after)


def gather_loads(head_load: torch.Tensor, group=None) -> np.ndarray:
    """All-gather every rank's per-head loads: [ranks, Hl] int64 on the host."""
    world = dist.get_world_size(group)
    parts = [torch.empty_like(head_load) for _ in range(world)]
    dist.all_gather(parts, head_load.contiguous(), group=group)
    return torch.stack(parts).cpu().numpy().astype(np.int64)


def make_plan(loads: np.ndarray, target: float, max_moves_per_rank: int) -> Plan:
    moves, after = rlb_plan(loads, target, max_moves_per_rank)
    return Plan(moves, loads, [int(x) for x in loads.sum(axis=1)], after)


def _exchange(ops) -> None:
    if ops:
        for req in dist.batch_isend_irecv(ops):
            req.wait()


def balanced_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cfg: Optional[RouteConfig] = None, *,
                       group=None, target: float = 1.05, max_moves_per_rank: int = 1,
                       kernels=None, state=None) -> Tuple[torch.Tensor, Plan]:
    """Block-sparse attention of this rank's heads with runtime head migration between ranks.
    q, k, v: [1, Hl, S, d], the same Hl, S, d and dtype on every rank; `state`: the routing of
    these heads when the caller already has it. Returns (O, plan)."""
    if q.shape[0] != 1:
        raise ValueError("expected [1, Hl, S, d] per rank")
    kernels = kernels or Kernels(cfg or RouteConfig())
    rank = dist.get_rank(group)
    peer = (lambda r: dist.get_global_rank(group, r)) if group is not None else (lambda r: r)
    _, Hl, S, d = q.shape

    if state is None:
        state = kernels.route(q, k)
    plan = make_plan(gather_loads(kernels.head_load(state), group), target, max_moves_per_rank)
    out = torch.empty_like(q)

    sent = [h for s, h, _ in plan.moves if s == rank]
    incoming = [(s, h) for s, h, dst in plan.moves if dst == rank]
    # 4. Q, K, V of the moved heads, in plan order on both sides of every pair of ranks
    ops = []
    qr = kr = vr = None
    if incoming:
        qr, kr, vr = (torch.empty((1, len(incoming), S, d), dtype=q.dtype, device=q.device) for _ in range(3))
    for s, h, dst in plan.moves:
        if s == rank:
            ops += [dist.P2POp(dist.isend, t[0, h], peer(dst), group) for t in (q, k, v)]
        elif dst == rank:
            slot = incoming.index((s, h))
            ops += [dist.P2POp(dist.irecv, t[0, slot], peer(s), group) for t in (qr, kr, vr)]
    reqs = dist.batch_isend_irecv(ops) if ops else []
    # ... while the heads this rank keeps are computed
    active = None
    if sent:
        active = [h not in sent for h in range(Hl)]
    if active is None or any(active):
        kernels.attend(q, k, v, state, active, out)
    for req in reqs:
        req.wait()
    # 5. the received heads, and their outputs back to their senders
    ops = []
    if incoming:
        out_r = torch.empty_like(qr)
        kernels.attend(qr, kr, vr, kernels.route(qr, kr), None, out_r)
        for slot, (s, h) in enumerate(incoming):
            ops.append(dist.P2POp(dist.isend, out_r[0, slot], peer(s), group))
    for s, h, dst in plan.moves:
        if s == rank:
            ops.append(dist.P2POp(dist.irecv, out[0, h], peer(dst), group))
    _exchange(ops)
    return out, plan
