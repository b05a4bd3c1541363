"""Sequence parallelism around the block-sparse layer (the Ulysses layout the FVAttn summary's
multi-GPU setting runs on, section "AI视频生成的阿喀琉斯之踵": sequence-sharded activations,
heads distributed across GPUs for attention).

Each of R ranks holds all H heads of its S/R-token slice of the sequence. One all-to-all turns
that into H/R heads over the whole sequence (routing needs every block of a head), the layer
routes and attends them (optionally with runtime head migration, rlb.balanced_attention), and one
all-to-all returns the outputs to the sequence layout. With overlap_pool=True the Q and K
exchange runs as R-1 shift steps (step s: send to rank+s, receive from rank-s, one batched
group per step) and the router's first pass (fvattn_route_pool) pools each received slice's
blocks while the later steps are still in flight; fvattn_route_finish completes the routing
once every slice is in.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch
import torch.distributed as dist

from . import RouteConfig
from . import rlb


def seq_to_head(x: torch.Tensor, group=None) -> torch.Tensor:
    """[1, H, S/R, d] (every head, this rank's sequence slice) -> [1, H/R, S, d] (this rank's
    heads, the whole sequence; slice r of the sequence came from rank r)."""
    R = dist.get_world_size(group)
    _, H, Sl, d = x.shape
    if H % R:
        raise ValueError(f"H={H} is not a multiple of {R} ranks")
    Hl = H // R
    send = x[0].reshape(R, Hl, Sl, d).contiguous()          # chunk r: the heads of rank r
    recv = torch.empty_like(send)                           # chunk r: sequence slice r of my heads
    dist.all_to_all_single(recv, send, group=group)
    return recv.permute(1, 0, 2, 3).reshape(1, Hl, R * Sl, d)


def head_to_seq(o: torch.Tensor, group=None) -> torch.Tensor:
    """Inverse of seq_to_head: [1, H/R, S, d] -> [1, H, S/R, d]."""
    R = dist.get_world_size(group)
    _, Hl, S, d = o.shape
    if S % R:
        raise ValueError(f"S={S} is not a multiple of {R} ranks")
    Sl = S // R
    send = o[0].reshape(Hl, R, Sl, d).permute(1, 0, 2, 3).contiguous()   # chunk r: sequence slice r
    recv = torch.empty_like(send)                                        # chunk r: heads of rank r
    dist.all_to_all_single(recv, send, group=group)
    return recv.reshape(1, R * Hl, Sl, d)


def seq_to_head_pooled(q: torch.Tensor, k: torch.Tensor, on_slice, group=None):
    """seq_to_head of q and k by R-1 shift steps, calling on_slice(qh, kh, r) on the current
    stream as soon as sequence slice r of this rank's heads is in place (own slice first)."""
    R = dist.get_world_size(group)
    rank = dist.get_rank(group)
    peer = (lambda r: dist.get_global_rank(group, r)) if group is not None else (lambda r: r)
    _, H, Sl, d = q.shape
    if H % R:
        raise ValueError(f"H={H} is not a multiple of {R} ranks")
    Hl = H // R
    send = [t[0].reshape(R, Hl, Sl, d).contiguous() for t in (q, k)]   # chunk r: the heads of rank r
    recv = [torch.empty_like(x) for x in send]                         # chunk r: slice r of my heads
    heads = [torch.empty((1, Hl, R * Sl, d), dtype=q.dtype, device=q.device) for _ in range(2)]
    steps = []
    for s in range(1, R):
        dst, src = (rank + s) % R, (rank - s) % R
        ops = []
        for x, y in zip(send, recv):
            ops += [dist.P2POp(dist.isend, x[dst], peer(dst), group), dist.P2POp(dist.irecv, y[src], peer(src), group)]
        steps.append((src, dist.batch_isend_irecv(ops)))

    def place(r):
        for h, y in zip(heads, recv):
            h[0, :, r * Sl:(r + 1) * Sl].copy_(y[r])
        on_slice(heads[0], heads[1], r)

    for h, x in zip(heads, send):
        h[0, :, rank * Sl:(rank + 1) * Sl].copy_(x[rank])
    on_slice(heads[0], heads[1], rank)
    for src, reqs in steps:
        for rq in reqs:
            rq.wait()
        place(src)
    return heads[0], heads[1]


def ulysses_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cfg: Optional[RouteConfig] = None, *,
                      group=None, balance: bool = False, target: float = 1.05, max_moves_per_rank: int = 1,
                      kernels=None, overlap_pool: bool = False) -> Tuple[torch.Tensor, Optional[rlb.Plan]]:
    """Block-sparse attention of sequence-sharded q, k, v ([1, H, S/R, d] on each rank; the
    sequence is the concatenation of the ranks' slices in rank order). Returns the output in the
    same layout and, with balance=True, the head-migration plan. overlap_pool pools each arriving
    slice's blocks during the exchange (slices must be whole 64-token blocks)."""
    kernels = kernels or rlb.Kernels(cfg or RouteConfig())
    Sl = q.shape[2]
    state = None
    if overlap_pool and Sl % 64 == 0:
        handle = None

        def on_slice(qh_, kh_, r):
            nonlocal handle
            if handle is None:
                handle = kernels.begin_route(qh_)
            kernels.pool_blocks(handle, qh_, kh_, r * Sl // 64, (r + 1) * Sl // 64)

        qh, kh = seq_to_head_pooled(q, k, on_slice, group)
        state = kernels.finish_route(handle, qh)
    else:
        qh, kh = (seq_to_head(t, group) for t in (q, k))
    vh = seq_to_head(v, group)
    plan = None
    if balance:
        oh, plan = rlb.balanced_attention(qh, kh, vh, group=group, target=target,
                                          max_moves_per_rank=max_moves_per_rank, kernels=kernels, state=state)
    else:
        oh = torch.empty_like(qh)
        kernels.attend(qh, kh, vh, state if state is not None else kernels.route(qh, kh), None, oh)
    return head_to_seq(oh, group), plan
