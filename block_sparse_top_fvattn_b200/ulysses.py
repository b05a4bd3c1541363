"""Sequence parallelism around the block-sparse layer (the Ulysses layout the FVAttn summary's
multi-GPU setting runs on, section "AI视频生成的阿喀琉斯之踵": sequence-sharded activations,
heads distributed across GPUs for attention).

Each of R ranks holds all H heads of its S/R-token slice of the sequence. One all-to-all turns
that into H/R heads over the whole sequence (routing needs every block of a head), the layer
routes and attends them (optionally with runtime head migration, rlb.balanced_attention), and one
all-to-all returns the outputs to the sequence layout. Pooling the blocks of each shard as it
arrives (overlapping the all-to-all with the router's first pass) is not done here: the
all-to-all completes before routing starts.
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


def ulysses_attention(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, cfg: Optional[RouteConfig] = None, *,
                      group=None, balance: bool = False, target: float = 1.05, max_moves_per_rank: int = 1,
                      kernels=None) -> Tuple[torch.Tensor, Optional[rlb.Plan]]:
    """Block-sparse attention of sequence-sharded q, k, v ([1, H, S/R, d] on each rank; the
    sequence is the concatenation of the ranks' slices in rank order). Returns the output in the
    same layout and, with balance=True, the head-migration plan."""
    kernels = kernels or rlb.Kernels(cfg or RouteConfig())
    qh, kh, vh = (seq_to_head(t, group) for t in (q, k, v))
    plan = None
    if balance:
        oh, plan = rlb.balanced_attention(qh, kh, vh, group=group, target=target,
                                          max_moves_per_rank=max_moves_per_rank, kernels=kernels)
    else:
        oh = torch.empty_like(qh)
        kernels.attend(qh, kh, vh, kernels.route(qh, kh), None, oh)
    return head_to_seq(oh, group), plan
