"""Oracle for runtime load balancing of heads across ranks (FVAttn blog summary, section
"RLB：不搞全局重洗，只做P2P“微创手术”，修复临界路径"). Integer loads, plain Python.

Test infrastructure only (see the package docstring); never used by the product path.

The summary's procedure: once the layer's sparse masks exist, each rank knows the load of
each of its heads (the number of blocks the head computes); the loads of all heads of all
ranks are exchanged; a greedy scheduler then repeatedly takes the most loaded rank as the
sender and the least loaded rank as the receiver and moves one head, the sender's heaviest,
point to point, until the imbalance factor is below a threshold or the migration budget
(about a fifth of a rank's heads) is used up. The imbalance factor is taken as max / mean of
the rank loads.

Readings where the summary is silent: ties between ranks and between heads go to the lower
index; only heads that started on the sender and have not moved yet can move (a head moves at
most once); a move is made only if it lowers the pair's maximum (receiver load + head load <
sender load), so the heaviest head that satisfies this is taken, and the plan stops when no
head of the sender does; the budget counts the heads a rank sends.
"""
from __future__ import annotations

from typing import List, Tuple

import numpy as np


def imbalance(rank_loads) -> float:
    """max / mean of the per-rank loads (1.0 when every rank is idle)."""
    L = [int(x) for x in rank_loads]
    total = sum(L)
    if total == 0:
        return 1.0
    return max(L) * len(L) / total


def rlb_plan(loads, target: float, max_moves_per_rank: int):
    """Greedy head migration plan.

    loads [R, Hl]: load of local head h of rank r. Returns (moves, rank_loads) where moves is
    the ordered list of (src rank, local head index on src, dst rank) and rank_loads the loads
    after the moves."""
    loads = np.asarray(loads, dtype=np.int64)
    R, Hl = loads.shape
    L = [int(x) for x in loads.sum(axis=1)]
    moved = np.zeros((R, Hl), dtype=bool)
    sent = [0] * R
    moves: List[Tuple[int, int, int]] = []
    while imbalance(L) > target:
        s = max(range(R), key=lambda r: (L[r], -r))          # most loaded, lowest index on ties
        d = min(range(R), key=lambda r: (L[r], r))           # least loaded, lowest index on ties
        if s == d or sent[s] >= max_moves_per_rank:
            break
        best = -1
        for h in range(Hl):
            w = int(loads[s, h])
            if moved[s, h] or not (L[d] + w < L[s]):
                continue
            if best < 0 or w > int(loads[s, best]):
                best = h
        if best < 0:
            break
        w = int(loads[s, best])
        L[s] -= w
        L[d] += w
        moved[s, best] = True
        sent[s] += 1
        moves.append((s, best, d))
    return moves, L
