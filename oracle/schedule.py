"""Oracle for the router's bookkeeping: CSR block lists, per-head loads, 128-row tile costs
and the longest-first (LPT) tile order. Integer arithmetic only.

Test infrastructure only (see the package docstring); never used by the product path.

Follows the FVAttn blog summary, section "RLB：不搞全局重洗…": the load of a head is the
number of blocks it has to compute, and the balancer moves the heaviest work first. On one
GPU the unit that is balanced is a tile of 128 query rows (two consecutive 64-token query
blocks of one head), whose cost is the number of distinct key blocks it must visit.
"""
from __future__ import annotations

import numpy as np


def csr_from_mask(mask):
    """row = bh*nb + i; row_ptr = exclusive prefix sum of the per-row counts; col_idx lists
    the selected key blocks of each row in ascending order."""
    mask = np.asarray(mask, dtype=bool)
    BH, nb, _ = mask.shape
    rows = mask.reshape(BH * nb, nb)
    counts = rows.sum(axis=1).astype(np.int64)
    row_ptr = np.zeros(BH * nb + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum(counts)
    col_idx = np.concatenate([np.nonzero(r)[0] for r in rows]).astype(np.int64) if BH * nb else np.zeros(0, np.int64)
    return row_ptr, col_idx


def head_loads(mask) -> np.ndarray:
    """Number of selected (query block, key block) pairs of each head: [BH] int64."""
    return np.asarray(mask, dtype=bool).sum(axis=(1, 2)).astype(np.int64)


def tile_costs(mask) -> np.ndarray:
    """[BH, ntiles] with ntiles = ceil(nb/2): the size of the union of the key-block sets of
    query blocks 2t and 2t+1 (just 2t when nb is odd and t is the last tile)."""
    mask = np.asarray(mask, dtype=bool)
    BH, nb, _ = mask.shape
    nt = -(-nb // 2)
    cost = np.zeros((BH, nt), dtype=np.int64)
    for t in range(nt):
        u = mask[:, 2 * t].copy()
        if 2 * t + 1 < nb:
            u |= mask[:, 2 * t + 1]
        cost[:, t] = u.sum(axis=1)
    return cost


def lpt_order(costs) -> np.ndarray:
    """Tile ids (bh*ntiles + t) sorted by cost, largest first; equal costs keep ascending id."""
    c = np.asarray(costs).reshape(-1)
    return np.argsort(-c, kind="stable").astype(np.int64)
