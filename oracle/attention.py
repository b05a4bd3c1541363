"""Oracle for block-sparse attention: exact softmax attention of every query token over the
tokens of its query block's selected key blocks. float64.

Test infrastructure only (see the package docstring); never used by the product path.

Follows the video-generation acceleration notes (wzjinhao.cn) §5.2, which expand the block
mask to a token mask and run a masked scaled-dot-product attention; key tokens at positions
>= S do not exist, so they take no part in any softmax.
"""
from __future__ import annotations

import numpy as np


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):          # torch tensor: bf16/fp32 -> fp64 is exact
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def _block_tokens(j: int, S: int, block: int) -> np.ndarray:
    return np.arange(j * block, min(S, (j + 1) * block))


def attention_block(Q, K, V, bh: int, i: int, sel_row, scale: float, block: int) -> np.ndarray:
    """Output rows of query block i of head bh: O_t = sum_u softmax_u(Q_t.K_u * scale) V_u,
    u over the valid tokens of the key blocks selected in `sel_row` (boolean [nb])."""
    S = Q.shape[1]
    rows = _block_tokens(i, S, block)
    cols = np.concatenate([_block_tokens(j, S, block) for j in np.nonzero(np.asarray(sel_row))[0]])
    q = _f64(Q[bh, rows[0]:rows[-1] + 1])
    k = _f64(K[bh][cols])
    v = _f64(V[bh][cols])
    s = (q @ k.T) * scale
    s = s - s.max(axis=1, keepdims=True)
    e = np.exp(s)
    return (e / e.sum(axis=1, keepdims=True)) @ v


def attention_rows(Q, K, V, mask, scale: float, items, block: int = 64) -> dict:
    """{(bh, i): output rows of query block i} for the requested (bh, i) items."""
    return {(bh, i): attention_block(Q, K, V, bh, i, mask[bh, i], scale, block) for bh, i in items}


def attention_sets(Q, K, V, mask, scale: float, block: int = 64) -> np.ndarray:
    """The full output [BH, S, d] in float64, one query block at a time."""
    BH, S, d = Q.shape
    nb = -(-S // block)
    out = np.empty((BH, S, d), dtype=np.float64)
    for bh in range(BH):
        for i in range(nb):
            rows = _block_tokens(i, S, block)
            out[bh, rows[0]:rows[-1] + 1] = attention_block(Q, K, V, bh, i, mask[bh, i], scale, block)
    return out


def attention_token_mask(Q, K, V, mask, scale: float, block: int = 64) -> np.ndarray:
    """Same output through the pages' literal route: block mask -> dense [S, S] token mask
    -> masked softmax over all keys. Small inputs only (O(S^2) memory)."""
    Qd, Kd, Vd = _f64(Q), _f64(K), _f64(V)
    BH, S, d = Qd.shape
    out = np.empty_like(Qd)
    for bh in range(BH):
        tok = np.repeat(np.repeat(np.asarray(mask[bh]), block, axis=0), block, axis=1)[:S, :S]
        s = (Qd[bh] @ Kd[bh].T) * scale
        s = np.where(tok, s, -np.inf)
        s = s - s.max(axis=1, keepdims=True)
        e = np.exp(s)
        out[bh] = (e / e.sum(axis=1, keepdims=True)) @ Vd[bh]
    return out


def selected_flops(mask, S: int, block: int, d: int) -> int:
    """Algorithmic FLOPs of attention over the selected blocks: 4*d per (query, key) token
    pair of a selected (query block, key block) pair, valid tokens only (2*d for Q.K and
    2*d for P.V)."""
    mask = np.asarray(mask, dtype=bool)
    nb = mask.shape[-1]
    n = np.array([min(S, (j + 1) * block) - j * block for j in range(nb)], dtype=np.int64)
    pairs = np.einsum("bij,i,j->", mask.astype(np.int64), n, n)
    return int(4 * d * pairs)


def attention_dense_mask(Q, K, V, tokmask, scale: float) -> np.ndarray:
    """Softmax attention of every query token over the key tokens its row of `tokmask`
    ([BH, S, S] bool) allows (the token-exact frame mode's definition). Small inputs only."""
    Qd, Kd, Vd = _f64(Q), _f64(K), _f64(V)
    out = np.empty_like(Qd)
    for bh in range(Qd.shape[0]):
        s = (Qd[bh] @ Kd[bh].T) * scale
        s = np.where(tokmask[bh], s, -np.inf)
        s = s - s.max(axis=1, keepdims=True)
        p = np.exp(s)
        out[bh] = (p / p.sum(axis=1, keepdims=True)) @ Vd[bh]
    return out
