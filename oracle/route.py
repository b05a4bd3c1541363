"""Oracle for the router: block pooling, block scores, row softmax, Top-p cut, forced
blocks and frame-level top-k. float64 NumPy, one plain step per function.

Test infrastructure only (see the package docstring); never used by the product path.
"""
from __future__ import annotations

import dataclasses
import itertools
import math
from typing import Optional

import numpy as np

EPS_GAP = 1e-6    # probability gap under which two blocks count as tied
EPS_MASS = 1e-5   # distance of a cumulative mass from p under which the cut counts as tied


@dataclasses.dataclass
class RouteCfg:
    """Routing configuration.

    mode         "topp" (FVAttn Top-p), "frame_topk" (Sol-Attn frame-level top-k) or "topk"
                 (a fixed number of key blocks per query block, the notes' teaching variant).
    p            Top-p mass threshold; p >= 1 selects every key block.
    block        tokens per block (the pages use 32 or 64; the library supports 64).
    force_diag   always keep key block i for query block i.
    local_window w > 0 forces the band |i - j| <= w (wzjinhao notes §5.2 "邻近块保底").
    frame_len    tokens per frame (0: no frame structure).
    topk_frames  k for frame mode.
    topk_blocks  k for "topk" mode.
    frame_window fw >= 0 forces the frames within +-fw of the query's frames; < 0 disables.
    force_first_frame  always keep the blocks of frame 0.
    scale        softmax scale; None means 1/sqrt(d).
    sasa_coef    augmentation coefficient in [0, 1] of slack-aware sparse augmentation
                 (sasa_tile_augment); 0 disables it. Top-p and "topk" modes only.
    sasa_trigger smallest slack, in key blocks, at which a row is augmented.
    frame_exact  frame mode: attention is token-exact (frame_token_mask) instead of over whole
                 key blocks.
    """
    mode: str = "topp"
    p: float = 0.9
    block: int = 64
    force_diag: bool = True
    local_window: int = 0
    frame_len: int = 0
    topk_frames: int = 0
    topk_blocks: int = 0
    frame_window: int = -1
    force_first_frame: bool = False
    scale: Optional[float] = None
    sasa_coef: float = 0.0
    sasa_trigger: int = 1
    frame_exact: bool = False


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):          # a torch tensor: bf16/fp32 -> fp64 is exact
        x = x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def pool_blocks(X, block: int) -> np.ndarray:
    """Mean of each block of `block` consecutive tokens, over the valid tokens only.

    X: [BH, S, d]. Returns [BH, nb, d], nb = ceil(S / block). The last block, when S is not a
    multiple of `block`, averages its S - (nb-1)*block real tokens (wzjinhao notes §5.2 pools
    block means; padding tokens are not data, so they are not averaged in).
    """
    X = _f64(X)
    BH, S, d = X.shape
    nb = -(-S // block)
    out = np.empty((BH, nb, d), dtype=np.float64)
    for i in range(nb):
        lo, hi = i * block, min(S, (i + 1) * block)
        out[:, i, :] = X[:, lo:hi, :].sum(axis=1) / (hi - lo)
    return out


def pool_frames(X, frame_len: int) -> np.ndarray:
    """Mean of each frame's tokens (Sol-Attn §2.1: a frame is represented by the average
    pool of its patch tokens). X: [BH, S, d] -> [BH, F, d]."""
    X = _f64(X)
    BH, S, d = X.shape
    F = -(-S // frame_len)
    out = np.empty((BH, F, d), dtype=np.float64)
    for f in range(F):
        lo, hi = f * frame_len, min(S, (f + 1) * frame_len)
        out[:, f, :] = X[:, lo:hi, :].sum(axis=1) / (hi - lo)
    return out


def block_scores(qbar: np.ndarray, kbar: np.ndarray, scale: float) -> np.ndarray:
    """Sc[bh, i, j] = <qbar[bh, i], kbar[bh, j]> * scale (wzjinhao notes §5.2: einsum of
    the block means divided by sqrt(d))."""
    return np.matmul(qbar, np.swapaxes(kbar, -1, -2)) * scale


def row_softmax(sc: np.ndarray) -> np.ndarray:
    """Softmax over the key-block axis: the distribution whose cumulative mass the Top-p
    cut compares with p."""
    m = sc.max(axis=-1, keepdims=True)
    e = np.exp(sc - m)
    return e / e.sum(axis=-1, keepdims=True)


def topp_row(pi: np.ndarray, p: float):
    """Top-p cut of one row (FVAttn summary, "AI视频生成的阿喀琉斯之踵": sort blocks by
    importance, descending, and take them in turn until the cumulative importance reaches p).

    Ties in pi go to the lower block index. Returns (order, k_star, csum): `order` is the
    descending order, `csum[k-1]` the mass of the first k blocks, and the selection is
    order[:k_star] with k_star the smallest k whose mass is >= p (all blocks when p >= 1 or
    when rounding keeps the total just under p).
    """
    nb = pi.shape[0]
    order = np.argsort(-pi, kind="stable")
    csum = np.cumsum(pi[order])
    if p >= 1.0:
        return order, nb, csum
    reach = np.nonzero(csum >= p)[0]
    k_star = int(reach[0]) + 1 if reach.size else nb
    return order, k_star, csum


def topk_row(sc: np.ndarray, k: int) -> np.ndarray:
    """The k highest block scores of one row (wzjinhao notes §5.2: scores.topk(topk_blocks));
    ties go to the lower block index. Returns the kept indices in descending score order."""
    order = np.argsort(-sc, kind="stable")
    return order[:min(k, sc.shape[0])]


def _frames_of_block(j: int, S: int, block: int, frame_len: int):
    lo = j * block
    hi = min(S, (j + 1) * block) - 1
    return lo // frame_len, hi // frame_len


def frame_incidence(S: int, block: int, frame_len: int) -> np.ndarray:
    """Boolean [F, nb]: entry (f, j) is true when key block j holds a valid token of frame f."""
    nb = -(-S // block)
    F = -(-S // frame_len)
    inc = np.zeros((F, nb), dtype=bool)
    for j in range(nb):
        f0, f1 = _frames_of_block(j, S, block, frame_len)
        inc[f0:f1 + 1, j] = True
    return inc


def _blocks_touching_frames(frames_sel: np.ndarray, inc: np.ndarray) -> np.ndarray:
    """Key blocks whose valid tokens intersect any selected frame (boolean [nb])."""
    return inc[np.asarray(frames_sel, dtype=bool)].any(axis=0)


def forced_blocks(S: int, cfg: RouteCfg) -> np.ndarray:
    """Mandatory key blocks for every query block, boolean [nb, nb] (same for all heads).

    Union of: the diagonal; the band |i-j| <= local_window (wzjinhao notes §5.2); the blocks
    of the frames within +-frame_window of the query block's frames, and of frame 0
    (Sol-Attn §2.2: neighbouring frames and the first frame are always kept).
    """
    bs = cfg.block
    nb = -(-S // bs)
    forced = np.zeros((nb, nb), dtype=bool)
    inc = frame_incidence(S, bs, cfg.frame_len) if cfg.frame_len > 0 else None
    for i in range(nb):
        if cfg.force_diag:
            forced[i, i] = True
        if cfg.local_window > 0:
            lo, hi = max(0, i - cfg.local_window), min(nb - 1, i + cfg.local_window)
            forced[i, lo:hi + 1] = True
        if cfg.frame_len > 0 and (cfg.frame_window >= 0 or cfg.force_first_frame):
            F = -(-S // cfg.frame_len)
            fsel = np.zeros(F, dtype=bool)
            f0, f1 = _frames_of_block(i, S, bs, cfg.frame_len)
            if cfg.frame_window >= 0:
                fsel[max(0, f0 - cfg.frame_window):min(F - 1, f1 + cfg.frame_window) + 1] = True
            if cfg.force_first_frame:
                fsel[0] = True
            forced[i] |= _blocks_touching_frames(fsel, inc)
    return forced


def frame_topk_select(qf: np.ndarray, kf: np.ndarray, S: int, cfg: RouteCfg, scale: float):
    """Frame-level top-k (Sol-Attn §2.1/§2.2): score every key frame against each query
    frame with the frame means, keep the k best (ties to the lower frame index), and expand
    to key blocks. A query block takes the union over the frames its tokens touch.

    qf, kf: [BH, F, d]. Returns (mask [BH, nb, nb] bool without forcing, frame_scores
    [BH, F, F], chosen [BH, F, F] bool).
    """
    BH, F, _ = qf.shape
    bs = cfg.block
    nb = -(-S // bs)
    fs = np.matmul(qf, np.swapaxes(kf, -1, -2)) * scale
    k = min(cfg.topk_frames, F)
    chosen = np.zeros((BH, F, F), dtype=bool)
    for bh in range(BH):
        for f in range(F):
            order = np.argsort(-fs[bh, f], kind="stable")
            chosen[bh, f, order[:k]] = True
    inc = frame_incidence(S, bs, cfg.frame_len)
    mask = np.zeros((BH, nb, nb), dtype=bool)
    for bh in range(BH):
        for i in range(nb):
            f0, f1 = _frames_of_block(i, S, bs, cfg.frame_len)
            fsel = chosen[bh, f0:f1 + 1].any(axis=0)
            mask[bh, i] = _blocks_touching_frames(fsel, inc)
    return mask, fs, chosen


def route(Q, K, cfg: RouteCfg):
    """The whole router on [BH, S, d] inputs. Returns a dict with
    mask [BH, nb, nb] (the final selection: routed set union forced set), routed (the set
    before forcing), forced [nb, nb], pi or frame scores, and near_tie [BH, nb]."""
    Q = _f64(Q)
    K = _f64(K)
    BH, S, d = Q.shape
    bs = cfg.block
    nb = -(-S // bs)
    scale = cfg.scale if cfg.scale is not None else 1.0 / math.sqrt(d)
    forced = forced_blocks(S, cfg)
    out = {"forced": forced, "nb": nb, "scale": scale}
    if cfg.mode == "topp":
        qbar, kbar = pool_blocks(Q, bs), pool_blocks(K, bs)
        pi = row_softmax(block_scores(qbar, kbar, scale))
        routed = np.zeros((BH, nb, nb), dtype=bool)
        kstar = np.zeros((BH, nb), dtype=np.int64)
        for bh in range(BH):
            for i in range(nb):
                order, ks, _ = topp_row(pi[bh, i], cfg.p)
                routed[bh, i, order[:ks]] = True
                kstar[bh, i] = ks
        out.update(pi=pi, kstar=kstar, qbar=qbar, kbar=kbar)
    elif cfg.mode == "topk":
        qbar, kbar = pool_blocks(Q, bs), pool_blocks(K, bs)
        sc = block_scores(qbar, kbar, scale)
        routed = np.zeros((BH, nb, nb), dtype=bool)
        for bh in range(BH):
            for i in range(nb):
                routed[bh, i, topk_row(sc[bh, i], cfg.topk_blocks)] = True
        out.update(scores=sc, qbar=qbar, kbar=kbar)
    elif cfg.mode == "frame_topk":
        qf, kf = pool_frames(Q, cfg.frame_len), pool_frames(K, cfg.frame_len)
        routed, fs, chosen = frame_topk_select(qf, kf, S, cfg, scale)
        out.update(frame_scores=fs, chosen=chosen)
        if cfg.frame_exact:
            out["frame_sets"] = np.stack([frame_sets(chosen[bh], cfg) for bh in range(BH)])
    else:
        raise ValueError(cfg.mode)
    out["routed"] = routed
    out["mask"] = routed | forced[None]
    out["near_tie"] = near_tie_rows(out, S, cfg)
    if cfg.sasa_coef > 0.0:
        if cfg.mode == "frame_topk":
            raise ValueError("slack-aware augmentation needs a per-block order (topp or topk mode)")
        key = out["pi"] if cfg.mode == "topp" else out["scores"]
        base = out["mask"]
        out["base_mask"] = base
        out["mask"] = sasa_tile_augment(base, key, cfg.sasa_coef, cfg.sasa_trigger)
        tie = out["near_tie"] | sasa_near_tie_rows(base, key, cfg.sasa_coef, cfg.sasa_trigger, cfg.mode)
        # a tile's augmentation reads both rows' sets, so a tie in either row reaches both
        partner = tie.copy()
        partner[:, 0:nb - nb % 2:2] |= tie[:, 1:nb - nb % 2 + 1:2]
        partner[:, 1::2] |= tie[:, 0:nb - nb % 2:2]
        out["base_near_tie"] = out["near_tie"]
        out["near_tie"] = partner
    return out


def _sasa_budget(coef: float, slack: int, trigger: int) -> int:
    """Blocks added to a row with `slack` free key-block steps: floor(coef * slack) once the
    slack reaches the trigger. coef is taken at float32 precision (the configuration's type)
    and the product formed in float64, where it is exact."""
    if slack <= 0 or slack < trigger:
        return 0
    return int(math.floor(float(np.float32(coef)) * slack))


def _sasa_candidates(mask_bh: np.ndarray, r: int):
    """Candidates of row r of one head: key blocks of its tile's union that r did not select
    (the tile's rows are query blocks 2t and 2t+1). None for a row without a partner."""
    nb = mask_bh.shape[0]
    partner = r ^ 1
    if partner >= nb:
        return None
    union = mask_bh[r] | mask_bh[partner]
    return np.nonzero(union & ~mask_bh[r])[0]


def sasa_tile_augment(mask: np.ndarray, key: np.ndarray, coef: float, trigger: int) -> np.ndarray:
    """Slack-aware sparse augmentation (FVAttn summary, section "SASA") on one GPU.

    The pages' slack is the idle time a rank would spend at a synchronisation point; SASA fills
    it, up to a budget set by an augmentation coefficient and a trigger threshold, with the
    highest-importance blocks that routing left out, reusing routing's importance order and
    never lengthening the critical path. On one GPU the synchronous unit is the 128-row
    attention tile: query blocks 2t and 2t+1 step through the union of their key blocks
    together, so a row's slack is the number of union blocks it did not select, and filling it
    costs no extra tile step. Row r with slack s >= trigger gains the floor(coef * s)
    candidates ranked highest by `key` (pi in Top-p mode, the block score in top-k mode; ties
    to the lower block index). Both rows are augmented from the sets before augmentation; the
    union, hence the tile's cost, is unchanged.

    mask [BH, nb, nb] bool (routed set union forced set), key [BH, nb, nb]. Returns a new mask.
    """
    out = mask.copy()
    BH, nb, _ = mask.shape
    for bh in range(BH):
        for r in range(nb):
            cand = _sasa_candidates(mask[bh], r)
            if cand is None:
                continue
            n = _sasa_budget(coef, cand.size, trigger)
            if n == 0:
                continue
            ranked = cand[np.argsort(-key[bh, r, cand], kind="stable")]
            out[bh, r, ranked[:n]] = True
    return out


def _gap_eps(v: float, mode: str) -> float:
    return EPS_GAP if mode == "topp" else EPS_GAP * max(1.0, abs(v))


def sasa_near_tie_rows(mask: np.ndarray, key: np.ndarray, coef: float, trigger: int, mode: str) -> np.ndarray:
    """Rows whose augmentation is decided by a key gap below the stated resolution: the last
    candidate added and the first one left out differ by less than EPS_GAP (in pi; in top-k
    mode relative to the score)."""
    BH, nb, _ = mask.shape
    near = np.zeros((BH, nb), dtype=bool)
    for bh in range(BH):
        for r in range(nb):
            cand = _sasa_candidates(mask[bh], r)
            if cand is None:
                continue
            n = _sasa_budget(coef, cand.size, trigger)
            if n == 0 or n >= cand.size:
                continue
            srt = np.sort(key[bh, r, cand])[::-1]
            near[bh, r] = (srt[n - 1] - srt[n]) < _gap_eps(srt[n - 1], mode)
    return near


def valid_sasa_row(key_row: np.ndarray, base_row: np.ndarray, partner_row: np.ndarray, final_row: np.ndarray,
                   coef: float, trigger: int, mode: str) -> bool:
    """Is `final_row` an acceptable augmentation of `base_row` (its tile partner's set
    `partner_row`) when the choice is a near-tie? It must keep the base set, add exactly the
    budget from the candidates only, and add no candidate ranked clearly below one it left out."""
    base_row, partner_row, final_row = (np.asarray(x, dtype=bool) for x in (base_row, partner_row, final_row))
    if np.any(base_row & ~final_row):
        return False
    cand_mask = (base_row | partner_row) & ~base_row
    added = final_row & ~base_row
    if np.any(added & ~cand_mask):
        return False
    n = _sasa_budget(coef, int(cand_mask.sum()), trigger)
    if int(added.sum()) != n:
        return False
    left = cand_mask & ~added
    if n == 0 or not left.any():
        return True
    lo_added = key_row[added].min()
    hi_left = key_row[left].max()
    return bool(lo_added >= hi_left - _gap_eps(lo_added, mode))


def near_tie_rows(r: dict, S: int, cfg: RouteCfg) -> np.ndarray:
    """Rows whose selection is decided by a difference below the stated resolution:
    a cumulative mass within EPS_MASS of p at the cut (k* or k*-1 blocks), or a probability
    gap under EPS_GAP between the last block kept and the first block left out. Top-k mode: a
    gap under EPS_GAP * max(1, |s|) between the k-th and the (k+1)-th score s (the scores are
    unnormalised logits, whose rounding grows with their magnitude). Frame mode: a frame-score
    gap under EPS_GAP at the top-k boundary of any frame the row touches."""
    mask = r["mask"]
    BH, nb, _ = mask.shape
    near = np.zeros((BH, nb), dtype=bool)
    if cfg.mode == "topk":
        k = min(cfg.topk_blocks, nb)
        if k >= nb:
            return near
        for bh in range(BH):
            for i in range(nb):
                srt = np.sort(r["scores"][bh, i])[::-1]
                near[bh, i] = (srt[k - 1] - srt[k]) < _gap_eps(srt[k - 1], "topk")
        return near
    if cfg.mode == "topp":
        if cfg.p >= 1.0:
            return near
        pi = r["pi"]
        for bh in range(BH):
            for i in range(nb):
                order, ks, csum = topp_row(pi[bh, i], cfg.p)
                srt = pi[bh, i][order]
                t = abs(csum[ks - 1] - cfg.p) < EPS_MASS
                if ks >= 2:
                    t |= abs(csum[ks - 2] - cfg.p) < EPS_MASS
                if ks < srt.shape[0]:
                    t |= (srt[ks - 1] - srt[ks]) < EPS_GAP
                near[bh, i] = t
        return near
    fs = r["frame_scores"]
    F = fs.shape[1]
    k = min(cfg.topk_frames, F)
    ftie = np.zeros((BH, F), dtype=bool)
    if k < F:
        for bh in range(BH):
            for f in range(F):
                srt = np.sort(fs[bh, f])[::-1]
                ftie[bh, f] = (srt[k - 1] - srt[k]) < EPS_GAP
    for i in range(nb):
        f0, f1 = _frames_of_block(i, S, cfg.block, cfg.frame_len)
        near[:, i] = ftie[:, f0:f1 + 1].any(axis=1)
    return near


def _kept_sets(scores: np.ndarray, k: int, eps: float):
    """Every set of k indices that the top-k rule can keep when scores closer than `eps` are
    taken as tied. With hi the k-th and lo the (k+1)-th highest score, an index is ranked
    clearly inside when its score is at least lo + eps (no tie with anything left out) and
    clearly outside when it is at most hi - eps; the set is the clearly-inside indices plus any
    choice of the rest. When hi - lo >= eps this is the top-k set alone. Yields boolean masks."""
    n = scores.shape[0]
    k = min(k, n)
    srt = np.sort(scores)[::-1]
    hi_cut = srt[k - 1]
    lo_cut = srt[k] if k < n else -np.inf
    must = (scores - lo_cut) >= eps
    band = ~must & ((hi_cut - scores) < eps)
    need = k - int(must.sum())
    for pick in itertools.combinations(np.nonzero(band)[0].tolist(), need):
        m = must.copy()
        m[list(pick)] = True
        yield m


def valid_near_tie_set(r: dict, bh: int, i: int, gpu_row: np.ndarray, S: int, cfg: RouteCfg) -> bool:
    """Is `gpu_row` (boolean [nb]) an acceptable selection for a near-tie row?

    A near-tie row's selection may differ from the oracle's only by the order of scores closer
    than the stated resolution (a gap under EPS_GAP, in probability units for Top-p, relative
    to the score in top-k mode, absolute for frame scores). So `gpu_row` must hold every forced
    block and be the forced set united with a selection the rule could make under such a
    reordering. Top-p: every block ranked clearly above the cut kept, none clearly below, and
    a kept mass of at least p - EPS_MASS. Top-k: exactly k routed blocks, chosen as in
    _kept_sets. Frame mode: per touched query frame exactly k key frames, chosen as in
    _kept_sets, united over the frames the query block touches and expanded to key blocks."""
    forced = r["forced"][i]
    gpu_row = np.asarray(gpu_row, dtype=bool)
    if np.any(forced & ~gpu_row):
        return False
    if cfg.mode == "topk":
        sc = r["scores"][bh, i]
        k = min(cfg.topk_blocks, sc.shape[0])
        eps = _gap_eps(np.sort(sc)[::-1][k - 1], "topk")
        return any(np.array_equal(m | forced, gpu_row) for m in _kept_sets(sc, k, eps))
    if cfg.mode == "topp":
        pi = r["pi"][bh, i]
        order, ks, csum = topp_row(pi, cfg.p)
        srt = pi[order]
        hi_cut = srt[ks - 1]
        lo_cut = srt[ks] if ks < pi.shape[0] else -np.inf
        must = ((pi - hi_cut) >= EPS_GAP) | forced
        may = ((lo_cut - pi) < EPS_GAP) | forced
        if pi[gpu_row].sum() < cfg.p - EPS_MASS:
            return False
        return bool(np.all(gpu_row[must]) and not np.any(gpu_row & ~may))
    fs = r["frame_scores"][bh]
    F = fs.shape[0]
    k = min(cfg.topk_frames, F)
    f0, f1 = _frames_of_block(i, S, cfg.block, cfg.frame_len)
    inc = frame_incidence(S, cfg.block, cfg.frame_len)
    options = [list(_kept_sets(fs[f], k, EPS_GAP)) for f in range(f0, f1 + 1)]
    if math.prod(len(o) for o in options) > 200_000:
        raise ValueError("too many tied frame choices to enumerate")
    for combo in itertools.product(*options):
        sel = np.logical_or.reduce(combo)
        if np.array_equal(_blocks_touching_frames(sel, inc) | forced, gpu_row):
            return True
    return False


# ---------------------------------------------------------------- token-exact frame selection

def frame_sets(chosen_bh: np.ndarray, cfg: RouteCfg) -> np.ndarray:
    """G [F, F] bool for one head: key frames a query token of frame f may attend in the
    token-exact frame mode: its top-k frames (Sol-Attn §2.1), the frames within +-frame_window
    of f (§2.2, neighbouring frames) and frame 0 when force_first_frame (§5.2)."""
    F = chosen_bh.shape[0]
    G = chosen_bh.astype(bool).copy()
    for f in range(F):
        if cfg.frame_window >= 0:
            G[f, max(0, f - cfg.frame_window):min(F - 1, f + cfg.frame_window) + 1] = True
        if cfg.force_first_frame:
            G[f, 0] = True
    return G


def block_forced(S: int, cfg: RouteCfg) -> np.ndarray:
    """[nb, nb] bool: the block-level forced blocks (diagonal, band |i-j| <= local_window)."""
    nb = -(-S // cfg.block)
    out = np.zeros((nb, nb), dtype=bool)
    for i in range(nb):
        if cfg.force_diag:
            out[i, i] = True
        if cfg.local_window > 0:
            out[i, max(0, i - cfg.local_window):min(nb - 1, i + cfg.local_window) + 1] = True
    return out


def frame_token_mask(G: np.ndarray, S: int, cfg: RouteCfg) -> np.ndarray:
    """[S, S] bool for one head, token-exact frame mode: query token t may attend key token u
    when frame(u) is in G[frame(t)], or when u's key block is a block-level forced block of t's
    query block (those are kept whole)."""
    fl, bs = cfg.frame_len, cfg.block
    fr = np.arange(S) // fl
    allowed = G[fr][:, fr]
    bf = block_forced(S, cfg)
    blk = np.arange(S) // bs
    return allowed | bf[blk][:, blk]


def frame_entry_code(G: np.ndarray, bf: np.ndarray, i: int, j: int, S: int, cfg: RouteCfg) -> int:
    """The 32-bit code of CSR entry (query block i, key block j) in token-exact frame mode:
    bits 0-3 allow[a][b] at bit 2a+b (a: the query block's first (0) or second (1) frame, b the
    same for the key block; a block spans at most two frames since frames are >= 64 tokens),
    bits 8-15 the first column of the key block's second frame (64 when it has one frame), bits
    16-23 the first row of the query block's second frame (64 likewise). A block-level forced
    entry allows all four."""
    fl, bs = cfg.frame_len, cfg.block
    qa, qb = _frames_of_block(i, S, bs, fl)
    ka, kb = _frames_of_block(j, S, bs, fl)
    qf, kf = (qa, qb), (ka, kb)
    bits = 0
    for a in range(2):
        for b in range(2):
            if bf[i, j] or G[qf[a], kf[b]]:
                bits |= 1 << (2 * a + b)
    kcol = kb * fl - j * bs if kb != ka else bs
    qrow = qb * fl - i * bs if qb != qa else bs
    return bits | (kcol << 8) | (qrow << 16)
