"""Pins of the oracle's near-tie rules and of frame top-k on frames that are not whole blocks.

The near-tie rules decide which differences between the GPU's selection and the oracle's are
excused, so each branch is pinned by hand-made rows on both sides of its resolution: Top-p
gaps in probability units, top-k gaps relative to the score (EPS_GAP * max(1, |s|)), frame
gaps absolute. A gap of exactly EPS_GAP is not a tie (ties are gaps *under* the resolution).
Frame top-k is pinned by hand-worked cases in which a query block straddles two frames whose
kept sets differ, so the block's row is their union. CPU only."""
import json
import os

import numpy as np
import pytest

import oracle
from oracle.route import EPS_GAP, frame_incidence

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")

# 2^-19 and 2^-19 - EPS_GAP differ by exactly EPS_GAP in fp64 (both are multiples of 2^-72).
A_EXACT = 2.0 ** -19
B_EXACT = A_EXACT - EPS_GAP
assert A_EXACT - B_EXACT == EPS_GAP


def _topk_r(row, forced=None):
    """A one-head router result whose nb query blocks all have the score row `row`."""
    row = np.asarray(row, dtype=np.float64)
    nb = row.shape[0]
    f = np.zeros((nb, nb), bool)
    if forced is not None:
        f[:] = np.asarray(forced, bool)
    return {"scores": np.tile(row, (1, nb, 1)), "mask": np.zeros((1, nb, nb), bool), "forced": f}


def _near_topk(rows, k):
    cfg = oracle.RouteCfg(mode="topk", topk_blocks=k)
    return np.array([oracle.near_tie_rows(_topk_r(row), 64 * len(row), cfg)[0, 0] for row in rows])


def _valid_topk(row, k, sel, forced=None):
    nb = len(row)
    gpu = np.zeros(nb, bool)
    gpu[list(sel)] = True
    return oracle.valid_near_tie_set(_topk_r(row, forced), 0, 0, gpu, 64 * nb,
                                     oracle.RouteCfg(mode="topk", topk_blocks=k))


# ---------------------------------------------------------------- top-k branch

def test_topk_near_tie_gap_is_relative_to_the_score():
    # |s| = 200: the resolution is 2e-4. A gap of 1.5e-4 is a tie (it would not be under an
    # absolute 1e-6); a gap of 3e-4 is not.
    near = _near_topk([[300.0, 200.0 + 1.5e-4, 200.0, 0.0], [300.0, 200.0 + 3e-4, 200.0, 0.0]], 2)
    assert near.tolist() == [True, False]


def test_topk_near_tie_gap_has_a_floor_of_one():
    # |s| < 1: the resolution is EPS_GAP itself (not EPS_GAP * |s|).
    near = _near_topk([[0.3, 0.2 + 0.5e-6, 0.2, 0.0], [0.3, 0.2 + 2e-6, 0.2, 0.0]], 2)
    assert near.tolist() == [True, False]


def test_topk_near_tie_exact_resolution_is_not_a_tie():
    near = _near_topk([[0.5, A_EXACT, B_EXACT, 0.0], [0.5, A_EXACT, A_EXACT, 0.0]], 2)
    assert near.tolist() == [False, True]            # gap == EPS_GAP: no tie; gap 0: tie


def test_topk_near_tie_k_at_least_nb_has_no_ties():
    assert not _near_topk([[1.0, 1.0, 1.0, 1.0]], 4).any()
    assert not _near_topk([[1.0, 1.0, 1.0, 1.0]], 9).any()


def test_topk_valid_set_relative_band():
    row = [300.0, 200.0 + 1.5e-4, 200.0, 0.0]
    assert _valid_topk(row, 2, {0, 1})
    assert _valid_topk(row, 2, {0, 2})                  # within 2e-4 of the cut
    assert not _valid_topk(row, 2, {0, 1, 2})           # k = 2 blocks, not 3
    assert not _valid_topk(row, 2, {1, 2})              # drops the block clearly above
    assert not _valid_topk(row, 2, {0, 3})              # takes a block clearly below
    assert not _valid_topk(row, 2, {0})
    far = [300.0, 200.0 + 3e-4, 200.0, 0.0]
    assert _valid_topk(far, 2, {0, 1}) and not _valid_topk(far, 2, {0, 2})


def test_topk_valid_set_small_scores_and_exact_resolution():
    assert _valid_topk([0.3, 0.2 + 0.5e-6, 0.2, 0.0], 2, {0, 2})
    assert not _valid_topk([0.3, 0.2 + 2e-6, 0.2, 0.0], 2, {0, 2})
    # k = 1 with A - B == EPS_GAP exactly: not a tie, so only A is a valid choice
    row = [A_EXACT, B_EXACT, 0.0]
    assert _valid_topk(row, 1, {0}) and not _valid_topk(row, 1, {1})
    # k = 2, the 2nd (X) and 3rd (B) scores tied, A - B == EPS_GAP exactly while A - X is
    # under it: A is clear of everything left out, so it stays; X and B are interchangeable
    X = B_EXACT + 0.25 * EPS_GAP
    row = [A_EXACT, X, B_EXACT]
    assert _valid_topk(row, 2, {0, 1}) and _valid_topk(row, 2, {0, 2})
    assert not _valid_topk(row, 2, {1, 2})
    # B and C tied for the second place, A clear of both
    row = [A_EXACT + EPS_GAP, B_EXACT, B_EXACT - 0.25 * EPS_GAP]
    assert _valid_topk(row, 2, {0, 1}) and _valid_topk(row, 2, {0, 2})
    assert not _valid_topk(row, 2, {1, 2})


def test_topk_valid_set_keeps_an_untied_kth_block():
    # scores 5 > 2 > 1 > 0, k = 2: no ties, only the top-2 set is valid
    row = [0.0, 1.0, 2.0, 5.0]
    assert _valid_topk(row, 2, {2, 3})
    assert not _valid_topk(row, 2, {1, 3}) and not _valid_topk(row, 2, {0, 3})


def test_topk_valid_set_with_forced_blocks():
    row = [300.0, 200.0 + 1.5e-4, 200.0, 0.0]
    assert _valid_topk(row, 2, {0, 1, 3}, forced=[0, 0, 0, 1])
    assert _valid_topk(row, 2, {0, 2, 3}, forced=[0, 0, 0, 1])
    assert not _valid_topk(row, 2, {0, 1, 2, 3}, forced=[0, 0, 0, 1])
    assert not _valid_topk(row, 2, {0, 1}, forced=[0, 0, 0, 1])          # forced block missing
    # a forced block inside the tie band may also be one of the k routed blocks
    assert _valid_topk(row, 2, {0, 2}, forced=[0, 0, 1, 0])
    assert _valid_topk(row, 2, {0, 1, 2}, forced=[0, 0, 1, 0])
    assert not _valid_topk(row, 2, {0, 2, 3}, forced=[0, 0, 1, 0])


def test_topk_valid_set_tie_at_the_kth_score():
    row = [3.0, 2.0, 2.0, 0.0]
    assert _near_topk([row], 2)[0]
    assert _valid_topk(row, 2, {0, 1}) and _valid_topk(row, 2, {0, 2})
    assert not _valid_topk(row, 2, {1, 2})


# ---------------------------------------------------------------- frame branch

# S = 300 tokens, frames of 100 (F = 3), 5 blocks; blocks 1 (tokens 64-127) and 3 (192-255)
# straddle frames 0|1 and 1|2. Frame of each block: 0: {0}, 1: {0,1}, 2: {1}, 3: {1,2}, 4: {2}.
# Key blocks of each frame: 0 -> {0,1}, 1 -> {1,2,3}, 2 -> {3,4}.
FRAME_CFG = oracle.RouteCfg(mode="frame_topk", topk_frames=1, frame_len=100, force_diag=False)


def _frame_r(fs):
    return {"frame_scores": np.asarray(fs, np.float64)[None], "mask": np.zeros((1, 5, 5), bool),
            "forced": np.zeros((5, 5), bool)}


def _valid_frame(fs, i, sel):
    gpu = np.zeros(5, bool)
    gpu[list(sel)] = True
    return oracle.valid_near_tie_set(_frame_r(fs), 0, i, gpu, 300, FRAME_CFG)


TIE_IN_LAST_FRAME = [[5.0, 1.0, 0.0], [0.0, 3.0, 1.0], [2.0 + 0.5e-6, 2.0, 0.0]]


def test_frame_near_tie_reaches_every_block_of_the_tied_frame():
    near = oracle.near_tie_rows(_frame_r(TIE_IN_LAST_FRAME), 300, FRAME_CFG)[0]
    # frame 2 is tied; block 3 touches it as its second frame
    assert near.tolist() == [False, False, False, True, True]


def test_frame_near_tie_gap_is_absolute():
    over = [[5.0, 1.0, 0.0], [0.0, 3.0, 1.0], [2.0 + 2e-6, 2.0, 0.0]]
    assert not oracle.near_tie_rows(_frame_r(over), 300, FRAME_CFG).any()
    big = [[5.0, 1.0, 0.0], [0.0, 3.0, 1.0], [200.0 + 1.5e-4, 200.0, 0.0]]
    assert not oracle.near_tie_rows(_frame_r(big), 300, FRAME_CFG).any()   # no relative band here
    exact = [[5.0, 1.0, 0.0], [0.0, 3.0, 1.0], [A_EXACT, B_EXACT, 0.0]]
    assert not oracle.near_tie_rows(_frame_r(exact), 300, FRAME_CFG).any()


def test_frame_valid_set_single_frame_row():
    # block 4 touches frame 2 only: its top-1 frame is 0 (blocks {0,1}) or, tied, 1 ({1,2,3})
    assert _valid_frame(TIE_IN_LAST_FRAME, 4, {0, 1})
    assert _valid_frame(TIE_IN_LAST_FRAME, 4, {1, 2, 3})
    assert not _valid_frame(TIE_IN_LAST_FRAME, 4, {0, 1, 2, 3})        # two frames, k = 1
    assert not _valid_frame(TIE_IN_LAST_FRAME, 4, {3, 4})              # frame 2: clearly below


def test_frame_valid_set_straddling_row_takes_the_union():
    # block 3 touches frames 1 (top-1: frame 1, clear) and 2 (tied between frames 0 and 1)
    assert _valid_frame(TIE_IN_LAST_FRAME, 3, {0, 1, 2, 3})
    assert _valid_frame(TIE_IN_LAST_FRAME, 3, {1, 2, 3})
    assert not _valid_frame(TIE_IN_LAST_FRAME, 3, {0, 1})              # misses frame 1's pick


# ---------------------------------------------------------------- frame top-k on straddling blocks

def _straddle_inputs(c):
    S, fl = c["S"], c["frame_len"]
    qf = np.asarray(c["qf"], dtype=np.float64)
    F = qf.shape[0]
    fr = np.arange(S) // fl
    Q = qf[fr][None]                                    # [1, S, F]
    K = np.eye(F)[fr][None]
    return Q, K


def _cases():
    return json.load(open(os.path.join(GOLDEN, "frame_topk_straddle_cases.json")))["cases"]


@pytest.mark.parametrize("case", range(2))
def test_frame_topk_straddle_golden(case):
    c = _cases()[case]
    Q, K = _straddle_inputs(c)
    cfg = oracle.RouteCfg(mode="frame_topk", topk_frames=c["topk"], frame_len=c["frame_len"], force_diag=False,
                          scale=1.0)
    r = oracle.route(Q, K, cfg)
    rows = [np.nonzero(r["mask"][0, i])[0].tolist() for i in range(r["nb"])]
    assert rows == c["expect_rows"]
    # the straddling rows differ from what their first frame alone would give
    qf, kf = oracle.pool_frames(Q, c["frame_len"]), oracle.pool_frames(K, c["frame_len"])
    np.testing.assert_array_equal(qf[0], np.asarray(c["qf"], np.float64))
    _, fs, chosen = oracle.frame_topk_select(qf, kf, c["S"], cfg, 1.0)
    inc = frame_incidence(c["S"], 64, c["frame_len"])
    straddle = [i for i in range(r["nb"]) if (i * 64) // c["frame_len"] != (min(c["S"], i * 64 + 64) - 1) // c["frame_len"]]
    assert straddle
    for i in straddle:
        f0 = (i * 64) // c["frame_len"]
        first_only = inc[chosen[0, f0]].any(axis=0)
        assert not np.array_equal(first_only, r["mask"][0, i]), i


def test_frame_topk_straddle_near_tie_rows():
    # case 2: frames 1 and 2 tie for the second place of query frame 0, so the rows of the
    # blocks touching frame 0 (blocks 0 and 1) are near-ties and nothing else is
    c = _cases()[1]
    Q, K = _straddle_inputs(c)
    cfg = oracle.RouteCfg(mode="frame_topk", topk_frames=2, frame_len=100, force_diag=False, scale=1.0)
    r = oracle.route(Q, K, cfg)
    assert r["near_tie"][0].tolist() == [True, True, False, False, False]
    # block 0 may take frames {0, 2} instead of {0, 1}: blocks {0, 1, 3, 4}
    alt = np.zeros(5, bool)
    alt[[0, 1, 3, 4]] = True
    assert oracle.valid_near_tie_set(r, 0, 0, alt, 300, cfg)
    assert not oracle.valid_near_tie_set(r, 0, 0, np.ones(5, bool), 300, cfg)   # three frames
    # block 1's union is every block whichever tied frame frame 0 keeps
    assert oracle.valid_near_tie_set(r, 0, 1, np.ones(5, bool), 300, cfg)
    assert not oracle.valid_near_tie_set(r, 0, 1, alt, 300, cfg)
