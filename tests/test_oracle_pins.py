"""Pins of the CPU oracle to facts that do not come from the oracle itself: closed forms,
hand-computed golden cases, brute force over all subsets, invariants and a library
routine (torch's scaled_dot_product_attention). CPU only."""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from oracle.route import EPS_GAP, EPS_MASS
from workloads import get_workload, make_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------- pooling (closed forms)

def test_pool_ramp_closed_form_with_ragged_tail():
    # X[t, c] = t + 1000 c: the mean of tokens lo..hi-1 is (lo + hi - 1)/2 + 1000 c.
    S, d = 200, 3
    X = (np.arange(S)[:, None] + 1000.0 * np.arange(d)[None, :])[None]
    m = oracle.pool_blocks(X, 64)
    assert m.shape == (1, 4, d)
    for i, (lo, hi) in enumerate([(0, 64), (64, 128), (128, 192), (192, 200)]):
        np.testing.assert_array_equal(m[0, i], (lo + hi - 1) / 2 + 1000.0 * np.arange(d))


def test_pool_constant_blocks():
    S, d = 64 * 5, 8
    X = np.repeat(np.arange(5, dtype=np.float64), 64)[None, :, None] * np.ones((2, 1, d))
    np.testing.assert_array_equal(oracle.pool_blocks(X, 64)[1, :, 0], np.arange(5.0))


def test_pool_frames_closed_form():
    S, fl = 250, 100
    X = np.arange(S, dtype=np.float64)[None, :, None]
    m = oracle.pool_frames(X, fl)[0, :, 0]
    np.testing.assert_array_equal(m, [49.5, 149.5, 224.5])


# ---------------------------------------------------------------- scores and softmax

def test_block_scores_hand():
    q = np.zeros((1, 2, 4)); k = np.zeros((1, 3, 4))
    q[0, 0, 0] = 2.0; q[0, 1, 1] = -1.0
    k[0, 0, 0] = 3.0; k[0, 1, 1] = 5.0; k[0, 2] = 1.0
    sc = oracle.block_scores(q, k, 0.5)
    np.testing.assert_array_equal(sc[0], [[3.0, 0.0, 1.0], [0.0, -2.5, -0.5]])


def test_softmax_closed_form():
    pi = oracle.row_softmax(np.log(np.array([[1.0, 2.0, 3.0, 4.0], [1.0, 3.0, 0.0 + 1e-300, 4.0]])))
    np.testing.assert_allclose(pi[0], [0.1, 0.2, 0.3, 0.4], rtol=1e-15)
    np.testing.assert_allclose(pi[1], [0.125, 0.375, 0.0, 0.5], atol=1e-15)
    # shift invariance of the logits
    x = np.random.default_rng(0).normal(size=(3, 7)) * 50
    np.testing.assert_allclose(oracle.row_softmax(x), oracle.row_softmax(x + 1234.5), rtol=1e-12)


# ---------------------------------------------------------------- Top-p cut

def test_topp_golden_hand_cases():
    cases = json.load(open(os.path.join(GOLDEN, "topp_hand_cases.json")))["cases"]
    for c in cases:
        pi = oracle.row_softmax(np.log(np.array(c["w"], dtype=np.float64))[None])[0]
        order, ks, _ = oracle.topp_row(pi, c["p"])
        assert sorted(order[:ks].tolist()) == c["expect"], c


def _brute_force_min_set(pi, p):
    """Smallest cardinality of any subset with mass >= p, and the best mass at that size."""
    n = pi.shape[0]
    for k in range(1, n + 1):
        best = max(sum(pi[list(s)]) for s in itertools.combinations(range(n), k))
        if best >= p:
            return k, best
    return n, pi.sum()


@pytest.mark.parametrize("seed", range(6))
def test_topp_minimal_prefix_brute_force(seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(2, 11))
    pi = oracle.row_softmax(rng.normal(size=n) * rng.uniform(0.3, 3.0))
    for p in (0.2, 0.5, 0.8, 0.9, 0.97):
        order, ks, csum = oracle.topp_row(pi, p)
        kmin, best = _brute_force_min_set(pi, p)
        if abs(csum[ks - 1] - p) < 1e-12 or abs(best - p) < 1e-12:
            continue
        assert ks == kmin
        assert abs(pi[order[:ks]].sum() - best) < 1e-12     # the prefix is a best set of that size


def test_topp_degenerate_rows():
    nb = 16
    one_hot = np.zeros(nb); one_hot[5] = 1.0
    order, ks, _ = oracle.topp_row(one_hot, 0.9)
    assert ks == 1 and order[0] == 5
    uni = np.full(nb, 1.0 / nb)
    assert oracle.topp_row(uni, 0.5)[1] == nb // 2
    assert oracle.topp_row(uni, 1.0)[1] == nb
    assert oracle.topp_row(uni, 1e-9)[1] == 1


def test_topp_nested_in_p():
    rng = np.random.default_rng(7)
    pi = oracle.row_softmax(rng.normal(size=40) * 2.0)
    prev = set()
    for p in (0.1, 0.3, 0.5, 0.8, 0.9, 0.95, 0.99, 1.0):
        order, ks, _ = oracle.topp_row(pi, p)
        cur = set(order[:ks].tolist())
        assert prev <= cur
        prev = cur
    assert prev == set(range(40))


def test_near_tie_flags():
    cfg = oracle.RouteCfg(p=0.9)
    # cut exactly at p: masses .5 .4 .1 -> c_2 = .9 (within EPS_MASS of p)
    r = {"pi": np.array([[[0.5, 0.4, 0.1]]]), "mask": np.ones((1, 1, 3), bool), "forced": np.eye(1, 3, dtype=bool)}
    assert oracle.near_tie_rows(r, 64 * 3, cfg)[0, 0]
    # clear cut, no tie
    r["pi"] = np.array([[[0.7, 0.05, 0.25]]])
    assert not oracle.near_tie_rows(r, 64 * 3, cfg)[0, 0]
    # probability gap below EPS_GAP at the boundary
    r["pi"] = np.array([[[0.85, 0.075 + 0.4 * EPS_GAP, 0.075 - 0.4 * EPS_GAP]]])
    assert oracle.near_tie_rows(r, 64 * 3, cfg)[0, 0]


# ---------------------------------------------------------------- forced blocks

def test_forced_diag_and_band_hand():
    f = oracle.forced_blocks(6 * 64, oracle.RouteCfg(force_diag=True, local_window=1))
    expect = np.zeros((6, 6), bool)
    for i in range(6):
        for j in range(max(0, i - 1), min(5, i + 1) + 1):
            expect[i, j] = True
    np.testing.assert_array_equal(f, expect)
    f0 = oracle.forced_blocks(6 * 64 - 10, oracle.RouteCfg(force_diag=True))
    np.testing.assert_array_equal(f0, np.eye(6, dtype=bool))


def test_forced_frames_golden():
    cases = json.load(open(os.path.join(GOLDEN, "frame_hand_cases.json")))["cases"]
    for c in cases:
        cfg = oracle.RouteCfg(force_diag=False, frame_len=c["frame_len"], frame_window=c["frame_window"],
                              force_first_frame=c["first"])
        f = oracle.forced_blocks(c["S"], cfg)
        assert np.nonzero(f[c["query_block"]])[0].tolist() == c["expect_blocks"], c


# ---------------------------------------------------------------- whole router invariants

def _small(name="single", **kw):
    w = get_workload(name, **kw)
    x = make_inputs(w)
    BH = w.B * w.H
    return w, x["q"].reshape(BH, w.S, w.d), x["k"].reshape(BH, w.S, w.d), x["v"].reshape(BH, w.S, w.d)


def test_route_invariants_and_p1_dense():
    w, Q, K, _ = _small(H=3, S=1000, frame_len=500, region_len=128, seed=11)
    for cfg in (oracle.RouteCfg(p=0.8, force_diag=True), oracle.RouteCfg(p=0.5, force_diag=False, local_window=2),
                oracle.RouteCfg(p=0.7, force_diag=True, frame_len=500, frame_window=0, force_first_frame=True)):
        r = oracle.route(Q, K, cfg)
        m = r["mask"]
        assert m.shape == (3, 16, 16)
        assert (m.sum(axis=2) >= 1).all()
        assert (m | ~r["forced"][None]).all()                      # forced subset of selected
        np.testing.assert_array_equal(m, r["routed"] | r["forced"][None])
        # the routed part has mass >= p in every row
        mass = (r["pi"] * r["routed"]).sum(axis=2)
        assert (mass >= cfg.p - 1e-12).all()
    r1 = oracle.route(Q, K, oracle.RouteCfg(p=1.0, force_diag=False))
    assert r1["mask"].all()


def test_route_selection_nested_in_p():
    w, Q, K, _ = _small(H=2, S=768, frame_len=256, region_len=64, seed=3, alpha=("const", 0.7))
    prev = None
    for p in (0.5, 0.8, 0.9, 0.95, 0.99, 1.0):
        m = oracle.route(Q, K, oracle.RouteCfg(p=p, force_diag=True))["mask"]
        if prev is not None:
            assert (m | ~prev).all()
        prev = m


def test_frame_mode_topk_ge_frames_is_dense():
    w, Q, K, _ = _small(H=2, S=900, frame_len=300, region_len=100, seed=5)
    r = oracle.route(Q, K, oracle.RouteCfg(mode="frame_topk", topk_frames=3, frame_len=300, force_diag=False))
    assert r["mask"].all()


def test_frame_mode_aligned_direct_construction():
    # Frames of 128 tokens = 2 blocks each: a key block is selected iff its frame is one of
    # the k frames whose mean key scores highest against the query block's frame mean.
    w, Q, K, _ = _small(H=2, S=1024, frame_len=128, region_len=64, seed=9)
    cfg = oracle.RouteCfg(mode="frame_topk", topk_frames=2, frame_len=128, force_diag=False)
    r = oracle.route(Q, K, cfg)
    Qd, Kd = Q.double().numpy(), K.double().numpy()
    F, nb = 8, 16
    for bh in range(2):
        qm = [Qd[bh, f * 128:(f + 1) * 128].mean(axis=0) for f in range(F)]
        km = [Kd[bh, f * 128:(f + 1) * 128].mean(axis=0) for f in range(F)]
        for i in range(nb):
            f = i // 2
            s = [float(np.dot(qm[f], km[g])) for g in range(F)]
            top = sorted(range(F), key=lambda g: (-s[g], g))[:2]
            expect = np.array([(j // 2) in top for j in range(nb)])
            np.testing.assert_array_equal(r["mask"][bh, i], expect)


def test_valid_near_tie_set_accepts_neighbours_and_rejects_far():
    cfg = oracle.RouteCfg(p=0.9, force_diag=True)
    pi = np.array([0.5, 0.4 + 2e-6, 0.1 - 2e-6, 0.0])
    r = {"pi": pi[None, None], "forced": np.eye(4, dtype=bool)[:1], "mask": None}
    assert oracle.valid_near_tie_set(r, 0, 0, np.array([1, 1, 0, 0], bool), 256, cfg)
    assert oracle.valid_near_tie_set(r, 0, 0, np.array([1, 1, 1, 0], bool), 256, cfg)
    assert not oracle.valid_near_tie_set(r, 0, 0, np.array([1, 0, 1, 0], bool), 256, cfg)
    assert not oracle.valid_near_tie_set(r, 0, 0, np.array([0, 1, 1, 0], bool), 256, cfg)


# ---------------------------------------------------------------- attention

def test_attention_full_coverage_equals_dense_sdpa():
    # The pages' own check (wzjinhao notes §5.3): b,h,l,d = 2,4,512,64, fp32, full coverage
    # must equal dense attention to max-abs < 1e-4.
    g = torch.Generator().manual_seed(0)
    q, k, v = (torch.randn(8, 512, 64, generator=g) for _ in range(3))
    mask = np.ones((8, 8, 8), bool)
    o = oracle.attention_sets(q, k, v, mask, 1 / 8.0)
    dense = torch.nn.functional.scaled_dot_product_attention(q.double(), k.double(), v.double()).numpy()
    assert np.abs(o - dense).max() < 1e-12
    dense32 = torch.nn.functional.scaled_dot_product_attention(q, k, v).numpy()
    assert np.abs(o - dense32).max() < 1e-4


def test_attention_single_block_and_tail_equal_sdpa_on_slice():
    g = torch.Generator().manual_seed(1)
    S = 200                                   # blocks 0..3, the last with 8 tokens
    q, k, v = (torch.randn(1, S, 32, dtype=torch.float64, generator=g) for _ in range(3))
    mask = np.zeros((1, 4, 4), bool)
    mask[0, 1, 3] = True                      # query block 1 sees only the ragged block 3
    mask[0, 3, [0, 3]] = True                 # query block 3 sees blocks 0 and 3
    mask[0, 0, 0] = mask[0, 2, 2] = True
    o = oracle.attention_sets(q, k, v, mask, 0.3)
    sd = torch.nn.functional.scaled_dot_product_attention
    ref1 = sd(q[:, 64:128], k[:, 192:200], v[:, 192:200], scale=0.3)
    np.testing.assert_allclose(o[0, 64:128], ref1[0].numpy(), atol=1e-13)
    cols = torch.cat([torch.arange(0, 64), torch.arange(192, 200)])
    ref3 = sd(q[:, 192:200], k[:, cols], v[:, cols], scale=0.3)
    np.testing.assert_allclose(o[0, 192:200], ref3[0].numpy(), atol=1e-13)


def test_attention_gather_equals_token_mask():
    w, Q, K, V = _small(H=2, S=700, frame_len=350, region_len=64, seed=2)
    rng = np.random.default_rng(4)
    nb = 11
    mask = rng.random((2, nb, nb)) < 0.3
    mask[:, np.arange(nb), np.arange(nb)] = True
    a = oracle.attention_sets(Q, K, V, mask, 0.1)
    b = oracle.attention_token_mask(Q, K, V, mask, 0.1)
    assert np.abs(a - b).max() < 1e-12


# ---------------------------------------------------------------- bookkeeping

def test_csr_loads_tiles_lpt_hand():
    m = np.zeros((2, 3, 3), bool)
    m[0, 0, [0, 2]] = True; m[0, 1, [1]] = True; m[0, 2, [0, 1, 2]] = True
    m[1, 0, [0]] = True; m[1, 1, [0, 1]] = True; m[1, 2, [2]] = True
    rp, ci = oracle.csr_from_mask(m)
    assert rp.tolist() == [0, 2, 3, 6, 7, 9, 10]
    assert ci.tolist() == [0, 2, 1, 0, 1, 2, 0, 0, 1, 2]
    assert oracle.head_loads(m).tolist() == [6, 4]
    c = oracle.tile_costs(m)                  # tiles: (0,1) and (2,) per head
    assert c.tolist() == [[3, 3], [2, 1]]
    assert oracle.lpt_order(c).tolist() == [0, 1, 2, 3]
    assert oracle.lpt_order(np.array([[1, 5], [5, 2]])).tolist() == [1, 2, 3, 0]


def test_selected_flops_hand():
    m = np.zeros((1, 2, 2), bool)
    m[0, 0, 1] = True; m[0, 1, 1] = True     # S = 100: block 0 = 64 tokens, block 1 = 36
    assert oracle.selected_flops(m, 100, 64, 16) == 4 * 16 * (64 * 36 + 36 * 36)


# ---------------------------------------------------------------- fixed top-k (notes §5.2)

def test_topk_row_hand_and_ties():
    sc = np.array([0.5, 2.0, -1.0, 2.0, 1.5])
    assert oracle.topk_row(sc, 1).tolist() == [1]                  # tie 2.0 / 2.0: lower index first
    assert oracle.topk_row(sc, 3).tolist() == [1, 3, 4]
    assert sorted(oracle.topk_row(sc, 9).tolist()) == [0, 1, 2, 3, 4]


def test_topk_mode_full_coverage_is_dense_like_the_notes_test():
    # The notes' own correctness check: topk_blocks = nb and local_window = nb -> dense.
    w, Q, K, V = _small(H=2, S=512, d=64, frame_len=256, region_len=64, dtype="f32", seed=0)
    r = oracle.route(Q, K, oracle.RouteCfg(mode="topk", topk_blocks=8, local_window=8, force_diag=False))
    assert r["mask"].all()
    o = oracle.attention_sets(Q, K, V, r["mask"], 1 / 8.0)
    dense = torch.nn.functional.scaled_dot_product_attention(Q.double(), K.double(), V.double()).numpy()
    assert np.abs(o - dense).max() < 1e-12


def test_topk_mode_matches_brute_force_ranking():
    w, Q, K, _ = _small(H=2, S=1000, frame_len=500, region_len=128, seed=21)
    cfg = oracle.RouteCfg(mode="topk", topk_blocks=3, force_diag=False)
    r = oracle.route(Q, K, cfg)
    Qd, Kd = Q.double().numpy(), K.double().numpy()
    nb = 16
    for bh in range(2):
        qm = [Qd[bh, i * 64:min(1000, i * 64 + 64)].mean(axis=0) for i in range(nb)]
        km = [Kd[bh, j * 64:min(1000, j * 64 + 64)].mean(axis=0) for j in range(nb)]
        for i in range(nb):
            s = [float(np.dot(qm[i], km[j])) for j in range(nb)]
            top = sorted(range(nb), key=lambda j: (-s[j], j))[:3]
            assert sorted(np.nonzero(r["mask"][bh, i])[0].tolist()) == sorted(top)


# ---------------------------------------------------------------- slack-aware augmentation (SASA)

def _sets_to_mask(sets, nb):
    m = np.zeros((1, nb, nb), dtype=bool)
    for i, s in enumerate(sets):
        m[0, i, s] = True
    return m


def test_sasa_golden_hand_cases():
    cases = json.load(open(os.path.join(GOLDEN, "sasa_hand_cases.json")))["cases"]
    for c in cases:
        nb = c["nb"]
        key = np.array(c["key"], dtype=np.float64)[None]
        out = oracle.sasa_tile_augment(_sets_to_mask(c["mask"], nb), key, c["coef"], c["trigger"])
        got = [np.nonzero(out[0, i])[0].tolist() for i in range(nb)]
        assert got == c["expect"], c["why"]


def _random_tile_masks(rng, BH, nb, density):
    mask = rng.random((BH, nb, nb)) < density
    mask[:, np.arange(nb), np.arange(nb)] = True        # every row non-empty, as routing guarantees
    return mask


@pytest.mark.parametrize("seed", range(8))
def test_sasa_budget_and_brute_force_best_mass(seed):
    # Closed-form count (floor(coef * slack) when slack >= trigger) and, by brute force over every
    # subset of the candidates of that size, the added set has the largest importance mass.
    rng = np.random.default_rng(seed)
    nb = int(rng.integers(2, 9))
    mask = _random_tile_masks(rng, 2, nb, 0.35)
    key = rng.random((2, nb, nb))
    coef = float(rng.choice([0.25, 0.5, 0.75, 1.0, 0.3]))
    trigger = int(rng.integers(0, 3))
    out = oracle.sasa_tile_augment(mask, key, coef, trigger)
    for bh in range(2):
        for r in range(nb):
            if r ^ 1 >= nb:
                assert np.array_equal(out[bh, r], mask[bh, r])
                continue
            union = mask[bh, r] | mask[bh, r ^ 1]
            cand = np.nonzero(union & ~mask[bh, r])[0]
            slack = cand.size
            n = math.floor(float(np.float32(coef)) * slack) if slack >= trigger and slack > 0 else 0
            added = np.nonzero(out[bh, r] & ~mask[bh, r])[0]
            assert added.size == n
            assert np.all(mask[bh, r] <= out[bh, r])
            if n:
                best = max(key[bh, r, list(s)].sum() for s in itertools.combinations(cand, n))
                assert key[bh, r, added].sum() == pytest.approx(best, rel=0, abs=1e-15)


@pytest.mark.parametrize("seed", range(4))
def test_sasa_tile_union_unchanged_and_coef_one_fills_union(seed):
    rng = np.random.default_rng(100 + seed)
    nb = 9
    mask = _random_tile_masks(rng, 3, nb, 0.3)
    key = rng.random((3, nb, nb))
    for coef in (0.5, 1.0):
        out = oracle.sasa_tile_augment(mask, key, coef, 1)
        for t in range(nb // 2):
            a, b = 2 * t, 2 * t + 1
            assert np.array_equal(out[:, a] | out[:, b], mask[:, a] | mask[:, b])   # tile cost unchanged
            if coef == 1.0:
                assert np.array_equal(out[:, a], mask[:, a] | mask[:, b])
                assert np.array_equal(out[:, b], mask[:, a] | mask[:, b])
        assert np.array_equal(out[:, nb - 1], mask[:, nb - 1])                      # odd tail, no partner
    assert np.array_equal(oracle.sasa_tile_augment(mask, key, 0.0, 1), mask)
    assert np.array_equal(oracle.sasa_tile_augment(mask, key, 1.0, nb + 1), mask)  # trigger never reached


def test_sasa_ties_go_to_lower_block_and_route_integration():
    # All candidates tied: the lowest indices are added. Through route(): the augmented mask keeps
    # the base mask, and the near-tie flags cover the tied rows.
    mask = _sets_to_mask([[0], [1, 2, 3, 4, 5]], 6)
    key = np.full((1, 6, 6), 0.1)
    out = oracle.sasa_tile_augment(mask, key, 0.5, 1)
    assert np.nonzero(out[0, 0])[0].tolist() == [0, 1, 2]
    assert oracle.sasa_near_tie_rows(mask, key, 0.5, 1, "topp")[0, 0]
    # a valid near-tie alternative: another 2 of the tied candidates
    alt = mask[0, 0].copy()
    alt[[4, 5]] = True
    assert oracle.valid_sasa_row(key[0, 0], mask[0, 0], mask[0, 1], alt, 0.5, 1, "topp")
    bad = mask[0, 0].copy()
    bad[[4]] = True                                        # wrong count
    assert not oracle.valid_sasa_row(key[0, 0], mask[0, 0], mask[0, 1], bad, 0.5, 1, "topp")

    x = make_inputs(get_workload("tiny"), device="cpu")
    BH = x["q"].shape[0] * x["q"].shape[1]
    Q = x["q"].reshape(BH, -1, x["q"].shape[-1])
    K = x["k"].reshape(BH, -1, x["k"].shape[-1])
    base = oracle.route(Q, K, oracle.RouteCfg(p=0.6))
    aug = oracle.route(Q, K, oracle.RouteCfg(p=0.6, sasa_coef=1.0, sasa_trigger=1))
    assert np.array_equal(aug["base_mask"], base["mask"])
    assert np.all(base["mask"] <= aug["mask"])
    assert aug["mask"].sum() > base["mask"].sum()
    assert np.array_equal(oracle.tile_costs(aug["mask"]), oracle.tile_costs(base["mask"]))


# ---------------------------------------------------------------- runtime load balancing (RLB)

def test_rlb_golden_hand_cases():
    cases = json.load(open(os.path.join(GOLDEN, "rlb_hand_cases.json")))["cases"]
    for c in cases:
        moves, L = oracle.rlb_plan(np.array(c["loads"]), c["target"], c["budget"])
        assert [list(mv) for mv in moves] == c["moves"], c["why"]
        assert L == c["rank_loads"], c["why"]


def test_rlb_imbalance_definition():
    assert oracle.imbalance([10, 10, 10]) == 1.0
    assert oracle.imbalance([3, 1]) == 1.5                 # max / mean = 3 / 2
    assert oracle.imbalance([0, 0]) == 1.0


@pytest.mark.parametrize("seed", range(10))
def test_rlb_invariants_random(seed):
    # Every move lowers the pair's maximum, so the maximum never rises and the imbalance never
    # grows; total load is conserved; a head moves at most once and only from its own rank; the
    # per-rank budget holds; the plan stops at the target or when the sender has no such head.
    rng = np.random.default_rng(seed)
    R, Hl = int(rng.integers(2, 9)), int(rng.integers(1, 7))
    loads = rng.integers(0, 1000, size=(R, Hl)) * (rng.random((R, Hl)) < 0.8)
    budget = int(rng.integers(0, 3))
    target = float(rng.choice([1.0, 1.05, 1.2]))
    moves, L = oracle.rlb_plan(loads, target, budget)
    cur = [int(x) for x in loads.sum(axis=1)]
    seen = set()
    sent = [0] * R
    for s, h, d in moves:
        assert (s, h) not in seen and s != d
        seen.add((s, h))
        w = int(loads[s, h])
        assert cur[d] + w < cur[s]
        before = max(cur)
        cur[s] -= w
        cur[d] += w
        assert max(cur) <= before
        sent[s] += 1
    assert cur == L and sum(L) == int(loads.sum())
    assert all(x <= budget for x in sent)
    assert oracle.imbalance(L) <= oracle.imbalance(loads.sum(axis=1))
    if moves == [] and budget > 0 and oracle.imbalance(L) > target:
        s = max(range(R), key=lambda r: (L[r], -r))
        d = min(range(R), key=lambda r: (L[r], r))
        assert all(not (L[d] + int(loads[s, h]) < L[s]) for h in range(Hl))


# ---------------------------------------------------------------- token-exact frame selection

def _exact_cfg(fl, **kw):
    base = dict(mode="frame_topk", frame_len=fl, topk_frames=1, force_diag=False, frame_exact=True)
    base.update(kw)
    return oracle.RouteCfg(**base)


def test_frame_exact_golden_hand_case():
    c = json.load(open(os.path.join(GOLDEN, "frame_exact_hand_case.json")))
    S, fl = c["S"], c["frame_len"]
    cfg = _exact_cfg(fl)
    G = np.array(c["G"], dtype=bool)
    tm = oracle.frame_token_mask(G, S, cfg)
    want = np.zeros((S, S), dtype=bool)
    want[0:96, 0:96] = True
    want[96:192, 192:256] = True
    want[192:256, 96:192] = True
    assert np.array_equal(tm, want), c["token_rule"]
    nb = S // 64
    support = [[j for j in range(nb) if tm[i * 64:(i + 1) * 64, j * 64:(j + 1) * 64].any()] for i in range(nb)]
    assert support == c["block_support"]
    bf = oracle.block_forced(S, cfg)
    for e in c["codes"]:
        code = oracle.frame_entry_code(G, bf, e["i"], e["j"], S, cfg)
        assert (code & 15, (code >> 8) & 255, (code >> 16) & 255) == (e["allow"], e["kcol"], e["qrow"]), e["why"]


@pytest.mark.parametrize("fl,seed", [(900, 0), (640, 1), (200, 2)])
def test_frame_exact_invariants(fl, seed):
    # The block support of the token mask is the block-granular frame selection; the entry codes
    # expand to exactly the token mask's 64 x 64 tiles; frames that are whole blocks give the
    # block mask itself; topk >= F allows everything.
    rng = np.random.default_rng(seed)
    S, d, BH = 1800, 16, 2
    Q = rng.standard_normal((BH, S, d))
    K = rng.standard_normal((BH, S, d))
    cfg = _exact_cfg(fl, topk_frames=2, frame_window=0 if seed == 1 else -1, force_first_frame=seed == 2,
                     force_diag=seed != 0, local_window=1 if seed == 2 else 0)
    r = oracle.route(Q, K, cfg)
    nb = -(-S // 64)
    bf = oracle.block_forced(S, cfg)
    for bh in range(BH):
        tm = oracle.frame_token_mask(r["frame_sets"][bh], S, cfg)
        for i in range(nb):
            for j in range(nb):
                tile = tm[i * 64:(i + 1) * 64, j * 64:(j + 1) * 64]
                assert tile.any() == r["mask"][bh, i, j], (bh, i, j)
                if r["mask"][bh, i, j]:
                    code = oracle.frame_entry_code(r["frame_sets"][bh], bf, i, j, S, cfg)
                    rows = np.arange(tile.shape[0]) >= ((code >> 16) & 255)
                    cols = np.arange(tile.shape[1]) >= ((code >> 8) & 255)
                    expand = (code >> (2 * rows[:, None] + cols[None, :])) & 1
                    assert np.array_equal(expand.astype(bool), tile), (bh, i, j)
    # frames of whole blocks: exact == block granular
    cfg64 = _exact_cfg(640, topk_frames=2)
    r64 = oracle.route(Q, K, cfg64)
    tm = oracle.frame_token_mask(r64["frame_sets"][0], S, cfg64)
    blk = np.arange(S) // 64
    assert np.array_equal(tm, r64["mask"][0][blk][:, blk])
    # every frame kept: dense
    rall = oracle.route(Q, K, _exact_cfg(fl, topk_frames=99))
    assert oracle.frame_token_mask(rall["frame_sets"][1], S, _exact_cfg(fl)).all()


def test_attention_dense_mask_matches_sdpa():
    rng = np.random.default_rng(5)
    Q, K, V = (torch.from_numpy(rng.standard_normal((2, 150, 32))) for _ in range(3))
    full = np.ones((2, 150, 150), dtype=bool)
    out = oracle.attention_dense_mask(Q, K, V, full, 1 / math.sqrt(32))
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V).numpy()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
    m = rng.random((2, 150, 150)) < 0.3
    m[:, np.arange(150), np.arange(150)] = True
    out = oracle.attention_dense_mask(Q, K, V, m, 0.2)
    ref = torch.nn.functional.scaled_dot_product_attention(Q, K, V, attn_mask=torch.from_numpy(m), scale=0.2).numpy()
    np.testing.assert_allclose(out, ref, rtol=0, atol=1e-12)
