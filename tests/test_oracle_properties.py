"""Property checks of the oracle against the mathematics, over many random cases (hypothesis):
the Top-p cut keeps the minimal descending prefix whose mass reaches p (every kept block at
least as likely as every dropped one, ties to the lower index, dropping the least likely kept
block falls short of p); block means are linear in the tokens and exact on constant blocks;
the softmax is shift invariant and sums to one; fixed top-k keeps exactly k blocks, the largest
scores. A plausible slip in the oracle (a reversed order, a strict/non-strict comparison, an
off-by-one in the prefix length) breaks one of these."""
import importlib

import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

R = importlib.import_module("oracle.route")

settings.register_profile("oracle", max_examples=120, deadline=None)
settings.load_profile("oracle")


rows = st.integers(min_value=1, max_value=40).flatmap(
    lambda n: st.lists(st.floats(min_value=-30, max_value=30, allow_nan=False, width=32), min_size=n, max_size=n))


@given(rows, st.floats(min_value=0.01, max_value=0.999))
def test_topp_is_the_minimal_descending_prefix(logits, p):
    sc = np.array(logits, dtype=np.float64)[None, :]
    pi = R.row_softmax(sc)[0]
    order, k, csum = R.topp_row(pi, p)
    kept = set(order[:k].tolist())
    dropped = [j for j in range(pi.size) if j not in kept]
    assert csum[k - 1] >= p or k == pi.size
    if k > 1:
        assert csum[k - 2] < p                      # one block fewer does not reach p
    for a in kept:                                  # every kept block ranks before every dropped one
        for b in dropped:
            assert pi[a] > pi[b] or (pi[a] == pi[b] and a < b)


@given(st.integers(min_value=1, max_value=3), st.integers(min_value=1, max_value=300),
       st.sampled_from([8, 16]), st.integers(min_value=0, max_value=2 ** 31 - 1))
def test_pool_is_linear_and_exact_on_constant_blocks(BH, S, d, seed):
    rng = np.random.default_rng(seed)
    X, Y = rng.standard_normal((BH, S, d)), rng.standard_normal((BH, S, d))
    a, b = 1.5, -0.25
    lhs = R.pool_blocks(a * X + b * Y, 64)
    rhs = a * R.pool_blocks(X, 64) + b * R.pool_blocks(Y, 64)
    np.testing.assert_allclose(lhs, rhs, rtol=1e-12, atol=1e-12)
    nb = -(-S // 64)
    C = np.repeat(np.arange(nb, dtype=np.float64), 64)[:S]
    const = np.broadcast_to(C[None, :, None], (BH, S, d)).copy()
    np.testing.assert_array_equal(R.pool_blocks(const, 64), np.broadcast_to(np.arange(nb)[None, :, None], (BH, nb, d)))


@given(rows, st.floats(min_value=-100, max_value=100, allow_nan=False))
def test_softmax_sums_to_one_and_is_shift_invariant(logits, c):
    sc = np.array(logits, dtype=np.float64)[None, :]
    pi = R.row_softmax(sc)[0]
    assert abs(pi.sum() - 1.0) < 1e-12 and np.all(pi >= 0)
    np.testing.assert_allclose(R.row_softmax(sc + c)[0], pi, rtol=1e-9, atol=1e-15)


@given(rows, st.integers(min_value=1, max_value=50))
def test_topk_keeps_the_k_largest_scores(logits, k):
    sc = np.array(logits, dtype=np.float64)
    sel = np.asarray(R.topk_row(sc, k))
    kept = set(np.flatnonzero(sel).tolist()) if sel.dtype == bool else set(sel.tolist())
    assert len(kept) == min(k, sc.size)
    dropped = [j for j in range(sc.size) if j not in kept]
    for a in kept:
        for b in dropped:
            assert sc[a] > sc[b] or (sc[a] == sc[b] and a < b)


@given(st.sampled_from([2, 4, 8, 16, 32]), st.data())
def test_topp_cut_reaching_p_exactly_keeps_that_prefix(n, data):
    # uniform rows of a power-of-two length: every prefix mass m/n is exact in binary, so a cut
    # at p = m/n must keep exactly m blocks ("reaches p": >=, not >), the lowest indices first
    m = data.draw(st.integers(min_value=1, max_value=n - 1))
    pi = R.row_softmax(np.zeros((1, n)))[0]
    order, k, csum = R.topp_row(pi, m / n)
    assert k == m and list(order[:k]) == list(range(m))
