"""The arithmetic behind the router's tensor-core block scores, checked on the CPU with exact
integers (Python ints / fractions): a block mean x with max|x| < 2^e is written as
N = rint(x 2^(39-e)) split into five signed 8-bit digits (balanced base-256 digits from the
bottom, the rest on top; e raised by one when the top digit would reach 128), so that
x ~ 2^e sum_a X_a 2^(-7-8a) within 2^(e-40); the 15 digit-pair dot products of levels a+b <= 4
then give the dot product of two means within the bound the GPU test uses. This pins the
scheme (digit ranges, exact reconstruction, the dropped-level bound), not the kernel."""
import math
from fractions import Fraction

import numpy as np
import pytest

SLICES = 5


def split(x: np.ndarray):
    """(e, digits[5][d]) of one block mean, as the scheme defines them."""
    mx = float(np.max(np.abs(x)))
    e = max(-900, math.frexp(mx)[1]) if mx > 0 else 0      # mx < 2^e
    if round(mx * 2.0 ** (39 - e)) > 127 * 2 ** 32:
        e += 1
    digits = np.zeros((SLICES, x.size), dtype=np.int64)
    for c, v in enumerate(x):
        n = int(round(float(v) * 2.0 ** (39 - e)))            # exact: |n| < 2^40 fits a double
        for a in range(SLICES - 1, 0, -1):
            dg = ((n + 128) & 255) - 128
            n = (n - dg) >> 8
            digits[a, c] = dg
        digits[0, c] = n
    return e, digits


def value(e, digits) -> list:
    return [Fraction(sum(int(digits[a, c]) * 2 ** (8 * (SLICES - 1 - a)) for a in range(SLICES)), 2 ** (39 - e))
            for c in range(digits.shape[1])]


def cases(rng):
    d = 128
    out = [rng.standard_normal(d), rng.standard_normal(d) * 1e-3, rng.standard_normal(d) * 300.0,
           np.zeros(d), np.full(d, -1.0), np.full(d, 1.0 - 2.0 ** -9)]     # -1: exact power; top-digit bump
    x = rng.standard_normal(d)
    x[0] = 0.999 * 2 ** 3                                                    # max just under a power of two
    out.append(x)
    return out


def test_digits_are_int8_and_reconstruct_within_2_pow_e_minus_40():
    rng = np.random.default_rng(0)
    for x in cases(rng):
        e, dg = split(x)
        assert dg.min() >= -128 and dg.max() <= 127
        rec = value(e, dg)
        for c, v in enumerate(x):
            assert abs(Fraction(float(v)) - rec[c]) <= Fraction(2) ** (e - 40)
        assert float(np.max(np.abs(x))) < 2.0 ** e


def test_level_sums_fit_fp32_exactly_and_dropped_levels_are_below_the_bound():
    rng = np.random.default_rng(1)
    xs = cases(rng)
    for qx in xs[:4]:
        for kx in xs[2:]:
            eq, dq = split(qx)
            ek, dk = split(kx)
            levels = [sum(int(np.dot(dq[a], dk[l - a])) for a in range(l + 1)) for l in range(SLICES)]
            assert all(abs(v) < 2 ** 24 for v in levels)          # exact in fp32 / int32 accumulators
            approx = sum(Fraction(levels[l], 2 ** (14 + 8 * l)) for l in range(SLICES)) * Fraction(2) ** (eq + ek)
            exact = sum(Fraction(float(a)) * Fraction(float(b)) for a, b in zip(qx, kx))
            # left out: levels 5..8 of the digits and the rounding of each mean (2^(e-40) per value)
            mq, mk = float(np.max(np.abs(qx))), float(np.max(np.abs(kx)))
            bound = Fraction(2) ** -30 * Fraction(2) ** (eq + ek) + \
                Fraction(2) ** -40 * (Fraction(2) ** eq * Fraction(sum(abs(float(b)) for b in kx)) +
                                      Fraction(2) ** ek * Fraction(sum(abs(float(a)) for a in qx)))
            assert abs(approx - exact) <= bound, float(abs(approx - exact) / bound)
            # the bound is far below the size of the products of nonzero means (max|x| >= 2^(e-2))
            if mq > 0 and mk > 0:
                assert float(bound) <= 2.0 ** -24 * mq * mk


@pytest.mark.parametrize("v", [1.0 - 2.0 ** -10, -(1.0 - 2.0 ** -10), 0.9961, 127.5 / 128])
def test_top_digit_bump(v):
    x = np.zeros(4)
    x[0] = v
    e, dg = split(x)
    assert dg.min() >= -128 and dg.max() <= 127
