"""The identity the CUDA path uses for 2-bit Adam's second scale, checked in
numpy on the CPU: the squared norm of the residual r = c - s1 sign(c) equals
sum_t [M2_t + n_t (mu_t - s1)^2] over 512-element tiles, with each tile's sums
taken in one sweep shifted by |c| of its first element.  This is the arithmetic
of twobit.cuh restated, set against the oracle's definition (the sum of the
squared float residuals), so that its error bound and its exact cases are
pinned without a GPU."""

import numpy as np
import pytest

TILE = 512


def second_scale_sq_by_tiles(c: np.ndarray, s1: np.float32) -> float:
    a = np.abs(c.astype(np.float64))
    total = 0.0
    for lo in range(0, a.size, TILE):
        x = a[lo:lo + TILE]
        K = x[0]
        d = x - K
        d1, d2 = d.sum(), (d * d).sum()
        n = x.size
        S = n * K + d1
        M2 = max(d2 - d1 * d1 / n, 0.0)
        mu = S / n
        total += M2 + n * (mu - float(s1)) ** 2
    return total


def residual_sq_as_defined(c: np.ndarray, s1: np.float32) -> float:
    r = c - np.where(c >= 0, s1, -s1).astype(np.float32)          # float residuals
    return float(np.sum(r.astype(np.float64) ** 2))


def first_scale(c: np.ndarray) -> np.float32:
    return np.float32(np.sqrt(np.sum(c.astype(np.float64) ** 2)) / np.sqrt(c.size))


@pytest.mark.parametrize("n", [1, 7, 512, 513, 4096 + 77, 100_000])
@pytest.mark.parametrize("dist", ["normal", "student_t", "uniform"])
def test_matches_the_float_residuals_within_their_rounding(n, dist):
    rng = np.random.default_rng([n, len(dist)])
    c = {"normal": rng.normal(0, 1e-3, n), "student_t": rng.standard_t(3, n) * 1e-3,
         "uniform": rng.uniform(-1e-3, 1e-3, n)}[dist].astype(np.float32)
    s1 = first_scale(c)
    got, want = second_scale_sq_by_tiles(c, s1), residual_sq_as_defined(c, s1)
    # the float residuals carry one rounding each: at most 2^-23 relative in the sum
    assert abs(got - want) <= 2.0 ** -23 * want + 1e-300


def test_equal_magnitudes_give_exactly_zero():
    for n in (1, 33, 512, 1000, 5000):
        c = np.where(np.arange(n) % 3 == 0, -1, 1).astype(np.float32) * np.float32(3.0517578e-05)
        s1 = first_scale(c)
        assert s1 == np.float32(3.0517578e-05)
        assert second_scale_sq_by_tiles(c, s1) == 0.0 == residual_sq_as_defined(c, s1)


def test_no_cancellation_when_magnitudes_sit_near_the_first_scale():
    rng = np.random.default_rng(7)
    n = 20_000
    c = (1.0 + 1e-6 * rng.standard_normal(n)).astype(np.float32) * np.where(rng.random(n) < 0.5, -1, 1)
    c = c.astype(np.float32)
    s1 = first_scale(c)
    got, want = second_scale_sq_by_tiles(c, s1), residual_sq_as_defined(c, s1)
    assert want > 0 and abs(got - want) <= 1e-6 * want


def test_the_raw_moment_form_would_cancel():
    """Why the shifted tile sums: sum c^2 - 2 s1 sum|c| + n s1^2 loses the
    residual entirely when the magnitudes sit near s1."""
    rng = np.random.default_rng(8)
    n = 20_000
    c = (1.0 + 1e-7 * rng.standard_normal(n)).astype(np.float32)
    s1 = first_scale(c)
    a = np.abs(c.astype(np.float64))
    raw = np.sum(a * a) - 2 * float(s1) * np.sum(a) + n * float(s1) ** 2
    want = residual_sq_as_defined(c, s1)
    assert abs(second_scale_sq_by_tiles(c, s1) - want) <= 1e-6 * want
    assert abs(raw - want) > 1e-3 * want
