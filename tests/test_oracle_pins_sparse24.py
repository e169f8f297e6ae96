"""Pins of the oracle's 2:4-sparse INT4 variant to things other than itself.

The pages evaluate QuEST on a 2:4-sparse INT4 format (atlas.scime.ai summary,
ablation table; pith.science review, results list and Figure 4a) without
spelling it out. The oracle reads it as: the same Hadamard transform and RMS;
in each run of four consecutive transformed values the two of largest magnitude
survive; survivors go onto the b-bit midrise grid whose step minimises the MSE
of the surviving values of an N(0,1) input; the trust mask applies the
half-interval rule to every value's total error (a pruned value is rebuilt as 0).

The pins: Monte Carlo of the kept-value law and its quantization MSE, a brute
force search for the step, order-statistic closed forms of the masked rates,
and the quantizer's outputs against scipy's Hadamard matrix and numpy's sort.
"""
import math

import numpy as np
import pytest
import scipy.linalg
import scipy.special

import oracle


def _kept_samples(n, seed):
    """Magnitudes that survive 2:4 pruning of n runs of four N(0,1) values."""
    z = np.abs(np.random.default_rng(seed).standard_normal((n, 4)))
    z.sort(axis=1)
    return z[:, 2:].reshape(-1)


def _midrise_err2(a, bits, delta):
    half = 1 << (bits - 1)
    i = np.minimum(np.floor(a / delta), half - 1)
    return (a - (i + 0.5) * delta) ** 2


@pytest.mark.parametrize("bits,delta", [(1, 2.0), (2, 1.2), (4, 0.36), (4, 0.5), (8, 0.032)])
def test_kept_mse_matches_monte_carlo(bits, delta):
    a = _kept_samples(2_000_000, 7 + bits)
    e2 = _midrise_err2(a, bits, delta)
    mc, se = e2.mean(), e2.std() / math.sqrt(e2.size)
    assert abs(oracle.sparse24_mse(bits, delta) - mc) < 4 * se + 1e-12


def test_kept_law_moments():
    # E|X| and E[X^2] of a surviving value by Monte Carlo against the oracle's MSE at
    # b = 1, where the error (a - delta/2)^2 expands to E[a^2] - delta E|a| + delta^2/4.
    a = _kept_samples(4_000_000, 3)
    m1, m2 = a.mean(), (a * a).mean()
    for delta in (0.5, 2.0, 3.0):
        expect = m2 - delta * m1 + delta * delta / 4
        assert oracle.sparse24_mse(1, delta) == pytest.approx(expect, rel=2e-3)
    # b = 1: the optimal level is the mean surviving magnitude
    alpha, d, _ = oracle.alpha_sparse24(1)
    assert d / 2 == pytest.approx(m1, rel=2e-3)


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_sparse_step_is_the_minimiser(bits):
    alpha, d, m = oracle.alpha_sparse24(bits)
    assert alpha == pytest.approx(d * 2 ** (bits - 1), rel=1e-15)
    grid = np.linspace(0.5 * d, 1.5 * d, 201)
    vals = np.array([oracle.sparse24_mse(bits, g) for g in grid])
    k = int(np.argmin(vals))
    assert abs(grid[k] - d) <= grid[1] - grid[0]
    assert m <= vals.min() + 1e-15
    # MSE is unimodal around the optimum on this grid
    assert np.all(np.diff(vals[:k + 1]) <= 1e-15) and np.all(np.diff(vals[k:]) >= -1e-15)


@pytest.mark.parametrize("bits", range(1, 9))
def test_sparse_clip_is_wider_than_dense(bits):
    # the survivors are the larger magnitudes, so their MSE-optimal clip edge is wider
    assert oracle.alpha_sparse24(bits)[0] > oracle.alpha(bits)[0]


@pytest.mark.parametrize("delta", [0.05, 0.06])
def test_sparse_fine_grid_is_granular(delta):
    # at b = 8 with the clip edge 128 delta >= 6.4 (survivors beyond it have mass
    # below 1e-8) the error is uniform within each cell: MSE ~ delta^2 / 12, the
    # textbook granular-noise result
    assert oracle.sparse24_mse(8, delta) == pytest.approx(delta * delta / 12, rel=1e-3)


def _half_normal_cdf(c):
    return scipy.special.erf(c / math.sqrt(2))


@pytest.mark.parametrize("bits", [1, 2, 4])
def test_masked_rates_match_order_statistics(bits):
    # Whole-row RMS on a long N(0,1) row. With F = P(|X| <= c), integrating the kept
    # density (6F^2 - 4F^3) dF gives P(|X| > c | kept) = 1 - 2F^3 + F^4 and the pruned
    # density (2 - 6F^2 + 4F^3) dF gives P(|X| > c | pruned) = 1 - 2F + 2F^3 - F^4.
    # With T = 1 a kept value is masked beyond the clip, |y| > alpha r, and a pruned
    # one beyond half a step, |y| > Delta / 2.
    n = 1 << 20
    x = np.random.default_rng(50 + bits).standard_normal((1, n))
    o = oracle.quantize_sparse24(x, bits=bits, had=128, rms_group=n, trust=1.0)
    alpha, _, _ = oracle.alpha_sparse24(bits)
    r = math.sqrt(np.mean(x ** 2))
    kept = o["kept"].astype(bool)
    assert kept.sum() == n // 2
    F = _half_normal_cdf(alpha * r)
    p_kept = 1 - 2 * F ** 3 + F ** 4
    rate_kept = 1 - o["mask"][kept].mean()
    assert abs(rate_kept - p_kept) < 4 * math.sqrt(p_kept * (1 - p_kept) / (n / 2)) + 2 / n
    F = _half_normal_cdf(0.5 * alpha * r / 2 ** (bits - 1))
    p_pruned = 1 - 2 * F + 2 * F ** 3 - F ** 4
    rate_pruned = 1 - o["mask"][~kept].mean()
    assert abs(rate_pruned - p_pruned) < 4 * math.sqrt(p_pruned * (1 - p_pruned) / (n / 2)) + 2 / n


@pytest.mark.parametrize("bits,trust,rms", [(4, 1.0, 128), (2, 0.7, 128), (4, 1.3, "row"), (1, 1.0, "row")])
def test_sparse_quantizer_against_definitions(bits, trust, rms):
    g = np.random.default_rng(9)
    x = g.standard_t(3, (5, 512))
    x[2, 128:256] = 0.0                                  # an all-zero group (rms 128)
    rg = 512 if rms == "row" else rms
    o = oracle.quantize_sparse24(x, bits=bits, had=128, rms_group=rg, trust=trust)
    H = scipy.linalg.hadamard(128) / math.sqrt(128)
    y = (x.reshape(5, 4, 128) @ H.T).reshape(5, 512)
    np.testing.assert_allclose(o["y"], y, atol=1e-12)
    # the two largest magnitudes of each run of four survive (no ties in this data)
    runs = np.abs(y).reshape(5, 128, 4)
    order = np.argsort(-runs, axis=-1, kind="stable")
    expect_kept = np.zeros_like(runs, dtype=np.uint8)
    np.put_along_axis(expect_kept, order[..., :2], 1, axis=-1)
    assert np.array_equal(o["kept"], expect_kept.reshape(5, 512))
    # step from the RMS of every value of the group (pruned ones included)
    alpha, _, _ = oracle.alpha_sparse24(bits)
    rms_v = np.sqrt((y.reshape(5, -1, rg) ** 2).mean(axis=-1))
    np.testing.assert_allclose(o["scale"], alpha * rms_v / 2 ** (bits - 1), rtol=1e-13)
    delta = np.repeat(o["scale"], rg, axis=1)
    with np.errstate(divide="ignore", invalid="ignore"):
        t = np.where(delta > 0, y / delta, 0.0)
    half = 1 << (bits - 1)
    q = np.clip(np.floor(t), -half, half - 1)
    kept = o["kept"].astype(bool) & (delta > 0)
    assert np.array_equal(o["q"][kept], q[kept])
    assert np.all(o["q"][~o["kept"].astype(bool)] == 0)
    np.testing.assert_allclose(o["yhat"], np.where(kept, (q + 0.5) * delta, 0.0), atol=1e-12)
    m = np.where(kept, np.abs(t - (q + 0.5)) <= trust / 2, np.abs(t) <= trust / 2)
    assert np.array_equal(o["mask"], m.astype(np.uint8) | (delta == 0))
    # the exemption distances
    srt = -np.sort(-runs, axis=-1)
    gap = np.repeat((srt[..., 1] - srt[..., 2]), 4, axis=-1).reshape(5, 512)
    with np.errstate(divide="ignore", invalid="ignore"):
        np.testing.assert_allclose(np.where(delta > 0, o["d_prune"], 0),
                                   np.where(delta > 0, gap / delta, 0), atol=1e-12)
    pr = ~o["kept"].astype(bool) & (delta > 0)
    np.testing.assert_allclose(o["d_mask"][pr], np.abs(np.abs(t[pr]) - trust / 2), atol=1e-12)


def test_sparse_tie_keeps_lower_index():
    # Equal magnitudes in the Hadamard domain, built exactly with 4-point blocks
    # (H_4 / 2 and its products with small integers are exact in binary): the lower
    # indices win the tie and the prune gap is exactly zero.
    H4 = scipy.linalg.hadamard(4) / 2.0
    y = np.array([[3.0, -3.0, 3.0, 3.0, -1.0, 2.0, 2.0, -2.0]])
    x = (y.reshape(1, 2, 4) @ H4).reshape(1, 8)     # H_4 / 2 is its own inverse
    o = oracle.quantize_sparse24(x, bits=4, had=4, rms_group=4)
    assert np.array_equal(o["y"], y)
    assert np.array_equal(o["kept"][0], [1, 1, 0, 0, 0, 1, 1, 0])
    assert np.all(o["d_prune"][0] == 0.0)
