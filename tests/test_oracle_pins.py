"""Pins of the oracle to things other than itself.

Each test checks the oracle against a closed form, a library routine, a
textbook table, an invariant of the method, or brute force, chosen so that a
plausible slip (a dropped term, a wrong sign or index, a transposed operand, an
off-by-one in the grid) fails at least one of them. No expected value here comes
from the CUDA library.
"""
import math
import os

import numpy as np
import pytest
import scipy.integrate
import scipy.linalg
import scipy.stats
import torch

import oracle

pytestmark = pytest.mark.filterwarnings("ignore::scipy.integrate.IntegrationWarning")


# ---------------------------------------------------------------------------
# Hadamard matrix
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("n", [2, 4, 8, 16, 32, 64, 128, 256])
def test_hadamard_matches_scipy_sylvester(n):
    # scipy.linalg.hadamard builds the Sylvester matrix in natural order.
    assert np.array_equal(oracle.hadamard(n), scipy.linalg.hadamard(n).astype(np.float64))


@pytest.mark.parametrize("n", [2, 4, 8, 16, 32, 64, 128])
def test_hadamard_orthogonality(n):
    H = oracle.hadamard(n)
    assert np.array_equal(H @ H.T, n * np.eye(n))


def test_hadamard_small_by_hand():
    assert np.array_equal(oracle.hadamard(2), np.array([[1, 1], [1, -1]], dtype=float))
    H4 = np.array([[1, 1, 1, 1], [1, -1, 1, -1], [1, 1, -1, -1], [1, -1, -1, 1]], dtype=float)
    assert np.array_equal(oracle.hadamard(4), H4)


def test_forward_transform_of_basis_vectors():
    # The transform of e_i is row i of H / sqrt(n) (H is symmetric).
    n = 128
    H = scipy.linalg.hadamard(n).astype(np.float64)
    for i in [0, 1, 5, 64, 127]:
        x = np.zeros((1, n))
        x[0, i] = 3.0
        y = oracle.quantize(x, bits=4, had=n)["y"][0]
        np.testing.assert_allclose(y, 3.0 * H[i] / math.sqrt(n), rtol=0, atol=1e-14)


def test_parseval_and_involution():
    g = np.random.default_rng(11)
    x = g.standard_normal((7, 384))
    y = oracle.quantize(x, bits=3, had=128)["y"]
    for b0 in range(0, 384, 128):
        np.testing.assert_allclose(np.sum(y[:, b0:b0 + 128] ** 2, axis=1),
                                   np.sum(x[:, b0:b0 + 128] ** 2, axis=1), rtol=1e-12)
    # The normalised transform is an involution: the backward with an all-ones mask
    # maps y back to x.
    back = oracle.trust_bwd(y, np.ones_like(y, dtype=np.uint8), had=128)
    np.testing.assert_allclose(back, x, rtol=0, atol=1e-12)


# ---------------------------------------------------------------------------
# Gaussian MSE and alpha_b
# ---------------------------------------------------------------------------

def _quad_mse(bits, delta):
    """Gaussian MSE of the midrise grid by adaptive quadrature, one cell at a time."""
    half = 1 << (bits - 1)
    total = 0.0
    for i in range(-half, half):
        level = (i + 0.5) * delta
        a = -np.inf if i == -half else i * delta
        b = np.inf if i == half - 1 else (i + 1) * delta
        val, _ = scipy.integrate.quad(lambda x: (x - level) ** 2 * scipy.stats.norm.pdf(x), a, b,
                                      epsabs=1e-14, epsrel=1e-12, limit=200)
        total += val
    return total


@pytest.mark.parametrize("bits,delta", [(1, 0.7), (1, 1.6), (2, 0.5), (2, 1.0), (3, 0.6),
                                        (4, 0.3352), (5, 0.2), (8, 0.03)])
def test_gauss_mse_matches_quadrature(bits, delta):
    assert oracle.gauss_mse(bits, delta) == pytest.approx(_quad_mse(bits, delta), rel=1e-9, abs=1e-13)


def test_alpha_one_bit_closed_form():
    # For one bit the optimal levels are +-E|X| = +-sqrt(2/pi), so the step is
    # 2 sqrt(2/pi), alpha_1 = 2^0 * step and the MSE is 1 - 2/pi.
    # A minimiser of a smooth function is only located to ~sqrt(machine eps) of its
    # argument: the MSE is flat to first order there.
    a, d, m = oracle.alpha(1)
    assert d == pytest.approx(2.0 * math.sqrt(2.0 / math.pi), abs=5e-8)
    assert a == pytest.approx(d, abs=0)
    assert m == pytest.approx(1.0 - 2.0 / math.pi, abs=1e-12)


@pytest.mark.parametrize("bits,step", [(2, 0.9957), (3, 0.5860), (4, 0.3352)])
def test_alpha_matches_max_1960_uniform_table(bits, step):
    # J. Max, "Quantizing for minimum distortion" (IRE Trans. IT-6, 1960), table of
    # optimum uniform quantizers for a unit-variance Gaussian: step sizes for
    # N = 4, 8, 16 output levels, printed to four digits.
    _, d, _ = oracle.alpha(bits)
    assert d == pytest.approx(step, abs=1.5e-4)


@pytest.mark.parametrize("bits", range(1, 9))
def test_alpha_is_grid_search_minimum(bits):
    a, d, m = oracle.alpha(bits)
    grid = d + np.arange(-2000, 2001) * 1e-6
    vals = np.array([oracle.gauss_mse(bits, float(v)) for v in grid])
    best = grid[np.argmin(vals)]
    assert abs(best - d) <= 1.5e-6
    assert m <= vals.min() + 1e-15
    # and the minimum is interior and unimodal on a coarse sweep
    coarse = np.linspace(0.2 * d, 3.0 * d, 400)
    cv = np.array([oracle.gauss_mse(bits, float(v)) for v in coarse])
    k = int(np.argmin(cv))
    assert 0 < k < len(coarse) - 1
    assert np.all(np.diff(cv[:k + 1]) <= 1e-15) and np.all(np.diff(cv[k:]) >= -1e-15)
    assert a == pytest.approx(d * 2 ** (bits - 1), rel=1e-15)


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
def test_alpha_mse_monte_carlo(bits):
    # Monte-Carlo MSE of the grid with step Delta* on 4M N(0,1) samples, quantized
    # by a direct table lookup of the 2^b levels (nearest level = midrise cell).
    _, d, m = oracle.alpha(bits)
    x = np.random.default_rng(100 + bits).standard_normal(4_000_000)
    levels = (np.arange(-(1 << (bits - 1)), 1 << (bits - 1)) + 0.5) * d
    idx = np.abs(x[:, None] - levels[None, :]).argmin(axis=1) if bits <= 4 else None
    if idx is None:  # nearest level without the big temporary
        idx = np.searchsorted((levels[:-1] + levels[1:]) / 2, x)
    err2 = (x - levels[idx]) ** 2
    se = err2.std() / math.sqrt(err2.size)
    assert abs(err2.mean() - m) < 4 * se


def test_mse_decreases_with_bits():
    ms = [oracle.alpha(b)[2] for b in range(1, 9)]
    assert all(ms[i + 1] < ms[i] / 2.5 for i in range(7))


# ---------------------------------------------------------------------------
# Forward quantizer
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bits", range(1, 9))
def test_codes_in_range_and_levels(bits):
    x = np.random.default_rng(bits).standard_t(3, size=(16, 512))
    o = oracle.quantize(x, bits=bits, had=128)
    lo, hi = -(1 << (bits - 1)), (1 << (bits - 1)) - 1
    assert o["q"].min() >= lo and o["q"].max() <= hi
    # dequantised values lie exactly on the symmetric grid (q + 1/2) * Delta
    d = np.repeat(o["scale"], 128, axis=1)
    np.testing.assert_allclose(o["yhat"] / d - 0.5, o["q"], rtol=0, atol=1e-9)
    # interior elements are within half a step of their level
    interior = np.abs(o["t"]) <= (1 << (bits - 1))
    assert np.all(np.abs(o["y"] - o["yhat"])[interior] <= 0.5 * d[interior] * (1 + 1e-12))


def test_one_bit_is_sign_quantizer_n2():
    # n = 2, b = 1: y = ((x0 + x1)/sqrt2, (x0 - x1)/sqrt2) and the code is the sign
    # bit: q = 0 iff y >= 0, else -1. Enumerate small integer inputs.
    for x0 in range(-3, 4):
        for x1 in range(-3, 4):
            if x0 == 0 and x1 == 0:
                continue
            o = oracle.quantize(np.array([[x0, x1]], dtype=float), bits=1, had=2)
            y = [x0 + x1, x0 - x1]
            assert list(o["q"][0]) == [0 if v >= 0 else -1 for v in y]


@pytest.mark.parametrize("bits", [1, 4, 8])
def test_scale_of_a_basis_vector_block(bits):
    # A block holding c * e_i transforms to values +-c / sqrt(n), so its RMS is
    # exactly c / sqrt(n) and its step alpha_b * c / (sqrt(n) * 2^(b-1)); every
    # pre-round value is +-2^(b-1) / alpha_b.
    n, c = 128, 5.0
    a, _, _ = oracle.alpha(bits)
    x = np.zeros((1, n))
    x[0, 37] = c
    o = oracle.quantize(x, bits=bits, had=n)
    assert o["scale"][0, 0] == pytest.approx(a * c / (math.sqrt(n) * 2 ** (bits - 1)), rel=1e-14)
    np.testing.assert_allclose(np.abs(o["t"][0]), 2 ** (bits - 1) / a, rtol=1e-13)


@pytest.mark.parametrize("rms_group", [128, 512])
def test_group_rms_equals_input_rms(rms_group):
    # Parseval: the RMS of the transformed group equals the RMS of the raw input
    # over the same columns, so Delta / alpha_b * 2^(b-1) must equal it.
    bits = 3
    x = np.random.default_rng(31).standard_t(4, size=(6, 1024))
    o = oracle.quantize(x, bits=bits, had=128, rms_group=rms_group)
    a, _, _ = oracle.alpha(bits)
    r_in = np.sqrt(np.mean(x.reshape(6, -1, rms_group) ** 2, axis=2))
    np.testing.assert_allclose(o["scale"] / a * 2 ** (bits - 1), r_in, rtol=1e-13)


def test_zero_group_reading():
    x = np.zeros((2, 256))
    x[1, 128:] = np.random.default_rng(3).standard_normal(128)
    o = oracle.quantize(x, bits=4, had=128)
    assert np.all(o["q"][0] == 0) and np.all(o["yhat"][0] == 0) and np.all(o["mask"][0] == 1)
    assert o["scale"][0, 0] == 0 and o["scale"][1, 0] == 0 and o["scale"][1, 1] > 0
    assert np.all(o["q"][1, :128] == 0)


@pytest.mark.parametrize("bits", [1, 3, 4, 8])
def test_scale_invariance(bits):
    # Multiplying the input by c > 0 multiplies Delta by c and leaves codes and mask
    # unchanged: the RMS normalisation has no absolute term. A power of two keeps
    # every operation exact.
    x = np.random.default_rng(7).standard_normal((8, 256))
    a = oracle.quantize(x, bits=bits)
    b = oracle.quantize(x * 8.0, bits=bits)
    assert np.array_equal(a["q"], b["q"]) and np.array_equal(a["mask"], b["mask"])
    np.testing.assert_allclose(b["scale"], 8.0 * a["scale"], rtol=1e-15)


@pytest.mark.parametrize("bits", [1, 2, 4, 8])
def test_sign_symmetry(bits):
    # The midrise grid is symmetric: negating the input maps code q to -1 - q
    # (away from decision boundaries) and keeps the mask.
    x = np.random.default_rng(9).standard_normal((8, 256))
    a = oracle.quantize(x, bits=bits)
    b = oracle.quantize(-x, bits=bits)
    ok = a["d_round"] > 1e-9
    assert np.array_equal(b["q"][ok], -1 - a["q"][ok])
    assert np.array_equal(a["mask"], b["mask"])


@pytest.mark.parametrize("bits", [1, 2, 3, 4, 8])
def test_code_histogram_matches_gaussian_cells(bits):
    # One long N(0,1) row with the RMS over the whole row (r ~ 1): code i must occur
    # with the Gaussian mass of its cell [i Delta*, (i+1) Delta*) (outer cells open).
    n = 1 << 20
    x = np.random.default_rng(20 + bits).standard_normal((1, n))
    o = oracle.quantize(x, bits=bits, had=128, rms_group=n)
    a, d, _ = oracle.alpha(bits)
    r = o["scale"][0, 0] / d
    half = 1 << (bits - 1)
    edges = np.concatenate([[-np.inf], np.arange(-half + 1, half) * d * r, [np.inf]])
    p = np.diff(scipy.stats.norm.cdf(edges))
    counts = np.bincount(o["q"][0] + half, minlength=2 * half)
    expected = p * n
    keep = expected > 20
    chi2 = np.sum((counts[keep] - expected[keep]) ** 2 / expected[keep])
    dof = max(int(keep.sum()) - 1, 1)
    assert chi2 < scipy.stats.chi2.ppf(1 - 1e-4, dof)


@pytest.mark.parametrize("bits", range(1, 9))
def test_mask_rate_is_gaussian_tail_mass(bits):
    # With T = 1 an element is masked iff it lies beyond the clip |y| > alpha_b r;
    # on N(0,1) the rate is 2 (1 - Phi(alpha_b)) (binomial tolerance, 4 sigma).
    n = 1 << 21
    x = np.random.default_rng(40 + bits).standard_normal((1, n))
    o = oracle.quantize(x, bits=bits, had=128, rms_group=n, trust=1.0)
    a, _, _ = oracle.alpha(bits)
    r = math.sqrt(np.mean(x ** 2))
    p = 2 * scipy.stats.norm.sf(a * r)
    rate = 1.0 - o["mask"].mean()
    assert abs(rate - p) < 4 * math.sqrt(p * (1 - p) / n) + 1.0 / n
    # the interior is never masked when T >= 1
    assert np.all(o["mask"][np.abs(o["t"]) <= (1 << (bits - 1))] == 1)


@pytest.mark.parametrize("bits,trust", [(1, 1.3), (2, 1.3), (4, 0.5), (3, 2.0)])
def test_trust_region_edges(bits, trust):
    # m = 0 iff the distance from t to its level exceeds T/2. For T >= 1 only the
    # outer cells can be masked, beyond |t| = 2^(b-1) + (T-1)/2; for T < 1 every
    # cell masks the outer (1-T)/2 of its width on both sides.
    x = np.random.default_rng(5).standard_normal((4, 1024)) * 3
    o = oracle.quantize(x, bits=bits, had=128, trust=trust)
    t, m = o["t"], o["mask"]
    half = 1 << (bits - 1)
    if trust >= 1:
        expect = (np.abs(t) <= half + (trust - 1) / 2).astype(np.uint8)
    else:
        frac = t - np.floor(t)
        inner = (frac >= (1 - trust) / 2) & (frac <= (1 + trust) / 2)
        expect = np.where(np.abs(t) < half, inner, 0).astype(np.uint8)
        # outer region: beyond the clip t lies further from the level than 1/2
    safe = _flip_distance(t, bits, trust) > 1e-9   # closed form, not the oracle's d_mask
    assert np.array_equal(m[safe], expect[safe])


# ---------------------------------------------------------------------------
# Mask-exemption distance d_mask. The parity checks exempt a mask bit whose t
# lies within 1e-5 relative of a flip point of the mask, so d_mask must be the
# true distance: were it 0 everywhere, every mask comparison would be skipped.
# The flip points come from the rule's closed form (half-interval mask,
# pith.science review, "What carries the argument"): for T >= 1 only the outer
# edge |t| = 2^(b-1) + (T-1)/2 flips; for T < 1 each cell k of the clamped grid
# flips at k + (1-T)/2 and k + (1+T)/2.
# ---------------------------------------------------------------------------

def _flip_points(bits, trust):
    half = 1 << (bits - 1)
    if trust >= 1:
        e = half + (trust - 1) / 2
        return np.array([-e, e])
    k = np.arange(-half, half, dtype=np.float64)
    return np.sort(np.concatenate([k + (1 - trust) / 2, k + (1 + trust) / 2]))


def _flip_distance(t, bits, trust):
    f = _flip_points(bits, trust)
    return np.abs(np.asarray(t)[..., None] - f).min(axis=-1)


def _mask_rule(t, bits, trust):
    """The mask as a function of t alone (closed form of m = [|t - (q+1/2)| <= T/2])."""
    half = 1 << (bits - 1)
    t = np.asarray(t, dtype=np.float64)
    if trust >= 1:
        return (np.abs(t) <= half + (trust - 1) / 2).astype(np.uint8)
    frac = t - np.floor(t)
    inner = (frac >= (1 - trust) / 2) & (frac <= (1 + trust) / 2)
    return np.where((t >= -half) & (t < half), inner, False).astype(np.uint8)


_DMASK_CASES = [(4, 1.0), (3, 0.8), (2, 1.3), (1, 1.0), (8, 1.0), (4, 0.5), (3, 2.0), (1, "s*")]


def _edge_input(bits, trust, seed, rows=6, cols=512):
    """x whose transformed groups put many t values within 0.3 of the mask's flip
    points. Each group's t = y half / (alpha r) is chosen first; r = rms(y) then
    equals half / alpha exactly when sum(y^2) = 128 (half / alpha)^2, which the
    last value of the group makes true; x = H y / sqrt(128) (H symmetric)."""
    g = np.random.default_rng(seed)
    half = 1 << (bits - 1)
    a, _, _ = oracle.alpha(bits)
    budget = 128 * (half / a) ** 2
    f = _flip_points(bits, trust)
    H = scipy.linalg.hadamard(128).astype(np.float64) / math.sqrt(128)
    y = np.empty((rows, cols))
    for r in range(rows):
        for b0 in range(0, cols, 128):
            v = g.standard_normal(128) * 0.2 * (half / a)
            n_near = int(min(48, 0.5 * budget / (np.max(np.abs(f)) + 0.3) ** 2))
            pts = g.choice(f, n_near) + g.uniform(-0.3, 0.3, n_near)
            v[:n_near] = pts
            rest = budget - np.sum(v[:127] ** 2)
            assert rest > 0
            v[127] = math.sqrt(rest)
            y[r, b0:b0 + 128] = g.permutation(v)
    return (y.reshape(rows, cols // 128, 128) @ H).reshape(rows, cols)


@pytest.mark.parametrize("bits,trust", _DMASK_CASES)
def test_mask_flip_distance_closed_form(bits, trust):
    # The oracle searches an element's own cell and both neighbours, which holds
    # every flip point within distance 1 of t (the clamped edge cells reach to
    # infinity), so the two agree exactly once capped at 1.
    if trust == "s*":
        trust = _golden("outer_trust_scale_1bit")
    x = _edge_input(bits, trust, 70 + bits)
    x[1, :128] = 0.0                                    # an all-zero group: no flips
    o = oracle.quantize(x, bits=bits, had=128, trust=trust)
    t, d = o["t"], o["d_mask"]
    zero = np.repeat(o["scale"] == 0, 128, axis=1)
    assert np.all(np.isinf(d[zero]))
    ref = _flip_distance(t[~zero], bits, trust)
    np.testing.assert_allclose(np.minimum(d[~zero], 1.0), np.minimum(ref, 1.0), rtol=0, atol=1e-12)
    # the data reach the flip points often enough for this to bite
    assert np.sum(ref < 0.3) > 50


@pytest.mark.parametrize("bits,trust", _DMASK_CASES)
def test_mask_flip_distance_is_tight(bits, trust):
    # Moving t by less than d_mask leaves the mask as the oracle set it; moving it
    # by just more than a finite d_mask changes it in one of the two directions.
    if trust == "s*":
        trust = _golden("outer_trust_scale_1bit")
    x = _edge_input(bits, trust, 80 + bits)
    o = oracle.quantize(x, bits=bits, had=128, trust=trust)
    t, m, d = o["t"], o["mask"], np.minimum(o["d_mask"], 1.0)
    assert np.array_equal(_mask_rule(t, bits, trust), m)
    for s in (-1.0, 1.0):
        assert np.array_equal(_mask_rule(t + s * 0.999 * d, bits, trust), m)
    near = o["d_mask"] < 0.5
    assert near.sum() > 50
    up = _mask_rule(t + 1.001 * d, bits, trust) != m
    down = _mask_rule(t - 1.001 * d, bits, trust) != m
    assert np.all((up | down)[near])
    # both mask values occur near the flips
    assert 0 < m[near].mean() < 1


def test_mse_of_quantizer_matches_closed_form():
    # The oracle's own dequantised output on a long Gaussian row (whole-row RMS)
    # reproduces the closed-form MSE at Delta*: ties the grid, the step and alpha
    # together.
    n = 1 << 21
    for bits in (2, 4):
        x = np.random.default_rng(60 + bits).standard_normal((1, n))
        o = oracle.quantize(x, bits=bits, had=128, rms_group=n)
        _, d, m = oracle.alpha(bits)
        r = math.sqrt(np.mean(x ** 2))        # Parseval: the RMS of y
        err = np.mean((o["y"] - o["yhat"]) ** 2) / r ** 2
        assert err == pytest.approx(m, rel=0.01)


# ---------------------------------------------------------------------------
# Trust backward
# ---------------------------------------------------------------------------

def test_trust_bwd_zero_mask_and_single_index():
    n = 128
    g = np.random.default_rng(4).standard_normal((3, 2 * n))
    assert np.all(oracle.trust_bwd(g, np.zeros_like(g, dtype=np.uint8), had=n) == 0)
    H = scipy.linalg.hadamard(n).astype(np.float64)
    for i in [0, 3, 77, 127]:
        m = np.zeros_like(g, dtype=np.uint8)
        m[:, n + i] = 1
        out = oracle.trust_bwd(g, m, had=n)
        assert np.all(out[:, :n] == 0)
        np.testing.assert_allclose(out[:, n:], g[:, n + i:n + i + 1] * H[i][None, :] / math.sqrt(n),
                                   rtol=0, atol=1e-14)


def test_trust_bwd_is_linear_and_transposed():
    # <T(m.g), x> = <m.g, H x / sqrt n>: the backward is the adjoint of the forward
    # transform applied to the masked gradient.
    g = np.random.default_rng(8).standard_normal((2, 256))
    x = np.random.default_rng(9).standard_normal((2, 256))
    m = (np.random.default_rng(10).random((2, 256)) < 0.7).astype(np.uint8)
    lhs = np.sum(oracle.trust_bwd(g, m, had=128) * x)
    y = oracle.quantize(x, bits=4)["y"]
    rhs = np.sum(m * g * y)
    assert lhs == pytest.approx(rhs, rel=1e-12)


# ---------------------------------------------------------------------------
# Integer GEMM and dequantisation
# ---------------------------------------------------------------------------

def test_gemm_matches_numpy_matmul():
    g = np.random.default_rng(13)
    a = g.integers(-128, 128, size=(37, 96)).astype(np.int8)
    b = g.integers(-128, 128, size=(23, 96)).astype(np.int8)
    assert np.array_equal(oracle.gemm_i8(a, b), a.astype(np.int64) @ b.astype(np.int64).T)


def test_gemm_closed_forms():
    K = 2048
    a = np.full((3, K), 15, dtype=np.int8)
    assert np.all(oracle.gemm_i8(a, a) == 225 * K)
    e = np.zeros((4, K), dtype=np.int8)
    for i in range(4):
        e[i, i * 7] = 1
    b = np.arange(5 * K, dtype=np.int64).reshape(5, K) % 100 - 50
    acc = oracle.gemm_i8(e, b.astype(np.int8))
    assert np.array_equal(acc, b[:, [0, 7, 14, 21]].T)
    assert oracle.gemm_i8(np.zeros((2, 0), np.int8), np.zeros((3, 0), np.int8)).sum() == 0


def test_dequant_linear_reproduces_float_product():
    # (q+1/2) Delta codes: Y = acc * Delta_a/2 * Delta_b/2 equals the product of the
    # dequantised operands (orthogonality keeps it in the Hadamard domain).
    g = np.random.default_rng(14)
    qa = g.integers(-8, 8, size=(5, 64))
    qb = g.integers(-8, 8, size=(6, 64))
    da, db = g.random(5) + 0.1, g.random(6) + 0.1
    acc = oracle.gemm_i8((2 * qa + 1).astype(np.int8), (2 * qb + 1).astype(np.int8))
    y = oracle.dequant_linear(acc, da, db)
    ref = ((qa + 0.5) * da[:, None]) @ ((qb + 0.5) * db[:, None]).T
    np.testing.assert_allclose(y, ref, rtol=1e-13)


# ---------------------------------------------------------------------------
# bfloat16 rounding
# ---------------------------------------------------------------------------

def test_bf16_rne_matches_torch_on_fp32_values():
    g = np.random.default_rng(15)
    v = np.concatenate([
        g.standard_normal(100000).astype(np.float32),
        (g.standard_normal(20000) * 1e-38).astype(np.float32),   # subnormal range
        np.clip(g.standard_normal(1000) * 3e38, -3.4e38, 3.4e38).astype(np.float32),   # near the top of the range
        np.array([0.0, -0.0, 1.0, -2.5, np.inf, -np.inf], dtype=np.float32),
    ])
    ref = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.bf16_rne(v.astype(np.float64)), ref)


def test_bf16_rne_ties_to_even_and_single_rounding():
    one = 1.0
    assert oracle.bf16_rne(np.array([one + 2 ** -8]))[0] == 0x3F80        # tie -> even (1.0)
    assert oracle.bf16_rne(np.array([one + 3 * 2 ** -8]))[0] == 0x3F82    # tie -> even (up)
    # just above a tie in fp64 (not representable in fp32): must round up, which a
    # double rounding through fp32 would get wrong
    assert oracle.bf16_rne(np.array([one + 2 ** -8 + 2 ** -40]))[0] == 0x3F81
    assert oracle.bf16_rne(np.array([-(one + 2 ** -8 + 2 ** -40)]))[0] == 0xBF81
    vals = oracle.bf16_bits_to_f64(np.array([0x3F80, 0xC020, 0x0001], dtype=np.uint16))
    assert list(vals) == [1.0, -2.5, 2.0 ** -133]


# --- per-group-scaled linear layer -------------------------------------------
def _grouped_case(M, N, K, seed):
    g = np.random.default_rng(seed)
    a = (2 * g.integers(-8, 8, size=(M, K)) + 1).astype(np.int8)
    b = (2 * g.integers(-8, 8, size=(N, K)) + 1).astype(np.int8)
    sa = np.exp(g.uniform(-6, -2, size=(M, K // 128)))
    sb = np.exp(g.uniform(-6, -2, size=(N, K // 128)))
    return a, b, sa, sb


def test_grouped_linear_equals_product_of_scaled_operands():
    # Scale-then-multiply with a library matmul against the oracle's
    # multiply-then-scale per group: the same bilinear form in another order.
    a, b, sa, sb = _grouped_case(7, 9, 512, 1)
    y, mag = oracle.linear_grouped(a, b, sa, sb)
    at = a.astype(np.float64) * np.repeat(sa / 2, 128, axis=1)
    bt = b.astype(np.float64) * np.repeat(sb / 2, 128, axis=1)
    ref = at @ bt.T
    assert np.allclose(y, ref, rtol=0, atol=1e-12 * np.max(mag))
    assert np.all(mag >= np.abs(y) * (1 - 1e-15))


def test_grouped_linear_with_row_constant_scales_is_the_row_scaled_layer():
    # Constant scales along K reduce the grouped layer to one int32 accumulator
    # per output and the per-row dequantisation.
    a, b, _, _ = _grouped_case(5, 6, 384, 2)
    ra = np.exp(np.random.default_rng(3).uniform(-5, -1, size=5))
    rb = np.exp(np.random.default_rng(4).uniform(-5, -1, size=6))
    y, _ = oracle.linear_grouped(a, b, np.repeat(ra[:, None], 3, axis=1), np.repeat(rb[:, None], 3, axis=1))
    ref = oracle.dequant_linear(oracle.gemm_i8(a, b), ra, rb)
    assert np.allclose(y, ref, rtol=1e-14, atol=0)


def test_grouped_linear_groups_are_independent():
    # Zeroing the scales of one group removes exactly that group's K-slice.
    a, b, sa, sb = _grouped_case(4, 5, 512, 5)
    sa0 = sa.copy()
    sa0[:, 2] = 0.0
    y0, _ = oracle.linear_grouped(a, b, sa0, sb)
    a_cut = a.copy()
    a_cut[:, 256:384] = 0
    y_cut, _ = oracle.linear_grouped(a_cut, b, sa, sb)
    assert np.allclose(y0, y_cut, rtol=1e-14, atol=0)


def test_e4m3_helpers_match_torch():
    # the test-side E4M3 codec against torch's float8_e4m3fn conversion
    import sys, os
    sys.path.insert(0, os.path.dirname(__file__))
    from parity import e4m3_decode, e4m3_encode_int
    c = np.arange(-15, 16)
    ref = torch.tensor(c, dtype=torch.float32).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(e4m3_encode_int(c), ref)
    allb = np.arange(256, dtype=np.uint8)
    tv = torch.from_numpy(allb).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    dv = e4m3_decode(allb)
    assert np.array_equal(np.isnan(tv), np.isnan(dv))
    assert np.array_equal(tv[~np.isnan(tv)], dv[~np.isnan(dv)])


def test_trust_bwd_linear_composition_pins():
    # the fused backward is the product followed by the pinned trust backward: pin
    # the product by a brute-force triple loop on a tiny case, and the whole chain
    # by two closed forms (all-ones mask and w_hat = [I; 0]: H G / sqrt(n) with G
    # the first K columns of g_y; all-zero mask: 0)
    g = np.random.default_rng(21)
    gy = g.standard_normal((3, 5))
    w = g.standard_normal((5, 16))
    m = g.integers(0, 2, size=(3, 16)).astype(np.uint8)
    G = np.zeros((3, 16))
    for i in range(3):
        for k in range(16):
            G[i, k] = sum(gy[i, n] * w[n, k] for n in range(5))
    assert np.allclose(oracle.trust_bwd_linear(gy, w, m, had=16), oracle.trust_bwd(G, m, had=16),
                       rtol=0, atol=1e-12)
    gy = g.standard_normal((4, 40))
    eye = np.zeros((40, 32))
    eye[:32, :32] = np.eye(32)
    H = scipy.linalg.hadamard(32) / np.sqrt(32)
    out = oracle.trust_bwd_linear(gy, eye, np.ones((4, 32), np.uint8), had=32)
    assert np.allclose(out, gy[:, :32] @ H.T, rtol=0, atol=1e-12)
    assert not oracle.trust_bwd_linear(gy, eye, np.zeros((4, 32), np.uint8), had=32).any()


def _golden(name):
    path = os.path.join(os.path.dirname(__file__), "golden", "pages_parameters.txt")
    with open(path) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                k, v = line.split()[:2]
                if k == name:
                    return float(v)
    raise KeyError(name)


def test_one_bit_outer_trust_from_the_pages():
    # The 1-bit runs widen the outer trust region with s* (printed by the pages), passed as
    # T: for T >= 1 the mask keeps |t| <= 2^(b-1) + (T-1)/2 = 1.15 at b = 1. On a long
    # N(0,1) row with whole-row RMS, t = y / (alpha_1 r) and the masked fraction is the
    # Gaussian tail mass beyond 1.15 alpha_1.
    s_star = _golden("outer_trust_scale_1bit")
    assert s_star == 1.30
    x = np.random.default_rng(13).standard_normal((1, 1 << 20))
    o = oracle.quantize(x, bits=1, had=128, rms_group=1 << 20, trust=s_star)
    edge = 1.0 + (s_star - 1.0) / 2.0
    assert np.array_equal(o["mask"], (np.abs(o["t"]) <= edge).astype(np.uint8))
    a1, _, _ = oracle.alpha(1)
    p = 2 * scipy.stats.norm.sf(edge * a1)
    rate = 1 - o["mask"].mean()
    assert abs(rate - p) < 4 * math.sqrt(p * (1 - p) / x.size)


def test_linear_bf16_pins():
    # brute-force triple loop on a tiny case, and the Hadamard-invariance the pages state:
    # transforming both operands' rows by the same orthogonal H leaves the product unchanged
    g = np.random.default_rng(23)
    x = g.standard_normal((3, 8))
    w = g.standard_normal((5, 8))
    y = oracle.linear_bf16(x, w)
    for i in range(3):
        for j in range(5):
            assert abs(y[i, j] - sum(x[i, k] * w[j, k] for k in range(8))) < 1e-12
    H = scipy.linalg.hadamard(8) / np.sqrt(8)
    assert np.allclose(oracle.linear_bf16(x @ H.T, w @ H.T), y, rtol=0, atol=1e-12)
