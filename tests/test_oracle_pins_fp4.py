"""Pins of the oracle's FP4 (E2M1) grid variant against things other than itself.

The pages report that QuEST also trains on an FP4 grid and that FP4 does slightly
worse than INT4, which the authors put down to a higher Gaussian MSE once
clipping is allowed (pith.science review, "What carries the argument" and its
results list). The oracle's reading: the same Hadamard transform and RMS, the 15
signed E2M1 values scaled by Delta = s* r with s* the Gaussian-MSE-optimal scale,
round to nearest, and a trust mask that keeps an element whose error is at most
T/2 of the grid interval holding it. These tests pin each step:

* the E2M1 decode table and round-to-nearest-even against ml_dtypes' float4_e2m1fn;
* the closed-form Gaussian MSE against numerical quadrature and Monte Carlo;
* s* against a brute-force scan, and the pages' qualitative claim (FP4 MSE above INT4's);
* the quantizer on hand-derived tiny inputs, and its outputs against their definitions
  recomputed independently (scipy's Hadamard matrix, numpy nearest-level search);
* the mask rate on Gaussian data against the tail mass 2(1 - Phi(s* (6 + T))).
"""
import math

import numpy as np
import pytest
from scipy import integrate, linalg, stats

import oracle

ml_dtypes = pytest.importorskip("ml_dtypes")

GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])   # OCP E2M1 magnitudes


def test_e2m1_decode_matches_library():
    lib = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)
    ours = np.array([oracle.e2m1_value(c) for c in range(16)])
    assert np.array_equal(ours, lib)
    assert np.array_equal(np.signbit(ours), np.signbit(lib))


def test_e2m1_round_matches_library():
    g = np.random.default_rng(0)
    # every tie point, both signs, the saturating range, +-0 and random values
    mids = 0.5 * (GRID[1:] + GRID[:-1])
    t = np.concatenate([mids, -mids, GRID, -GRID, [6.5, 7.0, 100.0, -9.0, 1e-30, -1e-30],
                        g.normal(0, 3, 4000)]).astype(np.float32)
    lib = t.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF
    ours = np.array([oracle.e2m1_round(float(v)) for v in t], dtype=np.uint8)
    bad = np.nonzero(lib != ours)[0]
    assert bad.size == 0, [(float(t[i]), int(lib[i]), int(ours[i])) for i in bad[:5]]


def test_fp4_mse_closed_form_against_quadrature():
    for s in (0.2, 0.48, 0.9):
        def integrand(x):
            q = GRID[np.argmin(np.abs(np.abs(x) / s - GRID))] * np.sign(x) * s
            return (x - q) ** 2 * stats.norm.pdf(x)
        # integrate cell by cell (the integrand jumps at the midpoints)
        edges = np.concatenate([[-12.0], -s * 0.5 * (GRID[1:] + GRID[:-1])[::-1], [0.0],
                                s * 0.5 * (GRID[1:] + GRID[:-1]), [12.0]])
        total = sum(integrate.quad(integrand, a, b, epsabs=1e-14, epsrel=1e-12)[0]
                    for a, b in zip(edges[:-1], edges[1:]))
        assert abs(oracle.fp4_gauss_mse(s) - total) < 1e-10 * max(1.0, total)


def test_fp4_scale_is_the_minimiser():
    s, mse = oracle.alpha_fp4()
    scan = np.linspace(0.05, 1.5, 2901)
    vals = np.array([oracle.fp4_gauss_mse(v) for v in scan])
    i = int(np.argmin(vals))
    assert abs(scan[i] - s) <= scan[1] - scan[0]
    fine = np.linspace(s - 1e-4, s + 1e-4, 2001)
    fv = np.array([oracle.fp4_gauss_mse(v) for v in fine])
    assert abs(fine[int(np.argmin(fv))] - s) <= 2e-7
    assert mse <= vals.min() + 1e-15
    # unimodal on the scan: decreasing, then increasing
    d = np.diff(vals)
    assert np.all(d[:i] < 0) and np.all(d[i:] > 0)


def test_fp4_mse_monte_carlo():
    s, mse = oracle.alpha_fp4()
    x = np.random.default_rng(1).standard_normal(4_000_000)
    q = GRID[np.argmin(np.abs(np.abs(x)[:, None] / s - GRID[None, :]), axis=1)] * np.sign(x) * s
    e = (x - q) ** 2
    assert abs(e.mean() - mse) < 4 * e.std() / math.sqrt(x.size)


def test_fp4_gaussian_mse_above_int4():
    # the pages' account of FP4 trailing INT4: higher Gaussian MSE once clipping is allowed
    _, mse_fp4 = oracle.alpha_fp4()
    _, _, mse_int4 = oracle.alpha(4)
    assert mse_fp4 > mse_int4


def test_fp4_tiny_hand_cases():
    s, _ = oracle.alpha_fp4()
    # n = 2: y = ((a+b)/sqrt2, (a-b)/sqrt2); x = (1, 1): y = (sqrt2, 0), rms = 1,
    # Delta = s*, t0 = sqrt2 / s* = 2.90 -> grid value 3 (code 0b0101), t1 = 0 -> +0
    o = oracle.quantize_fp4(np.array([[1.0, 1.0]]), had=2)
    assert o["scale"][0, 0] == pytest.approx(s, rel=1e-15)
    assert list(o["code"][0]) == [5, 0]
    assert o["yhat"][0, 0] == pytest.approx(3 * s, rel=1e-15)
    assert list(o["mask"][0]) == [1, 1]
    # n = 4, x = e0: y = (1/2)(1,1,1,1), rms = 1/2, t = 1/s* = 2.05 -> 2 (code 0b0100)
    o = oracle.quantize_fp4(np.array([[1.0, 0.0, 0.0, 0.0]]), had=4)
    assert list(o["code"][0]) == [4, 4, 4, 4]
    # x = (1, -1): y = (0, sqrt2) -> codes (+0, 3)
    o = oracle.quantize_fp4(np.array([[1.0, -1.0]]), had=2)
    assert list(o["code"][0]) == [0, 5]
    # x = (-1, -1): y = (-sqrt2, 0) -> code 0b1101 (-3) and +0
    o = oracle.quantize_fp4(np.array([[-1.0, -1.0]]), had=2)
    assert list(o["code"][0]) == [13, 0]
    # a zero group: Delta = 0, codes 0, mask 1
    o = oracle.quantize_fp4(np.zeros((1, 8)), had=8)
    assert o["scale"][0, 0] == 0 and not o["code"].any() and o["mask"].all()


@pytest.mark.parametrize("had,rms_group,trust", [(128, 128, 1.0), (32, 256, 1.0), (64, 64, 0.6),
                                                 (16, 512, 1.5)])
def test_fp4_quantizer_against_definitions(had, rms_group, trust):
    g = np.random.default_rng(had + rms_group)
    x = g.standard_t(3, size=(7, 512))
    o = oracle.quantize_fp4(x, had=had, rms_group=rms_group, trust=trust)
    H = linalg.hadamard(had) / math.sqrt(had)
    y = (x.reshape(7, -1, had) @ H.T).reshape(7, 512)
    assert np.allclose(o["y"], y, rtol=0, atol=1e-12)
    rms = np.sqrt((y.reshape(7, -1, rms_group) ** 2).mean(axis=2))
    s, _ = oracle.alpha_fp4()
    assert np.allclose(o["scale"], s * rms, rtol=1e-14)
    delta = np.repeat(s * rms, rms_group, axis=1)
    t = y / delta
    assert np.allclose(o["t"], t, rtol=1e-13)
    # nearest grid value by exhaustive search
    cand = np.concatenate([GRID, -GRID[1:]])
    dist = np.abs(t[..., None] - cand)
    best = dist.min(axis=-1)
    assert np.allclose(np.abs(t - o["value"]), best, atol=1e-12)
    assert np.array_equal(np.abs(o["value"]), np.abs(np.vectorize(oracle.e2m1_value)(o["code"])))
    assert np.allclose(o["yhat"], o["value"] * delta, rtol=1e-15)
    # mask: error within T/2 of the grid interval that holds |t| ([4, 6] beyond 6)
    a = np.abs(t)
    w = np.where(a < 2, 0.5, np.where(a < 4, 1.0, 2.0))
    assert np.array_equal(o["mask"], (np.abs(t - o["value"]) <= 0.5 * trust * w).astype(np.uint8))
    if trust >= 1.0:
        assert np.array_equal(o["mask"], (a <= 6 + trust).astype(np.uint8))


def test_fp4_mask_rate_matches_tail_mass():
    # whole-row RMS on a long Gaussian row: t ~ N(0,1) / s*, masked iff |t| > 7
    x = np.random.default_rng(5).standard_normal((1, 1 << 20))
    o = oracle.quantize_fp4(x, had=128, rms_group=1 << 20)
    s, _ = oracle.alpha_fp4()
    p = 2 * stats.norm.sf(7 * s)
    n = x.size
    rate = 1 - o["mask"].mean()
    assert abs(rate - p) < 4 * math.sqrt(p * (1 - p) / n)


def test_fp4_boundary_distances():
    x = np.random.default_rng(6).standard_normal((5, 256))
    o = oracle.quantize_fp4(x, had=128, trust=1.0)
    a = np.abs(o["t"])
    mids = 0.5 * (GRID[1:] + GRID[:-1])
    d = np.minimum(a, np.abs(a[..., None] - mids).min(axis=-1))
    assert np.allclose(o["d_round"], d, atol=1e-15)
    assert np.allclose(o["d_mask"], np.abs(a - 7.0), atol=1e-15)


# Mask-exemption distance on the FP4 grid. The mask m = [|t - Q| <= (T/2) w(t)]
# (the half-interval rule read on the local interval width) changes value only at
# |t| = 6 + T beyond the grid and, for T < 1, at v_k + (T/2) w_k and
# v_(k+1) - (T/2) w_k inside each interval [v_k, v_(k+1)] of width w_k. d_mask must
# be the distance to the nearest of them, or the parity checks' exemption band
# would hide mask mismatches.

def _fp4_flip_points(trust):
    pts = [6.0 + trust]
    if trust < 1.0:
        for k in range(7):
            w = GRID[k + 1] - GRID[k]
            pts += [GRID[k] + 0.5 * trust * w, GRID[k + 1] - 0.5 * trust * w]
    return np.array(pts)


def _fp4_edge_input(trust, seed, rows=6, cols=512):
    """x whose groups put many |t| within 0.3 of the flip points: with t = y / (s* r)
    and r = rms(y), t = y exactly when sum(y^2) = 128 / s*^2 (the last value of each
    group makes it so); x = H y / sqrt(128)."""
    g = np.random.default_rng(seed)
    s, _ = oracle.alpha_fp4()
    budget = 128 / s ** 2
    f = _fp4_flip_points(trust)
    H = linalg.hadamard(128).astype(np.float64) / math.sqrt(128)
    y = np.empty((rows, cols))
    for r in range(rows):
        for b0 in range(0, cols, 128):
            v = g.standard_normal(128) * 0.3
            n_near = int(min(48, 0.5 * budget / (np.max(f) + 0.3) ** 2))
            v[:n_near] = (g.choice(f, n_near) + g.uniform(-0.3, 0.3, n_near)) * np.sign(g.standard_normal(n_near))
            rest = budget - np.sum(v[:127] ** 2)
            assert rest > 0
            v[127] = math.sqrt(rest)
            y[r, b0:b0 + 128] = g.permutation(v)
    return (y.reshape(rows, cols // 128, 128) @ H).reshape(rows, cols)


def _fp4_mask_rule(t, trust):
    a = np.abs(t)
    q = GRID[np.abs(a[..., None] - GRID).argmin(axis=-1)]   # nearest magnitude (no ties here)
    w = np.where(a < 2, 0.5, np.where(a < 4, 1.0, 2.0))
    return (np.abs(a - q) <= 0.5 * trust * w).astype(np.uint8)


@pytest.mark.parametrize("trust", [0.5, 0.8, 1.0, 1.3, 2.0])
def test_fp4_mask_flip_distance(trust):
    x = _fp4_edge_input(trust, 90 + int(10 * trust))
    o = oracle.quantize_fp4(x, had=128, trust=trust)
    a, d = np.abs(o["t"]), o["d_mask"]
    ref = np.abs(a[..., None] - _fp4_flip_points(trust)).min(axis=-1)
    np.testing.assert_allclose(d, ref, rtol=0, atol=1e-12)
    assert np.sum(ref < 0.3) > 50
    # the distance is tight: less than d keeps the mask, just more flips it one way
    m = o["mask"]
    assert np.array_equal(_fp4_mask_rule(o["t"], trust), m)
    for sg in (-1.0, 1.0):
        assert np.array_equal(_fp4_mask_rule(o["t"] + sg * 0.999 * d, trust), m)
    near = d < 0.2
    flips = (_fp4_mask_rule(o["t"] + 1.001 * d, trust) != m) | (_fp4_mask_rule(o["t"] - 1.001 * d, trust) != m)
    assert np.all(flips[near])
