"""Pins of the oracle's Gaussian Lloyd-Max quantizers.

Each check ties the oracle to something other than its own formulas: a
printed table (Max 1960; the TurboQuant reference README's distortion
table), a closed form, numerical quadrature, Monte Carlo, or the
high-rate asymptote.
"""

import math

import numpy as np
import pytest
from scipy.integrate import quad

from oracle import codebook as cb


def test_one_bit_closed_form():
    levels, thr, d = cb.lloyd_max(1)
    # E[Z | Z > 0] = 2 phi(0) = sqrt(2/pi); D = 1 - 2/pi.
    assert np.allclose(levels, [-math.sqrt(2 / math.pi), math.sqrt(2 / math.pi)], atol=1e-14)
    assert np.array_equal(thr, [0.0])
    assert abs(d - (1 - 2 / math.pi)) < 1e-14


def test_max_1960_table(golden):
    for line in golden("lloyd_max_gaussian.txt"):
        b_s, lv_s, th_s, d_s = [p.strip() for p in line.split("|")]
        b = int(b_s)
        levels, thr, dist = cb.lloyd_max(b)
        half = len(levels) // 2
        # tolerance: half a unit of the printed last digit, at least 2e-4
        tol = lambda s: max(2e-4, 0.5 * 10.0 ** -len(s.split(".")[1]))
        for got, s in zip(levels[half:], lv_s.split()):
            assert abs(got - float(s)) <= tol(s), (b, got, s)
        assert np.array_equal(-levels[:half][::-1], levels[half:])
        for got, s in zip(thr[half:], th_s.split()):
            assert abs(got - float(s)) <= tol(s), (b, got, s)
        assert thr[half - 1] == 0.0
        assert abs(dist - float(d_s)) <= 0.5 * 10.0 ** -len(d_s.split(".")[1]), (b, dist, d_s)


def test_turboquant_distortion_table(golden):
    for line in golden("turboquant_distortion.txt"):
        b, theory, empirical = line.split()
        d = cb.lloyd_max(int(b))[2]
        assert abs(d - float(empirical)) <= 0.0006, (b, d, empirical)
        assert abs(d - float(theory)) <= 0.005, (b, d, theory)


@pytest.mark.parametrize("b", [2, 3, 4])
def test_conditions_by_quadrature(b):
    """Centroid and distortion checked by adaptive quadrature, not by the closed forms."""
    levels, thr, dist = cb.lloyd_max(b)
    edges = np.concatenate([[-np.inf], thr, [np.inf]])
    pdf = lambda z: math.exp(-0.5 * z * z) / math.sqrt(2 * math.pi)
    total = 0.0
    for k, lv in enumerate(levels):
        a, c = edges[k], edges[k + 1]
        p = quad(pdf, a, c, epsabs=1e-15, epsrel=1e-13)[0]
        m = quad(lambda z: z * pdf(z), a, c, epsabs=1e-15, epsrel=1e-13)[0] / p
        assert abs(m - lv) < 1e-10
        total += quad(lambda z: (z - lv) ** 2 * pdf(z), a, c, epsabs=1e-15, epsrel=1e-13)[0]
    # nearest-neighbour condition: thresholds halfway between levels
    assert np.allclose(thr, 0.5 * (levels[:-1] + levels[1:]), atol=1e-15)
    assert abs(total - dist) < 1e-12


def test_monte_carlo_distortion():
    rng = np.random.default_rng(42)
    z = rng.standard_normal(2_000_000)
    for b in range(1, 9):
        levels, _, dist = cb.lloyd_max(b)
        zq = cb.dequantize(cb.quantize(z, b), b)
        mse = np.mean((z - zq) ** 2)
        se = np.std((z - zq) ** 2) / math.sqrt(z.size)
        assert abs(mse - dist) < 6 * se, (b, mse, dist)


def test_high_rate_asymptote():
    # Panter-Dite: D(b) 4^b -> pi sqrt(3) / 2 as b grows, from below.
    limit = math.pi * math.sqrt(3) / 2
    ratios = [cb.lloyd_max(b)[2] * 4 ** b for b in range(1, 9)]
    assert all(np.diff(ratios) > 0)
    assert abs(ratios[-1] - limit) / limit < 0.01


def test_distortion_convex_decreasing():
    d = cb.distortion_table()
    assert d[0] == 1.0
    steps = -np.diff(d)
    assert np.all(steps > 0) and np.all(np.diff(steps) < 0)


def test_threshold_ties_take_lower_code():
    for b in range(1, 9):
        _, thr, _ = cb.lloyd_max(b)
        codes = cb.quantize(thr, b)
        assert np.array_equal(codes, np.arange(len(thr)))
        up = cb.quantize(np.nextafter(thr, np.inf), b)
        assert np.array_equal(up, np.arange(1, len(thr) + 1))
        assert cb.quantize(np.array([-1e9, 1e9]), b).tolist() == [0, 2 ** b - 1]


def test_symmetry():
    for b in range(1, 9):
        levels, thr, _ = cb.lloyd_max(b)
        assert np.array_equal(levels, -levels[::-1])
        assert np.array_equal(thr, -thr[::-1])
