"""Pins of the oracle's counter-based Gaussian stream."""

import math

import numpy as np
from scipy import stats

from oracle import rng


def test_splitmix64_reference_vector(golden):
    lines = golden("splitmix64.txt")
    seed, want = int(lines[0]), [int(x) for x in lines[1:]]
    got, _ = rng.splitmix64(seed, len(want))
    assert got == want


def test_gaussian_moments_and_ks():
    z = np.concatenate([rng.gaussians(7, h, 4000) for h in range(25)])
    n = z.size
    assert abs(z.mean()) < 5 / math.sqrt(n)
    assert abs(z.var() - 1.0) < 5 * math.sqrt(2.0 / n)
    assert stats.kstest(z, "norm").pvalue > 1e-4


def test_streams_differ_and_repeat():
    a = rng.qjl_matrix(42, 0, 5)
    b = rng.qjl_matrix(42, 1, 5)
    c = rng.qjl_matrix(43, 0, 5)
    assert a.shape == (5, 5)
    assert np.array_equal(a, rng.qjl_matrix(42, 0, 5))
    assert not np.allclose(a, b) and not np.allclose(a, c)
    # prefix property: a smaller matrix uses the first m*m draws of the stream
    assert np.array_equal(rng.qjl_matrix(42, 0, 2).reshape(-1), rng.gaussians(42, 0, 4))
