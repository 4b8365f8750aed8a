"""Pins of the oracle's calibration: eigenbasis, d_eff, kappa, scales, water-filling."""

import itertools
import math

import numpy as np
import pytest
from scipy import linalg as sla

from oracle import calibration as cal
from oracle import codebook as cb


def _spectrum_matrix(lam, seed=0):
    d = len(lam)
    q, r = np.linalg.qr(np.random.default_rng(seed).standard_normal((d, d)))
    q = q * np.sign(np.diag(r))
    return (q * np.asarray(lam, float)) @ q.T, q


def test_eigenbasis_orthonormal_and_residual():
    rng = np.random.default_rng(42)
    x = rng.standard_normal((300, 32)) * np.linspace(10, 0.1, 32)
    c = cal.second_moment(x)
    lam, v = cal.eigenbasis(c)
    assert np.all(np.diff(lam) <= 0) and np.all(lam >= 0)
    assert np.max(np.abs(v.T @ v - np.eye(32))) < 1e-12
    assert np.linalg.norm(c @ v - v * lam) / np.linalg.norm(c) < 1e-12
    # sign convention: the largest-magnitude entry of each eigenvector is positive
    for i in range(32):
        j = int(np.argmax(np.abs(v[:, i])))
        assert v[j, i] > 0


def test_eigenvalues_against_svd_and_general_solver():
    """The spectrum from two other routes: singular values of X, and the general eig solver."""
    rng = np.random.default_rng(1)
    x = rng.standard_normal((200, 24)) @ rng.standard_normal((24, 24))
    lam, _ = cal.eigenbasis(cal.second_moment(x))
    sv = np.linalg.svd(x, compute_uv=False)
    assert np.allclose(lam, sv ** 2 / x.shape[0], rtol=1e-10, atol=1e-12)
    w = np.sort(np.real(sla.eig(cal.second_moment(x))[0]))[::-1]
    assert np.allclose(lam, w, rtol=1e-9)


def test_second_moment_is_uncentred():
    x = np.ones((10, 4)) * 3.0
    # centred covariance would be 0; the uncentred second moment is 9 everywhere
    assert np.allclose(cal.second_moment(x), 9.0)


def test_deff_flat_spectrum_equals_d():
    for d in (32, 128, 256):
        assert cal.effective_dim(np.ones(d)) == d
        assert cal.spectral_gap(np.ones(d), d) == math.inf


def test_deff_rank4_equal_is_4():
    lam = np.zeros(32)
    lam[:4] = 7.0
    assert cal.participation_ratio(lam) == 4.0
    assert cal.effective_dim(lam) == 4
    assert cal.spectral_gap(lam, 4) == math.inf      # lambda[4] = 0
    # the same from sampled rank-4 data at large N
    rng = np.random.default_rng(42)
    u, _ = np.linalg.qr(rng.standard_normal((32, 4)))
    x = rng.standard_normal((100_000, 4)) @ u.T
    lam_s, _ = cal.eigenbasis(cal.second_moment(x))
    assert cal.effective_dim(lam_s) == 4


def test_deff_sharp_gap_spectrum():
    # conftest fixture sharp_gap_kv_data: 8 dims at 50, 24 at 1 (population).
    lam = np.array([50.0] * 8 + [1.0] * 24)
    pr = (8 * 50 + 24) ** 2 / (8 * 2500 + 24)
    assert abs(cal.participation_ratio(lam) - pr) < 1e-12
    assert cal.effective_dim(lam) == 9                 # 8.98 rounds to 9
    assert cal.spectral_gap(lam, 8) == 50.0
    assert cal.spectral_gap(lam, 9) == 1.0


def test_deff_marchenko_pastur_sampled_identity():
    # A sampled identity at N = 256, d = 32 has PR close to d / (1 + d / N) (not d).
    vals = []
    for s in range(20):
        x = np.random.default_rng(s).standard_normal((256, 32))
        vals.append(cal.participation_ratio(cal.eigenbasis(cal.second_moment(x))[0]))
    assert abs(np.mean(vals) - 32 / (1 + 32 / 256)) < 0.5


def test_deff_rounds_half_even():
    # Integer spectra whose participation ratio is exactly k + 1/2:
    # (2,1,1,1,1): 36/8 = 4.5 -> 4;  (5,5,2,1,1): 196/56 = 3.5 -> 4.
    assert cal.participation_ratio(np.array([2.0, 1, 1, 1, 1])) == 4.5
    assert cal.effective_dim(np.array([2.0, 1, 1, 1, 1])) == 4
    assert cal.participation_ratio(np.array([5.0, 5, 2, 1, 1])) == 3.5
    assert cal.effective_dim(np.array([5.0, 5, 2, 1, 1])) == 4


def test_scales():
    lam = np.array([4.0, 3.0, 2.0, 1.0])
    s = cal.scales(lam, normalize=True)
    assert abs(np.sum(s ** 2) - 1.0) < 1e-15
    assert np.allclose(cal.scales(lam, normalize=False), [2.0, math.sqrt(3), math.sqrt(2), 1.0])
    assert np.all(cal.scales(np.zeros(4), True) == 0)


def _brute_force(lam, n_bits, max_bits):
    dist = cb.distortion_table(max_bits)
    best = None
    for b in itertools.product(range(max_bits + 1), repeat=len(lam)):
        if sum(b) != n_bits:
            continue
        cost = sum(l * dist[k] for l, k in zip(lam, b))
        if best is None or cost < best - 1e-15:
            best = cost
    return best


@pytest.mark.parametrize("lam,n_bits", [
    ([5.0, 2.0, 1.0], 6), ([100.0, 1.0, 1.0, 0.5], 9), ([3.0, 3.0, 1.0, 1.0], 7),
    ([1000.0, 10.0, 1.0], 14), ([1.0, 1e-3, 1e-6, 0.0], 5)])
def test_water_fill_optimal_by_brute_force(lam, n_bits):
    lam = np.array(lam)
    b = cal.water_fill(lam, n_bits, 8)
    dist = cb.distortion_table(8)
    assert b.sum() == n_bits
    assert abs(np.sum(lam * dist[b]) - _brute_force(lam, n_bits, 8)) < 1e-12


def test_water_fill_budget_monotone_and_cap():
    rng = np.random.default_rng(3)
    lam = np.sort(rng.exponential(size=128) ** 3)[::-1]
    for n in (0, 1, 77, 384, 1024):
        b = cal.water_fill(lam, n, 8)
        assert b.sum() == n and b.max() <= 8
        assert np.all(np.diff(b) <= 0)             # sorted spectrum -> non-increasing bits
    with pytest.raises(ValueError):
        cal.water_fill(lam, 8 * 128 + 1, 8)


def test_water_fill_flat_is_uniform():
    b = cal.water_fill(np.ones(32), 96, 8)
    assert np.all(b == 3)
    b = cal.water_fill(np.ones(32), 100, 8)        # remainder to the lowest indices
    assert np.all(b[:4] == 4) and np.all(b[4:] == 3)


def test_water_fill_tracks_reverse_water_filling():
    # High-rate reverse water-filling: b_i ~ max(0, log2(lambda_i / theta) / 2).
    lam = np.concatenate([np.logspace(3, 2, 4), np.ones(124)])
    b = cal.water_fill(lam, 380, 8)
    lo, hi = 1e-9, 1e9
    for _ in range(200):
        th = math.sqrt(lo * hi)
        tot = np.sum(np.maximum(0, 0.5 * np.log2(lam / th)))
        lo, hi = (th, hi) if tot > 380 else (lo, th)
    cont = np.maximum(0, 0.5 * np.log2(lam / th))
    assert np.all(np.abs(b - cont) <= 1.0 + 1e-9)


def test_finalize_budget_identity():
    rng = np.random.default_rng(42)
    x = rng.standard_normal((512, 32)) * np.concatenate([np.full(8, math.sqrt(50)), np.ones(24)])
    c = cal.calibrate(x, avg_bits=3.0, is_key=True, qjl=True, seed=42, stream=0)
    assert c.total_bits == 96 and c.m == c.d_eff
    assert c.bits.sum() + c.m == c.total_bits          # codes + QJL bits = budget exactly
    assert c.words == 3 and c.S.shape == (c.m, c.m)
    v = cal.calibrate(x, avg_bits=3.0, is_key=False, seed=42, stream=1)
    assert v.m == 0 and v.bits.sum() == 96
    with pytest.raises(ValueError):
        cal.calibrate(x, avg_bits=3.01, is_key=False)
    o = cal.calibrate(x, avg_bits=3.0, is_key=True, d_eff_override=4)
    assert o.m == 4 and o.d_eff == c.d_eff


# ---------------------------------------------------------------- variants
def test_cumulative_variance_d_eff_exact_spectra():
    """Smallest k whose top-k eigenvalues hold the fraction of the trace:
    flat (0.9 x 32 = 28.8 -> 29), four equal spikes (3.6 -> 4), a spiked
    spectrum (0.9 x 208 = 187.2 reached at 100+50+20+10+8 ones -> 12), and an
    exact tie (half of 4 equal values is reached at 2, not 3)."""
    assert cal.effective_dim(np.ones(32), cumvar=0.9) == 29
    assert cal.effective_dim(np.array([1.0] * 4 + [0.0] * 28), cumvar=0.9) == 4
    spiked = np.array([100.0, 50.0, 20.0, 10.0] + [1.0] * 28)
    assert cal.effective_dim(spiked, cumvar=0.9) == 12
    assert cal.effective_dim(spiked) == 3            # participation ratio 3.32 for comparison
    assert cal.effective_dim(np.ones(4), cumvar=0.5) == 2
    assert cal.effective_dim(np.zeros(8), cumvar=0.9) == 8
    assert cal.effective_dim(np.ones(8), cumvar=1.0) == 8


def test_cumulative_variance_d_eff_in_the_record():
    x = np.random.default_rng(11).standard_normal((4000, 32)) * np.concatenate([np.full(4, 10.0), np.ones(28)])
    c = cal.calibrate(x, avg_bits=3.0, is_key=True, cumvar=0.9)
    want = cal.effective_dim(c.lam, cumvar=0.9)
    assert c.d_eff == want == c.m and c.flags & cal.FLAG_CUMVAR
    assert c.code_bits + c.m == c.total_bits == 96


def test_random_rotation_is_haar_distributed():
    """Q of QR with a positive diagonal of R is Haar-distributed: over many seeds
    a fixed entry has mean 0 and mean square 1/d (with isotropic data the
    variance ordering keeps the columns in place). A QR without the sign fix
    gives Q[0, 0] = -|g00| / ||g0|| < 0 every time."""
    d, n = 6, 3000
    q00 = np.empty(n)
    q23 = np.empty(n)
    for s in range(n):
        lam, v = cal.random_basis(np.eye(d), seed=1000 + s, stream=0)
        assert np.allclose(lam, 1.0)
        q00[s], q23[s] = v[0, 0], v[2, 3]
    se = math.sqrt(1.0 / d / n)
    assert abs(q00.mean()) < 5 * se and abs(q23.mean()) < 5 * se
    assert abs((q00 ** 2).mean() - 1.0 / d) < 0.1 / d
    assert abs((q23 ** 2).mean() - 1.0 / d) < 0.1 / d


def test_random_rotation_basis_properties():
    """Orthonormal, variances q_i^T C q_i summing to the trace, descending,
    and a different basis per stream and seed."""
    r = np.random.default_rng(12)
    x = r.standard_normal((3000, 16)) * np.linspace(5, 1, 16)
    c = cal.second_moment(x)
    lam, v = cal.random_basis(c, seed=7, stream=3)
    assert np.max(np.abs(v.T @ v - np.eye(16))) < 1e-12
    assert abs(lam.sum() - np.trace(c)) < 1e-10 * np.trace(c)
    assert np.all(np.diff(lam) <= 0)
    assert np.allclose(lam, np.einsum("ji,jk,ki->i", v, c, v))
    _, v2 = cal.random_basis(c, seed=7, stream=4)
    _, v3 = cal.random_basis(c, seed=8, stream=3)
    assert np.max(np.abs(v - v2)) > 0.1 and np.max(np.abs(v - v3)) > 0.1


def test_spectral_rotation_beats_random_rotation_on_spiked_data():
    """The A/B the README's spectral_rotation.py runs: on a spiked spectrum the
    calibrated eigenbasis concentrates the energy (small d_eff) and its
    water-filled expected distortion sum_i sigma_i^2 D(b_i) is lower than that
    of a random rotation at the same budget, whose per-direction variances
    are nearly flat."""
    r = np.random.default_rng(13)
    d = 64
    q, _ = np.linalg.qr(r.standard_normal((d, d)))
    lam = np.concatenate([np.full(4, 200.0), np.ones(d - 4)])
    x = (r.standard_normal((20000, d)) * np.sqrt(lam)) @ q.T
    spec = cal.calibrate(x, avg_bits=3.0, is_key=False, normalize=False)
    rand = cal.calibrate(x, avg_bits=3.0, is_key=False, normalize=False, rotation="random", seed=3)
    dist = cb.distortion_table()
    e_spec = float(np.sum(spec.sigma ** 2 * dist[spec.bits]))
    e_rand = float(np.sum(rand.sigma ** 2 * dist[rand.bits]))
    assert spec.d_eff <= 6 < rand.d_eff
    assert e_spec < 0.6 * e_rand
    assert rand.flags & cal.FLAG_RANDOM_ROTATION and not spec.flags & cal.FLAG_RANDOM_ROTATION
