"""Pins of the oracle's fitted per-regime codebooks (oracle/fitted.py).

SpectralQuant README, "Repository Structure": nonuniform_quantization.py,
"Lloyd-Max with per-regime codebooks"; the conftest fixture gaussian_data_1d
(a Lloyd-Max quantizer fitted to samples by iteration). Each pin is fixed by
the mathematics or worked by hand, not by re-running the oracle's formula.
"""

import itertools

import numpy as np
import pytest

from oracle import calibration as ocal
from oracle import codebook as ocb
from oracle import codec as ocodec
from oracle import fitted as ofit
from oracle import record as orec


def _mse(z, levels):
    thr = 0.5 * (levels[:-1] + levels[1:])
    return float(np.mean((z - levels[np.searchsorted(thr, z, side="left")]) ** 2))


def test_table_layout_offsets():
    # width b starts after the 2 + 4 + ... + 2^(b-1) levels (1 + 3 + ... thresholds) of the narrower widths
    assert [ofit.level_offset(b) for b in range(1, 9)] == [0, 2, 6, 14, 30, 62, 126, 254]
    assert [ofit.thresh_offset(b) for b in range(1, 9)] == [0, 1, 4, 11, 26, 57, 120, 247]
    assert ofit.N_LEVELS == 510 and ofit.N_THRESH == 502


def test_hand_worked_two_bit_fit():
    # Samples -4, -1, 0.5, 3 (ten of each), 2-bit start = Gaussian Lloyd-Max
    # levels +-0.4528, +-1.510 with thresholds 0, +-0.9816. Iteration 1: -4 and
    # -1 both lie below -0.9816 (cell 0, mean -2.5), cell 1 is empty and keeps
    # -0.4528, 0.5 is cell 2, 3 is cell 3. Iteration 2: thresholds -1.476,
    # 0.0236, 1.75 separate the four values, so each level is its value.
    s = np.repeat([-4.0, -1.0, 0.5, 3.0], 10)
    g = ocb.lloyd_max(2)[0]
    one = ofit.lloyd_fit(s, g, 1)
    assert one[0] == -2.5 and one[1] == g[1] and one[2] == 0.5 and one[3] == 3.0
    two = ofit.lloyd_fit(s, g, 2)
    np.testing.assert_array_equal(two, [-4.0, -1.0, 0.5, 3.0])
    np.testing.assert_array_equal(ofit.lloyd_fit(s, g, 30), [-4.0, -1.0, 0.5, 3.0])


def test_one_bit_fit_is_the_two_half_means():
    # One threshold at 0 (start +-sqrt(2/pi)); each level is the mean of its half line.
    rng = np.random.default_rng(3)
    z = rng.standard_t(4, 5001)
    lv = ofit.lloyd_fit(z, ocb.lloyd_max(1)[0], 1)
    assert lv[0] == pytest.approx(z[z <= 0].mean(), rel=1e-12)
    assert lv[1] == pytest.approx(z[z > 0].mean(), rel=1e-12)


@pytest.mark.parametrize("b,a,iters,tol", [(2, 2.0, 30, 2e-5), (3, 3.0, 300, 2e-4)])
def test_uniform_density_converges_to_the_uniform_quantizer(b, a, iters, tol):
    # For a uniform density on (-a, a) the Lloyd fixed point is the uniform
    # quantizer: levels at the cell centres a ((2k + 1) / 2^b - 1).
    z = ((np.arange(400000) + 0.5) / 400000 * 2 - 1) * a
    lv = ofit.lloyd_fit(z, ocb.lloyd_max(b)[0], iters)
    exact = ((2 * np.arange(1 << b) + 1) / (1 << b) - 1) * a
    assert np.max(np.abs(lv - exact)) < tol


def test_empty_outer_cells_keep_their_level():
    # Uniform on (-1, 1): the 3-bit start has outer thresholds +-1.748, so the
    # outermost cells never receive a sample and their levels stay +-2.152.
    z = (np.arange(10000) + 0.5) / 10000 * 2 - 1
    g = ocb.lloyd_max(3)[0]
    lv = ofit.lloyd_fit(z, g, 30)
    assert lv[0] == g[0] and lv[-1] == g[-1]
    assert np.all(np.diff(lv) > 0)


def test_fit_never_increases_the_sample_distortion():
    rng = np.random.default_rng(5)
    for b in (1, 2, 3, 4, 5):
        z = rng.standard_t(3, 20000) * 0.8
        g = ocb.lloyd_max(b)[0]
        prev = _mse(z, g)
        for it in (1, 2, 5, 30):
            cur = _mse(z, ofit.lloyd_fit(z, g, it))
            assert cur <= prev + 1e-15
            prev = cur


def test_converged_fit_is_the_best_partition_on_tiny_data():
    # Nine well-separated samples in four clusters: brute force over every
    # split of the sorted samples into four contiguous cells gives the optimum,
    # which the converged fit reaches (levels = cluster means).
    z = np.array([-5.1, -4.9, -5.0, -1.2, -0.8, 0.9, 1.1, 4.0, 4.2])
    best = np.inf
    srt = np.sort(z)
    for cuts in itertools.combinations(range(1, 9), 3):
        parts = np.split(srt, cuts)
        best = min(best, sum(float(np.sum((p - p.mean()) ** 2)) for p in parts) / z.size)
    lv = ofit.lloyd_fit(z, ocb.lloyd_max(2)[0], 200)
    assert _mse(z, lv) == pytest.approx(best, rel=1e-12)
    np.testing.assert_allclose(lv, [-5.0, -1.0, 1.0, 4.1], atol=1e-12)


def test_regimes_and_widths_are_fitted_apart():
    # Coordinates 0, 1 (signal, d_eff = 2) and 2..5 (noise) at 2 bits; coordinate
    # 6 (noise) at 1 bit. Signal samples take the values -4, -1, 0.5, 3; noise
    # samples -3, -0.7, 0.7, 3 (one per cell of the 2-bit start, so one
    # iteration lands on them); the 1-bit coordinate -7, 7. Each codebook
    # converges to its own group's values, none to another's.
    t = 40
    z = np.zeros((t, 7))
    z[:, 0] = np.tile([-4.0, -1.0, 0.5, 3.0], t // 4)
    z[:, 1] = np.tile([3.0, 0.5, -1.0, -4.0], t // 4)
    for i in range(2, 6):
        z[:, i] = np.tile([-3.0, -0.7, 0.7, 3.0], t // 4)
    z[:, 6] = np.tile([-7.0, 7.0], t // 2)
    bits = np.array([2, 2, 2, 2, 2, 2, 1])
    lv, th = ofit.fit_tables(z, bits, d_eff=2, iters=30)
    np.testing.assert_array_equal(ofit.codebook_of(lv, th, 0, 2)[0], [-4.0, -1.0, 0.5, 3.0])
    np.testing.assert_allclose(ofit.codebook_of(lv, th, 1, 2)[0], [-3.0, -0.7, 0.7, 3.0], rtol=0, atol=1e-15)
    np.testing.assert_array_equal(ofit.codebook_of(lv, th, 1, 1)[0], [-7.0, 7.0])
    np.testing.assert_allclose(ofit.codebook_of(lv, th, 1, 2)[1], [-1.85, 0.0, 1.85], rtol=0, atol=1e-14)
    # widths a regime does not use keep the Gaussian codebook
    np.testing.assert_array_equal(ofit.codebook_of(lv, th, 0, 1)[0], ocb.lloyd_max(1)[0])
    np.testing.assert_array_equal(ofit.codebook_of(lv, th, 0, 3)[1], ocb.lloyd_max(3)[1])


def _identity_head(d=8, d_eff=2, bits=(3, 3, 2, 2, 2, 2, 1, 1)):
    lam = np.array([100.0, 50.0] + [1.0] * (d - 2))
    cal = ocal.finalize(lam, np.eye(d), avg_bits=sum(bits) / d, is_key=False, normalize=False)
    cal.bits = np.array(bits, dtype=np.int64)
    cal.offsets = ocal.bit_offsets(cal.bits)
    cal.d_eff = d_eff
    cal.sigma = np.ones(d)
    return cal


def test_codec_codes_each_coordinate_with_its_regime_table():
    # Identity basis, sigma = 1, unnormalized: z = x. Hand-set tables: the
    # signal 3-bit codebook is 0..7, the noise 2-bit codebook is -30, -10, 10, 30
    # (thresholds -20, 0, 20), the noise 1-bit codebook is -1, 1.
    cal = _identity_head()
    g_lv, g_th = ofit.gaussian_tables()
    lv = np.stack([g_lv, g_lv])
    th = np.stack([g_th, g_th])
    o3, t3 = ofit.level_offset(3), ofit.thresh_offset(3)
    lv[0, o3:o3 + 8] = np.arange(8.0)
    th[0, t3:t3 + 7] = np.arange(7.0) + 0.5
    o2, t2 = ofit.level_offset(2), ofit.thresh_offset(2)
    lv[1, o2:o2 + 4] = [-30.0, -10.0, 10.0, 30.0]
    th[1, t2:t2 + 3] = [-20.0, 0.0, 20.0]
    cal.fit_lv, cal.fit_th = lv, th
    cal.flags |= ocal.FLAG_FITTED
    x = np.array([[2.2, 6.9, -25.0, -5.0, 0.0, 40.0, -0.1, 0.3]])
    out = ocodec.compress(x, cal)
    # 2.2 -> 2 (thresholds 0.5..6.5), 6.9 -> 7; noise 2-bit: -25 -> 0, -5 -> 1,
    # 0 -> 1 (tie takes the lower code), 40 -> 3; noise 1-bit (Gaussian
    # threshold 0): -0.1 -> 0, 0.3 -> 1
    np.testing.assert_array_equal(out["codes"][0], [2, 7, 0, 1, 1, 3, 0, 1])
    xh = ocodec.decompress(out["words"], out["norm"], out["rnorm"], cal, apply_qjl=False)
    g1 = ocb.lloyd_max(1)[0]
    np.testing.assert_allclose(xh[0], [2.0, 7.0, -30.0, -10.0, -10.0, 30.0, g1[0], g1[1]])


def test_fitted_calibration_codes_its_own_data_better():
    # Heavy-tailed calibration data: per regime and width, the fitted codebooks
    # give a sample distortion on the calibration z no larger than the Gaussian ones.
    rng = np.random.default_rng(11)
    d = 16
    q, _ = np.linalg.qr(rng.standard_normal((d, d)))
    x = (rng.standard_t(3, (3000, d)) * np.sqrt([200.0, 80.0] + [1.0] * (d - 2))) @ q.T
    g = ocal.calibrate(x, avg_bits=3.0, is_key=False)
    f = ocal.calibrate(x, avg_bits=3.0, is_key=False, codebooks="fitted")
    np.testing.assert_array_equal(g.bits, f.bits)
    assert f.fitted and not g.fitted
    _, y = ocodec.rotate(x, f)
    z = ocodec.scaled(y, f)
    for i in range(d):
        if f.bits[i] == 0:
            continue
        lvf, _ = f.codebook(i)
        lvg, _ = g.codebook(i)
        # per coordinate the pooled optimum need not win; pooled per group it must
        r = 0 if i < f.d_eff else 1
        cols = [j for j in range(d) if f.bits[j] == f.bits[i] and (0 if j < f.d_eff else 1) == r]
        assert _mse(z[:, cols].ravel(), lvf) <= _mse(z[:, cols].ravel(), lvg) + 1e-15


def test_record_round_trip_keeps_the_fitted_tables():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((512, 32)) * np.sqrt([40.0] * 4 + [1.0] * 28)
    cal = ocal.calibrate(x, avg_bits=3.0, is_key=True, codebooks="fitted", fit_iters=7)
    raw = orec.write(cal)
    assert len(raw) == orec.canonical_bytes(32)
    back = orec.read(raw)
    assert back.fitted and back.flags == cal.flags
    np.testing.assert_array_equal(back.fit_lv, cal.fit_lv)
    np.testing.assert_array_equal(back.fit_th, cal.fit_th)
    plain = orec.read(orec.write(ocal.calibrate(x, avg_bits=3.0, is_key=True)))
    assert not plain.fitted and plain.fit_lv is None
    # the section of a record without fitted codebooks is zero
    assert not any(orec.write(plain)[orec.canonical_bytes(32) - orec.FIT_BYTES:])
