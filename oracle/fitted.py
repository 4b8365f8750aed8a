"""Empirically fitted per-regime Lloyd codebooks (oracle, float64).

Test infrastructure: imported only by the tests, the smoke check and the
benchmark's CPU-baseline leg.

Sources
-------
* SpectralQuant README, "Repository Structure":
  ``nonuniform_quantization.py -- Lloyd-Max with per-regime codebooks``; the
  Chinese summary of the same repository calls them "Lloyd-Max codebooks per
  interval".
* spectralquant tests/conftest.py (v1 branch), fixture ``gaussian_data_1d``:
  5000 one-dimensional Gaussian samples "for Lloyd-Max quantizer tests",
  large enough for convergence tests, i.e. the quantizer is fitted to
  samples by Lloyd's iteration.

Readings taken (the pages print neither the regimes nor the fitting rule)
-------------------------------------------------------------------------
* Two regimes per head: the signal coordinates (rotated coordinates
  i < d_eff) and the noise coordinates (i >= d_eff), the split the method
  uses everywhere else (QJL on the signal dimensions only). Regime 0 is the
  signal regime, 1 the noise regime.
* In each regime, one codebook per bit width b that a coordinate of the
  regime uses, fitted to the pooled scaled coordinates z_{t,i} = y_{t,i} /
  sigma_i of the calibration vectors t over the regime's coordinates i of
  width b (the same z the compressor quantizes).
* Lloyd's algorithm from the Gaussian Lloyd-Max codebook of width b, for a
  fixed number of iterations (``FIT_ITERS`` unless the caller gives another):
  the thresholds are the midpoints of neighbouring levels, each sample takes
  the code the compressor gives it (the number of thresholds strictly
  below), and each level moves to the mean of its samples; a level with no
  sample keeps its value. The stored thresholds are the midpoints of the
  final levels. A fixed count (no convergence test) makes the steps
  identical on any machine. The means of ordered, disjoint cells are
  ordered and a kept level stays between its neighbours' new means, so the
  levels stay strictly increasing.
* Widths that no coordinate of a regime uses keep the Gaussian codebook
  (they are never used to code).

Table layout (the record's fitted-codebook section): levels [2][510] with
width b at offset 2**b - 2 (2**b levels, ascending) and thresholds [2][502]
with width b at offset 2**b - 1 - b (2**b - 1 thresholds), b = 1..8.
"""

from __future__ import annotations

import numpy as np

from . import codebook

FIT_ITERS = 30
N_LEVELS = sum(1 << b for b in range(1, codebook.MAX_BITS + 1))           # 510
N_THRESH = sum((1 << b) - 1 for b in range(1, codebook.MAX_BITS + 1))     # 502


def level_offset(b: int) -> int:
    """Offset of width b's levels in one regime's level table."""
    return (1 << b) - 2


def thresh_offset(b: int) -> int:
    """Offset of width b's thresholds in one regime's threshold table."""
    return (1 << b) - 1 - b


def gaussian_tables():
    """(levels [510], thresholds [502]) of the Gaussian Lloyd-Max codebooks."""
    lv = np.zeros(N_LEVELS)
    th = np.zeros(N_THRESH)
    for b in range(1, codebook.MAX_BITS + 1):
        levels, thr, _ = codebook.lloyd_max(b)
        lv[level_offset(b):level_offset(b) + (1 << b)] = levels
        th[thresh_offset(b):thresh_offset(b) + (1 << b) - 1] = thr
    return lv, th


def lloyd_fit(samples: np.ndarray, init_levels: np.ndarray, iters: int = FIT_ITERS) -> np.ndarray:
    """Levels after ``iters`` Lloyd iterations on ``samples`` from ``init_levels``."""
    z = np.asarray(samples, dtype=np.float64).reshape(-1)
    levels = np.asarray(init_levels, dtype=np.float64).copy()
    for _ in range(iters):
        thr = 0.5 * (levels[:-1] + levels[1:])
        codes = np.searchsorted(thr, z, side="left")          # thresholds strictly below z
        sums = np.bincount(codes, weights=z, minlength=levels.size)
        counts = np.bincount(codes, minlength=levels.size)
        levels = np.where(counts > 0, sums / np.maximum(counts, 1), levels)
    return levels


def regime_of(i: int, d_eff: int) -> int:
    """0 for a signal coordinate (i < d_eff), 1 for a noise coordinate."""
    return 0 if i < d_eff else 1


def fit_tables(z: np.ndarray, bits: np.ndarray, d_eff: int, iters: int = FIT_ITERS):
    """Per-regime tables (levels [2][510], thresholds [2][502]) fitted to the
    scaled calibration coordinates ``z`` [N, d] of a head with widths ``bits``."""
    z = np.asarray(z, dtype=np.float64)
    g_lv, g_th = gaussian_tables()
    lv = np.stack([g_lv, g_lv])
    th = np.stack([g_th, g_th])
    d = z.shape[1]
    for r in (0, 1):
        cols = [i for i in range(d) if regime_of(i, d_eff) == r]
        for b in range(1, codebook.MAX_BITS + 1):
            sel = [i for i in cols if int(bits[i]) == b]
            if not sel:
                continue
            o = level_offset(b)
            fitted = lloyd_fit(z[:, sel], g_lv[o:o + (1 << b)], iters)
            lv[r, o:o + (1 << b)] = fitted
            t = thresh_offset(b)
            th[r, t:t + (1 << b) - 1] = 0.5 * (fitted[:-1] + fitted[1:])
    return lv, th


def codebook_of(lv: np.ndarray, th: np.ndarray, regime: int, b: int):
    """(levels, thresholds) of width b in one regime of fitted tables."""
    o, t = level_offset(b), thresh_offset(b)
    return lv[regime, o:o + (1 << b)], th[regime, t:t + (1 << b) - 1]
