"""Gaussian Lloyd-Max scalar quantizers (oracle, float64).

Source: SpectralQuant README, "Repository Structure":
``nonuniform_quantization.py -- Lloyd-Max with per-regime codebooks``; the
Chinese summary of the same repository names the scheme "Lloyd-Max
per-interval codebooks" beside the water-filled bit allocation.

Reading taken (the pages print no codebook): every coordinate is quantized
after division by its own scale sigma_i, so one unit-variance Gaussian
Lloyd-Max quantizer per bit width b serves every coordinate; the "regime" of
a coordinate is its (sigma_i, b_i) pair. b = 0 means the coordinate is not
coded and reconstructs to 0.

The quantizer of b bits has 2**b levels l_0 < ... < l_{2**b-1} and the
2**b - 1 thresholds t_j = (l_j + l_{j+1}) / 2 (nearest-neighbour
condition). Each level is the conditional mean of N(0,1) over its cell
(centroid condition). The pair of conditions is solved by Lloyd's fixed-point
iteration. The Gaussian is symmetric, so only the positive half is iterated
and mirrored, which makes the middle threshold exactly 0.

Conditional moments of N(0,1) on a cell (a, c), with phi the density and
Phi the distribution function:
    P      = Phi(c) - Phi(a)
    E[Z]   = (phi(a) - phi(c)) / P
    E[Z^2] = 1 + (a phi(a) - c phi(c)) / P
The mean-squared distortion of the quantizer is the sum over cells of
P * (E[Z^2] - 2 l E[Z] + l^2).
"""

from __future__ import annotations

import functools
import math

import numpy as np
from scipy.special import erfc

MAX_BITS = 8
_SQRT2 = math.sqrt(2.0)
_INV_SQRT_2PI = 1.0 / math.sqrt(2.0 * math.pi)


def _phi(x: np.ndarray) -> np.ndarray:
    """Standard normal density; phi(+inf) = 0."""
    x = np.asarray(x, dtype=np.float64)
    with np.errstate(over="ignore"):
        return np.where(np.isinf(x), 0.0, _INV_SQRT_2PI * np.exp(-0.5 * x * x))


def _upper_tail(x: np.ndarray) -> np.ndarray:
    """Q(x) = 1 - Phi(x) = erfc(x / sqrt 2) / 2, accurate for large x."""
    return 0.5 * erfc(np.asarray(x, dtype=np.float64) / _SQRT2)


def _cell_moments(a: np.ndarray, c: np.ndarray):
    """P, E[Z | cell], E[Z^2 | cell] for cells (a, c) with 0 <= a < c <= inf."""
    p = _upper_tail(a) - _upper_tail(c)
    pa, pc = _phi(a), _phi(c)
    m1 = (pa - pc) / p
    a_pa = np.where(np.isinf(a), 0.0, np.where(np.isinf(a), 0.0, a) * pa)
    c_pc = np.where(np.isinf(c), 0.0, np.where(np.isinf(c), 0.0, c) * pc)
    m2 = 1.0 + (a_pa - c_pc) / p
    return p, m1, m2


def _positive_half(b: int, tol: float, max_iter: int):
    """Lloyd iteration on the positive half; returns the positive levels."""
    half = 1 << (b - 1)
    if half == 1:
        # One positive cell (0, inf): its centroid, sqrt(2/pi).
        _, m1, _ = _cell_moments(np.array([0.0]), np.array([np.inf]))
        return m1
    # Start from the centroids of equal-probability cells on (0, inf).
    q = np.linspace(0.5, 1.0, half + 1)[1:-1]          # Phi at the inner edges
    edges = np.sqrt(2.0) * _erfcinv(2.0 * (1.0 - q))
    lo = np.concatenate([[0.0], edges])
    hi = np.concatenate([edges, [np.inf]])
    _, levels, _ = _cell_moments(lo, hi)
    for _ in range(max_iter):
        inner = 0.5 * (levels[:-1] + levels[1:])
        lo = np.concatenate([[0.0], inner])
        hi = np.concatenate([inner, [np.inf]])
        _, new, _ = _cell_moments(lo, hi)
        step = np.max(np.abs(new - levels))
        levels = new
        if step < tol:
            break
    return levels


def _erfcinv(y: np.ndarray) -> np.ndarray:
    from scipy.special import erfcinv
    return erfcinv(y)


def _accelerated_positive_half(b: int, tol: float):
    """Lloyd's map solved by Newton's method on F(l) = lloyd(l) - l.

    Lloyd's fixed-point iteration alone converges very slowly for 7-8 bits.
    Newton steps on the same fixed-point equations (Jacobian by central
    differences) reach the same fixed point; plain Lloyd iterations are run
    before and after so that the result is Lloyd's fixed point to ``tol``.
    """
    levels = _positive_half(b, tol, 2000)
    half = levels.size
    if half == 1:
        return levels

    def lloyd(lv):
        inner = 0.5 * (lv[:-1] + lv[1:])
        lo = np.concatenate([[0.0], inner])
        hi = np.concatenate([inner, [np.inf]])
        return _cell_moments(lo, hi)[1]

    for _ in range(50):
        f = lloyd(levels) - levels
        if np.max(np.abs(f)) < tol:
            break
        h = 1e-7
        jac = np.empty((half, half))
        for k in range(half):
            e = np.zeros(half)
            e[k] = h
            jac[:, k] = ((lloyd(levels + e) - (levels + e)) - (lloyd(levels - e) - (levels - e))) / (2 * h)
        levels = levels - np.linalg.solve(jac, f)
    # Polish with plain Lloyd steps (a contraction near the fixed point).
    for _ in range(200):
        new = lloyd(levels)
        step = np.max(np.abs(new - levels))
        levels = new
        if step < tol:
            break
    return levels


@functools.lru_cache(maxsize=None)
def lloyd_max(b: int, tol: float = 1e-15):
    """Gaussian Lloyd-Max quantizer of ``b`` bits.

    Returns ``(levels, thresholds, distortion)``: 2**b ascending levels,
    2**b - 1 ascending thresholds, and D(b) = E[(Z - Q(Z))^2] for Z ~ N(0,1).
    ``b == 0`` returns a single level 0 with no thresholds and D(0) = 1.
    """
    if b == 0:
        return np.zeros(1), np.zeros(0), 1.0
    if not 1 <= b <= MAX_BITS:
        raise ValueError(f"bit width {b} outside 0..{MAX_BITS}")
    pos = _accelerated_positive_half(b, tol)
    levels = np.concatenate([-pos[::-1], pos])
    thresholds = 0.5 * (levels[:-1] + levels[1:])
    thresholds[len(thresholds) // 2] = 0.0
    return levels.copy(), thresholds.copy(), distortion(levels, thresholds)


def distortion(levels: np.ndarray, thresholds: np.ndarray) -> float:
    """E[(Z - Q(Z))^2] of a quantizer with the given cells, Z ~ N(0,1)."""
    edges = np.concatenate([[-np.inf], thresholds, [np.inf]])
    total = 0.0
    for k, lvl in enumerate(levels):
        a, c = edges[k], edges[k + 1]
        # Use the positive-side formulas through symmetry for cells below 0.
        if c <= 0.0:
            p, m1, m2 = _cell_moments(np.array([-c]), np.array([-a]))
            m1 = -m1
        elif a >= 0.0:
            p, m1, m2 = _cell_moments(np.array([a]), np.array([c]))
        else:  # a cell straddling 0 (odd level counts never occur here)
            p1, e1, s1 = _cell_moments(np.array([0.0]), np.array([c]))
            p2, e2, s2 = _cell_moments(np.array([0.0]), np.array([-a]))
            p = p1 + p2
            m1 = (p1 * e1 - p2 * e2) / p
            m2 = (p1 * s1 + p2 * s2) / p
        total += float(p[0] * (m2[0] - 2.0 * lvl * m1[0] + lvl * lvl))
    return total


def distortion_table(max_bits: int = MAX_BITS) -> np.ndarray:
    """D(b) for b = 0..max_bits (D(0) = 1: an uncoded coordinate)."""
    return np.array([lloyd_max(b)[2] for b in range(max_bits + 1)])


def quantize(z: np.ndarray, b: int) -> np.ndarray:
    """Code of each z: the number of thresholds strictly below z.

    A value exactly on a threshold takes the lower code.
    """
    _, thr, _ = lloyd_max(b)
    z = np.asarray(z, dtype=np.float64)
    return (z[..., None] > thr).sum(axis=-1).astype(np.int64)


def dequantize(codes: np.ndarray, b: int) -> np.ndarray:
    """Level of each code (0.0 for an uncoded coordinate, b == 0)."""
    if b == 0:
        return np.zeros(np.shape(codes))
    levels, _, _ = lloyd_max(b)
    return levels[np.asarray(codes, dtype=np.int64)]
