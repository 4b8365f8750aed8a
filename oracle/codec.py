"""Compression of key/value vectors into packed records, and the inverse (oracle).

Sources
-------
* SpectralQuant README, "Overview" and "Repository Structure":
  ``spectral_rotation.py`` (rotation into the calibrated eigenbasis),
  ``nonuniform_quantization.py`` (Lloyd-Max codebooks),
  ``selective_qjl.py`` (QJL correction on the signal dimensions only: error
  correction is dropped on the remaining noise dimensions), "Compression
  ratio ... analytical (bit accounting)".
* TurboQuant reference implementation README, "Project Structure":
  ``qjl.py -- Quantized Johnson-Lindenstrauss (1-bit inner product)`` and
  ``core.py -- TurboQuantMSE + TurboQuantProd`` (prior art for a b-bit
  quantizer plus one QJL sign bit per projection of the residual).

The steps, per vector x of one head with calibration ``cal``:
  1. norm = ||x|| (normalized mode; 1 otherwise) and u = x / norm (0 if norm = 0).
  2. y = V^T u: coordinates in the calibrated eigenbasis.
  3. z_i = y_i / sigma_i (0 where sigma_i = 0); code_i = number of the b_i-bit
     thresholds strictly below z_i; c_hat_i = level of code_i (0 if b_i = 0).
     The b-bit codebook is the Gaussian Lloyd-Max one, or, for a calibration
     with fitted codebooks, the one of coordinate i's regime (fitted.py).
  4. Keys with QJL, signal dims i < m: r = y[:m] - sigma[:m] * c_hat[:m],
     rho = ||r||, sign bit j = 1 if (S r)_j >= 0 else 0.
  5. Pack (reading taken; the pages fix no layout): one record of B bits per
     vector in ``words`` little-endian 32-bit words; stream bit k is bit k % 32
     of word k // 32. The codes of coordinates 0..d-1 with b_i > 0 come first,
     in coordinate order, each least-significant bit first, then the m QJL
     bits, then zeros. norm and rho are stored apart as float32.
Inverse: x_hat = norm * V (sigma * c_hat); with the QJL term,
x_hat += norm * V[:, :m] (sqrt(pi/2) / m * rho * S^T s), s_j = 2 bit_j - 1.
The QJL term is the unbiased estimator of the residual's inner products:
for a Gaussian row s, E[<s, q> sign<s, r>] = sqrt(2/pi) <q, r> / ||r||.
"""

from __future__ import annotations

import math

import numpy as np

from . import codebook
from .calibration import HeadCalib

QJL_SCALE = math.sqrt(math.pi / 2.0)
EXEMPT_REL = 1e-5


def rotate(x: np.ndarray, cal: HeadCalib):
    """(norm [T], y [T, d]) of the vectors ``x`` [T, d]."""
    x = np.asarray(x, dtype=np.float64)
    if cal.normalize:
        norm = np.sqrt(np.sum(x * x, axis=1))
    else:
        norm = np.ones(x.shape[0])
    safe = np.where(norm > 0.0, norm, 1.0)
    u = np.where(norm[:, None] > 0.0, x / safe[:, None], 0.0)
    y = u @ cal.V                       # y_i = sum_j V[j, i] u_j
    return norm, y


def scaled(y: np.ndarray, cal: HeadCalib) -> np.ndarray:
    """z = y / sigma per coordinate (0 where sigma = 0)."""
    safe = np.where(cal.sigma > 0.0, cal.sigma, 1.0)
    return np.where(cal.sigma > 0.0, y / safe, 0.0)


def quantize(z: np.ndarray, cal: HeadCalib) -> np.ndarray:
    """Codes [T, d] of the scaled coordinates (0 where b_i = 0)."""
    codes = np.zeros(z.shape, dtype=np.int64)
    for i in range(cal.d):
        if cal.bits[i] > 0:
            if cal.fitted:
                _, thr = cal.codebook(i)
                codes[:, i] = (z[:, i][:, None] > thr[None, :]).sum(axis=1)
            else:
                codes[:, i] = codebook.quantize(z[:, i], int(cal.bits[i]))
    return codes


def levels(codes: np.ndarray, cal: HeadCalib) -> np.ndarray:
    """Reconstruction levels c_hat [T, d] of the codes."""
    out = np.zeros(codes.shape)
    for i in range(cal.d):
        if cal.fitted and cal.bits[i] > 0:
            lv, _ = cal.codebook(i)
            out[:, i] = lv[np.asarray(codes[:, i], dtype=np.int64)]
        else:
            out[:, i] = codebook.dequantize(codes[:, i], int(cal.bits[i]))
    return out


def qjl_signs(y: np.ndarray, c_hat: np.ndarray, cal: HeadCalib):
    """(rho [T], bits [T, m], projections S r [T, m]) of the signal residual."""
    m = cal.m
    t = y.shape[0]
    if m == 0:
        return np.zeros(t), np.zeros((t, 0), dtype=np.int64), np.zeros((t, 0))
    r = y[:, :m] - cal.sigma[None, :m] * c_hat[:, :m]
    rho = np.sqrt(np.sum(r * r, axis=1))
    proj = r @ cal.S.T                   # (S r)_j = sum_k S[j, k] r_k
    return rho, (proj >= 0.0).astype(np.int64), proj


def pack(codes: np.ndarray, qbits: np.ndarray, cal: HeadCalib) -> np.ndarray:
    """Packed records [T, words] (uint32) of codes [T, d] and QJL bits [T, m]."""
    t = codes.shape[0]
    stream = np.zeros((t, cal.words * 32), dtype=np.uint8)
    for i in range(cal.d):
        for k in range(int(cal.bits[i])):
            stream[:, cal.offsets[i] + k] = (codes[:, i] >> k) & 1
    for j in range(cal.m):
        stream[:, cal.code_bits + j] = qbits[:, j]
    words = np.zeros((t, cal.words), dtype=np.uint64)
    for k in range(cal.words * 32):
        words[:, k // 32] |= stream[:, k].astype(np.uint64) << np.uint64(k % 32)
    return words.astype(np.uint32)


def unpack(words: np.ndarray, cal: HeadCalib):
    """(codes [T, d], QJL bits [T, m]) of packed records [T, words]."""
    words = np.asarray(words, dtype=np.uint32).astype(np.uint64)
    t = words.shape[0]

    def bit(k):
        return ((words[:, k // 32] >> np.uint64(k % 32)) & np.uint64(1)).astype(np.int64)

    codes = np.zeros((t, cal.d), dtype=np.int64)
    for i in range(cal.d):
        for k in range(int(cal.bits[i])):
            codes[:, i] |= bit(cal.offsets[i] + k) << k
    qbits = np.zeros((t, cal.m), dtype=np.int64)
    for j in range(cal.m):
        qbits[:, j] = bit(cal.code_bits + j)
    return codes, qbits


def compress(x: np.ndarray, cal: HeadCalib) -> dict:
    """All of steps 1-5 for vectors ``x`` [T, d].

    Returns the stored outputs (``words``, ``norm`` and ``rnorm`` as float32)
    and the float64 intermediates the parity exemptions need (``z``, ``proj``,
    ``norm64``, ``rho64``, ``codes``, ``qbits``).
    """
    norm, y = rotate(x, cal)
    z = scaled(y, cal)
    codes = quantize(z, cal)
    c_hat = levels(codes, cal)
    rho, qbits, proj = qjl_signs(y, c_hat, cal)
    return {
        "words": pack(codes, qbits, cal),
        "norm": norm.astype(np.float32),
        "rnorm": rho.astype(np.float32),
        "codes": codes, "qbits": qbits, "z": z, "y": y, "proj": proj,
        "norm64": norm, "rho64": rho,
    }


def decompress(words: np.ndarray, norm: np.ndarray, rnorm: np.ndarray, cal: HeadCalib,
               apply_qjl: bool = True) -> np.ndarray:
    """Reconstructed vectors [T, d] from packed records and the stored scalars."""
    codes, qbits = unpack(words, cal)
    c_hat = levels(codes, cal)
    norm = np.asarray(norm, dtype=np.float64)
    if not cal.normalize:
        norm = np.ones_like(norm)
    xhat = (c_hat * cal.sigma[None, :]) @ cal.V.T       # x_j = sum_i V[j, i] sigma_i c_i
    if apply_qjl and cal.m > 0:
        s = 2.0 * qbits - 1.0
        rho = np.asarray(rnorm, dtype=np.float64)
        corr = (QJL_SCALE / cal.m) * rho[:, None] * (s @ cal.S)   # (S^T s)_k
        xhat = xhat + corr @ cal.V[:, :cal.m].T
    return norm[:, None] * xhat


def exemptions(out: dict, cal: HeadCalib):
    """Which outputs may legitimately differ from a GPU's.

    A code is exempt when its z lies within 1e-5 * max(1, |t|) of one of its
    thresholds t. A token's QJL bits and rho are exempt when a signal-dim
    code is exempt, or bit j is when |(S r)_j| <= 1e-5 * ||S_j|| * rho.
    Returns (code_exempt [T, d] bool, qjl_exempt [T, m] bool, rho_exempt [T] bool).
    """
    z = out["z"]
    t = z.shape[0]
    code_ex = np.zeros(z.shape, dtype=bool)
    for i in range(cal.d):
        b = int(cal.bits[i])
        if b == 0:
            continue
        _, thr = cal.codebook(i)
        dist = np.abs(z[:, i:i + 1] - thr[None, :])
        code_ex[:, i] = np.any(dist <= EXEMPT_REL * np.maximum(1.0, np.abs(thr))[None, :], axis=1)
    m = cal.m
    rho_ex = np.zeros(t, dtype=bool)
    q_ex = np.zeros((t, m), dtype=bool)
    if m > 0:
        rho_ex = np.any(code_ex[:, :m], axis=1)
        srow = np.sqrt(np.sum(cal.S * cal.S, axis=1))
        q_ex = np.abs(out["proj"]) <= EXEMPT_REL * srow[None, :] * out["rho64"][:, None]
        q_ex |= rho_ex[:, None]
    return code_ex, q_ex, rho_ex
