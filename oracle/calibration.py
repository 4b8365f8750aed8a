"""Per-head eigenspectral calibration (oracle, float64).

Sources
-------
* SpectralQuant README, "Repository Structure": ``calibration.py --
  Eigenspectral calibration (PCA, d_eff, kappa)``; "Overview": a one-time
  calibration finds the few signal dimensions of the key vectors.
* spectralquant tests/conftest.py (v1 branch), fixture
  ``pre_computed_calibration``: C = X^T X / N (no centring), ``eigh``,
  reversal to descending order, d_eff = round((sum lambda)^2 / sum lambda^2),
  gap = lambda[d_eff - 1] / lambda[d_eff] (0-based) or inf when d_eff = d.
* The title of the method ("Water-Filled Bit Allocation") and the Chinese
  summary ("water-filling non-uniform bit allocation by spectral structure").

Readings taken where the pages are silent
-----------------------------------------
* Eigenvalues below zero (round-off) are clamped to 0.
* Sign of each eigenvector: its entry of largest magnitude is made positive
  (ties: the lowest index).
* d_eff rounds half to even (Python's ``round``) and is clamped to [1, d];
  an all-zero spectrum gives d_eff = d.
* Quantizer scale per coordinate. Normalized mode (default): the unit vector
  x/||x|| is quantized, and sigma_i = sqrt(lambda_i / sum lambda), the
  first-order second moment of its i-th rotated coordinate. Unnormalized
  mode: sigma_i = sqrt(lambda_i).
* Bit budget: B = avg_bits * d bits per vector, an integer. A key with QJL
  spends m = d_eff of them on sign bits, so the codes get B - m bits;
  otherwise the codes get all B. No coordinate takes more than 8 bits.
* Water-filling: greedy, one bit at a time, to the coordinate whose expected
  distortion drops most, lambda_i * (D(b_i) - D(b_i + 1)), among those below
  the cap; ties go to the lowest index. D is the Gaussian Lloyd-Max
  distortion table (D(0) = 1). Because D is convex and decreasing the greedy
  result minimises sum_i lambda_i D(b_i) over integer allocations.

Variants the README names ("Repository Structure": results/deff_sweep/ --
"participation ratio vs cumvar"; spectral_rotation.py -- "Spectral rotation
vs random rotation baseline"), with the readings taken:
* cumulative-variance d_eff: the smallest k >= 1 whose top-k eigenvalues hold
  at least a fraction ``cumvar`` of the trace (the pages give no fraction; the
  caller chooses it, 0.9 in the tests);
* random rotation: the basis is Q of the QR factorisation G = Q R (diag R > 0)
  of a d x d matrix G of N(0,1) draws, row-major, from the stream of seed
  ``seed ^ ROTATION_SALT`` and the head's index (the same SplitMix64 /
  Box-Muller stream as the QJL matrix, another seed), i.e. a Haar-random
  orthogonal matrix; lambda_i = q_i^T C q_i is the variance along column i,
  and the columns are ordered by descending variance (stable). Everything
  after the basis is unchanged.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

from . import codebook, rng

FLAG_IS_KEY = 1
FLAG_QJL = 2
FLAG_NORMALIZE = 4
FLAG_RANDOM_ROTATION = 8
FLAG_CUMVAR = 16
FLAG_FITTED = 32               # per-regime codebooks fitted to the calibration data (fitted.py)
ROTATION_SALT = 0x524F54       # seed salt of the random-rotation stream ("ROT")


def second_moment(x: np.ndarray) -> np.ndarray:
    """C = X^T X / N of the calibration vectors (rows of ``x``), uncentred."""
    x = np.asarray(x, dtype=np.float64)
    return x.T @ x / x.shape[0]


def eigenbasis(c: np.ndarray):
    """Eigenvalues (descending, >= 0) and orthonormal eigenvectors (columns)."""
    lam, vec = np.linalg.eigh(np.asarray(c, dtype=np.float64))
    lam = lam[::-1].copy()
    vec = vec[:, ::-1].copy()
    lam = np.maximum(lam, 0.0)
    for i in range(vec.shape[1]):
        j = int(np.argmax(np.abs(vec[:, i])))
        if vec[j, i] < 0.0:
            vec[:, i] = -vec[:, i]
    return lam, vec


def participation_ratio(lam: np.ndarray) -> float:
    """(sum lambda)^2 / sum lambda^2."""
    lam = np.asarray(lam, dtype=np.float64)
    s2 = float(np.sum(lam * lam))
    if s2 == 0.0:
        return float(lam.size)
    return float(np.sum(lam)) ** 2 / s2


def effective_dim(lam: np.ndarray, cumvar: float = 0.0) -> int:
    """d_eff: the participation ratio rounded half to even, within [1, d]; with
    0 < cumvar <= 1, the smallest k >= 1 whose top-k eigenvalues (descending)
    hold at least cumvar of the trace (d for an all-zero spectrum)."""
    d = len(lam)
    if cumvar > 0.0:
        lam = np.asarray(lam, dtype=np.float64)
        tr = float(np.sum(lam))
        if tr == 0.0:
            return d
        acc = 0.0
        for k in range(d):
            acc += float(lam[k])
            if acc >= cumvar * tr:
                return k + 1
        return d
    return int(min(max(round(participation_ratio(lam)), 1), d))


def random_basis(c: np.ndarray, seed: int, stream: int):
    """(variances, basis) of the random-rotation variant: Q of the QR
    factorisation of a seeded Gaussian matrix (diag R > 0), its columns ordered
    by descending variance q_i^T C q_i (stable)."""
    c = np.asarray(c, dtype=np.float64)
    d = c.shape[0]
    g = rng.gaussians(seed ^ ROTATION_SALT, stream, d * d).reshape(d, d)
    q, r = np.linalg.qr(g)
    q = q * np.sign(np.diagonal(r))[None, :]
    var = np.einsum("ji,jk,ki->i", q, c, q)
    order = np.argsort(-var, kind="stable")
    return np.maximum(var[order], 0.0), q[:, order].copy()


def spectral_gap(lam: np.ndarray, d_eff: int) -> float:
    """kappa = lambda[d_eff - 1] / lambda[d_eff] (0-based); inf if d_eff == d."""
    d = len(lam)
    if d_eff >= d or lam[d_eff] == 0.0:
        return float("inf")
    return float(lam[d_eff - 1] / lam[d_eff])


def scales(lam: np.ndarray, normalize: bool) -> np.ndarray:
    """Quantizer scale sigma_i of each rotated coordinate."""
    lam = np.asarray(lam, dtype=np.float64)
    if not normalize:
        return np.sqrt(lam)
    tr = float(np.sum(lam))
    if tr == 0.0:
        return np.zeros_like(lam)
    return np.sqrt(lam / tr)


def water_fill(lam: np.ndarray, n_bits: int, max_bits: int = codebook.MAX_BITS) -> np.ndarray:
    """Greedy integer allocation of ``n_bits`` bits over the coordinates."""
    lam = np.asarray(lam, dtype=np.float64)
    d = lam.size
    if n_bits < 0 or n_bits > max_bits * d:
        raise ValueError("bit budget outside [0, max_bits * d]")
    dist = codebook.distortion_table(max_bits)
    bits = np.zeros(d, dtype=np.int64)
    for _ in range(n_bits):
        gain = np.where(bits < max_bits,
                        lam * (dist[np.minimum(bits, max_bits - 1)] - dist[np.minimum(bits + 1, max_bits)]),
                        -np.inf)
        i = int(np.argmax(gain))          # first maximum = lowest index on ties
        bits[i] += 1
    return bits


def bit_offsets(bits: np.ndarray) -> np.ndarray:
    """Bit position of coordinate i's code in the packed record."""
    return np.concatenate([[0], np.cumsum(bits)[:-1]]).astype(np.int64)


@dataclass
class HeadCalib:
    """One head's calibration: everything the codec and attention read."""

    d: int
    d_eff: int            # participation ratio, rounded
    m: int                # QJL sign dimensions (0 without QJL)
    total_bits: int       # B: bits of one packed record
    code_bits: int        # sum of b_i
    words: int            # 32-bit words of one record, ceil(B / 32)
    flags: int
    sweeps: int
    stream: int           # head index of the QJL stream
    max_bits: int
    seed: int
    trace: float
    kappa: float
    avg_bits: float
    lam: np.ndarray       # [d] descending
    sigma: np.ndarray     # [d]
    V: np.ndarray         # [d, d], column i = eigenvector i
    S: np.ndarray         # [m, m] QJL projection
    bits: np.ndarray      # [d] int
    offsets: np.ndarray   # [d] int
    fit_lv: np.ndarray | None = None   # [2, 510] fitted levels (signal, noise regime) or None
    fit_th: np.ndarray | None = None   # [2, 502] fitted thresholds or None

    @property
    def is_key(self) -> bool:
        return bool(self.flags & FLAG_IS_KEY)

    @property
    def qjl(self) -> bool:
        return bool(self.flags & FLAG_QJL)

    @property
    def normalize(self) -> bool:
        return bool(self.flags & FLAG_NORMALIZE)

    @property
    def fitted(self) -> bool:
        return bool(self.flags & FLAG_FITTED)

    def codebook(self, i: int):
        """(levels, thresholds) that code coordinate i (its width b_i >= 1)."""
        b = int(self.bits[i])
        if self.fitted:
            from . import fitted
            return fitted.codebook_of(self.fit_lv, self.fit_th, fitted.regime_of(i, self.d_eff), b)
        levels, thr, _ = codebook.lloyd_max(b)
        return levels, thr


def budget(d: int, avg_bits: float) -> int:
    """B = avg_bits * d, which must be a whole number of bits."""
    total = avg_bits * d
    if abs(total - round(total)) > 1e-9 or total <= 0:
        raise ValueError(f"avg_bits * d = {total} is not a positive integer")
    return int(round(total))


def finalize(lam: np.ndarray, vec: np.ndarray, *, avg_bits: float, is_key: bool,
             qjl: bool = True, normalize: bool = True, d_eff_override: int = 0,
             max_bits: int = codebook.MAX_BITS, seed: int = 42, stream: int = 0,
             sweeps: int = 0, cumvar: float = 0.0, random_rotation: bool = False) -> HeadCalib:
    """Everything after the basis: d_eff, kappa, scales, bits, QJL matrix."""
    d = lam.size
    d_eff = effective_dim(lam, cumvar)
    kappa = spectral_gap(lam, d_eff)
    total = budget(d, avg_bits)
    use_qjl = bool(is_key and qjl)
    m = (d_eff_override if d_eff_override > 0 else d_eff) if use_qjl else 0
    if m > d:
        raise ValueError("QJL dimension above head_dim")
    code_bits = total - m
    if code_bits < 0 or code_bits > max_bits * d:
        raise ValueError("bit budget cannot hold the QJL bits and the codes")
    bits = water_fill(lam, code_bits, max_bits)
    flags = ((FLAG_IS_KEY if is_key else 0) | (FLAG_QJL if use_qjl else 0) | (FLAG_NORMALIZE if normalize else 0)
             | (FLAG_RANDOM_ROTATION if random_rotation else 0) | (FLAG_CUMVAR if cumvar > 0.0 else 0))
    return HeadCalib(
        d=d, d_eff=d_eff, m=m, total_bits=total, code_bits=code_bits,
        words=(total + 31) // 32, flags=flags, sweeps=sweeps, stream=stream,
        max_bits=max_bits, seed=seed, trace=float(np.sum(lam)), kappa=kappa,
        avg_bits=float(avg_bits), lam=lam.copy(), sigma=scales(lam, normalize),
        V=vec.copy(), S=rng.qjl_matrix(seed, stream, m), bits=bits,
        offsets=bit_offsets(bits))


def fit_codebooks(cal: HeadCalib, x: np.ndarray, iters: int | None = None) -> HeadCalib:
    """``cal`` with per-regime codebooks fitted to its calibration vectors
    ``x`` [N, d] (the z the compressor would quantize; see fitted.py)."""
    from . import codec, fitted
    it = fitted.FIT_ITERS if iters is None else iters
    _, y = codec.rotate(x, cal)
    z = codec.scaled(y, cal)
    lv, th = fitted.fit_tables(z, cal.bits, cal.d_eff, it)
    cal.fit_lv, cal.fit_th = lv, th
    cal.flags |= FLAG_FITTED
    return cal


def calibrate(x: np.ndarray, *, rotation: str = "spectral", codebooks: str = "gaussian",
              fit_iters: int | None = None, **kw) -> HeadCalib:
    """Calibrate one head from its calibration vectors ``x`` [N, d]; ``rotation``
    is "spectral" (the calibrated eigenbasis) or "random" (the A/B baseline);
    ``codebooks`` is "gaussian" (the shared Lloyd-Max tables) or "fitted"
    (per-regime tables fitted to ``x``)."""
    c = second_moment(x)
    if rotation == "random":
        lam, vec = random_basis(c, kw.get("seed", 42), kw.get("stream", 0))
        cal = finalize(lam, vec, random_rotation=True, **kw)
    else:
        lam, vec = eigenbasis(c)
        cal = finalize(lam, vec, **kw)
    if codebooks == "fitted":
        cal = fit_codebooks(cal, x, fit_iters)
    elif codebooks != "gaussian":
        raise ValueError(f"unknown codebooks {codebooks!r}")
    return cal
