"""Byte layout of one head's calibration record, canonical part (oracle side).

The CUDA library consumes calibration records as plain bytes, so a record
written here can be imported by the library and compared bit for bit. This
module writes and reads only the canonical part; the library appends its own
kernel-ready section after it (see the layout table in the public header).
All fields are little-endian.

  offset               type   field
  0                    u32    magic 0x31435153 ("SQC1")
  4                    u32    version (2)
  8                    i32    d
  12                   i32    d_eff (participation ratio, rounded)
  16                   i32    m (QJL sign dimensions; 0 without QJL)
  20                   i32    total_bits B
  24                   i32    code_bits (sum of b_i)
  28                   i32    words W = ceil(B / 32)
  32                   u32    flags: 1 key, 2 QJL, 4 normalized, 8 random rotation,
                              16 cumulative-variance d_eff, 32 fitted codebooks
  36                   i32    eigensolver sweeps (0 when not from the library)
  40                   i32    stream (head index of the QJL Gaussian stream)
  44                   i32    max_bits
  48                   u64    seed
  56                   f64    trace (sum of eigenvalues)
  64                   f64    kappa (spectral gap; +inf when d_eff = d)
  72                   f64    avg_bits
  80                   u32    library use (0 here)
  84 .. 127                   zero
  128                  f64    lambda[d], descending
  128 + 8d             f64    sigma[d]
  128 + 16d            f64    V[d*d], row-major: V[j*d + i] = component j of eigenvector i
  128 + 16d + 8d^2     f64    S[d*d]: the m x m QJL matrix row-major in its first m*m slots
  128 + 16d + 16d^2    u8     bits[d]
  128 + 17d + 16d^2    i32    offset[d] (bit position of coordinate i's code)
  128 + 21d + 16d^2    f64    fitted levels [2][510] (signal, noise regime; width b
                              at 2^b - 2), zero unless flag 32
  8288 + 21d + 16d^2   f64    fitted thresholds [2][502] (width b at 2^b - 1 - b)
  16320 + 21d + 16d^2         end of the canonical part
"""

from __future__ import annotations

import struct

import numpy as np

from . import fitted
from .calibration import FLAG_FITTED, HeadCalib

MAGIC = 0x31435153
VERSION = 2
HEADER = 128
FIT_BYTES = 8 * 2 * (fitted.N_LEVELS + fitted.N_THRESH)


def canonical_bytes(d: int) -> int:
    """Size of the canonical part of a record for head_dim ``d``."""
    return HEADER + 21 * d + 16 * d * d + FIT_BYTES


def write(cal: HeadCalib) -> bytes:
    """Canonical bytes of ``cal``."""
    d = cal.d
    buf = bytearray(canonical_bytes(d))
    struct.pack_into("<IIiiiiiiIiii", buf, 0, MAGIC, VERSION, d, cal.d_eff, cal.m,
                     cal.total_bits, cal.code_bits, cal.words, cal.flags, cal.sweeps,
                     cal.stream, cal.max_bits)
    struct.pack_into("<Qddd", buf, 48, cal.seed & ((1 << 64) - 1), cal.trace, cal.kappa, cal.avg_bits)
    o = HEADER
    buf[o:o + 8 * d] = np.asarray(cal.lam, "<f8").tobytes(); o += 8 * d
    buf[o:o + 8 * d] = np.asarray(cal.sigma, "<f8").tobytes(); o += 8 * d
    buf[o:o + 8 * d * d] = np.asarray(cal.V, "<f8").reshape(-1).tobytes(); o += 8 * d * d
    s = np.zeros(d * d)
    s[:cal.m * cal.m] = np.asarray(cal.S, np.float64).reshape(-1)
    buf[o:o + 8 * d * d] = s.astype("<f8").tobytes(); o += 8 * d * d
    buf[o:o + d] = np.asarray(cal.bits, np.uint8).tobytes(); o += d
    buf[o:o + 4 * d] = np.asarray(cal.offsets, "<i4").tobytes(); o += 4 * d
    if cal.flags & FLAG_FITTED:
        lv = np.asarray(cal.fit_lv, "<f8").reshape(-1)
        th = np.asarray(cal.fit_th, "<f8").reshape(-1)
        buf[o:o + lv.nbytes] = lv.tobytes()
        buf[o + lv.nbytes:o + lv.nbytes + th.nbytes] = th.tobytes()
    o += FIT_BYTES
    assert o == canonical_bytes(d)
    return bytes(buf)


def read(raw: bytes) -> HeadCalib:
    """HeadCalib from canonical bytes (extra trailing bytes are ignored)."""
    raw = bytes(raw)
    (magic, version, d, d_eff, m, total, code_bits, words, flags, sweeps, stream,
     max_bits) = struct.unpack_from("<IIiiiiiiIiii", raw, 0)
    if magic != MAGIC or version != VERSION:
        raise ValueError("not a version-2 calibration record")
    seed, trace, kappa, avg_bits = struct.unpack_from("<Qddd", raw, 48)
    o = HEADER

    def take(n, dtype):
        nonlocal o
        a = np.frombuffer(raw, dtype=dtype, count=n, offset=o).copy()
        o += n * np.dtype(dtype).itemsize
        return a

    lam = take(d, "<f8")
    sigma = take(d, "<f8")
    V = take(d * d, "<f8").reshape(d, d)
    S = take(d * d, "<f8")[:m * m].reshape(m, m)
    bits = take(d, np.uint8).astype(np.int64)
    offsets = take(d, "<i4").astype(np.int64)
    fit_lv = take(2 * fitted.N_LEVELS, "<f8").reshape(2, fitted.N_LEVELS)
    fit_th = take(2 * fitted.N_THRESH, "<f8").reshape(2, fitted.N_THRESH)
    fit = bool(flags & FLAG_FITTED)
    return HeadCalib(d=d, d_eff=d_eff, m=m, total_bits=total, code_bits=code_bits,
                     words=words, flags=flags, sweeps=sweeps, stream=stream,
                     max_bits=max_bits, seed=seed, trace=trace, kappa=kappa,
                     avg_bits=avg_bits, lam=lam, sigma=sigma, V=V, S=S, bits=bits,
                     offsets=offsets, fit_lv=fit_lv if fit else None, fit_th=fit_th if fit else None)
