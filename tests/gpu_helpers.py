"""Helpers shared by the GPU parity tests: oracle records on the device,
exemption masks, and the comparison rules.

Tolerances (stated once, used by every parity test):
* packed codes and QJL bits: bit-exact after masking the fields the oracle
  marks exempt (z within 1e-5 * max(1, |t|) of a threshold; a QJL projection
  within 1e-5 * ||S_j|| * rho of 0; all QJL bits and rho of a token with an
  exempt signal-dim code);
* stored norms: relative 1e-6 (a float32 rounding of the float64 value);
* rho: relative 1e-5 on non-exempt tokens (float64 residual stored as float32);
* reconstruction: relative L2 per vector <= 1e-4 (vectors without exempt codes);
* attention scores: relative L2 per (batch, query head) row <= 1e-3;
* attention outputs: relative L2 per (batch, query head) <= 2e-3;
* exempt fields of one comparison: exempt codes at most 2e-3 of the codes
  compared plus 2, and QJL bits exempt through their own band (not through an
  exempt signal code of their token) at most 2e-3 of the bits plus 2, so that
  an over-permissive exemption rule cannot hide a mismatch. (A code of b bits
  lies within 1e-5 of one of its 2^b - 1 thresholds with probability of order
  2e-5 2^b / 6, about 1e-3 for the 8-bit signal codes.)
"""

from __future__ import annotations

import numpy as np
import torch

from compressed_attention_head_b200 import sq
from oracle import calibration as ocal
from oracle import codec as ocodec
from oracle import record as orec

TOL_NORM = 1e-6
TOL_RHO = 1e-5
TOL_RECON = 1e-4
TOL_SCORES = 1e-3
TOL_OUT = 2e-3
MAX_EXEMPT_FRACTION = 2e-3


def records_to_device(cals, device="cuda") -> torch.Tensor:
    """Oracle HeadCalibs -> imported device records (the library builds its derived part)."""
    d = cals[0].d
    size = sq.sq_calib_bytes(d)
    host = np.zeros(len(cals) * size, dtype=np.uint8)
    for i, c in enumerate(cals):
        raw = np.frombuffer(orec.write(c), dtype=np.uint8)
        host[i * size:i * size + raw.size] = raw
    dev = torch.from_numpy(host).to(device)
    status = torch.full((len(cals),), -1, dtype=torch.int32, device=device)
    sq.sq_calib_import(dev, len(cals), d, status)
    torch.cuda.synchronize()
    assert status.cpu().tolist() == [0] * len(cals)
    return dev


def read_records(dev: torch.Tensor, n: int, d: int):
    raw = dev.cpu().numpy().tobytes()
    size = sq.sq_calib_bytes(d)
    return [orec.read(raw[i * size:(i + 1) * size]) for i in range(n)]


def calibrate_oracle(x_cal: torch.Tensor, avg_bits, is_key, qjl=True, normalize=True, seed=42, d_eff_override=0):
    """One oracle HeadCalib per head of x_cal [n_heads, N, d] (stream = head index)."""
    return [ocal.calibrate(x_cal[h].double().cpu().numpy(), avg_bits=avg_bits, is_key=is_key, qjl=qjl,
                           normalize=normalize, seed=seed, stream=h, d_eff_override=d_eff_override)
            for h in range(x_cal.shape[0])]


def exempt_mask(out: dict, cal) -> np.ndarray:
    """uint32 [T, W] mask of the record bits that may differ from the oracle's."""
    code_ex, q_ex, _ = ocodec.exemptions(out, cal)
    t = code_ex.shape[0]
    mask = np.zeros((t, cal.words * 32), dtype=bool)
    for i in range(cal.d):
        b = int(cal.bits[i])
        if b:
            mask[code_ex[:, i], cal.offsets[i]:cal.offsets[i] + b] = True
    for j in range(cal.m):
        mask[q_ex[:, j], cal.code_bits + j] = True
    words = np.zeros((t, cal.words), dtype=np.uint64)
    for k in range(cal.words * 32):
        words[:, k // 32] |= mask[:, k].astype(np.uint64) << np.uint64(k % 32)
    return words.astype(np.uint32)


def compare_compressed(gpu_words: np.ndarray, gpu_norm: np.ndarray, gpu_rnorm, x: np.ndarray, cal):
    """Checks one head's GPU records against the oracle; returns exemption counts."""
    out = ocodec.compress(x, cal)
    mask = exempt_mask(out, cal)
    diff = (gpu_words ^ out["words"]) & ~mask
    bad = np.argwhere(diff != 0)
    assert bad.size == 0, f"{len(bad)} words differ, first at token/word {bad[:5].tolist()}"
    ref_n = out["norm64"]
    assert np.all(np.abs(gpu_norm - ref_n) <= TOL_NORM * np.maximum(ref_n, 1e-30)), "norm mismatch"
    code_ex, q_ex, rho_ex = ocodec.exemptions(out, cal)
    n_codes = code_ex.shape[0] * int(np.count_nonzero(cal.bits))
    n_code_ex = int(code_ex.sum())
    assert n_code_ex <= MAX_EXEMPT_FRACTION * n_codes + 2, f"{n_code_ex} exempt codes of {n_codes}"
    if cal.m > 0:
        band_ex = int((q_ex & ~rho_ex[:, None]).sum())
        assert band_ex <= MAX_EXEMPT_FRACTION * q_ex.size + 2, f"{band_ex} exempt QJL bits of {q_ex.size}"
    if cal.m > 0:
        ok = ~rho_ex
        ref_r = out["rho64"][ok]
        got = np.asarray(gpu_rnorm)[ok]
        assert np.all(np.abs(got - ref_r) <= TOL_RHO * np.maximum(ref_r, 1e-30) + 1e-12), "rho mismatch"
    return int(code_ex.sum()), int(q_ex.sum())


def rel_l2_rows(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    num = np.linalg.norm(a - b, axis=-1)
    den = np.linalg.norm(b, axis=-1)
    return num / np.maximum(den, 1e-300)
