"""Calibration stability: the spread of compression quality across independent
calibration draws.

The SpectralQuant README lists "Calibration stability (CV=3.9%)" among its
results (``run_calibration_stability.py``, ``results/calibration_stability/``):
calibration is a one-time step on a sample of vectors, and the quality of the
compression it yields should not depend much on which sample was drawn.

The study, for one workload shape and its first ``heads`` KV heads of one layer:
  * ``n_draws`` independent calibration sets of ``n_cal`` vectors per head (the
    same population: the synthetic generator's head model), each calibrated on
    the GPU with sq_calibrate;
  * one fixed evaluation set of ``n_eval`` vectors per head, compressed with
    each draw's records (sq_compress_kv) and reconstructed (sq_decompress_kv;
    keys with their QJL term, values without one);
  * the quality readout of a draw: the mean cosine similarity of the
    reconstructed vectors against the originals;
  * the coefficient of variation (standard deviation / mean, population
    standard deviation) of the readout across the draws, for keys and values.
Every codec step runs in libsq; torch holds the buffers and averages the
readout.
"""

from __future__ import annotations

import math

import torch

from . import sq


def _readout(x: torch.Tensor, xh: torch.Tensor) -> float:
    """Mean cosine similarity of the rows of xh against the rows of x (float64)."""
    x = x.double()
    xh = xh.double()
    num = (x * xh).sum(-1)
    den = x.norm(dim=-1) * xh.norm(dim=-1)
    cos = torch.where(den > 0, num / den.clamp_min(1e-300), torch.ones_like(num))
    return float(cos.mean().item())


def calibration_stability(name: str, n_draws: int = 8, n_eval: int = 4096, heads: int = 2, layer: int = 0,
                          device: str = "cuda", bits: float | None = None) -> dict:
    """Per-draw readouts and their coefficient of variation for keys and values
    (see the module docstring). ``bits`` overrides the workload's bits per
    coordinate for both sides."""
    from synthetic.workloads import CONFIGS, make_workload

    cfg = dict(CONFIGS[name])
    g = cfg["n_q"] // cfg["n_kv"]
    cfg.update(n_kv=heads, n_q=heads * g)
    if bits is not None:
        cfg["bits_k"] = cfg["bits_v"] = float(bits)
    d = cfg["d"]
    ev = make_workload(cfg, layer, device=device, batch=1, tokens=n_eval, with_calibration=False)
    out = {"keys": [], "values": []}
    recon = torch.empty(1, heads, n_eval, d, dtype=torch.float32, device=device)
    for draw in range(n_draws):
        cal = make_workload(cfg, layer, device=device, batch=1, tokens=1, calib_draw=draw + 1)
        ncal = cal.k_cal.shape[1]
        for side, x_cal, x_eval, b, is_key in (("keys", cal.k_cal, ev.k, cfg["bits_k"], True),
                                                ("values", cal.v_cal, ev.v, cfg["bits_v"], False)):
            p = sq.calib_params(d, heads, b, is_key)
            recs = sq.alloc_records(heads, d, device)
            ws = torch.empty(sq.sq_calibrate_workspace(p, ncal), dtype=torch.uint8, device=device)
            status = torch.zeros(heads, dtype=torch.int32, device=device)
            sq.sq_calibrate(p, x_cal.contiguous(), ncal, ncal * d, d, recs, ws, status)
            cache = sq.alloc_cache(1, heads, n_eval, sq.sq_record_words(p), is_key and p.qjl == 1, device)
            xe = x_eval.contiguous()
            if is_key:
                sq.sq_compress_kv(recs, None, xe, None, 1, heads, d, n_eval, None, cache, None)
            else:
                sq.sq_compress_kv(None, recs, None, xe, 1, heads, d, n_eval, None, None, cache)
            sq.sq_decompress_kv(recs, cache, d, 0, n_eval, is_key, recon)
            torch.cuda.synchronize(device)
            if int((status != 0).sum().item()):
                raise RuntimeError(f"calibration draw {draw} of the {side} did not converge")
            out[side].append(_readout(xe.reshape(-1, d), recon.reshape(-1, d)))
    res = {"workload": name, "draws": n_draws, "eval_vectors_per_head": n_eval, "heads": heads,
           "calibration_vectors_per_head": cfg["n_cal"]}
    for side, vals in out.items():
        mean = sum(vals) / len(vals)
        sd = math.sqrt(sum((v - mean) ** 2 for v in vals) / len(vals))
        res[side] = {"per_draw": vals, "mean": mean, "cv": sd / mean if mean else float("nan")}
    return res
