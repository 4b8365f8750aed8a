"""Synthetic keys, values and queries with the spectra the pages report.

The pages measure real models (Qwen2.5 1.5B/7B/14B, Llama-3.1-8B, Mistral-7B,
Gemma-2-9B); no weights or datasets are available, so seeded Gaussian draws
with matching second-moment structure stand in for them:

* SpectralQuant README, "Key Findings": key vectors concentrate their energy
  in 3-4 % of head_dim (d_eff ~ 4 for keys) and values are much flatter
  (d_eff ~ 40-55).
* TurboQuant reference implementation README, "K/V Norm Disparity" (mean key
  norms 274.0 for Qwen2.5-7B and 778.6 for Qwen2.5-1.5B, value norms 2.6-4.3)
  and "Outlier-Aware Mixed Precision" (5-20 % of key channels with 10-100x
  the median RMS).
* spectralquant tests/conftest.py, fixture ``sharp_gap_kv_data``: diagonal
  spectra of 50 on the signal dims and 1 elsewhere, head_dim 32, 256 tokens,
  seed 42.

Recipe, per (layer, KV head) with its own seeded generator:
  keys   k = (z * sqrt(lam)) Q^T, z ~ N(0, I), Q Haar-orthogonal; lam = spikes
         log-spaced from 1e3 down to 1e2 on ``k_spikes`` dims, 1 elsewhere;
         then per-channel multipliers (outlier channels raised to ``outlier_rms``
         x the median channel RMS, or heavy-tailed |t_3| multipliers
         normalised to median 1); then one scale so that the RMS key norm is
         ``k_norm``.
  values v = (z * sqrt(lam_v)) Q_v^T, lam_v = 50 on ``v_spikes`` dims, 1
         elsewhere, scaled to RMS norm ``v_norm``.
  query  a fresh draw from the key distribution, scaled so that the standard
         deviation of q.k / sqrt(d) over keys is 2 (unscaled logits of
         ||q|| ||k|| / sqrt(d) ~ 1e3 would make softmax one-hot).
  calibration vectors: a separate draw of ``n_cal`` tokens from the same
         distributions.
The tiny case follows the conftest fixture instead: keys N(0, diag(50 x 8,
1 x 24)) rotated by a random orthogonal matrix, values N(0, diag(50 x 12,
1 x 20)) unrotated, float32.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

# name -> shape of the workload. "mode" says what the benchmark step does:
# prefill = compress a prompt of ``ctx`` tokens, then one decode step;
# decode  = one decode step over a cache of ``ctx`` tokens per sequence.
CONFIGS = {
    "tiny": dict(layers=1, n_q=4, n_kv=4, d=32, dtype="f32", batch=1, ctx=256, n_cal=256,
                 bits_k=3.0, bits_v=3.0, mode="prefill", tiny=True, seed=42),
    "llama8b": dict(layers=32, n_q=32, n_kv=8, d=128, dtype="f16", batch=1, ctx=2048, n_cal=2048,
                    bits_k=3.0, bits_v=3.0, k_spikes=4, outliers=6, outlier_rms=20.0, t_scales=False,
                    k_norm=150.0, v_spikes=48, v_norm=3.0, mode="prefill", seed=42),
    "qwen14b": dict(layers=48, n_q=40, n_kv=8, d=128, dtype="f16", batch=4, ctx=8192, n_cal=2048,
                    bits_k=2.5, bits_v=3.0, k_spikes=4, outliers=0, outlier_rms=20.0, t_scales=False,
                    k_norm=270.0, v_spikes=48, v_norm=3.0, mode="decode", seed=42),
    "qwen1_5b_long": dict(layers=28, n_q=12, n_kv=2, d=128, dtype="f16", batch=16, ctx=32768, n_cal=2048,
                          bits_k=3.0, bits_v=3.0, k_spikes=4, outliers=0, outlier_rms=20.0, t_scales=True,
                          k_norm=780.0, v_spikes=40, v_norm=4.3, mode="decode", seed=42),
    "gemma9b_sweep": dict(layers=42, n_q=16, n_kv=8, d=256, dtype="bf16", batch=64, ctx=4096, n_cal=2048,
                          bits_k=3.0, bits_v=3.0, k_spikes=8, outliers=0, outlier_rms=20.0, t_scales=False,
                          k_norm=150.0, v_spikes=110, v_norm=3.0, mode="decode", seed=42,
                          sweep_bits=(2.0, 2.5, 3.0, 3.5, 4.0)),
}

TORCH_DTYPE = {"f32": torch.float32, "f16": torch.float16, "bf16": torch.bfloat16}
_STREAMS = {"model": 0, "calib": 1, "data": 2, "query": 3}


def _seed(base: int, *parts: int) -> int:
    ss = np.random.SeedSequence([base, *[int(p) for p in parts]])
    return int(ss.generate_state(1, dtype=np.uint64)[0] & ((1 << 63) - 1))


def _gen(device, base: int, *parts: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed(base, *parts))
    return g


@dataclass
class HeadModel:
    """Second-moment structure of one (layer, KV head, kind) population."""

    basis: torch.Tensor      # [d, d] orthogonal
    lam: torch.Tensor        # [d] variances along the basis
    chan: torch.Tensor       # [d] per-channel multipliers in the original basis
    scale: float             # overall scale

    def covariance(self) -> torch.Tensor:
        c = (self.basis * self.lam[None, :]) @ self.basis.T
        c = self.chan[:, None] * c * self.chan[None, :]
        return (self.scale ** 2) * c


def _haar(d: int, gen: torch.Generator, device) -> torch.Tensor:
    a = torch.randn(d, d, generator=gen, device=device, dtype=torch.float64)
    q, r = torch.linalg.qr(a)
    return q * torch.sign(torch.diagonal(r))[None, :]


def head_model(cfg: dict, layer: int, head: int, kind: str, device="cpu") -> HeadModel:
    d = cfg["d"]
    kid = 0 if kind == "k" else 1
    gen = _gen(device, cfg["seed"], _STREAMS["model"], layer, head, kid)
    f64 = dict(device=device, dtype=torch.float64)
    if cfg.get("tiny"):
        n_sig = 8 if kind == "k" else 12
        lam = torch.cat([torch.full((n_sig,), 50.0, **f64), torch.ones(d - n_sig, **f64)])
        basis = _haar(d, gen, device) if kind == "k" else torch.eye(d, **f64)
        return HeadModel(basis, lam, torch.ones(d, **f64), 1.0)
    basis = _haar(d, gen, device)
    chan = torch.ones(d, **f64)
    if kind == "k":
        k = cfg["k_spikes"]
        lam = torch.ones(d, **f64)
        lam[:k] = torch.logspace(3.0, 2.0, k, **f64)
        rms = torch.sqrt(torch.diagonal((basis * lam[None, :]) @ basis.T))
        if cfg.get("t_scales"):
            # |t_3| = |N| / sqrt(chi2_3 / 3), normalised to median 1.
            n = torch.randn(d, generator=gen, **f64)
            chi = (torch.randn(3, d, generator=gen, **f64) ** 2).sum(0) / 3.0
            t = torch.abs(n / torch.sqrt(chi))
            chan = t / torch.median(t)
        if cfg.get("outliers", 0):
            idx = torch.randperm(d, generator=gen, device=device)[: cfg["outliers"]]
            target = cfg["outlier_rms"] * torch.median(rms * chan)
            chan[idx] = target / rms[idx]
        norm2 = float(torch.sum((chan * rms) ** 2))
        scale = cfg["k_norm"] / math.sqrt(norm2)
    else:
        lam = torch.ones(d, **f64)
        lam[: cfg["v_spikes"]] = 50.0
        scale = cfg["v_norm"] / math.sqrt(float(lam.sum()))
    return HeadModel(basis, lam, chan, scale)


def draw(model: HeadModel, n: int, gen: torch.Generator, device, out_dtype=torch.float32) -> torch.Tensor:
    """``n`` vectors [n, d] from the head's distribution."""
    d = model.lam.numel()
    z = torch.randn(n, d, generator=gen, device=device, dtype=torch.float32)
    b = (model.basis * torch.sqrt(model.lam)[None, :]).T.to(torch.float32)      # [d, d]
    x = (z @ b) * (model.chan * model.scale).to(torch.float32)[None, :]
    return x.to(out_dtype)


@dataclass
class Workload:
    """Inputs of one layer: keys/values [B, n_kv, T, d], calibration [n_kv, N, d], queries [B, n_q, d]."""

    cfg: dict
    layer: int
    k: torch.Tensor
    v: torch.Tensor
    k_cal: torch.Tensor
    v_cal: torch.Tensor
    q: torch.Tensor
    models: dict = field(default_factory=dict)


def make_workload(name_or_cfg, layer: int = 0, *, device="cpu", batch: int | None = None,
                  tokens: int | None = None, n_cal: int | None = None, data_stream: int = 0,
                  with_calibration: bool = True, calib_draw: int = 0) -> Workload:
    """Draw one layer's inputs. ``tokens`` overrides the context length;
    ``calib_draw`` selects an independent draw of the calibration vectors from
    the same population (same head model, keys, values and queries)."""
    cfg = CONFIGS[name_or_cfg] if isinstance(name_or_cfg, str) else name_or_cfg
    bsz = cfg["batch"] if batch is None else batch
    t = cfg["ctx"] if tokens is None else tokens
    ncal = cfg["n_cal"] if n_cal is None else n_cal
    dt = TORCH_DTYPE[cfg["dtype"]]
    n_kv, n_q, d = cfg["n_kv"], cfg["n_q"], cfg["d"]
    group = n_q // n_kv
    k = torch.empty(bsz, n_kv, t, d, device=device, dtype=dt)
    v = torch.empty_like(k)
    k_cal = torch.empty(n_kv, ncal, d, device=device, dtype=dt)
    v_cal = torch.empty_like(k_cal)
    q = torch.empty(bsz, n_q, d, device=device, dtype=dt)
    models = {}
    for h in range(n_kv):
        mk = head_model(cfg, layer, h, "k", device)
        mv = head_model(cfg, layer, h, "v", device)
        models[h] = (mk, mv)
        gk = _gen(device, cfg["seed"], _STREAMS["data"], layer, h, 0, data_stream)
        gv = _gen(device, cfg["seed"], _STREAMS["data"], layer, h, 1, data_stream)
        k[:, h] = draw(mk, bsz * t, gk, device, dt).reshape(bsz, t, d)
        v[:, h] = draw(mv, bsz * t, gv, device, dt).reshape(bsz, t, d)
        if with_calibration:
            extra = (calib_draw,) if calib_draw else ()
            gck = _gen(device, cfg["seed"], _STREAMS["calib"], layer, h, 0, *extra)
            gcv = _gen(device, cfg["seed"], _STREAMS["calib"], layer, h, 1, *extra)
            k_cal[h] = draw(mk, ncal, gck, device, dt)
            v_cal[h] = draw(mv, ncal, gcv, device, dt)
        gq = _gen(device, cfg["seed"], _STREAMS["query"], layer, h, data_stream)
        qs = draw(mk, bsz * group, gq, device, torch.float64).reshape(bsz, group, d)
        ck = mk.covariance()
        var = torch.einsum("bgi,ij,bgj->bg", qs, ck, qs)
        qs = qs * (2.0 * math.sqrt(d) / torch.sqrt(var))[..., None]
        q[:, h * group:(h + 1) * group] = qs.to(dt)
    return Workload(cfg, layer, k, v, k_cal, v_cal, q, models)
