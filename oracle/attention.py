"""Decode attention read straight from the packed cache (oracle, float64).

Sources
-------
* SpectralQuant README, "Headline Results": per-step decode latency of
  attention over the compressed cache (512 tokens), and "Key Findings" 3
  (faster than TurboQuant at 512/1024/2048 tokens).
* SpectralQuant README, "Overview": keys carry the QJL correction on their
  signal dimensions only; values are quantized without it ("KV spectral
  asymmetry": value spectra are much flatter).

For batch row b and query head h, with KV head g = h // G (contiguous
grouped-query mapping, G = n_q / n_kv) and L = seq_len[b]:
  q'    = V_K^T q                           (query in the key eigenbasis)
  dot_t = sum_i q'_i sigma_K,i c_hat_t,i
  qjl_t = sqrt(pi/2) / m * rho_t * sum_j (S q'[:m])_j s_t,j    (keys with QJL)
  s_t   = scale * ||k_t|| * (dot_t + qjl_t)                     (t < L)
  p     = softmax(s)                  (float64, max subtracted)
  acc_i = sum_t p_t ||v_t|| c_hat^V_t,i
  o     = V_V (sigma_V * acc)
This equals dense softmax attention of q over the decompressed keys (with
the QJL term) and values (without it), which the tests check.
Readings taken: scale defaults to 1/sqrt(d); no logit soft-cap, window or
positional rotation is applied (none is part of the compressed path).
"""

from __future__ import annotations

import math

import numpy as np

from . import codec
from .calibration import HeadCalib


def attend_one(q: np.ndarray, k_words, k_norm, k_rnorm, v_words, v_norm,
               cal_k: HeadCalib, cal_v: HeadCalib, scale: float):
    """(output [d], scores [L]) of one query vector over one packed KV head."""
    q = np.asarray(q, dtype=np.float64)
    qp = cal_k.V.T @ q
    codes, qbits = codec.unpack(k_words, cal_k)
    c_hat = codec.levels(codes, cal_k)
    dot = c_hat @ (cal_k.sigma * qp)
    if cal_k.m > 0:
        sq = cal_k.S @ qp[:cal_k.m]
        s = 2.0 * qbits - 1.0
        dot = dot + (codec.QJL_SCALE / cal_k.m) * np.asarray(k_rnorm, np.float64) * (s @ sq)
    kn = np.asarray(k_norm, np.float64) if cal_k.normalize else np.ones(len(dot))
    scores = scale * kn * dot
    if scores.size == 0:
        return np.zeros(cal_v.d), scores
    p = np.exp(scores - np.max(scores))
    p /= np.sum(p)
    vcodes, _ = codec.unpack(v_words, cal_v)
    v_hat = codec.levels(vcodes, cal_v)
    vn = np.asarray(v_norm, np.float64) if cal_v.normalize else np.ones(len(p))
    acc = (p * vn) @ v_hat
    return cal_v.V @ (cal_v.sigma * acc), scores


def attn_decode(q, k_words, k_norm, k_rnorm, v_words, v_norm, cals_k, cals_v,
                seq_lens, scale: float | None = None):
    """Decode attention for every batch row and query head.

    q [B, n_q, d]; k_words / v_words [B, n_kv, cap, W]; k_norm, k_rnorm,
    v_norm [B, n_kv, cap]; ``cals_k`` / ``cals_v``: one HeadCalib per KV head;
    seq_lens [B]. Returns (out [B, n_q, d], scores [B, n_q, max_len] with NaN
    past each row's length).
    """
    q = np.asarray(q, dtype=np.float64)
    bsz, n_q, d = q.shape
    n_kv = len(cals_k)
    group = n_q // n_kv
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    max_len = int(max(seq_lens)) if len(seq_lens) else 0
    out = np.zeros((bsz, n_q, d))
    scores = np.full((bsz, n_q, max_len), np.nan)
    for b in range(bsz):
        n = int(seq_lens[b])
        for h in range(n_q):
            g = h // group
            rnorm = k_rnorm[b, g, :n] if k_rnorm is not None else np.zeros(n)
            o, s = attend_one(q[b, h], k_words[b, g, :n], k_norm[b, g, :n], rnorm,
                              v_words[b, g, :n], v_norm[b, g, :n], cals_k[g], cals_v[g], scale)
            out[b, h] = o
            scores[b, h, :n] = s
    return out, scores


def attn_prefill(q, k_words, k_norm, k_rnorm, v_words, v_norm, cals_k, cals_v, starts, scale: float | None = None):
    """Causal attention of a chunk of queries over the packed cache (prefill).

    q [B, n_q, T, d]; query t of row b sits at position starts[b] + t and
    attends to the packed tokens 0 .. starts[b] + t of its KV head, exactly as
    one decode query over that prefix (``attend_one``). Returns out [B, n_q, T, d].
    Reading taken: the pages measure the method over sequence lengths 512-2048
    (SpectralQuant README, "Key Findings" 3) without stating how prompts pass
    through attention; causal attention over the compressed cache is the plain
    reading.
    """
    q = np.asarray(q, dtype=np.float64)
    bsz, n_q, t_len, d = q.shape
    n_kv = len(cals_k)
    group = n_q // n_kv
    if scale is None or scale <= 0:
        scale = 1.0 / math.sqrt(d)
    out = np.zeros((bsz, n_q, t_len, d))
    for b in range(bsz):
        for h in range(n_q):
            g = h // group
            for t in range(t_len):
                n = int(starts[b]) + t + 1
                rnorm = k_rnorm[b, g, :n] if k_rnorm is not None else np.zeros(n)
                out[b, h, t], _ = attend_one(q[b, h, t], k_words[b, g, :n], k_norm[b, g, :n], rnorm,
                                             v_words[b, g, :n], v_norm[b, g, :n], cals_k[g], cals_v[g], scale)
    return out


def dense_attention(q: np.ndarray, keys: np.ndarray, values: np.ndarray, scale: float):
    """Softmax attention of one query over explicit keys [L, d] and values [L, d]."""
    s = scale * (np.asarray(keys, np.float64) @ np.asarray(q, np.float64))
    p = np.exp(s - np.max(s))
    p /= np.sum(p)
    return p @ np.asarray(values, np.float64), s
