"""Pins of the oracle's decode attention over the packed cache."""

import math

import numpy as np
import torch

from oracle import attention, calibration as cal, codec
from synthetic import make_workload


def _build(cfg_name="tiny", g=1, tokens=256, n_kv=2, bits_k=3.0, bits_v=3.0, seq=None):
    w = make_workload(cfg_name, tokens=tokens)
    n_kv = min(n_kv, w.cfg["n_kv"])
    ck, cv, kw, kn, kr, vw, vn = [], [], [], [], [], [], []
    for h in range(n_kv):
        a = cal.calibrate(w.k_cal[h].double().numpy(), avg_bits=bits_k, is_key=True, seed=42, stream=h)
        b = cal.calibrate(w.v_cal[h].double().numpy(), avg_bits=bits_v, is_key=False, seed=42, stream=100 + h)
        ok = codec.compress(w.k[0, h].double().numpy(), a)
        ov = codec.compress(w.v[0, h].double().numpy(), b)
        ck.append(a); cv.append(b)
        kw.append(ok["words"]); kn.append(ok["norm"]); kr.append(ok["rnorm"])
        vw.append(ov["words"]); vn.append(ov["norm"])
    q = np.random.default_rng(0).standard_normal((1, n_kv * g, w.cfg["d"])) * 0.5
    st = lambda xs: np.stack(xs)[None]
    return q, st(kw), st(kn), st(kr), st(vw), st(vn), ck, cv


def test_equals_dense_attention_on_decompressed_vectors():
    for g in (1, 3):
        q, kw, kn, kr, vw, vn, ck, cv = _build(g=g)
        scale = 1 / math.sqrt(q.shape[-1])
        out, scores = attention.attn_decode(q, kw, kn, kr, vw, vn, ck, cv, [kw.shape[2]], scale)
        for h in range(q.shape[1]):
            kv = h // g
            keys = codec.decompress(kw[0, kv], kn[0, kv], kr[0, kv], ck[kv], apply_qjl=True)
            vals = codec.decompress(vw[0, kv], vn[0, kv], None, cv[kv], apply_qjl=False)
            o, s = attention.dense_attention(q[0, h], keys, vals, scale)
            assert np.allclose(scores[0, h], s, rtol=1e-11, atol=1e-11)
            assert np.allclose(out[0, h], o, rtol=1e-11, atol=1e-13)


def test_single_token_returns_its_value():
    q, kw, kn, kr, vw, vn, ck, cv = _build(tokens=8)
    out, _ = attention.attn_decode(q, kw, kn, kr, vw, vn, ck, cv, [1], None)
    v0 = codec.decompress(vw[0, 0, :1], vn[0, 0, :1], None, cv[0], apply_qjl=False)[0]
    assert np.allclose(out[0, 0], v0, rtol=1e-12, atol=1e-14)


def test_ragged_lengths_and_nan_padding():
    q, kw, kn, kr, vw, vn, ck, cv = _build(tokens=40)
    q2 = np.concatenate([q, q])
    kw2, kn2, kr2, vw2, vn2 = (np.concatenate([a, a]) for a in (kw, kn, kr, vw, vn))
    out, scores = attention.attn_decode(q2, kw2, kn2, kr2, vw2, vn2, ck, cv, [40, 17], None)
    assert np.all(np.isnan(scores[1, :, 17:])) and not np.any(np.isnan(scores[1, :, :17]))
    o17, _ = attention.attn_decode(q, kw[:, :, :17], kn[:, :, :17], kr[:, :, :17], vw[:, :, :17],
                                   vn[:, :, :17], ck, cv, [17], None)
    assert np.allclose(out[1], o17[0], rtol=1e-12)


def test_uniform_scores_average_values():
    """A zero query gives equal weights: the output is the mean decompressed value."""
    q, kw, kn, kr, vw, vn, ck, cv = _build(tokens=32)
    out, scores = attention.attn_decode(np.zeros_like(q), kw, kn, kr, vw, vn, ck, cv, [32], None)
    assert np.all(scores == 0.0)
    vals = codec.decompress(vw[0, 0], vn[0, 0], None, cv[0], apply_qjl=False)
    assert np.allclose(out[0, 0], vals.mean(axis=0), rtol=1e-12, atol=1e-14)


def test_dense_attention_matches_library_softmax_attention():
    """The oracle's dense reference against PyTorch's scaled_dot_product_attention
    (float64, CPU) on random keys, values and queries, several lengths and
    scales, including a query that makes the softmax nearly one-hot."""
    rng = np.random.default_rng(7)
    for L, d, scale in [(1, 32, 0.2), (17, 64, 1 / 8), (300, 128, 1 / math.sqrt(128)), (64, 32, 40.0)]:
        keys = rng.standard_normal((L, d))
        vals = rng.standard_normal((L, d))
        q = rng.standard_normal(d)
        o, s = attention.dense_attention(q, keys, vals, scale)
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(q)[None, None, None], torch.from_numpy(keys)[None, None],
            torch.from_numpy(vals)[None, None], scale=scale)[0, 0, 0].numpy()
        assert np.allclose(o, ref, rtol=1e-12, atol=1e-12)
        assert np.allclose(s, scale * keys @ q, rtol=1e-13, atol=1e-13)


def test_prefill_equals_causal_dense_attention_on_decompressed_vectors():
    """The prefill oracle against PyTorch's causal scaled_dot_product_attention
    (float64) over the decompressed keys (with their QJL term) and values: a
    chunk of 9 queries at positions 23 .. 31 of a 32-token cache, G = 2."""
    g = 2
    q, kw, kn, kr, vw, vn, ck, cv = _build(g=g, tokens=32)
    rng = np.random.default_rng(3)
    t_len, start = 9, 23
    qs = rng.standard_normal((1, q.shape[1], t_len, q.shape[2])) * 0.5
    scale = 1 / math.sqrt(q.shape[2])
    out = attention.attn_prefill(qs, kw, kn, kr, vw, vn, ck, cv, [start], scale)
    for h in range(qs.shape[1]):
        kv = h // g
        keys = codec.decompress(kw[0, kv], kn[0, kv], kr[0, kv], ck[kv], apply_qjl=True)
        vals = codec.decompress(vw[0, kv], vn[0, kv], None, cv[kv], apply_qjl=False)
        # query t sees keys 0 .. start + t: a boolean mask over the 32 keys
        mask = np.arange(32)[None, :] <= (start + np.arange(t_len))[:, None]
        ref = torch.nn.functional.scaled_dot_product_attention(
            torch.from_numpy(qs[0, h])[None, None], torch.from_numpy(keys)[None, None],
            torch.from_numpy(vals)[None, None], attn_mask=torch.from_numpy(mask)[None, None], scale=scale)[0, 0]
        assert np.allclose(out[0, h], ref.numpy(), rtol=1e-10, atol=1e-12)


def test_prefill_last_query_is_a_decode_query():
    """The last query of a chunk ending at the cache's end attends to the whole
    cache: it equals attn_decode of the same query at that length."""
    q, kw, kn, kr, vw, vn, ck, cv = _build(g=1, tokens=20)
    qs = np.repeat(q[:, :, None, :], 4, axis=2)
    out = attention.attn_prefill(qs, kw, kn, kr, vw, vn, ck, cv, [16], None)
    dec, _ = attention.attn_decode(q, kw, kn, kr, vw, vn, ck, cv, [20], None)
    assert np.allclose(out[0, :, 3], dec[0], rtol=1e-13, atol=1e-14)
    dec16, _ = attention.attn_decode(q, kw, kn, kr, vw, vn, ck, cv, [17], None)
    assert np.allclose(out[0, :, 0], dec16[0], rtol=1e-13, atol=1e-14)
