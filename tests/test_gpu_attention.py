"""GPU parity of decode attention over the packed cache against the oracle.

The oracle is fed the GPU's own packed cache (and the same imported
calibration records), which isolates attention from code-flip exemptions of
the compressor: scores must match per row within 1e-3 relative L2 and the
outputs within 2e-3.
"""

import math

import numpy as np
import pytest
import torch

from gpu_helpers import TOL_OUT, TOL_SCORES, calibrate_oracle, records_to_device, rel_l2_rows
from oracle import attention as oattn
from synthetic import CONFIGS, make_workload

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

from compressed_attention_head_b200 import sq  # noqa: E402


def _run(name, batch, ctx, seq_lens, heads=None, bits_k=None, bits_v=None, qjl=True, out_dtype=torch.float32,
         cap=None, d_eff_override=0):
    w = make_workload(name, batch=batch, tokens=ctx)
    cfg = w.cfg
    nkv = heads or cfg["n_kv"]
    group = cfg["n_q"] // cfg["n_kv"]
    nq = nkv * group
    d = cfg["d"]
    ck = calibrate_oracle(w.k_cal[:nkv], cfg["bits_k"] if bits_k is None else bits_k, True, qjl=qjl,
                          d_eff_override=d_eff_override)
    cv = calibrate_oracle(w.v_cal[:nkv], cfg["bits_v"] if bits_v is None else bits_v, False)
    rk, rv = records_to_device(ck), records_to_device(cv)
    cap = cap or ((ctx + 15) // 16) * 16
    kc = sq.alloc_cache(batch, nkv, cap, ck[0].words, ck[0].m > 0)
    vc = sq.alloc_cache(batch, nkv, cap, cv[0].words, False)
    k = w.k[:, :nkv].contiguous().cuda()
    v = w.v[:, :nkv].contiguous().cuda()
    sq.sq_compress_kv(rk, rv, k, v, batch, nkv, d, ctx, None, kc, vc)
    q = w.q[:, :nq].contiguous().cuda()
    lens = torch.tensor(seq_lens, dtype=torch.int32, device="cuda")
    max_ctx = max(max(seq_lens), 1)
    ws = torch.empty(sq.sq_attn_workspace(batch, nq, nkv, d, max_ctx), dtype=torch.uint8, device="cuda")
    out = torch.empty(batch, nq, d, dtype=out_dtype, device="cuda")
    scores = torch.full((batch, nq, max_ctx), float("nan"), device="cuda")
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    sq.sq_attn_decode(rk, rv, kc, vc, lens, batch, nq, nkv, d, max_ctx, q, 0.0, out, scores, ws, flags)
    torch.cuda.synchronize()
    ref_out, ref_scores = oattn.attn_decode(
        q.double().cpu().numpy(), kc.words_u32(), kc.norm.cpu().numpy(),
        kc.rnorm.cpu().numpy() if kc.rnorm is not None else None, vc.words_u32(), vc.norm.cpu().numpy(),
        ck, cv, seq_lens, 1.0 / math.sqrt(d))
    return out.float().cpu().numpy(), scores.cpu().numpy(), ref_out, ref_scores, flags.item()


def _assert_close(out, scores, ref_out, ref_scores, seq_lens, out_tol=TOL_OUT):
    for b, n in enumerate(seq_lens):
        if n == 0:
            assert np.all(out[b] == 0.0)
            continue
        err_s = rel_l2_rows(scores[b, :, :n], ref_scores[b, :, :n])
        assert np.max(err_s) <= TOL_SCORES, np.max(err_s)
        err_o = rel_l2_rows(out[b], ref_out[b])
        assert np.max(err_o) <= out_tol, np.max(err_o)


@pytest.mark.parametrize("name,batch,ctx,lens,heads", [
    ("tiny", 1, 256, [256], None),                         # G = 1
    ("llama8b", 2, 600, [600, 333], 2),                     # G = 4, ragged tail
    ("qwen14b", 2, 1100, [1100, 1], 2),                     # G = 5, one-token row
    ("qwen1_5b_long", 1, 2100, [2100], 2),                  # G = 6, several splits
    ("gemma9b_sweep", 2, 300, [300, 129], 2),               # G = 2, d = 256
])
def test_attention_parity(name, batch, ctx, lens, heads):
    out, scores, ref_out, ref_scores, flags = _run(name, batch, ctx, lens, heads=heads)
    assert flags == 0
    _assert_close(out, scores, ref_out, ref_scores, lens)


@pytest.mark.parametrize("bits", [2.0, 3.5])
@pytest.mark.parametrize("qjl", [True, False])
def test_attention_gemma_bits(bits, qjl):
    out, scores, ref_out, ref_scores, _ = _run("gemma9b_sweep", 1, 200, [200], heads=1, bits_k=bits, bits_v=bits,
                                               qjl=qjl)
    _assert_close(out, scores, ref_out, ref_scores, [200])


def test_attention_empty_row_and_half_output():
    out, scores, ref_out, ref_scores, flags = _run("llama8b", 2, 64, [0, 64], heads=1, out_dtype=torch.float16)
    assert flags == 0
    _assert_close(out, scores, ref_out, ref_scores, [0, 64], out_tol=2e-3 + 1e-3)


def test_attention_seq_len_past_bound_is_flagged():
    w = make_workload("tiny", batch=1, tokens=32)
    ck = calibrate_oracle(w.k_cal[:1], 3.0, True)
    cv = calibrate_oracle(w.v_cal[:1], 3.0, False)
    rk, rv = records_to_device(ck), records_to_device(cv)
    kc = sq.alloc_cache(1, 1, 32, ck[0].words, True)
    vc = sq.alloc_cache(1, 1, 32, cv[0].words, False)
    q = w.q[:, :1].contiguous().cuda()
    lens = torch.tensor([40], dtype=torch.int32, device="cuda")
    ws = torch.empty(sq.sq_attn_workspace(1, 1, 1, 32, 32), dtype=torch.uint8, device="cuda")
    out = torch.empty(1, 1, 32, device="cuda")
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    sq.sq_attn_decode(rk, rv, kc, vc, lens, 1, 1, 1, 32, 32, q, 0.0, out, None, ws, flags)
    torch.cuda.synchronize()
    assert flags.item() & sq.SQ_FLAG_SEQLEN
    with pytest.raises(sq.SqError) as e:
        sq.sq_attn_decode(rk, rv, kc, vc, lens, 1, 1, 1, 32, 32, q, 0.0, out, None, ws[:16], flags)
    assert e.value.status == sq.SQ_ERR_WORKSPACE


@pytest.mark.parametrize("name,ctx,heads", [("llama8b", 700, 2), ("gemma9b_sweep", 300, 2), ("qwen14b", 1500, 1)])
def test_every_partial_kernel_matches_the_oracle(name, ctx, heads):
    """The three attention partial kernels (tcgen05, SIMT, mma.sync) against the
    oracle on the same packed cache."""
    outs = {}
    try:
        for path in (0, 1, 2):
            sq.sq_set_option(sq.SQ_OPT_ATTN_PATH, path)
            outs[path] = _run(name, 1, ctx, [ctx], heads=heads)
    finally:
        sq.sq_set_option(sq.SQ_OPT_ATTN_PATH, 0)
    for path, (o, sc, r_o, r_s, flags) in outs.items():
        assert flags == 0, path
        _assert_close(o, sc, r_o, r_s, [ctx])


def test_full_size_decode_sampled_rows():
    """Qwen2.5-14B-shaped decode step (batch 4 at context 8192, one layer's 8 KV /
    40 query heads, the launch shape of one layer): every output and score row
    of two KV heads against the oracle."""
    out, scores, ref_out, ref_scores, flags = _run("qwen14b", 4, 8192, [8192, 8191, 4097, 8192], heads=2)
    assert flags == 0
    _assert_close(out, scores, ref_out, ref_scores, [8192, 8191, 4097, 8192])


def test_attention_more_than_sixteen_qjl_dimensions():
    """Keys with m = 24 QJL sign dimensions (d_eff_override) through the default
    (tensor-core) path: the signs take two 16-column blocks."""
    out, scores, ref_out, ref_scores, flags = _run("llama8b", 2, 300, [300, 257], heads=2, d_eff_override=24)
    assert flags == 0
    _assert_close(out, scores, ref_out, ref_scores, [300, 257])


def test_attention_head_dim_64():
    """head_dim 64 (a Llama-shaped head at half the width): G = 4, ragged rows."""
    cfg = dict(CONFIGS["llama8b"], d=64)
    out, scores, ref_out, ref_scores, flags = _run(cfg, 2, 500, [500, 77], heads=2)
    assert flags == 0
    _assert_close(out, scores, ref_out, ref_scores, [500, 77])


def _bench_shape_sampled(name, n_layers, batch, ctx, rows, distinct_heads=2, distinct_rows=None):
    """Decode attention in the launch configuration of the benchmark step (all
    layers folded into the KV-head index, batch x context of the workload,
    max_ctx = context + 1 for the appended token): the packed caches of
    ``distinct_heads`` KV heads and ``distinct_rows`` batch rows are compressed
    once and repeated over the layers' heads and the batch, and sampled (batch
    row, query head) rows are checked against the oracle."""
    cfg = CONFIGS[name]
    d, g = cfg["d"], cfg["n_q"] // cfg["n_kv"]
    # only the distinct heads are drawn (on the device: millions of vectors)
    nb = distinct_rows or batch
    w = make_workload(dict(cfg, n_kv=distinct_heads, n_q=distinct_heads * g), batch=nb, tokens=ctx,
                      device="cuda")
    ck = calibrate_oracle(w.k_cal[:distinct_heads], cfg["bits_k"], True)
    cv = calibrate_oracle(w.v_cal[:distinct_heads], cfg["bits_v"], False)
    nkv = n_layers * cfg["n_kv"]
    nq = nkv * g
    rk1, rv1 = records_to_device(ck), records_to_device(cv)
    size = sq.sq_calib_bytes(d)
    rep = nkv // distinct_heads
    rk = rk1.view(distinct_heads, size).repeat(rep, 1).reshape(-1).contiguous()
    rv = rv1.view(distinct_heads, size).repeat(rep, 1).reshape(-1).contiguous()
    cap = ((ctx + 1 + 31) // 32) * 32
    k1 = sq.alloc_cache(nb, distinct_heads, cap, ck[0].words, True)
    v1 = sq.alloc_cache(nb, distinct_heads, cap, cv[0].words, False)
    sq.sq_compress_kv(rk1, rv1, w.k.contiguous(), w.v.contiguous(), nb, distinct_heads, d, ctx, None, k1, v1)
    del w.k, w.v
    rb = batch // nb
    kc, vc = k1.tiled(rb, rep), v1.tiled(rb, rep)
    q = w.q.repeat(rb, rep, 1).contiguous()
    lens_l = [ctx - (7 * b) % 301 for b in range(batch)]
    lens = torch.tensor(lens_l, dtype=torch.int32, device="cuda")
    max_ctx = ctx + 1
    ws = torch.empty(sq.sq_attn_workspace(batch, nq, nkv, d, max_ctx), dtype=torch.uint8, device="cuda")
    out = torch.empty(batch, nq, d, device="cuda")
    scores = torch.full((batch, nq, max_ctx), float("nan"), device="cuda")
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    sq.sq_attn_decode(rk, rv, kc, vc, lens, batch, nq, nkv, d, max_ctx, q, 0.0, out, scores, ws, flags)
    torch.cuda.synchronize()
    assert flags.item() == 0
    kw, vw = k1.words_u32(), v1.words_u32()
    kn, kr, vn = k1.norm.cpu().numpy(), k1.rnorm.cpu().numpy(), v1.norm.cpu().numpy()
    scale = 1.0 / math.sqrt(d)
    for (b, h) in rows:
        gh = h // g
        src, sb = gh % distinct_heads, b % nb
        n = lens_l[b]
        ro, rs = oattn.attend_one(q[b, h].double().cpu().numpy(), kw[sb, src, :n], kn[sb, src, :n],
                                  kr[sb, src, :n], vw[sb, src, :n], vn[sb, src, :n], ck[src], cv[src], scale)
        got_s = scores[b, h, :n].cpu().numpy()
        got_o = out[b, h].cpu().numpy()
        assert rel_l2_rows(got_s[None], rs[None])[0] <= TOL_SCORES, (b, h)
        assert rel_l2_rows(got_o[None], ro[None])[0] <= TOL_OUT, (b, h)
    return sq.sq_attn_workspace(batch, nq, nkv, d, max_ctx)


def test_decode_qwen1_5b_long_bench_shape_sampled():
    """Qwen2.5-1.5B-shaped decode as benchmarked: batch 16 at context 32768, 28
    layers x 2 KV heads folded (56 KV / 336 query heads, head_dim 128)."""
    _bench_shape_sampled("qwen1_5b_long", 28, 16, 32768,
                         rows=[(0, 0), (3, 7), (9, 200), (15, 335), (12, 101)])


def test_decode_gemma_bench_shape_sampled():
    """Gemma-2-9B-shaped decode as benchmarked: batch 64 at context 4096, 42
    layers x 8 KV heads folded (336 KV / 672 query heads, head_dim 256, bf16)."""
    _bench_shape_sampled("gemma9b_sweep", 42, 64, 4096,
                         rows=[(0, 0), (63, 671), (17, 300), (40, 5), (33, 450)], distinct_rows=2)


@pytest.mark.parametrize("name,batch,ctx,heads", [("llama8b", 3, 700, 2), ("gemma9b_sweep", 2, 300, 2),
                                                  ("qwen14b", 2, 1100, 1), ("tiny", 2, 100, 2)])
def test_decode_step_appends_then_attends(name, batch, ctx, heads):
    """sq_decode_step: each row's new token compressed at its own position and
    attended together with the prefix before it. The new records equal the
    oracle's, the outputs and scores equal the oracle's attention over the
    resulting cache, and they equal the separate calls (sq_compress_kv of one
    token, then sq_attn_decode) on a second cache. Covers the two-launch
    tcgen05 step (head_dim 128 and 256) and the separate-launch path (head_dim 32)."""
    from gpu_helpers import compare_compressed
    w = make_workload(name, batch=batch, tokens=ctx)
    cfg = w.cfg
    g = cfg["n_q"] // cfg["n_kv"]
    nkv = min(heads, cfg["n_kv"])
    nq, d = nkv * g, cfg["d"]
    ck = calibrate_oracle(w.k_cal[:nkv], cfg["bits_k"], True)
    cv = calibrate_oracle(w.v_cal[:nkv], cfg["bits_v"], False)
    rk, rv = records_to_device(ck), records_to_device(cv)
    cap = ctx + 32
    caches = []
    for _ in range(2):
        kc = sq.alloc_cache(batch, nkv, cap, ck[0].words, True)
        vc = sq.alloc_cache(batch, nkv, cap, cv[0].words, False)
        sq.sq_compress_kv(rk, rv, w.k[:, :nkv, :ctx - 1].contiguous().cuda(), w.v[:, :nkv, :ctx - 1].contiguous().cuda(),
                          batch, nkv, d, ctx - 1, None, kc, vc)
        caches.append((kc, vc))
    pos_l = [ctx - 1 - (37 * b) % 61 for b in range(batch)]
    pos = torch.tensor(pos_l, dtype=torch.int32, device="cuda")
    k_new = w.k[:, :nkv, ctx - 1:].contiguous().cuda()
    v_new = w.v[:, :nkv, ctx - 1:].contiguous().cuda()
    q = w.q[:, :nq].contiguous().cuda()
    max_ctx = ctx
    ws = torch.empty(sq.sq_attn_workspace(batch, nq, nkv, d, max_ctx), dtype=torch.uint8, device="cuda")
    outs, scs = [], []
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    (kc, vc), (kc2, vc2) = caches
    out = torch.empty(batch, nq, d, device="cuda")
    sc = torch.full((batch, nq, max_ctx), float("nan"), device="cuda")
    sq.sq_decode_step(rk, rv, kc, vc, k_new, v_new, q, pos, batch, nq, nkv, d, max_ctx, 0.0, out, sc, ws, flags)
    out2 = torch.empty_like(out)
    sc2 = torch.full_like(sc, float("nan"))
    sq.sq_compress_kv(rk, rv, k_new, v_new, batch, nkv, d, 1, pos, kc2, vc2, flags)
    sq.sq_attn_decode(rk, rv, kc2, vc2, pos + 1, batch, nq, nkv, d, max_ctx, q, 0.0, out2, sc2, ws, flags)
    torch.cuda.synchronize()
    assert flags.item() == 0
    assert np.array_equal(kc.words_u32(), kc2.words_u32()) and np.array_equal(vc.words_u32(), vc2.words_u32())
    kw, vw = kc.words_u32(), vc.words_u32()
    for b, p in enumerate(pos_l):
        for h in range(nkv):
            compare_compressed(kw[b, h, p:p + 1], kc.norm[b, h, p:p + 1].cpu().numpy(),
                               kc.rnorm[b, h, p:p + 1].cpu().numpy(), k_new[b, h].double().cpu().numpy(), ck[h])
            compare_compressed(vw[b, h, p:p + 1], vc.norm[b, h, p:p + 1].cpu().numpy(), None,
                               v_new[b, h].double().cpu().numpy(), cv[h])
    lens = [p + 1 for p in pos_l]
    ref_out, ref_sc = oattn.attn_decode(q.double().cpu().numpy(), kw, kc.norm.cpu().numpy(), kc.rnorm.cpu().numpy(),
                                        vw, vc.norm.cpu().numpy(), ck, cv, lens, 1.0 / math.sqrt(d))
    o, s = out.cpu().numpy(), sc.cpu().numpy()
    _assert_close(o, s, ref_out, ref_sc, lens)
    np.testing.assert_allclose(o, out2.cpu().numpy(), rtol=1e-5, atol=1e-6)


@pytest.mark.parametrize("name,batch,prefix,chunk,heads", [
    ("llama8b", 2, 300, 37, 1),          # G = 4: blocks of 4 positions, a partial last block
    ("qwen14b", 1, 129, 31, 1),          # G = 5: blocks of 3 positions (15 columns)
    ("gemma9b_sweep", 2, 100, 19, 1),    # G = 2, head_dim 256: blocks of 8 positions
    ("qwen1_5b_long", 1, 600, 40, 1),    # G = 6: blocks of 2 positions, several splits
    ("tiny", 2, 60, 21, 2),              # head_dim 32: the SIMT partials
])
def test_prefill_attention_matches_the_oracle(name, batch, prefix, chunk, heads):
    """sq_attn_prefill: each query token of a chunk at position start[b] + t
    attends causally to the packed cache 0 .. start[b] + t (ragged starts per
    row); every (row, head, token) output against the oracle."""
    w = make_workload(name, batch=batch, tokens=prefix + chunk)
    cfg = w.cfg
    g = cfg["n_q"] // cfg["n_kv"]
    nkv = min(heads, cfg["n_kv"])
    nq, d = nkv * g, cfg["d"]
    ck = calibrate_oracle(w.k_cal[:nkv], cfg["bits_k"], True)
    cv = calibrate_oracle(w.v_cal[:nkv], cfg["bits_v"], False)
    rk, rv = records_to_device(ck), records_to_device(cv)
    T = prefix + chunk
    kc = sq.alloc_cache(batch, nkv, T, ck[0].words, True)
    vc = sq.alloc_cache(batch, nkv, T, cv[0].words, False)
    sq.sq_compress_kv(rk, rv, w.k[:, :nkv].contiguous().cuda(), w.v[:, :nkv].contiguous().cuda(), batch, nkv, d, T,
                      None, kc, vc)
    gen = torch.Generator().manual_seed(5)
    qs = w.q[:, :nq, None, :].float() * (1.0 + 0.3 * torch.randn(batch, nq, chunk, 1, generator=gen))
    qs = qs.to(w.q.dtype).contiguous().cuda()
    starts_l = [prefix - 13 * b for b in range(batch)]
    starts = torch.tensor(starts_l, dtype=torch.int32, device="cuda")
    ws = torch.empty(sq.sq_attn_prefill_workspace(batch, nq, nkv, d, chunk, T), dtype=torch.uint8, device="cuda")
    out = torch.full((batch, nq, chunk, d), float("nan"), device="cuda")
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    sq.sq_attn_prefill(rk, rv, kc, vc, starts, batch, nq, nkv, d, chunk, T, qs, 0.0, out, ws, flags)
    torch.cuda.synchronize()
    assert flags.item() == 0
    ref = oattn.attn_prefill(qs.double().cpu().numpy(), kc.words_u32(), kc.norm.cpu().numpy(),
                             kc.rnorm.cpu().numpy(), vc.words_u32(), vc.norm.cpu().numpy(), ck, cv, starts_l,
                             1.0 / math.sqrt(d))
    got = out.cpu().numpy()
    err = rel_l2_rows(got.reshape(-1, d), ref.reshape(-1, d))
    assert np.max(err) <= TOL_OUT, np.max(err)
