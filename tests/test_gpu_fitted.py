"""Fitted per-regime codebooks on the GPU, through the C ABI, against the oracle.

SpectralQuant README, "Repository Structure": nonuniform_quantization.py,
"Lloyd-Max with per-regime codebooks". The fit (sq_calibrate with
codebooks = 1) is compared with the oracle's fit on the same basis; compress,
append, decompress and decode attention with fitted records are compared
with the oracle element by element (oracle records imported, so the two sides
code with identical tables).
"""

import math

import numpy as np
import pytest
import torch

from gpu_helpers import (TOL_OUT, TOL_RECON, TOL_SCORES, compare_compressed, read_records, records_to_device,
                         rel_l2_rows)
from oracle import attention as oattn
from oracle import calibration as ocal
from oracle import codec as ocodec
from oracle import fitted as ofit
from oracle import record as orec
from synthetic import make_workload

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

from compressed_attention_head_b200 import sq  # noqa: E402


def _oracle_fitted(x_cal, bits, is_key, iters=ofit.FIT_ITERS):
    return [ocal.calibrate(x_cal[h].double().cpu().numpy(), avg_bits=bits, is_key=is_key, seed=42, stream=h,
                           codebooks="fitted", fit_iters=iters) for h in range(x_cal.shape[0])]


@pytest.mark.parametrize("name,is_key,iters", [("llama8b", True, 30), ("llama8b", False, 30),
                                               ("qwen1_5b_long", True, 12), ("gemma9b_sweep", False, 30)])
def test_gpu_fit_matches_the_oracle_fit_on_the_same_basis(name, is_key, iters):
    w = make_workload(name, batch=1, tokens=1)
    cfg = w.cfg
    heads, d = 2, cfg["d"]
    x = (w.k_cal if is_key else w.v_cal)[:heads].contiguous().cuda()
    n = x.shape[1]
    bits = cfg["bits_k"] if is_key else cfg["bits_v"]
    p = sq.calib_params(d, heads, bits, is_key, codebooks=1, fit_iters=iters)
    recs = sq.alloc_records(heads, d, "cuda")
    ws = torch.empty(sq.sq_calibrate_workspace(p, n), dtype=torch.uint8, device="cuda")
    status = torch.zeros(heads, dtype=torch.int32, device="cuda")
    sq.sq_calibrate(p, x, n, n * d, d, recs, ws, status)
    torch.cuda.synchronize()
    assert status.cpu().tolist() == [0] * heads
    got = read_records(recs, heads, d)
    g_lv, g_th = ofit.gaussian_tables()
    for h, cg in enumerate(got):
        assert cg.fitted
        # the oracle's fit on the GPU's basis, widths and d_eff
        base = orec.read(orec.write(cg))
        base.flags &= ~ocal.FLAG_FITTED
        ref = ocal.fit_codebooks(base, x[h].double().cpu().numpy(), iters)
        for r in (0, 1):
            used = {int(cg.bits[i]) for i in range(d) if cg.bits[i] > 0 and (0 if i < cg.d_eff else 1) == r}
            for b in range(1, 9):
                lv_g, th_g = ofit.codebook_of(cg.fit_lv, cg.fit_th, r, b)
                lv_o, th_o = ofit.codebook_of(ref.fit_lv, ref.fit_th, r, b)
                if b in used:
                    np.testing.assert_allclose(lv_g, lv_o, rtol=0, atol=1e-9 * max(1.0, np.max(np.abs(lv_o))))
                    np.testing.assert_allclose(th_g, th_o, rtol=0, atol=1e-9 * max(1.0, np.max(np.abs(lv_o))))
                    assert np.all(np.diff(lv_g) > 0)
                else:   # never used to code: the Gaussian tables (the library's own solver)
                    np.testing.assert_allclose(lv_g, g_lv[ofit.level_offset(b):ofit.level_offset(b) + (1 << b)],
                                               rtol=0, atol=1e-9)


def test_gpu_fit_records_import_and_code_like_the_oracle():
    # the GPU-calibrated record, read back into the oracle, codes the evaluation
    # vectors exactly as the GPU does (compress through the reference kernels)
    w = make_workload("llama8b", batch=1, tokens=300)
    d = w.cfg["d"]
    x_cal = w.k_cal[:2].contiguous().cuda()
    n = x_cal.shape[1]
    p = sq.calib_params(d, 2, 3.0, True, codebooks=1)
    recs = sq.alloc_records(2, d, "cuda")
    ws = torch.empty(sq.sq_calibrate_workspace(p, n), dtype=torch.uint8, device="cuda")
    sq.sq_calibrate(p, x_cal, n, n * d, d, recs, ws, None)
    cals = read_records(recs, 2, d)
    k = w.k[:, :2].contiguous().cuda()
    cache = sq.alloc_cache(1, 2, 320, cals[0].words, True)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    sq.sq_compress_kv(recs, None, k, None, 1, 2, d, 300, None, cache, None, flags)
    torch.cuda.synchronize()
    assert flags.item() == 0
    words = cache.words_u32()
    for h in range(2):
        compare_compressed(words[0, h, :300], cache.norm[0, h, :300].cpu().numpy(),
                           cache.rnorm[0, h, :300].cpu().numpy(), k[0, h].double().cpu().numpy(), cals[h])


@pytest.mark.parametrize("name,dtype,is_key,n_tok", [
    ("llama8b", torch.float16, True, 700),     # fp16 head_dim 128: the tensor-core pass leaves fitted heads to the reference pass
    ("llama8b", torch.float32, False, 333),
    ("gemma9b_sweep", torch.bfloat16, True, 130),
    ("llama8b", torch.float16, True, 3),        # append kernel (fewer than 16 tokens)
])
def test_compress_and_decompress_with_fitted_records(name, dtype, is_key, n_tok):
    w = make_workload(name, batch=2, tokens=max(n_tok, 1))
    cfg = w.cfg
    d, heads = cfg["d"], 2
    cals = _oracle_fitted(w.k_cal[:heads] if is_key else w.v_cal[:heads], cfg["bits_k"] if is_key else cfg["bits_v"],
                          is_key)
    recs = records_to_device(cals)
    x = (w.k if is_key else w.v)[:, :heads, :n_tok].to(dtype).contiguous().cuda()
    cap = ((n_tok + 31) // 32) * 32
    cache = sq.alloc_cache(2, heads, cap, cals[0].words, is_key and cals[0].m > 0)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    if is_key:
        sq.sq_compress_kv(recs, None, x, None, 2, heads, d, n_tok, None, cache, None, flags)
    else:
        sq.sq_compress_kv(None, recs, None, x, 2, heads, d, n_tok, None, None, cache, flags)
    torch.cuda.synchronize()
    assert flags.item() == 0
    words = cache.words_u32()
    if n_tok >= 100:
        # the case tells fitted from Gaussian tables: the oracle's codes differ
        gauss = orec.read(orec.write(cals[0]))
        gauss.flags &= ~ocal.FLAG_FITTED
        xs = x[0, 0].double().cpu().numpy()
        differ = np.mean(ocodec.compress(xs, cals[0])["codes"] != ocodec.compress(xs, gauss)["codes"])
        assert differ > 1e-3, differ
    for b in range(2):
        for h in range(heads):
            rn = cache.rnorm[b, h, :n_tok].cpu().numpy() if cache.rnorm is not None else None
            compare_compressed(words[b, h, :n_tok], cache.norm[b, h, :n_tok].cpu().numpy(), rn,
                               x[b, h].double().cpu().numpy(), cals[h])
    out = torch.empty(2, heads, n_tok, d, dtype=torch.float32, device="cuda")
    sq.sq_decompress_kv(recs, cache, d, 0, n_tok, is_key, out)
    torch.cuda.synchronize()
    for b in range(2):
        for h in range(heads):
            rn = cache.rnorm[b, h, :n_tok].cpu().numpy() if cache.rnorm is not None else None
            ref = ocodec.decompress(words[b, h, :n_tok], cache.norm[b, h, :n_tok].cpu().numpy(), rn, cals[h],
                                    apply_qjl=is_key)
            assert np.max(rel_l2_rows(out[b, h].cpu().numpy(), ref)) <= TOL_RECON


def _attention_case(name="qwen14b", batch=2, ctx=600, lens=(600, 257), heads=2):
    w = make_workload(name, batch=batch, tokens=ctx)
    cfg = w.cfg
    g = cfg["n_q"] // cfg["n_kv"]
    d, nq = cfg["d"], heads * g
    ck = _oracle_fitted(w.k_cal[:heads], cfg["bits_k"], True)
    cv = _oracle_fitted(w.v_cal[:heads], cfg["bits_v"], False)
    rk, rv = records_to_device(ck), records_to_device(cv)
    cap = ((ctx + 31) // 32) * 32
    kc = sq.alloc_cache(batch, heads, cap, ck[0].words, ck[0].m > 0)
    vc = sq.alloc_cache(batch, heads, cap, cv[0].words, False)
    sq.sq_compress_kv(rk, rv, w.k[:, :heads].contiguous().cuda(), w.v[:, :heads].contiguous().cuda(), batch, heads,
                      d, ctx, None, kc, vc)
    q = w.q[:, :nq].contiguous().cuda()
    seq = torch.tensor(list(lens), dtype=torch.int32, device="cuda")
    return ck, cv, rk, rv, kc, vc, q, seq, batch, nq, heads, d, ctx


def test_decode_attention_with_fitted_records_on_the_simt_path():
    ck, cv, rk, rv, kc, vc, q, seq, batch, nq, heads, d, ctx = _attention_case()
    ws = torch.empty(sq.sq_attn_workspace(batch, nq, heads, d, ctx), dtype=torch.uint8, device="cuda")
    out = torch.empty(batch, nq, d, device="cuda")
    scores = torch.full((batch, nq, ctx), float("nan"), device="cuda")
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    sq.sq_set_option(sq.SQ_OPT_ATTN_PATH, 1)
    try:
        sq.sq_attn_decode(rk, rv, kc, vc, seq, batch, nq, heads, d, ctx, q, 0.0, out, scores, ws, flags)
        torch.cuda.synchronize()
    finally:
        sq.sq_set_option(sq.SQ_OPT_ATTN_PATH, 0)
    assert flags.item() == 0
    lens = seq.cpu().tolist()
    ref_out, ref_sc = oattn.attn_decode(q.double().cpu().numpy(), kc.words_u32(), kc.norm.cpu().numpy(),
                                        kc.rnorm.cpu().numpy(), vc.words_u32(), vc.norm.cpu().numpy(), ck, cv, lens,
                                        1.0 / math.sqrt(d))
    s, o = scores.cpu().numpy(), out.cpu().numpy()
    for b, n in enumerate(lens):
        assert np.max(rel_l2_rows(s[b, :, :n], ref_sc[b, :, :n])) <= TOL_SCORES
        assert np.max(rel_l2_rows(o[b], ref_out[b])) <= TOL_OUT


def test_tensor_core_attention_refuses_fitted_records():
    ck, cv, rk, rv, kc, vc, q, seq, batch, nq, heads, d, ctx = _attention_case(ctx=300, lens=(300, 40))
    ws = torch.empty(sq.sq_attn_workspace(batch, nq, heads, d, ctx), dtype=torch.uint8, device="cuda")
    out = torch.empty(batch, nq, d, device="cuda")
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    sq.sq_attn_decode(rk, rv, kc, vc, seq, batch, nq, heads, d, ctx, q, 0.0, out, None, ws, flags)
    torch.cuda.synchronize()
    assert flags.item() & sq.SQ_FLAG_RECORD


def test_import_rejects_fitted_tables_out_of_order():
    w = make_workload("llama8b", batch=1, tokens=1)
    cal = _oracle_fitted(w.v_cal[:1], 3.0, False, iters=3)[0]
    b = int(cal.bits[-1])
    o = ofit.level_offset(b)
    cal.fit_lv[1, o], cal.fit_lv[1, o + 1] = cal.fit_lv[1, o + 1], cal.fit_lv[1, o]
    size = sq.sq_calib_bytes(cal.d)
    host = np.zeros(size, dtype=np.uint8)
    raw = np.frombuffer(orec.write(cal), dtype=np.uint8)
    host[:raw.size] = raw
    dev = torch.from_numpy(host).cuda()
    status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    sq.sq_calib_import(dev, 1, cal.d, status)
    torch.cuda.synchronize()
    assert status.item() == sq.SQ_ERR_RECORD
