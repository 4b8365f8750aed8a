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
from synthetic import make_workload

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

from compressed_attention_head_b200 import sq  # noqa: E402


def _run(name, batch, ctx, seq_lens, heads=None, bits_k=None, bits_v=None, qjl=True, out_dtype=torch.float32,
         cap=None):
    w = make_workload(name, batch=batch, tokens=ctx)
    cfg = w.cfg
    nkv = heads or cfg["n_kv"]
    group = cfg["n_q"] // cfg["n_kv"]
    nq = nkv * group
    d = cfg["d"]
    ck = calibrate_oracle(w.k_cal[:nkv], cfg["bits_k"] if bits_k is None else bits_k, True, qjl=qjl)
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


@pytest.mark.parametrize("name,ctx,heads", [("llama8b", 700, 2), ("gemma9b_sweep", 300, 2)])
def test_tensor_core_partials_match_simt_partials(name, ctx, heads):
    """Both attention paths against the oracle on the same packed cache."""
    try:
        sq.sq_set_option(sq.SQ_OPT_ATTN_PATH, 1)
        o1, s1, r_o, r_s, _ = _run(name, 1, ctx, [ctx], heads=heads)
        sq.sq_set_option(sq.SQ_OPT_ATTN_PATH, 0)
        o0, s0, _, _, _ = _run(name, 1, ctx, [ctx], heads=heads)
    finally:
        sq.sq_set_option(sq.SQ_OPT_ATTN_PATH, 0)
    _assert_close(o1, s1, r_o, r_s, [ctx])
    _assert_close(o0, s0, r_o, r_s, [ctx])


def test_full_size_decode_sampled_rows():
    """Qwen2.5-14B-shaped decode step (batch 4 at context 8192, one layer's 8 KV /
    40 query heads, the launch shape of one layer): every output and score row
    of two KV heads against the oracle."""
    out, scores, ref_out, ref_scores, flags = _run("qwen14b", 4, 8192, [8192, 8191, 4097, 8192], heads=2)
    assert flags == 0
    _assert_close(out, scores, ref_out, ref_scores, [8192, 8191, 4097, 8192])
