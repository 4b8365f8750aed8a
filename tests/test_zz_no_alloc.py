"""The no-allocation decode-attention entry point (collected last on purpose).

Callers that cannot allocate device memory where they run decode attention
(a serving loop whose device memory is reserved once at start-up, plug-ins
without the host application's allocator) call sq_attn_decode_noalloc,
whose scratch is a fixed array inside libsq. This checks, through the C ABI,
that two calls in a row give the same outputs and scores as sq_attn_decode
with a caller workspace, within the attention tolerances, and that shapes
needing more scratch than the array are refused before any launch.
"""

import numpy as np
import pytest
import torch

from gpu_helpers import TOL_OUT, TOL_SCORES, calibrate_oracle, records_to_device, rel_l2_rows
from synthetic import make_workload

pytestmark = pytest.mark.gpu

if not torch.cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

from compressed_attention_head_b200 import sq  # noqa: E402


def _setup(name="llama8b", batch=2, ctx=700, heads=2):
    w = make_workload(name, batch=batch, tokens=ctx)
    cfg = w.cfg
    group = cfg["n_q"] // cfg["n_kv"]
    nq, d = heads * group, cfg["d"]
    ck = calibrate_oracle(w.k_cal[:heads], cfg["bits_k"], True)
    cv = calibrate_oracle(w.v_cal[:heads], cfg["bits_v"], False)
    rk, rv = records_to_device(ck), records_to_device(cv)
    kc = sq.alloc_cache(batch, heads, ctx, ck[0].words, True)
    vc = sq.alloc_cache(batch, heads, ctx, cv[0].words, False)
    sq.sq_compress_kv(rk, rv, w.k[:, :heads].contiguous().cuda(), w.v[:, :heads].contiguous().cuda(), batch, heads,
                      d, ctx, None, kc, vc)
    q = w.q[:, :nq].contiguous().cuda()
    lens = torch.tensor([ctx, ctx - 123][:batch], dtype=torch.int32, device="cuda")
    return rk, rv, kc, vc, lens, batch, nq, heads, d, ctx, q


def test_noalloc_matches_workspace_call_twice():
    rk, rv, kc, vc, lens, batch, nq, nkv, d, ctx, q = _setup()
    ws = torch.empty(sq.sq_attn_workspace(batch, nq, nkv, d, ctx), dtype=torch.uint8, device="cuda")
    ref_out = torch.empty(batch, nq, d, device="cuda")
    ref_sc = torch.zeros(batch, nq, ctx, device="cuda")
    sq.sq_attn_decode(rk, rv, kc, vc, lens, batch, nq, nkv, d, ctx, q, 0.0, ref_out, ref_sc, ws)
    torch.cuda.synchronize()
    for _ in range(2):
        out = torch.full((batch, nq, d), float("nan"), device="cuda")
        sc = torch.zeros(batch, nq, ctx, device="cuda")
        flags = torch.zeros(1, dtype=torch.int32, device="cuda")
        sq.sq_attn_decode_noalloc(rk, rv, kc, vc, lens, batch, nq, nkv, d, ctx, q, 0.0, out, sc, flags)
        torch.cuda.synchronize()
        assert flags.item() == 0
        o, r = out.cpu().numpy(), ref_out.cpu().numpy()
        assert np.max(rel_l2_rows(o.reshape(-1, d), r.reshape(-1, d))) <= TOL_OUT
        s, rs = sc.cpu().numpy(), ref_sc.cpu().numpy()
        for b in range(batch):
            n = int(lens[b])
            assert np.max(rel_l2_rows(s[b, :, :n], rs[b, :, :n])) <= TOL_SCORES


def test_noalloc_refuses_shapes_beyond_its_array():
    rk, rv, kc, vc, lens, batch, nq, nkv, d, ctx, q = _setup(batch=1, ctx=64, heads=1)
    big_batch, big_q, big_kv, big_ctx = 64, 4096, 256, 4096
    need = sq.sq_attn_workspace(big_batch, big_q, big_kv, d, big_ctx)
    assert need > sq.SQ_ATTN_NOALLOC_MAX_BYTES
    out = torch.empty(1, nq, d, device="cuda")
    # a cache description with the oversized shape: refused on the host, nothing launched
    bad_k = sq.PackedCache(kc.codes, kc.norm, kc.rnorm, big_batch, big_kv, kc.cap, kc.words)
    bad_v = sq.PackedCache(vc.codes, vc.norm, vc.rnorm, big_batch, big_kv, vc.cap, vc.words)
    with pytest.raises(sq.SqError) as e:
        sq.sq_attn_decode_noalloc(rk, rv, bad_k, bad_v, lens, big_batch, big_q, big_kv, d, big_ctx, q, 0.0, out)
    assert e.value.status == sq.SQ_ERR_WORKSPACE
