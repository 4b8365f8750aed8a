"""GPU parity of compress / decompress / append against the oracle.

The oracle's calibration records are imported into the library (the
eigenvectors of a degenerate noise subspace are not unique, so compression
parity is checked on one shared calibration; the GPU calibration itself is
checked separately by invariants). Inputs come from the seeded synthetic
generators; nothing the oracle reads comes from the CUDA path except the
packed cache that decompress and attention parity feed it on purpose.
"""

import numpy as np
import pytest
import torch

from gpu_helpers import (TOL_RECON, calibrate_oracle, compare_compressed, exempt_mask, records_to_device,
                         rel_l2_rows)
from oracle import codec as ocodec
from synthetic import CONFIGS, make_workload

pytestmark = pytest.mark.gpu

cuda = pytest.importorskip("torch").cuda
if not cuda.is_available():
    pytest.skip("needs a CUDA GPU", allow_module_level=True)

from compressed_attention_head_b200 import sq  # noqa: E402


def _case(name, batch=2, tokens=333, heads=None, bits_k=None, bits_v=None, qjl=True, normalize=True):
    w = make_workload(name, batch=batch, tokens=tokens)
    cfg = w.cfg
    nh = min(heads, cfg["n_kv"]) if heads else cfg["n_kv"]
    bk = cfg["bits_k"] if bits_k is None else bits_k
    bv = cfg["bits_v"] if bits_v is None else bits_v
    ck = calibrate_oracle(w.k_cal[:nh], bk, True, qjl=qjl, normalize=normalize)
    cv = calibrate_oracle(w.v_cal[:nh], bv, False, normalize=normalize)
    k = w.k[:, :nh].contiguous()
    v = w.v[:, :nh].contiguous()
    return w, ck, cv, k, v, nh


def _compress(ck, cv, k, v, cap=None, start=None, flags=None):
    batch, nh, t, d = k.shape
    rk = records_to_device(ck)
    rv = records_to_device(cv)
    cap = cap or t
    kc = sq.alloc_cache(batch, nh, cap, ck[0].words, ck[0].m > 0)
    vc = sq.alloc_cache(batch, nh, cap, cv[0].words, False)
    sp = None if start is None else torch.tensor(start, dtype=torch.int32, device="cuda")
    sq.sq_compress_kv(rk, rv, k.cuda(), v.cuda(), batch, nh, d, t, sp, kc, vc, flags)
    torch.cuda.synchronize()
    return rk, rv, kc, vc


def _check_side(cache, cals, x, t0=0):
    words = cache.words_u32()
    norm = cache.norm.cpu().numpy()
    rn = cache.rnorm.cpu().numpy() if cache.rnorm is not None else None
    n_ex = 0
    t = x.shape[2]
    for b in range(x.shape[0]):
        for h in range(x.shape[1]):
            xs = x[b, h].double().cpu().numpy()
            e1, e2 = compare_compressed(words[b, h, t0:t0 + t], norm[b, h, t0:t0 + t],
                                        rn[b, h, t0:t0 + t] if rn is not None else None, xs, cals[h])
            n_ex += e1 + e2
    return n_ex


@pytest.mark.parametrize("name", ["tiny", "llama8b", "qwen14b", "qwen1_5b_long", "gemma9b_sweep"])
def test_compress_parity_configs(name):
    heads = None if name in ("tiny", "llama8b") else 4
    w, ck, cv, k, v, nh = _case(name, heads=heads, tokens=333 if name != "tiny" else 256,
                                batch=2 if name != "tiny" else 1)
    _, _, kc, vc = _compress(ck, cv, k, v)
    ex = _check_side(kc, ck, k) + _check_side(vc, cv, v)
    total = k.numel() + v.numel()
    assert ex < 1e-3 * total


@pytest.mark.parametrize("bits", [2.0, 2.5, 3.0, 3.5, 4.0])
@pytest.mark.parametrize("qjl", [True, False])
def test_gemma_bit_sweep_parity(bits, qjl):
    w, ck, cv, k, v, nh = _case("gemma9b_sweep", batch=1, tokens=130, heads=2, bits_k=bits, bits_v=bits, qjl=qjl)
    _, _, kc, vc = _compress(ck, cv, k, v)
    _check_side(kc, ck, k)
    _check_side(vc, cv, v)
    assert (kc.rnorm is not None) == qjl


def test_unnormalized_mode_parity():
    w, ck, cv, k, v, nh = _case("llama8b", batch=1, tokens=100, heads=2, normalize=False)
    _, _, kc, vc = _compress(ck, cv, k, v)
    _check_side(kc, ck, k)
    _check_side(vc, cv, v)
    assert torch.all(kc.norm[:, :, :100] == 1.0)


@pytest.mark.parametrize("name", ["tiny", "qwen14b", "gemma9b_sweep"])
def test_decompress_parity(name):
    w, ck, cv, k, v, nh = _case(name, batch=1, tokens=150, heads=2)
    rk, rv, kc, vc = _compress(ck, cv, k, v)
    d = k.shape[-1]
    for cache, cals, recs, qjl in ((kc, ck, rk, True), (kc, ck, rk, False), (vc, cv, rv, False)):
        out = torch.empty(1, nh, 150, d, device="cuda")
        sq.sq_decompress_kv(recs, cache, d, 0, 150, qjl, out)
        torch.cuda.synchronize()
        words = cache.words_u32()
        for h in range(nh):
            ref = ocodec.decompress(words[0, h, :150], cache.norm[0, h, :150].cpu().numpy(),
                                    cache.rnorm[0, h, :150].cpu().numpy() if cache.rnorm is not None else None,
                                    cals[h], apply_qjl=qjl)
            err = rel_l2_rows(out[0, h].cpu().numpy(), ref)
            assert np.max(err) <= TOL_RECON, (name, h, np.max(err))


def test_append_decode_tokens_at_start_pos():
    """One new token per row written at each row's own position (ragged lengths)."""
    w, ck, cv, k, v, nh = _case("qwen14b", batch=3, tokens=1, heads=2)
    start = [5, 0, 47]
    _, _, kc, vc = _compress(ck, cv, k, v, cap=64, start=start)
    words = kc.words_u32()
    for b, s in enumerate(start):
        for h in range(nh):
            compare_compressed(words[b, h, s:s + 1], kc.norm[b, h, s:s + 1].cpu().numpy(),
                               kc.rnorm[b, h, s:s + 1].cpu().numpy(), k[b, h].double().numpy(), ck[h])
            # untouched slots stay zero
            others = np.delete(np.arange(64), s)
            assert np.all(words[b, h, others] == 0)


def test_zero_tokens_is_noop_and_capacity_flag():
    w, ck, cv, k, v, nh = _case("tiny", batch=1, tokens=32, heads=2)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    rk, rv, kc, vc = _compress(ck, cv, k[:, :, :0], v[:, :, :0], cap=32, flags=flags)
    assert flags.item() == 0 and torch.all(kc.codes == 0)
    # 32 tokens at start 16 into a 32-slot cache overflow: flagged, nothing written
    _, _, kc2, _ = _compress(ck, cv, k, v, cap=32, start=[16], flags=flags)
    assert flags.item() & sq.SQ_FLAG_CAPACITY
    assert torch.all(kc2.codes == 0)


def test_record_mismatch_flag():
    w, ck, cv, k, v, nh = _case("tiny", batch=1, tokens=16, heads=1)
    rk = records_to_device(ck)
    kc = sq.alloc_cache(1, 1, 16, ck[0].words + 1, True)       # wrong word count
    vc = sq.alloc_cache(1, 1, 16, cv[0].words, False)
    rv = records_to_device(cv)
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    sq.sq_compress_kv(rk, rv, k.cuda(), v.cuda(), 1, 1, 32, 16, None, kc, vc, flags)
    torch.cuda.synchronize()
    assert flags.item() & sq.SQ_FLAG_RECORD
    assert torch.all(kc.codes == 0)


def test_argument_errors():
    w, ck, cv, k, v, nh = _case("tiny", batch=1, tokens=16, heads=1)
    rk = records_to_device(ck)
    kc = sq.alloc_cache(1, 1, 16, ck[0].words, True)
    with pytest.raises(sq.SqError) as e:
        sq.sq_compress_kv(rk, None, k.cuda(), None, 1, 1, 48, 16, None, kc, None)
    assert e.value.status == sq.SQ_ERR_UNSUPPORTED
    with pytest.raises(sq.SqError) as e:
        sq.sq_compress_kv(rk, None, k.cuda(), None, 2, 1, 32, 16, None, kc, None)   # batch mismatch
    assert e.value.status == sq.SQ_ERR_ARG


@pytest.mark.parametrize("name,tokens", [("llama8b", 1000), ("qwen14b", 777), ("qwen1_5b_long", 129)])
def test_tensor_core_path_matches_oracle_and_reference_kernel(name, tokens):
    """The fp16 head_dim-128 tensor-core compress against the oracle and against
    the float64 reference kernel. Both decide every code exactly up to float64
    rounding (~1e-13 relative), so their records are identical bit for bit
    outside the fields the oracle marks exempt (a z within 1e-5 of a threshold,
    a QJL projection within the band of 0), where the two float64 evaluations,
    summed in different orders, may round to different sides."""
    w, ck, cv, k, v, nh = _case(name, batch=2, tokens=tokens, heads=4)
    try:
        sq.sq_set_option(sq.SQ_OPT_COMPRESS_PATH, 0)
        _, _, kc, vc = _compress(ck, cv, k, v)
        sq.sq_set_option(sq.SQ_OPT_COMPRESS_PATH, 1)
        _, _, kr, vr = _compress(ck, cv, k, v)
    finally:
        sq.sq_set_option(sq.SQ_OPT_COMPRESS_PATH, 0)
    _check_side(kc, ck, k)
    _check_side(vc, cv, v)
    for a, b, cals, x in ((kc, kr, ck, k), (vc, vr, cv, v)):
        wa, wb = a.words_u32(), b.words_u32()
        for bi in range(x.shape[0]):
            for h in range(nh):
                out = ocodec.compress(x[bi, h].double().numpy(), cals[h])
                mask = exempt_mask(out, cals[h])
                diff = (wa[bi, h, :tokens] ^ wb[bi, h, :tokens]) & ~mask
                assert not diff.any(), (bi, h, np.argwhere(diff != 0)[:4].tolist())
        # value norms are summed in float32 on the tensor-core path: equal up to
        # the stated norm tolerance (keys are summed in float64 on both)
        assert torch.allclose(a.norm, b.norm, rtol=1e-6, atol=0)
    assert torch.allclose(kc.rnorm, kr.rnorm, rtol=1e-6, atol=0)


@pytest.mark.parametrize("cfg,tokens,batch,dtype", [
    ("gemma9b_sweep", 77, 2, None),                          # bf16, head_dim 256: a ragged last block of 32
    ("gemma9b_sweep", 4096, 1, None),                        # the decode-cache prompt of one row
    ("qwen14b", 40, 2, None),                                # fp16 head_dim 128 under one 64-token tile
    ("llama8b", 150, 2, torch.float32),                      # f32 head_dim 128
    (dict(CONFIGS["llama8b"], d=64), 300, 2, None),          # fp16 head_dim 64: a ragged last block of 128
    (dict(CONFIGS["llama8b"], d=64, dtype="bf16"), 16, 1, None),   # the shortest prompt it takes
])
def test_block_kernel_matches_reference_kernel(cfg, tokens, batch, dtype):
    """The block-tiled float64 compress (every prompt of >= 16 tokens that the
    tensor-core kernel does not take) sums each rotated coordinate in the same
    order as the one-warp-per-vector reference kernel, and ||x|| with the same
    lane-strided sum: records, norms and QJL norms identical bit for bit, and
    parity with the oracle."""
    w, ck, cv, k, v, nh = _case(cfg, batch=batch, tokens=tokens, heads=2)
    if dtype is not None:
        k, v = k.to(dtype), v.to(dtype)
    try:
        sq.sq_set_option(sq.SQ_OPT_COMPRESS_PATH, 0)
        _, _, kc, vc = _compress(ck, cv, k, v)
        sq.sq_set_option(sq.SQ_OPT_COMPRESS_PATH, 1)
        _, _, kr, vr = _compress(ck, cv, k, v)
    finally:
        sq.sq_set_option(sq.SQ_OPT_COMPRESS_PATH, 0)
    for a, b in ((kc, kr), (vc, vr)):
        assert torch.equal(a.codes, b.codes)
        assert torch.equal(a.norm, b.norm)
    assert torch.equal(kc.rnorm, kr.rnorm)
    ex = _check_side(kc, ck, k) + _check_side(vc, cv, v)
    assert ex < 1e-3 * (k.numel() + v.numel())


def test_full_size_prefill_in_bench_launch_configuration():
    """Llama-shaped prompt: all 32 layers x 8 KV heads (2048 tokens) compressed in one
    call, as the benchmark times it; sampled (head, token) records against the oracle."""
    cfg = CONFIGS["llama8b"]
    L, nkv, d, T = cfg["layers"], cfg["n_kv"], cfg["d"], cfg["ctx"]
    ks, vs, cks, cvs = [], [], [], []
    for layer in range(L):
        w = make_workload("llama8b", layer, batch=1, tokens=T)
        ks.append(w.k)
        vs.append(w.v)
        cks += calibrate_oracle(w.k_cal, cfg["bits_k"], True)
        cvs += calibrate_oracle(w.v_cal, cfg["bits_v"], False)
    k = torch.cat(ks, 1).contiguous()
    v = torch.cat(vs, 1).contiguous()
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    _, _, kc, vc = _compress(cks, cvs, k, v, flags=flags)
    assert flags.item() == 0
    rng = np.random.default_rng(7)
    kw, vw = kc.words_u32(), vc.words_u32()
    for _ in range(48):
        h = int(rng.integers(0, L * nkv))
        ts = np.sort(rng.choice(T, size=16, replace=False))
        xk = k[0, h, ts].double().numpy()
        xv = v[0, h, ts].double().numpy()
        compare_compressed(kw[0, h, ts], kc.norm[0, h, ts].cpu().numpy(), kc.rnorm[0, h, ts].cpu().numpy(), xk,
                           cks[h])
        compare_compressed(vw[0, h, ts], vc.norm[0, h, ts].cpu().numpy(), None, xv, cvs[h])


@pytest.mark.parametrize("name,batch,ntok", [("qwen14b", 11, 3), ("tiny", 5, 15), ("gemma9b_sweep", 9, 1),
                                             ("llama8b", 1, 1), ("qwen1_5b_long", 2, 1), ("tiny", 1, 3),
                                             ("qwen14b", 3, 1), ("llama8b", 2, 3)])
def test_append_groups_of_vectors(name, batch, ntok):
    """Decode-step compress of several tokens for many rows (blocks of 1, 2, 4 or
    8 vectors of a head, a ragged last group), each row at its own position,
    against the oracle."""
    w, ck, cv, k, v, nh = _case(name, batch=batch, tokens=ntok, heads=2)
    rng = np.random.default_rng(3)
    cap = 64
    start = [int(s) for s in rng.integers(0, cap - ntok + 1, size=batch)]
    _, _, kc, vc = _compress(ck, cv, k, v, cap=cap, start=start)
    kw, vw = kc.words_u32(), vc.words_u32()
    for b, s in enumerate(start):
        for h in range(nh):
            compare_compressed(kw[b, h, s:s + ntok], kc.norm[b, h, s:s + ntok].cpu().numpy(),
                               kc.rnorm[b, h, s:s + ntok].cpu().numpy(), k[b, h].double().numpy(), ck[h])
            compare_compressed(vw[b, h, s:s + ntok], vc.norm[b, h, s:s + ntok].cpu().numpy(), None,
                               v[b, h].double().numpy(), cv[h])
            others = np.setdiff1d(np.arange(cap), np.arange(s, s + ntok))
            assert np.all(kw[b, h, others] == 0) and np.all(vw[b, h, others] == 0)


@pytest.mark.parametrize("name,batch,tokens,heads,slab_heads,dtype", [
    ("llama8b", 2, 333, 3, 1, torch.float16),        # tensor-core path, one head per piece
    ("qwen14b", 3, 200, 4, 3, torch.float16),        # pieces of 3 heads and a ragged last piece
    ("tiny", 2, 100, 4, 2, torch.float32),           # float64 reference path, head_dim 32
    ("gemma9b_sweep", 2, 100, 2, 1, torch.bfloat16), # block-tiled float64 path, head_dim 256
    ("llama8b", 2, 150, 2, 2, torch.float32),        # block-tiled float64 path, f32 inputs
])
def test_host_input_compress_matches_device_input(name, batch, tokens, heads, slab_heads, dtype):
    """sq_compress_kv_host (pinned host inputs, copies overlapped through a
    small staging buffer) writes exactly what sq_compress_kv writes from device
    inputs, at per-row start positions, and matches the oracle."""
    w, ck, cv, k, v, nh = _case(name, batch=batch, tokens=tokens, heads=heads)
    k, v = k.to(dtype), v.to(dtype)
    d = k.shape[-1]
    cap = ((tokens + 40 + 15) // 16) * 16
    start = [int(s) for s in np.random.default_rng(5).integers(0, cap - tokens + 1, size=batch)]
    rk, rv, kd, vd = _compress(ck, cv, k, v, cap=cap, start=start)
    kh = sq.alloc_cache(batch, nh, cap, ck[0].words, ck[0].m > 0)
    vh = sq.alloc_cache(batch, nh, cap, cv[0].words, False)
    sp = torch.tensor(start, dtype=torch.int32, device="cuda")
    row = tokens * d * k.element_size()
    slab = ((slab_heads * row + 255) // 256) * 256
    staging = torch.empty(2 * slab, dtype=torch.uint8, device="cuda")
    flags = torch.zeros(1, dtype=torch.int32, device="cuda")
    sq.sq_compress_kv_host(rk, rv, k.pin_memory(), v.pin_memory(), batch, nh, d, tokens, sp, kh, vh, staging, flags)
    torch.cuda.synchronize()
    assert flags.item() == 0
    assert np.array_equal(kh.words_u32(), kd.words_u32()) and np.array_equal(vh.words_u32(), vd.words_u32())
    assert torch.equal(kh.norm, kd.norm) and torch.equal(vh.norm, vd.norm)
    if kd.rnorm is not None:
        assert torch.equal(kh.rnorm, kd.rnorm)
    b, h = batch - 1, nh - 1
    s0 = start[b]
    compare_compressed(kh.words_u32()[b, h, s0:s0 + tokens], kh.norm[b, h, s0:s0 + tokens].cpu().numpy(),
                       kh.rnorm[b, h, s0:s0 + tokens].cpu().numpy() if kh.rnorm is not None else None,
                       k[b, h].double().numpy(), ck[h])
    with pytest.raises(sq.SqError) as e:
        sq.sq_compress_kv_host(rk, rv, k.pin_memory(), v.pin_memory(), batch, nh, d, tokens, sp, kh, vh,
                               staging[: 2 * row - 1], flags)
    assert e.value.status == sq.SQ_ERR_WORKSPACE


@pytest.mark.parametrize("name,tokens", [("llama8b", 200), ("tiny", 40), ("gemma9b_sweep", 20)])
def test_zero_vectors_compress_like_the_oracle(name, tokens):
    """Zero vectors (norm 0, so every z is 0): 0 is the middle threshold of every
    width and ties take the lower code, so the record of a zero vector is fixed
    and must equal the oracle's bit for bit (the codes are all on a threshold,
    hence outside the exemption rule's use); its norm is 0 and its rho is the
    norm of the lower levels' residual. The other tokens keep ordinary parity.
    Covers the tensor-core path (fp16, head_dim 128, >= 64 tokens) and the
    float64 kernel (float32 head_dim 32; bf16 head_dim 256)."""
    w, ck, cv, k, v, nh = _case(name, batch=1, tokens=tokens, heads=2)
    zero = [0, 5, tokens - 1]
    k[:, :, zero] = 0
    v[:, :, zero] = 0
    _, _, kc, vc = _compress(ck, cv, k, v)
    keep = np.setdiff1d(np.arange(tokens), zero)
    for cache, cals, x in ((kc, ck, k), (vc, cv, v)):
        words = cache.words_u32()
        norm = cache.norm.cpu().numpy()
        rn = cache.rnorm.cpu().numpy() if cache.rnorm is not None else None
        for h in range(nh):
            xs = x[0, h].double().numpy()
            out = ocodec.compress(xs, cals[h])
            assert np.array_equal(words[0, h, zero], out["words"][zero]), (name, h)
            assert np.all(norm[0, h, zero] == 0.0)
            if rn is not None:
                np.testing.assert_allclose(rn[0, h, zero], out["rnorm"][zero], rtol=1e-6)
            compare_compressed(words[0, h, keep], norm[0, h, keep], rn[0, h, keep] if rn is not None else None,
                               xs[keep], cals[h])
