"""The C-ABI library: it loads without a GPU, exports every entry point the
public header declares, and its host-only calls behave as documented."""

import ctypes
import os
import re

import numpy as np
import pytest

from compressed_attention_head_b200 import build as sqbuild
from compressed_attention_head_b200 import sq
from oracle import codebook as ocb
from oracle import record as orec

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in sorted(os.listdir(os.path.join(ROOT, "include"))):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(sq_[a-z0-9_]+)\s*\(", text))
    return names


@pytest.fixture(scope="module")
def libsq():
    sqbuild.build()
    return sq.lib()


def test_exports_every_declared_symbol(libsq):
    declared = _declared()
    assert {"sq_calibrate", "sq_compress_kv", "sq_decompress_kv", "sq_attn_decode"} <= declared
    for name in declared:
        assert hasattr(libsq, name), name
        assert name in sq._SIGNATURES, f"binding misses {name}"


def test_status_strings_and_version(libsq):
    assert sq.sq_abi_version() == 3
    for s in range(8):
        assert sq.sq_status_str(s) and "unknown" not in sq.sq_status_str(s)
    assert "unknown" in sq.sq_status_str(99)


def test_record_geometry_matches_the_documented_layout(libsq):
    for d in (32, 64, 128, 256):
        n = sq.sq_calib_bytes(d)
        assert n % 256 == 0 and n >= orec.canonical_bytes(d)
    assert sq.sq_calib_bytes(48) == 0


def test_record_words(libsq):
    assert sq.sq_record_words(sq.calib_params(128, 1, 2.5, True)) == 10
    assert sq.sq_record_words(sq.calib_params(128, 1, 3.0, True)) == 12
    assert sq.sq_record_words(sq.calib_params(256, 1, 3.5, False)) == 28
    assert sq.sq_record_words(sq.calib_params(32, 1, 3.01, False)) == 0     # not a whole number of bits
    assert sq.sq_record_words(sq.calib_params(40, 1, 3.0, False)) == 0     # unsupported head_dim


def test_library_codebook_matches_oracle(libsq):
    for b in range(1, 9):
        lv, th, dist = sq.sq_codebook(b)
        l2, t2, d2 = ocb.lloyd_max(b)
        assert np.max(np.abs(lv - l2)) < 1e-10
        assert np.max(np.abs(th - t2)) < 1e-10
        assert abs(dist - d2) < 1e-14
    assert sq.lib().sq_codebook(0, None, None, None) == sq.SQ_ERR_ARG
    assert sq.lib().sq_codebook(9, None, None, None) == sq.SQ_ERR_ARG


def test_argument_errors_need_no_gpu(libsq):
    L = sq.lib()
    p = sq.calib_params(48, 1, 3.0, True)
    assert L.sq_calibrate(ctypes.byref(p), None, 0, 16, 0, 48, None, None, 0, None, None) == sq.SQ_ERR_UNSUPPORTED
    p = sq.calib_params(32, 1, 3.0, True)
    assert L.sq_calibrate(ctypes.byref(p), None, 0, 16, 0, 32, None, None, 0, None, None) == sq.SQ_ERR_ARG
    assert L.sq_calib_import(None, 1, 32, None, None) == sq.SQ_ERR_ARG
    assert L.sq_compress_kv(None, None, None, None, 1, 1, 1, 32, 0, None, None, None, None, None) == sq.SQ_OK
    assert L.sq_compress_kv(None, None, None, None, 1, 1, 1, 32, 4, None, None, None, None, None) == sq.SQ_ERR_ARG
    assert L.sq_attn_workspace(1, 3, 2, 128, 100) > 0
    assert L.sq_attn_workspace(1, 1, 1, 100, 100) == 0


def test_host_compress_staging_and_argument_errors(libsq):
    """sq_compress_host_staging sizes (two 256-byte-rounded slabs of whole heads,
    about 16 MiB each) and the host-input compress's checks, which run before
    any CUDA call."""
    L = sq.lib()
    row = 2048 * 128 * 2                                    # one fp16 head of 2048 tokens
    assert L.sq_compress_host_staging(1, 256, 128, sq.SQ_F16, 2048) == 2 * 32 * row
    assert L.sq_compress_host_staging(4, 2, 128, sq.SQ_F16, 2048) == 2 * 2 * row
    assert L.sq_compress_host_staging(1, 8, 32, sq.SQ_F32, 3) == 2 * 3072         # 8 heads of 384 B per slab
    assert L.sq_compress_host_staging(1, 3, 32, sq.SQ_F32, 1) == 2 * 512          # 3 heads of 128 B, rounded up
    assert L.sq_compress_host_staging(1, 8, 48, sq.SQ_F16, 64) == 0
    assert L.sq_compress_host_staging(1, 8, 128, sq.SQ_F16, 0) == 0
    fake = 1 << 20                                           # aligned addresses, never dereferenced
    cache = sq.sq_cache(fake, fake, fake, 1, 2, 64, 12)
    args = (fake, None, fake, None, sq.SQ_F16, 1, 2, 128, 64, None, ctypes.byref(cache), None)
    one_head = 64 * 128 * 2
    assert L.sq_compress_kv_host(*args, None, 1 << 20, None, None) == sq.SQ_ERR_ARG          # no staging
    assert L.sq_compress_kv_host(*args, fake + 16, 1 << 20, None, None) == sq.SQ_ERR_ARG     # misaligned staging
    assert L.sq_compress_kv_host(*args, fake, 2 * one_head - 1, None, None) == sq.SQ_ERR_WORKSPACE
    assert L.sq_compress_kv_host(fake, None, None, None, sq.SQ_F16, 1, 2, 128, 64, None, None, None, fake,
                                 1 << 20, None, None) == sq.SQ_ERR_ARG                       # nothing to compress
    assert L.sq_compress_kv_host(*args[:8], 0, *args[9:], None, 0, None, None) == sq.SQ_OK    # n_tok = 0
    assert L.sq_compress_kv_host(fake, None, fake, None, sq.SQ_F16, 1, 2, 48, 64, None, ctypes.byref(cache),
                                 None, fake, 1 << 20, None, None) == sq.SQ_ERR_UNSUPPORTED


def _splits_from_workspace(L, batch, n_q, n_kv, d, ctx):
    """The split count a workspace was sized for: floats of w, u, the split
    partials, then one uint32 counter per (batch, KV head)."""
    nbytes = L.sq_attn_workspace(batch, n_q, n_kv, d, ctx) - 4 * batch * n_kv
    floats = nbytes // 4
    per_head = floats // (batch * n_q) - 2 * d
    assert per_head % (d + 2) == 0
    return per_head // (d + 2)


def _chunk(ctx, S):
    return -(-(-(-ctx // S)) // 128) * 128


def _valid(ctx):
    return [S for S in range(1, 257) if -(-ctx // _chunk(ctx, S)) == S]


def _splits_mma(batch, n_kv, d, ctx):
    """mma.sync partials: 148 SMs x 3 (d 128) / 4 (d 64) / 1 (d 256) resident
    blocks; cost waves x (1 + 2 tiles per block), the smaller S on ties."""
    slots = 148 * (4 if d <= 64 else (3 if d <= 128 else 1))
    units = batch * n_kv

    def cost(S):
        return -(-units * S // slots) * (1 + 2 * (_chunk(ctx, S) // 128))
    return min(_valid(ctx), key=lambda S: (cost(S), S))


def _splits_td(batch, n_kv, d, ctx, ng=None):
    """tcgen05 partials: one block per SM (148) whose ng warp groups (at most 4
    for d 64, 3 for d 128 and 256; fewer when the records' buffers do not fit)
    take the tiles; cost waves x (1 + tiles per group)."""
    ng = ng or (4 if d <= 64 else 3)
    units = batch * n_kv

    def cost(S):
        return -(-units * S // 148) * (1 + -(-(_chunk(ctx, S) // 128) // ng))
    return min(_valid(ctx), key=lambda S: (cost(S), S))


def test_attention_split_count(libsq):
    """The context split counts behind sq_attn_workspace: every split holds
    tokens (spans of whole 128-token tiles), each partial kernel's count
    minimises its documented wave cost, and the workspace holds the largest
    count over the partial kernels and the tcgen05 kernel's group counts (which
    kernel and how many groups a call takes depends on its records)."""
    L = sq.lib()
    for (batch, n_kv, g, d, ctx) in [(1, 256, 4, 128, 2049), (4, 384, 5, 128, 8193), (16, 56, 6, 128, 32769),
                                     (1, 2, 1, 64, 600), (2, 3, 2, 128, 1), (3, 7, 1, 128, 100000),
                                     (1, 1, 1, 128, 300000), (64, 336, 2, 256, 4097)]:
        s = _splits_from_workspace(L, batch, n_kv * g, n_kv, d, ctx)
        assert 1 <= s <= 256
        ngmax = 4 if d <= 64 else 3
        want = max([_splits_mma(batch, n_kv, d, ctx)] + [_splits_td(batch, n_kv, d, ctx, ng) for ng in range(1, ngmax + 1)])
        assert s == want, (batch, n_kv, d, ctx)
    # the decode shapes of the benchmark (split counts of the tcgen05 kernel)
    assert _splits_td(4, 384, 128, 8193) == 2
    assert _splits_td(16, 56, 128, 32769) >= 1


def test_header_constants_match_the_binding():
    """Every #define and enum value of the public header that the binding
    mirrors has the same value there."""
    text = open(os.path.join(ROOT, "include", "sq.h")).read()
    defines = {m.group(1): int(m.group(2).rstrip("u"), 0)     # plain literals only, not expressions
               for m in re.finditer(r"^#define\s+(SQ_\w+)\s+(0x[0-9a-fA-F]+u?|\d+u?)\s*(?:/\*.*)?$", text, re.M)}
    enums = {m.group(1): int(m.group(2)) for m in re.finditer(r"\b(SQ_[A-Z0-9_]+)\s*=\s*(\d+)", text)}
    mirrored = 0
    for name, value in {**defines, **enums}.items():
        if hasattr(sq, name):
            assert getattr(sq, name) == value, name
            mirrored += 1
    for name in ("SQ_FLAG_CAPACITY", "SQ_FLAG_RECORD", "SQ_FLAG_SEQLEN", "SQ_FLAG_TIMEOUT", "SQ_ERR_WORKSPACE",
                 "SQ_F16", "SQ_ATTN_NOALLOC_MAX_BYTES"):
        assert name in defines or name in enums, name
    assert mirrored >= 10
