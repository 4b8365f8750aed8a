"""Python binding of libsq: the C-ABI entry points under the same names.

Argument marshalling only: every step of the compressed-KV path runs in the
CUDA library. PyTorch supplies device memory and streams. A missing or
unloadable libsq raises at import of the first call; there is no fallback.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libsq.so")

SQ_OK, SQ_ERR_ARG, SQ_ERR_UNSUPPORTED, SQ_ERR_CUDA = 0, 1, 2, 3
SQ_ERR_NOT_CONVERGED, SQ_ERR_CAPACITY, SQ_ERR_WORKSPACE, SQ_ERR_RECORD = 4, 5, 6, 7
SQ_F32, SQ_F16, SQ_BF16 = 0, 1, 2
SQ_FLAG_CAPACITY, SQ_FLAG_RECORD, SQ_FLAG_SEQLEN, SQ_FLAG_TIMEOUT = 1, 2, 4, 0x80000000
DTYPE_CODE = {torch.float32: SQ_F32, torch.float16: SQ_F16, torch.bfloat16: SQ_BF16}


class SqError(RuntimeError):
    def __init__(self, status: int, what: str):
        detail = f" [{lib().sq_last_error().decode()}]" if status == SQ_ERR_CUDA else ""
        super().__init__(f"{what}: {sq_status_str(status)} ({status}){detail}")
        self.status = status


class sq_calib_params(ctypes.Structure):
    _fields_ = [("d", ctypes.c_int), ("n_heads", ctypes.c_int), ("avg_bits", ctypes.c_double),
                ("is_key", ctypes.c_int), ("qjl", ctypes.c_int), ("normalize", ctypes.c_int),
                ("d_eff_override", ctypes.c_int), ("max_bits", ctypes.c_int), ("seed", ctypes.c_uint64),
                ("max_sweeps", ctypes.c_int), ("tol", ctypes.c_double), ("rotation", ctypes.c_int),
                ("cumvar", ctypes.c_double), ("codebooks", ctypes.c_int), ("fit_iters", ctypes.c_int)]


class sq_cache(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("norm", ctypes.c_void_p), ("rnorm", ctypes.c_void_p),
                ("batch", ctypes.c_int), ("n_heads", ctypes.c_int), ("cap", ctypes.c_int64),
                ("words", ctypes.c_int)]


_lib = None
_P = ctypes.c_void_p
_SIGNATURES = {
    "sq_abi_version": (ctypes.c_int, []),
    "sq_status_str": (ctypes.c_char_p, [ctypes.c_int]),
    "sq_last_error": (ctypes.c_char_p, []),
    "sq_calib_bytes": (ctypes.c_size_t, [ctypes.c_int]),
    "sq_record_words": (ctypes.c_int, [ctypes.POINTER(sq_calib_params)]),
    "sq_codebook": (ctypes.c_int, [ctypes.c_int, _P, _P, _P]),
    "sq_init": (ctypes.c_int, []),
    "sq_set_option": (ctypes.c_int, [ctypes.c_int, ctypes.c_int]),
    "sq_calibrate_workspace": (ctypes.c_size_t, [ctypes.POINTER(sq_calib_params), ctypes.c_int64]),
    "sq_calibrate": (ctypes.c_int, [ctypes.POINTER(sq_calib_params), _P, ctypes.c_int, ctypes.c_int64,
                                    ctypes.c_int64, ctypes.c_int64, _P, _P, ctypes.c_size_t, _P, _P]),
    "sq_calib_import": (ctypes.c_int, [_P, ctypes.c_int, ctypes.c_int, _P, _P]),
    "sq_compress_kv": (ctypes.c_int, [_P, _P, _P, _P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_int64, _P, ctypes.POINTER(sq_cache), ctypes.POINTER(sq_cache),
                                      _P, _P]),
    "sq_compress_host_staging": (ctypes.c_size_t, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                   ctypes.c_int64]),
    "sq_compress_kv_host": (ctypes.c_int, [_P, _P, _P, _P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int64, _P, ctypes.POINTER(sq_cache), ctypes.POINTER(sq_cache),
                                           _P, ctypes.c_size_t, _P, _P]),
    "sq_decompress_kv": (ctypes.c_int, [_P, ctypes.POINTER(sq_cache), ctypes.c_int, ctypes.c_int64,
                                        ctypes.c_int64, ctypes.c_int, _P, _P, _P]),
    "sq_attn_workspace": (ctypes.c_size_t, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int64]),
    "sq_attn_decode": (ctypes.c_int, [_P, _P, ctypes.POINTER(sq_cache), ctypes.POINTER(sq_cache), _P,
                                      ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64,
                                      _P, ctypes.c_int, ctypes.c_float, _P, ctypes.c_int, _P, _P,
                                      ctypes.c_size_t, _P, _P]),
    "sq_decode_step": (ctypes.c_int, [_P, _P, ctypes.POINTER(sq_cache), ctypes.POINTER(sq_cache), _P, _P, _P,
                                      ctypes.c_int, _P, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                      ctypes.c_int64, ctypes.c_float, _P, ctypes.c_int, _P, _P, ctypes.c_size_t, _P,
                                      _P]),
    "sq_attn_prefill_workspace": (ctypes.c_size_t, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                    ctypes.c_int64, ctypes.c_int64]),
    "sq_attn_prefill": (ctypes.c_int, [_P, _P, ctypes.POINTER(sq_cache), ctypes.POINTER(sq_cache), _P, ctypes.c_int,
                                       ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64, ctypes.c_int64, _P,
                                       ctypes.c_int, ctypes.c_float, _P, ctypes.c_int, _P, ctypes.c_size_t, _P, _P]),
    "sq_attn_decode_noalloc": (ctypes.c_int, [_P, _P, ctypes.POINTER(sq_cache), ctypes.POINTER(sq_cache), _P,
                                              ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                              ctypes.c_int64, _P, ctypes.c_int, ctypes.c_float, _P, ctypes.c_int,
                                              _P, _P, _P]),
    "sq_wait_selftest": (ctypes.c_int, [ctypes.c_uint32, _P, _P]),
}

SQ_ATTN_NOALLOC_MAX_BYTES = 8 << 20


def lib() -> ctypes.CDLL:
    """The loaded libsq (raises if it is missing: build it with build.py)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libsq not built: {LIB_PATH} is missing "
                               "(run python -m compressed_attention_head_b200.build)")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(status: int, what: str) -> None:
    if status != SQ_OK:
        raise SqError(status, what)


# --------------------------------------------------------------------------- host-only calls
def sq_abi_version() -> int:
    return lib().sq_abi_version()


def sq_status_str(status: int) -> str:
    return lib().sq_status_str(status).decode()


def sq_calib_bytes(d: int) -> int:
    return lib().sq_calib_bytes(d)


def calib_params(d, n_heads, avg_bits, is_key, qjl=True, normalize=True, d_eff_override=0, max_bits=8,
                 seed=42, max_sweeps=30, tol=1e-13, rotation=0, cumvar=0.0, codebooks=0,
                 fit_iters=0) -> sq_calib_params:
    """rotation: 0 calibrated eigenbasis, 1 random rotation (A/B baseline);
    cumvar: 0 participation-ratio d_eff, else the cumulative-variance fraction;
    codebooks: 0 shared Gaussian Lloyd-Max, 1 per-regime codebooks fitted to the
    calibration vectors (fit_iters Lloyd iterations, 0 = the library's 30)."""
    return sq_calib_params(d, n_heads, float(avg_bits), int(bool(is_key)), int(bool(qjl)), int(bool(normalize)),
                           int(d_eff_override), int(max_bits), int(seed) & ((1 << 64) - 1), int(max_sweeps),
                           float(tol), int(rotation), float(cumvar), int(codebooks), int(fit_iters))


def sq_record_words(params: sq_calib_params) -> int:
    return lib().sq_record_words(ctypes.byref(params))


def sq_codebook(b: int):
    """(levels, thresholds, D) of the library's b-bit Gaussian Lloyd-Max quantizer."""
    lv = np.zeros(1 << b)
    th = np.zeros((1 << b) - 1)
    dist = ctypes.c_double()
    _check(lib().sq_codebook(b, lv.ctypes.data, th.ctypes.data, ctypes.addressof(dist)), "sq_codebook")
    return lv, th, dist.value


def sq_calibrate_workspace(params: sq_calib_params, n_tokens: int) -> int:
    return lib().sq_calibrate_workspace(ctypes.byref(params), n_tokens)


def sq_attn_workspace(batch, n_q_heads, n_kv_heads, d, max_ctx) -> int:
    return lib().sq_attn_workspace(batch, n_q_heads, n_kv_heads, d, max_ctx)


# --------------------------------------------------------------------------- device buffers
@dataclass
class PackedCache:
    """Caller-owned device arrays of one packed cache (see sq_cache in sq.h)."""

    codes: torch.Tensor          # int32 [batch, n_heads, cap / 32, words, 32], read as uint32
    norm: torch.Tensor           # float32 [batch, n_heads, cap]
    rnorm: torch.Tensor | None   # float32 [batch, n_heads, cap] or None
    batch: int
    n_heads: int
    cap: int
    words: int

    def struct(self) -> sq_cache:
        return sq_cache(self.codes.data_ptr(), self.norm.data_ptr(),
                        self.rnorm.data_ptr() if self.rnorm is not None else None,
                        self.batch, self.n_heads, self.cap, self.words)

    def words_u32(self) -> np.ndarray:
        """The records as [batch, n_heads, cap, words] uint32 (undoing the 32-token interleave)."""
        c = self.codes.cpu().numpy().view(np.uint32)
        return np.ascontiguousarray(c.transpose(0, 1, 2, 4, 3)).reshape(self.batch, self.n_heads, self.cap,
                                                                        self.words)

    def tiled(self, rep_batch: int, rep_heads: int) -> "PackedCache":
        """A new cache holding this one repeated rep_batch times over the batch and
        rep_heads times over the heads (row (b, h) = this row (b % batch, h % n_heads))."""
        return PackedCache(self.codes.repeat(rep_batch, rep_heads, 1, 1, 1),
                           self.norm.repeat(rep_batch, rep_heads, 1),
                           self.rnorm.repeat(rep_batch, rep_heads, 1) if self.rnorm is not None else None,
                           self.batch * rep_batch, self.n_heads * rep_heads, self.cap, self.words)


def alloc_cache(batch, n_heads, cap, words, with_rnorm, device="cuda") -> PackedCache:
    """Zeroed packed cache; cap is rounded up to a multiple of 32."""
    cap = ((int(cap) + 31) // 32) * 32
    codes = torch.zeros(batch, n_heads, cap // 32, words, 32, dtype=torch.int32, device=device)
    norm = torch.zeros(batch, n_heads, cap, dtype=torch.float32, device=device)
    rnorm = torch.zeros_like(norm) if with_rnorm else None
    return PackedCache(codes, norm, rnorm, batch, n_heads, cap, words)


def alloc_records(n_heads: int, d: int, device="cuda") -> torch.Tensor:
    """Zeroed storage for n_heads calibration records (uint8, record after record)."""
    return torch.zeros(n_heads * sq_calib_bytes(d), dtype=torch.uint8, device=device)


# --------------------------------------------------------------------------- launching calls
def sq_init() -> None:
    _check(lib().sq_init(), "sq_init")


SQ_OPT_COMPRESS_PATH = 1
SQ_OPT_ATTN_PATH = 2
SQ_OPT_TC_ERROR_BOUND = 3


def sq_set_option(option: int, value: int) -> None:
    _check(lib().sq_set_option(option, value), "sq_set_option")


def sq_calibrate(params, x, n_tokens, stride_head, stride_tok, calib_out, ws, status=None, stream=None):
    _check(lib().sq_calibrate(ctypes.byref(params), _ptr(x), DTYPE_CODE[x.dtype], n_tokens, stride_head,
                              stride_tok, _ptr(calib_out), _ptr(ws), ws.numel() * ws.element_size(),
                              _ptr(status), _stream(stream)), "sq_calibrate")


def sq_calib_import(calib, n_heads, d, status=None, stream=None):
    _check(lib().sq_calib_import(_ptr(calib), n_heads, d, _ptr(status), _stream(stream)), "sq_calib_import")


def sq_compress_kv(calib_k, calib_v, k, v, batch, n_heads, d, n_tok, start_pos, kc, vc, flags=None,
                   stream=None):
    x = k if k is not None else v
    kcs = kc.struct() if kc is not None else None
    vcs = vc.struct() if vc is not None else None
    _check(lib().sq_compress_kv(_ptr(calib_k), _ptr(calib_v), _ptr(k), _ptr(v), DTYPE_CODE[x.dtype], batch,
                                n_heads, d, n_tok, _ptr(start_pos),
                                ctypes.byref(kcs) if kcs is not None else None,
                                ctypes.byref(vcs) if vcs is not None else None, _ptr(flags),
                                _stream(stream)), "sq_compress_kv")


def sq_compress_host_staging(batch, n_heads, d, dtype, n_tok) -> int:
    return lib().sq_compress_host_staging(batch, n_heads, d, DTYPE_CODE[dtype], n_tok)


def sq_compress_kv_host(calib_k, calib_v, k, v, batch, n_heads, d, n_tok, start_pos, kc, vc, staging, flags=None,
                        stream=None):
    """k, v: CPU tensors (pinned for overlapped copies); staging: a device uint8 tensor."""
    x = k if k is not None else v
    for t in (k, v):
        if t is not None and (t.is_cuda or not t.is_contiguous()):
            raise ValueError("sq_compress_kv_host takes contiguous host tensors")
    kcs = kc.struct() if kc is not None else None
    vcs = vc.struct() if vc is not None else None
    _check(lib().sq_compress_kv_host(_ptr(calib_k), _ptr(calib_v), _ptr(k), _ptr(v), DTYPE_CODE[x.dtype], batch,
                                     n_heads, d, n_tok, _ptr(start_pos),
                                     ctypes.byref(kcs) if kcs is not None else None,
                                     ctypes.byref(vcs) if vcs is not None else None, _ptr(staging),
                                     staging.numel() * staging.element_size() if staging is not None else 0,
                                     _ptr(flags), _stream(stream)), "sq_compress_kv_host")


def sq_decompress_kv(calib, cache, d, t0, n_tok, apply_qjl, out, flags=None, stream=None):
    cs = cache.struct()
    _check(lib().sq_decompress_kv(_ptr(calib), ctypes.byref(cs), d, t0, n_tok, int(bool(apply_qjl)), _ptr(out),
                                  _ptr(flags), _stream(stream)), "sq_decompress_kv")


def sq_attn_decode(calib_k, calib_v, kc, vc, seq_lens, batch, n_q_heads, n_kv_heads, d, max_ctx, q, scale, out,
                   scores_out=None, ws=None, flags=None, stream=None):
    kcs, vcs = kc.struct(), vc.struct()
    _check(lib().sq_attn_decode(_ptr(calib_k), _ptr(calib_v), ctypes.byref(kcs), ctypes.byref(vcs),
                                _ptr(seq_lens), batch, n_q_heads, n_kv_heads, d, max_ctx, _ptr(q),
                                DTYPE_CODE[q.dtype], float(scale), _ptr(out), DTYPE_CODE[out.dtype],
                                _ptr(scores_out), _ptr(ws), ws.numel() * ws.element_size() if ws is not None else 0,
                                _ptr(flags), _stream(stream)), "sq_attn_decode")


def sq_attn_prefill_workspace(batch, n_q_heads, n_kv_heads, d, n_qtok, max_ctx) -> int:
    return lib().sq_attn_prefill_workspace(batch, n_q_heads, n_kv_heads, d, n_qtok, max_ctx)


def sq_attn_prefill(calib_k, calib_v, kc, vc, start, batch, n_q_heads, n_kv_heads, d, n_qtok, max_ctx, q, scale, out,
                    ws, flags=None, stream=None):
    """Causal attention of q [batch, n_q, n_qtok, d] at positions start[b] + t (see sq.h)."""
    kcs, vcs = kc.struct(), vc.struct()
    _check(lib().sq_attn_prefill(_ptr(calib_k), _ptr(calib_v), ctypes.byref(kcs), ctypes.byref(vcs), _ptr(start),
                                 batch, n_q_heads, n_kv_heads, d, n_qtok, max_ctx, _ptr(q), DTYPE_CODE[q.dtype],
                                 float(scale), _ptr(out), DTYPE_CODE[out.dtype], _ptr(ws),
                                 ws.numel() * ws.element_size(), _ptr(flags), _stream(stream)), "sq_attn_prefill")


def sq_decode_step(calib_k, calib_v, kc, vc, k_new, v_new, q, pos, batch, n_q_heads, n_kv_heads, d, max_ctx, scale,
                   out, scores_out=None, ws=None, flags=None, stream=None):
    """Append the new token at pos[b] and attend over pos[b] + 1 tokens (see sq.h)."""
    kcs, vcs = kc.struct(), vc.struct()
    _check(lib().sq_decode_step(_ptr(calib_k), _ptr(calib_v), ctypes.byref(kcs), ctypes.byref(vcs), _ptr(k_new),
                                _ptr(v_new), _ptr(q), DTYPE_CODE[q.dtype], _ptr(pos), batch, n_q_heads, n_kv_heads, d,
                                max_ctx, float(scale), _ptr(out), DTYPE_CODE[out.dtype], _ptr(scores_out), _ptr(ws),
                                ws.numel() * ws.element_size() if ws is not None else 0, _ptr(flags),
                                _stream(stream)), "sq_decode_step")


def sq_attn_decode_noalloc(calib_k, calib_v, kc, vc, seq_lens, batch, n_q_heads, n_kv_heads, d, max_ctx, q, scale,
                           out, scores_out=None, flags=None, stream=None):
    """sq_attn_decode with the library's fixed scratch array instead of a workspace
    (for callers that cannot allocate device memory; see sq.h)."""
    kcs, vcs = kc.struct(), vc.struct()
    _check(lib().sq_attn_decode_noalloc(_ptr(calib_k), _ptr(calib_v), ctypes.byref(kcs), ctypes.byref(vcs),
                                        _ptr(seq_lens), batch, n_q_heads, n_kv_heads, d, max_ctx, _ptr(q),
                                        DTYPE_CODE[q.dtype], float(scale), _ptr(out), DTYPE_CODE[out.dtype],
                                        _ptr(scores_out), _ptr(flags), _stream(stream)), "sq_attn_decode_noalloc")


def sq_wait_selftest(limit_us, flags, stream=None):
    """One GPU thread waits on an mbarrier nothing arrives on for limit_us
    microseconds with the library's bounded-wait helper, then sets
    SQ_FLAG_TIMEOUT in flags (see sq.h)."""
    _check(lib().sq_wait_selftest(int(limit_us), _ptr(flags), _stream(stream)), "sq_wait_selftest")
