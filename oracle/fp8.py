"""FP8 E4M3 storage for the paged cache, in numpy: test infrastructure only.

Not on the pages, which store K/V in 16-bit; this is a plain extension that
halves the bytes a decode step reads. The format is the OCP 8-bit E4M3 ("fn":
no infinities): sign bit 7, exponent bits 6-3 (bias 7), mantissa bits 2-0;
exponent 0 holds the subnormals m * 2^-9; 0x7F / 0xFF are NaN; the largest
finite magnitude is 448. One fp32 scale per tensor: stored = e4m3(x / scale),
value = scale * decode(stored).

Quantization is round to nearest, ties to the even code, with out-of-range
magnitudes saturated to 448 (reading: the usual "satfinite" conversion; the
kernel's append does the same, and the pins check it against torch's own
float8_e4m3fn conversion wherever that one is defined). The quotient x / scale
is taken in fp32 with one correctly rounded division before it is rounded to a
code: a quantised code is an integer decided by floating point, so both sides
take it in the kernel's precision (the inputs are 16-bit, exact in fp32).
"""

import ctypes

import numpy as np
import torch

from . import decode as _decode

_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = _decode._load()
        lib.oracle_decode_e4m3.argtypes = [ctypes.c_uint8]
        lib.oracle_decode_e4m3.restype = ctypes.c_double
        p, i64 = ctypes.c_void_p, ctypes.c_int64
        lib.oracle_paged_decode_fp8.argtypes = [p, p, p, ctypes.c_double, ctypes.c_double, p, p,
                                                i64, i64, i64, i64, i64, i64, i64,
                                                ctypes.c_double, ctypes.c_int, ctypes.c_int, p]
        lib.oracle_paged_decode_fp8.restype = ctypes.c_int
        _lib = lib
    return _lib


def decode_table():
    """fp64 value of every code 0 .. 255 (NaN for 0x7F and 0xFF)."""
    lib = _load()
    return np.array([lib.oracle_decode_e4m3(c) for c in range(256)], dtype=np.float64)


def quantize(x, scale):
    """Codes (uint8) of fp32(x / scale): round to nearest, ties to even code,
    saturate at 448. x is any float array (taken as fp32); NaN gives 0x7F."""
    y = (np.asarray(x, dtype=np.float32) / np.float32(scale)).astype(np.float64)
    table = decode_table()
    mags = table[:127]  # codes 0 .. 126: the finite non-negative values, increasing
    a = np.minimum(np.abs(y), mags[-1])
    hi = np.clip(np.searchsorted(mags, a, side="left"), 0, 126)  # first >= a
    lo = np.maximum(hi - 1, 0)
    d_lo, d_hi = a - mags[lo], mags[hi] - a
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0) & (hi != lo))
    code = np.where(pick_hi, hi, lo).astype(np.uint8)
    code = np.where(np.signbit(y), code | np.uint8(0x80), code)  # the sign, zeros included
    return np.where(np.isnan(y), np.uint8(0x7F), code).astype(np.uint8)


def paged_decode_fp8(q, k_cache, v_cache, k_scale, v_scale, block_tables, seq_lens, scale,
                     threads=0):
    """fp64 decode over uint8 E4M3 caches [NB, Hkv, S, D]; q [B, H, D] fp16/bf16."""
    B, H, D = q.shape
    NB, Hkv, S, D2 = k_cache.shape
    if D2 != D or H % Hkv:
        raise _decode.OracleError("shape mismatch")
    qb = q.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    kb = np.ascontiguousarray(torch.as_tensor(k_cache).cpu().numpy().astype(np.uint8))
    vb = np.ascontiguousarray(torch.as_tensor(v_cache).cpu().numpy().astype(np.uint8))
    bt = np.ascontiguousarray(torch.as_tensor(block_tables).cpu().numpy().astype(np.int32))
    sl = np.ascontiguousarray(torch.as_tensor(seq_lens).cpu().numpy().astype(np.int32))
    out = np.zeros((B, H, D), np.float64)
    ptr = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    rc = _load().oracle_paged_decode_fp8(
        ptr(qb), ptr(kb), ptr(vb), float(k_scale), float(v_scale), ptr(bt), ptr(sl), B, H, Hkv,
        D, S, NB, bt.shape[1], float(scale), 0 if q.dtype == torch.float16 else 1, int(threads),
        ptr(out))
    if rc:
        raise _decode.OracleError(f"oracle_paged_decode_fp8 returned {rc}")
    return out
