"""fp64 paged decode attention, the oracle (test infrastructure only).

Thin ctypes marshalling around ``oracle.cpp``; all arithmetic is in that file.
What is computed, per request i and head h, is the plain definition from
"vLLM KV Cache and PagedAttention Explained", "Appendix: The Attention Score
Formula": out = softmax(scale * q K^T) V over the request's first seq_lens[i]
tokens, where token t is read from physical block block_tables[i][t // S] at
offset t % S ("PagedAttention" card, "OS paging과 같은 발상"), in the
[Block, Head, Block_Size, Head_D] layout of "vLLM의 PagedAttention 아키텍처와 GPU
메모리 최적화 원리", section 4.

``partition_stats`` returns, for partitions of P tokens, the partition's max
score m, its sum of exp(s - m) and its exp(s - m)-weighted sum of V: the
quantities a split-KV ("FlashDecoding", "PagedAttention" card,
"헷갈리기 쉬운 구분") pass produces, by definition.
"""

import ctypes

import numpy as np
import torch

from . import build as _build

_DTYPE_CODE = {torch.float16: 0, torch.bfloat16: 1}
_lib = None


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(_build.build())
        p = ctypes.c_void_p
        i64 = ctypes.c_int64
        lib.oracle_paged_decode.argtypes = [p, p, p, p, p, i64, i64, i64, i64, i64, i64, i64,
                                            ctypes.c_double, ctypes.c_int, p, i64, ctypes.c_int, p]
        lib.oracle_paged_decode.restype = ctypes.c_int
        lib.oracle_partition_stats.argtypes = [p, p, p, p, p, i64, i64, i64, i64, i64, i64,
                                               ctypes.c_double, ctypes.c_int, i64, i64,
                                               ctypes.c_int, p, p, p]
        lib.oracle_partition_stats.restype = ctypes.c_int
        lib.oracle_paged_prefill.argtypes = [p, p, p, p, p, p, i64, i64, i64, i64, i64, i64, i64,
                                             ctypes.c_double, ctypes.c_int, ctypes.c_int, p]
        lib.oracle_paged_prefill.restype = ctypes.c_int
        lib.oracle_decode16.argtypes = [ctypes.c_uint16, ctypes.c_int]
        lib.oracle_decode16.restype = ctypes.c_double
        _lib = lib
    return _lib


def _bits(t) -> np.ndarray:
    """The raw 16-bit patterns of an fp16/bf16 tensor (or a uint16 array of them),
    as a contiguous uint16 array."""
    if isinstance(t, np.ndarray):
        return np.ascontiguousarray(t, dtype=np.uint16)
    t = t.detach().to("cpu").contiguous()
    return t.view(torch.int16).numpy().view(np.uint16)


def _i32(t) -> np.ndarray:
    return np.ascontiguousarray(torch.as_tensor(t).to("cpu").numpy(), dtype=np.int32)


def _ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data)


class OracleError(RuntimeError):
    pass


def decode16(bits: int, dtype: torch.dtype) -> float:
    """One fp16/bf16 bit pattern decoded to a Python float by the oracle."""
    return _load().oracle_decode16(bits, _DTYPE_CODE[dtype])


def paged_decode(q, k_cache, v_cache, block_tables, seq_lens, scale, pairs=None, threads=0,
                 dtype=None):
    """fp64 attention output.

    q [B, H, D]; k_cache, v_cache [NB, Hkv, S, D] (fp16 or bf16, same dtype as q),
    Hkv dividing H: query head h reads KV head h // (H // Hkv) (grouped-query
    attention; Hkv == H is the pages' one KV head per query head);
    block_tables [B, MB] int32; seq_lens [B] int32. ``pairs`` is an optional
    sequence of (request, head) pairs; the result is then [len(pairs), D],
    otherwise [B, H, D]. ``threads`` = 0 uses every host core. The 16-bit inputs
    may also be uint16 numpy arrays of bit patterns, with ``dtype`` naming them.
    """
    B, H, D = q.shape
    NB, Hkv, S, D2 = k_cache.shape
    if D2 != D or H % Hkv != 0 or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise OracleError("shape mismatch")
    if dtype is None:
        if q.dtype != k_cache.dtype or q.dtype != v_cache.dtype:
            raise OracleError("dtype mismatch")
        dtype = q.dtype
    qb, kb, vb = _bits(q), _bits(k_cache), _bits(v_cache)
    bt = _i32(block_tables).reshape(B, -1)
    sl = _i32(seq_lens).reshape(B)
    MB = bt.shape[1]
    if pairs is None:
        pa, n, out = None, B * H, np.zeros((B, H, D), np.float64)
    else:
        pa = np.ascontiguousarray(np.asarray(pairs, dtype=np.int64).reshape(-1, 2))
        n, out = pa.shape[0], np.zeros((pa.shape[0], D), np.float64)
    rc = _load().oracle_paged_decode(
        _ptr(qb), _ptr(kb), _ptr(vb), _ptr(bt), _ptr(sl), B, H, Hkv, D, S, NB, MB, float(scale),
        _DTYPE_CODE[dtype], None if pa is None else _ptr(pa), n, int(threads), _ptr(out))
    if rc:
        raise OracleError(f"oracle_paged_decode returned {rc}")
    return out


def partition_stats(q, k_cache, v_cache, block_tables, seq_lens, scale, partition, n_parts=None,
                    threads=0):
    """(m, l, acc) per (request, head, partition), fp64 natural-log units.

    m, l: [B, H, NP]; acc: [B, H, NP, D]; NP defaults to the most partitions any
    request needs. Partitions past a request's end hold (-inf, 0, 0).
    """
    B, H, D = q.shape
    NB, _, S, _ = k_cache.shape
    qb, kb, vb = _bits(q), _bits(k_cache), _bits(v_cache)
    bt = _i32(block_tables).reshape(B, -1)
    sl = _i32(seq_lens).reshape(B)
    if n_parts is None:
        n_parts = max(1, -(-int(sl.max(initial=0)) // partition))
    m = np.zeros((B, H, n_parts), np.float64)
    l = np.zeros((B, H, n_parts), np.float64)
    acc = np.zeros((B, H, n_parts, D), np.float64)
    rc = _load().oracle_partition_stats(
        _ptr(qb), _ptr(kb), _ptr(vb), _ptr(bt), _ptr(sl), B, H, D, S, NB, bt.shape[1],
        float(scale), _DTYPE_CODE[q.dtype], int(partition), int(n_parts), int(threads),
        _ptr(m), _ptr(l), _ptr(acc))
    if rc:
        raise OracleError(f"oracle_partition_stats returned {rc}")
    return m, l, acc


def paged_prefill(q, k_cache, v_cache, block_tables, seq_lens, q_start, scale, threads=0):
    """fp64 causal prefill attention over the paged cache ("vLLM KV Cache and
    PagedAttention Explained", Step 6 "Prefill"): q [T, H, D] holds the new tokens
    of every request (request i's rows q_start[i] .. q_start[i+1] - 1, the last
    q_start[i+1] - q_start[i] of its seq_lens[i] cached tokens); row j of request
    i attends to cache tokens 0 .. seq_lens[i] - n_i + j; query head h reads KV
    head h // (H // Hkv) of the [NB, Hkv, S, D] caches. Returns [T, H, D]."""
    T, H, D = q.shape
    NB, Hkv, S, D2 = k_cache.shape
    if D2 != D or H % Hkv:
        raise OracleError("shape mismatch")
    qb, kb, vb = _bits(q), _bits(k_cache), _bits(v_cache)
    sl = _i32(seq_lens).reshape(-1)
    B = sl.shape[0]
    bt = _i32(block_tables).reshape(B, -1)
    qs = _i32(q_start).reshape(B + 1)
    out = np.zeros((T, H, D), np.float64)
    rc = _load().oracle_paged_prefill(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(bt), _ptr(sl), _ptr(qs),
                                      B, H, Hkv, D, S, NB, bt.shape[1], float(scale),
                                      _DTYPE_CODE[q.dtype], int(threads), _ptr(out))
    if rc:
        raise OracleError(f"oracle_paged_prefill returned {rc}")
    return out
