"""ctypes binding of libpagedattn.so: argument marshalling only.

Every function has the name of the C entry point it calls (include/pagedattn.h)
and passes torch tensors' data pointers and the current torch CUDA stream; no
step of the path runs in Python. A missing library raises at load time: there
is no fallback.
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libpagedattn.so")

PA_OK, PA_ERR_INVALID, PA_ERR_OOM, PA_ERR_OUT_OF_RANGE, PA_ERR_CUDA = range(5)
PA_F16, PA_BF16, PA_F32 = range(3)
PA_DEVERR_BLOCK_ID, PA_DEVERR_SEQ_LEN, PA_DEVERR_SLOT, PA_DEVERR_TIMEOUT = 1, 2, 4, 8

_DT = {torch.float16: PA_F16, torch.bfloat16: PA_BF16, torch.float32: PA_F32}

_lib = None

_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
_SIGNATURES = {
    "pa_status_string": ([_i32], ctypes.c_char_p),
    "pa_version": ([], _i32),
    "pa_kv_append": ([_vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _vp], _i32),
    "pa_decode_workspace_bytes": ([_i32, _i32, _i32, _i32, _i32, _i32], _sz),
    "pa_decode_plan": ([_i32, _i32, _i32, _i32, _i32, _i32, _vp, _vp], _i32),
    "pa_decode_plan_grouped": ([_i32, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _vp], _i32),
    "pa_decode": ([_vp, _i32, _vp, _vp, _vp, _vp, _i32, _vp, ctypes.c_float, _i32, _i32, _i32,
                   _i32, _i32, _i32, _i32, _i32, _vp, _sz, _vp], _i32),
    "pa_get_device_error": ([_vp, _vp], _i32),
    "pa_check_slots": ([_vp, _i64, _i64, _vp], _i32),
    "pa_decode_append": ([_vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, ctypes.c_float, _i32,
                          _i32, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _sz, _vp], _i32),
    "pa_decode_gqa": ([_vp, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, ctypes.c_float, _i32,
                       _i32, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _sz, _vp], _i32),
    "pa_decode_noalloc": ([_vp, _i32, _vp, _vp, _vp, _vp, _i32, _vp, ctypes.c_float, _i32, _i32,
                           _i32, _i32, _i32, _i32, _i32, _i32, _vp], _i32),
    "pa_noalloc_scratch_bytes": ([], _sz),
    # k, v, in_dt, slot_mapping, k_cache, v_cache, k_scale, v_scale, T, H, D, S, NB, stream
    "pa_kv_append_fp8": ([_vp, _vp, _i32, _vp, _vp, _vp, ctypes.c_float, ctypes.c_float, _i32,
                          _i32, _i32, _i32, _i32, _vp], _i32),
    # out, out_dt, q, q_dt, k_cache, v_cache, k_scale, v_scale, block_tables, MB, seq_lens,
    # scale, B, H, D, S, NB, partition, max_seq_len, workspace, ws_bytes, stream
    "pa_decode_fp8": ([_vp, _i32, _vp, _i32, _vp, _vp, ctypes.c_float, ctypes.c_float, _vp, _i32,
                       _vp, ctypes.c_float, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _vp, _sz,
                       _vp], _i32),
    "pa_decode_gqa_fp8": ([_vp, _i32, _vp, _i32, _vp, _vp, ctypes.c_float, ctypes.c_float, _vp,
                           _i32, _vp, ctypes.c_float, _i32, _i32, _i32, _i32, _i32, _i32, _i32,
                           _i32, _vp, _sz, _vp], _i32),
    "pa_decode_append_fp8": ([_vp, _i32, _vp, _i32, _vp, _vp, _vp, _vp, ctypes.c_float,
                              ctypes.c_float, _vp, _i32, _vp, ctypes.c_float, _i32, _i32, _i32,
                              _i32, _i32, _i32, _i32, _vp, _sz, _vp], _i32),
    # out, out_dt, q, k_cache, v_cache, block_tables, MB, seq_lens, q_start, scale,
    # B, H, Hkv, D, S, NB, dt, T, max_q_len, stream
    "pa_prefill": ([_vp, _i32, _vp, _vp, _vp, _vp, _i32, _vp, _vp, ctypes.c_float, _i32, _i32,
                    _i32, _i32, _i32, _i32, _i32, _i32, _i32, _vp], _i32),
    "pa_stepper_create": ([_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _i32,
                           ctypes.c_float, _i32, _i32, _i32, _i32, _vp, _vp], _i32),
    "pa_stepper_destroy": ([_vp], None),
    "pa_stepper_step": ([_vp, _vp, _vp, _vp, _vp], _i32),
    "pa_stepper_output": ([_vp, _i64, _vp], _i32),
    "pa_stepper_drain": ([_vp], _i32),
    "pa_alloc_create": ([_i32, _i32, _vp, _vp], _i32),
    "pa_alloc_destroy": ([_vp], None),
    "pa_seq_grow": ([_vp, _i64, _i32], _i32),
    "pa_seq_free": ([_vp, _i64], _i32),
    "pa_seq_len": ([_vp, _i64, _vp], _i32),
    "pa_seq_block_table": ([_vp, _i64, _vp, _i32, _vp], _i32),
    "pa_build_slot_mapping": ([_vp, _vp, _vp, _vp, _i32, _vp], _i32),
    "pa_build_block_tables": ([_vp, _vp, _i32, _i32, _vp], _i32),
    "pa_prepare_step": ([_vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp], _i32),
    "pa_alloc_stats": ([_vp, _vp, _vp, _vp], _i32),
    "pa_seq_fork": ([_vp, _i64, _i64], _i32),
    "pa_alloc_take_copies": ([_vp, _vp, _i32, _vp], _i32),
    "pa_alloc_refcounts": ([_vp, _vp, _i32], _i32),
    "pa_copy_blocks": ([_vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _vp], _i32),
    "pa_alloc_dump": ([_vp, _vp, _i32, _vp], _i32),
}


class PagedAttnError(RuntimeError):
    def __init__(self, code, where):
        name = lib().pa_status_string(code).decode() if _lib is not None else str(code)
        super().__init__(f"{where}: {name}")
        self.code = code


def open_library(path):
    """Loads the library build at `path` with the C signatures declared here."""
    if not os.path.exists(path):
        raise ImportError(f"{path} is missing: run `python -m paged_kv_cache_driven_b200.build`")
    handle = ctypes.CDLL(path)
    for name, (args, res) in _SIGNATURES.items():
        fn = getattr(handle, name)
        fn.argtypes = args
        fn.restype = res
    return handle


def lib():
    """The loaded library (loaded on first use; raises if it was never built)."""
    global _lib
    if _lib is None:
        _lib = open_library(LIB_PATH)
    return _lib


def use_library(handle):
    """Makes `handle` (from open_library) the library the functions here call;
    returns the one it replaces (None if none was loaded yet)."""
    global _lib
    old, _lib = _lib, handle
    return old


def _check(rc, where):
    if rc != PA_OK:
        raise PagedAttnError(rc, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _cuda(t, name):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


# ---------------------------------------------------------------------------
# device entry points
# ---------------------------------------------------------------------------

def pa_kv_append(k, v, slot_mapping, k_cache, v_cache, stream=None):
    """Scatters k, v [T, H, D] into k_cache, v_cache [NB, H, S, D] at slot_mapping [T] (int64)."""
    for n, t in (("k", k), ("v", v), ("slot_mapping", slot_mapping), ("k_cache", k_cache),
                 ("v_cache", v_cache)):
        _cuda(t, n)
    if slot_mapping.dtype != torch.int64:
        raise ValueError("slot_mapping must be int64")
    if not (k.dtype == v.dtype == k_cache.dtype == v_cache.dtype):
        raise ValueError("k, v and the caches must share one dtype")
    T, H, D = k.shape
    NB, H2, S, D2 = k_cache.shape
    if (H2, D2) != (H, D) or v.shape != k.shape or v_cache.shape != k_cache.shape \
            or slot_mapping.shape != (T,):
        raise ValueError("shape mismatch")
    _check(lib().pa_kv_append(_ptr(k), _ptr(v), _ptr(slot_mapping), _ptr(k_cache), _ptr(v_cache),
                              T, H, D, S, NB, _DT[k.dtype], _stream(stream)), "pa_kv_append")


def pa_decode_workspace_bytes(B, H, D, S, max_seq_len, partition=0):
    return int(lib().pa_decode_workspace_bytes(B, H, D, S, max_seq_len, partition))


def pa_decode_plan(B, H, D, S, max_seq_len, partition=0):
    """(partition_tokens, num_partitions); (0, 1) = single pass."""
    P, NP = ctypes.c_int(), ctypes.c_int()
    _check(lib().pa_decode_plan(B, H, D, S, max_seq_len, partition, ctypes.byref(P),
                                ctypes.byref(NP)), "pa_decode_plan")
    return P.value, NP.value


def pa_decode_plan_grouped(B, H, Hkv, D, S, max_seq_len, partition=0):
    """The plan of pa_decode_gqa / pa_decode_gqa_fp8: (partition_tokens,
    num_partitions); (0, 1) = single pass."""
    P, NP = ctypes.c_int(), ctypes.c_int()
    _check(lib().pa_decode_plan_grouped(B, H, Hkv, D, S, max_seq_len, partition,
                                        ctypes.byref(P), ctypes.byref(NP)),
           "pa_decode_plan_grouped")
    return P.value, NP.value


def pa_decode(out, q, k_cache, v_cache, block_tables, seq_lens, scale, max_seq_len,
              partition=0, workspace=None, stream=None):
    """out [B, H, D] (fp32/fp16/bf16) = softmax(q K^T * scale) V through block tables.

    workspace: a CUDA uint8 tensor of at least pa_decode_workspace_bytes(...)
    bytes, or None when that size is 0.
    """
    for n, t in (("out", out), ("q", q), ("k_cache", k_cache), ("v_cache", v_cache),
                 ("block_tables", block_tables), ("seq_lens", seq_lens)):
        _cuda(t, n)
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("block_tables and seq_lens must be int32")
    B, H, D = q.shape
    NB, Hc, S, _ = k_cache.shape
    if Hc != H:
        raise ValueError("the cache has a different head count: use pa_decode_gqa")
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    if workspace is not None:
        _cuda(workspace, "workspace")
    _check(lib().pa_decode(_ptr(out), _DT[out.dtype], _ptr(q), _ptr(k_cache), _ptr(v_cache),
                           _ptr(block_tables), MB, _ptr(seq_lens), float(scale), B, H, D, S, NB,
                           _DT[q.dtype], int(partition), int(max_seq_len), _ptr(workspace),
                           ws_bytes, _stream(stream)), "pa_decode")


def pa_decode_append(out, q, k_new, v_new, k_cache, v_cache, block_tables, seq_lens, scale,
                     max_seq_len, partition=0, workspace=None, stream=None):
    """One decode step in one launch: writes k_new, v_new [B, H, D] at each
    request's last position (seq_lens[i] - 1), then decodes as pa_decode."""
    for n, t in (("out", out), ("q", q), ("k_new", k_new), ("v_new", v_new), ("k_cache", k_cache),
                 ("v_cache", v_cache), ("block_tables", block_tables), ("seq_lens", seq_lens)):
        _cuda(t, n)
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("block_tables and seq_lens must be int32")
    if k_new.shape != q.shape or v_new.shape != q.shape or k_new.dtype != q.dtype:
        raise ValueError("k_new, v_new must match q")
    B, H, D = q.shape
    NB, _, S, _ = k_cache.shape
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().pa_decode_append(_ptr(out), _DT[out.dtype], _ptr(q), _ptr(k_new), _ptr(v_new),
                                  _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), MB,
                                  _ptr(seq_lens), float(scale), B, H, D, S, NB, _DT[q.dtype],
                                  int(partition), int(max_seq_len), _ptr(workspace), ws_bytes,
                                  _stream(stream)), "pa_decode_append")


def pa_decode_gqa(out, q, k_cache, v_cache, block_tables, seq_lens, scale, max_seq_len,
                  k_new=None, v_new=None, partition=0, workspace=None, stream=None):
    """Grouped-query decode: q/out [B, H, D], caches [NB, Hkv, S, D] with H a
    multiple of Hkv; optional k_new, v_new [B, Hkv, D] appended first."""
    for n, t in (("out", out), ("q", q), ("k_cache", k_cache), ("v_cache", v_cache),
                 ("block_tables", block_tables), ("seq_lens", seq_lens)):
        _cuda(t, n)
    if (k_new is None) != (v_new is None):
        raise ValueError("k_new and v_new go together")
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("block_tables and seq_lens must be int32")
    B, H, D = q.shape
    NB, Hkv, S, _ = k_cache.shape
    if k_new is not None:
        _cuda(k_new, "k_new")
        _cuda(v_new, "v_new")
        if tuple(k_new.shape) != (B, Hkv, D) or tuple(v_new.shape) != (B, Hkv, D):
            raise ValueError("k_new, v_new must be [B, Hkv, D]")
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().pa_decode_gqa(_ptr(out), _DT[out.dtype], _ptr(q), _ptr(k_new), _ptr(v_new),
                               _ptr(k_cache), _ptr(v_cache), _ptr(block_tables), MB,
                               _ptr(seq_lens), float(scale), B, H, Hkv, D, S, NB, _DT[q.dtype],
                               int(partition), int(max_seq_len), _ptr(workspace), ws_bytes,
                               _stream(stream)), "pa_decode_gqa")


def pa_check_slots(slots, n_slots):
    """Host check of a slot mapping (a CPU int64 tensor): raises PagedAttnError
    (PA_ERR_OUT_OF_RANGE or PA_ERR_INVALID, with the offending index) if a slot
    is past n_slots or appears twice; negative slots are padding."""
    if slots.is_cuda or slots.dtype != torch.int64:
        raise ValueError("slots must be a CPU int64 tensor")
    s = slots.contiguous()
    bad = ctypes.c_int64(-1)
    st = lib().pa_check_slots(_ptr(s), s.numel(), int(n_slots), ctypes.byref(bad))
    if st != PA_OK:
        raise PagedAttnError(st, f"pa_check_slots: entry {bad.value}")


def pa_prefill(out, q, k_cache, v_cache, block_tables, seq_lens, q_start, scale, max_q_len,
               stream=None):
    """Causal paged prefill attention: q/out [T, H, D] packed by request
    (request i's rows q_start[i] .. q_start[i+1] - 1, the last of its seq_lens[i]
    cached tokens); caches [NB, Hkv, S, D]; q_start int32 [B + 1] on the device."""
    for n, t in (("out", out), ("q", q), ("k_cache", k_cache), ("v_cache", v_cache),
                 ("block_tables", block_tables), ("seq_lens", seq_lens), ("q_start", q_start)):
        _cuda(t, n)
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32 or \
            q_start.dtype != torch.int32:
        raise ValueError("block_tables, seq_lens and q_start must be int32")
    T, H, D = q.shape
    NB, Hkv, S, _ = k_cache.shape
    B = seq_lens.numel()
    if q_start.numel() != B + 1 or tuple(out.shape) != (T, H, D):
        raise ValueError("q_start must be [B + 1] and out [T, H, D]")
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    _check(lib().pa_prefill(_ptr(out), _DT[out.dtype], _ptr(q), _ptr(k_cache), _ptr(v_cache),
                            _ptr(block_tables), MB, _ptr(seq_lens), _ptr(q_start), float(scale),
                            B, H, Hkv, D, S, NB, _DT[q.dtype], T, int(max_q_len),
                            _stream(stream)), "pa_prefill")


def pa_kv_append_fp8(k, v, slot_mapping, k_cache, v_cache, k_scale, v_scale, stream=None):
    """Scatter k, v [T, H, D] (fp16/bf16) into uint8 E4M3 caches [NB, H, S, D]
    as codes of fp32(x / scale), round to nearest even, saturated at 448."""
    for n, t in (("k", k), ("v", v), ("slot_mapping", slot_mapping), ("k_cache", k_cache),
                 ("v_cache", v_cache)):
        _cuda(t, n)
    if k_cache.dtype != torch.uint8 or v_cache.dtype != torch.uint8:
        raise ValueError("E4M3 caches are uint8 tensors of codes")
    if slot_mapping.dtype != torch.int64:
        raise ValueError("slot_mapping must be int64")
    T, H, D = k.shape
    NB, H2, S, D2 = k_cache.shape
    if (H2, D2) != (H, D) or tuple(v.shape) != tuple(k.shape):
        raise ValueError("shape mismatch")
    _check(lib().pa_kv_append_fp8(_ptr(k), _ptr(v), _DT[k.dtype], _ptr(slot_mapping), _ptr(k_cache),
                                  _ptr(v_cache), float(k_scale), float(v_scale), T, H, D, S, NB,
                                  _stream(stream)), "pa_kv_append_fp8")


def pa_decode_fp8(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, seq_lens, scale,
                  max_seq_len, partition=0, workspace=None, stream=None):
    """Decode over uint8 E4M3 caches [NB, H, S, D] with per-tensor scales."""
    for n, t in (("out", out), ("q", q), ("k_cache", k_cache), ("v_cache", v_cache),
                 ("block_tables", block_tables), ("seq_lens", seq_lens)):
        _cuda(t, n)
    if k_cache.dtype != torch.uint8 or v_cache.dtype != torch.uint8:
        raise ValueError("E4M3 caches are uint8 tensors of codes")
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("block_tables and seq_lens must be int32")
    B, H, D = q.shape
    NB, H2, S, _ = k_cache.shape
    if H2 != H:
        raise ValueError("the E4M3 decode has one KV head per query head")
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().pa_decode_fp8(_ptr(out), _DT[out.dtype], _ptr(q), _DT[q.dtype], _ptr(k_cache),
                               _ptr(v_cache), float(k_scale), float(v_scale), _ptr(block_tables),
                               MB, _ptr(seq_lens), float(scale), B, H, D, S, NB, int(partition),
                               int(max_seq_len), _ptr(workspace), ws_bytes, _stream(stream)),
           "pa_decode_fp8")


def pa_decode_gqa_fp8(out, q, k_cache, v_cache, k_scale, v_scale, block_tables, seq_lens, scale,
                      max_seq_len, partition=0, workspace=None, stream=None):
    """Decode over uint8 E4M3 caches [NB, Hkv, S, D] for q [B, H, D] with H a
    multiple of Hkv (query head h reads KV head h // (H // Hkv))."""
    for n, t in (("out", out), ("q", q), ("k_cache", k_cache), ("v_cache", v_cache),
                 ("block_tables", block_tables), ("seq_lens", seq_lens)):
        _cuda(t, n)
    if k_cache.dtype != torch.uint8 or v_cache.dtype != torch.uint8:
        raise ValueError("E4M3 caches are uint8 tensors of codes")
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("block_tables and seq_lens must be int32")
    B, H, D = q.shape
    NB, Hkv, S, _ = k_cache.shape
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().pa_decode_gqa_fp8(_ptr(out), _DT[out.dtype], _ptr(q), _DT[q.dtype],
                                   _ptr(k_cache), _ptr(v_cache), float(k_scale), float(v_scale),
                                   _ptr(block_tables), MB, _ptr(seq_lens), float(scale), B, H, Hkv,
                                   D, S, NB, int(partition), int(max_seq_len), _ptr(workspace),
                                   ws_bytes, _stream(stream)), "pa_decode_gqa_fp8")


def pa_decode_append_fp8(out, q, k_new, v_new, k_cache, v_cache, k_scale, v_scale, block_tables,
                         seq_lens, scale, max_seq_len, partition=0, workspace=None, stream=None):
    """pa_kv_append_fp8 of k_new / v_new [B, H, D] at each request's last position,
    then pa_decode_fp8, in one launch (same bits as the two calls)."""
    for n, t in (("out", out), ("q", q), ("k_new", k_new), ("v_new", v_new),
                 ("k_cache", k_cache), ("v_cache", v_cache), ("block_tables", block_tables),
                 ("seq_lens", seq_lens)):
        _cuda(t, n)
    if k_cache.dtype != torch.uint8 or v_cache.dtype != torch.uint8:
        raise ValueError("E4M3 caches are uint8 tensors of codes")
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("block_tables and seq_lens must be int32")
    B, H, D = q.shape
    NB, H2, S, _ = k_cache.shape
    if H2 != H or tuple(k_new.shape) != (B, H, D) or tuple(v_new.shape) != (B, H, D):
        raise ValueError("k_new / v_new must be [B, H, D] with one KV head per query head")
    if k_new.dtype != q.dtype or v_new.dtype != q.dtype:
        raise ValueError("k_new / v_new must have q's dtype")
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib().pa_decode_append_fp8(
        _ptr(out), _DT[out.dtype], _ptr(q), _DT[q.dtype], _ptr(k_new), _ptr(v_new),
        _ptr(k_cache), _ptr(v_cache), float(k_scale), float(v_scale), _ptr(block_tables), MB,
        _ptr(seq_lens), float(scale), B, H, D, S, NB, int(partition), int(max_seq_len),
        _ptr(workspace), ws_bytes, _stream(stream)), "pa_decode_append_fp8")


def pa_decode_noalloc(out, q, k_cache, v_cache, block_tables, seq_lens, scale, max_seq_len,
                      partition=0, stream=None):
    """pa_decode without a workspace argument: for callers that cannot allocate
    device memory. The split-KV partials go to the library's static device array
    (PA_NOALLOC_SCRATCH_BYTES); a split that needs more raises PA_ERR_OOM."""
    for n, t in (("out", out), ("q", q), ("k_cache", k_cache), ("v_cache", v_cache),
                 ("block_tables", block_tables), ("seq_lens", seq_lens)):
        _cuda(t, n)
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("block_tables and seq_lens must be int32")
    B, H, D = q.shape
    NB, _, S, _ = k_cache.shape
    MB = block_tables.shape[1] if block_tables.dim() == 2 else 0
    _check(lib().pa_decode_noalloc(_ptr(out), _DT[out.dtype], _ptr(q), _ptr(k_cache),
                                   _ptr(v_cache), _ptr(block_tables), MB, _ptr(seq_lens),
                                   float(scale), B, H, D, S, NB, _DT[q.dtype], int(partition),
                                   int(max_seq_len), _stream(stream)), "pa_decode_noalloc")


def pa_noalloc_scratch_bytes():
    """Size of the library's static scratch array that pa_decode_noalloc uses."""
    return int(lib().pa_noalloc_scratch_bytes())


def pa_copy_blocks(k_cache, v_cache, src_dst, stream=None):
    """Copies physical blocks src -> dst (device int32 [n, 2]) in both caches."""
    for n, t in (("k_cache", k_cache), ("v_cache", v_cache), ("src_dst", src_dst)):
        _cuda(t, n)
    if src_dst.dtype != torch.int32:
        raise ValueError("src_dst must be int32")
    NB, H, S, D = k_cache.shape
    n = src_dst.shape[0] if src_dst.numel() else 0
    _check(lib().pa_copy_blocks(_ptr(k_cache), _ptr(v_cache), _ptr(src_dst), n, H, S, D, NB,
                                _DT[k_cache.dtype], _stream(stream)), "pa_copy_blocks")


def pa_get_device_error(stream=None):
    """Synchronises the stream, then reads and clears the device error word."""
    flags = ctypes.c_uint32()
    _check(lib().pa_get_device_error(_stream(stream), ctypes.byref(flags)), "pa_get_device_error")
    return flags.value


# ---------------------------------------------------------------------------
# host allocator
# ---------------------------------------------------------------------------

def _host_i64(seq):
    a = (ctypes.c_int64 * len(seq))(*[int(x) for x in seq])
    return a


def _host_i32(seq):
    return (ctypes.c_int * len(seq))(*[int(x) for x in seq])


class BlockAllocator:
    """The library's host block allocator (pa_alloc_*, pa_seq_*, pa_build_*)."""

    def __init__(self, num_blocks, block_size, initial_order=None):
        self.num_blocks, self.block_size = num_blocks, block_size
        handle = ctypes.c_void_p()
        order = None if initial_order is None else _host_i32(initial_order)
        _check(lib().pa_alloc_create(num_blocks, block_size, order, ctypes.byref(handle)),
               "pa_alloc_create")
        self._h = handle

    def close(self):
        if self._h:
            lib().pa_alloc_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def pa_seq_grow(self, seq_id, new_len):
        _check(lib().pa_seq_grow(self._h, int(seq_id), int(new_len)), "pa_seq_grow")

    def pa_seq_free(self, seq_id):
        _check(lib().pa_seq_free(self._h, int(seq_id)), "pa_seq_free")

    def pa_seq_len(self, seq_id):
        n = ctypes.c_int()
        _check(lib().pa_seq_len(self._h, int(seq_id), ctypes.byref(n)), "pa_seq_len")
        return n.value

    def pa_seq_block_table(self, seq_id):
        n = ctypes.c_int()
        cap = self.num_blocks
        buf = (ctypes.c_int32 * max(cap, 1))()
        _check(lib().pa_seq_block_table(self._h, int(seq_id), buf, cap, ctypes.byref(n)),
               "pa_seq_block_table")
        return list(buf[:n.value])

    def pa_build_slot_mapping(self, seq_ids, start_pos, n_tok, out=None):
        """int64 slots; writes into ``out`` (a CPU int64 tensor) when given."""
        total = sum(int(x) for x in n_tok)
        if out is None:
            out = torch.empty(total, dtype=torch.int64)
        _check(lib().pa_build_slot_mapping(self._h, _host_i64(seq_ids), _host_i32(start_pos),
                                           _host_i32(n_tok), len(seq_ids), _ptr(out)),
               "pa_build_slot_mapping")
        return out

    def pa_build_block_tables(self, seq_ids, max_blocks, out=None):
        if out is None:
            out = torch.empty((len(seq_ids), max_blocks), dtype=torch.int32)
        _check(lib().pa_build_block_tables(self._h, _host_i64(seq_ids), len(seq_ids), max_blocks,
                                           _ptr(out)), "pa_build_block_tables")
        return out

    def pa_prepare_step(self, seq_ids, n_new, max_blocks, slots=None, tables=None, lens=None):
        """Grows every sequence by n_new tokens and fills the given CPU tensors (pinned
        memory welcome): slots int64 [n*n_new], tables int32 [n, max_blocks], lens int32 [n]."""
        ids = seq_ids if isinstance(seq_ids, ctypes.Array) else _host_i64(seq_ids)
        _check(lib().pa_prepare_step(self._h, ids, len(ids), int(n_new), int(max_blocks),
                                     _ptr(slots), _ptr(tables), _ptr(lens)), "pa_prepare_step")

    def pa_alloc_stats(self):
        f, u, w = ctypes.c_int(), ctypes.c_int64(), ctypes.c_int64()
        _check(lib().pa_alloc_stats(self._h, ctypes.byref(f), ctypes.byref(u), ctypes.byref(w)),
               "pa_alloc_stats")
        return f.value, u.value, w.value

    def pa_seq_fork(self, parent, child):
        _check(lib().pa_seq_fork(self._h, int(parent), int(child)), "pa_seq_fork")

    def pa_alloc_take_copies(self):
        """The queued copy-on-write pairs as a CPU int32 tensor [n, 2] (queue cleared)."""
        n = ctypes.c_int()
        cap = self.num_blocks
        out = torch.empty((max(cap, 1), 2), dtype=torch.int32)
        _check(lib().pa_alloc_take_copies(self._h, _ptr(out), cap, ctypes.byref(n)),
               "pa_alloc_take_copies")
        return out[:n.value].clone()

    def pa_alloc_refcounts(self):
        out = torch.empty(max(self.num_blocks, 1), dtype=torch.int32)
        _check(lib().pa_alloc_refcounts(self._h, _ptr(out), self.num_blocks), "pa_alloc_refcounts")
        return out[:self.num_blocks].tolist()

    def pa_alloc_dump(self):
        n = ctypes.c_int()
        cap = self.num_blocks
        buf = (ctypes.c_int32 * max(cap, 1))()
        _check(lib().pa_alloc_dump(self._h, buf, cap, ctypes.byref(n)), "pa_alloc_dump")
        return list(buf[:n.value])
