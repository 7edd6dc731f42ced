"""The C-ABI library loads without a GPU, exports every symbol the header
declares, and rejects bad arguments on the host before launching anything."""

import ctypes
import os
import re

import pytest

from paged_kv_cache_driven_b200 import binding, build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return binding.lib()


def declared_functions():
    names = set()
    inc = os.path.join(ROOT, "include")
    for f in os.listdir(inc):
        if f.endswith(".h"):
            text = open(os.path.join(inc, f)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names |= set(re.findall(r"\b(pa_[a-z0-9_]+)\s*\(", text))
    return sorted(names)


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 18
    for n in names:
        assert hasattr(lib, n), n
    assert set(binding._SIGNATURES) >= set(names)


def test_version_and_status_strings(lib):
    assert lib.pa_version() == 100
    assert lib.pa_status_string(0) == b"PA_OK"
    assert lib.pa_status_string(2) == b"PA_ERR_OOM"


NULL = None
P = ctypes.c_void_p(16 * 1024)  # an aligned address the host checks never dereference


def decode_args(**kw):
    a = dict(out=P, out_dt=binding.PA_F32, q=P, k=P, v=P, bt=P, MB=8, sl=P, scale=0.1, B=2, H=4,
             D=128, S=16, NB=16, dt=binding.PA_BF16, partition=0, max_seq_len=100, ws=NULL,
             ws_bytes=0, stream=NULL)
    a.update(kw)
    return [a[k] for k in ("out", "out_dt", "q", "k", "v", "bt", "MB", "sl", "scale", "B", "H", "D",
                           "S", "NB", "dt", "partition", "max_seq_len", "ws", "ws_bytes", "stream")]


@pytest.mark.parametrize("bad", [
    dict(D=96), dict(D=512), dict(S=4), dict(S=64), dict(dt=binding.PA_F32), dict(out_dt=7),
    dict(q=NULL), dict(k=NULL), dict(out=NULL), dict(bt=NULL), dict(sl=NULL),
    dict(q=ctypes.c_void_p(16 * 1024 + 8)), dict(H=0), dict(B=-1), dict(MB=0),
    dict(partition=24), dict(partition=-2), dict(max_seq_len=8 * 16 + 1), dict(max_seq_len=-1),
    dict(scale=float("nan")), dict(scale=float("inf")), dict(B=70000),
    dict(max_seq_len=100, partition=16),  # needs a workspace, none given
])
def test_decode_rejects_bad_arguments_on_host(lib, bad):
    assert lib.pa_decode(*decode_args(**bad)) == binding.PA_ERR_INVALID


def test_decode_zero_batch_is_noop(lib):
    assert lib.pa_decode(*decode_args(B=0, q=NULL, out=NULL)) == binding.PA_OK


def test_workspace_and_plan(lib):
    assert binding.pa_decode_workspace_bytes(64, 40, 128, 16, 512) == 0
    assert binding.pa_decode_plan(64, 40, 128, 16, 512) == (0, 1)
    assert binding.pa_decode_plan(64, 40, 128, 16, 2048) == (512, 4)
    assert binding.pa_decode_plan(64, 40, 128, 16, 2048, partition=-1) == (0, 1)
    assert binding.pa_decode_plan(64, 40, 128, 16, 2048, partition=256) == (256, 8)
    # small grids: partitions halve while the grid has fewer CTAs than SMs (148
    # without a device); a count of 3, 5, 6 or 7 is then rounded to a power of
    # two (the next, else the previous) if the grid stays within 2 CTAs per SM:
    # one request of 1332 tokens on 32 heads -> 256 x 6 -> 176 x 8 (256 CTAs)
    assert binding.pa_decode_plan(1, 32, 128, 16, 1332) == (176, 8)
    # on 40 heads 8 partitions would be 320 CTAs: 4 of 336 tokens instead
    assert binding.pa_decode_plan(1, 40, 128, 16, 1332) == (336, 4)
    # 3 partitions of 64 -> 4 of 48 (S = 16)
    assert binding.pa_decode_plan(1, 32, 128, 16, 150) == (48, 4)
    assert binding.pa_decode_plan(2, 32, 128, 16, 280) == (80, 4)
    # 270 tokens in blocks of 32: 8 partitions of 64 tokens, the last three empty
    assert binding.pa_decode_plan(1, 1, 128, 32, 270) == (64, 8)
    # 1332 tokens in blocks of 32 on 32 heads: 8 of 192 (the eighth empty)
    assert binding.pa_decode_plan(1, 32, 128, 32, 1332) == (192, 8)
    assert binding.pa_decode_plan(1, 1, 128, 16, 8192) == (64, 128)
    # long contexts: up to 2048-token partitions while >= 8 CTAs per SM remain
    assert binding.pa_decode_plan(8, 32, 128, 16, 131072) == (2048, 64)
    assert binding.pa_decode_plan(2, 4, 128, 16, 40000) == (512, 79)  # too few CTAs to grow
    assert binding.pa_decode_plan(64, 40, 128, 16, 8192) == (512, 16)  # below 32K: 512
    assert binding.pa_decode_plan(1, 32, 128, 8, 100) == (64, 2)
    n = 64 * 40 * 4
    want = ((n * 8 + 255) // 256) * 256 + n * 128 * 4
    assert binding.pa_decode_workspace_bytes(64, 40, 128, 16, 2048) == want
    with pytest.raises(binding.PagedAttnError):
        binding.pa_decode_plan(1, 1, 128, 16, 100, partition=20)


def test_grouped_plan(lib):
    """Grouped-query heads: the partition pass has B * Hkv * ceil(G / 16) CTAs
    per partition; a grid within 2 CTAs per SM (296 without a device) at 512
    tokens halves its partitions (down to 128) while it stays within that."""
    # 64 query heads on 8 KV heads: 8 CTAs per partition for one request
    assert binding.pa_decode_plan_grouped(1, 64, 8, 128, 16, 1332) == (128, 11)
    assert binding.pa_decode_plan_grouped(1, 64, 8, 128, 16, 4096) == (128, 32)
    assert binding.pa_decode_plan_grouped(4, 64, 8, 128, 16, 2048) == (256, 8)  # 512 CTAs at 128
    assert binding.pa_decode_plan_grouped(1, 64, 8, 128, 16, 100) == (0, 1)
    # blocks of 32 still halve to 128; 8 KV heads x 2 chunks (G = 32)
    assert binding.pa_decode_plan_grouped(1, 256, 8, 128, 32, 1332) == (128, 11)
    # larger grids, explicit partitions and Hkv == H take pa_decode_plan's choice
    assert binding.pa_decode_plan_grouped(64, 64, 8, 128, 16, 2048) == (512, 4)
    assert binding.pa_decode_plan_grouped(1, 64, 8, 128, 16, 1332, partition=64) == (64, 21)
    assert binding.pa_decode_plan_grouped(1, 32, 32, 128, 16, 1332) == \
        binding.pa_decode_plan(1, 32, 128, 16, 1332)
    for bad in ((1, 64, 0), (1, 64, 7), (1, 0, 1)):
        with pytest.raises(binding.PagedAttnError):
            binding.pa_decode_plan_grouped(*bad, 128, 16, 1332)
    # the workspace covers the grouped plan of every Hkv (H = 64: at most 11
    # partitions of 1332 tokens; the one-head-per-KV-head plan has 4)
    assert binding.pa_decode_plan(1, 64, 128, 16, 1332)[1] == 4
    n = 1 * 64 * 11
    want = ((n * 8 + 255) // 256) * 256 + n * 128 * 4
    assert binding.pa_decode_workspace_bytes(1, 64, 128, 16, 1332) == want


def append_args(**kw):
    a = dict(k=P, v=P, slots=P, kc=P, vc=P, T=4, H=2, D=64, S=16, NB=8, dt=binding.PA_F16,
             stream=NULL)
    a.update(kw)
    return [a[k] for k in ("k", "v", "slots", "kc", "vc", "T", "H", "D", "S", "NB", "dt", "stream")]


@pytest.mark.parametrize("bad", [
    dict(D=60), dict(T=-1), dict(H=0), dict(S=0), dict(dt=binding.PA_F32), dict(k=NULL),
    dict(slots=NULL), dict(kc=ctypes.c_void_p(16 * 1024 + 2)),
])
def test_append_rejects_bad_arguments_on_host(lib, bad):
    assert lib.pa_kv_append(*append_args(**bad)) == binding.PA_ERR_INVALID


def test_append_zero_tokens_is_noop(lib):
    assert lib.pa_kv_append(*append_args(T=0, k=NULL, v=NULL)) == binding.PA_OK


def test_stepper_rejects_bad_arguments_on_host(lib):
    h = ctypes.c_void_p()
    a = binding.BlockAllocator(8, 16)
    base = [a._h, P, P, 4, 2, 64, 16, 8, 8, binding.PA_BF16, binding.PA_F32, 0.1, 100, 0, 1, 2,
            NULL, ctypes.byref(h)]
    for idx, bad in [(0, NULL), (1, NULL), (3, 0), (9, binding.PA_F32), (10, 9), (12, 8 * 16 + 1),
                     (15, 0), (15, 9), (13, 24)]:
        args = list(base)
        args[idx] = bad
        assert lib.pa_stepper_create(*args) == binding.PA_ERR_INVALID, idx
    assert lib.pa_stepper_step(NULL, P, P, NULL, NULL) == binding.PA_ERR_INVALID
    assert lib.pa_stepper_output(NULL, 0, ctypes.byref(h)) == binding.PA_ERR_INVALID


def prefill_args(**kw):
    a = dict(out=P, out_dt=binding.PA_F32, q=P, k=P, v=P, bt=P, MB=8, sl=P, qs=P, scale=0.1, B=2,
             H=4, Hkv=4, D=128, S=16, NB=16, dt=binding.PA_BF16, T=100, max_q_len=64, stream=NULL)
    a.update(kw)
    return [a[k] for k in ("out", "out_dt", "q", "k", "v", "bt", "MB", "sl", "qs", "scale", "B",
                           "H", "Hkv", "D", "S", "NB", "dt", "T", "max_q_len", "stream")]


@pytest.mark.parametrize("bad", [
    dict(D=96), dict(D=512), dict(S=4), dict(S=256), dict(dt=binding.PA_F32), dict(out_dt=9),
    dict(scale=0.0), dict(scale=-1.0), dict(scale=float("nan")), dict(Hkv=3), dict(Hkv=0),
    dict(q=NULL), dict(qs=NULL), dict(bt=NULL), dict(out=ctypes.c_void_p(16 * 1024 + 4)),
    dict(NB=0), dict(NB=1 << 28), dict(T=-1), dict(max_q_len=-1), dict(B=-1), dict(B=65536),
    dict(max_q_len=65535 * 128 + 1),
])
def test_prefill_rejects_bad_arguments_on_host(lib, bad):
    assert lib.pa_prefill(*prefill_args(**bad)) == binding.PA_ERR_INVALID


def test_prefill_nothing_to_do_is_noop(lib):
    for kw in (dict(B=0), dict(T=0), dict(max_q_len=0)):
        assert lib.pa_prefill(*prefill_args(q=NULL, out=NULL, **kw)) == binding.PA_OK


def fp8_decode_args(**kw):
    a = dict(out=P, out_dt=binding.PA_F32, q=P, q_dt=binding.PA_BF16, k=P, v=P, ks=0.05, vs=0.08,
             bt=P, MB=8, sl=P, scale=0.1, B=2, H=4, D=128, S=16, NB=16, partition=0,
             max_seq_len=100, ws=NULL, ws_bytes=0, stream=NULL)
    a.update(kw)
    return [a[k] for k in ("out", "out_dt", "q", "q_dt", "k", "v", "ks", "vs", "bt", "MB", "sl",
                           "scale", "B", "H", "D", "S", "NB", "partition", "max_seq_len", "ws",
                           "ws_bytes", "stream")]


@pytest.mark.parametrize("bad", [
    dict(ks=0.0), dict(vs=-1.0), dict(ks=float("inf")), dict(vs=float("nan")), dict(D=96),
    dict(q_dt=binding.PA_F32), dict(S=4), dict(k=NULL), dict(q=ctypes.c_void_p(16 * 1024 + 8)),
    dict(max_seq_len=100, partition=16),  # needs a workspace, none given
])
def test_decode_fp8_rejects_bad_arguments_on_host(lib, bad):
    assert lib.pa_decode_fp8(*fp8_decode_args(**bad)) == binding.PA_ERR_INVALID


def test_decode_fp8_zero_batch_is_noop(lib):
    assert lib.pa_decode_fp8(*fp8_decode_args(B=0, q=NULL, out=NULL)) == binding.PA_OK


def fp8_gqa_args(Hkv=2, **kw):
    a = fp8_decode_args(**kw)
    return a[:14] + [Hkv] + a[14:]  # Hkv after H


@pytest.mark.parametrize("bad", [
    dict(Hkv=3), dict(Hkv=0), dict(Hkv=8), dict(ks=0.0), dict(D=96), dict(k=NULL),
    dict(q_dt=binding.PA_F32), dict(max_seq_len=100, partition=16),
])
def test_decode_gqa_fp8_rejects_bad_arguments_on_host(lib, bad):
    assert lib.pa_decode_gqa_fp8(*fp8_gqa_args(**bad)) == binding.PA_ERR_INVALID


def test_decode_gqa_fp8_zero_batch_is_noop(lib):
    assert lib.pa_decode_gqa_fp8(*fp8_gqa_args(B=0, q=NULL, out=NULL)) == binding.PA_OK


def fp8_decode_append_args(kn=P, vn=P, **kw):
    a = fp8_decode_args(**kw)
    return a[:4] + [kn, vn] + a[4:]  # k_new, v_new after q_dt


@pytest.mark.parametrize("bad", [
    dict(kn=NULL), dict(vn=NULL), dict(kn=ctypes.c_void_p(16 * 1024 + 8)),
    dict(vn=ctypes.c_void_p(16 * 1024 + 2)), dict(ks=0.0), dict(D=96), dict(k=NULL),
    dict(q_dt=binding.PA_F32), dict(max_seq_len=100, partition=16),
])
def test_decode_append_fp8_rejects_bad_arguments_on_host(lib, bad):
    assert lib.pa_decode_append_fp8(*fp8_decode_append_args(**bad)) == binding.PA_ERR_INVALID


def test_decode_append_fp8_zero_batch_is_noop(lib):
    args = fp8_decode_append_args(kn=NULL, vn=NULL, B=0, q=NULL, out=NULL)
    assert lib.pa_decode_append_fp8(*args) == binding.PA_OK


def fp8_append_args(**kw):
    a = dict(k=P, v=P, in_dt=binding.PA_BF16, slots=P, kc=P, vc=P, ks=0.05, vs=0.08, T=4, H=2,
             D=64, S=16, NB=8, stream=NULL)
    a.update(kw)
    return [a[k] for k in ("k", "v", "in_dt", "slots", "kc", "vc", "ks", "vs", "T", "H", "D", "S",
                           "NB", "stream")]


@pytest.mark.parametrize("bad", [
    dict(D=8), dict(D=72), dict(ks=0.0), dict(vs=float("nan")), dict(in_dt=binding.PA_F32),
    dict(T=-1), dict(slots=NULL), dict(kc=ctypes.c_void_p(16 * 1024 + 8)),
])
def test_append_fp8_rejects_bad_arguments_on_host(lib, bad):
    assert lib.pa_kv_append_fp8(*fp8_append_args(**bad)) == binding.PA_ERR_INVALID


def test_append_fp8_zero_tokens_is_noop(lib):
    assert lib.pa_kv_append_fp8(*fp8_append_args(T=0, k=NULL, v=NULL)) == binding.PA_OK


def test_gqa_rejects_heads_not_a_multiple(lib):
    args = decode_args(H=6)
    # pa_decode_gqa(out, out_dt, q, k_new, v_new, k_cache, v_cache, bt, MB, sl, scale, B, H, Hkv,
    #               D, S, NB, dt, partition, max_seq_len, ws, ws_bytes, stream)
    out, out_dt, q, k, v, bt, MB, sl, scale, B, H, D, S, NB, dt, part, msl, ws, wsb, st = args
    assert lib.pa_decode_gqa(out, out_dt, q, NULL, NULL, k, v, bt, MB, sl, scale, B, H, 4, D, S,
                             NB, dt, part, msl, ws, wsb, st) == binding.PA_ERR_INVALID


def noalloc_args(**kw):
    """pa_decode_noalloc's arguments: pa_decode's without the workspace."""
    a = decode_args(**kw)
    return a[:17] + [a[19]]


@pytest.mark.parametrize("bad", [
    dict(D=96), dict(S=4), dict(dt=binding.PA_F32), dict(q=NULL), dict(out=NULL), dict(bt=NULL),
    dict(MB=0), dict(H=0), dict(B=70000), dict(partition=24), dict(scale=float("nan")),
    dict(max_seq_len=8 * 16 + 1),
    # bad arguments whose split would also be far larger than the static array:
    # the argument check comes first, so these are PA_ERR_INVALID, not PA_ERR_OOM
    dict(B=64, H=40, MB=8192, max_seq_len=8192 * 16 + 1, partition=512),
    dict(B=64, H=40, MB=8192, max_seq_len=131072, partition=512, q=NULL),
    dict(B=64, H=70000, MB=8192, max_seq_len=131072, partition=512),
])
def test_noalloc_rejects_bad_arguments_before_the_size_check(lib, bad):
    assert lib.pa_decode_noalloc(*noalloc_args(**bad)) == binding.PA_ERR_INVALID


def test_noalloc_size_check_and_exported_limit(lib):
    limit = binding.pa_noalloc_scratch_bytes()
    # the header's #define and the library agree
    text = open(os.path.join(ROOT, "include", "pagedattn.h")).read()
    m = re.search(r"#define PA_NOALLOC_SCRATCH_BYTES \((\d+)u << (\d+)\)", text)
    assert m and limit == int(m.group(1)) << int(m.group(2))
    # a valid call whose split needs more than the array is PA_ERR_OOM
    big = dict(B=64, H=40, MB=8192, max_seq_len=131072, partition=512)
    need = binding.pa_decode_workspace_bytes(64, 40, 128, 16, 131072, 512)
    assert need > limit
    assert lib.pa_decode_noalloc(*noalloc_args(**big)) == binding.PA_ERR_OOM
    assert lib.pa_decode_noalloc(*noalloc_args(B=0, q=NULL, out=NULL)) == binding.PA_OK


def test_grouped_plan_invariants(lib):
    """For a seeded spread of batch sizes, head groupings, block sizes and
    lengths: every plan covers the length in whole blocks, and the workspace
    pa_decode_workspace_bytes reports holds the partials of the grouped plan of
    any KV-head count (the entry points refuse a smaller one)."""
    import random
    rng = random.Random(7)
    D = 128
    for _ in range(400):
        B = rng.choice([1, 2, 3, 4, 8, 16, 33, 64, 200])
        H = rng.choice([1, 2, 8, 32, 40, 64, 128])
        divisors = [k for k in range(1, H + 1) if H % k == 0]
        Hkv = rng.choice(divisors)
        S = rng.choice([8, 16, 32])
        L = rng.choice([0, 1, 15, 100, 513, 1332, 2048, 4096, 40000, 131072])
        P, NP = binding.pa_decode_plan_grouped(B, H, Hkv, D, S, L)
        if NP == 1:
            assert P == 0
        else:
            # whole blocks, the length covered; a re-cut into a power of two
            # may leave the last one or two partitions without a token
            assert P % S == 0 and P >= 48 and P * NP >= L and NP - -(-L // P) <= 2
        n = B * H * NP
        need = 0 if NP == 1 else ((n * 8 + 255) // 256) * 256 + n * D * 4
        assert binding.pa_decode_workspace_bytes(B, H, D, S, L) >= need, (B, H, Hkv, S, L)
