"""FP8 E4M3 KV cache (a storage extension, not on the pages): pa_kv_append_fp8
bit for bit against the oracle's quantizer, and pa_decode_fp8 against the
oracle's decode over the same codes, at the decode tolerance, with NaN codes
poisoning every byte a request does not own; small cases element by element,
the LLaMA-2-13B decode shape on sampled pairs."""

import math

import numpy as np
import pytest
import torch

from helpers import MAX_ABS, REL_L2, assert_parity, sample_pairs
from oracle import fp8 as ofp8
from paged_kv_cache_driven_b200 import binding, workloads

pytestmark = pytest.mark.gpu
DEV = "cuda"
NAN_CODE = 0x7F


def fp8_case(lens, H, D, S, in_dt, seed, k_scale=0.05, v_scale=0.08):
    """A decode case whose caches are filled through pa_kv_append_fp8 from the
    16-bit case's K/V rows; unused bytes are NaN codes. Returns (case, kc8, vc8)."""
    case = workloads.decode_case(lens, H=H, D=D, S=S, dtype=in_dt, seed=seed, device=DEV,
                                 poison=False)
    NB = case.k_cache.shape[0]
    kc8 = torch.full((NB, H, S, D), NAN_CODE, dtype=torch.uint8, device=DEV)
    vc8 = torch.full_like(kc8, NAN_CODE)
    for i, L in enumerate(case.seq_lens_host):
        if L == 0:
            continue
        blocks = torch.tensor(case.tables_host[i], device=DEV)
        k = case.k_cache[blocks].permute(0, 2, 1, 3).reshape(-1, H, D)[:L].contiguous()
        v = case.v_cache[blocks].permute(0, 2, 1, 3).reshape(-1, H, D)[:L].contiguous()
        slots = (blocks.repeat_interleave(S) * S + torch.arange(S, device=DEV).repeat(len(blocks)))[:L]
        binding.pa_kv_append_fp8(k, v, slots.to(torch.int64), kc8, vc8, k_scale, v_scale)
    torch.cuda.synchronize()
    assert binding.pa_get_device_error() == 0
    return case, kc8, vc8


@pytest.mark.parametrize("in_dt", [torch.bfloat16, torch.float16])
def test_append_fp8_bit_exact(in_dt):
    g = torch.Generator().manual_seed(1)
    T, H, D, S, NB = 300, 4, 128, 16, 40
    k = (torch.randn(T, H, D, generator=g) * 3).to(in_dt)
    v = (torch.randn(T, H, D, generator=g) * 3).to(in_dt)
    k[0, 0, :4] = torch.tensor([500.0, -1e4, 0.0, -0.0]).to(in_dt)  # saturation and zeros
    slots = torch.randperm(NB * S, generator=g)[:T].to(torch.int64)
    slots[5] = -1  # padding: skipped
    kc8 = torch.full((NB, H, S, D), NAN_CODE, dtype=torch.uint8, device=DEV)
    vc8 = torch.full_like(kc8, NAN_CODE)
    binding.pa_kv_append_fp8(k.to(DEV), v.to(DEV), slots.to(DEV), kc8, vc8, 0.05, 0.08)
    torch.cuda.synchronize()
    assert binding.pa_get_device_error() == 0
    want_k = np.full((NB, H, S, D), NAN_CODE, np.uint8)
    want_v = want_k.copy()
    kq = ofp8.quantize(k.float().numpy(), 0.05)
    vq = ofp8.quantize(v.float().numpy(), 0.08)
    for t, s in enumerate(slots.tolist()):
        if s >= 0:
            want_k[s // S, :, s % S, :] = kq[t]
            want_v[s // S, :, s % S, :] = vq[t]
    assert np.array_equal(kc8.cpu().numpy(), want_k)
    assert np.array_equal(vc8.cpu().numpy(), want_v)
    # a slot past the pool is flagged and skipped
    bad = torch.tensor([NB * S + 3], dtype=torch.int64, device=DEV)
    binding.pa_kv_append_fp8(k[:1].to(DEV), v[:1].to(DEV), bad, kc8, vc8, 0.05, 0.08)
    assert binding.pa_get_device_error() & binding.PA_DEVERR_SLOT


def run_fp8(case, kc8, vc8, out_dt=torch.float32, partition=0, k_scale=0.05, v_scale=0.08):
    B, H, D = case.q.shape
    S = kc8.shape[2]
    maxlen = max(case.seq_lens_host + [0])
    out = torch.empty((B, H, D), dtype=out_dt, device=DEV)
    wsb = binding.pa_decode_workspace_bytes(B, H, D, S, maxlen, partition)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=DEV)
    binding.pa_decode_fp8(out, case.q, kc8, vc8, k_scale, v_scale, case.block_tables,
                          case.seq_lens, case.scale, maxlen, partition=partition, workspace=ws)
    torch.cuda.synchronize()
    assert binding.pa_get_device_error() == 0
    return out


@pytest.mark.parametrize("D,S", [(64, 8), (64, 16), (64, 32), (128, 8), (128, 16), (128, 32),
                                 (256, 8), (256, 16), (256, 32)])
@pytest.mark.parametrize("partition", [0, -1])
def test_decode_fp8_small(D, S, partition):
    lens = [0, 1, S - 1, S, 3 * S + 5, 700]
    case, kc8, vc8 = fp8_case(lens, H=3, D=D, S=S, in_dt=torch.bfloat16, seed=D + S)
    out = run_fp8(case, kc8, vc8, partition=partition)
    want = ofp8.paged_decode_fp8(case.q.cpu(), kc8.cpu(), vc8.cpu(), 0.05, 0.08,
                                 case.block_tables.cpu(), case.seq_lens.cpu(), case.scale)
    assert_parity(out.cpu().numpy(), want, f"fp8 D={D} S={S} p={partition}")
    assert np.all(out[0].cpu().numpy() == 0)  # L = 0


@pytest.mark.parametrize("q_dt,out_dt", [(torch.float16, torch.float16),
                                         (torch.bfloat16, torch.bfloat16)])
def test_decode_fp8_dtypes(q_dt, out_dt):
    case, kc8, vc8 = fp8_case([50, 333, 1000], H=4, D=128, S=16, in_dt=q_dt, seed=3)
    out = run_fp8(case, kc8, vc8, out_dt=out_dt)
    want = ofp8.paged_decode_fp8(case.q.cpu(), kc8.cpu(), vc8.cpu(), 0.05, 0.08,
                                 case.block_tables.cpu(), case.seq_lens.cpu(), case.scale)
    got = out.float().cpu().numpy()
    ulp = 2.0 ** -8 if out_dt == torch.bfloat16 else 2.0 ** -11
    assert np.abs(got - want).max() <= MAX_ABS + ulp * np.abs(want).max()


def test_decode_fp8_llama13b_shape_sampled():
    """40 heads, head_dim 128, block 16, batch 64, L ~ U[1, 2048]: the bench's
    decode shape with an E4M3 cache, in its launch configuration."""
    lens = workloads.uniform_lengths(64, 1, 2048, 0)
    case, kc8, vc8 = fp8_case(lens, H=40, D=128, S=16, in_dt=torch.bfloat16, seed=0)
    out = run_fp8(case, kc8, vc8)
    pairs = sample_pairs(case, 24)
    # the oracle on the sampled (request, head) pairs: a one-head sub-problem each
    qs, ks, vs, tabs, Ls = [], [], [], [], []
    off = 0
    for i, h in pairs:
        L = case.seq_lens_host[i]
        blocks = torch.tensor(case.tables_host[i], device=DEV)
        ks.append(kc8[blocks, h].unsqueeze(1).cpu())
        vs.append(vc8[blocks, h].unsqueeze(1).cpu())
        qs.append(case.q[i, h].view(1, 1, -1).cpu())
        tabs.append(list(range(off, off + len(blocks))))
        Ls.append(L)
        off += len(blocks)
    MB = max(len(t) for t in tabs)
    bt = torch.full((len(pairs), MB), -1, dtype=torch.int32)
    for r, t in enumerate(tabs):
        bt[r, :len(t)] = torch.tensor(t, dtype=torch.int32)
    want = ofp8.paged_decode_fp8(torch.cat(qs), torch.cat(ks), torch.cat(vs), 0.05, 0.08, bt,
                                 torch.tensor(Ls, dtype=torch.int32), case.scale)[:, 0]
    got = torch.stack([out[i, h] for i, h in pairs]).cpu().numpy()
    assert_parity(got, want, "fp8 13B shape")
    assert bool(torch.isfinite(out).all())


@pytest.mark.parametrize("D", [128, 256])
@pytest.mark.parametrize("q_mag", [1e-3, 1.0, 3e3])
def test_decode_fp8_query_magnitude(D, q_mag):
    """Tiny, unit and large queries all match the oracle (a 3e3 query times
    codes up to 448 would overflow an f16 product), including a split into
    32-token partitions."""
    lens = [5, 40, 333]
    case, kc8, vc8 = fp8_case(lens, H=2, D=D, S=16, in_dt=torch.bfloat16, seed=7)
    case.q.mul_(q_mag)
    for partition in (0, 32):
        out = run_fp8(case, kc8, vc8, partition=partition)
        want = ofp8.paged_decode_fp8(case.q.cpu(), kc8.cpu(), vc8.cpu(), 0.05, 0.08,
                                     case.block_tables.cpu(), case.seq_lens.cpu(), case.scale)
        assert_parity(out.cpu().numpy(), want, f"fp8 D={D} |q|~{q_mag} p={partition}")


def test_decode_fp8_bad_block_id_is_skipped_and_flagged():
    """A table entry outside the pool is never loaded: the kernel flags it and
    leaves that block's tokens out; the other requests are unaffected."""
    case, kc8, vc8 = fp8_case([64, 48], H=2, D=128, S=16, in_dt=torch.bfloat16, seed=9)
    want = ofp8.paged_decode_fp8(case.q.cpu(), kc8.cpu(), vc8.cpu(), 0.05, 0.08,
                                 case.block_tables.cpu(), case.seq_lens.cpu(), case.scale)
    bt = case.block_tables.clone()
    bt[0, 1] = kc8.shape[0] + 7
    B, H, D = case.q.shape
    out = torch.empty((B, H, D), dtype=torch.float32, device=DEV)
    binding.pa_decode_fp8(out, case.q, kc8, vc8, 0.05, 0.08, bt, case.seq_lens, case.scale, 64,
                          partition=-1)
    assert binding.pa_get_device_error() & binding.PA_DEVERR_BLOCK_ID
    assert_parity(out[1:].cpu().numpy(), want[1:], "fp8 neighbour of a bad id")
    assert bool(torch.isfinite(out[0]).all())


@pytest.mark.parametrize("lens,H,D,S,in_dt,out_dt,partition", [
    ([0, 1, 17, 300, 1000], 3, 128, 16, torch.bfloat16, torch.float32, 0),
    ([0, 1, 17, 300, 1000], 3, 128, 16, torch.bfloat16, torch.float32, -1),
    ([5, 64, 333], 2, 64, 8, torch.float16, torch.bfloat16, 32),
    ([7, 129, 700], 2, 256, 32, torch.bfloat16, torch.float16, 64),
    ([1332], 32, 128, 16, torch.bfloat16, torch.float32, 0),  # a cluster plan: 8 x 176 tokens
    # large grids (more than two CTAs per SM): the half-width CTAs of small units
    ([(37 * i) % 600 + 1 for i in range(24)], 8, 128, 16, torch.bfloat16, torch.float32, 64),
    ([(53 * i) % 500 + 1 for i in range(24)], 4, 64, 8, torch.float16, torch.float32, 32),
])
def test_decode_append_fp8_equals_two_calls(lens, H, D, S, in_dt, out_dt, partition):
    """pa_decode_append_fp8 quantizes each request's new row into its last slot
    inside the decode launch: the same cache bytes as pa_kv_append_fp8 (and as
    the oracle's quantizer), the same output bits as pa_kv_append_fp8 followed
    by pa_decode_fp8, and the oracle's decode of those codes."""
    case, kc8, vc8 = fp8_case(lens, H=H, D=D, S=S, in_dt=in_dt, seed=sum(lens) + D)
    B = len(lens)
    g = torch.Generator(device=DEV).manual_seed(D + S)
    k_new = (torch.randn((B, H, D), generator=g, device=DEV) * 4).to(in_dt)
    v_new = (torch.randn((B, H, D), generator=g, device=DEV) * 4).to(in_dt)
    k_new[-1, 0, :3] = torch.tensor([1e4, -1e4, 0.0], device=DEV).to(in_dt)  # saturation
    slots = torch.tensor([case.tables_host[i][(L - 1) // S] * S + (L - 1) % S if L > 0 else -1
                          for i, L in enumerate(lens)], dtype=torch.int64, device=DEV)
    kc_a, vc_a = kc8.clone(), vc8.clone()
    binding.pa_kv_append_fp8(k_new, v_new, slots, kc_a, vc_a, 0.05, 0.08)
    out_a = run_fp8(case, kc_a, vc_a, out_dt=out_dt, partition=partition)
    kc_b, vc_b = kc8.clone(), vc8.clone()
    maxlen = max(lens)
    out_b = torch.empty((B, H, D), dtype=out_dt, device=DEV)
    wsb = binding.pa_decode_workspace_bytes(B, H, D, S, maxlen, partition)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=DEV)
    binding.pa_decode_append_fp8(out_b, case.q, k_new, v_new, kc_b, vc_b, 0.05, 0.08,
                                 case.block_tables, case.seq_lens, case.scale, maxlen,
                                 partition=partition, workspace=ws)
    torch.cuda.synchronize()
    assert binding.pa_get_device_error() == 0
    assert torch.equal(kc_a, kc_b) and torch.equal(vc_a, vc_b), "cache bytes differ"
    bits = torch.int32 if out_dt == torch.float32 else torch.int16
    assert torch.equal(out_a.view(bits), out_b.view(bits)), "output bits differ"
    # the appended codes are the oracle quantizer's
    kq = ofp8.quantize(k_new.float().cpu().numpy(), 0.05)
    vq = ofp8.quantize(v_new.float().cpu().numpy(), 0.08)
    kcb, vcb = kc_b.cpu().numpy(), vc_b.cpu().numpy()
    for i, s in enumerate(slots.tolist()):
        if s >= 0:
            assert np.array_equal(kcb[s // S, :, s % S, :], kq[i])
            assert np.array_equal(vcb[s // S, :, s % S, :], vq[i])
    if out_dt == torch.float32:
        want = ofp8.paged_decode_fp8(case.q.cpu(), kc_b.cpu(), vc_b.cpu(), 0.05, 0.08,
                                     case.block_tables.cpu(), case.seq_lens.cpu(), case.scale)
        assert_parity(out_b.cpu().numpy(), want, f"fused fp8 append {lens} D={D}")


def fp8_gqa_case(lens, H, Hkv, D, S, in_dt, seed, k_scale=0.05, v_scale=0.08):
    """fp8_case with Hkv KV heads in the caches ([NB, Hkv, S, D]) and H query heads."""
    case = workloads.decode_case(lens, H=H, D=D, S=S, dtype=in_dt, seed=seed, device=DEV,
                                 poison=False, Hkv=Hkv)
    NB = case.k_cache.shape[0]
    kc8 = torch.full((NB, Hkv, S, D), NAN_CODE, dtype=torch.uint8, device=DEV)
    vc8 = torch.full_like(kc8, NAN_CODE)
    for i, L in enumerate(case.seq_lens_host):
        if L == 0:
            continue
        blocks = torch.tensor(case.tables_host[i], device=DEV)
        k = case.k_cache[blocks].permute(0, 2, 1, 3).reshape(-1, Hkv, D)[:L].contiguous()
        v = case.v_cache[blocks].permute(0, 2, 1, 3).reshape(-1, Hkv, D)[:L].contiguous()
        slots = (blocks.repeat_interleave(S) * S + torch.arange(S, device=DEV).repeat(len(blocks)))[:L]
        binding.pa_kv_append_fp8(k, v, slots.to(torch.int64), kc8, vc8, k_scale, v_scale)
    torch.cuda.synchronize()
    assert binding.pa_get_device_error() == 0
    return case, kc8, vc8


def run_gqa_fp8(case, kc8, vc8, out_dt=torch.float32, partition=0):
    B, H, D = case.q.shape
    S = kc8.shape[2]
    maxlen = max(case.seq_lens_host + [0])
    out = torch.empty((B, H, D), dtype=out_dt, device=DEV)
    wsb = binding.pa_decode_workspace_bytes(B, H, D, S, maxlen, partition)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=DEV)
    binding.pa_decode_gqa_fp8(out, case.q, kc8, vc8, 0.05, 0.08, case.block_tables,
                              case.seq_lens, case.scale, maxlen, partition=partition, workspace=ws)
    torch.cuda.synchronize()
    assert binding.pa_get_device_error() == 0
    return out


@pytest.mark.parametrize("G,D,S,in_dt,partition", [
    (8, 128, 16, torch.bfloat16, 0), (8, 128, 16, torch.bfloat16, 64),
    (2, 64, 8, torch.float16, -1), (4, 256, 32, torch.bfloat16, 64),
    (16, 128, 16, torch.float16, 0), (3, 128, 8, torch.bfloat16, 32),
    (8, 64, 32, torch.bfloat16, 0), (12, 256, 16, torch.float16, 0),
])
def test_decode_gqa_fp8(G, D, S, in_dt, partition):
    """Grouped-query heads over E4M3 caches (tensor cores, f16 products) against
    the oracle's decode over the same codes, every output element."""
    lens = [0, 1, S - 1, 16, 17, 300, 1000]
    Hkv = 2
    case, kc8, vc8 = fp8_gqa_case(lens, H=G * Hkv, Hkv=Hkv, D=D, S=S, in_dt=in_dt, seed=G + D + S)
    out = run_gqa_fp8(case, kc8, vc8, partition=partition)
    want = ofp8.paged_decode_fp8(case.q.cpu(), kc8.cpu(), vc8.cpu(), 0.05, 0.08,
                                 case.block_tables.cpu(), case.seq_lens.cpu(), case.scale)
    assert_parity(out.cpu().numpy(), want, f"fp8 gqa G={G} D={D} S={S} p={partition}")
    assert np.all(out[0].cpu().numpy() == 0)  # L = 0


@pytest.mark.parametrize("q_mag", [1e-3, 3e3])
def test_decode_gqa_fp8_query_magnitude(q_mag):
    """Each query head is scaled into f16 by its own power of two: tiny and large
    queries (and heads of different magnitudes in one group) match the oracle."""
    case, kc8, vc8 = fp8_gqa_case([5, 40, 333], H=16, Hkv=2, D=128, S=16,
                                  in_dt=torch.bfloat16, seed=11)
    case.q.mul_(q_mag)
    case.q[:, 1::2].mul_(64.0)  # neighbouring heads four orders of magnitude apart
    for out_dt in (torch.float32, torch.bfloat16):
        out = run_gqa_fp8(case, kc8, vc8, out_dt=out_dt)
        want = ofp8.paged_decode_fp8(case.q.cpu(), kc8.cpu(), vc8.cpu(), 0.05, 0.08,
                                     case.block_tables.cpu(), case.seq_lens.cpu(), case.scale)
        got = out.float().cpu().numpy()
        if out_dt == torch.float32:
            assert_parity(got, want, f"fp8 gqa |q|~{q_mag}")
        else:
            assert np.abs(got - want).max() <= MAX_ABS + 2.0 ** -8 * np.abs(want).max()


def test_decode_gqa_fp8_one_group_is_decode_fp8():
    """Hkv == H goes to pa_decode_fp8: the same bits."""
    case, kc8, vc8 = fp8_case([7, 300, 999], H=4, D=128, S=16, in_dt=torch.bfloat16, seed=5)
    a = run_fp8(case, kc8, vc8)
    b = run_gqa_fp8(case, kc8, vc8)
    assert torch.equal(a.view(torch.int32), b.view(torch.int32))


def test_decode_gqa_fp8_llama70b_shape_sampled():
    """64 query heads on 8 KV heads, head_dim 128, block 16, batch 64, L ~ U[1, 2048]
    over an E4M3 cache, in the automatic plan, on sampled (request, head) pairs."""
    lens = workloads.uniform_lengths(64, 1, 2048, 0)
    case, kc8, vc8 = fp8_gqa_case(lens, H=64, Hkv=8, D=128, S=16, in_dt=torch.bfloat16, seed=0)
    out = run_gqa_fp8(case, kc8, vc8)
    pairs = sample_pairs(case, 24)
    G = 8
    qs, ks, vs, tabs, Ls = [], [], [], [], []
    off = 0
    for i, h in pairs:
        blocks = torch.tensor(case.tables_host[i], device=DEV)
        ks.append(kc8[blocks, h // G].unsqueeze(1).cpu())
        vs.append(vc8[blocks, h // G].unsqueeze(1).cpu())
        qs.append(case.q[i, h].view(1, 1, -1).cpu())
        tabs.append(list(range(off, off + len(blocks))))
        Ls.append(case.seq_lens_host[i])
        off += len(blocks)
    MB = max(len(t) for t in tabs)
    bt = torch.full((len(pairs), MB), -1, dtype=torch.int32)
    for r, t in enumerate(tabs):
        bt[r, :len(t)] = torch.tensor(t, dtype=torch.int32)
    want = ofp8.paged_decode_fp8(torch.cat(qs), torch.cat(ks), torch.cat(vs), 0.05, 0.08, bt,
                                 torch.tensor(Ls, dtype=torch.int32), case.scale)[:, 0]
    got = torch.stack([out[i, h] for i, h in pairs]).cpu().numpy()
    assert_parity(got, want, "fp8 70B shape")
    assert bool(torch.isfinite(out).all())


def test_decode_gqa_fp8_bad_block_id_is_skipped_and_flagged():
    case, kc8, vc8 = fp8_gqa_case([64, 48], H=8, Hkv=2, D=128, S=16, in_dt=torch.bfloat16,
                                  seed=9)
    want = ofp8.paged_decode_fp8(case.q.cpu(), kc8.cpu(), vc8.cpu(), 0.05, 0.08,
                                 case.block_tables.cpu(), case.seq_lens.cpu(), case.scale)
    bt = case.block_tables.clone()
    bt[0, 1] = kc8.shape[0] + 7
    B, H, D = case.q.shape
    out = torch.empty((B, H, D), dtype=torch.float32, device=DEV)
    binding.pa_decode_gqa_fp8(out, case.q, kc8, vc8, 0.05, 0.08, bt, case.seq_lens, case.scale,
                              64, partition=-1)
    assert binding.pa_get_device_error() & binding.PA_DEVERR_BLOCK_ID
    assert_parity(out[1:].cpu().numpy(), want[1:], "fp8 gqa neighbour of a bad id")
    assert bool(torch.isfinite(out[0]).all())
