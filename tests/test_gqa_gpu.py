"""Grouped-query decode (pa_decode_gqa; query head h reads KV head h // G) on
the GPU against the fp64 oracle, against pa_decode when G = 1, and its fused
append against the two-call path."""

import numpy as np
import pytest
import torch

from helpers import assert_parity, oracle_full, oracle_pairs, run_decode, sample_pairs
from oracle import append as oracle_append
from oracle import decode as oracle_decode
from paged_kv_cache_driven_b200 import binding, workloads

pytestmark = pytest.mark.gpu
DEV = "cuda"


def gqa_case(lens, Hkv, G, D, S, dtype, seed, extra=3):
    return workloads.decode_case(lens, H=Hkv * G, D=D, S=S, dtype=dtype, seed=seed, device=DEV,
                                 Hkv=Hkv, pool_blocks=sum(-(-L // S) for L in lens) + extra)


@pytest.mark.parametrize("G", [2, 3, 4, 8, 16])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_group_sizes(G, dtype):
    S = 16
    lens = [0, 1, S - 1, S + 1, 333, 1000, 2047]
    case = gqa_case(lens, Hkv=2, G=G, D=128, S=S, dtype=dtype, seed=G)
    want = oracle_full(case)
    for partition in (0, -1, 64):
        out, _ = run_decode(case, partition=partition)
        o = out.cpu()
        assert torch.all(o[0] == 0)
        assert_parity(o.numpy(), want, f"G={G} p={partition}")
    assert binding.pa_get_device_error() == 0


@pytest.mark.parametrize("D,S", [(64, 8), (64, 32), (128, 8), (128, 32), (256, 8), (256, 16),
                                 (256, 32), (64, 16)])
def test_shapes(D, S):
    lens = [1, 2 * S + 3, 700, 1500]
    case = gqa_case(lens, Hkv=2, G=4, D=D, S=S, dtype=torch.bfloat16, seed=D + S)
    want = oracle_full(case)
    for partition in (0, 4 * S):
        out, _ = run_decode(case, partition=partition)
        assert_parity(out.cpu().numpy(), want, f"D={D} S={S} p={partition}")
    assert binding.pa_get_device_error() == 0


def test_one_group_equals_pa_decode_bitwise():
    case = workloads.llama13b_decode(seed=2, device=DEV, batch=8)
    B, H, D = case.q.shape
    S = case.k_cache.shape[2]
    maxlen = max(case.seq_lens_host)
    ws = torch.empty(binding.pa_decode_workspace_bytes(B, H, D, S, maxlen) + 16,
                     dtype=torch.uint8, device=DEV)
    a = torch.empty((B, H, D), dtype=torch.float32, device=DEV)
    b = torch.empty_like(a)
    binding.pa_decode(a, case.q, case.k_cache, case.v_cache, case.block_tables, case.seq_lens,
                      case.scale, maxlen, workspace=ws)
    binding.pa_decode_gqa(b, case.q, case.k_cache, case.v_cache, case.block_tables,
                          case.seq_lens, case.scale, maxlen, workspace=ws)
    assert torch.equal(a, b)


@pytest.mark.parametrize("G", [3, 8])
@pytest.mark.parametrize("partition", [0, 32])
def test_fused_append_equals_two_calls_and_oracle(G, partition):
    S, Hkv, D = 16, 4, 128
    lens = [1, S, S + 1, 500, 1023]
    case = gqa_case(lens, Hkv=Hkv, G=G, D=D, S=S, dtype=torch.bfloat16, seed=11 + G)
    B, H = len(lens), Hkv * G
    g = torch.Generator(device=DEV).manual_seed(5)
    k_new = torch.randn((B, Hkv, D), generator=g, device=DEV, dtype=torch.bfloat16)
    v_new = torch.randn((B, Hkv, D), generator=g, device=DEV, dtype=torch.bfloat16)
    slots = torch.tensor([case.tables_host[i][(L - 1) // S] * S + (L - 1) % S
                          for i, L in enumerate(lens)], dtype=torch.int64)
    maxlen = max(lens)
    ws = torch.empty(binding.pa_decode_workspace_bytes(B, H, D, S, maxlen, partition) + 16,
                     dtype=torch.uint8, device=DEV)
    kb, vb = case.k_cache.cpu(), case.v_cache.cpu()
    kc2, vc2 = case.k_cache.clone(), case.v_cache.clone()
    binding.pa_kv_append(k_new, v_new, slots.to(DEV), kc2, vc2)
    ref = torch.empty((B, H, D), dtype=torch.float32, device=DEV)
    binding.pa_decode_gqa(ref, case.q, kc2, vc2, case.block_tables, case.seq_lens, case.scale,
                          maxlen, partition=partition, workspace=ws)
    out = torch.empty_like(ref)
    binding.pa_decode_gqa(out, case.q, case.k_cache, case.v_cache, case.block_tables,
                          case.seq_lens, case.scale, maxlen, k_new=k_new, v_new=v_new,
                          partition=partition, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    assert torch.equal(case.k_cache.view(torch.int16), kc2.view(torch.int16))
    assert torch.equal(case.v_cache.view(torch.int16), vc2.view(torch.int16))
    kc, vc = oracle_append.kv_append(k_new.cpu(), v_new.cpu(), slots, kb, vb)
    want = oracle_decode.paged_decode(case.q.cpu(), torch.from_numpy(kc.view(np.int16)).view(
        torch.bfloat16), torch.from_numpy(vc.view(np.int16)).view(torch.bfloat16),
        case.block_tables.cpu(), case.seq_lens.cpu(), case.scale)
    assert_parity(out.cpu().numpy(), want, f"fused GQA G={G}")
    assert torch.equal(out[0].cpu(), v_new[0].float().cpu().repeat_interleave(G, dim=0))
    assert binding.pa_get_device_error() == 0


def test_llama70b_shape_full_size_sampled():
    """64 query heads over 8 KV heads, head_dim 128, bf16, batch 64, U[1, 2048]."""
    case = workloads.llama70b_decode(seed=0, device=DEV)
    out, _ = run_decode(case)
    pairs = sample_pairs(case, 48)
    got = np.stack([out[i, h].cpu().numpy() for i, h in pairs])
    assert_parity(got, oracle_pairs(case, pairs), "llama70b full size")
    assert binding.pa_get_device_error() == 0
