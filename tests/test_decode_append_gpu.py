"""pa_decode_append (append the new token at each request's last position, then
decode, in one launch) against the two-call path pa_kv_append + pa_decode (bit
for bit: output and cache) and against the oracle (numpy scatter + fp64 decode)."""

import numpy as np
import pytest
import torch

from helpers import assert_parity
from oracle import append as oracle_append
from oracle import decode as oracle_decode
from paged_kv_cache_driven_b200 import binding, workloads

pytestmark = pytest.mark.gpu
DEV = "cuda"


def last_slots(case):
    S = case.k_cache.shape[2]
    return torch.tensor([case.tables_host[i][(L - 1) // S] * S + (L - 1) % S if L > 0 else -1
                         for i, L in enumerate(case.seq_lens_host)], dtype=torch.int64)


def run_both(case, partition, out_dtype=torch.float32, seed=0):
    B, H, D = case.q.shape
    S = case.k_cache.shape[2]
    g = torch.Generator(device=DEV).manual_seed(seed + 77)
    k_new = torch.randn((B, H, D), generator=g, device=DEV, dtype=case.q.dtype)
    v_new = torch.randn((B, H, D), generator=g, device=DEV, dtype=case.q.dtype)
    maxlen = max(case.seq_lens_host)
    ws_bytes = binding.pa_decode_workspace_bytes(B, H, D, S, maxlen, partition)
    ws = torch.empty(ws_bytes + 16, dtype=torch.uint8, device=DEV)
    # the two-call path on copies of the cache
    kc2, vc2 = case.k_cache.clone(), case.v_cache.clone()
    binding.pa_kv_append(k_new, v_new, last_slots(case).to(DEV), kc2, vc2)
    ref = torch.empty((B, H, D), dtype=out_dtype, device=DEV)
    binding.pa_decode(ref, case.q, kc2, vc2, case.block_tables, case.seq_lens, case.scale, maxlen,
                      partition=partition, workspace=ws)
    # the fused path on the case's own cache
    k_before, v_before = case.k_cache.cpu(), case.v_cache.cpu()
    out = torch.empty((B, H, D), dtype=out_dtype, device=DEV)
    binding.pa_decode_append(out, case.q, k_new, v_new, case.k_cache, case.v_cache,
                             case.block_tables, case.seq_lens, case.scale, maxlen,
                             partition=partition, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(out, ref)
    # bit patterns: the pools hold NaN poison, which never compares equal
    assert torch.equal(case.k_cache.view(torch.int16), kc2.view(torch.int16))
    assert torch.equal(case.v_cache.view(torch.int16), vc2.view(torch.int16))
    return out, k_new, v_new, k_before, v_before


@pytest.mark.parametrize("partition", [0, -1, 16, 64])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_fused_equals_two_calls_and_oracle(partition, dtype):
    S = 16
    lens = [1, S - 1, S, S + 1, 2 * S, 200, 777, 1024, 1025, 2048]
    case = workloads.decode_case(lens, H=6, D=128, S=S, dtype=dtype, seed=5, device=DEV)
    out, k_new, v_new, kb, vb = run_both(case, partition)
    kc, vc = oracle_append.kv_append(k_new.cpu(), v_new.cpu(), last_slots(case), kb, vb)
    want = oracle_decode.paged_decode(case.q.cpu(), torch.from_numpy(kc.view(np.int16)).view(dtype),
                                      torch.from_numpy(vc.view(np.int16)).view(dtype),
                                      case.block_tables.cpu(), case.seq_lens.cpu(), case.scale)
    assert_parity(out.cpu().numpy(), want, f"fused p={partition}")
    # a request of one token attends only to its new token: out = v_new exactly
    assert torch.equal(out[0].cpu(), v_new[0].float().cpu())
    assert binding.pa_get_device_error() == 0


@pytest.mark.parametrize("D,S", [(64, 8), (64, 32), (128, 8), (128, 32), (256, 8), (256, 16),
                                 (256, 32), (64, 16)])
def test_fused_all_shapes(D, S):
    lens = [0, 1, S, 3 * S + 1, 900, 1600]
    case = workloads.decode_case(lens, H=3, D=D, S=S, dtype=torch.bfloat16, seed=D * S,
                                 device=DEV, pool_blocks=sum(-(-L // S) for L in lens) + 4)
    for partition in (0, 4 * S):
        out, *_ = run_both(case, partition, out_dtype=torch.bfloat16, seed=partition)
        assert torch.all(out[0] == 0)  # L = 0: no append, zero output
    assert binding.pa_get_device_error() == 0


def test_fused_llama13b_full_size():
    """The bench's workload in its launch configuration, against the two-call path."""
    case = workloads.llama13b_decode(seed=0, device=DEV)
    run_both(case, 0, out_dtype=torch.bfloat16)
    assert binding.pa_get_device_error() == 0
