"""KV append (slot_mapping scatter) on the GPU: bit-exact against the oracle's
numpy scatter, with every untouched byte of the cache unchanged."""

import numpy as np
import pytest
import torch

from oracle import append as oracle_append
from oracle.allocator_model import BlockPoolModel
from paged_kv_cache_driven_b200 import binding, workloads

pytestmark = pytest.mark.gpu
DEV = "cuda"


def bits(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def check_append(k, v, slots, kc, vc):
    want_k, want_v = oracle_append.kv_append(k.cpu(), v.cpu(), slots.cpu(), kc.cpu(), vc.cpu())
    binding.pa_kv_append(k, v, slots, kc, vc)
    assert np.array_equal(bits(kc), want_k)
    assert np.array_equal(bits(vc), want_v)


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("D,S", [(64, 8), (128, 16), (256, 32), (8, 16), (136, 8)])
def test_decode_append_one_token_per_request(dtype, D, S):
    g = torch.Generator().manual_seed(D * S)
    NB, H, T = 40, 5, 23
    kc = torch.randn(NB, H, S, D, generator=g).to(dtype).to(DEV)
    vc = torch.randn(NB, H, S, D, generator=g).to(dtype).to(DEV)
    k = torch.randn(T, H, D, generator=g).to(dtype).to(DEV)
    v = torch.randn(T, H, D, generator=g).to(dtype).to(DEV)
    slots = torch.randperm(NB * S, generator=g)[:T].to(torch.int64)
    slots[[2, 9]] = -1  # padding tokens are skipped
    check_append(k, v, slots.to(DEV), kc, vc)
    assert binding.pa_get_device_error() == 0


def test_prefill_scale_append():
    """16 requests x U[512, 4096] tokens (H 32, D 128, bf16) scattered through
    slot mappings built by the oracle's allocator model into a shuffled pool."""
    case = workloads.prefill_append(seed=0, device=DEV)
    NB, H, S, D = case.k_cache.shape
    model = BlockPoolModel(NB, S, initial_order=case.block_order)
    for r, n in enumerate(case.n_tokens):
        model.grow(r, n)
    slots = torch.tensor(model.slot_mapping(list(range(len(case.n_tokens))), [0] * 16,
                                            case.n_tokens), dtype=torch.int64)
    assert slots.numel() == case.k.shape[0]
    check_append(case.k, case.v, slots.to(DEV), case.k_cache, case.v_cache)
    assert binding.pa_get_device_error() == 0


def test_zero_tokens_and_all_padding():
    kc = torch.randn(4, 2, 16, 64, device=DEV).half()
    vc = torch.randn(4, 2, 16, 64, device=DEV).half()
    before = (kc.clone(), vc.clone())
    k = torch.randn(0, 2, 64, device=DEV).half()
    binding.pa_kv_append(k, k, torch.empty(0, dtype=torch.int64, device=DEV), kc, vc)
    k = torch.randn(5, 2, 64, device=DEV).half()
    binding.pa_kv_append(k, k, torch.full((5,), -1, dtype=torch.int64, device=DEV), kc, vc)
    assert torch.equal(kc, before[0]) and torch.equal(vc, before[1])


def test_slot_past_pool_is_skipped_and_flagged():
    NB, H, S, D = 6, 2, 8, 64
    kc = torch.randn(NB, H, S, D, device=DEV).half()
    vc = torch.randn(NB, H, S, D, device=DEV).half()
    k = torch.randn(3, H, D, device=DEV).half()
    v = torch.randn(3, H, D, device=DEV).half()
    slots = torch.tensor([5, NB * S + 3, 17], dtype=torch.int64, device=DEV)
    want_k, want_v = oracle_append.kv_append(k.cpu(), v.cpu(),
                                             torch.tensor([5, -1, 17]), kc.cpu(), vc.cpu())
    binding.pa_kv_append(k, v, slots, kc, vc)
    assert binding.pa_get_device_error() & binding.PA_DEVERR_SLOT
    assert np.array_equal(bits(kc), want_k) and np.array_equal(bits(vc), want_v)
    assert binding.pa_get_device_error() == 0
