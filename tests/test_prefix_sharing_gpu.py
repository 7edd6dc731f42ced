"""Prefix sharing with copy-on-write ("vLLM KV Cache and PagedAttention
Explained", Step 9) on the GPU: pa_copy_blocks bit for bit against the oracle's
block copy, and parallel sampling from one shared prompt (fork, decode steps
whose writes into the shared partly filled block are preceded by the queued
copies) against an oracle mirror: allocator model, numpy copies and scatters,
fp64 decode."""

import math

import numpy as np
import pytest
import torch

from helpers import assert_parity
from oracle import append as oracle_append
from oracle import decode as oracle_decode
from oracle.allocator_model import BlockPoolModel
from paged_kv_cache_driven_b200 import binding
from paged_kv_cache_driven_b200.binding import BlockAllocator

pytestmark = pytest.mark.gpu
DEV = "cuda"


def bits(t):
    return t.cpu().view(torch.int16).numpy().view(np.uint16)


def test_copy_blocks_bit_exact():
    g = torch.Generator().manual_seed(0)
    NB, H, S, D = 50, 6, 16, 128
    kc = torch.randn(NB, H, S, D, generator=g).to(torch.bfloat16).to(DEV)
    vc = torch.randn(NB, H, S, D, generator=g).to(torch.bfloat16).to(DEV)
    pairs = [(3, 10), (7, 11), (3, 12), (40, 0)]
    want_k, want_v = bits(kc).copy(), bits(vc).copy()
    oracle_append.copy_blocks_into(want_k, want_v, pairs)
    binding.pa_copy_blocks(kc, vc, torch.tensor(pairs, dtype=torch.int32, device=DEV))
    assert np.array_equal(bits(kc), want_k) and np.array_equal(bits(vc), want_v)
    binding.pa_copy_blocks(kc, vc, torch.empty((0, 2), dtype=torch.int32, device=DEV))
    assert binding.pa_get_device_error() == 0
    # an id outside the pool is skipped and flagged, the other pair still copies
    binding.pa_copy_blocks(kc, vc, torch.tensor([[1, NB + 5], [2, 13]], dtype=torch.int32,
                                                device=DEV))
    assert binding.pa_get_device_error() & binding.PA_DEVERR_BLOCK_ID
    oracle_append.copy_blocks_into(want_k, want_v, [(2, 13)])
    assert np.array_equal(bits(kc), want_k)


@pytest.mark.parametrize("fused", [True, False], ids=["fused", "two_calls"])
def test_parallel_sampling_from_a_shared_prompt(fused):
    g = torch.Generator().manual_seed(1)
    n, prompt, steps = 5, 100, 24
    H, S, D = 8, 16, 128
    NB = 60
    order = torch.randperm(NB, generator=g).tolist()
    dt = torch.bfloat16
    nan = float("nan")
    kc = torch.full((NB, H, S, D), nan, dtype=dt, device=DEV)
    vc = torch.full((NB, H, S, D), nan, dtype=dt, device=DEV)
    alloc = BlockAllocator(NB, S, initial_order=order)
    model = BlockPoolModel(NB, S, initial_order=order)
    mk, mv = bits(kc).copy(), bits(vc).copy()
    # prompt prefill: one request, then n samples forked from it
    pk = torch.randn(prompt, H, D, generator=g).to(dt)
    pv = torch.randn(prompt, H, D, generator=g).to(dt)
    alloc.pa_seq_grow(100, prompt)
    model.grow(100, prompt)
    slots = alloc.pa_build_slot_mapping([100], [0], [prompt])
    assert slots.tolist() == model.slot_mapping([100], [0], [prompt])
    binding.pa_kv_append(pk.to(DEV), pv.to(DEV), slots.to(DEV), kc, vc)
    oracle_append.scatter_into(bits(pk), bits(pv), slots.numpy(), mk, mv)
    ids = list(range(n))
    for k in ids:
        alloc.pa_seq_fork(100, k)
        model.fork(100, k)
    alloc.pa_seq_free(100)
    model.release(100)
    assert alloc.pa_alloc_refcounts() == model.refs
    MB = -(-(prompt + steps) // S)
    ws = torch.empty(binding.pa_decode_workspace_bytes(n, H, D, S, prompt + steps, 32) + 16,
                     dtype=torch.uint8, device=DEV)
    copies_seen = 0
    for step in range(steps):
        h_slots = torch.empty(n, dtype=torch.int64)
        h_tables = torch.empty((n, MB), dtype=torch.int32)
        h_lens = torch.empty(n, dtype=torch.int32)
        alloc.pa_prepare_step(ids, 1, MB, h_slots, h_tables, h_lens)
        pairs = alloc.pa_alloc_take_copies()
        want_slots = []
        for k in ids:
            model.grow(k, model.lens[k] + 1)
            want_slots += model.slot_mapping([k], [model.lens[k] - 1], [1])
        want_pairs = model.take_copies()
        assert [tuple(x) for x in pairs.tolist()] == want_pairs
        assert h_slots.tolist() == want_slots and h_tables.tolist() == model.block_tables(ids, MB)
        copies_seen += len(want_pairs)
        # device: the copies first, then the step's append and decode
        binding.pa_copy_blocks(kc, vc, pairs.to(DEV))
        q = torch.randn(n, H, D, generator=g).to(dt)
        kn = torch.randn(n, H, D, generator=g).to(dt)
        vn = torch.randn(n, H, D, generator=g).to(dt)
        out = torch.empty((n, H, D), dtype=torch.float32, device=DEV)
        tables_d, lens_d = h_tables.to(DEV), h_lens.to(DEV)
        maxlen = int(h_lens.max())
        if fused:
            binding.pa_decode_append(out, q.to(DEV), kn.to(DEV), vn.to(DEV), kc, vc, tables_d,
                                     lens_d, D ** -0.5, maxlen, partition=32, workspace=ws)
        else:
            binding.pa_kv_append(kn.to(DEV), vn.to(DEV), h_slots.to(DEV), kc, vc)
            binding.pa_decode(out, q.to(DEV), kc, vc, tables_d, lens_d, D ** -0.5, maxlen,
                              partition=32, workspace=ws)
        # the mirror
        oracle_append.copy_blocks_into(mk, mv, want_pairs)
        oracle_append.scatter_into(bits(kn), bits(vn), np.array(want_slots), mk, mv)
        want = oracle_decode.paged_decode(bits(q), mk, mv, np.array(model.block_tables(ids, MB),
                                          dtype=np.int32), np.array([model.lens[k] for k in ids],
                                          dtype=np.int32), D ** -0.5, dtype=dt)
        assert_parity(out.cpu().numpy(), want, f"sampling step {step}")
    assert copies_seen == n - 1  # the shared partly filled prompt block, for all writers but the last
    torch.cuda.synchronize()
    assert np.array_equal(bits(kc), mk) and np.array_equal(bits(vc), mv)
    assert binding.pa_get_device_error() == 0
