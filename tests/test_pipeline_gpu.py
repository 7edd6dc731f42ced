"""HostFedDecoder / pa_stepper_* (decode steps fed from pinned host memory,
copies overlapped with kernels on a second stream) against the same steps run one call at a time,
and its last step against the oracle."""

import math

import numpy as np
import torch
import pytest

from helpers import assert_parity
from oracle import decode as oracle_decode
from paged_kv_cache_driven_b200 import binding, workloads
from paged_kv_cache_driven_b200.binding import BlockAllocator
from paged_kv_cache_driven_b200.pipeline import HostFedDecoder

pytestmark = pytest.mark.gpu
DEV = "cuda"


def setup(seed, B=12, H=6, D=128, S=16, steps=6):
    lens = workloads.uniform_lengths(B, 1, 1500, seed)
    NB = sum(-(-(L + steps) // S) for L in lens) + 3
    order = torch.randperm(NB, generator=torch.Generator().manual_seed(seed)).tolist()
    g = torch.Generator(device=DEV).manual_seed(seed)
    kc = torch.randn((NB, H, S, D), generator=g, device=DEV, dtype=torch.bfloat16)
    vc = torch.randn((NB, H, S, D), generator=g, device=DEV, dtype=torch.bfloat16)
    alloc = BlockAllocator(NB, S, initial_order=order)
    for i, L in enumerate(lens):
        alloc.pa_seq_grow(i, L)
    inputs = [torch.randn((3, B, H, D), generator=g, device=DEV, dtype=torch.bfloat16)
              .cpu().pin_memory() for _ in range(steps)]
    MB = -(-(max(lens) + steps) // S)
    return lens, kc, vc, alloc, inputs, MB


@pytest.mark.parametrize("fused", [True, False])
def test_pipelined_steps_equal_sequential_steps(fused):
    steps = 6
    lens0, kc, vc, alloc, inputs, MB = setup(0, steps=steps)
    B = len(lens0)
    H, S, D = kc.shape[1], kc.shape[2], kc.shape[3]
    kc_ref, vc_ref = kc.clone(), vc.clone()
    _, _, _, alloc_ref, _, _ = setup(0, steps=steps)
    ids = list(range(B))
    max_len = max(lens0) + steps

    fed = HostFedDecoder(alloc, kc, vc, B, MB, max_len, out_dtype=torch.float32, fused=fused)
    got, prev = [], None
    for n in range(steps):
        step_no, _ = fed.step(ids, inputs[n])
        assert step_no == n
        if prev is not None:  # read step n-1 while step n is in flight
            got.append(fed.output(prev))
        prev = step_no
    fed.drain()
    torch.cuda.synchronize()
    got.append(fed.output(prev))
    with pytest.raises(binding.PagedAttnError):
        fed.output(0)  # its staging set has been reused
    fed.close()

    ws = torch.empty(binding.pa_decode_workspace_bytes(B, H, D, S, max_len, 0) + 16,
                     dtype=torch.uint8, device=DEV)
    for n in range(steps):
        slots = torch.empty(B, dtype=torch.int64)
        tables = torch.empty((B, MB), dtype=torch.int32)
        lens = torch.empty(B, dtype=torch.int32)
        alloc_ref.pa_prepare_step(ids, 1, MB, slots, tables, lens)
        q, k, v = (x.to(DEV) for x in inputs[n])  # [3, B, H, D] unpacks to q, k, v
        binding.pa_kv_append(k, v, slots.to(DEV), kc_ref, vc_ref)
        out = torch.empty((B, H, D), dtype=torch.float32, device=DEV)
        binding.pa_decode(out, q, kc_ref, vc_ref, tables.to(DEV), lens.to(DEV), D ** -0.5,
                          int(lens.max()), workspace=ws)
        assert torch.equal(got[n], out.cpu()), f"step {n}"
    assert torch.equal(kc, kc_ref) and torch.equal(vc, vc_ref)
    assert alloc.pa_alloc_dump() == alloc_ref.pa_alloc_dump()
    # the last step against the oracle
    want = oracle_decode.paged_decode(inputs[-1][0], kc.cpu(), vc.cpu(), tables, lens, D ** -0.5)
    assert_parity(got[-1].numpy(), want, "pipelined last step")
    assert binding.pa_get_device_error() == 0
