"""pa_decode_noalloc: decode for callers that cannot allocate device memory.

Some callers of this library cannot call cudaMalloc: a plugin whose host
framework owns every device allocation and hands it no allocator, or a serving
process that fixes its device-memory budget at start-up and must not allocate
(or risk a device-wide synchronisation) while it serves. For them,
pa_decode_noalloc keeps the split-KV partials in a static device array inside
the library instead of a caller-provided workspace.

This file is collected last so that a run stopping at the first failure has
already run every other test; it must pass alone in a fresh process too.
"""

import pytest
import torch

from helpers import assert_parity, run_decode
from paged_kv_cache_driven_b200 import binding, workloads

pytestmark = pytest.mark.gpu
DEV = "cuda"


def noalloc(case, partition, out_dtype=torch.float32):
    out = torch.empty(case.q.shape, dtype=out_dtype, device=DEV)
    binding.pa_decode_noalloc(out, case.q, case.k_cache, case.v_cache, case.block_tables,
                              case.seq_lens, case.scale, max(case.seq_lens_host),
                              partition=partition)
    return out


@pytest.mark.parametrize("partition", [0, 64])
def test_noalloc_matches_pa_decode_twice_in_a_row(partition):
    """Two calls in a row, on two different batches, each against pa_decode with
    a caller-provided workspace: the second call reuses the array the first one
    left its partials in."""
    for seed in (0, 1):
        case = workloads.llama13b_decode(seed=seed, device=DEV, batch=8)
        B, H, D = case.q.shape
        S = case.k_cache.shape[2]
        need = binding.pa_decode_workspace_bytes(B, H, D, S, max(case.seq_lens_host), partition)
        assert 0 < need <= binding.pa_noalloc_scratch_bytes()  # the split really uses the array
        want, _ = run_decode(case, partition=partition)
        got = noalloc(case, partition)
        torch.cuda.synchronize()
        assert_parity(got.cpu().numpy(), want.cpu().numpy(), f"no-alloc seed {seed}")
        assert torch.equal(got, want)  # same kernels, same order: identical bits
    assert binding.pa_get_device_error() == 0


def test_noalloc_rejects_a_split_larger_than_the_array():
    """A split whose partials exceed PA_NOALLOC_SCRATCH_BYTES is refused on the
    host with PA_ERR_OOM before anything is launched."""
    B, H, D, S = 64, 40, 128, 16
    big = binding.pa_decode_workspace_bytes(B, H, D, S, 131072, 512)
    assert big > binding.pa_noalloc_scratch_bytes()
    q = torch.zeros((B, H, D), dtype=torch.bfloat16, device=DEV)
    out = torch.empty((B, H, D), dtype=torch.float32, device=DEV)
    tables = torch.full((B, 8192), -1, dtype=torch.int32, device=DEV)
    lens = torch.zeros(B, dtype=torch.int32, device=DEV)
    kc = torch.zeros((4, H, S, D), dtype=torch.bfloat16, device=DEV)
    before = out.clone()
    with pytest.raises(binding.PagedAttnError) as e:
        binding.pa_decode_noalloc(out, q, kc, kc, tables, lens, 0.1, 131072, partition=512)
    assert e.value.code == binding.PA_ERR_OOM
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int32), before.view(torch.int32))  # nothing ran
