"""The shape sweep at full size: block_size {8, 16, 32} x head_dim {64, 128, 256}
x batch {1, 32, 256}, 32 heads, fp16 and bf16, seq_lens uniform in [16, 8192],
in the automatic launch configuration; sampled outputs against the oracle."""

import numpy as np
import pytest
import torch

from helpers import assert_parity, oracle_pairs, run_decode, sample_pairs
from paged_kv_cache_driven_b200 import binding, workloads

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16], ids=["fp16", "bf16"])
@pytest.mark.parametrize("B", [1, 32, 256])
@pytest.mark.parametrize("D", [64, 128, 256])
@pytest.mark.parametrize("S", [8, 16, 32])
def test_sweep_point(S, D, B, dtype):
    seed = S * 100000 + D * 1000 + B * 10 + (dtype == torch.bfloat16)
    case = workloads.sweep_case(S, D, B, dtype, seed=seed, device=DEV)
    out, _ = run_decode(case)
    pairs = sample_pairs(case, 12 if B > 1 else 8, seed=seed)
    got = np.stack([out[i, h].cpu().numpy() for i, h in pairs])
    assert_parity(got, oracle_pairs(case, pairs), f"S={S} D={D} B={B} {dtype}")
    assert binding.pa_get_device_error() == 0
    del case, out
    torch.cuda.empty_cache()
