"""Split-KV (FlashDecoding-style) partition pass and log-sum-exp reduce on the
GPU, against the oracle's per-partition statistics and its full result."""

import math

import numpy as np
import pytest
import torch

from helpers import assert_parity, oracle_full, oracle_pairs, run_decode, sample_pairs
from oracle import decode as oracle_decode
from paged_kv_cache_driven_b200 import binding, workloads

pytestmark = pytest.mark.gpu
DEV = "cuda"
LOG2E = 1.0 / math.log(2.0)


def workspace_views(ws, B, H, NP, D):
    n = B * H * NP
    f = ws.view(torch.float32)
    m = f[:n].view(B, H, NP)
    l = f[n:2 * n].view(B, H, NP)
    off = ((n * 8 + 255) // 256) * 256 // 4
    acc = f[off:off + n * D].view(B, H, NP, D)
    return m, l, acc


@pytest.mark.parametrize("P", [16, 64, 512])
def test_partition_stats_match_oracle(P):
    """m (base 2), l and the unnormalised acc of every written partition."""
    S, D, H = 16, 128, 3
    lens = [P + 1, 3 * P, 5 * P - 7, 2 * P + S]
    case = workloads.decode_case(lens, H=H, D=D, S=S, dtype=torch.bfloat16, seed=P, device=DEV)
    maxlen = max(lens)
    out, ws = run_decode(case, partition=P)
    _, NP = binding.pa_decode_plan(len(lens), H, D, S, maxlen, P)
    m, l, acc = (x.cpu().double().numpy() for x in workspace_views(ws, len(lens), H, NP, D))
    om, ol, oacc = oracle_decode.partition_stats(case.q.cpu(), case.k_cache.cpu(),
                                                 case.v_cache.cpu(), case.block_tables.cpu(),
                                                 case.seq_lens.cpu(), case.scale, P, NP)
    for i, L in enumerate(lens):
        n = -(-L // P)
        # the kernel keeps m in base-2 units: m2 = m * log2(e)
        np.testing.assert_allclose(m[i, :, :n], om[i, :, :n] * LOG2E, rtol=0, atol=2e-4)
        np.testing.assert_allclose(l[i, :, :n], ol[i, :, :n], rtol=2e-4, atol=0)
        assert_parity(acc[i, :, :n] / ol[i, :, :n, None], oacc[i, :, :n] / ol[i, :, :n, None],
                      f"partition acc P={P} request {i}")
    assert_parity(out.cpu().numpy(), oracle_full(case), f"merged P={P}")


@pytest.mark.parametrize("P", [16, 32, 128, 512, 4096])
def test_any_partition_size_gives_the_same_result(P):
    case = workloads.llama13b_decode(seed=7, device=DEV, batch=6)
    want = oracle_full(case)
    out, _ = run_decode(case, partition=P)
    assert_parity(out.cpu().numpy(), want, f"P={P}")
    single, _ = run_decode(case, partition=-1)
    assert_parity(single.cpu().numpy(), want, "single pass")
    assert binding.pa_get_device_error() == 0


def test_long_context_reduced():
    """Long-context shape (32 heads, head_dim 128, bf16) at lengths 32K-40K, 2 requests."""
    case = workloads.long_context_decode(seed=1, device=DEV, batch=2, lo=32768, hi=40000, H=4)
    out, _ = run_decode(case)
    P, NP = binding.pa_decode_plan(2, 4, 128, 16, max(case.seq_lens_host))
    assert NP > 1 and P % 16 == 0  # split
    assert_parity(out.cpu().numpy(), oracle_full(case), "long context reduced")


def test_long_context_full_size_sampled():
    """Batch 8, lengths U[32768, 131072], 32 heads: 512-token partitions and the
    reduce, checked on sampled outputs including the longest request."""
    case = workloads.long_context_decode(seed=0, device=DEV)
    out, _ = run_decode(case)
    pairs = sample_pairs(case, 16)
    got = np.stack([out[i, h].cpu().numpy() for i, h in pairs])
    assert_parity(got, oracle_pairs(case, pairs), "long context full size")
    assert binding.pa_get_device_error() == 0


@pytest.mark.parametrize("fill", ["zeros", "ones", "random", "nan"])
def test_any_workspace_contents(fill):
    """The result does not depend on what the workspace held before (every
    partial the merge reads is written by the same call), and one workspace
    serves calls of other partition sizes and of a grouped-query shape."""
    case = workloads.llama13b_decode(seed=3, device=DEV, batch=6)
    B, H, D = case.q.shape
    S, maxlen = 16, max(case.seq_lens_host)
    want = oracle_full(case)
    gq = workloads.llama70b_decode(seed=4, device=DEV, batch=3)
    Bg, Hg, _ = gq.q.shape
    gmax = max(gq.seq_lens_host)
    size = max([binding.pa_decode_workspace_bytes(B, H, D, S, maxlen, P) for P in (16, 64, 512)]
               + [binding.pa_decode_workspace_bytes(Bg, Hg, D, S, gmax, 64)])
    ws = torch.empty(size, dtype=torch.uint8, device=DEV)
    if fill == "zeros":
        ws.zero_()
    elif fill == "ones":
        ws.fill_(0xFF)
    elif fill == "random":
        ws.copy_(torch.randint(0, 256, (size,), dtype=torch.uint8, generator=torch.Generator()
                               .manual_seed(5)).to(DEV))
    else:
        ws.view(torch.float32)[: size // 4].fill_(float("nan"))
    for P in (64, 16, 512, 64):
        out = torch.empty((B, H, D), dtype=torch.float32, device=DEV)
        binding.pa_decode(out, case.q, case.k_cache, case.v_cache, case.block_tables,
                          case.seq_lens, case.scale, maxlen, partition=P, workspace=ws)
        assert_parity(out.cpu().numpy(), want, f"{fill} P={P}")
    out = torch.empty((Bg, Hg, D), dtype=torch.float32, device=DEV)
    binding.pa_decode_gqa(out, gq.q, gq.k_cache, gq.v_cache, gq.block_tables, gq.seq_lens,
                          gq.scale, gmax, partition=64, workspace=ws)
    assert_parity(out.cpu().numpy(), oracle_full(gq), f"{fill} grouped heads")
    assert binding.pa_get_device_error() == 0
