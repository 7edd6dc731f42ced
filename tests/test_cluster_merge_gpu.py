"""Small grids merge a split request inside a thread-block cluster.

FlashDecoding's split-KV ("PagedAttention" card, "헷갈리기 쉬운 구분") cuts a
request into partitions and merges their partial results by log-sum-exp. When
the automatic plan splits into 2, 4 or 8 partitions on a grid that fits within
two CTAs per SM, the partitions of one (request, head) run as one cluster and
partition 0 merges the others' (acc, m, l) through distributed shared memory;
an explicit partition length takes the workspace and the merge kernel instead.
Both forms must give the same bits, and the oracle's result within tolerance.
"""

import numpy as np
import pytest
import torch

from helpers import assert_parity, oracle_full, run_decode
from oracle import append as oracle_append
from paged_kv_cache_driven_b200 import binding, workloads

pytestmark = pytest.mark.gpu
DEV = "cuda"

# (lengths, heads, head_dim, block_size, dtype): each plans 2, 4 or 8 partitions
CASES = [
    ([1332], 32, 128, 16, torch.bfloat16),          # 8 x 176 tokens, 256 CTAs
    ([1332], 40, 128, 16, torch.float16),           # 4 x 336
    ([1332, 17], 16, 64, 16, torch.float16),        # 8; the short request is direct, 7 CTAs idle
    ([1332, 0, 1, 700], 8, 256, 32, torch.bfloat16),  # 4; empty, one-token and half-idle clusters
    ([100], 32, 128, 8, torch.float16),             # 2 x 64
    ([150], 32, 64, 16, torch.bfloat16),            # 4 x 48
    ([2048, 2048], 16, 128, 16, torch.bfloat16),    # 8 x 256, every partition full
    ([700, 20], 20, 64, 8, torch.float16),          # 4 x 176
]


def cluster_plan(B, H, D, S, maxlen):
    P, NP = binding.pa_decode_plan(B, H, D, S, maxlen, 0)
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert NP in (2, 4, 8) and B * H * NP <= 2 * sms, (P, NP)
    return P, NP


def same_bits(a, b):
    return torch.equal(a.contiguous().view(torch.int32 if a.element_size() == 4 else torch.int16),
                       b.contiguous().view(torch.int32 if b.element_size() == 4 else torch.int16))


@pytest.mark.parametrize("lens,H,D,S,dt", CASES)
def test_cluster_merge_matches_workspace_merge_and_oracle(lens, H, D, S, dt):
    case = workloads.decode_case(lens, H=H, D=D, S=S, dtype=dt, seed=sum(lens) + H, device=DEV)
    P, _ = cluster_plan(len(lens), H, D, S, max(lens))
    for out_dt in (torch.float32, dt):
        auto, _ = run_decode(case, out_dtype=out_dt, partition=0)
        ws, _ = run_decode(case, out_dtype=out_dt, partition=P)
        assert same_bits(auto, ws), f"cluster and workspace merges differ ({out_dt})"
    auto32, _ = run_decode(case, partition=0)
    assert_parity(auto32.cpu().numpy(), oracle_full(case), f"cluster merge {lens} H={H} D={D}")
    assert binding.pa_get_device_error() == 0


def test_cluster_merge_fused_append():
    """pa_decode_append on a cluster plan: the same output and cache bytes as the
    workspace form, and the appended rows where the slot mapping puts them."""
    lens = [1332, 17, 700]
    H, D, S = 10, 128, 16
    case = workloads.decode_case(lens, H=H, D=D, S=S, dtype=torch.bfloat16, seed=11,
                                 device=DEV, pool_blocks=200, max_blocks=96)
    P, _ = cluster_plan(len(lens), H, D, S, max(lens))
    g = torch.Generator(device=DEV).manual_seed(5)
    k_new = torch.randn((len(lens), H, D), generator=g, device=DEV).to(torch.bfloat16)
    v_new = torch.randn((len(lens), H, D), generator=g, device=DEV).to(torch.bfloat16)
    results = []
    for part in (0, P):
        kc, vc = case.k_cache.clone(), case.v_cache.clone()
        out = torch.empty((len(lens), H, D), dtype=torch.float32, device=DEV)
        wsb = binding.pa_decode_workspace_bytes(len(lens), H, D, S, max(lens), part)
        ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=DEV)
        binding.pa_decode_append(out, case.q, k_new, v_new, kc, vc, case.block_tables,
                                 case.seq_lens, case.scale, max(lens), partition=part,
                                 workspace=ws)
        results.append((out, kc, vc))
    (o0, k0, v0), (o1, k1, v1) = results
    assert same_bits(o0, o1)
    assert torch.equal(k0.view(torch.int16), k1.view(torch.int16))
    assert torch.equal(v0.view(torch.int16), v1.view(torch.int16))
    # the new rows sit at position L - 1 of each request
    slots = [case.tables_host[i][(L - 1) // S] * S + (L - 1) % S for i, L in enumerate(lens)]
    kc_want = case.k_cache.clone().cpu().view(torch.int16).numpy()
    vc_want = case.v_cache.clone().cpu().view(torch.int16).numpy()
    oracle_append.scatter_into(k_new.cpu().view(torch.int16).numpy(),
                               v_new.cpu().view(torch.int16).numpy(), slots, kc_want, vc_want)
    assert np.array_equal(k0.cpu().view(torch.int16).numpy(), kc_want)
    assert np.array_equal(v0.cpu().view(torch.int16).numpy(), vc_want)
    assert binding.pa_get_device_error() == 0


def test_cluster_merge_fp8():
    """pa_decode_fp8 on a cluster plan gives the workspace form's bits."""
    lens = [1332]
    H, D, S = 32, 128, 16
    case = workloads.decode_case(lens, H=H, D=D, S=S, dtype=torch.bfloat16, seed=3, device=DEV)
    P, _ = cluster_plan(1, H, D, S, max(lens))
    NB = case.k_cache.shape[0]
    kc8 = torch.empty((NB, H, S, D), dtype=torch.uint8, device=DEV)
    vc8 = torch.empty_like(kc8)
    slots = torch.arange(NB * S, dtype=torch.int64, device=DEV)
    flat = lambda c: c.permute(0, 2, 1, 3).reshape(-1, H, D).contiguous()  # noqa: E731
    binding.pa_kv_append_fp8(flat(case.k_cache), flat(case.v_cache), slots, kc8, vc8, 0.05, 0.08)
    outs = []
    for part in (0, P):
        out = torch.empty((1, H, D), dtype=torch.float32, device=DEV)
        wsb = binding.pa_decode_workspace_bytes(1, H, D, S, max(lens), part)
        ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=DEV)
        binding.pa_decode_fp8(out, case.q, kc8, vc8, 0.05, 0.08, case.block_tables,
                              case.seq_lens, case.scale, max(lens), partition=part, workspace=ws)
        outs.append(out)
    assert same_bits(outs[0], outs[1])
    assert torch.isfinite(outs[0]).all()
    assert binding.pa_get_device_error() == 0


def test_cluster_merge_in_a_cuda_graph():
    """A cluster launch captured in a CUDA graph replays to the eager bits."""
    lens = [1332, 17]
    H, D, S = 16, 128, 16
    case = workloads.decode_case(lens, H=H, D=D, S=S, dtype=torch.bfloat16, seed=21, device=DEV)
    cluster_plan(len(lens), H, D, S, max(lens))
    eager, _ = run_decode(case, partition=0)
    out = torch.empty_like(eager)
    wsb = binding.pa_decode_workspace_bytes(len(lens), H, D, S, max(lens), 0)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=DEV)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):  # warm-up outside the capture (attribute set-up)
        binding.pa_decode(out, case.q, case.k_cache, case.v_cache, case.block_tables,
                          case.seq_lens, case.scale, max(lens), partition=0, workspace=ws)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    out.zero_()
    with torch.cuda.graph(g):
        binding.pa_decode(out, case.q, case.k_cache, case.v_cache, case.block_tables,
                          case.seq_lens, case.scale, max(lens), partition=0, workspace=ws)
    for _ in range(3):
        out.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert same_bits(out, eager)
    del g
    assert binding.pa_get_device_error() == 0
