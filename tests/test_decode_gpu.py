"""Paged decode attention on the GPU against the fp64 oracle, through the C ABI."""

import math

import numpy as np
import pytest
import torch

from helpers import assert_parity, oracle_full, oracle_pairs, parity_stats, run_decode, sample_pairs
from paged_kv_cache_driven_b200 import binding, workloads

pytestmark = pytest.mark.gpu
DEV = "cuda"


def clean_error_word():
    assert binding.pa_get_device_error() == 0


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_worked_example_all_outputs(seed):
    """4 requests of 6/50/8/100 tokens, fp16, 64-block permuted pool, NaN-poisoned."""
    case = workloads.worked_example(seed=seed, device=DEV)
    out, _ = run_decode(case)
    torch.cuda.synchronize()
    assert_parity(out.cpu().numpy(), oracle_full(case), "worked example")
    clean_error_word()


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_llama13b_shape_reduced_batch(seed):
    """40 heads, head_dim 128, bf16, lengths U[1, 2048]; 8 requests, every output checked."""
    case = workloads.llama13b_decode(seed=seed, device=DEV, batch=8)
    out, _ = run_decode(case)
    assert_parity(out.cpu().numpy(), oracle_full(case), "llama13b batch 8")
    clean_error_word()


def test_llama13b_full_size_sampled():
    """The full batch-64 workload in the launch configuration the bench times
    (automatic partitioning), checked on sampled (request, head) outputs."""
    case = workloads.llama13b_decode(seed=0, device=DEV)
    out, _ = run_decode(case)
    pairs = sample_pairs(case, 48)
    got = np.stack([out[i, h].cpu().numpy() for i, h in pairs])
    assert_parity(got, oracle_pairs(case, pairs), "llama13b full size")
    clean_error_word()


@pytest.mark.parametrize("out_dtype", [torch.float16, torch.bfloat16])
def test_low_precision_output_is_rounded_fp32(out_dtype):
    """fp16/bf16 output = round-to-nearest-even of the kernel's own fp32 result."""
    case = workloads.llama13b_decode(seed=3, device=DEV, batch=8)
    for partition in (0, -1, 256):
        f32, _ = run_decode(case, torch.float32, partition=partition)
        lp, _ = run_decode(case, out_dtype, partition=partition)
        assert torch.equal(lp.view(torch.int16), f32.to(out_dtype).view(torch.int16))
    want = oracle_full(case)
    got = lp.double().cpu().numpy()
    # rounding the output adds at most half an ulp of the output format
    ulp = 2.0 ** -10 if out_dtype == torch.float16 else 2.0 ** -7
    bound = 4e-3 + 0.5 * ulp * np.maximum(np.abs(want), 2.0 ** -14) * 2
    assert np.all(np.abs(got - want) <= bound)
    if out_dtype == torch.float16:
        assert_parity(got, want, "fp16 output")


def test_deterministic_bitwise():
    case = workloads.llama13b_decode(seed=4, device=DEV, batch=16)
    a, _ = run_decode(case)
    b, _ = run_decode(case)
    assert torch.equal(a, b)


def test_block_id_relabelling_invariance():
    """Relabel every physical block; the kernel's output must not change at all."""
    case = workloads.llama13b_decode(seed=5, device=DEV, batch=8)
    base, _ = run_decode(case)
    NB = case.k_cache.shape[0]
    pi = torch.randperm(NB, generator=torch.Generator().manual_seed(9)).to(DEV)
    k2 = torch.empty_like(case.k_cache)
    v2 = torch.empty_like(case.v_cache)
    k2[pi] = case.k_cache
    v2[pi] = case.v_cache
    bt = case.block_tables
    bt2 = torch.where(bt >= 0, pi[bt.clamp(min=0).long()].to(torch.int32), bt)
    case.k_cache, case.v_cache, case.block_tables = k2, v2, bt2
    got, _ = run_decode(case)
    assert torch.equal(got, base)


def test_edge_lengths_and_poison():
    """L = 0 (zeros), L = 1 (= V), block-boundary lengths, NaN everywhere unowned."""
    S = 16
    lens = [0, 1, S - 1, S, S + 1, 2 * S, 5 * S + 7, 1023, 1024, 1025, 3000]
    case = workloads.decode_case(lens, H=5, D=128, S=S, dtype=torch.bfloat16, seed=11,
                                 device=DEV, pool_blocks=sum(-(-L // S) for L in lens) + 17)
    for partition in (0, -1, 16, 512):
        out, _ = run_decode(case, partition=partition)
        o = out.cpu()
        assert torch.all(o[0] == 0)
        blk = case.tables_host[1][0]
        assert torch.equal(o[1], case.v_cache[blk, :, 0, :].float().cpu())
        assert_parity(o.numpy(), oracle_full(case), f"edges partition={partition}")
    clean_error_word()


@pytest.mark.parametrize("D,S", [(64, 8), (64, 32), (128, 8), (128, 32), (256, 8), (256, 16),
                                 (256, 32), (64, 16)])
@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_shapes_small(D, S, dtype):
    lens = [1, 2 * S + 3, 700, 1500, S * 9]
    case = workloads.decode_case(lens, H=3, D=D, S=S, dtype=dtype, seed=D + S, device=DEV,
                                 pool_blocks=sum(-(-L // S) for L in lens) + 5)
    want = oracle_full(case)
    for partition in (0, -1, 4 * S):
        out, _ = run_decode(case, partition=partition)
        assert_parity(out.cpu().numpy(), want, f"D={D} S={S} p={partition}")
    clean_error_word()


def test_out_of_range_block_id_is_skipped_and_flagged():
    """A table entry outside [0, NB) is never dereferenced; the error word says so."""
    case = workloads.decode_case([40, 40], H=2, D=64, S=16, dtype=torch.float16, seed=2,
                                 device=DEV)
    bt = case.block_tables.clone()
    bt[1, 1] = case.k_cache.shape[0] + 1000
    case.block_tables = bt
    out, _ = run_decode(case)
    flags = binding.pa_get_device_error()
    assert flags & binding.PA_DEVERR_BLOCK_ID
    # request 0 is untouched by the bad entry of request 1
    case.block_tables = case.block_tables.clone()
    want = oracle_pairs(case, [(0, 0), (0, 1)])
    assert_parity(out[0].cpu().numpy(), want, "unaffected request")
    clean_error_word()


def test_seq_len_past_table_is_clamped_and_flagged():
    case = workloads.decode_case([20, 30], H=2, D=64, S=16, dtype=torch.float16, seed=3,
                                 device=DEV, max_blocks=2)
    sl = case.seq_lens.clone()
    sl[0] = 1000  # beyond MB * S = 32
    case.seq_lens = sl
    run_decode(case, max_seq_len=32)
    assert binding.pa_get_device_error() & binding.PA_DEVERR_SEQ_LEN
    clean_error_word()


def test_stream_argument_is_honoured():
    case = workloads.llama13b_decode(seed=6, device=DEV, batch=4)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        out, _ = run_decode(case, stream=s)
    s.synchronize()
    ref, _ = run_decode(case)
    assert torch.equal(out, ref)
