"""Paged prefill attention (pa_prefill) against the oracle's causal prefill
("vLLM KV Cache and PagedAttention Explained", Step 6 "Prefill and Decode"):
element by element on small cases that span several 128-row query tiles and
128-key tiles with ragged tails, with and without earlier context, for every
block size, head size, cache and output dtype; sampled rows at the prompt
prefill workload's full size; and the edge cases (requests with no new tokens,
a single token, a grid wider than needed, bad table entries)."""

import numpy as np
import pytest
import torch

from helpers import (MAX_ABS, REL_L2, assert_parity, oracle_prefill_full, oracle_prefill_rows,
                     run_prefill)
from paged_kv_cache_driven_b200 import binding, workloads

pytestmark = pytest.mark.gpu
DEV = "cuda"


def check(pc, out_dtype=torch.float32, what="", **kw):
    out = run_prefill(pc, out_dtype=out_dtype, **kw)
    torch.cuda.synchronize()
    assert binding.pa_get_device_error() == 0
    want = oracle_prefill_full(pc)
    got = out.float().cpu().numpy()
    if out_dtype == torch.float32:
        return assert_parity(got, want, what)
    # a 16-bit output adds one rounding of the result
    ulp = 2.0 ** -8 if out_dtype == torch.bfloat16 else 2.0 ** -11
    assert np.all(np.isfinite(got))
    assert np.abs(got - want).max() <= MAX_ABS + ulp * np.abs(want).max(), what


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float16])
def test_prompts_tiles_and_tails(dt):
    """Plain prompts: 1 row, less than a tile, exactly one tile, one past, three
    ragged tiles."""
    pc = workloads.prefill_case([0] * 5, [1, 77, 128, 129, 300], H=3, D=128, S=16, dtype=dt,
                                seed=1, device=DEV)
    check(pc, what=f"prompts {dt}")


@pytest.mark.parametrize("S", [8, 16, 32, 64, 128])
def test_block_sizes_with_context(S):
    """Chunked prefill: new tokens after context already cached; the causal
    diagonal falls inside a key tile and inside a block."""
    pc = workloads.prefill_case([0, 13, 200, 511], [140, 60, 257, 3], H=2, D=128, S=S,
                                dtype=torch.bfloat16, seed=S, device=DEV)
    check(pc, what=f"S={S}")


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("S", [8, 32])
def test_head_dim_64(dt, S):
    pc = workloads.prefill_case([5, 0, 130], [200, 129, 66], H=4, D=64, S=S, dtype=dt, seed=7,
                                device=DEV)
    check(pc, what=f"D=64 S={S} {dt}")


@pytest.mark.parametrize("dt", [torch.bfloat16, torch.float16])
@pytest.mark.parametrize("S", [8, 16, 64, 128])
def test_head_dim_256(dt, S):
    """head_dim 256: one 128-row query tile per CTA; prompts and chunks that
    span several query and key tiles with ragged tails, with context."""
    pc = workloads.prefill_case([0, 37, 200, 0], [1, 129, 300, 256], H=2, D=256, S=S, dtype=dt,
                                seed=S + 256, device=DEV)
    check(pc, what=f"D=256 S={S} {dt}")


def test_head_dim_256_grouped_and_outputs():
    """head_dim 256 with grouped query heads (6 on 2) and 16-bit outputs."""
    pc = workloads.prefill_case([5, 0], [140, 260], H=6, D=256, S=16, dtype=torch.bfloat16,
                                seed=9, device=DEV, Hkv=2)
    check(pc, what="D=256 gqa")
    check(pc, out_dtype=torch.bfloat16, what="D=256 bf16 out")


@pytest.mark.parametrize("odt", [torch.bfloat16, torch.float16])
def test_output_dtypes(odt):
    pc = workloads.prefill_case([0, 40], [150, 90], H=2, D=128, S=16, dtype=torch.bfloat16,
                                seed=3, device=DEV)
    check(pc, out_dtype=odt, what=f"out {odt}")


def test_grouped_query_heads():
    """Eight query heads on two KV heads: query head h reads KV head h // 4."""
    pc = workloads.prefill_case([0, 100], [200, 70], H=8, D=128, S=16, dtype=torch.bfloat16,
                                seed=4, device=DEV, Hkv=2)
    check(pc, what="gqa")


def test_long_context_chunk():
    """A 256-token chunk after 3000 cached tokens (24 key tiles per query tile)."""
    pc = workloads.prefill_case([3000], [256], H=2, D=128, S=16, dtype=torch.bfloat16, seed=5,
                                device=DEV)
    check(pc, what="long context")


def test_edge_cases():
    # requests with no new tokens produce no rows and disturb nothing
    pc = workloads.prefill_case([10, 0, 64, 0], [0, 33, 0, 1], H=2, D=128, S=16,
                                dtype=torch.bfloat16, seed=6, device=DEV)
    check(pc, what="empty requests")
    # a grid wider than the longest request
    check(pc, what="wide grid", max_q_len=1000)
    # nothing to do
    empty = torch.empty((0, 2, 128), dtype=torch.float32, device=DEV)
    c = pc.cache
    binding.pa_prefill(empty, pc.q[:0], c.k_cache, c.v_cache, c.block_tables, c.seq_lens,
                       torch.zeros(5, dtype=torch.int32, device=DEV), c.scale, 0)
    assert binding.pa_get_device_error() == 0


def test_bad_inputs_are_flagged():
    pc = workloads.prefill_case([0, 20], [40, 50], H=2, D=128, S=16, dtype=torch.bfloat16,
                                seed=8, device=DEV)
    c = pc.cache
    good = run_prefill(pc)
    # a table entry outside the pool: flagged; the other request is unaffected
    bt = c.block_tables.clone()
    bt[0, 1] = c.k_cache.shape[0] + 3
    out = torch.full_like(good, 7.0)
    binding.pa_prefill(out, pc.q, c.k_cache, c.v_cache, bt, c.seq_lens, pc.q_start, c.scale,
                       pc.max_q_len)
    assert binding.pa_get_device_error() & binding.PA_DEVERR_BLOCK_ID
    assert torch.equal(out[40:], good[40:])
    # more new tokens than cached ones: that request is skipped and flagged
    lens = c.seq_lens.clone()
    lens[1] = 10
    out = torch.full_like(good, 7.0)
    binding.pa_prefill(out, pc.q, c.k_cache, c.v_cache, c.block_tables, lens, pc.q_start,
                       c.scale, pc.max_q_len)
    assert binding.pa_get_device_error() & binding.PA_DEVERR_SEQ_LEN
    assert torch.equal(out[:40], good[:40]) and bool((out[40:] == 7.0).all())
    # max_q_len below a request's new tokens: flagged, not silently truncated
    binding.pa_prefill(out, pc.q, c.k_cache, c.v_cache, c.block_tables, c.seq_lens, pc.q_start,
                       c.scale, 45)
    assert binding.pa_get_device_error() & binding.PA_DEVERR_SEQ_LEN
    # host-side checks launch nothing: an unsupported block size, a scale <= 0
    NB, H, S, D = c.k_cache.shape
    small = c.k_cache.new_zeros((NB, H, 4, D))
    with pytest.raises(binding.PagedAttnError):
        binding.pa_prefill(out, pc.q, small, small, c.block_tables, c.seq_lens, pc.q_start,
                           c.scale, pc.max_q_len)
    with pytest.raises(binding.PagedAttnError):
        binding.pa_prefill(out, pc.q, c.k_cache, c.v_cache, c.block_tables, c.seq_lens,
                           pc.q_start, 0.0, pc.max_q_len)


def test_prompt_prefill_full_size_sampled():
    """The prompt prefill workload (16 prompts of U[512, 4096] tokens, 32 heads,
    head_dim 128, block 16, bf16) in the launch the benchmark times; sampled
    rows: first and last rows of the longest and shortest prompts, rows at tile
    edges, random ones."""
    pc = workloads.prompt_prefill(device=DEV)
    out = run_prefill(pc)
    torch.cuda.synchronize()
    assert binding.pa_get_device_error() == 0
    g = torch.Generator().manual_seed(0)
    order = sorted(range(len(pc.new_lens)), key=lambda i: pc.new_lens[i])
    picks = []
    for i in (order[0], order[-1]):
        n = pc.new_lens[i]
        for j in (0, 127, 128, n - 1):
            picks.append((i, min(j, n - 1), int(torch.randint(0, 32, (1,), generator=g))))
    while len(picks) < 48:
        i = int(torch.randint(0, len(pc.new_lens), (1,), generator=g))
        j = int(torch.randint(0, pc.new_lens[i], (1,), generator=g))
        picks.append((i, j, int(torch.randint(0, 32, (1,), generator=g))))
    want = oracle_prefill_rows(pc, picks)
    qs = pc.q_start.cpu().tolist()
    got = torch.stack([out[qs[i] + j, h] for i, j, h in picks]).cpu().numpy()
    assert_parity(got, want, "prompt prefill sampled rows")
    assert bool(torch.isfinite(out).all())


@pytest.mark.parametrize("dt,Hkv", [(torch.float16, 32), (torch.bfloat16, 8)],
                         ids=["fp16", "gqa_64q_8kv"])
def test_chunked_prefill_large_sampled(dt, Hkv):
    """Chunked prefill at scale: 8 requests with U[0, 6000] cached tokens and
    U[300, 2500] new ones, head_dim 128, block 16; fp16 with 32 heads, and 64
    query heads on 8 KV heads (LLaMA-2-70B-shaped groups). Sampled rows against
    the oracle's decode of the row's prefix."""
    g = torch.Generator().manual_seed(11)
    ctx = torch.randint(0, 6001, (8,), generator=g).tolist()
    new = torch.randint(300, 2501, (8,), generator=g).tolist()
    H = 32 if Hkv == 32 else 64
    pc = workloads.prefill_case(ctx, new, H=H, D=128, S=16, dtype=dt, seed=12, device=DEV,
                                Hkv=Hkv)
    out = run_prefill(pc)
    torch.cuda.synchronize()
    assert binding.pa_get_device_error() == 0
    picks = []
    for i in range(8):
        for j in (0, new[i] - 1, int(torch.randint(0, new[i], (1,), generator=g))):
            picks.append((i, j, int(torch.randint(0, H, (1,), generator=g))))
    want = oracle_prefill_rows(pc, picks)
    qs = pc.q_start.cpu().tolist()
    got = torch.stack([out[qs[i] + j, h] for i, j, h in picks]).cpu().numpy()
    assert_parity(got, want, f"chunked prefill {dt} Hkv={Hkv}")
    assert bool(torch.isfinite(out).all())


@pytest.mark.parametrize("v_scale", [1.0, 2.0 ** 20, 2.0 ** -8, 2.0 ** 30, 2.0 ** -14])
def test_bf16_value_magnitudes(v_scale):
    """bf16 caches with V from 2^-14 to 2^30 times N(0, 1): every scale matches
    the oracle relative to the scale of V (the output is linear in V),
    including context, ragged tiles and a key tile past the end."""
    pc = workloads.prefill_case([0, 37, 300], [140, 200, 66], H=2, D=128, S=16,
                                dtype=torch.bfloat16, seed=11, device=DEV)
    c = pc.cache
    c.v_cache.copy_((c.v_cache.float() * v_scale).to(torch.bfloat16))
    out = run_prefill(pc)
    torch.cuda.synchronize()
    assert binding.pa_get_device_error() == 0
    want = oracle_prefill_full(pc)
    assert_parity(out.cpu().numpy() / v_scale, want / v_scale, f"V x {v_scale}")


def test_bf16_mixed_tile_modes():
    """One request whose V tiles (128 tokens each) alternate between 2^18 and
    2^28 times N(0, 1), so that rows mix key tiles of very different
    magnitude."""
    pc = workloads.prefill_case([0], [600], H=2, D=128, S=16, dtype=torch.bfloat16, seed=12,
                                device=DEV)
    c = pc.cache
    S = c.k_cache.shape[2]
    table = c.tables_host[0]
    c.v_cache.copy_((c.v_cache.float() * 2.0 ** 18).to(torch.bfloat16))
    for j in range(0, 600, 256):  # tokens j .. j + 127 of every other key tile: x 2^10 more
        for blk in table[j // S:(j + 128) // S]:
            c.v_cache[blk] = (c.v_cache[blk].float() * 2.0 ** 10).to(torch.bfloat16)
    out = run_prefill(pc)
    torch.cuda.synchronize()
    assert binding.pa_get_device_error() == 0
    want = oracle_prefill_full(pc)
    scale = float(np.abs(want).max())
    assert_parity(out.cpu().numpy() / scale, want / scale, "mixed tile modes")
