"""Pins for the allocator model and the waste arithmetic (CPU only).

Each expected value below is printed by the pages (tests/golden/worked_example.txt,
with its citation) or follows from the ceiling definition by brute force.
"""

import os
import random

import pytest

from oracle.allocator_model import INVALID, OOM, OUT_OF_RANGE, BlockPoolModel, PoolError
from oracle import waste

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example.txt")


def golden():
    vals = {}
    with open(GOLDEN) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if not line:
                continue
            k, v = (x.strip() for x in line.split("=", 1))
            parts = v.split()
            vals[k] = [float(p) if "." in p else int(p) for p in parts]
            if len(parts) == 1:
                vals[k] = vals[k][0]
    return vals


G = golden()


def test_worked_example_blocks_and_waste():
    """6단계: 6/50/8/100 tokens -> 1/4/1/7 = 13 blocks; requests 1 and 3 waste 10 and 8."""
    S = G["block_size"]
    pool = BlockPoolModel(64, S)
    for i, L in enumerate(G["seq_lens"]):
        pool.grow(i, L)
    counts = [len(pool.block_table(i)) for i in range(4)]
    assert counts == G["paged_blocks_per_request"]
    assert sum(counts) == G["paged_total_blocks"]
    blocks, tail = waste.paged_allocation(G["seq_lens"], S)
    assert blocks == counts
    assert tail[0] == G["annotated_waste_slots_request1"]
    assert tail[2] == G["annotated_waste_slots_request3"]
    # The page's "18 slots" is the sum of the two annotated requests; the true
    # total over all four is 13 * 16 - 164 = 44 (recorded, not corrected).
    assert tail[0] + tail[2] == G["paged_waste_slots"]
    assert tail == [10, 14, 8, 12] and sum(tail) == 44
    free, used, wasted = pool.stats()
    assert (free, used, wasted) == (64 - 13, 164, 44)


def test_worked_example_identity_order_matches_5단계():
    """5단계: request A gets block 0 and request B starts at blocks 1, 2, 3.

    The page lists only three blocks for B's 50 tokens, against its own 6단계
    (four blocks) and ceil(50/16) = 4; the model gives B a fourth block.
    """
    pool = BlockPoolModel(64, 16)
    pool.grow("A", 6)
    pool.grow("B", 50)
    assert pool.block_table("A") == [0]
    assert pool.block_table("B")[:3] == [1, 2, 3]
    assert len(pool.block_table("B")) == 4


def test_waste_arithmetic_matches_page():
    """6단계: 0.78 MB per token, 1.6 GB per reservation, 6.4 GB total, ~127 MB used,
    ~6.27 GB (98%) wasted; paged 13 blocks ~162 MB, 18 slots ~14 MB, ~9%."""
    per_tok = waste.kv_bytes_per_token(layers=40, hidden=5120, bytes_per_elem=2)
    assert per_tok == 819200
    mib = per_tok / 2**20
    assert round(mib, 2) == G["kv_mb_per_token"]
    mb = G["kv_mb_per_token"]  # the page's rounded figure, used for its own arithmetic
    lens = G["seq_lens"]
    reserved, used, wasted = waste.static_reservation(lens, G["max_model_len"], mb)
    assert round(G["max_model_len"] * mb / 1000, 1) == G["static_gb_per_request"]
    assert round(reserved / 1000, 1) == G["static_total_gb"]
    assert int(used) == G["static_used_mb"]
    assert round((G["static_total_gb"] * 1000 - G["static_used_mb"]) / 1000, 2) == G["static_waste_gb"]
    assert round(100 * wasted / reserved) == G["static_waste_pct"]
    blocks, _ = waste.paged_allocation(lens, G["block_size"])
    total_mb = sum(blocks) * G["block_size"] * mb
    assert round(total_mb) == G["paged_total_mb"]
    waste_mb = G["paged_waste_slots"] * mb
    assert round(waste_mb) == G["paged_waste_mb"]
    assert round(100 * waste_mb / total_mb) == G["paged_waste_pct"]
    # With the true 44 tail slots the paged waste would be 21%.
    assert round(100 * 44 * mb / total_mb) == 21


@pytest.mark.parametrize("S", [8, 16, 32])
def test_blocks_needed_brute_force(S):
    """ceil(len/S) blocks, growth exactly when a token starts a new block."""
    pool = BlockPoolModel(8, S)
    prev = 0
    for L in range(0, 4 * S + 1):
        pool.grow("r", L)
        n = len(pool.block_table("r"))
        # brute force: count the distinct blocks the tokens 0..L-1 fall into
        assert n == len({t // S for t in range(L)})
        grew = n - prev
        assert grew == (1 if (L >= 1 and L % S == 1) or (S == 1 and L >= 1) else 0)
        prev = n


def test_page_block_boundary_examples():
    S = G["block_size"]
    pool = BlockPoolModel(8, S)
    pool.grow("a", 6)
    assert len(pool.block_table("a")) == G["prefill_blocks_for_6_tokens"]
    pool.grow("a", G["first_token_of_second_block"] - 1)
    assert len(pool.block_table("a")) == 1
    pool.grow("a", G["first_token_of_second_block"])
    assert len(pool.block_table("a")) == 2
    assert waste.paged_allocation([32], S)[1] == [G["waste_32_tokens"]]
    assert waste.paged_allocation([17], S)[1] == [G["waste_17_tokens"]]


def test_max_waste_and_mean_waste_property():
    """Step 5: at most block_size - 1 slots per request; the mean stays under half a block."""
    rng = random.Random(0)
    S = 16
    lens = [rng.randint(1, 5000) for _ in range(20000)]
    _, tail = waste.paged_allocation(lens, S)
    assert max(tail) == G["max_waste_slots"] == S - 1
    assert min(tail) == 0
    assert sum(tail) / len(tail) < S / 2


def test_page_slots_in_block_42():
    """Step 5/7: prompt tokens in slots 0-5 of block 42, the first decoded token in slot 6."""
    S = G["block_size"]
    order = [G["example_block"]] + [b for b in range(64) if b != G["example_block"]]
    pool = BlockPoolModel(64, S, initial_order=order)
    pool.grow("req", 6)
    assert pool.block_table("req") == [G["example_block"]]
    slots = pool.slot_mapping(["req"], [0], [6])
    assert slots == [G["example_block"] * S + o for o in G["example_prompt_slots"]]
    pool.grow("req", 7)
    assert pool.slot_mapping(["req"], [6], [1]) == [G["example_block"] * S + G["example_decode_slot"]]


def test_page_request_b_blocks():
    """Step 5: any free blocks serve; logical 0/1/2 -> physical 7/23/61."""
    want = G["example_request_b_blocks"]
    order = want + [b for b in range(100) if b not in want]
    pool = BlockPoolModel(100, 16, initial_order=order)
    pool.grow("B", 40)
    assert pool.block_table("B") == want
    assert pool.block_tables(["B"], 5) == [want + [-1, -1]]


def test_free_then_reuse_lifo():
    """Step 7 item 7: a released block can be handed to the very next request."""
    pool = BlockPoolModel(16, 16)
    pool.grow("a", 40)  # blocks 0, 1, 2
    pool.grow("b", 5)   # block 3
    ta = pool.block_table("a")
    pool.release("a")
    pool.grow("c", 20)  # two blocks: the last two pushed come back first
    assert pool.block_table("c") == [ta[2], ta[1]]
    pool.grow("d", 1)
    assert pool.block_table("d") == [ta[0]]
    assert sorted(pool.dump() + pool.block_table("b") + pool.block_table("c")
                  + pool.block_table("d")) == list(range(16))


def test_oom_leaves_state_unchanged():
    pool = BlockPoolModel(4, 16)
    pool.grow("a", 33)  # 3 blocks
    before = (pool.dump(), pool.block_table("a"), pool.stats())
    with pytest.raises(PoolError) as e:
        pool.grow("b", 17)  # needs 2, one left
    assert e.value.code == OOM
    assert (pool.dump(), pool.block_table("a"), pool.stats()) == before
    assert "b" not in pool.tables


def test_errors():
    pool = BlockPoolModel(4, 16)
    pool.grow("a", 10)
    with pytest.raises(PoolError) as e:
        pool.grow("a", 5)
    assert e.value.code == INVALID
    with pytest.raises(PoolError) as e:
        pool.slot_mapping(["a"], [5], [6])
    assert e.value.code == OUT_OF_RANGE
    with pytest.raises(PoolError) as e:
        pool.release("zz")
    assert e.value.code == INVALID
    with pytest.raises(PoolError):
        BlockPoolModel(4, 16, initial_order=[0, 1, 1, 3])


def test_pool_conservation_random_walk():
    """Invariant: free + held blocks always partition the pool; held = sum ceil(len/S)."""
    rng = random.Random(1)
    S, NB = 8, 200
    order = list(range(NB))
    rng.shuffle(order)
    pool = BlockPoolModel(NB, S, initial_order=order)
    live = {}
    for step in range(3000):
        op = rng.random()
        if op < 0.5 and live:
            sid = rng.choice(list(live))
            new = live[sid] + rng.randint(0, 20)
            try:
                pool.grow(sid, new)
                live[sid] = new
            except PoolError as e:
                assert e.code == OOM
        elif op < 0.7 and live:
            sid = rng.choice(list(live))
            pool.release(sid)
            del live[sid]
        else:
            sid = step
            L = rng.randint(0, 60)
            try:
                pool.grow(sid, L)
                live[sid] = L
            except PoolError as e:
                assert e.code == OOM
        held = [b for t in pool.tables.values() for b in t]
        assert sorted(held + pool.dump()) == list(range(NB))
        assert len(held) == sum(-(-L // S) for L in live.values())


# ---------------------------------------------------------------------------
# Prefix sharing and copy-on-write ("vLLM KV Cache and PagedAttention
# Explained", Step 9 "Safe Sharing with Copy-on-Write").
# ---------------------------------------------------------------------------

def _order_first(*ids, n=100):
    return list(ids) + [b for b in range(n) if b not in ids]


def test_shared_prefix_block_refcount_three():
    """A system prompt of 8 tokens in physical block 5, shared by requests A, B
    and C: reference count 3, all three tables name block 5."""
    pool = BlockPoolModel(100, 16, initial_order=_order_first(5))
    pool.grow("prompt", 8)
    assert pool.block_table("prompt") == [5]
    for r in "ABC":
        pool.fork("prompt", r)
    pool.release("prompt")
    assert pool.refs[5] == 3
    assert [pool.block_table(r) for r in "ABC"] == [[5], [5], [5]]
    assert 5 not in pool.dump()


def test_page_tables_for_a_block_aligned_prefix():
    """Step 9's tables: block 5 shared, logical block 1 private per request
    (12, 37, 61). They arise when the shared prefix fills its block, so each
    request's own tokens start a new block and nothing is copied."""
    pool = BlockPoolModel(100, 16, initial_order=_order_first(5, 12, 37, 61))
    pool.grow("prompt", 16)
    for r in "ABC":
        pool.fork("prompt", r)
    pool.release("prompt")
    for r in "ABC":
        pool.grow(r, 17)
    assert [pool.block_table(r) for r in "ABC"] == [[5, 12], [5, 37], [5, 61]]
    assert pool.refs[5] == 3 and pool.take_copies() == []


def test_copy_on_write_repoints_only_the_writer():
    """Writing into the shared, partly filled block copies it for the writer;
    the others keep block 5; the last holder writes in place."""
    pool = BlockPoolModel(100, 16, initial_order=_order_first(5, 40, 41))
    pool.grow("prompt", 8)
    for r in "ABC":
        pool.fork("prompt", r)
    pool.release("prompt")
    pool.grow("A", 9)                       # A's 9th token goes into block 5's slot 8
    assert pool.block_table("A") == [40] and pool.take_copies() == [(5, 40)]
    assert pool.block_table("B") == [5] and pool.block_table("C") == [5] and pool.refs[5] == 2
    pool.grow("B", 10)
    assert pool.block_table("B") == [41] and pool.take_copies() == [(5, 41)]
    pool.grow("C", 9)                       # only C still names block 5: no copy
    assert pool.block_table("C") == [5] and pool.take_copies() == [] and pool.refs[5] == 1
    assert pool.slot_mapping(["C"], [8], [1]) == [5 * 16 + 8]
    for r in "ABC":
        pool.release(r)
    assert sorted(pool.dump()) == list(range(100)) and set(pool.refs) == {0}


def test_parallel_sampling_saves_blocks():
    """n samples forked from one prompt hold the prompt's full blocks once."""
    S, prompt, n, gen = 16, 1000, 8, 100
    shared = BlockPoolModel(1000, S)
    shared.grow("p", prompt)
    for k in range(n):
        shared.fork("p", k)
    shared.release("p")
    for k in range(n):
        shared.grow(k, prompt + gen)
    private = BlockPoolModel(1000, S)
    for k in range(n):
        private.grow(k, prompt + gen)
    used_shared = 1000 - len(shared.free)
    used_private = 1000 - len(private.free)
    full_prompt_blocks = prompt // S
    assert used_private - used_shared == (n - 1) * full_prompt_blocks
    assert len(shared.take_copies()) == n - 1   # the partly filled prompt block, per writer but the last


def test_cow_counts_in_oom_and_leaves_state_unchanged():
    pool = BlockPoolModel(2, 16)
    pool.grow("p", 8)
    pool.fork("p", "q")
    pool.grow("x", 16)          # the pool is now empty
    before = (pool.dump(), dict(pool.tables), list(pool.refs))
    with pytest.raises(PoolError) as e:
        pool.grow("q", 9)       # needs a private copy of the shared block
    assert e.value.code == OOM
    assert (pool.dump(), dict(pool.tables), list(pool.refs)) == before
