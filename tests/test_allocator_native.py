"""The library's C++ block allocator against the oracle's Python model: every
table, slot mapping, statistic and the free list itself must match bit for bit
(CPU only; the allocator never touches the GPU)."""

import random

import pytest
import torch

from oracle.allocator_model import OOM, BlockPoolModel, PoolError
from paged_kv_cache_driven_b200 import binding
from paged_kv_cache_driven_b200.binding import BlockAllocator, PagedAttnError


def same_state(native, model, seq_ids):
    assert native.pa_alloc_dump() == model.dump()
    assert native.pa_alloc_stats() == model.stats()
    for sid in seq_ids:
        assert native.pa_seq_block_table(sid) == model.block_table(sid)
        assert native.pa_seq_len(sid) == model.lens[sid]


def test_worked_example_native():
    """6단계: 6/50/8/100 tokens -> 1/4/1/7 = 13 blocks, 44 empty tail slots."""
    a = BlockAllocator(64, 16)
    m = BlockPoolModel(64, 16)
    for i, L in enumerate([6, 50, 8, 100]):
        a.pa_seq_grow(i, L)
        m.grow(i, L)
    assert [len(a.pa_seq_block_table(i)) for i in range(4)] == [1, 4, 1, 7]
    assert a.pa_alloc_stats() == (51, 164, 44)
    same_state(a, m, range(4))


def test_block_42_slots_native():
    order = [42] + [b for b in range(64) if b != 42]
    a = BlockAllocator(64, 16, initial_order=order)
    a.pa_seq_grow(7, 6)
    assert a.pa_build_slot_mapping([7], [0], [6]).tolist() == [42 * 16 + k for k in range(6)]
    a.pa_seq_grow(7, 7)
    assert a.pa_build_slot_mapping([7], [6], [1]).tolist() == [42 * 16 + 6]


def test_errors_match_model():
    a = BlockAllocator(4, 16)
    a.pa_seq_grow(1, 33)
    with pytest.raises(PagedAttnError) as e:
        a.pa_seq_grow(2, 17)
    assert e.value.code == binding.PA_ERR_OOM
    with pytest.raises(PagedAttnError) as e:
        a.pa_seq_grow(1, 10)
    assert e.value.code == binding.PA_ERR_INVALID
    with pytest.raises(PagedAttnError) as e:
        a.pa_build_slot_mapping([1], [30], [5])
    assert e.value.code == binding.PA_ERR_OUT_OF_RANGE
    with pytest.raises(PagedAttnError) as e:
        a.pa_seq_free(99)
    assert e.value.code == binding.PA_ERR_INVALID
    with pytest.raises(PagedAttnError) as e:
        a.pa_build_block_tables([1], 2)
    assert e.value.code == binding.PA_ERR_OUT_OF_RANGE
    with pytest.raises(PagedAttnError):
        BlockAllocator(4, 16, initial_order=[0, 1, 2, 2])
    with pytest.raises(PagedAttnError):
        a.pa_prepare_step([1, 1], 1, 8)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_random_walk_bit_exact(seed):
    rng = random.Random(seed)
    S = rng.choice([8, 16, 32])
    NB = 300
    order = list(range(NB))
    rng.shuffle(order)
    a = BlockAllocator(NB, S, initial_order=order)
    m = BlockPoolModel(NB, S, initial_order=order)
    live = {}
    next_id = 0
    for step in range(1500):
        op = rng.random()
        if op < 0.45 and live:
            sid = rng.choice(sorted(live))
            new = live[sid] + rng.randint(0, 3 * S)
            try:
                m.grow(sid, new)
                exp = None
            except PoolError as e:
                exp = e.code
            if exp is None:
                a.pa_seq_grow(sid, new)
                live[sid] = new
            else:
                with pytest.raises(PagedAttnError) as e:
                    a.pa_seq_grow(sid, new)
                assert e.value.code == exp == OOM
        elif op < 0.65 and live:
            sid = rng.choice(sorted(live))
            a.pa_seq_free(sid)
            m.release(sid)
            del live[sid]
        elif op < 0.8 and live:
            ids = rng.sample(sorted(live), min(len(live), rng.randint(1, 6)))
            n_new = rng.randint(1, 2)
            MB = max(-(-(live[s] + n_new) // S) for s in ids) + rng.randint(0, 2)
            slots = torch.empty(len(ids) * n_new, dtype=torch.int64)
            tables = torch.empty((len(ids), MB), dtype=torch.int32)
            lens = torch.empty(len(ids), dtype=torch.int32)
            # the model: all-or-nothing growth, then slots / tables / lengths
            need = sum(-(-(live[s] + n_new) // S) - len(m.tables[s]) for s in ids)
            if need > len(m.free):
                with pytest.raises(PagedAttnError) as e:
                    a.pa_prepare_step(ids, n_new, MB, slots, tables, lens)
                assert e.value.code == binding.PA_ERR_OOM
            else:
                a.pa_prepare_step(ids, n_new, MB, slots, tables, lens)
                want_slots = []
                for s in ids:
                    m.grow(s, live[s] + n_new)
                    want_slots += m.slot_mapping([s], [live[s]], [n_new])
                    live[s] += n_new
                assert slots.tolist() == want_slots
                assert tables.tolist() == m.block_tables(ids, MB)
                assert lens.tolist() == [live[s] for s in ids]
        else:
            sid = next_id
            next_id += 1
            L = rng.randint(0, 10 * S)
            try:
                m.grow(sid, L)
                a.pa_seq_grow(sid, L)
                live[sid] = L
            except PoolError:
                with pytest.raises(PagedAttnError):
                    a.pa_seq_grow(sid, L)
        if step % 50 == 0 or step > 1450:
            same_state(a, m, live)
            if live:
                ids = sorted(live)
                MB = max(len(m.tables[s]) for s in ids) + 1
                assert a.pa_build_block_tables(ids, MB).tolist() == m.block_tables(ids, MB)
                starts = [rng.randint(0, live[s]) for s in ids]
                ns = [rng.randint(0, live[s] - p) for s, p in zip(ids, starts)]
                assert a.pa_build_slot_mapping(ids, starts, ns).tolist() == \
                    m.slot_mapping(ids, starts, ns)


def same_sharing_state(native, model):
    assert native.pa_alloc_refcounts() == model.refs
    got = native.pa_alloc_take_copies().tolist()
    assert [tuple(x) for x in got] == model.take_copies()


def test_copy_on_write_page_example_native():
    order = [5, 40, 41] + [b for b in range(100) if b not in (5, 40, 41)]
    a = BlockAllocator(100, 16, initial_order=order)
    m = BlockPoolModel(100, 16, initial_order=order)
    for x in (a, m):
        (x.pa_seq_grow if x is a else x.grow)(0, 8)
    for r in (1, 2, 3):
        a.pa_seq_fork(0, r)
        m.fork(0, r)
    a.pa_seq_free(0)
    m.release(0)
    assert a.pa_alloc_refcounts()[5] == 3
    a.pa_seq_grow(1, 9)
    m.grow(1, 9)
    assert a.pa_seq_block_table(1) == [40] and a.pa_seq_block_table(2) == [5]
    same_sharing_state(a, m)
    same_state(a, m, [1, 2, 3])
    with pytest.raises(PagedAttnError) as e:
        a.pa_seq_fork(99, 7)
    assert e.value.code == binding.PA_ERR_INVALID
    with pytest.raises(PagedAttnError) as e:
        a.pa_seq_fork(1, 2)
    assert e.value.code == binding.PA_ERR_INVALID


@pytest.mark.parametrize("seed", [3, 4, 5])
def test_random_walk_with_forks_bit_exact(seed):
    rng = random.Random(seed)
    S = rng.choice([8, 16, 32])
    NB = 400
    order = list(range(NB))
    rng.shuffle(order)
    a = BlockAllocator(NB, S, initial_order=order)
    m = BlockPoolModel(NB, S, initial_order=order)
    live = {}
    next_id = 0
    for step in range(1500):
        op = rng.random()
        if op < 0.15 and live:  # fork
            parent = rng.choice(sorted(live))
            child = next_id
            next_id += 1
            a.pa_seq_fork(parent, child)
            m.fork(parent, child)
            live[child] = live[parent]
        elif op < 0.5 and live:  # grow (may copy on write)
            sid = rng.choice(sorted(live))
            new = live[sid] + rng.randint(1, S + 2)
            try:
                m.grow(sid, new)
            except PoolError as e:
                with pytest.raises(PagedAttnError) as ee:
                    a.pa_seq_grow(sid, new)
                assert ee.value.code == e.code
            else:
                a.pa_seq_grow(sid, new)
                live[sid] = new
        elif op < 0.65 and live:  # one decode step for a few sequences
            ids = rng.sample(sorted(live), min(len(live), rng.randint(1, 5)))
            MB = max(-(-(live[s] + 1) // S) for s in ids) + 1
            slots = torch.empty(len(ids), dtype=torch.int64)
            tables = torch.empty((len(ids), MB), dtype=torch.int32)
            lens = torch.empty(len(ids), dtype=torch.int32)
            need = sum(-(-(live[s] + 1) // S) - len(m.tables[s]) + (1 if m._cow_needed(s, live[s] + 1) else 0)
                       for s in ids)
            if need > len(m.free):
                with pytest.raises(PagedAttnError):
                    a.pa_prepare_step(ids, 1, MB, slots, tables, lens)
            else:
                a.pa_prepare_step(ids, 1, MB, slots, tables, lens)
                want = []
                for s in ids:
                    m.grow(s, live[s] + 1)
                    want += m.slot_mapping([s], [live[s]], [1])
                    live[s] += 1
                assert slots.tolist() == want
                assert tables.tolist() == m.block_tables(ids, MB)
        elif op < 0.8 and live:
            sid = rng.choice(sorted(live))
            a.pa_seq_free(sid)
            m.release(sid)
            del live[sid]
        else:
            sid = next_id
            next_id += 1
            L = rng.randint(0, 6 * S)
            try:
                m.grow(sid, L)
            except PoolError:
                with pytest.raises(PagedAttnError):
                    a.pa_seq_grow(sid, L)
            else:
                a.pa_seq_grow(sid, L)
                live[sid] = L
        if step % 25 == 0:
            same_state(a, m, live)
            same_sharing_state(a, m)
            # every block is free or named by a table, with the right count
            counts = [0] * NB
            for t in m.tables.values():
                for b in t:
                    counts[b] += 1
            assert counts == m.refs
            assert sorted(set(b for t in m.tables.values() for b in t) | set(m.dump())) == \
                list(range(NB))


def test_check_slots_host():
    """The host-side slot check: duplicates and slots past the pool are refused
    (the append kernels do not detect duplicates), padding is allowed, and every
    slot mapping the allocator builds passes."""
    ok = torch.tensor([5, -1, 7, 0, -1, 63], dtype=torch.int64)
    binding.pa_check_slots(ok, 64)
    binding.pa_check_slots(torch.empty(0, dtype=torch.int64), 64)
    with pytest.raises(PagedAttnError) as e:
        binding.pa_check_slots(torch.tensor([5, 9, 5], dtype=torch.int64), 64)
    assert e.value.code == binding.PA_ERR_INVALID and "entry 2" in str(e.value)
    with pytest.raises(PagedAttnError) as e:
        binding.pa_check_slots(torch.tensor([5, 64], dtype=torch.int64), 64)
    assert e.value.code == binding.PA_ERR_OUT_OF_RANGE and "entry 1" in str(e.value)
    a = BlockAllocator(64, 16)
    for sid, L in enumerate([6, 50, 8, 100]):
        a.pa_seq_grow(sid, L)
    slots = a.pa_build_slot_mapping([0, 1, 2, 3], [0, 0, 0, 0], [6, 50, 8, 100])
    binding.pa_check_slots(slots, 64 * 16)
