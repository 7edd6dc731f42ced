"""The continuous-batching loop (40 heads, head_dim 128, bf16, lognormal prompts,
geometric stops, shuffled free list) against an oracle mirror that replays the
same random draws with the oracle's allocator model, numpy scatter and fp64
decode. Allocator state, block tables and slot mappings are compared bit for
bit every step; the cache bit for bit and the decode output at the tolerance
on the mirrored heads."""

import numpy as np
import pytest
import torch

from helpers import assert_parity
from oracle import append as oracle_append
from oracle import decode as oracle_decode
from oracle.allocator_model import BlockPoolModel
from paged_kv_cache_driven_b200 import binding, workloads
from paged_kv_cache_driven_b200.batching import ContinuousBatching

pytestmark = pytest.mark.gpu
DEV = "cuda"


def host_bits(t, heads):
    return t[:, heads].contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


class OracleMirror:
    """Replays the loop with oracle components, for the heads in ``heads``."""

    def __init__(self, loop, heads, MB):
        self.loop, self.heads, self.MB = loop, list(heads), MB
        NB, S, D = loop.num_blocks, loop.S, loop.D
        self.model = BlockPoolModel(NB, S, initial_order=loop.block_order)
        nan_bits = torch.tensor([float("nan")], dtype=loop.dtype).view(torch.int16).numpy().view(np.uint16)[0]
        self.kc = np.full((NB, len(self.heads), S, D), nan_bits, np.uint16)
        self.vc = np.full((NB, len(self.heads), S, D), nan_bits, np.uint16)
        self.budget = {}
        self.batch = []
        for b in range(loop.batch):
            self.admit(b, loop.initial_lens[b], loop.budgets[b])

    def admit(self, sid, L, budget):
        self.model.grow(sid, L)
        slots = self.model.slot_mapping([sid], [0], [L])
        k, v = self.loop.prompt_kv(sid, L, DEV)
        oracle_append.scatter_into(host_bits(k, self.heads), host_bits(v, self.heads), slots,
                                   self.kc, self.vc)
        self.budget[sid] = max(1, int(budget))
        return sid

    def step(self, rec, check):
        ids = rec["ids"]
        starts = [self.model.lens[s] for s in ids]
        for s in ids:
            self.model.grow(s, self.model.lens[s] + 1)
        slots = self.model.slot_mapping(ids, starts, [1] * len(ids))
        assert rec["slots"].tolist() == slots
        assert rec["lens"].tolist() == [self.model.lens[s] for s in ids]
        assert rec["tables"].tolist() == self.model.block_tables(ids, self.MB)
        oracle_append.scatter_into(host_bits(rec["k"], self.heads), host_bits(rec["v"], self.heads),
                                   slots, self.kc, self.vc)
        # decode of the mirrored heads, through the model's tables
        q = host_bits(rec["q"], self.heads)
        bt = np.array(self.model.block_tables(ids, self.MB), dtype=np.int32)
        lens = np.array([self.model.lens[s] for s in ids], dtype=np.int32)
        want = None
        if check:
            want = oracle_decode.paged_decode(q, self.kc, self.vc, bt, lens,
                                              1.0 / np.sqrt(self.loop.D), dtype=self.loop.dtype)
        # retirements and admissions, in batch-slot order
        retired, admitted = [], iter(rec["admitted"])
        for s in ids:
            self.budget[s] -= 1
            if self.budget[s] == 0:
                self.model.release(s)
                del self.budget[s]
                retired.append(s)
                sid, L, budget = next(admitted)
                self.admit(sid, L, budget)
        assert retired == rec["retired"]
        return want


def run_loop(batch, H, steps, check_steps, heads, seed, fused=False):
    loop = workloads.batching_loop(seed=seed, batch=batch, H=H)
    drv = ContinuousBatching(loop, DEV, max_steps=steps, fused=fused)
    mirror = OracleMirror(loop, heads, drv.MB)
    assert drv.alloc.pa_alloc_dump() == mirror.model.dump()
    n_retired = 0
    for step in range(steps):
        rec = drv.step(step)
        out = rec["out"][:, heads].cpu().numpy()
        want = mirror.step(rec, step in check_steps)
        n_retired += len(rec["retired"])
        assert drv.alloc.pa_alloc_dump() == mirror.model.dump()
        assert drv.alloc.pa_alloc_stats() == mirror.model.stats()
        if step in check_steps:
            assert_parity(out, want, f"step {step}")
            torch.cuda.synchronize()
            assert np.array_equal(host_bits(drv.k_cache, heads), mirror.kc), f"K cache, step {step}"
            assert np.array_equal(host_bits(drv.v_cache, heads), mirror.vc), f"V cache, step {step}"
    assert binding.pa_get_device_error() == 0
    return n_retired


@pytest.mark.parametrize("fused", [False, True], ids=["two_calls", "fused"])
def test_batching_loop_reduced_every_step(fused):
    """Batch 16, 4 heads, 64 steps: every output, every cache byte, every step."""
    n = run_loop(batch=16, H=4, steps=64, check_steps=set(range(64)), heads=[0, 1, 2, 3], seed=1,
                 fused=fused)
    assert n > 0  # some requests retired and were replaced


@pytest.mark.parametrize("fused", [False, True], ids=["two_calls", "fused"])
def test_batching_loop_full_size(fused):
    """Batch 256, 40 heads, a 66,560-block shuffled pool, 64 steps: allocator state
    every step; cache and decode on two mirrored heads at three steps."""
    n = run_loop(batch=256, H=40, steps=64, check_steps={0, 31, 63}, heads=[0, 39], seed=0,
                 fused=fused)
    assert n > 50  # mean budget 128: about 40% of 256 requests stop within 64 steps
