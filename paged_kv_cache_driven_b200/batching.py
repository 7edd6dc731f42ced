"""Continuous-batching decode loop over the paged KV cache.

"vLLM KV Cache and PagedAttention Explained", Step 8 "Continuous Batching in
vLLM": as soon as a request finishes, its batch slot is refilled with a new
request, and because each request's KV lives in its own physical blocks only
the finished request's blocks are freed and handed on (Step 7 item 7). Each
step is the decode loop of 7단계 "전체 흐름 요약": the new token's K/V is appended
to the cache, then attention reads the cached K/V.

One step, in this order (the order is part of the contract the tests check):
  1. host: every active request grows by one token (pa_prepare_step: new blocks
     at block boundaries, the new tokens' slots, padded block tables, lengths);
  2. host -> device copies of slots, tables and lengths;
  3. pa_kv_append of the step's new K/V, then pa_decode over every request's
     cached tokens including the new one (or both in one pa_decode_append);
  4. host: each request's token budget drops by one; for batch slots in index
     order, a finished request is freed (pa_seq_free) and its slot immediately
     refilled by the next arrival: grow to its prompt length and append its
     prompt K/V through slot_mapping (the prefill write of Step 6 "Prefill").

Random draws (lengths, budgets, token values, the shuffled free list) come from
``workloads.BatchingLoop``; everything else runs in the library. The host time
spent in allocator calls (grow, slot mapping, tables, free) is summed in
``host_s`` and reported per step in the step's record, with the device slot
mappings of the step's admissions.

With ``graph=True`` the device part of step 2-3 (the three uploads from the
pinned staging set and the append + decode launches) is a CUDA graph: the
first step that uses a staging set runs it eagerly and captures it, later steps
with that set replay it. The graph fixes every pointer and size, so the step's
q/k/v are first copied into fixed device buffers and decode is planned for the
largest length the loop can reach (``max_len``) instead of the step's own
maximum; the eager path does the same when ``fixed_plan`` is set, so the two
give the same bits.
"""

import ctypes
import math
import time

import numpy as np
import torch

from . import binding


class StagingRing:
    """Pinned host buffers for each step's slots, block tables and lengths (and
    the slot mappings of the step's admitted prompts), ``depth`` sets deep. The
    host fills set k while the copies of earlier sets may still be in flight;
    before a set is refilled, the event recorded after its copies is waited on,
    so the host never rewrites memory a pending copy still reads. (A copy from
    pageable memory would instead make the host wait for the whole stream.)"""

    PROMPT_SLOTS = 1 << 16  # admitted prompt tokens per step that fit the pinned slab

    def __init__(self, n_seq, max_blocks, n_new=1, depth=2):
        self.sets = [dict(slots=torch.empty(n_seq * n_new, dtype=torch.int64).pin_memory(),
                          tables=torch.empty((n_seq, max_blocks), dtype=torch.int32).pin_memory(),
                          lens=torch.empty(n_seq, dtype=torch.int32).pin_memory(),
                          prompt=torch.empty(self.PROMPT_SLOTS, dtype=torch.int64).pin_memory(),
                          prompt_used=0)
                     for _ in range(depth)]
        self.events = [None] * depth
        self.k = 0

    def acquire(self):
        i = self.k % len(self.sets)
        if self.events[i] is not None:
            self.events[i].synchronize()
        self.sets[i]["prompt_used"] = 0
        return self.sets[i]

    def release(self, stream=None):
        ev = torch.cuda.Event()
        ev.record(stream if stream is not None else torch.cuda.current_stream())
        self.events[self.k % len(self.sets)] = ev
        self.k += 1


class ContinuousBatching:
    def __init__(self, loop, device, max_steps=64, poison=True, fused=False, graph=False,
                 fixed_plan=False, keep_records=True):
        self.loop = loop
        self.fused = fused  # pa_decode_append instead of pa_kv_append + pa_decode
        self.graph = graph
        self.fixed_plan = fixed_plan or graph
        self.device = device
        B, H, D, S = loop.batch, loop.H, loop.D, loop.S
        self.B, self.H, self.D, self.S = B, H, D, S
        self.max_len = 4096 + max_steps
        self.MB = -(-self.max_len // S)
        NB = loop.num_blocks
        fill = float("nan") if poison else 0.0
        self.k_cache = torch.full((NB, H, S, D), fill, dtype=loop.dtype, device=device)
        self.v_cache = torch.full((NB, H, S, D), fill, dtype=loop.dtype, device=device)
        self.alloc = binding.BlockAllocator(NB, S, initial_order=loop.block_order)
        self.scale = 1.0 / math.sqrt(D)
        self.serial = 0
        self.keep_records = keep_records  # step records carry copies of slots, tables, lengths
        self.sid = []  # per batch slot: its sequence id
        self.ids_c = (ctypes.c_int64 * B)()  # the same, as the allocator takes it
        self.budget = np.zeros(B, dtype=np.int64)  # per batch slot: tokens left to decode
        self.staging = StagingRing(B, self.MB)
        self.d_slots = torch.empty(B, dtype=torch.int64, device=device)
        self.d_tables = torch.empty((B, self.MB), dtype=torch.int32, device=device)
        self.d_lens = torch.empty(B, dtype=torch.int32, device=device)
        self.out = torch.empty((B, H, D), dtype=torch.float32, device=device)
        ws = binding.pa_decode_workspace_bytes(B, H, D, S, self.max_len, 0)
        self.ws = torch.empty(max(ws, 16), dtype=torch.uint8, device=device)
        self.q_buf = torch.empty((B, H, D), dtype=loop.dtype, device=device)
        self.k_buf = torch.empty_like(self.q_buf)
        self.v_buf = torch.empty_like(self.q_buf)
        self.graphs = [None] * len(self.staging.sets)
        self.events = []  # (kind, seq_id, serial, prompt_len) for admissions / retirements
        self.host_s = 0.0  # seconds spent in allocator calls (grow, slots, tables, free)
        self.prompt_slots = []  # device slot mappings of the admissions since the last step
        for b in range(B):
            self._admit(b, loop.initial_lens[b], loop.budgets[b])

    def _admit(self, b, prompt_len, budget, h=None):
        """Creates a request in batch slot b, allocates its prompt blocks and
        appends its prompt K/V. During a step (h: the step's staging set) the
        slot mapping goes up from the set's pinned slab, asynchronously."""
        sid = self.serial
        self.serial += 1
        pinned = h is not None and h["prompt_used"] + prompt_len <= StagingRing.PROMPT_SLOTS
        t = time.perf_counter()
        self.alloc.pa_seq_grow(sid, prompt_len)
        if pinned:
            off = h["prompt_used"]
            h_slots = self.alloc.pa_build_slot_mapping(
                [sid], [0], [prompt_len], out=h["prompt"][off:off + prompt_len])
            h["prompt_used"] = off + prompt_len
        else:
            h_slots = self.alloc.pa_build_slot_mapping([sid], [0], [prompt_len])
        self.host_s += time.perf_counter() - t
        k, v = self.loop.prompt_kv(sid, prompt_len, self.device)
        slots = h_slots.to(self.device, non_blocking=pinned)
        binding.pa_kv_append(k, v, slots, self.k_cache, self.v_cache)
        self.prompt_slots.append(slots)
        self.events.append(("admit", sid, prompt_len))
        if b < len(self.sid):
            self.sid[b] = sid
        else:
            self.sid.append(sid)
        self.ids_c[b] = sid
        self.budget[b] = max(1, int(budget))

    def seq_ids(self):
        return list(self.sid)

    def _device_step(self, h, max_len):
        """Uploads from staging set h, then append + decode (eager or under capture)."""
        self.d_slots.copy_(h["slots"], non_blocking=True)
        self.d_tables.copy_(h["tables"], non_blocking=True)
        self.d_lens.copy_(h["lens"], non_blocking=True)
        q, k, v = (self.q_buf, self.k_buf, self.v_buf) if self.fixed_plan else self._qkv
        if self.fused:
            binding.pa_decode_append(self.out, q, k, v, self.k_cache, self.v_cache,
                                     self.d_tables, self.d_lens, self.scale, max_len,
                                     partition=0, workspace=self.ws)
        else:
            binding.pa_kv_append(k, v, self.d_slots, self.k_cache, self.v_cache)
            binding.pa_decode(self.out, q, self.k_cache, self.v_cache, self.d_tables,
                              self.d_lens, self.scale, max_len, partition=0, workspace=self.ws)

    def step(self, step_idx):
        """One decode step; returns a record of what it did (for checking and timing)."""
        ids = self.seq_ids()
        set_idx = self.staging.k % len(self.staging.sets)
        h = self.staging.acquire()
        host0 = self.host_s
        self.prompt_slots = []
        t = time.perf_counter()
        self.alloc.pa_prepare_step(self.ids_c, 1, self.MB, h["slots"], h["tables"], h["lens"])
        self.host_s += time.perf_counter() - t
        q, k, v = self.loop.token_kv(step_idx, self.B, self.device)
        self._qkv = (q, k, v)
        if self.fixed_plan:
            self.q_buf.copy_(q)
            self.k_buf.copy_(k)
            self.v_buf.copy_(v)
        max_len = self.max_len if self.fixed_plan else int(h["lens"].max())
        if self.graph and self.graphs[set_idx] is not None:
            self.graphs[set_idx].replay()
        else:
            self._device_step(h, max_len)
            if self.graph:  # capture this staging set's step for the steps that reuse it
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    self._device_step(h, max_len)
                self.graphs[set_idx] = g
        if self.keep_records:
            record = dict(ids=ids, slots=h["slots"].clone(), lens=h["lens"].clone(),
                          tables=h["tables"].clone(), q=q, k=k, v=v, out=self.out, retired=[],
                          admitted=[])
        else:
            record = dict(ids=ids, retired=[], admitted=[])
        self.budget -= 1
        for b in np.flatnonzero(self.budget <= 0).tolist():  # batch slots in index order
            old = self.sid[b]
            t = time.perf_counter()
            self.alloc.pa_seq_free(old)
            self.host_s += time.perf_counter() - t
            self.events.append(("retire", old, 0))
            L, budget = self.loop.arrival()
            self._admit(b, L, budget, h)
            record["retired"].append(old)
            record["admitted"].append((self.sid[b], L, int(self.budget[b])))
        self.staging.release()
        record["host_s"] = self.host_s - host0
        record["prompt_slots"] = self.prompt_slots
        return record
