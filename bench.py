#!/usr/bin/env python
"""Benchmark of the paged decode hot path on B200.

Workload: LLaMA-2-13B-shaped single-layer decode -- 40 heads, head_dim 128,
block_size 16, bf16, batch 64, seq_lens uniform in [1, 2048], physical blocks a
seeded random permutation of the pool (synthetic N(0, 1) data).

One step = the whole hot path for one batch: append the 64 new tokens' K/V
through slot_mapping (pa_kv_append), then decode attention over every request's
cached tokens (pa_decode: partition pass + log-sum-exp reduce).

  value  -- KV GB/s with all inputs resident in HBM (device-timed, CUDA events)
  e2e    -- the same metric through the C ABI with host buffers: every step
            grows the block tables on the host allocator (pa_prepare_step), copies
            q/k/v, slots, tables and lengths from pinned host memory, runs the
            kernels and copies the output back
  roofline -- the decode call (its algorithmic bytes / its event-timed duration)
            against the measured HBM copy bandwidth

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl reference]
For N > 1 launch under torch.distributed.run; every rank decodes its own batch
(weak scaling, no data-path collective).

Other workloads (--workload, one GPU, one JSON line each): long_context and
sweep (decode-only calls of the other decode configurations), llama70b
(grouped-query decode), llama13b_fp8 (the headline decode shape over an FP8
E4M3 cache) and prompt_prefill (causal paged prefill attention, TFLOP/s against
the measured bf16 tensor peak).
"""

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from paged_kv_cache_driven_b200 import binding, workloads  # noqa: E402
from paged_kv_cache_driven_b200.pipeline import HostFedDecoder  # noqa: E402

H, D, S, BATCH, MAX_LEN = 40, 128, 16, 64, 2048
DTYPE = torch.bfloat16
ELEM = 2
METRIC = "paged decode attention KV GB/s"
E2E_MIN_STEPS = 200
WORKLOAD = "llama2-13b-shaped single-layer decode: 40 heads, head_dim 128, block 16, bf16, " \
           "batch 64, seq_lens U[1,2048], permuted pool"


def decode_bytes(lens):
    """Algorithmic bytes of one decode call: K and V of every live token, q and
    out, the block-table entries read and the seq_lens."""
    kv = sum(H * (2 * L * D * ELEM + 2 * D * ELEM) for L in lens)
    return kv + sum(4 * (-(-L // S)) for L in lens) + 4 * len(lens)


def append_bytes(T, slots=True):
    """New tokens' K and V read and written; plus the int64 slots when the
    append goes through slot_mapping (the fused step derives them on device)."""
    return T * H * D * ELEM * 4 + (8 * T if slots else 0)


class ClockSampler:
    """SM clock and throttle-reason samples taken while the timed region runs.

    Polls NVML (read-only queries) from a background thread about every
    millisecond, so even a timed region of a few milliseconds gets samples;
    ``mark_start`` / ``mark_end`` bracket the region and only samples inside it
    are summarised. Falls back to an nvidia-smi poll if NVML is unavailable."""

    REASONS = (("hw_slowdown", 0x8), ("hw_thermal_slowdown", 0x40),
               ("sw_thermal_slowdown", 0x20), ("sw_power_cap", 0x4),
               ("hw_power_brake_slowdown", 0x80))

    def __init__(self, local_index):
        import threading
        visible = os.environ.get("CUDA_VISIBLE_DEVICES")
        ids = [x.strip() for x in visible.split(",")] if visible else []
        self.dev_id = ids[local_index] if local_index < len(ids) else str(local_index)
        self.samples = []
        self.window = [None, None]
        self._stop = threading.Event()
        self._ready = threading.Event()  # set once the first sample (or a failure) is in
        self._thread = threading.Thread(target=self._run, daemon=True)
        self.max_mhz = None
        self.source = None

    def _handle(self, nv):
        if self.dev_id.isdigit():
            return nv.nvmlDeviceGetHandleByIndex(int(self.dev_id))
        return nv.nvmlDeviceGetHandleByUUID(self.dev_id)

    def _run(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._handle(nv)
            self.max_mhz = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            self.source = "nvml"
            while not self._stop.is_set():
                t = time.perf_counter()
                mhz = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                reasons = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                self.samples.append((t, float(mhz), int(reasons)))
                self._ready.set()
                time.sleep(0.001)
            nv.nvmlShutdown()
        except Exception:
            self._run_smi()
        finally:
            self._ready.set()

    def _run_smi(self):
        q = "clocks.sm,clocks.max.sm,clocks_event_reasons.active"
        try:
            proc = subprocess.Popen(["nvidia-smi", f"--id={self.dev_id}", f"--query-gpu={q}",
                                     "--format=csv,noheader,nounits", "-lms", "100"],
                                    stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            return
        self.source = "nvidia-smi"
        while not self._stop.is_set():
            line = proc.stdout.readline()
            if not line:
                break
            f = [x.strip() for x in line.split(",")]
            try:
                self.max_mhz = float(f[1])
                self.samples.append((time.perf_counter(), float(f[0]), int(f[2], 16)))
                self._ready.set()
            except (ValueError, IndexError):
                continue
        proc.terminate()

    def __enter__(self):
        self._thread.start()
        self._ready.wait(timeout=10.0)  # the timed region starts only once sampling runs
        return self

    def __exit__(self, *exc):
        self._stop.set()
        self._thread.join(timeout=10)

    def mark_start(self):
        self.window[0] = time.perf_counter()

    def mark_end(self):
        self.window[1] = time.perf_counter()

    def summary(self):
        t0, t1 = self.window
        inside = [s for s in self.samples if t0 is not None and t1 is not None and t0 <= s[0] <= t1]
        reasons = sorted({n for _, _, r in inside for n, bit in self.REASONS if r & bit})
        mhz = [m for _, m, _ in inside]
        return {"sm_mhz": statistics.median(mhz) if mhz else None, "sm_max_mhz": self.max_mhz,
                "reasons": reasons, "samples": len(mhz), "source": self.source}


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def kernel_source_hash():
    """Hash of the headline call's kernels (the partition pass and the split-KV
    merge, with the device helpers they use), comments and blank lines removed,
    so a profile stays attached to the kernel code it measured and nothing else."""
    import re
    h = hashlib.sha256()
    for f in ("pa_decode.cuh", "pa_device.cuh"):
        with open(os.path.join(ROOT, "paged_kv_cache_driven_b200", "csrc", f)) as fh:
            text = re.sub(r"/\*.*?\*/", "", fh.read(), flags=re.S)
        lines = [re.sub(r"//.*", "", l).rstrip() for l in text.splitlines()]
        h.update("\n".join(l for l in lines if l.strip()).encode())
    return h.hexdigest()[:16]


def profiled_traffic():
    """DRAM bytes per decode call from the committed ncu summary, if it was taken
    on the current kernel source; else None."""
    p = os.path.join(ROOT, "profiles", "paged_decode_llama13b_traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        rec = json.load(f)
    if rec.get("kernel_source_hash") != kernel_source_hash():
        return None
    return rec.get("dram_bytes_per_decode_call")


class Workload:
    """The batch, its pool and the host allocator that owns its block tables."""

    def __init__(self, seed, device, extra_tokens):
        self.device = device
        lens = workloads.uniform_lengths(BATCH, 1, MAX_LEN, seed)
        self.lens0 = lens
        NB = sum(-(-(L + extra_tokens) // S) for L in lens)
        g = torch.Generator().manual_seed(seed + 17)
        order = torch.randperm(NB, generator=g).tolist()
        dg = torch.Generator(device=device).manual_seed(seed + 29)
        self.k_cache = torch.randn((NB, H, S, D), generator=dg, device=device, dtype=DTYPE)
        self.v_cache = torch.randn((NB, H, S, D), generator=dg, device=device, dtype=DTYPE)
        self.q = torch.randn((BATCH, H, D), generator=dg, device=device, dtype=DTYPE)
        self.k_new = torch.randn((BATCH, H, D), generator=dg, device=device, dtype=DTYPE)
        self.v_new = torch.randn((BATCH, H, D), generator=dg, device=device, dtype=DTYPE)
        self.out = torch.empty((BATCH, H, D), device=device, dtype=DTYPE)
        self.NB = NB
        self.MB = -(-(MAX_LEN + extra_tokens) // S)
        self.max_len = MAX_LEN + extra_tokens
        self.alloc = binding.BlockAllocator(NB, S, initial_order=order)
        self.seq_ids = list(range(BATCH))
        # the prompts (all but the newest token) are already cached
        for i, L in enumerate(lens):
            self.alloc.pa_seq_grow(i, L - 1)
        # device-resident step: the newest token of each request at position L - 1
        slots = torch.empty(BATCH, dtype=torch.int64)
        tables = torch.empty((BATCH, self.MB), dtype=torch.int32)
        lens_t = torch.empty(BATCH, dtype=torch.int32)
        self.alloc.pa_prepare_step(self.seq_ids, 1, self.MB, slots, tables, lens_t)
        self.lens = lens_t.tolist()
        self.max_seq = max(self.lens)
        self.slots_d = slots.to(device)
        self.tables_d = tables.to(device)
        self.lens_d = lens_t.to(device)
        ws = binding.pa_decode_workspace_bytes(BATCH, H, D, S, self.max_len, 0)
        self.ws = torch.empty(max(ws, 16), dtype=torch.uint8, device=device)
        self.plan = binding.pa_decode_plan(BATCH, H, D, S, self.max_seq, 0)
        self.scale = 1.0 / math.sqrt(D)
        self.e2e_ready = False

    def prepare_e2e(self):
        """Pinned host inputs and the host-fed step pipeline of the end-to-end step."""
        self.e2e_ready = True
        self.h_qkv = torch.stack([self.q, self.k_new, self.v_new]).cpu().pin_memory()
        self.fed = HostFedDecoder(self.alloc, self.k_cache, self.v_cache, BATCH, self.MB,
                                  self.max_len, out_dtype=DTYPE, fused=True)

    def launches_per_step(self, fused=True):
        """Kernels one step launches: the partition pass, the split-KV merge
        kernel when the plan splits and does not merge inside clusters (a
        cluster merge needs 2, 4 or 8 partitions and a grid of at most two CTAs
        per SM), and for the unfused step the append."""
        _, NP = binding.pa_decode_plan(BATCH, H, D, S, self.max_seq, 0)
        sms = torch.cuda.get_device_properties(self.device).multi_processor_count
        cluster = NP in (2, 4, 8) and BATCH * H * NP <= 2 * sms
        merge = 1 if NP > 1 and not cluster else 0
        return 1 + merge + (0 if fused else 1)

    def device_step(self, ev_decode=None, fused=True):
        """One step on device-resident inputs. Fused: pa_decode_append (the new
        tokens' K/V written at their last positions inside the decode launch);
        unfused: pa_kv_append through slot_mapping, then pa_decode."""
        if not fused:
            binding.pa_kv_append(self.k_new, self.v_new, self.slots_d, self.k_cache, self.v_cache)
        if ev_decode is not None:
            ev_decode[0].record()
        if fused:
            binding.pa_decode_append(self.out, self.q, self.k_new, self.v_new, self.k_cache,
                                     self.v_cache, self.tables_d, self.lens_d, self.scale,
                                     self.max_seq, partition=0, workspace=self.ws)
        else:
            binding.pa_decode(self.out, self.q, self.k_cache, self.v_cache, self.tables_d,
                              self.lens_d, self.scale, self.max_seq, partition=0,
                              workspace=self.ws)
        if ev_decode is not None:
            ev_decode[1].record()

    def e2e_step(self):
        """One decode step through the public API from host memory: the host
        allocator grows every request by one token, q/k/v, tables and lengths are
        copied from pinned host memory, the decode (with the append) runs, the
        output is copied back."""
        if not self.e2e_ready:
            self.prepare_e2e()
        self.fed.step(self.seq_ids, self.h_qkv)

    def e2e_drain(self):
        self.fed.drain()

    def h2d_bytes(self):
        return self.fed.h2d_bytes()

    def d2h_bytes(self):
        return self.fed.d2h_bytes()


def dist_setup(n_gpus):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    elif n_gpus > 1:
        raise SystemExit("for --gpus N > 1 launch with torch.distributed.run")
    return rank, world, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x, world, device):
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(x, world, device):
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM)
    return float(t.item())


class CpuOracleSample:
    """A bounded sample of a decode workload's (request, head) pairs for the fp64
    CPU oracle, sized so that one pass takes about ``pass_seconds`` (or the
    whole workload, if that is quicker). ``q``, ``k_cache``, ``v_cache`` may sit
    on any device; only the sampled pairs' blocks are copied to the host, once."""

    def __init__(self, q, k_cache, v_cache, tables_host, lens, scale, pass_seconds, cores):
        from oracle import decode as oracle_decode  # test infrastructure: CPU-baseline legs only

        self._decode = oracle_decode.paged_decode
        self.q, self.k_cache, self.v_cache = q, k_cache, v_cache
        self.tables_host, self.lens, self.scale, self.cores = tables_host, lens, scale, cores
        B, Hq, _ = q.shape
        self.B, self.H = B, Hq
        g = torch.Generator().manual_seed(123)
        all_pairs = [(i, h) for i in range(B) for h in range(Hq)]
        perm = torch.randperm(len(all_pairs), generator=g).tolist()
        n = min(len(all_pairs), 2 * cores)
        while True:
            self.pairs = [all_pairs[k] for k in perm[:n]]
            self.prob = self._sub_problem(self.pairs)
            dt = self.run()
            if dt >= pass_seconds * 0.5 or n >= len(all_pairs):
                break
            n = min(len(all_pairs), max(2 * n, int(n * pass_seconds / max(dt, 1e-3))))
        Dh = q.shape[2]
        e = k_cache.element_size()
        self.tokens = sum(lens[i] for i, _ in self.pairs)
        self.nbytes = sum(2 * lens[i] * Dh * e for i, _ in self.pairs)

    def _sub_problem(self, pairs):
        S, Dh = self.k_cache.shape[2], self.q.shape[2]
        G = self.q.shape[1] // self.k_cache.shape[1]
        ks, vs, qs, rows, lens = [], [], [], [], []
        off = 0
        for i, h in pairs:
            L = self.lens[i]
            blocks = torch.tensor(self.tables_host[i][: -(-L // S)], dtype=torch.long,
                                  device=self.k_cache.device)
            ks.append(self.k_cache[blocks, h // G].unsqueeze(1).cpu())
            vs.append(self.v_cache[blocks, h // G].unsqueeze(1).cpu())
            qs.append(self.q[i, h].view(1, 1, Dh).cpu())
            rows.append(list(range(off, off + len(blocks))))
            lens.append(L)
            off += len(blocks)
        MB = max(max(len(r) for r in rows), 1)
        bt = torch.full((len(pairs), MB), -1, dtype=torch.int32)
        for r, row in enumerate(rows):
            bt[r, :len(row)] = torch.tensor(row, dtype=torch.int32)
        return (torch.cat(qs), torch.cat(ks), torch.cat(vs), bt,
                torch.tensor(lens, dtype=torch.int32))

    def run(self):
        t0 = time.perf_counter()
        self._decode(*self.prob, self.scale, threads=self.cores)
        return time.perf_counter() - t0

    def describe(self, passes, seconds):
        return (f"{len(self.pairs)} of {self.B * self.H} (request, head) pairs of the workload "
                f"({self.tokens} tokens) x {passes} passes, {seconds:.1f} s on {self.cores} "
                f"thread{'s' if self.cores > 1 else ''}")


def cpu_baseline_case(q, k_cache, v_cache, tables_host, lens, scale, target_seconds, cores):
    """The oracle as it stands, timed on this host on a bounded sample of a decode
    workload: (GB/s of KV, description)."""
    smp = CpuOracleSample(q, k_cache, v_cache, tables_host, lens, scale,
                          min(target_seconds, 10.0), cores)
    passes, total = 0, 0.0
    while total < target_seconds * 0.7 or passes == 0:
        total += smp.run()
        passes += 1
    return passes * smp.nbytes / total / 1e9, smp.describe(passes, total)


def cpu_baseline_legs(q, k_cache, v_cache, tables_host, lens, scale, seconds=8.0):
    """The oracle on all host threads and on one thread, with the host's
    processor count: the cpu_baseline object of a bench line."""
    cores = os.cpu_count() or 1
    v, desc = cpu_baseline_case(q, k_cache, v_cache, tables_host, lens, scale, seconds, cores)
    v1, desc1 = cpu_baseline_case(q, k_cache, v_cache, tables_host, lens, scale, seconds, 1)
    return {"value": round(v, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
            "sample": desc, "nproc": cores,
            "single_thread": {"value": round(v1, 4), "unit": "GB/s", "cores": 1,
                              "sample": desc1}}


def cpu_baseline(wl, target_seconds, cores):
    """The headline workload's oracle leg: (GB/s of KV, description)."""
    tables = wl.tables_d.cpu().tolist()
    return cpu_baseline_case(wl.q, wl.k_cache, wl.v_cache, tables, wl.lens, wl.scale,
                             target_seconds, cores)


def run_reference(args):
    """The reference arm: the fp64 CPU oracle on the host cores, rank 0 only. Each
    step is one pass over a bounded sample of the workload. The workload is
    built on the host by the seeded generators alone (same shape and length mix
    as the native arm's, block tables a seeded permutation of an exactly sized
    pool), so nothing of the product library runs or loads here."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    lens = workloads.uniform_lengths(BATCH, 1, MAX_LEN, args.seed)
    case = workloads.decode_case(lens, H=H, D=D, S=S, dtype=DTYPE, seed=args.seed, device="cpu",
                                 poison=False)
    cores = os.cpu_count() or 1
    per_step = min(5.0, max(0.05, 150.0 / (args.steps + args.warmup)))
    smp = CpuOracleSample(case.q, case.k_cache, case.v_cache, case.tables_host,
                          case.seq_lens_host, case.scale, per_step, cores)
    for _ in range(args.warmup):
        smp.run()
    total = sum(smp.run() for _ in range(args.steps))
    value = args.steps * smp.nbytes / total / 1e9
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(1e3 * total / args.steps, 3),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOAD, "l2": "inputs larger than L2"},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores,
                             "kind": "oracle", "sample": smp.describe(args.steps, total)},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def decode_bytes_case(case):
    """Algorithmic bytes of one decode call on a workloads.DecodeCase: K and V of
    every live token of every KV head, q and out of every query head, the table
    entries read and the lengths."""
    B, Hq, Dc = case.q.shape
    Hkv, Sc = case.k_cache.shape[1], case.k_cache.shape[2]
    e = case.q.element_size()
    return sum(Hkv * 2 * L * Dc * e + Hq * 2 * Dc * e + 4 * (-(-L // Sc))
               for L in case.seq_lens_host) + 4 * B


L2_FLUSHED = "flushed before each call: 256 MB write, then 256 MB read"


class L2Flush:
    """Empties L2 (126 MB) before a timed call: a 256 MB write, then a 256 MB
    read. The read evicts the write's dirty lines, so L2 holds neither the
    call's inputs nor dirty lines whose write-back the timed call would pay for
    (after a write alone, a call that reads more than L2 writes about 126 MB
    back to HBM while it runs)."""

    def __init__(self, device):
        self.w = torch.empty(256 << 20, dtype=torch.uint8, device=device)
        self.r = torch.ones(64 << 20, dtype=torch.float32, device=device)
        self.sink = torch.empty((), dtype=torch.float32, device=device)
        self.k = 0

    def __call__(self):
        self.k += 1
        self.w.fill_(self.k & 0xff)
        torch.sum(self.r, dim=0, out=self.sink)


def time_decode_case(case, iters, warmup, partition=0):
    """Median event-timed pa_decode call with L2 flushed (L2Flush) before each."""
    B, Hc, Dc = case.q.shape
    Sc = case.k_cache.shape[2]
    maxlen = max(case.seq_lens_host)
    out = torch.empty((B, Hc, Dc), dtype=case.q.dtype, device=case.q.device)
    wsb = binding.pa_decode_workspace_bytes(B, Hc, Dc, Sc, maxlen, partition)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=case.q.device)
    flush = L2Flush(case.q.device)
    times = []
    for k in range(warmup + iters):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        if case.k_cache.shape[1] != Hc:
            binding.pa_decode_gqa(out, case.q, case.k_cache, case.v_cache, case.block_tables,
                                  case.seq_lens, case.scale, maxlen, partition=partition,
                                  workspace=ws)
        else:
            binding.pa_decode(out, case.q, case.k_cache, case.v_cache, case.block_tables,
                              case.seq_lens, case.scale, maxlen, partition=partition,
                              workspace=ws)
        b.record()
        torch.cuda.synchronize()
        if k >= warmup:
            times.append(a.elapsed_time(b))
    if binding.pa_get_device_error():
        raise SystemExit("device error word set")
    Hkv = case.k_cache.shape[1]
    return statistics.median(times), binding.pa_decode_plan_grouped(B, Hc, Hkv, Dc, Sc, maxlen,
                                                                      partition)


def time_decode_fp8(seed, iters, warmup):
    """The LLaMA-2-13B decode shape over an E4M3 cache (filled by pa_kv_append_fp8
    from the bf16 case): median event-timed pa_decode_fp8 call with L2 flushed
    before each, and the same for pa_decode_append_fp8 (each request's new row
    quantized into its last slot inside the launch); returns (ms, KV bytes,
    plan, fused-append ms)."""
    device = torch.device("cuda", 0)
    case = workloads.llama13b_decode(seed=seed, device=device)
    B, Hc, Dc = case.q.shape
    NB, _, Sc, _ = case.k_cache.shape
    kc8 = torch.empty((NB, Hc, Sc, Dc), dtype=torch.uint8, device=device)
    vc8 = torch.empty_like(kc8)
    slots = torch.arange(NB * Sc, dtype=torch.int64, device=device)
    binding.pa_kv_append_fp8(case.k_cache.permute(0, 2, 1, 3).reshape(-1, Hc, Dc).contiguous(),
                             case.v_cache.permute(0, 2, 1, 3).reshape(-1, Hc, Dc).contiguous(),
                             slots, kc8, vc8, 0.05, 0.08)
    del case.k_cache, case.v_cache
    maxlen = max(case.seq_lens_host)
    out = torch.empty((B, Hc, Dc), dtype=DTYPE, device=device)
    wsb = binding.pa_decode_workspace_bytes(B, Hc, Dc, Sc, maxlen, 0)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=device)
    flush = L2Flush(device)
    g = torch.Generator(device=device).manual_seed(seed + 77)
    k_new = torch.randn((B, Hc, Dc), generator=g, device=device).to(DTYPE)
    v_new = torch.randn((B, Hc, Dc), generator=g, device=device).to(DTYPE)

    def timed(call):
        times = []
        for k in range(warmup + iters):
            flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            call()
            b.record()
            torch.cuda.synchronize()
            if k >= warmup:
                times.append(a.elapsed_time(b))
        if binding.pa_get_device_error():
            raise SystemExit("device error word set")
        return statistics.median(times)

    ms = timed(lambda: binding.pa_decode_fp8(out, case.q, kc8, vc8, 0.05, 0.08, case.block_tables,
                                             case.seq_lens, case.scale, maxlen, partition=0,
                                             workspace=ws))
    ms_fused = timed(lambda: binding.pa_decode_append_fp8(
        out, case.q, k_new, v_new, kc8, vc8, 0.05, 0.08, case.block_tables, case.seq_lens,
        case.scale, maxlen, partition=0, workspace=ws))
    nbytes = sum(Hc * (2 * L * Dc + 2 * Dc * 2) + 4 * (-(-L // Sc)) for L in case.seq_lens_host) \
        + 4 * B
    return ms, nbytes, binding.pa_decode_plan(B, Hc, Dc, Sc, maxlen, 0), ms_fused


def time_decode_gqa_fp8(seed, iters, warmup):
    """The LLaMA-2-70B decode shape (64 query heads on 8 KV heads) over an E4M3
    cache filled by pa_kv_append_fp8 from the bf16 case: median event-timed
    pa_decode_gqa_fp8 call with L2 flushed before each; returns (ms, KV bytes,
    plan)."""
    device = torch.device("cuda", 0)
    case = workloads.llama70b_decode(seed=seed, device=device)
    B, Hq, Dc = case.q.shape
    NB, Hkv, Sc, _ = case.k_cache.shape
    kc8 = torch.empty((NB, Hkv, Sc, Dc), dtype=torch.uint8, device=device)
    vc8 = torch.empty_like(kc8)
    slots = torch.arange(NB * Sc, dtype=torch.int64, device=device)
    binding.pa_kv_append_fp8(case.k_cache.permute(0, 2, 1, 3).reshape(-1, Hkv, Dc).contiguous(),
                             case.v_cache.permute(0, 2, 1, 3).reshape(-1, Hkv, Dc).contiguous(),
                             slots, kc8, vc8, 0.05, 0.08)
    del case.k_cache, case.v_cache
    maxlen = max(case.seq_lens_host)
    out = torch.empty((B, Hq, Dc), dtype=DTYPE, device=device)
    wsb = binding.pa_decode_workspace_bytes(B, Hq, Dc, Sc, maxlen, 0)
    ws = torch.empty(max(wsb, 16), dtype=torch.uint8, device=device)
    flush = L2Flush(device)
    times = []
    for k in range(warmup + iters):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        binding.pa_decode_gqa_fp8(out, case.q, kc8, vc8, 0.05, 0.08, case.block_tables,
                                  case.seq_lens, case.scale, maxlen, partition=0, workspace=ws)
        b.record()
        torch.cuda.synchronize()
        if k >= warmup:
            times.append(a.elapsed_time(b))
    if binding.pa_get_device_error():
        raise SystemExit("device error word set")
    nbytes = sum(Hkv * 2 * L * Dc + Hq * 2 * Dc * 2 + 4 * (-(-L // Sc))
                 for L in case.seq_lens_host) + 4 * B
    return statistics.median(times), nbytes, binding.pa_decode_plan_grouped(B, Hq, Hkv, Dc, Sc,
                                                                             maxlen, 0)


def latency_floors(device, iters, warmup):
    """The small-batch floor, timed like the sweep's calls (L2 flushed, events
    around the call): a launch of a one-element fill (a kernel that does
    nothing measurable), and a decode of a single CTA (one request of 16
    tokens, one head, head_dim 128: one length, one table entry and one 8 KB
    K/V block to load)."""
    flush = L2Flush(device)
    x = torch.empty(1, dtype=torch.float32, device=device)
    case = workloads.decode_case([16], H=1, D=128, S=16, dtype=torch.bfloat16, seed=0,
                                 device=device)
    out = torch.empty((1, 1, 128), dtype=torch.bfloat16, device=device)

    def med(fn):
        ts = []
        for k in range(warmup + iters):
            flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize()
            if k >= warmup:
                ts.append(a.elapsed_time(b) * 1e3)
        return round(statistics.median(ts), 2)

    return {"empty_launch": med(lambda: x.fill_(0.0)),
            "single_cta_decode": med(lambda: binding.pa_decode(
                out, case.q, case.k_cache, case.v_cache, case.block_tables, case.seq_lens,
                case.scale, 16, partition=0, workspace=None))}


def run_shape_workloads(args):
    """--workload long_context | sweep: decode-only KV GB/s of the other
    configurations, one JSON line per case (L2 flushed before every call)."""
    device = torch.device("cuda", 0)
    peak, peak_kind = measured_peak()
    if args.workload == "long_context":
        cases = [("long_context", lambda: workloads.long_context_decode(seed=args.seed,
                                                                        device=device))]
    elif args.workload == "llama13b_fp8":
        ms, nbytes, plan, ms_fused = time_decode_fp8(args.seed, args.steps, args.warmup)
        gbs = nbytes / (ms / 1e3) / 1e9
        print(json.dumps({"workload": "llama13b_fp8_e4m3_cache", "ms": round(ms, 4),
                          "gb_s": round(gbs, 1), "frac_of_peak": round(gbs / peak, 3),
                          "kv_bytes": nbytes, "tok_s_layer": round(64 / (ms / 1e3), 1),
                          "fused_append_ms": round(ms_fused, 4),
                          "partition": {"tokens": plan[0], "num": plan[1]},
                          "l2": L2_FLUSHED}), flush=True)
        return
    elif args.workload == "llama70b":
        cases = [("llama70b_gqa_64q_8kv", lambda: workloads.llama70b_decode(seed=args.seed,
                                                                            device=device))]
    elif args.workload == "llama70b_fp8":
        ms, nbytes, plan = time_decode_gqa_fp8(args.seed, args.steps, args.warmup)
        gbs = nbytes / (ms / 1e3) / 1e9
        print(json.dumps({"workload": "llama70b_gqa_64q_8kv_fp8_e4m3_cache", "ms": round(ms, 4),
                          "gb_s": round(gbs, 1), "frac_of_peak": round(gbs / peak, 3),
                          "kv_bytes": nbytes, "tok_s_layer": round(64 / (ms / 1e3), 1),
                          "partition": {"tokens": plan[0], "num": plan[1]},
                          "l2": L2_FLUSHED}), flush=True)
        return
    else:
        cases = []
        for Sx in (8, 16, 32):
            for Dx in (64, 128, 256):
                for Bx in (1, 32, 256):
                    for dt in (torch.float16, torch.bfloat16):
                        name = f"S{Sx}_D{Dx}_B{Bx}_{'fp16' if dt == torch.float16 else 'bf16'}"
                        cases.append((name, (lambda Sx=Sx, Dx=Dx, Bx=Bx, dt=dt: workloads.sweep_case(
                            Sx, Dx, Bx, dt, seed=args.seed, device=device))))
    # the oracle is timed on one case of each configuration (the long-context
    # case, one mid-size point of the sweep)
    cpu_cases = {"long_context", "S16_D128_B32_bf16"}
    if args.case:
        cases = [(n, m) for n, m in cases if n == args.case]
        if not cases:
            raise SystemExit(f"no case named {args.case}")
    rows = []
    for name, make in cases:
        case = make()
        ms, plan = time_decode_case(case, args.steps, args.warmup)
        nbytes = decode_bytes_case(case)
        gbs = nbytes / (ms / 1e3) / 1e9
        row = {"workload": name, "ms": round(ms, 4), "gb_s": round(gbs, 1),
               "frac_of_peak": round(gbs / peak, 3), "kv_bytes": nbytes,
               "tok_s_layer": round(case.q.shape[0] / (ms / 1e3), 1),
               "partition": {"tokens": plan[0], "num": plan[1]}, "l2": L2_FLUSHED}
        if name in cpu_cases and not args.no_cpu_baseline:
            row["cpu_baseline"] = cpu_baseline_legs(case.q, case.k_cache, case.v_cache,
                                                    case.tables_host, case.seq_lens_host,
                                                    case.scale)
        rows.append(row)
        print(json.dumps(row), flush=True)
        del case
        torch.cuda.empty_cache()
    big = [r for r in rows if r["kv_bytes"] > 1 << 30]
    floors = latency_floors(device, args.steps, args.warmup) if args.workload == "sweep" else None
    summary = {"metric": METRIC + " (decode only)", "workload": args.workload,
               "peak": peak, "peak_kind": peak_kind, "cases": len(rows), "latency_floors_us": floors,
               "min_frac_over_1GB": min((r["frac_of_peak"] for r in big), default=None),
               "median_frac_over_1GB": statistics.median([r["frac_of_peak"] for r in big])
               if big else None}
    print(json.dumps(summary), flush=True)


def run_worked_example(args):
    """--workload worked_example: the pages' four requests of 6/50/8/100 tokens
    (4 heads, head_dim 64, fp16). The whole cache is 256 KB: even with L2
    flushed before each call the GPU time is a launch- and latency-bound
    figure, not a bandwidth one. The line's point is the oracle leg on the same
    inputs (all threads and one)."""
    device = torch.device("cuda", 0)
    case = workloads.worked_example(seed=args.seed, device=device)
    ms, plan = time_decode_case(case, args.steps, args.warmup)
    nbytes = decode_bytes_case(case)
    row = {"workload": "worked_example_6_50_8_100", "ms": round(ms, 4),
           "gb_s": round(nbytes / (ms / 1e3) / 1e9, 2), "kv_bytes": nbytes,
           "note": "256 KB cache; launch- and latency-bound", "l2": L2_FLUSHED,
           "partition": {"tokens": plan[0], "num": plan[1]}}
    if not args.no_cpu_baseline:
        row["cpu_baseline"] = cpu_baseline_legs(case.q, case.k_cache, case.v_cache,
                                                case.tables_host, case.seq_lens_host, case.scale,
                                                seconds=3.0)
    print(json.dumps(row), flush=True)


APPEND_WORKLOAD = "prefill-scale append: 16 requests of U[512,4096] tokens, 32 heads, " \
                  "head_dim 128, block 16, bf16, slots from the host allocator over a shuffled pool"


def run_append_workload(args):
    """--workload prefill_append: pa_kv_append of a prefill-sized batch of new
    tokens through slot_mapping (the shape sweep's append), KV GB/s against the
    measured HBM copy bandwidth. Algorithmic bytes: the new tokens' K and V read
    and written plus the int64 slots, T*H*D*e*4 + 8T. Median of event-timed calls
    with L2 flushed (L2Flush) before each."""
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    if args.workload == "prefill_append_small":  # a profiling-sized case: 4 x 4096 tokens
        case = workloads.prefill_append(seed=args.seed, device=device, n_req=4, lo=4096, hi=4096)
    else:
        case = workloads.prefill_append(seed=args.seed, device=device)
    T, Hc, Dc = case.k.shape
    NB, _, Sc, _ = case.k_cache.shape
    alloc = binding.BlockAllocator(NB, Sc, initial_order=case.block_order)
    ids = list(range(len(case.n_tokens)))
    for i, n in zip(ids, case.n_tokens):
        alloc.pa_seq_grow(i, n)
    slots = alloc.pa_build_slot_mapping(ids, [0] * len(ids), case.n_tokens).to(device)
    alloc.close()
    e = case.k.element_size()
    nbytes = T * Hc * Dc * e * 4 + 8 * T
    flush = L2Flush(device)
    times = []
    with ClockSampler(0) as clk:
        clk.mark_start()
        for k in range(args.warmup + args.steps):
            flush()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            binding.pa_kv_append(case.k, case.v, slots, case.k_cache, case.v_cache)
            b.record()
            torch.cuda.synchronize()
            if k >= args.warmup:
                times.append(a.elapsed_time(b))
        clk.mark_end()
    if binding.pa_get_device_error():
        raise SystemExit("device error word set")
    ms = statistics.median(times)
    peak, peak_kind = measured_peak()
    gbs = nbytes / (ms / 1e3) / 1e9
    print(json.dumps({"workload": APPEND_WORKLOAD if args.workload == "prefill_append" else
                      "prefill-scale append, profiling size: 4 requests of 4096 tokens",
                      "tokens": T, "ms": round(ms, 4),
                      "gb_s": round(gbs, 1), "frac_of_peak": round(gbs / peak, 3),
                      "peak": peak, "peak_kind": peak_kind, "bytes_per_call": nbytes,
                      "kernel": "kv_append_kernel (one launch)", "calls": args.steps,
                      "l2": L2_FLUSHED, "clocks": clk.summary()}), flush=True)


BATCHING_WORKLOAD = "continuous batching: 40 heads, head_dim 128, block 16, bf16, batch 256, " \
                    "prompts lognormal(median 300, sigma 1) clipped to [1,4096], geometric stops " \
                    "(mean 128), shuffled free list"


def run_batching_workload(args):
    """--workload batching: the continuous-batching loop (the pages' Step 8), 64
    timed steps after W warm-up steps, on the same draws three ways:

    * eager, two calls per step (pa_kv_append through slot_mapping, pa_decode);
    * eager, fused (pa_decode_append);
    * CUDA graph, fused: the step's uploads and launch captured per staging set
      and replayed, decode planned for the loop's largest length.

    Each reports the wall-clock step time (host and device overlapped as the
    loop runs them), the host time spent in allocator calls per step and its
    share. The device phases are then replayed back to back from the eager
    run's recorded steps (uploads from pinned memory, append, decode, the
    admissions' prompt appends), so their event times carry no host gaps.
    Token and prompt K/V are drawn once before the timed steps (input synthesis
    stays out of them); the pool is 256 * ceil((4096 + 64 + W) / 16) blocks so
    the warm-up steps fit."""
    from paged_kv_cache_driven_b200.batching import ContinuousBatching

    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    K, W = 64, args.warmup
    pre = None

    def make_loop():
        nonlocal pre
        loop = workloads.batching_loop(seed=args.seed, headroom=64 + W)
        if pre is None:
            g = torch.Generator(device=device).manual_seed(args.seed + 4242)
            shape = (K + W, 3, loop.batch, loop.H, loop.D)
            tok = torch.randn(shape, generator=g, device=device, dtype=loop.dtype)
            pk = torch.randn((4096, loop.H, loop.D), generator=g, device=device, dtype=loop.dtype)
            pv = torch.randn((4096, loop.H, loop.D), generator=g, device=device, dtype=loop.dtype)
            pre = (tok, pk, pv)
        tok, pk, pv = pre
        loop.token_kv = lambda step, n, dev: (tok[step, 0, :n], tok[step, 1, :n], tok[step, 2, :n])
        loop.prompt_kv = lambda serial, n, dev: (pk[:n], pv[:n])
        return loop

    def run(fused, graph, keep=False):
        loop = make_loop()
        cb = ContinuousBatching(loop, device, max_steps=64 + W, poison=False, fused=fused,
                                graph=graph, keep_records=keep)
        for k in range(W):
            cb.step(k)
        torch.cuda.synchronize()
        host0 = cb.host_s
        recs = []
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0 = time.perf_counter()
        e0.record()
        for k in range(W, W + K):
            r = cb.step(k)
            if keep:
                recs.append(dict(slots=r["slots"], tables=r["tables"], lens=r["lens"],
                                 prompt_slots=r["prompt_slots"]))
        e1.record()
        torch.cuda.synchronize()
        wall = (time.perf_counter() - t0) / K
        dev_ms = e0.elapsed_time(e1) / K
        if binding.pa_get_device_error():
            raise SystemExit("device error word set")
        host = (cb.host_s - host0) / K
        res = {"step_ms": round(wall * 1e3, 4), "device_span_ms": round(dev_ms, 4),
               "tok_s_layer": round(loop.batch / wall, 1), "host_alloc_ms": round(host * 1e3, 4),
               "host_share": round(host / wall, 4)}
        return res, cb, recs

    with ClockSampler(0) as clk:
        clk.mark_start()
        two_call, cb, recs = run(fused=False, graph=False, keep=True)
        # device phases replayed back to back from the recorded steps
        tok, pk, pv = pre
        B, Hc, Dc, Sc = cb.B, cb.H, cb.D, cb.S
        for r in recs:  # pinned before the replay, so no host work sits between its phases
            for key in ("slots", "tables", "lens"):
                r[key] = r[key].pin_memory()
        marks = []
        for k, r in enumerate(recs):
            ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
            ev[0].record()
            cb.d_slots.copy_(r["slots"], non_blocking=True)
            cb.d_tables.copy_(r["tables"], non_blocking=True)
            cb.d_lens.copy_(r["lens"], non_blocking=True)
            ev[1].record()
            binding.pa_kv_append(tok[W + k, 1], tok[W + k, 2], cb.d_slots, cb.k_cache, cb.v_cache)
            ev[2].record()
            binding.pa_decode(cb.out, tok[W + k, 0], cb.k_cache, cb.v_cache, cb.d_tables,
                              cb.d_lens, cb.scale, int(r["lens"].max()), partition=0,
                              workspace=cb.ws)
            ev[3].record()
            for ps in r["prompt_slots"]:
                n = ps.numel()
                binding.pa_kv_append(pk[:n], pv[:n], ps, cb.k_cache, cb.v_cache)
            ev[4].record()
            marks.append(ev)
        torch.cuda.synchronize()
        if binding.pa_get_device_error():
            raise SystemExit("device error word set")
        ph = [[a.elapsed_time(b) for a, b in zip(ev[:-1], ev[1:])] for ev in marks]
        dec_bytes = [sum(Hc * (2 * L * Dc * 2 + 2 * Dc * 2) + 4 * (-(-L // Sc))
                         for L in r["lens"].tolist()) + 4 * B for r in recs]
        dec_ms = [p[2] for p in ph]
        admissions = sum(len(r["prompt_slots"]) for r in recs) / K
        prompt_tokens = sum(ps.numel() for r in recs for ps in r["prompt_slots"]) / K
        two_call["device_phases_ms"] = {
            "upload": round(statistics.mean(p[0] for p in ph), 4),
            "append": round(statistics.mean(p[1] for p in ph), 4),
            "decode": round(statistics.mean(dec_ms), 4),
            "admission_prompt_appends": round(statistics.mean(p[3] for p in ph), 4),
            "sum": round(statistics.mean(sum(p) for p in ph), 4)}
        two_call["decode_kv_gb_s"] = round(sum(dec_bytes) / (sum(dec_ms) / 1e3) / 1e9, 1)
        two_call["admissions_per_step"] = round(admissions, 3)
        two_call["prompt_tokens_per_step"] = round(prompt_tokens, 1)
        del cb, recs, marks
        torch.cuda.empty_cache()
        fused, cb, _ = run(fused=True, graph=False)
        del cb
        torch.cuda.empty_cache()
        graphed, cb, _ = run(fused=True, graph=True)
        del cb
        torch.cuda.empty_cache()
        clk.mark_end()
    peak, peak_kind = measured_peak()
    line = {"metric": "continuous-batching decode step tok/s/layer", "workload": BATCHING_WORKLOAD,
            "steps": K, "warmup": W, "batch": 256,
            "eager_two_calls": two_call, "eager_fused": fused, "graph_fused": graphed,
            "hbm_peak": peak, "peak_kind": peak_kind,
            "decode_frac_of_peak": round(two_call["decode_kv_gb_s"] / peak, 3),
            "clocks": clk.summary()}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# Prompt prefill: causal paged prefill attention (pa_prefill) on the tensor cores
# ---------------------------------------------------------------------------

PREFILL_METRIC = "paged prefill attention TFLOP/s"
PREFILL_WORKLOAD = "prompt prefill: 16 prompts of U[512,4096] tokens, 32 heads, head_dim 128, " \
                   "block 16, bf16, permuted pool, causal"


def prefill_flops(new_lens, ctx_lens, Hq, Dh):
    """Algorithmic FLOPs of causal prefill: q.k and p.v (2 * D each) for every
    (new token, head, key it sees) triple; new token j of a request with c
    cached tokens sees c + j + 1 keys."""
    return sum(Hq * 4 * Dh * (n * c + n * (n + 1) // 2) for n, c in zip(new_lens, ctx_lens))


def measured_tensor_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured (cuBLAS bf16 burst)"
    return 1590.0, "fallback"


def prefill_cpu_baseline(target_seconds, cores, seed):
    """The oracle's causal prefill on one prompt of the workload's shape (32 heads,
    head_dim 128, block 16) on the host cores, its length sized to about
    target_seconds: (TFLOP/s, description)."""
    from oracle import decode as oracle_decode  # test infrastructure: CPU-baseline leg only

    n, total, passes = 128, 0.0, 0
    while True:
        pc = workloads.prefill_case([0], [n], H=32, D=128, S=16, dtype=DTYPE, seed=seed,
                                    device="cpu")
        c = pc.cache
        t0 = time.perf_counter()
        oracle_decode.paged_prefill(pc.q, c.k_cache, c.v_cache, c.block_tables, c.seq_lens,
                                    pc.q_start, c.scale, threads=cores)
        dt = time.perf_counter() - t0
        if dt >= target_seconds * 0.3 or n >= 4096:
            total, passes = dt, 1
            break
        n = min(4096, int(n * max(1.5, min(4.0, (target_seconds * 0.5 / max(dt, 1e-3)) ** 0.5))))
    fl = prefill_flops([n], [0], 32, 128)
    return fl / total / 1e12, (f"one {n}-token prompt x 32 heads (causal, fp64) x {passes} pass, "
                               f"{total:.1f} s on {cores} threads")


def prefill_trace_phases(buf):
    """Per-phase medians (SM cycles) from the trace build's stamps
    [CTA][slot][key tile] (slot meanings in pa_prefill.cuh), over the
    steady-state key tiles of the traced CTAs: the first two and the last key
    tile of each CTA are left out."""
    agg = {}

    def add(k, v):
        if v > 0:
            agg.setdefault(k, []).append(int(v))

    for cta in range(buf.shape[0]):
        if buf[cta, 31, 0] == 0:
            continue
        nk = int((buf[cta, 20, :] > 0).sum())
        # the CTA's start to its first scores (tile 0, first half), and its
        # whole run
        if buf[cta, 0, 0]:
            add("CTA start to its first scores ready (prologue)", buf[cta, 0, 0] - buf[cta, 31, 0])
        if buf[cta, 30, 0]:
            add("CTA start to end", buf[cta, 30, 0] - buf[cta, 31, 0])
        for j in range(2, nk - 1):
            for t in range(2):
                for hw in range(2):
                    k = 2 * t + hw
                    s0 = buf[cta, k, j]
                    if s0 == 0 or buf[cta, 16 + k, j] == 0:
                        continue
                    add("softmax: scores from tensor memory and the row max",
                        buf[cta, 4 + k, j] - s0)
                    add("softmax: the max exchange between the two halves",
                        buf[cta, 8 + k, j] - buf[cta, 4 + k, j])
                    add("softmax: weights P (exp2, hi + lo packing, stores)",
                        buf[cta, 12 + k, j] - buf[cta, 8 + k, j])
                    add("softmax: output rescale and fences",
                        buf[cta, 16 + k, j] - buf[cta, 12 + k, j])
                    add("softmax of one query tile and key tile (per warpgroup)",
                        buf[cta, 16 + k, j] - s0)
                    if buf[cta, k, j + 1]:
                        add("from a warpgroup's P-ready arrival to its next scores",
                            buf[cta, k, j + 1] - buf[cta, 16 + k, j])
            for t in range(2):
                if buf[cta, 20 + t, j] and buf[cta, 22 + t, j]:
                    add(f"MMA warp: P(j) of tile {t} seen to its P.V and next S issued",
                        buf[cta, 22 + t, j] - buf[cta, 20 + t, j])
            if buf[cta, 20, j + 1]:
                add("one key tile for both query tiles (period)",
                    buf[cta, 20, j + 1] - buf[cta, 20, j])
    return {k: {"median": int(statistics.median(v)), "n": len(v)} for k, v in agg.items()}


def run_prefill_trace(args):
    """--workload prefill_trace: where the prefill kernel's time goes. The
    profiling-size prompt case (4 prompts of 2048 tokens, 8 heads) runs on the
    library proper and on the trace build (libpagedattn_trace.so, from
    `python -m paged_kv_cache_driven_b200.build --trace`: the same kernel with
    clock stamps at its hand-offs); the two outputs must be the same bits, and
    the trace build's stamps of one launch are reduced to per-phase medians in
    SM cycles (prefill_trace_phases)."""
    import ctypes
    import numpy as np
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    pc = workloads.prompt_prefill(seed=args.seed, device=device, n_req=4, lo=2048, hi=2048, H=8)
    c = pc.cache
    T, Hq, Dh = pc.q.shape

    def run(out):
        binding.pa_prefill(out, pc.q, c.k_cache, c.v_cache, c.block_tables, c.seq_lens,
                           pc.q_start, c.scale, pc.max_q_len)

    def timed(out):
        for _ in range(args.warmup):
            run(out)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        run(out)
        b.record()
        torch.cuda.synchronize()
        return a.elapsed_time(b)

    ref = torch.empty((T, Hq, Dh), dtype=DTYPE, device=device)
    ms_plain = timed(ref)
    if binding.pa_get_device_error():
        raise SystemExit("device error word set")
    path = os.path.join(ROOT, "paged_kv_cache_driven_b200", "libpagedattn_trace.so")
    th = binding.open_library(path)
    th.pa_prefill_trace_read.argtypes = [ctypes.c_void_p, ctypes.c_size_t]
    th.pa_prefill_trace_read.restype = ctypes.c_int
    th.pa_prefill_trace_clear.restype = ctypes.c_int
    prev = binding.use_library(th)
    try:
        got = torch.empty_like(ref)
        for _ in range(args.warmup):
            run(got)
        torch.cuda.synchronize()
        if th.pa_prefill_trace_clear() != 0:
            raise SystemExit("pa_prefill_trace_clear failed")
        ms_trace = timed(got)
        buf = np.zeros((64, 32, 48), dtype=np.int64)
        if th.pa_prefill_trace_read(ctypes.c_void_p(buf.ctypes.data), buf.nbytes) != 0:
            raise SystemExit("pa_prefill_trace_read failed")
        if binding.pa_get_device_error():
            raise SystemExit("device error word set (trace build)")
    finally:
        binding.use_library(prev)
    same = torch.equal(ref.view(torch.int16), got.view(torch.int16))
    print(json.dumps({"workload": "prompt prefill, profiling size: 4 prompts of 2048 tokens, "
                                  "8 heads, head_dim 128, block 16, bf16, causal",
                      "launch_ms": round(ms_plain, 4), "launch_ms_trace_build": round(ms_trace, 4),
                      "same_bits_as_library": same, "traced_ctas": int((buf[:, 31, 0] > 0).sum()),
                      "cycles": prefill_trace_phases(buf)}), flush=True)
    if not same:
        raise SystemExit("the trace build's output differs from the library's")


def run_prefill_workload(args):
    """--workload prompt_prefill: pa_prefill over the prompt prefill workload,
    TFLOP/s against the measured bf16 tensor peak, plus an end-to-end prefill
    step through the C ABI from host buffers (host allocator, uploads of the
    prompts' q/k/v, pa_kv_append, pa_prefill, download of the output)."""
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    if args.workload == "prompt_prefill_small":  # a profiling-sized case of the same kernel
        pc = workloads.prompt_prefill(seed=args.seed, device=device, n_req=4, lo=2048, hi=2048,
                                      H=8)
    elif args.workload == "prompt_prefill_d256":  # the same prompts at head_dim 256
        pc = workloads.prompt_prefill(seed=args.seed, device=device, D=256)
    else:
        pc = workloads.prompt_prefill(seed=args.seed, device=device)
    c = pc.cache
    T, Hq, Dh = pc.q.shape
    flops = prefill_flops(pc.new_lens, pc.ctx_lens, Hq, Dh)
    out = torch.empty((T, Hq, Dh), dtype=DTYPE, device=device)
    stream = torch.cuda.current_stream()

    def call():
        binding.pa_prefill(out, pc.q, c.k_cache, c.v_cache, c.block_tables, c.seq_lens,
                           pc.q_start, c.scale, pc.max_q_len)

    for _ in range(args.warmup):
        call()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(0) as clk:
        clk.mark_start()
        start.record(stream)
        for a, b in evs:
            a.record(stream)
            call()
            b.record(stream)
        end.record(stream)
        torch.cuda.synchronize()
        clk.mark_end()
    total_ms = start.elapsed_time(end)
    call_ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    if binding.pa_get_device_error():
        raise SystemExit("device error word set")
    value = flops * args.steps / (total_ms / 1e3) / 1e12
    achieved = flops / (call_ms / 1e3) / 1e12
    peak, peak_kind = measured_tensor_peak()

    # ---- end to end: the same prompts from host buffers ------------------------
    kh = torch.randn((T, c.k_cache.shape[1], Dh), dtype=torch.float32).to(DTYPE).pin_memory()
    vh = torch.randn((T, c.k_cache.shape[1], Dh), dtype=torch.float32).to(DTYPE).pin_memory()
    qh = pc.q.cpu().pin_memory()
    oh = torch.empty((T, Hq, Dh), dtype=DTYPE).pin_memory()
    B = len(pc.new_lens)
    NB = c.k_cache.shape[0]
    MB = c.block_tables.shape[1]
    qs_h = pc.q_start.cpu().pin_memory()
    dq = torch.empty_like(pc.q)
    dk = torch.empty((T, c.k_cache.shape[1], Dh), dtype=DTYPE, device=device)
    dv = torch.empty_like(dk)
    dslots = torch.empty(T, dtype=torch.int64, device=device)
    dtab = torch.empty((B, MB), dtype=torch.int32, device=device)
    dlens = torch.empty(B, dtype=torch.int32, device=device)
    dqs = torch.empty(B + 1, dtype=torch.int32, device=device)
    h2d = d2h = 0

    def e2e_step():
        nonlocal h2d, d2h
        alloc = binding.BlockAllocator(NB, c.k_cache.shape[2])
        ids = list(range(B))
        for i, n in zip(ids, pc.new_lens):
            alloc.pa_seq_grow(i, n)
        slots = alloc.pa_build_slot_mapping(ids, [0] * B, pc.new_lens).pin_memory()
        tables = alloc.pa_build_block_tables(ids, MB).pin_memory()
        lens = torch.tensor(pc.new_lens, dtype=torch.int32).pin_memory()
        for dst, src in ((dq, qh), (dk, kh), (dv, vh), (dslots, slots), (dtab, tables),
                         (dlens, lens), (dqs, qs_h)):
            dst.copy_(src, non_blocking=True)
        binding.pa_kv_append(dk, dv, dslots, c.k_cache, c.v_cache)
        binding.pa_prefill(out, dq, c.k_cache, c.v_cache, dtab, dlens, dqs, c.scale,
                           pc.max_q_len)
        oh.copy_(out, non_blocking=True)
        h2d = sum(t.numel() * t.element_size() for t in (qh, kh, vh, slots, tables, lens, qs_h))
        d2h = oh.numel() * oh.element_size()
        alloc.close()

    for _ in range(args.warmup):
        e2e_step()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    if binding.pa_get_device_error():
        raise SystemExit("device error word set")
    e2e_value = flops * args.steps / (e2e_ms / 1e3) / 1e12

    cpu = None
    if not args.no_cpu_baseline:
        cores = os.cpu_count() or 1
        v, desc = prefill_cpu_baseline(12.0, cores, args.seed)
        cpu = {"value": round(v, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
               "sample": desc}
    line = {
        "metric": PREFILL_METRIC, "value": round(value, 2), "unit": "TFLOP/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 4), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": {"prompt_prefill": PREFILL_WORKLOAD,
                                "prompt_prefill_d256": PREFILL_WORKLOAD.replace("head_dim 128",
                                                                                "head_dim 256")}.get(
                       args.workload,
                       "prompt prefill, profiling size: 4 prompts of 2048 tokens, 8 heads"),
                   "prompt_tokens": T, "heads": Hq,
                   "head_dim": Dh, "block_size": c.k_cache.shape[2], "flops_per_step": flops,
                   "l2": "inputs larger than L2 (0.9 GB or more of q and K/V vs 126 MB L2)",
                   "parallelism": "dp1"},
        "roofline": {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak,
                     "unit": "TFLOP/s", "frac": round(achieved / peak, 4), "peak_kind": peak_kind,
                     "traffic": None, "kernel": "paged_prefill_kernel (one launch per step)",
                     "call_ms": round(call_ms, 4), "algorithmic_flops_per_launch": flops,
                     "tensor_work_per_launch": "bf16 weights enter P.V as two terms, so the "
                                               "tensor cores do 1.5x the algorithmic FLOPs"},
        "e2e": {"value": round(e2e_value, 2), "unit": "TFLOP/s",
                "api": "host BlockAllocator (grow, slot mapping, tables), pinned uploads, "
                       "pa_kv_append, pa_prefill, output download",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": round(e2e_ms / args.steps, 4)},
        "gpu_launches": args.steps,
        "clocks": clk.summary(),
    }
    if cpu is not None:
        line["cpu_baseline"] = cpu
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--case", default=None,
                    help="with --workload sweep: time only this case (e.g. S16_D128_B1_bf16)")
    ap.add_argument("--workload", default="llama13b",
                    choices=["llama13b", "long_context", "sweep", "llama70b", "llama70b_fp8",
                             "llama13b_fp8",
                             "prompt_prefill", "prompt_prefill_small", "prompt_prefill_d256",
                             "worked_example",
                             "prefill_append", "prefill_append_small", "batching",
                             "prefill_trace"],
                    help="llama13b: the headline step (default); the others time decode-only "
                         "calls of the long-context, shape-sweep and LLaMA-2-70B-shaped "
                         "grouped-query configurations, paged prefill attention over "
                         "16 prompts (prompt_prefill), the pages' worked example, the "
                         "prefill-scale append, or the continuous-batching loop; "
                         "prefill_trace: per-phase clock stamps of the prefill kernel "
                         "(needs `python -m paged_kv_cache_driven_b200.build --trace`)")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
        return
    if args.workload.startswith("prompt_prefill"):
        binding.lib()
        run_prefill_workload(args)
        return
    extra = {"worked_example": run_worked_example, "prefill_append": run_append_workload,
             "prefill_append_small": run_append_workload, "batching": run_batching_workload,
             "prefill_trace": run_prefill_trace}
    if args.workload in extra:
        binding.lib()
        extra[args.workload](args)
        return
    if args.workload != "llama13b":
        binding.lib()
        run_shape_workloads(args)
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    binding.lib()  # fail loudly if the library is missing
    rank, world, local = dist_setup(args.gpus)
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    # the end-to-end leg runs at least E2E_MIN_STEPS steps, so that its one pipeline
    # fill and drain weigh the same whatever --steps is
    e2e_steps = max(args.steps, E2E_MIN_STEPS)
    extra = args.warmup + e2e_steps + 8
    wl = Workload(seed=args.seed + 1000 * rank, device=device, extra_tokens=extra)
    stream = torch.cuda.current_stream()

    # ---- device-resident steps -------------------------------------------------
    def timed_steps(fused, sampler=None):
        for _ in range(args.warmup):
            wl.device_step(fused=fused)
        torch.cuda.synchronize()
        barrier(world)
        torch.cuda.synchronize()
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        calls = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                 for _ in range(args.steps)]
        if sampler is not None:
            sampler.mark_start()
        start.record(stream)
        for k in range(args.steps):
            wl.device_step(calls[k], fused=fused)
        end.record(stream)
        torch.cuda.synchronize()
        if sampler is not None:
            sampler.mark_end()
        barrier(world)
        torch.cuda.synchronize()
        total = max_over_ranks(start.elapsed_time(end), world, device)
        call_ms = statistics.mean(a.elapsed_time(b) for a, b in calls)
        flags = binding.pa_get_device_error()
        if flags:
            raise SystemExit(f"device error word set: {flags:#x}")
        return total, call_ms

    # the two-call step (pa_kv_append through slot_mapping, then pa_decode), for reference
    unfused_ms, unfused_dec_ms = timed_steps(fused=False)
    # the fused step, timed for the headline with clocks sampled inside the region
    with ClockSampler(local) as clk:
        ms_total, dec_ms = timed_steps(fused=True, sampler=clk)
    step_bytes = decode_bytes(wl.lens) + append_bytes(BATCH, slots=False)
    total_bytes = sum_over_ranks(step_bytes * args.steps, world, device)
    value = total_bytes / (ms_total / 1e3) / 1e9
    ms_per_step = ms_total / args.steps
    dec_gbs = step_bytes / (dec_ms / 1e3) / 1e9
    unfused_bytes = decode_bytes(wl.lens) + append_bytes(BATCH)
    unfused = {"ms_per_step": round(unfused_ms / args.steps, 4),
               "gb_s": round(sum_over_ranks(unfused_bytes * args.steps, world, device)
                             / (unfused_ms / 1e3) / 1e9, 2),
               "pa_decode_ms": round(unfused_dec_ms, 4),
               "pa_decode_gb_s": round(decode_bytes(wl.lens) / (unfused_dec_ms / 1e3) / 1e9, 2)}
    peak, peak_kind = measured_peak()

    # ---- end-to-end steps through the C ABI from host buffers ------------------
    for _ in range(args.warmup):
        wl.e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e_start.record(stream)
    for _ in range(e2e_steps):
        wl.e2e_step()
    wl.e2e_drain()  # the last result copies are inside the timed region
    e_end.record(stream)
    torch.cuda.synchronize()
    # every e2e step grew each request by one token: timed step j decoded L + W + j + 1
    e2e_bytes = sum(decode_bytes([L + args.warmup + j + 1 for L in wl.lens])
                    + append_bytes(BATCH, slots=False) for j in range(e2e_steps))
    assert [wl.alloc.pa_seq_len(i) for i in wl.seq_ids] == \
        [L + args.warmup + e2e_steps for L in wl.lens]
    barrier(world)
    e2e_ms = max_over_ranks(e_start.elapsed_time(e_end), world, device)
    e2e_total = sum_over_ranks(e2e_bytes, world, device)
    e2e_value = e2e_total / (e2e_ms / 1e3) / 1e9
    flags = binding.pa_get_device_error()
    if flags:
        raise SystemExit(f"device error word set: {flags:#x}")

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cores = os.cpu_count() or 1
        v, desc = cpu_baseline(wl, 12.0, cores)
        cpu = {"value": round(v, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
               "sample": desc}

    if rank == 0:
        tok_s_layer = BATCH * world / (ms_per_step / 1e3)
        line = {
            "metric": METRIC, "value": round(value, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 4),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "batch_per_gpu": BATCH, "heads": H, "head_dim": D,
                       "block_size": S, "kv_bytes_per_step": step_bytes,
                       "partition": {"tokens": wl.plan[0], "num": wl.plan[1]},
                       "l2": "inputs larger than L2 (1.3 GB of KV per step vs 126 MB L2)",
                       "parallelism": f"dp{world} (independent batches, no collective)"},
            "decode_tok_s_layer": round(tok_s_layer, 1),
            "step": "pa_decode_append: the 64 new tokens' K/V appended inside the decode launch",
            "unfused_step": unfused,
            "roofline": {"bound": "hbm", "achieved": round(dec_gbs, 2), "peak": peak,
                         "unit": "GB/s", "frac": round(dec_gbs / peak, 4),
                         "peak_kind": peak_kind, "traffic": profiled_traffic(),
                         "peak_note": "peak is a STREAM-style copy (reads and writes mixed); "
                                      "a read-only stream can exceed it, so frac is a fraction "
                                      "of copy bandwidth and may pass 1",
                         "frac_of_copy_bw": round(dec_gbs / peak, 4),
                         "frac_of_nominal_8000": round(dec_gbs / 8000.0, 4),
                         "kernel": "pa_decode_append call: paged_decode_partition_kernel<APPEND> "
                                   "+ splitkv_reduce_kernel (launched as a programmatic "
                                   "dependent); timed together as one call",
                         "call_ms": round(dec_ms, 4),
                         "algorithmic_bytes_per_launch": step_bytes},
            "e2e": {"value": round(e2e_value, 2), "unit": "GB/s",
                    "api": "pa_stepper_step (host allocator step, uploads, pa_decode_append, "
                           "download; every request grows by one token per step)",
                    "h2d_bytes_per_step": wl.h2d_bytes(), "d2h_bytes_per_step": wl.d2h_bytes(),
                    "steps": e2e_steps, "ms_per_step": round(e2e_ms / e2e_steps, 4)},
            "gpu_launches": wl.launches_per_step(fused=True) * args.steps,
            "clocks": clk.summary(),
        }
        if cpu is not None:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
