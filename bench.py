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

H, D, S, BATCH, MAX_LEN = 40, 128, 16, 64, 2048
DTYPE = torch.bfloat16
ELEM = 2
METRIC = "paged decode attention KV GB/s"
WORKLOAD = "llama2-13b-shaped single-layer decode: 40 heads, head_dim 128, block 16, bf16, " \
           "batch 64, seq_lens U[1,2048], permuted pool"


def decode_bytes(lens):
    """Algorithmic bytes of one decode call: K and V of every live token, q and
    out, the block-table entries read and the seq_lens."""
    kv = sum(H * (2 * L * D * ELEM + 2 * D * ELEM) for L in lens)
    return kv + sum(4 * (-(-L // S)) for L in lens) + 4 * len(lens)


def append_bytes(T):
    return T * H * D * ELEM * 4 + 8 * T


class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index):
        visible = os.environ.get("CUDA_VISIBLE_DEVICES")
        ids = [x.strip() for x in visible.split(",")] if visible else []
        self.idx = ids[device_index] if device_index < len(ids) else str(device_index)
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.idx}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in getattr(self, "lines", []):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


def kernel_source_hash():
    h = hashlib.sha256()
    for f in ("pa_decode.cuh", "pa_device.cuh", "pa_api.cu"):
        with open(os.path.join(ROOT, "paged_kv_cache_driven_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
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
        # pinned host buffers of the end-to-end step
        self.h_q = self.q.cpu().pin_memory()
        self.h_k = self.k_new.cpu().pin_memory()
        self.h_v = self.v_new.cpu().pin_memory()
        self.h_slots = torch.empty(BATCH, dtype=torch.int64).pin_memory()
        self.h_tables = torch.empty((BATCH, self.MB), dtype=torch.int32).pin_memory()
        self.h_lens = torch.empty(BATCH, dtype=torch.int32).pin_memory()
        self.h_out = torch.empty((BATCH, H, D), dtype=DTYPE).pin_memory()
        self.d_q = torch.empty_like(self.q)
        self.d_k = torch.empty_like(self.k_new)
        self.d_v = torch.empty_like(self.v_new)
        self.d_slots = torch.empty(BATCH, dtype=torch.int64, device=device)
        self.d_tables = torch.empty((BATCH, self.MB), dtype=torch.int32, device=device)
        self.d_lens = torch.empty(BATCH, dtype=torch.int32, device=device)

    def launches_per_step(self):
        return 2 + (1 if self.plan[1] > 1 else 0)

    def device_step(self, ev_decode=None):
        binding.pa_kv_append(self.k_new, self.v_new, self.slots_d, self.k_cache, self.v_cache)
        if ev_decode is not None:
            ev_decode[0].record()
        binding.pa_decode(self.out, self.q, self.k_cache, self.v_cache, self.tables_d, self.lens_d,
                          self.scale, self.max_seq, partition=0, workspace=self.ws)
        if ev_decode is not None:
            ev_decode[1].record()

    def e2e_step(self):
        """One decode step through the public API from host memory. Returns the
        sequence lengths it decoded."""
        self.alloc.pa_prepare_step(self.seq_ids, 1, self.MB, self.h_slots, self.h_tables,
                                   self.h_lens)
        self.d_q.copy_(self.h_q, non_blocking=True)
        self.d_k.copy_(self.h_k, non_blocking=True)
        self.d_v.copy_(self.h_v, non_blocking=True)
        self.d_slots.copy_(self.h_slots, non_blocking=True)
        self.d_tables.copy_(self.h_tables, non_blocking=True)
        self.d_lens.copy_(self.h_lens, non_blocking=True)
        binding.pa_kv_append(self.d_k, self.d_v, self.d_slots, self.k_cache, self.v_cache)
        binding.pa_decode(self.out, self.d_q, self.k_cache, self.v_cache, self.d_tables,
                          self.d_lens, self.scale, int(self.h_lens.max()), partition=0,
                          workspace=self.ws)
        self.h_out.copy_(self.out, non_blocking=True)
        return self.h_lens.tolist()

    def h2d_bytes(self):
        return (3 * BATCH * H * D * ELEM + 8 * BATCH + 4 * BATCH * self.MB + 4 * BATCH)

    def d2h_bytes(self):
        return BATCH * H * D * ELEM


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


def cpu_oracle_sample(wl, target_seconds, cores):
    """Times the fp64 CPU oracle on a bounded sample of this workload's
    (request, head) pairs; returns (GB/s of KV, description)."""
    from oracle import decode as oracle_decode  # test infrastructure: the CPU baseline leg only

    tables = wl.tables_d.cpu()

    def sub_problem(pairs):
        ks, vs, qs, rows, lens = [], [], [], [], []
        off = 0
        for i, h in pairs:
            L = wl.lens[i]
            blocks = tables[i, : -(-L // S)].long().to(wl.device)
            ks.append(wl.k_cache[blocks, h].unsqueeze(1).cpu())
            vs.append(wl.v_cache[blocks, h].unsqueeze(1).cpu())
            qs.append(wl.q[i, h].view(1, 1, D).cpu())
            rows.append(list(range(off, off + len(blocks))))
            lens.append(L)
            off += len(blocks)
        MB = max(len(r) for r in rows)
        bt = torch.full((len(pairs), MB), -1, dtype=torch.int32)
        for r, row in enumerate(rows):
            bt[r, :len(row)] = torch.tensor(row, dtype=torch.int32)
        return (torch.cat(qs), torch.cat(ks), torch.cat(vs), bt,
                torch.tensor(lens, dtype=torch.int32))

    g = torch.Generator().manual_seed(123)
    all_pairs = [(i, h) for i in range(BATCH) for h in range(H)]
    perm = torch.randperm(len(all_pairs), generator=g).tolist()
    # calibrate on a few pairs, then size the sample for ~target_seconds
    n = 2 * cores
    while True:
        pairs = [all_pairs[k] for k in perm[:n]]
        prob = sub_problem(pairs)
        t0 = time.perf_counter()
        oracle_decode.paged_decode(*prob, wl.scale, threads=cores)
        dt = time.perf_counter() - t0
        if dt >= target_seconds * 0.5 or n >= len(all_pairs):
            break
        n = min(len(all_pairs), max(n * 2, int(n * target_seconds / max(dt, 1e-3))))
    nbytes = sum(2 * wl.lens[i] * D * ELEM for i, _ in pairs)
    desc = (f"{len(pairs)} of {BATCH * H} (request, head) pairs of the workload, "
            f"{sum(wl.lens[i] for i, _ in pairs)} tokens, {dt:.1f} s on {cores} threads")
    return nbytes / dt / 1e9, desc, dt


def run_reference(args):
    """The reference arm: the fp64 CPU oracle on the host cores, rank 0 only."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    device = "cuda" if torch.cuda.is_available() else "cpu"
    wl = Workload(seed=0, device=device, extra_tokens=0)
    cores = os.cpu_count() or 1
    vals = []
    for _ in range(args.warmup):
        cpu_oracle_sample(wl, 1.0, cores)
    desc = ""
    for _ in range(args.steps):
        v, desc, _ = cpu_oracle_sample(wl, 5.0, cores)
        vals.append(v)
    value = statistics.mean(vals)
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": {"workload": WORKLOAD, "l2": "inputs larger than L2"},
            "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": cores,
                             "kind": "oracle", "sample": desc},
            "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        raise SystemExit("--warmup must be at least 3")
    if args.impl == "reference":
        run_reference(args)
        return
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device")
    binding.lib()  # fail loudly if the library is missing
    rank, world, local = dist_setup(args.gpus)
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    extra = args.warmup + args.steps + 8
    wl = Workload(seed=args.seed + 1000 * rank, device=device, extra_tokens=extra)
    stream = torch.cuda.current_stream()

    # ---- device-resident steps -------------------------------------------------
    for _ in range(args.warmup):
        wl.device_step()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    dec_events = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(args.steps)]
    with ClockSampler(device.index if device.index is not None else 0) as clk:
        start.record(stream)
        for k in range(args.steps):
            wl.device_step(dec_events[k])
        end.record(stream)
        torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    ms_total = max_over_ranks(start.elapsed_time(end), world, device)
    dec_ms = statistics.mean(a.elapsed_time(b) for a, b in dec_events)
    flags = binding.pa_get_device_error()
    if flags:
        raise SystemExit(f"device error word set: {flags:#x}")
    step_bytes = decode_bytes(wl.lens) + append_bytes(BATCH)
    total_bytes = sum_over_ranks(step_bytes * args.steps, world, device)
    value = total_bytes / (ms_total / 1e3) / 1e9
    ms_per_step = ms_total / args.steps
    dec_gbs = decode_bytes(wl.lens) / (dec_ms / 1e3) / 1e9
    peak, peak_kind = measured_peak()

    # ---- end-to-end steps through the C ABI from host buffers ------------------
    for _ in range(args.warmup):
        wl.e2e_step()
    torch.cuda.synchronize()
    barrier(world)
    torch.cuda.synchronize()
    e_start, e_end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e2e_bytes = 0
    e_start.record(stream)
    for _ in range(args.steps):
        lens = wl.e2e_step()
        e2e_bytes += decode_bytes(lens) + append_bytes(BATCH)
    e_end.record(stream)
    torch.cuda.synchronize()
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
        v, desc, _ = cpu_oracle_sample(wl, 15.0, cores)
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
            "decode_only": {"ms": round(dec_ms, 4), "gb_s": round(dec_gbs, 2),
                            "tok_s_layer": round(BATCH / (dec_ms / 1e3), 1)},
            "roofline": {"bound": "hbm", "achieved": round(dec_gbs, 2), "peak": peak,
                         "unit": "GB/s", "frac": round(dec_gbs / peak, 4),
                         "peak_kind": peak_kind, "traffic": profiled_traffic(),
                         "kernel": "pa_decode (paged_decode_partition_kernel + splitkv_reduce_kernel)",
                         "algorithmic_bytes_per_launch": decode_bytes(wl.lens)},
            "e2e": {"value": round(e2e_value, 2), "unit": "GB/s",
                    "h2d_bytes_per_step": wl.h2d_bytes(), "d2h_bytes_per_step": wl.d2h_bytes(),
                    "ms_per_step": round(e2e_ms / args.steps, 4)},
            "gpu_launches": wl.launches_per_step() * args.steps,
            "clocks": clk.summary(),
        }
        if cpu is not None:
            line["cpu_baseline"] = cpu
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
