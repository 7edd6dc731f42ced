"""Shared test utilities: run the CUDA path through the C ABI, run the oracle on
the same seeded inputs, and compare at the stated tolerance."""

import numpy as np
import torch

from oracle import decode as oracle_decode
from paged_kv_cache_driven_b200 import binding

# Attention outputs (fp16/bf16 inputs, fp32 accumulation, fp32 output) against
# the fp64 oracle on N(0, 1) inputs.
MAX_ABS = 4e-3
REL_L2 = 1e-3


def parity_stats(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    err = np.abs(got - want)
    rel = np.linalg.norm((got - want).ravel()) / max(np.linalg.norm(want.ravel()), 1e-300)
    return float(err.max(initial=0.0)), float(rel)


def assert_parity(got, want, what=""):
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    mx, rel = parity_stats(got, want)
    assert mx <= MAX_ABS and rel <= REL_L2, f"{what}: max|d|={mx:.3e} relL2={rel:.3e}"
    return mx, rel


def run_decode(case, out_dtype=torch.float32, partition=0, max_seq_len=None, stream=None):
    """pa_decode on a workloads.DecodeCase; returns the output tensor."""
    B, H, D = case.q.shape
    S = case.k_cache.shape[2]
    if max_seq_len is None:
        max_seq_len = max(case.seq_lens_host + [0])
    out = torch.empty((B, H, D), dtype=out_dtype, device=case.q.device)
    ws_bytes = binding.pa_decode_workspace_bytes(B, H, D, S, max_seq_len, partition)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=case.q.device) if ws_bytes else None
    if case.k_cache.shape[1] != H:  # grouped query heads
        binding.pa_decode_gqa(out, case.q, case.k_cache, case.v_cache, case.block_tables,
                              case.seq_lens, case.scale, max_seq_len, partition=partition,
                              workspace=ws, stream=stream)
    else:
        binding.pa_decode(out, case.q, case.k_cache, case.v_cache, case.block_tables,
                          case.seq_lens, case.scale, max_seq_len, partition=partition,
                          workspace=ws, stream=stream)
    return out, ws


def oracle_full(case, threads=0):
    """The oracle over every (request, head) of a small case (copies it to the host)."""
    return oracle_decode.paged_decode(case.q.cpu(), case.k_cache.cpu(), case.v_cache.cpu(),
                                      case.block_tables.cpu(), case.seq_lens.cpu(), case.scale,
                                      threads=threads)


def oracle_pairs(case, pairs, threads=0):
    """The oracle on sampled (request, head) pairs of a case of any size.

    Only the sampled pairs' blocks are copied to the host: each pair becomes a
    one-head request whose blocks are renumbered 0..n-1 (a relabelling of
    physical ids, which the oracle's pins show leaves the result unchanged).
    Returns [len(pairs), D] fp64.
    """
    S = case.k_cache.shape[2]
    D = case.q.shape[2]
    G = case.q.shape[1] // case.k_cache.shape[1]  # query heads per KV head
    ks, vs, qs, tables, lens = [], [], [], [], []
    off = 0
    for i, h in pairs:
        L = case.seq_lens_host[i]
        blocks = case.tables_host[i][: -(-L // S)]
        n = len(blocks)
        idx = torch.tensor(blocks, dtype=torch.long, device=case.k_cache.device)
        ks.append(case.k_cache[idx, h // G].unsqueeze(1).cpu())
        vs.append(case.v_cache[idx, h // G].unsqueeze(1).cpu())
        qs.append(case.q[i, h].view(1, 1, D).cpu())
        tables.append(list(range(off, off + n)))
        lens.append(L)
        off += n
    MB = max([len(t) for t in tables] + [1])
    bt = torch.full((len(pairs), MB), -1, dtype=torch.int32)
    for r, t in enumerate(tables):
        bt[r, :len(t)] = torch.tensor(t, dtype=torch.int32)
    kc = torch.cat(ks) if off else torch.zeros((1, 1, S, D), dtype=case.q.dtype)
    vc = torch.cat(vs) if off else torch.zeros((1, 1, S, D), dtype=case.q.dtype)
    out = oracle_decode.paged_decode(torch.cat(qs), kc, vc, bt, torch.tensor(lens, dtype=torch.int32),
                                     case.scale, threads=threads)
    return out[:, 0, :]


def sample_pairs(case, n, seed=0):
    """n (request, head) pairs: the longest and shortest requests, then random ones."""
    g = torch.Generator().manual_seed(seed)
    B, H = case.q.shape[0], case.q.shape[1]
    lens = case.seq_lens_host
    order = sorted(range(B), key=lambda i: lens[i])
    picks = [(order[-1], 0), (order[-1], H - 1), (order[0], H // 2)]
    while len(picks) < n:
        i = int(torch.randint(0, B, (1,), generator=g))
        h = int(torch.randint(0, H, (1,), generator=g))
        picks.append((i, h))
    return picks[:n]


def run_prefill(pc, out_dtype=torch.float32, max_q_len=None, stream=None):
    """pa_prefill on a workloads.PrefillCase; returns out [T, H, D]."""
    T, H, D = pc.q.shape
    out = torch.empty((T, H, D), dtype=out_dtype, device=pc.q.device)
    c = pc.cache
    binding.pa_prefill(out, pc.q, c.k_cache, c.v_cache, c.block_tables, c.seq_lens, pc.q_start,
                       c.scale, pc.max_q_len if max_q_len is None else max_q_len, stream=stream)
    return out


def oracle_prefill_full(pc, threads=0):
    """The oracle's causal prefill over a whole small case."""
    c = pc.cache
    return oracle_decode.paged_prefill(pc.q.cpu(), c.k_cache.cpu(), c.v_cache.cpu(),
                                       c.block_tables.cpu(), c.seq_lens.cpu(), pc.q_start.cpu(),
                                       c.scale, threads=threads)


def oracle_prefill_rows(pc, picks, threads=0):
    """The oracle on sampled (request, new-token index, head) triples of a case of
    any size. Row j of request i is the decode of that query over the first
    ctx_i + j + 1 cached tokens (the oracle's pins show the two agree), so each
    triple becomes a one-head decode over only the blocks it reads. Returns
    [len(picks), D] fp64."""
    c = pc.cache
    S = c.k_cache.shape[2]
    D = pc.q.shape[2]
    G = pc.q.shape[1] // c.k_cache.shape[1]
    qs = pc.q_start.cpu().tolist()
    ks, vs, qrows, tables, lens = [], [], [], [], []
    off = 0
    for i, j, h in picks:
        L = pc.ctx_lens[i] + j + 1
        blocks = c.tables_host[i][: -(-L // S)]
        idx = torch.tensor(blocks, dtype=torch.long, device=c.k_cache.device)
        ks.append(c.k_cache[idx, h // G].unsqueeze(1).cpu())
        vs.append(c.v_cache[idx, h // G].unsqueeze(1).cpu())
        qrows.append(pc.q[qs[i] + j, h].view(1, 1, D).cpu())
        tables.append(list(range(off, off + len(blocks))))
        lens.append(L)
        off += len(blocks)
    MB = max(len(t) for t in tables)
    bt = torch.full((len(picks), MB), -1, dtype=torch.int32)
    for r, t in enumerate(tables):
        bt[r, :len(t)] = torch.tensor(t, dtype=torch.int32)
    out = oracle_decode.paged_decode(torch.cat(qrows), torch.cat(ks), torch.cat(vs), bt,
                                     torch.tensor(lens, dtype=torch.int32), c.scale,
                                     threads=threads)
    return out[:, 0, :]
