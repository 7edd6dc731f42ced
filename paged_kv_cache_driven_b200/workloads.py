"""Seeded synthetic inputs for the paged decode path.

These generators are the one module that both the CUDA path and the CPU oracle
consume; they hold none of the method's arithmetic (no slot computation, no
attention, no allocator policy). They only draw random numbers and lay them out
in the shapes the pages describe:

* the [Block, Head, Block_Size, Head_D] cache ("vLLM의 PagedAttention 아키텍처와
  GPU 메모리 최적화 원리", section 4), filled with N(0, 1) values;
* per-request block tables whose physical ids are a seeded random permutation of
  the pool ("vLLM KV Cache and PagedAttention Explained", Step 5: ids 42, 7, 23,
  61 are arbitrary), padded with -1;
* seq_lens drawn from the length mixes of the serving examples.

Structure (lengths, permutations, budgets) is drawn on the CPU with
``torch.Generator('cpu')`` so it is identical on every machine; bulk values are
drawn on the target device. Every byte a request does not own -- tail slots past
its length, blocks no table names -- is set to NaN ("poison"), so any read that
is not masked shows up in the output.
"""

from dataclasses import dataclass, field
import math

import torch

_BLOCK_POISON = float("nan")


@dataclass
class DecodeCase:
    """One batch of decode inputs, all tensors on ``device``."""

    q: torch.Tensor             # [B, H, D]
    k_cache: torch.Tensor       # [NB, H, S, D]
    v_cache: torch.Tensor       # [NB, H, S, D]
    block_tables: torch.Tensor  # [B, MB] int32, -1 padded
    seq_lens: torch.Tensor      # [B] int32
    scale: float
    seq_lens_host: list = field(default_factory=list)
    tables_host: list = field(default_factory=list)

    @property
    def shape(self):
        NB, H, S, D = self.k_cache.shape
        return dict(B=self.q.shape[0], H=H, D=D, S=S, NB=NB, MB=self.block_tables.shape[1])


def _cpu_gen(seed):
    return torch.Generator("cpu").manual_seed(int(seed))


def _dev_gen(seed, device):
    return torch.Generator(device=device).manual_seed(int(seed) + 0x5EED)


def uniform_lengths(n, lo, hi, seed):
    """n integers uniform in [lo, hi]."""
    return torch.randint(lo, hi + 1, (n,), generator=_cpu_gen(seed)).tolist()


def lognormal_lengths(n, median, sigma, lo, hi, gen):
    """round(exp(N(ln median, sigma))) clipped to [lo, hi]."""
    x = torch.empty(n, dtype=torch.float64).log_normal_(math.log(median), sigma, generator=gen)
    return x.round().clamp(lo, hi).to(torch.int64).tolist()


def decode_case(seq_lens, H, D, S, dtype, seed, device, pool_blocks=None, poison=True,
                max_blocks=None, Hkv=None):
    """A batch of single-query decode inputs (Hkv KV heads in the cache, H query
    heads; Hkv defaults to H).

    Request i holds the first ceil(L_i / S) ids of its share of a random
    permutation of the pool; ``pool_blocks`` (default: exactly enough) sets the
    pool size; ``max_blocks`` (default: the widest table) the table width.
    """
    gen = _cpu_gen(seed)
    B = len(seq_lens)
    nblk = [-(-int(L) // S) for L in seq_lens]
    need = sum(nblk)
    NB = need if pool_blocks is None else int(pool_blocks)
    if NB < need:
        raise ValueError("pool too small for the requested lengths")
    MB = max(nblk + [1]) if max_blocks is None else int(max_blocks)
    perm = torch.randperm(NB, generator=gen)
    tables = torch.full((B, MB), -1, dtype=torch.int32)
    tables_host = []
    off = 0
    for i, n in enumerate(nblk):
        ids = perm[off:off + n]
        tables[i, :n] = ids.to(torch.int32)
        tables_host.append(ids.tolist())
        off += n
    dgen = _dev_gen(seed, device)
    Hc = H if Hkv is None else Hkv
    q = torch.randn((B, H, D), generator=dgen, device=device, dtype=torch.float32).to(dtype)
    k_cache = torch.randn((NB, Hc, S, D), generator=dgen, device=device, dtype=dtype)
    v_cache = torch.randn((NB, Hc, S, D), generator=dgen, device=device, dtype=dtype)
    if poison:
        unused = perm[need:].to(device)
        if unused.numel():
            k_cache[unused] = _BLOCK_POISON
            v_cache[unused] = _BLOCK_POISON
        for i, L in enumerate(seq_lens):
            tail = int(L) % S
            if tail and nblk[i]:
                b = tables_host[i][-1]
                k_cache[b, :, tail:, :] = _BLOCK_POISON
                v_cache[b, :, tail:, :] = _BLOCK_POISON
    return DecodeCase(q=q, k_cache=k_cache, v_cache=v_cache,
                      block_tables=tables.to(device), seq_lens=torch.tensor(
                          [int(L) for L in seq_lens], dtype=torch.int32, device=device),
                      scale=1.0 / math.sqrt(D), seq_lens_host=[int(L) for L in seq_lens],
                      tables_host=tables_host)


# ---------------------------------------------------------------------------
# The five workloads, named by what they are.
# ---------------------------------------------------------------------------

def worked_example(seed=0, device="cpu"):
    """Four requests of 6/50/8/100 tokens ("vLLM KV Cache and PagedAttention
    Explained", 6단계), block_size 16, 4 heads, head_dim 64, fp16, in a 64-block
    pool whose ids are a seeded permutation; 51 blocks are unused and poisoned."""
    return decode_case([6, 50, 8, 100], H=4, D=64, S=16, dtype=torch.float16, seed=seed,
                       device=device, pool_blocks=64)


def llama13b_decode(seed=0, device="cpu", batch=64, max_len=2048):
    """LLaMA-2-13B-shaped single-layer decode: 40 heads, head_dim 128, block 16,
    bf16, batch 64, seq_lens uniform in [1, 2048], pool sized exactly."""
    lens = uniform_lengths(batch, 1, max_len, seed)
    return decode_case(lens, H=40, D=128, S=16, dtype=torch.bfloat16, seed=seed, device=device)


def long_context_decode(seed=0, device="cpu", batch=8, lo=32768, hi=131072, H=32):
    """Long-context split-KV decode: batch 8, seq_lens uniform in [32768, 131072],
    32 heads, head_dim 128, block 16, bf16, permuted pool."""
    lens = uniform_lengths(batch, lo, hi, seed)
    return decode_case(lens, H=H, D=128, S=16, dtype=torch.bfloat16, seed=seed, device=device)


def llama70b_decode(seed=0, device="cpu", batch=64, max_len=2048):
    """LLaMA-2-70B-shaped single-layer decode (grouped-query attention, not on the
    pages): 64 query heads sharing 8 KV heads, head_dim 128, block 16, bf16,
    seq_lens uniform in [1, 2048]."""
    lens = uniform_lengths(batch, 1, max_len, seed)
    return decode_case(lens, H=64, D=128, S=16, dtype=torch.bfloat16, seed=seed, device=device,
                       Hkv=8)


def sweep_case(S, D, B, dtype, seed=0, device="cpu", H=32, lo=16, hi=8192):
    """One point of the shape sweep: 32 heads, seq_lens uniform in [16, 8192]."""
    lens = uniform_lengths(B, lo, hi, seed)
    return decode_case(lens, H=H, D=D, S=S, dtype=dtype, seed=seed, device=device)


@dataclass
class PrefillCase:
    """Prefill inputs: the cache already holds every request's tokens (context
    and new), q [T, H, D] packs the new tokens' queries request after request."""

    cache: DecodeCase        # caches, tables, seq_lens (total tokens per request)
    q: torch.Tensor          # [T, H, D]
    q_start: torch.Tensor    # [B + 1] int32, on the device
    new_lens: list           # new tokens per request
    ctx_lens: list           # tokens cached before them

    @property
    def max_q_len(self):
        return max(self.new_lens + [0])


def prefill_case(ctx_lens, new_lens, H, D, S, dtype, seed, device, Hkv=None, pool_blocks=None):
    """Request i has ctx_lens[i] tokens cached earlier and new_lens[i] new ones,
    all already in the (poisoned, permuted) cache; q holds the new tokens' queries."""
    lens = [int(c) + int(n) for c, n in zip(ctx_lens, new_lens)]
    cache = decode_case(lens, H=H, D=D, S=S, dtype=dtype, seed=seed, device=device, Hkv=Hkv,
                        pool_blocks=pool_blocks)
    T = sum(int(n) for n in new_lens)
    g = _dev_gen(seed + 77, device)
    q = torch.randn((T, H, D), generator=g, device=device, dtype=torch.float32).to(dtype)
    starts = [0]
    for n in new_lens:
        starts.append(starts[-1] + int(n))
    return PrefillCase(cache=cache, q=q, q_start=torch.tensor(starts, dtype=torch.int32,
                                                               device=device),
                       new_lens=[int(n) for n in new_lens], ctx_lens=[int(c) for c in ctx_lens])


def prompt_prefill(seed=0, device="cpu", n_req=16, lo=512, hi=4096, H=32, D=128, S=16,
                   dtype=torch.bfloat16):
    """Prompt prefill attention: 16 prompts of uniform [512, 4096] tokens, no
    earlier context, 32 heads, head_dim 128, block 16, bf16, permuted pool."""
    n_tok = torch.randint(lo, hi + 1, (n_req,), generator=_cpu_gen(seed)).tolist()
    return prefill_case([0] * n_req, n_tok, H=H, D=D, S=S, dtype=dtype, seed=seed, device=device)


@dataclass
class AppendCase:
    """Tokens to scatter: k, v [T, H, D], plus where each request's tokens go."""

    k: torch.Tensor
    v: torch.Tensor
    k_cache: torch.Tensor
    v_cache: torch.Tensor
    n_tokens: list           # tokens per request, in order
    block_order: list        # the order in which pool ids are handed out


def prefill_append(seed=0, device="cpu", n_req=16, lo=512, hi=4096, H=32, D=128, S=16,
                   dtype=torch.bfloat16, spare_blocks=64):
    """Prefill-scale append: 16 requests of uniform [512, 4096] tokens each, their
    K/V to be scattered into a pool handed out in a seeded random order."""
    gen = _cpu_gen(seed)
    n_tok = torch.randint(lo, hi + 1, (n_req,), generator=gen).tolist()
    NB = sum(-(-n // S) for n in n_tok) + spare_blocks
    order = torch.randperm(NB, generator=gen).tolist()
    T = sum(n_tok)
    dgen = _dev_gen(seed, device)
    k = torch.randn((T, H, D), generator=dgen, device=device, dtype=dtype)
    v = torch.randn((T, H, D), generator=dgen, device=device, dtype=dtype)
    k_cache = torch.randn((NB, H, S, D), generator=dgen, device=device, dtype=dtype)
    v_cache = torch.randn((NB, H, S, D), generator=dgen, device=device, dtype=dtype)
    return AppendCase(k=k, v=v, k_cache=k_cache, v_cache=v_cache, n_tokens=n_tok,
                      block_order=order)


@dataclass
class BatchingLoop:
    """Random draws of the continuous-batching loop (40 heads, head_dim 128, bf16).

    initial_lens: prompt lengths of the first ``batch`` requests.
    budgets: decode tokens each of those requests produces before it stops.
    arrivals: an endless stream of (prompt_len, budget) for replacements.
    block_order: the shuffled order in which the free list hands out ids.
    """

    batch: int
    H: int
    D: int
    S: int
    dtype: torch.dtype
    num_blocks: int
    initial_lens: list
    budgets: list
    block_order: list
    seed: int
    _gen: torch.Generator = None

    def arrival(self):
        """(prompt_len, budget) of the next replacement request."""
        L = lognormal_lengths(1, 300, 1.0, 1, 4096, self._gen)[0]
        b = int(torch.empty(1, dtype=torch.float64).geometric_(1.0 / 128, generator=self._gen)
                .item())
        return L, b

    def token_kv(self, step, n, device):
        """q, k, v [n, H, D] for the tokens decoded at ``step``."""
        g = _dev_gen(self.seed * 1000003 + step, device)
        shape = (n, self.H, self.D)
        return (torch.randn(shape, generator=g, device=device, dtype=self.dtype),
                torch.randn(shape, generator=g, device=device, dtype=self.dtype),
                torch.randn(shape, generator=g, device=device, dtype=self.dtype))

    def prompt_kv(self, req_serial, n, device):
        """k, v [n, H, D] for a prompt's prefill append."""
        g = _dev_gen(self.seed * 7919 + 104729 * (req_serial + 1), device)
        shape = (n, self.H, self.D)
        return (torch.randn(shape, generator=g, device=device, dtype=self.dtype),
                torch.randn(shape, generator=g, device=device, dtype=self.dtype))


def batching_loop(seed=0, batch=256, H=40, D=128, S=16, dtype=torch.bfloat16, max_len=4096,
                  headroom=64):
    """The continuous-batching loop: batch 256, prompt lengths lognormal with median
    300 clipped to [1, 4096], geometric stop budgets with mean 128, a pool of
    batch * ceil((4096 + 64) / 16) blocks handed out in a seeded shuffled order."""
    gen = _cpu_gen(seed)
    lens = lognormal_lengths(batch, 300, 1.0, 1, max_len, gen)
    budgets = torch.empty(batch, dtype=torch.float64).geometric_(1.0 / 128, generator=gen)
    NB = batch * (-(-(max_len + headroom) // S))
    order = torch.randperm(NB, generator=gen).tolist()
    return BatchingLoop(batch=batch, H=H, D=D, S=S, dtype=dtype, num_blocks=NB,
                        initial_lens=lens, budgets=[int(b) for b in budgets.tolist()],
                        block_order=order, seed=seed, _gen=gen)
