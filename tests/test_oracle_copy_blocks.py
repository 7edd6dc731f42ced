"""Pin for the oracle's copy-on-write block copy (CPU only).

"vLLM KV Cache and PagedAttention Explained", Step 9 "Safe Sharing with
Copy-on-Write": before a sequence writes into a physical block that another
table also names, the block is copied to a private block and the writer's table
is repointed. The device half of that is a bit copy of whole physical blocks
(every head, K and V). ``oracle.append.copy_blocks_into`` is the expected value
for ``pa_copy_blocks``; here it is pinned against an independent formulation:
torch ``index_copy_`` along the block dimension of the [NB, H, S, D] caches,
with every source block read (gathered) before any destination is written.

The test also shows that plausible mistakes in the oracle (copying K only,
swapping source and destination, copying one head, dropping a pair that shares
its source with another) fail the pin; the mistakes are planted in local copies
of the function, on the CPU.
"""

import numpy as np
import torch

from oracle import append as oracle_append


def bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def by_index_copy(kc, vc, pairs):
    """Independent formulation: gather every source block first, then write
    them at their destinations with index_copy_ on dim 0."""
    src = torch.tensor([s for s, _ in pairs], dtype=torch.int64)
    dst = torch.tensor([d for _, d in pairs], dtype=torch.int64)
    outs = []
    for c in (kc, vc):
        c2 = c.clone()
        if len(pairs):
            c2.index_copy_(0, dst, c.index_select(0, src))
        outs.append(bits(c2))
    return outs


def cases():
    """(k_cache, v_cache, pairs) with distinct destinations that are not
    sources, as pa_copy_blocks requires."""
    g = torch.Generator().manual_seed(21)
    out = []
    for NB, H, S, D, dtype in ((12, 3, 8, 16, torch.float16), (30, 4, 16, 64, torch.bfloat16)):
        kc = torch.randn(NB, H, S, D, generator=g).to(dtype)
        vc = torch.randn(NB, H, S, D, generator=g).to(dtype)
        perm = torch.randperm(NB, generator=g).tolist()
        srcs, dsts = perm[:3], perm[3:9]
        # several pairs share a source (parallel sampling: one shared prompt
        # block copied for several writers), one pair has its own source
        pairs = [(srcs[0], dsts[0]), (srcs[0], dsts[1]), (srcs[1], dsts[2]),
                 (srcs[0], dsts[3]), (srcs[2], dsts[4])]
        out.append((kc, vc, pairs))
        out.append((kc, vc, []))               # nothing queued: nothing changes
        out.append((kc, vc, [(srcs[1], dsts[5])]))
    return out


def agrees(copy_fn):
    """True when copy_fn (the oracle's signature) equals the independent
    formulation on every case, and leaves every block that is not a destination
    with its bytes."""
    for kc, vc, pairs in cases():
        want_k, want_v = by_index_copy(kc, vc, pairs)
        got_k, got_v = bits(kc).copy(), bits(vc).copy()
        copy_fn(got_k, got_v, pairs)
        if not (np.array_equal(got_k, want_k) and np.array_equal(got_v, want_v)):
            return False
        dst = {d for _, d in pairs}
        keep = [b for b in range(kc.shape[0]) if b not in dst]
        if not (np.array_equal(got_k[keep], bits(kc)[keep])
                and np.array_equal(got_v[keep], bits(vc)[keep])):
            return False
        for s, d in pairs:  # each destination is now a bit copy of its source
            if not (np.array_equal(got_k[d], bits(kc)[s]) and np.array_equal(got_v[d], bits(vc)[s])):
                return False
    return True


def test_copy_blocks_into_matches_index_copy():
    assert agrees(oracle_append.copy_blocks_into)


def test_copy_blocks_pin_catches_plausible_mistakes():
    def k_only(kc, vc, pairs):
        for s, d in pairs:
            kc[d] = kc[s]

    def swapped(kc, vc, pairs):
        for s, d in pairs:
            kc[s] = kc[d]
            vc[s] = vc[d]

    def one_head(kc, vc, pairs):
        for s, d in pairs:
            kc[d, 0] = kc[s, 0]
            vc[d, 0] = vc[s, 0]

    def first_per_source(kc, vc, pairs):
        seen = set()
        for s, d in pairs:
            if s in seen:
                continue
            seen.add(s)
            kc[d] = kc[s]
            vc[d] = vc[s]

    def v_into_k(kc, vc, pairs):
        for s, d in pairs:
            kc[d] = vc[s]
            vc[d] = vc[s]

    for mutant in (k_only, swapped, one_head, first_per_source, v_into_k):
        assert not agrees(mutant), mutant.__name__


def test_copy_then_decode_reads_the_same_tokens():
    """After the copy, a table that names the private block instead of the
    shared one decodes to the same attention output (the fp64 oracle), which is
    what the writer needs before it appends its own token."""
    from oracle import decode as oracle_decode

    kc, vc, pairs = cases()[3]
    s, d = pairs[0]
    k2, v2 = bits(kc).copy(), bits(vc).copy()
    oracle_append.copy_blocks_into(k2, v2, pairs)
    H, D = kc.shape[1], kc.shape[3]
    S = kc.shape[2]
    q = torch.randn(1, H, D, generator=torch.Generator().manual_seed(5)).to(kc.dtype)
    lens = torch.tensor([S], dtype=torch.int32)
    shared = oracle_decode.paged_decode(q, k2, v2, torch.tensor([[s]], dtype=torch.int32), lens,
                                        0.125, dtype=kc.dtype)
    private = oracle_decode.paged_decode(q, k2, v2, torch.tensor([[d]], dtype=torch.int32), lens,
                                         0.125, dtype=kc.dtype)
    assert np.array_equal(shared, private)
