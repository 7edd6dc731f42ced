"""Pins for the fp64 decode oracle and the append oracle (CPU only).

The oracle is pinned to things other than itself:
* torch's own fp16/bf16 -> fp64 conversion, for every one of the 65536 bit patterns;
* contiguous-KV attention computed by torch's scaled_dot_product_attention in
  fp64 (the "PagedAttention" card, "Kernel은 무엇이 달라지는가": the paged kernel
  computes the same attention without gathering the blocks into one tensor);
* invariance under any relabelling of physical block ids ("vLLM KV Cache and
  PagedAttention Explained", Step 5: ids 42 / 7, 23, 61 are arbitrary);
* closed forms: one token, equal keys, zero query, two tokens (a sigmoid);
* the log-sum-exp merge of per-partition statistics reproducing the full result;
* torch's index_copy_ for the slot_mapping scatter.
"""

import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import append as oracle_append
from oracle import decode as oracle_decode


def make_paged(contig_k, contig_v, S, pool_extra, gen):
    """Scatter per-request contiguous K/V [L_i, H, D] into a permuted paged pool.

    Returns (k_cache, v_cache, block_tables, seq_lens). Unowned bytes are NaN.
    """
    lens = [k.shape[0] for k in contig_k]
    H, D = contig_k[0].shape[1], contig_k[0].shape[2]
    nblk = [-(-L // S) for L in lens]
    NB = sum(nblk) + pool_extra
    perm = torch.randperm(NB, generator=gen)
    dtype = contig_k[0].dtype
    kc = torch.full((NB, H, S, D), float("nan"), dtype=dtype)
    vc = torch.full((NB, H, S, D), float("nan"), dtype=dtype)
    MB = max(nblk + [1])
    bt = torch.full((len(lens), MB), -1, dtype=torch.int32)
    off = 0
    for i, L in enumerate(lens):
        for j in range(nblk[i]):
            b = int(perm[off + j])
            bt[i, j] = b
            n = min(S, L - j * S)
            kc[b, :, :n, :] = contig_k[i][j * S:j * S + n].transpose(0, 1)
            vc[b, :, :n, :] = contig_v[i][j * S:j * S + n].transpose(0, 1)
        off += nblk[i]
    return kc, vc, bt, torch.tensor(lens, dtype=torch.int32)


def dense_reference(q, contig_k, contig_v, scale):
    """fp64 attention of each request over its contiguous K/V, by torch SDPA."""
    outs = []
    for i in range(q.shape[0]):
        qi = q[i].double().unsqueeze(1)                 # [H, 1, D]
        ki = contig_k[i].double().transpose(0, 1)       # [H, L, D]
        vi = contig_v[i].double().transpose(0, 1)
        if ki.shape[1] == 0:
            outs.append(torch.zeros(q.shape[1], q.shape[2], dtype=torch.float64))
            continue
        outs.append(F.scaled_dot_product_attention(qi, ki, vi, scale=scale).squeeze(1))
    return torch.stack(outs).numpy()


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
def test_decode16_matches_torch_for_every_bit_pattern(oracle_lib, dtype):
    bits = np.arange(65536, dtype=np.uint16)
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(dtype).double().numpy()
    got = np.array([oracle_decode.decode16(int(b), dtype) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(nan, np.isnan(got))
    assert np.array_equal(ref[~nan], got[~nan])


@pytest.mark.parametrize("dtype", [torch.float16, torch.bfloat16])
@pytest.mark.parametrize("S,D", [(8, 1), (16, 2), (16, 4), (32, 64), (16, 128), (8, 256)])
def test_paged_equals_contiguous_sdpa(oracle_lib, dtype, S, D):
    gen = torch.Generator().manual_seed(S * 1000 + D)
    H = 3
    lens = [1, S - 1, S, S + 1, 3 * S + 5, 7 * S]
    ks = [torch.randn(L, H, D, generator=gen).to(dtype) for L in lens]
    vs = [torch.randn(L, H, D, generator=gen).to(dtype) for L in lens]
    q = torch.randn(len(lens), H, D, generator=gen).to(dtype)
    kc, vc, bt, sl = make_paged(ks, vs, S, pool_extra=5, gen=gen)
    scale = 1.0 / math.sqrt(D)
    got = oracle_decode.paged_decode(q, kc, vc, bt, sl, scale)
    want = dense_reference(q, ks, vs, scale)
    np.testing.assert_allclose(got, want, rtol=1e-12, atol=1e-12)


def test_permutation_invariance(oracle_lib):
    gen = torch.Generator().manual_seed(7)
    S, H, D = 16, 2, 32
    lens = [6, 50, 8, 100]
    ks = [torch.randn(L, H, D, generator=gen).half() for L in lens]
    vs = [torch.randn(L, H, D, generator=gen).half() for L in lens]
    q = torch.randn(4, H, D, generator=gen).half()
    kc, vc, bt, sl = make_paged(ks, vs, S, pool_extra=51, gen=gen)
    base = oracle_decode.paged_decode(q, kc, vc, bt, sl, 0.125)
    for trial in range(3):
        pi = torch.randperm(kc.shape[0], generator=gen)
        kc2 = torch.empty_like(kc)
        vc2 = torch.empty_like(vc)
        kc2[pi] = kc
        vc2[pi] = vc
        bt2 = torch.where(bt >= 0, pi[bt.clamp(min=0).long()].to(torch.int32), bt)
        got = oracle_decode.paged_decode(q, kc2, vc2, bt2, sl, 0.125)
        assert np.array_equal(got, base)


def test_closed_forms(oracle_lib):
    gen = torch.Generator().manual_seed(3)
    S, H, D = 8, 2, 16
    # one token: the output is that token's V exactly
    k1 = [torch.randn(1, H, D, generator=gen).to(torch.bfloat16)]
    v1 = [torch.randn(1, H, D, generator=gen).to(torch.bfloat16)]
    q = torch.randn(1, H, D, generator=gen).to(torch.bfloat16)
    kc, vc, bt, sl = make_paged(k1, v1, S, 2, gen)
    out = oracle_decode.paged_decode(q, kc, vc, bt, sl, 0.3)
    assert np.array_equal(out[0], v1[0][0].double().numpy())
    # equal keys (or a zero query): the output is the mean of V
    L = 3 * S + 3
    kk = torch.randn(1, H, D, generator=gen).to(torch.bfloat16).expand(L, H, D).contiguous()
    vv = torch.randn(L, H, D, generator=gen).to(torch.bfloat16)
    kc, vc, bt, sl = make_paged([kk], [vv], S, 4, gen)
    out = oracle_decode.paged_decode(q, kc, vc, bt, sl, 0.3)
    np.testing.assert_allclose(out[0], vv.double().mean(0).numpy(), rtol=0, atol=1e-14)
    kr = torch.randn(L, H, D, generator=gen).to(torch.bfloat16)
    kc, vc, bt, sl = make_paged([kr], [vv], S, 4, gen)
    out = oracle_decode.paged_decode(torch.zeros_like(q), kc, vc, bt, sl, 0.3)
    np.testing.assert_allclose(out[0], vv.double().mean(0).numpy(), rtol=0, atol=1e-14)
    # two tokens: weights sigmoid(s0 - s1) and sigmoid(s1 - s0)
    k2 = torch.randn(2, H, D, generator=gen).to(torch.bfloat16)
    v2 = torch.randn(2, H, D, generator=gen).to(torch.bfloat16)
    kc, vc, bt, sl = make_paged([k2], [v2], S, 0, gen)
    out = oracle_decode.paged_decode(q, kc, vc, bt, sl, 0.3)
    qd, kd, vd = q[0].double(), k2.double(), v2.double()
    for h in range(H):
        s0 = 0.3 * float(qd[h] @ kd[0, h])
        s1 = 0.3 * float(qd[h] @ kd[1, h])
        w0 = 1.0 / (1.0 + math.exp(s1 - s0))
        want = w0 * vd[0, h] + (1.0 - w0) * vd[1, h]
        np.testing.assert_allclose(out[0, h], want.numpy(), rtol=0, atol=1e-14)


def test_empty_request_and_bad_block(oracle_lib):
    gen = torch.Generator().manual_seed(4)
    H, D, S = 2, 8, 8
    ks = [torch.randn(L, H, D, generator=gen).half() for L in (0, 9)]
    vs = [torch.randn(L, H, D, generator=gen).half() for L in (0, 9)]
    q = torch.randn(2, H, D, generator=gen).half()
    kc, vc, bt, sl = make_paged(ks, vs, S, 1, gen)
    out = oracle_decode.paged_decode(q, kc, vc, bt, sl, 0.5)
    assert np.all(out[0] == 0.0)
    assert np.all(np.isfinite(out[1]))
    bad = bt.clone()
    bad[1, 0] = kc.shape[0]
    with pytest.raises(oracle_decode.OracleError):
        oracle_decode.paged_decode(q, kc, vc, bad, sl, 0.5)


def test_pairs_subset_matches_full(oracle_lib):
    gen = torch.Generator().manual_seed(5)
    H, D, S = 4, 16, 16
    lens = [30, 1, 77]
    ks = [torch.randn(L, H, D, generator=gen).half() for L in lens]
    vs = [torch.randn(L, H, D, generator=gen).half() for L in lens]
    q = torch.randn(3, H, D, generator=gen).half()
    kc, vc, bt, sl = make_paged(ks, vs, S, 3, gen)
    full = oracle_decode.paged_decode(q, kc, vc, bt, sl, 0.25, threads=1)
    pairs = [(2, 3), (0, 1), (1, 0)]
    sub = oracle_decode.paged_decode(q, kc, vc, bt, sl, 0.25, pairs=pairs, threads=3)
    for k, (i, h) in enumerate(pairs):
        assert np.array_equal(sub[k], full[i, h])


@pytest.mark.parametrize("P", [8, 16, 48, 512])
def test_partition_stats_merge_to_full(oracle_lib, P):
    """FlashDecoding split: log-sum-exp merge of the partitions = the full softmax."""
    gen = torch.Generator().manual_seed(P)
    H, D, S = 2, 32, 8
    lens = [1, 7, 8, 9, 100, 333]
    ks = [torch.randn(L, H, D, generator=gen).to(torch.bfloat16) for L in lens]
    vs = [torch.randn(L, H, D, generator=gen).to(torch.bfloat16) for L in lens]
    q = torch.randn(len(lens), H, D, generator=gen).to(torch.bfloat16)
    kc, vc, bt, sl = make_paged(ks, vs, S, 2, gen)
    scale = 1 / math.sqrt(D)
    m, l, acc = oracle_decode.partition_stats(q, kc, vc, bt, sl, scale, P)
    M = m.max(axis=2, keepdims=True)
    w = np.exp(m - M)
    merged = (w[..., None] * acc).sum(2) / (w * l).sum(2)[..., None]
    want = dense_reference(q, ks, vs, scale)
    np.testing.assert_allclose(merged, want, rtol=1e-12, atol=1e-12)
    # each nonempty partition's max term contributes exactly exp(0) = 1 to l
    for i, L in enumerate(lens):
        n = -(-L // P)
        assert np.all(l[i, :, :n] >= 1.0)
        assert np.all(np.isneginf(m[i, :, n:])) and np.all(l[i, :, n:] == 0)
    # the partition max is the max of the dense scores over that range
    for i, L in enumerate(lens):
        s = scale * torch.einsum("hd,lhd->hl", q[i].double(), ks[i].double())
        for p in range(-(-L // P)):
            np.testing.assert_allclose(m[i, :, p], s[:, p * P:(p + 1) * P].max(1).values.numpy(),
                                       rtol=0, atol=1e-13)


def test_append_matches_index_copy(oracle_lib):
    """The scatter equals torch.index_copy_ on the [NB*S, H, D] token view."""
    gen = torch.Generator().manual_seed(11)
    NB, H, S, D, T = 10, 3, 8, 16, 25
    kc = torch.randn(NB, H, S, D, generator=gen).half()
    vc = torch.randn(NB, H, S, D, generator=gen).half()
    k = torch.randn(T, H, D, generator=gen).half()
    v = torch.randn(T, H, D, generator=gen).half()
    slots = torch.randperm(NB * S, generator=gen)[:T].to(torch.int64)
    slots[3] = -1
    slots[17] = -5
    nk, nv = oracle_append.kv_append(k, v, slots, kc, vc)
    keep = slots >= 0
    for cache, new, src in ((kc, nk, k), (vc, nv, v)):
        tok = cache.permute(0, 2, 1, 3).reshape(NB * S, H, D).clone()
        tok.index_copy_(0, slots[keep], src[keep])
        want = tok.reshape(NB, S, H, D).permute(0, 2, 1, 3).contiguous()
        assert np.array_equal(new, want.view(torch.int16).numpy().view(np.uint16))
    # the skipped tokens' values appear nowhere they were not already
    assert np.array_equal(nk.reshape(-1).shape, kc.reshape(-1).shape)


def test_oracle_sensitivity_to_plausible_mistakes(oracle_lib):
    """A wrong scale, a table entry that names another request's block, or an
    off-by-one length all move the result well beyond the parity tolerance, so
    the pins above would catch such a mistake in the oracle. (Swapping two full
    blocks of one request would not: attention without positions is invariant
    under any reordering of its tokens.)"""
    gen = torch.Generator().manual_seed(12)
    H, D, S = 2, 64, 16
    lens = [40, 70]
    ks = [torch.randn(L, H, D, generator=gen).half() for L in lens]
    vs = [torch.randn(L, H, D, generator=gen).half() for L in lens]
    q = torch.randn(2, H, D, generator=gen).half()
    kc, vc, bt, sl = make_paged(ks, vs, S, 0, gen)
    want = dense_reference(q, ks, vs, 0.125)
    base = oracle_decode.paged_decode(q, kc, vc, bt, sl, 0.125)
    assert np.abs(base - want).max() < 1e-12
    assert np.abs(oracle_decode.paged_decode(q, kc, vc, bt, sl, 0.125 * 1.1) - want).max() > 4e-3
    bt2 = bt.clone()
    bt2[1, 0] = bt[0, 0]
    assert np.abs(oracle_decode.paged_decode(q, kc, vc, bt2, sl, 0.125) - want).max() > 4e-3
    sl2 = sl.clone()
    sl2[0] -= 1
    assert np.abs(oracle_decode.paged_decode(q, kc, vc, bt, sl2, 0.125) - want).max() > 4e-3


@pytest.mark.parametrize("G", [2, 4, 8])
def test_grouped_query_heads_equal_sdpa_with_gqa(oracle_lib, G):
    """Grouped-query attention (query head h reads KV head h // G; not on the
    pages): equal to torch SDPA with enable_gqa on the contiguous K/V, and to
    the one-KV-head-per-query-head oracle on a cache with every KV head
    repeated G times."""
    gen = torch.Generator().manual_seed(G)
    Hkv, D, S = 2, 64, 16
    H = Hkv * G
    lens = [1, 17, 40, 130]
    ks = [torch.randn(L, Hkv, D, generator=gen).to(torch.bfloat16) for L in lens]
    vs = [torch.randn(L, Hkv, D, generator=gen).to(torch.bfloat16) for L in lens]
    q = torch.randn(len(lens), H, D, generator=gen).to(torch.bfloat16)
    kc, vc, bt, sl = make_paged(ks, vs, S, 3, gen)
    got = oracle_decode.paged_decode(q, kc, vc, bt, sl, 0.125)
    for i in range(len(lens)):
        want = F.scaled_dot_product_attention(
            q[i].double().unsqueeze(1), ks[i].double().transpose(0, 1),
            vs[i].double().transpose(0, 1), scale=0.125, enable_gqa=True).squeeze(1)
        np.testing.assert_allclose(got[i], want.numpy(), rtol=1e-12, atol=1e-12)
    rep = oracle_decode.paged_decode(q, kc.repeat_interleave(G, dim=1),
                                     vc.repeat_interleave(G, dim=1), bt, sl, 0.125)
    assert np.array_equal(got, rep)


@pytest.mark.parametrize("ctx", [0, 5, 37])
def test_prefill_equals_causal_sdpa(oracle_lib, ctx):
    """Causal prefill over the paged cache ("vLLM KV Cache and PagedAttention
    Explained", Step 6 "Prefill"): equal to torch SDPA with a causal mask shifted
    by the context already cached; its last row equals the decode of that
    request."""
    gen = torch.Generator().manual_seed(ctx + 1)
    H, D, S = 2, 32, 8
    news = [1, 9, 30]
    lens = [ctx + n for n in news]
    ks = [torch.randn(L, H, D, generator=gen).to(torch.bfloat16) for L in lens]
    vs = [torch.randn(L, H, D, generator=gen).to(torch.bfloat16) for L in lens]
    kc, vc, bt, sl = make_paged(ks, vs, S, 2, gen)
    q = torch.randn(sum(news), H, D, generator=gen).to(torch.bfloat16)
    q_start = torch.tensor([0] + list(np.cumsum(news)), dtype=torch.int32)
    got = oracle_decode.paged_prefill(q, kc, vc, bt, sl, q_start, 0.2)
    for i, (L, n) in enumerate(zip(lens, news)):
        qi = q[q_start[i]:q_start[i + 1]].double().transpose(0, 1)       # [H, n, D]
        ki, vi = ks[i].double().transpose(0, 1), vs[i].double().transpose(0, 1)
        pos = torch.arange(L - n, L).unsqueeze(1)
        mask = torch.arange(L).unsqueeze(0) <= pos                         # [n, L]
        want = F.scaled_dot_product_attention(qi, ki, vi, attn_mask=mask, scale=0.2)
        np.testing.assert_allclose(got[q_start[i]:q_start[i + 1]], want.transpose(0, 1).numpy(),
                                   rtol=1e-12, atol=1e-12)
    last = torch.stack([q[q_start[i + 1] - 1] for i in range(len(news))])
    dec = oracle_decode.paged_decode(last, kc, vc, bt, sl, 0.2)
    for i in range(len(news)):
        assert np.array_equal(got[q_start[i + 1] - 1], dec[i])


def test_prefill_grouped_heads_equal_sdpa_gqa(oracle_lib):
    """Grouped KV heads in prefill: query head h reads KV head h // G; equal to
    torch SDPA with enable_gqa and the shifted causal mask."""
    gen = torch.Generator().manual_seed(11)
    H, Hkv, D, S = 6, 2, 16, 4
    ctx, news = [3, 0], [7, 10]
    lens = [c + n for c, n in zip(ctx, news)]
    ks = [torch.randn(L, Hkv, D, generator=gen).to(torch.float16) for L in lens]
    vs = [torch.randn(L, Hkv, D, generator=gen).to(torch.float16) for L in lens]
    kc, vc, bt, sl = make_paged(ks, vs, S, 3, gen)
    q = torch.randn(sum(news), H, D, generator=gen).to(torch.float16)
    q_start = torch.tensor([0, news[0], sum(news)], dtype=torch.int32)
    got = oracle_decode.paged_prefill(q, kc, vc, bt, sl, q_start, 0.3)
    for i, (L, n) in enumerate(zip(lens, news)):
        qi = q[q_start[i]:q_start[i + 1]].double().transpose(0, 1)
        ki, vi = ks[i].double().transpose(0, 1), vs[i].double().transpose(0, 1)
        mask = torch.arange(L).unsqueeze(0) <= torch.arange(L - n, L).unsqueeze(1)
        want = F.scaled_dot_product_attention(qi, ki, vi, attn_mask=mask, scale=0.3,
                                              enable_gqa=True)
        np.testing.assert_allclose(got[q_start[i]:q_start[i + 1]], want.transpose(0, 1).numpy(),
                                   rtol=1e-12, atol=1e-12)
