"""Pins of the oracle's FP8 E4M3 cache format (not on the pages; a storage
extension): the decode table against torch's float8_e4m3fn for all 256 codes,
the quantizer against torch's conversion wherever torch defines it plus the
saturation and tie rules of the format, and decode over an FP8 cache against
torch SDPA on the dequantized K/V."""

import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import fp8 as ofp8

pytestmark = pytest.mark.skipif(not hasattr(torch, "float8_e4m3fn"), reason="torch fp8 dtype")


def test_decode_table_matches_torch():
    codes = torch.arange(256, dtype=torch.uint8)
    want = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = ofp8.decode_table()
    assert np.array_equal(np.isnan(got), np.isnan(want))
    ok = ~np.isnan(want)
    assert np.array_equal(got[ok], want[ok])
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and got[0x08] == 2.0 ** -6
    assert np.isnan(got[0x7F]) and np.isnan(got[0xFF])


def test_quantize_matches_torch_in_range():
    g = torch.Generator().manual_seed(0)
    x = torch.cat([torch.randn(20000, generator=g, dtype=torch.float32) * s
                   for s in (1e-3, 0.1, 1.0, 30.0, 200.0)])
    x = x[x.abs() <= 448]
    want = x.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = ofp8.quantize(x.numpy(), 1.0)
    assert np.array_equal(got, want)


def test_quantize_rules():
    table = ofp8.decode_table()
    # saturation at 448 (the largest finite code 0x7E), both signs
    assert ofp8.quantize(np.array([449.0, 1e6, -1e6]), 1.0).tolist() == [0x7E, 0x7E, 0xFE]
    # exact grid points map to themselves (finite codes of both signs)
    codes = np.array([c for c in range(256) if not np.isnan(table[c])], dtype=np.uint8)
    assert np.array_equal(ofp8.quantize(table[codes], 1.0), codes)
    # midpoints between neighbours go to the even code
    for c in range(0, 126):
        mid = (table[c] + table[c + 1]) / 2
        q = int(ofp8.quantize(np.array([mid]), 1.0)[0])
        assert q == (c if c % 2 == 0 else c + 1)
    # the scale divides first, in fp32
    assert ofp8.quantize(np.array([3.0]), 2.0)[0] == ofp8.quantize(np.array([1.5]), 1.0)[0]
    x = torch.randn(5000, generator=torch.Generator().manual_seed(3)).to(torch.bfloat16).float()
    want = (x / torch.tensor(0.037)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(ofp8.quantize(x.numpy(), 0.037), want)


@pytest.mark.parametrize("H,Hkv", [(4, 4), (8, 2)])
def test_paged_decode_fp8_equals_sdpa_on_dequantized(H, Hkv):
    g = torch.Generator().manual_seed(H)
    D, S, lens = 32, 8, [1, 13, 40]
    NB = sum(-(-L // S) for L in lens) + 2
    k_scale, v_scale = 0.05, 0.08
    kc = torch.from_numpy(ofp8.quantize(torch.randn(NB, Hkv, S, D, generator=g).numpy(), k_scale))
    vc = torch.from_numpy(ofp8.quantize(torch.randn(NB, Hkv, S, D, generator=g).numpy(), v_scale))
    perm = torch.randperm(NB, generator=g).tolist()
    MB = max(-(-L // S) for L in lens)
    bt = torch.full((len(lens), MB), -1, dtype=torch.int32)
    off = 0
    for i, L in enumerate(lens):
        n = -(-L // S)
        bt[i, :n] = torch.tensor(perm[off:off + n], dtype=torch.int32)
        off += n
    q = torch.randn(len(lens), H, D, generator=g).to(torch.bfloat16)
    scale = 1 / math.sqrt(D)
    got = ofp8.paged_decode_fp8(q, kc, vc, k_scale, v_scale, bt, torch.tensor(lens), scale)
    table = torch.from_numpy(ofp8.decode_table())
    for i, L in enumerate(lens):
        blocks = bt[i, : -(-L // S)].long()
        kd = (table[kc[blocks].long()] * k_scale).permute(1, 0, 2, 3).reshape(Hkv, -1, D)[:, :L]
        vd = (table[vc[blocks].long()] * v_scale).permute(1, 0, 2, 3).reshape(Hkv, -1, D)[:, :L]
        want = F.scaled_dot_product_attention(q[i].double().unsqueeze(1), kd, vd, scale=scale,
                                              enable_gqa=True).squeeze(1)
        np.testing.assert_allclose(got[i], want.numpy(), rtol=1e-12, atol=1e-12)
