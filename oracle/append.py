"""The slot_mapping scatter of new tokens' K/V into the paged cache, in numpy.

Test infrastructure only. Follows "vLLM KV Cache and PagedAttention Explained",
Step 6 "Decode" and Step 7 item 5 (K7/V7 of the new token are stored in slot 6
of block 42) and Step 6 "Prefill" (K1..K6/V1..V6 are written to the cache), in
the [Block, Head, Block_Size, Head_D] layout of "vLLM의 PagedAttention 아키텍처와
GPU 메모리 최적화 원리", section 4. Reading where the pages are silent: a slot is
the integer block * block_size + offset, and a negative slot means "skip this
token" (padding).
"""

import numpy as np
import torch


def _bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def scatter_into(k_bits, v_bits, slots, kc_bits, vc_bits):
    """In-place form on uint16 bit arrays: k_bits, v_bits [T, H, D]; caches [NB, H, S, D]."""
    slots = np.asarray(slots, dtype=np.int64)
    S = kc_bits.shape[2]
    for t in range(slots.shape[0]):
        s = int(slots[t])
        if s < 0:
            continue
        block, offset = divmod(s, S)
        kc_bits[block, :, offset, :] = k_bits[t]
        vc_bits[block, :, offset, :] = v_bits[t]


def kv_append(k, v, slot_mapping, k_cache, v_cache):
    """Returns (k_cache', v_cache') as uint16 bit arrays after the scatter.

    k, v [T, H, D]; slot_mapping [T] int64; caches [NB, H, S, D]. The inputs
    are not modified. Every token with slot >= 0 has its [H, D] rows written to
    block slot // S at offset slot % S for every head; all other cache bytes
    keep their values.
    """
    kc, vc = _bits(k_cache).copy(), _bits(v_cache).copy()
    slots = np.asarray(torch.as_tensor(slot_mapping).to("cpu").numpy(), dtype=np.int64)
    scatter_into(_bits(k), _bits(v), slots, kc, vc)
    return kc, vc


def copy_blocks_into(kc_bits, vc_bits, pairs):
    """Copy-on-write, device half ("vLLM KV Cache and PagedAttention Explained",
    Step 9): physical block dst becomes a bit copy of block src, every head, in
    both caches, for each (src, dst) pair in order. In place on uint16 arrays."""
    for src, dst in pairs:
        kc_bits[dst] = kc_bits[src]
        vc_bits[dst] = vc_bits[src]
