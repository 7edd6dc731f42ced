"""Memory-waste arithmetic of static reservation versus paged allocation.

Test infrastructure only. Follows "vLLM KV Cache and PagedAttention Explained",
6단계 (LLaMA-2-13B on an A100 40GB, max_model_len 2048, requests of 6/50/8/100
tokens) and Step 5 "Why Waste Stays Below 4%" (waste lives only in each request's
last block, at most block_size - 1 slots).
"""


def kv_bytes_per_token(layers, hidden, bytes_per_elem=2):
    """K and V for every layer: 2 * layers * hidden * bytes."""
    return 2 * layers * hidden * bytes_per_elem


def static_reservation(seq_lens, max_model_len, bytes_per_token):
    """(reserved bytes, used bytes, wasted bytes) when each request holds max_model_len tokens."""
    reserved = len(seq_lens) * max_model_len * bytes_per_token
    used = sum(seq_lens) * bytes_per_token
    return reserved, used, reserved - used


def paged_allocation(seq_lens, block_size):
    """(blocks per request, empty tail slots per request) under on-demand blocks."""
    blocks = [-(-n // block_size) for n in seq_lens]
    waste = [b * block_size - n for b, n in zip(blocks, seq_lens)]
    return blocks, waste
