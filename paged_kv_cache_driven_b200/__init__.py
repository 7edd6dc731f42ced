"""B200-native (sm_100a) paged KV cache: slot_mapping append, block-table-driven
single-query decode attention with split-KV (16-bit or FP8 E4M3 caches,
grouped-query heads, fused append), causal paged prefill attention on the
tensor cores, copy-on-write block copies, a host block allocator and a host-fed
step executor, all behind the C ABI of ``libpagedattn.so``
(``include/pagedattn.h``).

The Python layer is marshalling only (``binding``); every step of the path runs
in the library. Importing this package does not load the library; the first
call does, and raises if it was never built.
"""

from .binding import (  # noqa: F401
    PA_BF16, PA_DEVERR_BLOCK_ID, PA_DEVERR_SEQ_LEN, PA_DEVERR_SLOT, PA_DEVERR_TIMEOUT,
    PA_ERR_CUDA, PA_ERR_INVALID, PA_ERR_OOM, PA_ERR_OUT_OF_RANGE, PA_F16, PA_F32, PA_OK,
    BlockAllocator, PagedAttnError, lib, pa_decode, pa_decode_append, pa_decode_append_fp8,
    pa_decode_fp8, pa_decode_gqa_fp8,
    pa_decode_gqa, pa_decode_noalloc, pa_decode_plan, pa_decode_plan_grouped,
    pa_decode_workspace_bytes,
    pa_copy_blocks, pa_get_device_error, pa_kv_append, pa_kv_append_fp8, pa_prefill,
)
