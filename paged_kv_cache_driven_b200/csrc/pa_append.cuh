// KV append: the slot_mapping scatter of new tokens' K/V into the paged cache.
//
// "vLLM KV Cache and PagedAttention Explained", Step 6 "Decode" and Step 7
// item 5 (the new token's K/V is stored in slot 6 of block 42) and Step 6
// "Prefill" (K1..K6 / V1..V6 written to the cache); the layout is the
// [Block, Head, Block_Size, Head_D] tensor of "vLLM의 PagedAttention 아키텍처와
// GPU 메모리 최적화 원리", section 4.
//
// A pure copy, bound by HBM: each thread moves one 16-byte vector of K and the
// same vector of V. Consecutive threads take consecutive vectors of a token's
// [H, D] rows, so reads of k / v are fully coalesced and each destination row
// (D * 2 bytes, contiguous in the cache) is written by D / 8 adjacent threads.
#pragma once

#include "pa_device.cuh"

namespace pa {

__global__ void __launch_bounds__(256)
    kv_append_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                     const int64_t* __restrict__ slots, uint4* __restrict__ k_cache,
                     uint4* __restrict__ v_cache, int64_t total, int H, int vpr, int S,
                     int64_t n_slots) {
  const int64_t per_token = static_cast<int64_t>(H) * vpr;
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = idx / per_token;
    const int64_t rem = idx - t * per_token;
    const int64_t h = rem / vpr;
    const int64_t c = rem - h * vpr;
    const int64_t slot = __ldg(slots + t);
    if (slot < 0) continue;  // padding
    if (slot >= n_slots) {
      raise_error(PA_DEVERR_SLOT);
      continue;
    }
    const int64_t blk = slot / S;
    const int64_t off = slot - blk * S;
    const int64_t dst = ((blk * H + h) * S + off) * vpr + c;
    const uint4 kv = __ldcs(k + idx);  // read once: streaming
    const uint4 vv = __ldcs(v + idx);
    k_cache[dst] = kv;
    v_cache[dst] = vv;
  }
}

}  // namespace pa
