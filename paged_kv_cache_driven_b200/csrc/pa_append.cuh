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

// The same scatter into an FP8 E4M3 cache (a storage extension, not on the
// pages): each element is stored as the E4M3 code of fp32(x / scale) (one
// correctly rounded division, then round to nearest even, saturated at 448),
// K and V with their own per-tensor scale. One thread per 8 elements: a
// 16-byte vector of 16-bit input becomes an 8-byte vector of codes.
template <typename T>
__global__ void __launch_bounds__(256)
    kv_append_fp8_kernel(const uint4* __restrict__ k, const uint4* __restrict__ v,
                         const int64_t* __restrict__ slots, uint2* __restrict__ k_cache,
                         uint2* __restrict__ v_cache, float k_scale, float v_scale, int64_t total,
                         int H, int vpr, int S, int64_t n_slots) {
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
    float kf[8], vf[8];
    convert_frag<T>(__ldcs(k + idx), kf);
    convert_frag<T>(__ldcs(v + idx), vf);
    uint32_t kw[4], vw[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      kw[e] = float2_to_e4m3x2(__fdiv_rn(kf[2 * e], k_scale), __fdiv_rn(kf[2 * e + 1], k_scale));
      vw[e] = float2_to_e4m3x2(__fdiv_rn(vf[2 * e], v_scale), __fdiv_rn(vf[2 * e + 1], v_scale));
    }
    k_cache[dst] = make_uint2(kw[0] | (kw[1] << 16), kw[2] | (kw[3] << 16));
    v_cache[dst] = make_uint2(vw[0] | (vw[1] << 16), vw[2] | (vw[3] << 16));
  }
}

// Copy-on-write, device half ("vLLM KV Cache and PagedAttention Explained",
// Step 9): copies whole physical blocks, every head, of K and V from src to
// dst for each (src, dst) pair. One thread per 16-byte vector; the pairs come
// from the allocator's queue and name distinct destinations.
__global__ void __launch_bounds__(256)
    copy_blocks_kernel(uint4* __restrict__ k_cache, uint4* __restrict__ v_cache,
                       const int32_t* __restrict__ src_dst, int64_t total, int64_t vec_per_block,
                       int NB) {
  for (int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; idx < total;
       idx += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t pair = idx / vec_per_block;
    const int64_t c = idx - pair * vec_per_block;
    const int32_t src = __ldg(src_dst + 2 * pair);
    const int32_t dst = __ldg(src_dst + 2 * pair + 1);
    if (static_cast<unsigned>(src) >= static_cast<unsigned>(NB) ||
        static_cast<unsigned>(dst) >= static_cast<unsigned>(NB)) {
      if (c == 0) raise_error(PA_DEVERR_BLOCK_ID);
      continue;
    }
    const uint4 kv = k_cache[src * vec_per_block + c];
    const uint4 vv = v_cache[src * vec_per_block + c];
    k_cache[dst * vec_per_block + c] = kv;
    v_cache[dst * vec_per_block + c] = vv;
  }
}

}  // namespace pa
