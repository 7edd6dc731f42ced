// Kernels that move cache bytes: the slot_mapping append (16-bit and E4M3
// caches) and the copy-on-write block copy, with their launchers. Grids stride
// beyond about 16 CTAs per SM.

#include "pa_append.cuh"
#include "pa_launch.h"

namespace pa {
namespace host {
namespace {

unsigned grid_for(int64_t total) {
  int64_t blocks = ceil_div(total, 256);
  const int64_t cap = 148LL * 16;
  return static_cast<unsigned>(blocks > cap ? cap : blocks);
}

}  // namespace

pa_status launch_kv_append(const void* k, const void* v, const int64_t* slots, void* k_cache,
                           void* v_cache, int T, int H, int D, int S, int NB, cudaStream_t stream) {
  const int vpr = D / 8;  // 16-byte vectors per row
  const int64_t total = static_cast<int64_t>(T) * H * vpr;
  kv_append_kernel<<<grid_for(total), 256, 0, stream>>>(
      static_cast<const uint4*>(k), static_cast<const uint4*>(v), slots,
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), total, H, vpr, S,
      static_cast<int64_t>(NB) * S);
  return cuda_status();
}

pa_status launch_kv_append_fp8(const void* k, const void* v, pa_dtype in_dt, const int64_t* slots,
                               void* k_cache, void* v_cache, float k_scale, float v_scale, int T,
                               int H, int D, int S, int NB, cudaStream_t stream) {
  const int vpr = D / 8;  // 8-element vectors per row
  const int64_t total = static_cast<int64_t>(T) * H * vpr;
  const int64_t n_slots = static_cast<int64_t>(NB) * S;
  if (in_dt == PA_BF16)
    kv_append_fp8_kernel<__nv_bfloat16><<<grid_for(total), 256, 0, stream>>>(
        static_cast<const uint4*>(k), static_cast<const uint4*>(v), slots,
        static_cast<uint2*>(k_cache), static_cast<uint2*>(v_cache), k_scale, v_scale, total, H,
        vpr, S, n_slots);
  else
    kv_append_fp8_kernel<__half><<<grid_for(total), 256, 0, stream>>>(
        static_cast<const uint4*>(k), static_cast<const uint4*>(v), slots,
        static_cast<uint2*>(k_cache), static_cast<uint2*>(v_cache), k_scale, v_scale, total, H,
        vpr, S, n_slots);
  return cuda_status();
}

pa_status launch_copy_blocks(void* k_cache, void* v_cache, const int32_t* src_dst, int n, int H,
                             int S, int D, int NB, cudaStream_t stream) {
  const int64_t vpb = static_cast<int64_t>(H) * S * D / 8;  // 16-byte vectors per block
  const int64_t total = vpb * n;
  copy_blocks_kernel<<<grid_for(total), 256, 0, stream>>>(
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), src_dst, total, vpb, NB);
  return cuda_status();
}

bool take_error_append(unsigned int* bits) { return take_error_word(bits); }

}  // namespace host
}  // namespace pa
