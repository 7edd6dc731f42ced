// Internal interface of the library (not installed, not part of the C ABI):
// the kernel parameter blocks, and the host-side launchers that each
// translation unit holding kernels exports to the C-ABI layer (pa_api.cu).
// Kernels are split over several translation units (decode, grouped-query
// decode, FP8 decode, prefill, append) so they compile in parallel; each unit
// has its own device error word, which pa_get_device_error() gathers.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "pagedattn.h"

namespace pa {

struct DecodeParams {
  void* out;                   // [B, H, D] final output (dtype TO)
  const void* q;               // [B, H, D]
  const void* k_cache;         // [NB, H, S, D]
  const void* v_cache;         // [NB, H, S, D]
  const int32_t* block_tables; // [B, MB]
  const int32_t* seq_lens;     // [B]
  float* ws_m;                 // [B, H, NP]
  float* ws_l;                 // [B, H, NP]
  float* ws_acc;               // [B, H, NP, D]
  const void* k_new;           // [B, H, D] fused append: the new token's K (or null)
  const void* v_new;           // [B, H, D] fused append: the new token's V (or null)
  float q_scale;               // scale * log2(e)
  int MB, B, H, NB;
  int Hkv;   // KV heads in the cache; query head h reads KV head h / (H / Hkv)
  int P;     // tokens per partition (multiple of S)
  int NP;    // partitions in the grid
  int L_cap; // lengths are clamped to this (MB*S, or NP*P when split)
  float v_scale;  // V = v_scale * stored value (1 for 16-bit caches; E4M3 caches)
};

// The parameters of the FP8 fused append (pa_decode_append_fp8): K's
// per-tensor scale, which the quantizer divides by (q_scale holds it folded
// with the softmax scale). A type of its own, so that the other kernels'
// parameter block stays as it is.
struct DecodeParamsQ8 : DecodeParams {
  float k_scale;
};

struct PrefillParams {
  void* out;                    // [T, H, D] TO
  const void* k_cache;          // [NB, Hkv, S, D] T
  const void* v_cache;
  const int32_t* block_tables;  // [B, MB]
  const int32_t* seq_lens;      // [B] tokens in the cache, new ones included
  const int32_t* q_start;       // [B + 1] first query row of each request
  float scale_log2;             // scale * log2(e)
  int MB, B, H, Hkv, NB, T, max_q_len;
};

namespace host {

constexpr int kMaxDevices = 64;

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

inline pa_status cuda_status() { return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA; }

// The shared-memory opt-in is a per-device property of a kernel function.
template <typename K>
bool opt_in_smem(K kern, int bytes, bool (&configured)[kMaxDevices]) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return false;
  if (!configured[dev]) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
        cudaSuccess)
      return false;
    configured[dev] = true;
  }
  return true;
}

// Tensor maps (pa_api.cu). row_map: a cache [NB, Hkv, S, D] of 16-bit elements
// as a 2-D array of NB * Hkv * S rows of D elements, boxes of 64 elements x
// box_rows rows, 128-byte swizzle (the last few maps are cached). query_map: the
// packed queries [T, H, D] as (D, H, T), boxes of 64 elements x 1 head x 128 rows.
bool row_map(CUtensorMap* out, const void* base, int64_t rows, int D, int box_rows, pa_dtype dt);
// row_map_codes: the same view of a cache of one-byte E4M3 codes; a box is one
// whole D-byte row x box_rows rows, unswizzled.
bool row_map_codes(CUtensorMap* out, const void* base, int64_t rows, int D, int box_rows);
bool query_map(CUtensorMap* out, const void* q, int64_t T, int H, int D, pa_dtype dt);

// Launchers (asynchronous on `stream`; the arguments are already checked).
// cluster: launch the partition pass in clusters of prm.NP CTAs (NP of 2, 4
// or 8) that merge a split among themselves, instead of the merge kernel.
// wide: the grid (B * H * NP CTAs) holds at most four CTAs per SM, so the
// partition pass takes its wide CTA shapes (DecodeTiling, WIDE); a cluster
// launch (at most two CTAs per SM) always does.
pa_status launch_decode16(const DecodeParams& prm, pa_dtype dt, pa_dtype out_dt, int D, int S,
                          bool append, bool cluster, bool wide,
                          cudaStream_t stream);                        // pa_k_decode.cu
pa_status launch_grouped(const DecodeParams& prm, pa_dtype dt, pa_dtype out_dt, int D, int S,
                         bool append, cudaStream_t stream);             // pa_k_gqa.cu
// grouped-query heads over E4M3 caches (q_dt: the queries' 16-bit type)
pa_status launch_grouped_fp8(const DecodeParams& prm, pa_dtype q_dt, pa_dtype out_dt, int D,
                             int S, cudaStream_t stream);               // pa_k_gqa.cu
// append: the new tokens' rows (prm.k_new / v_new, dtype q_dt) are quantized
// with k_scale and prm.v_scale and written into the caches inside the launch.
pa_status launch_decode_fp8(const DecodeParams& prm, pa_dtype q_dt, pa_dtype out_dt, int D,
                            int S, bool cluster, bool wide, bool append, float k_scale,
                            cudaStream_t stream);                       // pa_k_fp8.cu
pa_status launch_prefill(const PrefillParams& prm, const void* q, pa_dtype dt, pa_dtype out_dt,
                         int D, int S, cudaStream_t stream);            // pa_k_prefill.cu
pa_status launch_kv_append(const void* k, const void* v, const int64_t* slots, void* k_cache,
                           void* v_cache, int T, int H, int D, int S, int NB,
                           cudaStream_t stream);                        // pa_k_append.cu
pa_status launch_kv_append_fp8(const void* k, const void* v, pa_dtype in_dt,
                               const int64_t* slots, void* k_cache, void* v_cache, float k_scale,
                               float v_scale, int T, int H, int D, int S, int NB,
                               cudaStream_t stream);
pa_status launch_copy_blocks(void* k_cache, void* v_cache, const int32_t* src_dst, int n, int H,
                             int S, int D, int NB, cudaStream_t stream);

// Each unit's device error word, read and cleared (ORed into *bits).
bool take_error_decode16(unsigned int* bits);
bool take_error_grouped(unsigned int* bits);
bool take_error_fp8(unsigned int* bits);
bool take_error_prefill(unsigned int* bits);
bool take_error_append(unsigned int* bits);

}  // namespace host
}  // namespace pa
