// Kernels of grouped-query decode (pa_decode_gqa and pa_decode_gqa_fp8 with
// H > Hkv): the tensor-core partition pass over 16-bit or E4M3 caches, and
// its launchers (the split-KV merge is splitkv_reduce_kernel).

#include <climits>
#include <type_traits>

#include "pa_gqa.cuh"
#include "pa_launch.h"

namespace pa {
namespace host {
namespace {

// One CTA per (partition, KV head, request, chunk of up to 16 query heads).
// TC: the cache element type (T, or E4M3 codes).
template <typename T, typename TO, int D, int S, bool APPEND, int NHT, typename TC = T>
pa_status launch(const DecodeParams& prm, cudaStream_t stream) {
  using Tg = GqaTiling<D, sizeof(TC)>;
  auto kern = paged_decode_gqa_kernel<T, TO, D, S, APPEND, NHT, TC>;
  static bool configured[kMaxDevices] = {};
  if (!opt_in_smem(kern, Tg::SMEM, configured)) return PA_ERR_CUDA;
  const int64_t rows = static_cast<int64_t>(prm.NB) * prm.Hkv * S;
  if (rows <= 0 || rows > INT_MAX) return PA_ERR_INVALID;  // TMA row coordinates are int32
  CUtensorMap tmk, tmv;
  if constexpr (sizeof(TC) == 1) {
    if (!row_map_codes(&tmk, prm.k_cache, rows, D, S < 16 ? S : 16) ||
        !row_map_codes(&tmv, prm.v_cache, rows, D, S < 16 ? S : 16))
      return PA_ERR_CUDA;
  } else {
    const pa_dtype dt = std::is_same<T, __half>::value ? PA_F16 : PA_BF16;
    if (!row_map(&tmk, prm.k_cache, rows, D, S < 16 ? S : 16, dt) ||
        !row_map(&tmv, prm.v_cache, rows, D, S < 16 ? S : 16, dt))
      return PA_ERR_CUDA;
  }
  const int G = prm.H / prm.Hkv;
  const dim3 grid(prm.NP, prm.Hkv * ((G + 15) / 16), prm.B);
  kern<<<grid, (Tg::NC + 1) * 32, Tg::SMEM, stream>>>(prm, tmk, tmv);
  if (launch_splitkv_reduce<TO, D>(prm, stream) != cudaSuccess) return PA_ERR_CUDA;
  return cuda_status();
}

template <typename T, typename TO, bool APPEND, typename TC = T>
pa_status by_shape(const DecodeParams& prm, int D, int S, cudaStream_t st) {
  const bool wide = prm.H / prm.Hkv > 8;  // two 8-head column tiles per CTA
#define PA_CASE(DD, SS)                                                         \
  if (D == DD && S == SS)                                                       \
    return wide ? launch<T, TO, DD, SS, APPEND, 2, TC>(prm, st)                 \
                : launch<T, TO, DD, SS, APPEND, 1, TC>(prm, st);
  PA_CASE(64, 8) PA_CASE(64, 16) PA_CASE(64, 32)
  PA_CASE(128, 8) PA_CASE(128, 16) PA_CASE(128, 32)
  PA_CASE(256, 8) PA_CASE(256, 16) PA_CASE(256, 32)
#undef PA_CASE
  return PA_ERR_INVALID;
}

template <typename T, bool APPEND, typename TC = T>
pa_status by_out(const DecodeParams& prm, pa_dtype out_dt, int D, int S, cudaStream_t st) {
  switch (out_dt) {
    case PA_F32: return by_shape<T, float, APPEND, TC>(prm, D, S, st);
    case PA_F16: return by_shape<T, __half, APPEND, TC>(prm, D, S, st);
    case PA_BF16: return by_shape<T, __nv_bfloat16, APPEND, TC>(prm, D, S, st);
  }
  return PA_ERR_INVALID;
}

}  // namespace

pa_status launch_grouped(const DecodeParams& prm, pa_dtype dt, pa_dtype out_dt, int D, int S,
                         bool append, cudaStream_t stream) {
  if (append)
    return dt == PA_F16 ? by_out<__half, true>(prm, out_dt, D, S, stream)
                        : by_out<__nv_bfloat16, true>(prm, out_dt, D, S, stream);
  return dt == PA_F16 ? by_out<__half, false>(prm, out_dt, D, S, stream)
                      : by_out<__nv_bfloat16, false>(prm, out_dt, D, S, stream);
}

pa_status launch_grouped_fp8(const DecodeParams& prm, pa_dtype q_dt, pa_dtype out_dt, int D,
                             int S, cudaStream_t stream) {
  return q_dt == PA_F16 ? by_out<__half, false, __nv_fp8_e4m3>(prm, out_dt, D, S, stream)
                        : by_out<__nv_bfloat16, false, __nv_fp8_e4m3>(prm, out_dt, D, S, stream);
}

bool take_error_grouped(unsigned int* bits) { return take_error_word(bits); }

}  // namespace host
}  // namespace pa
