// Kernels of pa_decode_fp8 and pa_decode_append_fp8: the partition pass over
// E4M3 caches (one-byte cache elements, per-tensor scales; with or without the
// quantized fused append, plain or in clusters) and the split-KV merge, with
// their launcher.

#include <type_traits>

#include "pa_decode.cuh"
#include "pa_launch.h"

namespace pa {
namespace host {
namespace {

// One CTA per (partition, head, request). Prm: DecodeParams, or DecodeParamsQ8
// for the fused append (APPEND).
// wide: the grid holds at most two CTAs per SM (DecodeTiling's WIDE shapes;
// cluster launches always are).
template <typename T, typename TO, int D, int S, bool APPEND, typename Prm>
pa_status launch(const Prm& prm, bool cluster, bool wide, cudaStream_t stream) {
  using Tn = DecodeTiling<D, S, 1, false>;
  using Tw = DecodeTiling<D, S, 1, true>;
  constexpr bool two = Tn::NW != Tw::NW;  // otherwise one plain kernel serves both
  using E = __nv_fp8_e4m3;
  auto kern_n = paged_decode_partition_kernel<T, TO, D, S, APPEND, E, false, Prm>;
  auto kern_w = paged_decode_partition_kernel<T, TO, D, S, APPEND, E, false, Prm, two>;
  auto kern_cl = paged_decode_partition_kernel<T, TO, D, S, APPEND, E, true, Prm>;
  static bool conf_n[kMaxDevices] = {}, conf_w[kMaxDevices] = {}, conf_cl[kMaxDevices] = {};
  const bool w = wide && two;
  if (!(w ? opt_in_smem(kern_w, Tw::SMEM, conf_w) : opt_in_smem(kern_n, Tn::SMEM, conf_n)) ||
      !opt_in_smem(kern_cl, Tw::SMEM_CL, conf_cl))
    return PA_ERR_CUDA;
  if (launch_partition_pass<TO, D>(w ? kern_w : kern_n, kern_cl, cluster, prm,
                                   (w ? Tw::NW : Tn::NW) * 32, w ? Tw::SMEM : Tn::SMEM,
                                   Tw::NW * 32, Tw::SMEM_CL, stream) != cudaSuccess)
    return PA_ERR_CUDA;
  return cuda_status();
}

template <typename T, typename TO, bool APPEND, typename Prm>
pa_status by_shape(const Prm& prm, int D, int S, bool cl, bool wide, cudaStream_t st) {
#define PA_CASE(DD, SS) \
  if (D == DD && S == SS) return launch<T, TO, DD, SS, APPEND>(prm, cl, wide, st);
  PA_CASE(64, 8) PA_CASE(64, 16) PA_CASE(64, 32)
  PA_CASE(128, 8) PA_CASE(128, 16) PA_CASE(128, 32)
  PA_CASE(256, 8) PA_CASE(256, 16) PA_CASE(256, 32)
#undef PA_CASE
  return PA_ERR_INVALID;
}

template <typename T, bool APPEND, typename Prm>
pa_status by_out(const Prm& prm, pa_dtype out_dt, int D, int S, bool cl, bool wide,
                 cudaStream_t st) {
  switch (out_dt) {
    case PA_F32: return by_shape<T, float, APPEND>(prm, D, S, cl, wide, st);
    case PA_F16: return by_shape<T, __half, APPEND>(prm, D, S, cl, wide, st);
    case PA_BF16: return by_shape<T, __nv_bfloat16, APPEND>(prm, D, S, cl, wide, st);
  }
  return PA_ERR_INVALID;
}

template <bool APPEND, typename Prm>
pa_status by_q(const Prm& prm, pa_dtype q_dt, pa_dtype out_dt, int D, int S, bool cl,
               bool wide, cudaStream_t st) {
  return q_dt == PA_F16 ? by_out<__half, APPEND>(prm, out_dt, D, S, cl, wide, st)
                        : by_out<__nv_bfloat16, APPEND>(prm, out_dt, D, S, cl, wide, st);
}

}  // namespace

pa_status launch_decode_fp8(const DecodeParams& prm, pa_dtype q_dt, pa_dtype out_dt, int D,
                            int S, bool cluster, bool wide, bool append, float k_scale,
                            cudaStream_t stream) {
  if (!append) return by_q<false>(prm, q_dt, out_dt, D, S, cluster, wide, stream);
  DecodeParamsQ8 q8;
  static_cast<DecodeParams&>(q8) = prm;
  q8.k_scale = k_scale;
  return by_q<true>(q8, q_dt, out_dt, D, S, cluster, wide, stream);
}

bool take_error_fp8(unsigned int* bits) { return take_error_word(bits); }

}  // namespace host
}  // namespace pa
