// Kernels of pa_decode / pa_decode_append with one KV head per query head:
// the partition pass (whose CTAs merge a split request among themselves in a
// cluster launch, or leave partials for the merge kernel) and the merge kernel,
// for every cache dtype, output dtype, head size and block size, and their
// launcher.

#include <type_traits>

#include "pa_decode.cuh"
#include "pa_launch.h"

namespace pa {
namespace host {
namespace {

// One CTA per (partition, head, request). wide: the grid holds at most two
// CTAs per SM (DecodeTiling's WIDE shapes; cluster launches always are).
template <typename T, typename TO, int D, int S, bool APPEND>
pa_status launch(const DecodeParams& prm, bool cluster, bool wide, cudaStream_t stream) {
  using Tn = DecodeTiling<D, S, 2, false>;
  using Tw = DecodeTiling<D, S, 2, true>;
  constexpr bool two = Tn::NW != Tw::NW;  // otherwise one plain kernel serves both
  auto kern_n = paged_decode_partition_kernel<T, TO, D, S, APPEND>;
  auto kern_w = paged_decode_partition_kernel<T, TO, D, S, APPEND, T, false, DecodeParams, two>;
  auto kern_cl = paged_decode_partition_kernel<T, TO, D, S, APPEND, T, true>;
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

template <typename T, typename TO, bool APPEND>
pa_status by_shape(const DecodeParams& prm, int D, int S, bool cl, bool wide, cudaStream_t st) {
#define PA_CASE(DD, SS) \
  if (D == DD && S == SS) return launch<T, TO, DD, SS, APPEND>(prm, cl, wide, st);
  PA_CASE(64, 8) PA_CASE(64, 16) PA_CASE(64, 32)
  PA_CASE(128, 8) PA_CASE(128, 16) PA_CASE(128, 32)
  PA_CASE(256, 8) PA_CASE(256, 16) PA_CASE(256, 32)
#undef PA_CASE
  return PA_ERR_INVALID;
}

template <typename T, bool APPEND>
pa_status by_out(const DecodeParams& prm, pa_dtype out_dt, int D, int S, bool cl, bool wide,
                 cudaStream_t st) {
  switch (out_dt) {
    case PA_F32: return by_shape<T, float, APPEND>(prm, D, S, cl, wide, st);
    case PA_F16: return by_shape<T, __half, APPEND>(prm, D, S, cl, wide, st);
    case PA_BF16: return by_shape<T, __nv_bfloat16, APPEND>(prm, D, S, cl, wide, st);
  }
  return PA_ERR_INVALID;
}

}  // namespace

pa_status launch_decode16(const DecodeParams& prm, pa_dtype dt, pa_dtype out_dt, int D, int S,
                          bool append, bool cluster, bool wide, cudaStream_t stream) {
  if (append)
    return dt == PA_F16 ? by_out<__half, true>(prm, out_dt, D, S, cluster, wide, stream)
                        : by_out<__nv_bfloat16, true>(prm, out_dt, D, S, cluster, wide, stream);
  return dt == PA_F16 ? by_out<__half, false>(prm, out_dt, D, S, cluster, wide, stream)
                      : by_out<__nv_bfloat16, false>(prm, out_dt, D, S, cluster, wide, stream);
}

bool take_error_decode16(unsigned int* bits) { return take_error_word(bits); }

}  // namespace host
}  // namespace pa
