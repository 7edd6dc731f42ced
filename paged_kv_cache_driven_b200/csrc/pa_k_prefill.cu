// Kernels of pa_prefill: causal paged prefill attention on the fifth-generation
// tensor cores, for both 16-bit cache dtypes, every output dtype, head size 64,
// 128 and 256 and block sizes 8 .. 128, and their launcher.

#include <type_traits>

#include "pa_launch.h"
#include "pa_prefill.cuh"

namespace pa {
namespace host {
namespace {

// One CTA per (256 query rows, query head, request). The grid runs the heads
// fastest, then a request's row blocks from the last (the longest, with the
// most keys) to the first, then the requests: a request's longest CTAs of
// every head start first, and its K/V stays in L2 while its heads run (one
// 4096-token prompt on 32 heads: 0.278 -> 0.231 ms against row blocks fastest).
template <typename T, typename TO, int D, int S>
pa_status launch(const PrefillParams& prm, const void* q, cudaStream_t stream) {
  using Tl = PrefillTiling<D, std::is_same<T, __nv_bfloat16>::value>;
  auto kern = paged_prefill_kernel<T, TO, D, S>;
  static bool configured[kMaxDevices] = {};
  if (!opt_in_smem(kern, Tl::SMEM, configured)) return PA_ERR_CUDA;
  const pa_dtype dt = std::is_same<T, __half>::value ? PA_F16 : PA_BF16;
  const int64_t rows = static_cast<int64_t>(prm.NB) * prm.Hkv * S;
  CUtensorMap tmq, tmk, tmv;
  if (!query_map(&tmq, q, prm.T, prm.H, D, dt) || !row_map(&tmk, prm.k_cache, rows, D, S, dt) ||
      !row_map(&tmv, prm.v_cache, rows, D, S, dt))
    return PA_ERR_CUDA;
  const dim3 grid(prm.H, static_cast<unsigned>(ceil_div(prm.max_q_len, Tl::NQT * Tl::BM)), prm.B);
  kern<<<grid, Tl::THREADS, Tl::SMEM, stream>>>(prm, tmq, tmk, tmv);
  return cuda_status();
}

template <typename T, typename TO>
pa_status by_shape(const PrefillParams& prm, const void* q, int D, int S, cudaStream_t st) {
#define PA_CASE(DD, SS) \
  if (D == DD && S == SS) return launch<T, TO, DD, SS>(prm, q, st);
  PA_CASE(64, 8) PA_CASE(64, 16) PA_CASE(64, 32) PA_CASE(64, 64) PA_CASE(64, 128)
  PA_CASE(128, 8) PA_CASE(128, 16) PA_CASE(128, 32) PA_CASE(128, 64) PA_CASE(128, 128)
  PA_CASE(256, 8) PA_CASE(256, 16) PA_CASE(256, 32) PA_CASE(256, 64) PA_CASE(256, 128)
#undef PA_CASE
  return PA_ERR_INVALID;
}

template <typename T>
pa_status by_out(const PrefillParams& prm, const void* q, pa_dtype out_dt, int D, int S,
                 cudaStream_t st) {
  switch (out_dt) {
    case PA_F32: return by_shape<T, float>(prm, q, D, S, st);
    case PA_F16: return by_shape<T, __half>(prm, q, D, S, st);
    case PA_BF16: return by_shape<T, __nv_bfloat16>(prm, q, D, S, st);
  }
  return PA_ERR_INVALID;
}

}  // namespace

pa_status launch_prefill(const PrefillParams& prm, const void* q, pa_dtype dt, pa_dtype out_dt,
                         int D, int S, cudaStream_t stream) {
  return dt == PA_BF16 ? by_out<__nv_bfloat16>(prm, q, out_dt, D, S, stream)
                       : by_out<__half>(prm, q, out_dt, D, S, stream);
}

bool take_error_prefill(unsigned int* bits) { return take_error_word(bits); }

}  // namespace host
}  // namespace pa

#ifdef PA_PREFILL_TRACE
// Trace build only: the stamp buffer g_prefill_trace ([64][32][48] int64, see
// pa_prefill.cuh), copied to host memory `dst` of `bytes` (which must be its
// size), or set to zero. Return 0 on success.
extern "C" int pa_prefill_trace_read(void* dst, size_t bytes) {
  if (!dst || bytes != sizeof(pa::g_prefill_trace)) return 1;
  return cudaMemcpyFromSymbol(dst, pa::g_prefill_trace, bytes) == cudaSuccess ? 0 : 2;
}
extern "C" int pa_prefill_trace_clear(void) {
  void* addr = nullptr;
  if (cudaGetSymbolAddress(&addr, pa::g_prefill_trace) != cudaSuccess) return 2;
  return cudaMemset(addr, 0, sizeof(pa::g_prefill_trace)) == cudaSuccess ? 0 : 2;
}
#endif
