// The device half of the C ABI (pagedattn.h): argument validation, launch
// planning, tensor-map encoding and kernel dispatch for pa_kv_append,
// pa_decode / pa_decode_append / pa_decode_gqa / pa_decode_noalloc,
// pa_prefill and pa_copy_blocks, and the device error word. Every check runs
// on the host before anything is launched.

#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <climits>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>
#include <type_traits>

#include "pa_append.cuh"
#include "pa_decode.cuh"
#include "pa_gqa.cuh"
#include "pa_prefill.cuh"
#include "pagedattn.h"

namespace {

constexpr int kDefaultPartition = 512;  // tokens per split-KV partition when splitting
constexpr int kMaxDevices = 64;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool cache_dtype_ok(pa_dtype dt) { return dt == PA_F16 || dt == PA_BF16; }

bool out_dtype_ok(pa_dtype dt) { return dt == PA_F16 || dt == PA_BF16 || dt == PA_F32; }

bool decode_shape_ok(int D, int S) {
  return (D == 64 || D == 128 || D == 256) && (S == 8 || S == 16 || S == 32);
}

int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }

// SMs of the current device (148 on B200; also the answer without a device).
int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    cudaGetLastError();  // clear the error state of the failed query
    return 148;
  }
  return n;
}

// Chooses the partition length. Returns false on an invalid `partition`.
//   -1      never split: one partition covering any length up to MB * S
//   > 0     that many tokens (a multiple of S)
//   0       automatic: 512-token partitions, halved (down to 64 tokens, staying a
//           multiple of S) while the grid would hold fewer than about four
//           waves of CTAs (three CTAs per SM), so that small batches still
//           spread over every SM; no split if one partition covers every request
bool plan(int B, int H, int S, int max_seq_len, int partition, int* P_out, int* NP_out) {
  if (max_seq_len < 0 || S <= 0) return false;
  int P;
  if (partition < 0) {
    if (partition != -1) return false;
    *P_out = 0;
    *NP_out = 1;
    return true;
  } else if (partition > 0) {
    if (partition % S != 0) return false;
    P = partition;
  } else {
    P = kDefaultPartition;
    const int64_t target = 4LL * 3 * sm_count();
    const int64_t pairs = static_cast<int64_t>(B > 0 ? B : 1) * (H > 0 ? H : 1);
    while (P > 64 && (P / 2) % S == 0 && pairs * ceil_div(max_seq_len, P) < target) P /= 2;
  }
  const int64_t np = ceil_div(max_seq_len, P);
  if (np <= 1) {
    *P_out = 0;
    *NP_out = 1;
    return true;
  }
  if (np * P > INT_MAX) return false;
  *P_out = P;
  *NP_out = static_cast<int>(np);
  return true;
}

size_t workspace_for(int B, int H, int D, int NP) {
  if (NP <= 1) return 0;
  const size_t n = static_cast<size_t>(B) * H * NP;
  return align256(n * 2 * sizeof(float)) + n * D * sizeof(float);
}

pa_status cuda_status() {
  return cudaGetLastError() == cudaSuccess ? PA_OK : PA_ERR_CUDA;
}

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

template <typename TO, int D>
void launch_reduce(const pa::DecodeParams& prm, cudaStream_t stream) {
  if (prm.NP > 1) {
    const int64_t pairs = static_cast<int64_t>(prm.B) * prm.H;
    pa::splitkv_reduce_kernel<TO, D>
        <<<static_cast<unsigned>((pairs + 3) / 4), 128, 0, stream>>>(prm);
  }
}

// One KV head per query head (or an odd group size): the multi-head kernel,
// each CTA reading its query head's KV head.
template <typename T, typename TO, int D, int S, bool APPEND>
pa_status launch_decode(const pa::DecodeParams& prm, cudaStream_t stream) {
  using Tl = pa::DecodeTiling<D, S>;
  auto kern = pa::paged_decode_partition_kernel<T, TO, D, S, APPEND>;
  static bool configured[kMaxDevices] = {};
  if (!opt_in_smem(kern, Tl::SMEM, configured)) return PA_ERR_CUDA;
  const dim3 grid(prm.NP, prm.H, prm.B);
  kern<<<grid, Tl::NW * 32, Tl::SMEM, stream>>>(prm);
  launch_reduce<TO, D>(prm, stream);
  return cuda_status();
}

// ---- tensor maps of the caches, for the tiled TMA loads ---------------------
// Each cache [NB, Hkv, S, D] is viewed as a 2-D array of NB * Hkv * S rows of D
// elements; a box is 64 elements x min(S, 16) rows with the 128-byte swizzle.
// Encoding goes through the driver's cuTensorMapEncodeTiled (looked up once);
// the last few maps are kept, keyed by everything they encode, since a cache is
// decoded over and over.

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

struct RowMapKey {
  const void* base;
  int64_t rows;
  int D, box_rows, dt;
  bool operator==(const RowMapKey& o) const {
    return base == o.base && rows == o.rows && D == o.D && box_rows == o.box_rows && dt == o.dt;
  }
};

bool row_map(CUtensorMap* out, const void* base, int64_t rows, int D, int box_rows, pa_dtype dt) {
  static std::mutex mu;
  static RowMapKey keys[16];
  static CUtensorMap maps[16];
  static int used = 0, next = 0;
  const RowMapKey key{base, rows, D, box_rows, static_cast<int>(dt)};
  std::lock_guard<std::mutex> lock(mu);
  for (int k = 0; k < used; ++k)
    if (keys[k] == key) {
      *out = maps[k];
      return true;
    }
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * 2};
  const cuuint32_t box[2] = {64, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  CUtensorMap map;
  if (fn(&map, dt == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
         2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  const int slot = used < 16 ? used++ : next;
  next = (slot + 1) % 16;
  keys[slot] = key;
  maps[slot] = map;
  *out = map;
  return true;
}

// Grouped query heads: one CTA per (partition, KV head, request, chunk of up to
// 16 query heads), the contraction on the tensor cores.
template <typename T, typename TO, int D, int S, bool APPEND, int NHT>
pa_status launch_grouped(const pa::DecodeParams& prm, cudaStream_t stream) {
  using Tg = pa::GqaTiling<D>;
  auto kern = pa::paged_decode_gqa_kernel<T, TO, D, S, APPEND, NHT>;
  static bool configured[kMaxDevices] = {};
  if (!opt_in_smem(kern, Tg::SMEM, configured)) return PA_ERR_CUDA;
  const int64_t rows = static_cast<int64_t>(prm.NB) * prm.Hkv * S;
  if (rows <= 0 || rows > INT_MAX) return PA_ERR_INVALID;  // TMA row coordinates are int32
  const pa_dtype dt = std::is_same<T, __half>::value ? PA_F16 : PA_BF16;
  CUtensorMap tmk, tmv;
  if (!row_map(&tmk, prm.k_cache, rows, D, S < 16 ? S : 16, dt) ||
      !row_map(&tmv, prm.v_cache, rows, D, S < 16 ? S : 16, dt))
    return PA_ERR_CUDA;
  const int G = prm.H / prm.Hkv;
  const dim3 grid(prm.NP, prm.Hkv * ((G + 15) / 16), prm.B);
  kern<<<grid, (Tg::NC + 1) * 32, Tg::SMEM, stream>>>(prm, tmk, tmv);
  launch_reduce<TO, D>(prm, stream);
  return cuda_status();
}

// E4M3 cache: the multi-head kernel with one-byte cache elements.
template <typename T, typename TO, int D, int S>
pa_status launch_decode_fp8(const pa::DecodeParams& prm, cudaStream_t stream) {
  using Tl = pa::DecodeTiling<D, S, 1>;
  auto kern = pa::paged_decode_partition_kernel<T, TO, D, S, false, __nv_fp8_e4m3>;
  static bool configured[kMaxDevices] = {};
  if (!opt_in_smem(kern, Tl::SMEM, configured)) return PA_ERR_CUDA;
  const dim3 grid(prm.NP, prm.H, prm.B);
  kern<<<grid, Tl::NW * 32, Tl::SMEM, stream>>>(prm);
  launch_reduce<TO, D>(prm, stream);
  return cuda_status();
}

template <typename T, typename TO>
pa_status dispatch_fp8_shape(const pa::DecodeParams& prm, int D, int S, cudaStream_t st) {
#define PA_CASE(DD, SS) \
  if (D == DD && S == SS) return launch_decode_fp8<T, TO, DD, SS>(prm, st);
  PA_CASE(64, 8) PA_CASE(64, 16) PA_CASE(64, 32)
  PA_CASE(128, 8) PA_CASE(128, 16) PA_CASE(128, 32)
  PA_CASE(256, 8) PA_CASE(256, 16) PA_CASE(256, 32)
#undef PA_CASE
  return PA_ERR_INVALID;
}

template <typename T, typename TO, bool APPEND>
pa_status dispatch_shape(const pa::DecodeParams& prm, int D, int S, cudaStream_t st) {
  const bool grouped = prm.H != prm.Hkv;
#define PA_CASE(DD, SS)                                                            \
  if (D == DD && S == SS)                                                          \
    return grouped ? (prm.H / prm.Hkv <= 8 ? launch_grouped<T, TO, DD, SS, APPEND, 1>(prm, st)   \
                                           : launch_grouped<T, TO, DD, SS, APPEND, 2>(prm, st)) \
                   : launch_decode<T, TO, DD, SS, APPEND>(prm, st);
  PA_CASE(64, 8) PA_CASE(64, 16) PA_CASE(64, 32)
  PA_CASE(128, 8) PA_CASE(128, 16) PA_CASE(128, 32)
  PA_CASE(256, 8) PA_CASE(256, 16) PA_CASE(256, 32)
#undef PA_CASE
  return PA_ERR_INVALID;
}

template <typename T, bool APPEND>
pa_status dispatch_out(const pa::DecodeParams& prm, pa_dtype out_dt, int D, int S,
                       cudaStream_t st) {
  switch (out_dt) {
    case PA_F32: return dispatch_shape<T, float, APPEND>(prm, D, S, st);
    case PA_F16: return dispatch_shape<T, __half, APPEND>(prm, D, S, st);
    case PA_BF16: return dispatch_shape<T, __nv_bfloat16, APPEND>(prm, D, S, st);
  }
  return PA_ERR_INVALID;
}

// ---- paged prefill -------------------------------------------------------------
// The packed queries [T, H, D] as a 3-D tensor map (D, H, T) whose box is one
// 64-element column block of one head for 128 consecutive query rows; rows
// past T read as zeros.
bool query_map(CUtensorMap* out, const void* q, int64_t T, int H, int D, pa_dtype dt) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(T)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * 2,
                                 static_cast<cuuint64_t>(H) * D * 2};
  const cuuint32_t box[3] = {64, 1, 128};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(out, dt == PA_BF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16,
            3, const_cast<void*>(q), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename T, typename TO, int D, int S>
pa_status launch_prefill(const pa::PrefillParams& prm, const void* q, cudaStream_t stream) {
  using Tl = pa::PrefillTiling<D, std::is_same<T, __nv_bfloat16>::value>;
  auto kern = pa::paged_prefill_kernel<T, TO, D, S>;
  static bool configured[kMaxDevices] = {};
  if (!opt_in_smem(kern, Tl::SMEM, configured)) return PA_ERR_CUDA;
  const pa_dtype dt = std::is_same<T, __half>::value ? PA_F16 : PA_BF16;
  const int64_t rows = static_cast<int64_t>(prm.NB) * prm.Hkv * S;
  CUtensorMap tmq, tmk, tmv;
  if (!query_map(&tmq, q, prm.T, prm.H, D, dt) || !row_map(&tmk, prm.k_cache, rows, D, S, dt) ||
      !row_map(&tmv, prm.v_cache, rows, D, S, dt))
    return PA_ERR_CUDA;
  const dim3 grid(static_cast<unsigned>(ceil_div(prm.max_q_len, Tl::NQT * Tl::BM)), prm.H, prm.B);
  kern<<<grid, Tl::THREADS, Tl::SMEM, stream>>>(prm, tmq, tmk, tmv);
  return cuda_status();
}

template <typename T, typename TO>
pa_status dispatch_prefill_shape(const pa::PrefillParams& prm, const void* q, int D, int S,
                                 cudaStream_t st) {
#define PA_CASE(DD, SS) \
  if (D == DD && S == SS) return launch_prefill<T, TO, DD, SS>(prm, q, st);
  PA_CASE(64, 8) PA_CASE(64, 16) PA_CASE(64, 32) PA_CASE(64, 64) PA_CASE(64, 128)
  PA_CASE(128, 8) PA_CASE(128, 16) PA_CASE(128, 32) PA_CASE(128, 64) PA_CASE(128, 128)
#undef PA_CASE
  return PA_ERR_INVALID;
}

template <typename T>
pa_status dispatch_prefill(const pa::PrefillParams& prm, const void* q, pa_dtype out_dt, int D,
                           int S, cudaStream_t st) {
  switch (out_dt) {
    case PA_F32: return dispatch_prefill_shape<T, float>(prm, q, D, S, st);
    case PA_F16: return dispatch_prefill_shape<T, __half>(prm, q, D, S, st);
    case PA_BF16: return dispatch_prefill_shape<T, __nv_bfloat16>(prm, q, D, S, st);
  }
  return PA_ERR_INVALID;
}

}  // namespace

extern "C" {

const char* pa_status_string(pa_status s) {
  switch (s) {
    case PA_OK: return "PA_OK";
    case PA_ERR_INVALID: return "PA_ERR_INVALID";
    case PA_ERR_OOM: return "PA_ERR_OOM";
    case PA_ERR_OUT_OF_RANGE: return "PA_ERR_OUT_OF_RANGE";
    case PA_ERR_CUDA: return "PA_ERR_CUDA";
  }
  return "PA_ERR_UNKNOWN";
}

int pa_version(void) { return 100; }

pa_status pa_kv_append(const void* k, const void* v, const int64_t* slot_mapping, void* k_cache,
                       void* v_cache, int T, int H, int D, int S, int NB, pa_dtype dt,
                       void* stream) {
  if (T < 0 || H <= 0 || D <= 0 || S <= 0 || NB < 0 || !cache_dtype_ok(dt)) return PA_ERR_INVALID;
  if (D % 8 != 0) return PA_ERR_INVALID;  // rows move as 16-byte vectors
  if (T == 0) return PA_OK;
  if (!k || !v || !slot_mapping || !k_cache || !v_cache) return PA_ERR_INVALID;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID;
  const int vpr = D / 8;
  const int64_t total = static_cast<int64_t>(T) * H * vpr;
  const int64_t n_slots = static_cast<int64_t>(NB) * S;
  int64_t blocks = ceil_div(total, 256);
  const int64_t cap = 148LL * 16;  // grid-stride beyond ~16 CTAs per SM
  if (blocks > cap) blocks = cap;
  pa::kv_append_kernel<<<static_cast<unsigned>(blocks), 256, 0,
                         static_cast<cudaStream_t>(stream)>>>(
      static_cast<const uint4*>(k), static_cast<const uint4*>(v), slot_mapping,
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), total, H, vpr, S, n_slots);
  return cuda_status();
}

pa_status pa_copy_blocks(void* k_cache, void* v_cache, const int32_t* src_dst, int n, int H,
                         int S, int D, int NB, pa_dtype dt, void* stream) {
  if (n < 0 || H <= 0 || S <= 0 || D <= 0 || NB < 0 || !cache_dtype_ok(dt) || D % 8 != 0)
    return PA_ERR_INVALID;
  if (n == 0) return PA_OK;
  if (!k_cache || !v_cache || !src_dst || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID;
  const int64_t vpb = static_cast<int64_t>(H) * S * D / 8;  // 16-byte vectors per block
  const int64_t total = vpb * n;
  int64_t blocks = ceil_div(total, 256);
  if (blocks > 148LL * 16) blocks = 148LL * 16;
  pa::copy_blocks_kernel<<<static_cast<unsigned>(blocks), 256, 0,
                           static_cast<cudaStream_t>(stream)>>>(
      static_cast<uint4*>(k_cache), static_cast<uint4*>(v_cache), src_dst, total, vpb, NB);
  return cuda_status();
}

pa_status pa_decode_plan(int B, int H, int D, int S, int max_seq_len, int partition,
                         int* partition_tokens, int* num_partitions) {
  (void)B;
  (void)H;
  (void)D;
  if (!partition_tokens || !num_partitions) return PA_ERR_INVALID;
  int P, NP;
  if (!plan(B, H, S, max_seq_len, partition, &P, &NP)) return PA_ERR_INVALID;
  *partition_tokens = P;
  *num_partitions = NP;
  return PA_OK;
}

size_t pa_decode_workspace_bytes(int B, int H, int D, int S, int max_seq_len, int partition) {
  int P, NP;
  if (B < 0 || H <= 0 || D <= 0 || !plan(B, H, S, max_seq_len, partition, &P, &NP)) return 0;
  return workspace_for(B, H, D, NP);
}

}  // extern "C"

namespace {

// pa_decode and pa_decode_append: k_new / v_new null = plain decode.
pa_status decode_impl(void* out, pa_dtype out_dt, const void* q, const void* k_new,
                      const void* v_new, const void* k_cache, const void* v_cache,
                      const int32_t* block_tables, int MB, const int32_t* seq_lens, float scale,
                      int B, int H, int Hkv, int D, int S, int NB, pa_dtype dt, int partition,
                      int max_seq_len, void* workspace, size_t ws_bytes, void* stream) {
  if (B < 0 || H <= 0 || NB < 0 || MB < 0) return PA_ERR_INVALID;
  if (Hkv <= 0 || H % Hkv != 0) return PA_ERR_INVALID;
  if (!cache_dtype_ok(dt) || !out_dtype_ok(out_dt) || !decode_shape_ok(D, S)) return PA_ERR_INVALID;
  if (!std::isfinite(scale)) return PA_ERR_INVALID;
  if (B > 65535 || H > 65535) return PA_ERR_INVALID;  // grid y / z limits
  const int64_t L_max = static_cast<int64_t>(MB) * S;
  if (L_max > INT_MAX || max_seq_len < 0 || max_seq_len > L_max) return PA_ERR_INVALID;
  int P, NP;
  if (!plan(B, H, S, max_seq_len, partition, &P, &NP)) return PA_ERR_INVALID;
  if (B == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !seq_lens || MB == 0)
    return PA_ERR_INVALID;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID;
  const size_t need = workspace_for(B, H, D, NP);
  if (need > 0 && (!workspace || ws_bytes < need || !aligned16(workspace))) return PA_ERR_INVALID;

  pa::DecodeParams prm{};
  prm.out = out;
  prm.q = q;
  prm.k_cache = k_cache;
  prm.v_cache = v_cache;
  prm.block_tables = block_tables;
  prm.seq_lens = seq_lens;
  prm.q_scale = scale * 1.4426950408889634f;  // log2(e)
  prm.v_scale = 1.f;
  prm.MB = MB;
  prm.B = B;
  prm.H = H;
  prm.Hkv = Hkv;
  prm.NB = NB;
  if (NP > 1) {
    const size_t n = static_cast<size_t>(B) * H * NP;
    prm.ws_m = static_cast<float*>(workspace);
    prm.ws_l = prm.ws_m + n;
    prm.ws_acc = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                          align256(n * 2 * sizeof(float)));
    prm.P = P;
    prm.NP = NP;
    prm.L_cap = static_cast<int>(std::min<int64_t>(L_max, static_cast<int64_t>(NP) * P));
  } else {
    prm.P = static_cast<int>(L_max > 0 ? L_max : S);  // one partition covers every block
    prm.NP = 1;
    prm.L_cap = static_cast<int>(L_max);
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  prm.k_new = k_new;
  prm.v_new = v_new;
  if (k_new) {
    if (dt == PA_F16) return dispatch_out<__half, true>(prm, out_dt, D, S, st);
    return dispatch_out<__nv_bfloat16, true>(prm, out_dt, D, S, st);
  }
  if (dt == PA_F16) return dispatch_out<__half, false>(prm, out_dt, D, S, st);
  return dispatch_out<__nv_bfloat16, false>(prm, out_dt, D, S, st);
}

}  // namespace

extern "C" {

pa_status pa_decode(void* out, pa_dtype out_dt, const void* q, const void* k_cache,
                    const void* v_cache, const int32_t* block_tables, int MB,
                    const int32_t* seq_lens, float scale, int B, int H, int D, int S, int NB,
                    pa_dtype dt, int partition, int max_seq_len, void* workspace,
                    size_t ws_bytes, void* stream) {
  return decode_impl(out, out_dt, q, nullptr, nullptr, k_cache, v_cache, block_tables, MB,
                     seq_lens, scale, B, H, H, D, S, NB, dt, partition, max_seq_len, workspace,
                     ws_bytes, stream);
}

pa_status pa_decode_append(void* out, pa_dtype out_dt, const void* q, const void* k_new,
                           const void* v_new, void* k_cache, void* v_cache,
                           const int32_t* block_tables, int MB, const int32_t* seq_lens,
                           float scale, int B, int H, int D, int S, int NB, pa_dtype dt,
                           int partition, int max_seq_len, void* workspace, size_t ws_bytes,
                           void* stream) {
  if (B > 0 && (!k_new || !v_new || !aligned16(k_new) || !aligned16(v_new)))
    return PA_ERR_INVALID;
  return decode_impl(out, out_dt, q, B > 0 ? k_new : nullptr, v_new, k_cache, v_cache,
                     block_tables, MB, seq_lens, scale, B, H, H, D, S, NB, dt, partition,
                     max_seq_len, workspace, ws_bytes, stream);
}

pa_status pa_decode_gqa(void* out, pa_dtype out_dt, const void* q, const void* k_new,
                        const void* v_new, void* k_cache, void* v_cache,
                        const int32_t* block_tables, int MB, const int32_t* seq_lens, float scale,
                        int B, int H, int Hkv, int D, int S, int NB, pa_dtype dt, int partition,
                        int max_seq_len, void* workspace, size_t ws_bytes, void* stream) {
  if ((k_new == nullptr) != (v_new == nullptr)) return PA_ERR_INVALID;
  if (k_new && B > 0 && (!aligned16(k_new) || !aligned16(v_new))) return PA_ERR_INVALID;
  return decode_impl(out, out_dt, q, B > 0 ? k_new : nullptr, v_new, k_cache, v_cache,
                     block_tables, MB, seq_lens, scale, B, H, Hkv, D, S, NB, dt, partition,
                     max_seq_len, workspace, ws_bytes, stream);
}

pa_status pa_prefill(void* out, pa_dtype out_dt, const void* q, const void* k_cache,
                     const void* v_cache, const int32_t* block_tables, int MB,
                     const int32_t* seq_lens, const int32_t* q_start, float scale, int B, int H,
                     int Hkv, int D, int S, int NB, pa_dtype dt, int T, int max_q_len,
                     void* stream) {
  if (B < 0 || H <= 0 || Hkv <= 0 || H % Hkv != 0 || T < 0 || max_q_len < 0 || MB < 0 || NB < 0)
    return PA_ERR_INVALID;
  if (!cache_dtype_ok(dt) || !out_dtype_ok(out_dt)) return PA_ERR_INVALID;
  if (!(D == 64 || D == 128) || !(S == 8 || S == 16 || S == 32 || S == 64 || S == 128))
    return PA_ERR_INVALID;
  if (!std::isfinite(scale) || !(scale > 0.f)) return PA_ERR_INVALID;
  if (B == 0 || T == 0 || max_q_len == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !seq_lens || !q_start)
    return PA_ERR_INVALID;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID;
  if (NB == 0 || static_cast<int64_t>(NB) * Hkv * S > INT_MAX) return PA_ERR_INVALID;
  if (ceil_div(max_q_len, 128) > INT_MAX / 2 || H > 65535 || B > 65535) return PA_ERR_INVALID;
  pa::PrefillParams prm;
  prm.out = out;
  prm.k_cache = k_cache;
  prm.v_cache = v_cache;
  prm.block_tables = block_tables;
  prm.seq_lens = seq_lens;
  prm.q_start = q_start;
  prm.scale_log2 = static_cast<float>(static_cast<double>(scale) * 1.4426950408889634);
  prm.MB = MB;
  prm.B = B;
  prm.H = H;
  prm.Hkv = Hkv;
  prm.NB = NB;
  prm.T = T;
  prm.max_q_len = max_q_len;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  return dt == PA_BF16 ? dispatch_prefill<__nv_bfloat16>(prm, q, out_dt, D, S, st)
                       : dispatch_prefill<__half>(prm, q, out_dt, D, S, st);
}

pa_status pa_kv_append_fp8(const void* k, const void* v, pa_dtype in_dt,
                           const int64_t* slot_mapping, void* k_cache, void* v_cache,
                           float k_scale, float v_scale, int T, int H, int D, int S, int NB,
                           void* stream) {
  if (T < 0 || H <= 0 || D <= 0 || S <= 0 || NB < 0 || !cache_dtype_ok(in_dt)) return PA_ERR_INVALID;
  if (D % 16 != 0) return PA_ERR_INVALID;  // 8-byte code vectors, 16-byte cache rows
  if (!(std::isfinite(k_scale) && k_scale > 0.f && std::isfinite(v_scale) && v_scale > 0.f))
    return PA_ERR_INVALID;
  if (T == 0) return PA_OK;
  if (!k || !v || !slot_mapping || !k_cache || !v_cache) return PA_ERR_INVALID;
  if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID;
  const int vpr = D / 8;
  const int64_t total = static_cast<int64_t>(T) * H * vpr;
  const int64_t n_slots = static_cast<int64_t>(NB) * S;
  int64_t blocks = ceil_div(total, 256);
  const int64_t cap = 148LL * 16;
  if (blocks > cap) blocks = cap;
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (in_dt == PA_BF16)
    pa::kv_append_fp8_kernel<__nv_bfloat16><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        static_cast<const uint4*>(k), static_cast<const uint4*>(v), slot_mapping,
        static_cast<uint2*>(k_cache), static_cast<uint2*>(v_cache), k_scale, v_scale, total, H,
        vpr, S, n_slots);
  else
    pa::kv_append_fp8_kernel<__half><<<static_cast<unsigned>(blocks), 256, 0, st>>>(
        static_cast<const uint4*>(k), static_cast<const uint4*>(v), slot_mapping,
        static_cast<uint2*>(k_cache), static_cast<uint2*>(v_cache), k_scale, v_scale, total, H,
        vpr, S, n_slots);
  return cuda_status();
}

pa_status pa_decode_fp8(void* out, pa_dtype out_dt, const void* q, pa_dtype q_dt,
                        const void* k_cache, const void* v_cache, float k_scale, float v_scale,
                        const int32_t* block_tables, int MB, const int32_t* seq_lens, float scale,
                        int B, int H, int D, int S, int NB, int partition, int max_seq_len,
                        void* workspace, size_t ws_bytes, void* stream) {
  if (B < 0 || H <= 0 || NB < 0 || MB < 0) return PA_ERR_INVALID;
  if (!cache_dtype_ok(q_dt) || !out_dtype_ok(out_dt) || !decode_shape_ok(D, S)) return PA_ERR_INVALID;
  if (!std::isfinite(scale)) return PA_ERR_INVALID;
  if (!(std::isfinite(k_scale) && k_scale > 0.f && std::isfinite(v_scale) && v_scale > 0.f))
    return PA_ERR_INVALID;
  if (B > 65535 || H > 65535) return PA_ERR_INVALID;
  const int64_t L_max = static_cast<int64_t>(MB) * S;
  if (L_max > INT_MAX || max_seq_len < 0 || max_seq_len > L_max) return PA_ERR_INVALID;
  int P, NP;
  if (!plan(B, H, S, max_seq_len, partition, &P, &NP)) return PA_ERR_INVALID;
  if (B == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !seq_lens || MB == 0)
    return PA_ERR_INVALID;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID;
  const size_t need = workspace_for(B, H, D, NP);
  if (need > 0 && (!workspace || ws_bytes < need || !aligned16(workspace))) return PA_ERR_INVALID;
  pa::DecodeParams prm{};
  prm.out = out;
  prm.q = q;
  prm.k_cache = k_cache;
  prm.v_cache = v_cache;
  prm.block_tables = block_tables;
  prm.seq_lens = seq_lens;
  prm.q_scale = scale * k_scale * 1.4426950408889634f;  // K's scale folded into q, log2(e)
  prm.v_scale = v_scale;
  prm.MB = MB;
  prm.B = B;
  prm.H = H;
  prm.Hkv = H;
  prm.NB = NB;
  if (NP > 1) {
    const size_t n = static_cast<size_t>(B) * H * NP;
    prm.ws_m = static_cast<float*>(workspace);
    prm.ws_l = prm.ws_m + n;
    prm.ws_acc = reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) +
                                          align256(n * 2 * sizeof(float)));
    prm.P = P;
    prm.NP = NP;
    prm.L_cap = static_cast<int>(std::min<int64_t>(L_max, static_cast<int64_t>(NP) * P));
  } else {
    prm.P = static_cast<int>(L_max > 0 ? L_max : S);
    prm.NP = 1;
    prm.L_cap = static_cast<int>(L_max);
  }
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (q_dt == PA_F16) {
    switch (out_dt) {
      case PA_F32: return dispatch_fp8_shape<__half, float>(prm, D, S, st);
      case PA_F16: return dispatch_fp8_shape<__half, __half>(prm, D, S, st);
      case PA_BF16: return dispatch_fp8_shape<__half, __nv_bfloat16>(prm, D, S, st);
    }
  } else {
    switch (out_dt) {
      case PA_F32: return dispatch_fp8_shape<__nv_bfloat16, float>(prm, D, S, st);
      case PA_F16: return dispatch_fp8_shape<__nv_bfloat16, __half>(prm, D, S, st);
      case PA_BF16: return dispatch_fp8_shape<__nv_bfloat16, __nv_bfloat16>(prm, D, S, st);
    }
  }
  return PA_ERR_INVALID;
}

pa_status pa_get_device_error(void* stream, uint32_t* flags) {
  if (!flags) return PA_ERR_INVALID;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return PA_ERR_CUDA;
  unsigned int v = 0;
  if (cudaMemcpyFromSymbol(&v, pa::g_error_word, sizeof(v)) != cudaSuccess) return PA_ERR_CUDA;
  const unsigned int zero = 0;
  if (cudaMemcpyToSymbol(pa::g_error_word, &zero, sizeof(zero)) != cudaSuccess) return PA_ERR_CUDA;
  *flags = v;
  return PA_OK;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// pa_decode_noalloc: decode whose split-KV partials live in a static device
// array instead of a caller-provided workspace, for callers that cannot
// allocate device memory (see pagedattn.h). It reuses pa_decode unchanged.
// ---------------------------------------------------------------------------

namespace {

static __device__ __align__(256) unsigned char g_noalloc_scratch[PA_NOALLOC_SCRATCH_BYTES];

// Device address of g_noalloc_scratch per device, looked up on the first call
// made with that device current. The host-side name of the array is only a
// stand-in for the symbol, never a usable device address.
std::atomic<void*> g_noalloc_scratch_addr[kMaxDevices];

}  // namespace

extern "C" pa_status pa_decode_noalloc(void* out, pa_dtype out_dt, const void* q,
                                       const void* k_cache, const void* v_cache,
                                       const int32_t* block_tables, int MB,
                                       const int32_t* seq_lens, float scale, int B, int H, int D,
                                       int S, int NB, pa_dtype dt, int partition, int max_seq_len,
                                       void* stream) {
  int P, NP;
  if (B < 0 || H <= 0 || !decode_shape_ok(D, S) || !plan(B, H, S, max_seq_len, partition, &P, &NP))
    return PA_ERR_INVALID;
  const size_t need = workspace_for(B, H, D, NP);
  if (need > PA_NOALLOC_SCRATCH_BYTES) return PA_ERR_OOM;  // larger than the static array
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PA_ERR_CUDA;
  void* scratch = g_noalloc_scratch_addr[dev].load(std::memory_order_acquire);
  if (!scratch) {
    if (cudaGetSymbolAddress(&scratch, g_noalloc_scratch) != cudaSuccess || !scratch)
      return PA_ERR_CUDA;
    g_noalloc_scratch_addr[dev].store(scratch, std::memory_order_release);
  }
  return pa_decode(out, out_dt, q, k_cache, v_cache, block_tables, MB, seq_lens, scale, B, H, D, S,
                   NB, dt, partition, max_seq_len, scratch, PA_NOALLOC_SCRATCH_BYTES, stream);
}
