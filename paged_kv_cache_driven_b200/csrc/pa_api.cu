// The C-ABI layer (pagedattn.h): argument validation, launch planning, the
// split-KV workspace layout, tensor-map encoding and dispatch to the launchers
// of the translation units that hold the kernels (pa_k_*.cu), the device
// error words, and pa_decode_noalloc's static scratch. Every check runs on the
// host before anything is launched.

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

#include "pa_launch.h"
#include "pagedattn.h"

using pa::host::ceil_div;
using pa::host::kMaxDevices;

namespace {

constexpr int kDefaultPartition = 512;  // tokens per split-KV partition when splitting

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

bool cache_dtype_ok(pa_dtype dt) { return dt == PA_F16 || dt == PA_BF16; }

bool out_dtype_ok(pa_dtype dt) { return dt == PA_F16 || dt == PA_BF16 || dt == PA_F32; }

bool decode_shape_ok(int D, int S) {
  return (D == 64 || D == 128 || D == 256) && (S == 8 || S == 16 || S == 32);
}

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
//           multiple of S) while the grid would hold fewer CTAs than the device
//           has SMs, so that small batches still spread over every SM; no split
//           if one partition covers every request. (Measured at batch 1, 32
//           heads, 1.3K tokens: 256-token partitions, 192 CTAs, are fastest for
//           head sizes 64 to 256; 64-token ones, 672 CTAs, are 40 % slower,
//           each CTA's fixed start and end costing more than its short stream.)
//           Contexts of 32K tokens and more take partitions of up to 2048
//           tokens while the grid keeps 8 CTAs per SM.
//           A small grid then has a partition count of 3, 5, 6 or 7 rounded
//           to a power of two (the next, else the previous; partitions re-cut
//           evenly in whole blocks) when the grid stays within two CTAs per SM,
//           so that its split can merge inside a cluster (cluster_merge).
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
    const int64_t target = sm_count();
    const int64_t pairs = static_cast<int64_t>(B > 0 ? B : 1) * (H > 0 ? H : 1);
    while (P > 64 && (P / 2) % S == 0 && pairs * ceil_div(max_seq_len, P) < target) P /= 2;
    // long contexts (32K tokens and more) take partitions of up to 2048 tokens
    // while the grid keeps at least 8 CTAs per SM: fewer partials and per-CTA
    // starts (8 x U[32K, 131K] tokens on 32 heads: 1.627 ms against 1.658 ms
    // at 512; shorter requests run best at 512)
    if (max_seq_len >= 32768)
      while (P < 2048 && pairs * ceil_div(max_seq_len, 2 * P) >= 8 * target) P *= 2;
    const int64_t n = ceil_div(max_seq_len, P);
    if (n > 2 && n < 8 && (n & (n - 1)) != 0) {
      const int64_t up = n < 4 ? 4 : 8;
      for (const int64_t c : {up, up / 2}) {
        if (pairs * c > 2 * target) continue;
        // c partitions of a whole number of blocks; where blocks do not divide
        // evenly the last one or two hold no token (they only join the merge)
        *P_out = static_cast<int>(ceil_div(ceil_div(max_seq_len, c), S) * S);
        *NP_out = static_cast<int>(c);
        return true;
      }
    }
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

// The automatic plan for grouped-query heads (Hkv < H): the partition pass then
// has B * Hkv * ceil(G / 16) CTAs per partition (G = H / Hkv), up to 16 query
// heads per CTA. Where that grid at 512-token partitions holds at most two
// CTAs per SM, the partitions are halved (down to 128 tokens, multiples of S)
// while the grid stays within that bound: a small grid is resident at once,
// so shorter partitions shorten every CTA's stream (64 query heads on 8 KV
// heads, head_dim 128: one request of 1,332 tokens 19.5 -> 15.4 us, four of
// 2,048 23.6 -> 19.5 us). Larger grids, explicit partitions and one KV head per
// query head take plan().
bool plan_grouped(int B, int H, int Hkv, int S, int max_seq_len, int partition, int* P_out,
                  int* NP_out) {
  if (Hkv <= 0 || Hkv >= H || H % Hkv != 0 || partition != 0 || max_seq_len < 0 || S <= 0)
    return plan(B, H, S, max_seq_len, partition, P_out, NP_out);
  const int64_t ctas = static_cast<int64_t>(B > 0 ? B : 1) * Hkv * ceil_div(H / Hkv, 16);
  const int64_t cap = 2 * static_cast<int64_t>(sm_count());
  int P = kDefaultPartition;
  if (ctas * ceil_div(max_seq_len, P) > cap) return plan(B, H, S, max_seq_len, 0, P_out, NP_out);
  while (P > 128 && (P / 2) % S == 0 && ctas * ceil_div(max_seq_len, P / 2) <= cap) P /= 2;
  const int64_t np = ceil_div(max_seq_len, P);
  *P_out = np <= 1 ? 0 : P;
  *NP_out = np <= 1 ? 1 : static_cast<int>(np);
  return true;
}

// Whether a partition pass of B x H x NP CTAs holds at most two CTAs per SM
// (a small grid: resident at once, so its split can merge inside clusters).
bool small_grid(int B, int H, int NP) {
  return static_cast<int64_t>(B) * H * NP <= 2 * static_cast<int64_t>(sm_count());
}

// Whether the partition pass takes its wide CTA shapes (DecodeTiling, WIDE):
// grids of at most four CTAs per SM, the small grids among them (head_dim 64,
// block 8, 512 CTAs: 21.5 us wide against 23.6 narrow).
bool wide_grid(int B, int H, int NP) {
  return static_cast<int64_t>(B) * H * NP <= 4 * static_cast<int64_t>(sm_count());
}

// Whether an automatic split of NP partitions over B x H (request, head) pairs
// merges inside clusters instead of through the workspace and the merge
// kernel: NP is a portable cluster size (2, 4 or 8; the cluster spans the
// grid's x dimension, the partitions of one pair), and the grid fits within two
// CTAs per SM, so that it is resident at once and the CTAs that wait at their
// cluster's barrier hold no SM another CTA is queued for. Large grids keep the
// merge kernel, which overlaps their last wave.
bool cluster_merge(int B, int H, int NP) {
  if (NP != 2 && NP != 4 && NP != 8) return false;
  return small_grid(B, H, NP);
}

// Split-KV workspace: m and l [B, H, NP], then (256-byte aligned) acc [B, H, NP, D].
size_t acc_offset(size_t n) { return align256(n * 2 * sizeof(float)); }

size_t workspace_for(int B, int H, int D, int NP) {
  if (NP <= 1) return 0;
  const size_t n = static_cast<size_t>(B) * H * NP;
  return acc_offset(n) + n * D * sizeof(float);
}

// Points the kernel parameters at the workspace parts for NP > 1 partitions.
void set_split(pa::DecodeParams& prm, void* workspace, int B, int H, int P, int NP,
               int64_t L_max) {
  const size_t n = static_cast<size_t>(B) * H * NP;
  uint8_t* base = static_cast<uint8_t*>(workspace);
  prm.ws_m = reinterpret_cast<float*>(base);
  prm.ws_l = prm.ws_m + n;
  prm.ws_acc = reinterpret_cast<float*>(base + acc_offset(n));
  prm.P = P;
  prm.NP = NP;
  prm.L_cap = static_cast<int>(std::min<int64_t>(L_max, static_cast<int64_t>(NP) * P));
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

}  // namespace

namespace pa {
namespace host {

// kind: 0 = f16, 1 = bf16: boxes of 64 elements, so every box row is 128 bytes,
// the 128-byte swizzle's width; 2 = one-byte E4M3 codes: a box spans the whole
// D-byte row, unswizzled (the consumer converts it to 16-bit tiles itself).
static bool row_map_kind(CUtensorMap* out, const void* base, int64_t rows, int D, int box_rows,
                         int kind) {
  static std::mutex mu;
  static RowMapKey keys[16];
  static CUtensorMap maps[16];
  static int used = 0, next = 0;
  const RowMapKey key{base, rows, D, box_rows, kind};
  std::lock_guard<std::mutex> lock(mu);
  for (int k = 0; k < used; ++k)
    if (keys[k] == key) {
      *out = maps[k];
      return true;
    }
  auto fn = encode_fn();
  if (!fn) return false;
  const bool codes = kind == 2;
  const cuuint64_t esize = codes ? 1 : 2;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(D) * esize};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(codes ? D : 128 / esize),
                             static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  const CUtensorMapDataType type =
      codes ? CU_TENSOR_MAP_DATA_TYPE_UINT8
            : (kind == 1 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16);
  CUtensorMap map;
  if (fn(&map, type, 2, const_cast<void*>(base), dims, strides, box, estr,
         CU_TENSOR_MAP_INTERLEAVE_NONE,
         codes ? CU_TENSOR_MAP_SWIZZLE_NONE : CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return false;
  const int slot = used < 16 ? used++ : next;
  next = (slot + 1) % 16;
  keys[slot] = key;
  maps[slot] = map;
  *out = map;
  return true;
}

bool row_map(CUtensorMap* out, const void* base, int64_t rows, int D, int box_rows, pa_dtype dt) {
  return row_map_kind(out, base, rows, D, box_rows, dt == PA_BF16 ? 1 : 0);
}

bool row_map_codes(CUtensorMap* out, const void* base, int64_t rows, int D, int box_rows) {
  return row_map_kind(out, base, rows, D, box_rows, 2);
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

}  // namespace host
}  // namespace pa

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
  return pa::host::launch_kv_append(k, v, slot_mapping, k_cache, v_cache, T, H, D, S, NB,
                                    static_cast<cudaStream_t>(stream));
}

pa_status pa_copy_blocks(void* k_cache, void* v_cache, const int32_t* src_dst, int n, int H,
                         int S, int D, int NB, pa_dtype dt, void* stream) {
  if (n < 0 || H <= 0 || S <= 0 || D <= 0 || NB < 0 || !cache_dtype_ok(dt) || D % 8 != 0)
    return PA_ERR_INVALID;
  if (n == 0) return PA_OK;
  if (!k_cache || !v_cache || !src_dst || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID;
  return pa::host::launch_copy_blocks(k_cache, v_cache, src_dst, n, H, S, D, NB,
                                      static_cast<cudaStream_t>(stream));
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
  // grouped-query heads may split finer (plan_grouped); one KV head has the
  // fewest CTAs per partition and so the most partitions
  int Pg, NPg;
  if (H > 1 && plan_grouped(B, H, 1, S, max_seq_len, partition, &Pg, &NPg)) NP = std::max(NP, NPg);
  return workspace_for(B, H, D, NP);
}

pa_status pa_decode_plan_grouped(int B, int H, int Hkv, int D, int S, int max_seq_len,
                                 int partition, int* partition_tokens, int* num_partitions) {
  (void)D;
  if (!partition_tokens || !num_partitions || Hkv <= 0 || H <= 0 || H % Hkv != 0)
    return PA_ERR_INVALID;
  int P, NP;
  if (!plan_grouped(B, H, Hkv, S, max_seq_len, partition, &P, &NP)) return PA_ERR_INVALID;
  *partition_tokens = P;
  *num_partitions = NP;
  return PA_OK;
}

}  // extern "C"

namespace {

// The host checks of pa_decode's arguments, workspace aside (shared by its
// variants). On PA_OK, *P / *NP hold the plan and *noop is set for B == 0.
pa_status decode_check(const void* out, pa_dtype out_dt, const void* q, const void* k_cache,
                       const void* v_cache, const int32_t* block_tables, int MB,
                       const int32_t* seq_lens, float scale, int B, int H, int Hkv, int D, int S,
                       int NB, pa_dtype dt, int partition, int max_seq_len, int* P, int* NP,
                       bool* noop) {
  *noop = false;
  if (B < 0 || H <= 0 || NB < 0 || MB < 0) return PA_ERR_INVALID;
  if (Hkv <= 0 || H % Hkv != 0) return PA_ERR_INVALID;
  if (!cache_dtype_ok(dt) || !out_dtype_ok(out_dt) || !decode_shape_ok(D, S)) return PA_ERR_INVALID;
  if (!std::isfinite(scale)) return PA_ERR_INVALID;
  if (B > 65535 || H > 65535) return PA_ERR_INVALID;  // grid y / z limits
  const int64_t L_max = static_cast<int64_t>(MB) * S;
  if (L_max > INT_MAX || max_seq_len < 0 || max_seq_len > L_max) return PA_ERR_INVALID;
  if (!plan_grouped(B, H, Hkv, S, max_seq_len, partition, P, NP)) return PA_ERR_INVALID;
  if (B == 0) {
    *noop = true;
    return PA_OK;
  }
  if (!out || !q || !k_cache || !v_cache || !block_tables || !seq_lens || MB == 0)
    return PA_ERR_INVALID;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID;
  return PA_OK;
}

// pa_decode and pa_decode_append: k_new / v_new null = plain decode.
pa_status decode_impl(void* out, pa_dtype out_dt, const void* q, const void* k_new,
                      const void* v_new, const void* k_cache, const void* v_cache,
                      const int32_t* block_tables, int MB, const int32_t* seq_lens, float scale,
                      int B, int H, int Hkv, int D, int S, int NB, pa_dtype dt, int partition,
                      int max_seq_len, void* workspace, size_t ws_bytes, void* stream) {
  int P, NP;
  bool noop;
  const pa_status chk = decode_check(out, out_dt, q, k_cache, v_cache, block_tables, MB, seq_lens,
                                     scale, B, H, Hkv, D, S, NB, dt, partition, max_seq_len, &P,
                                     &NP, &noop);
  if (chk != PA_OK || noop) return chk;
  const int64_t L_max = static_cast<int64_t>(MB) * S;
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
    set_split(prm, workspace, B, H, P, NP, L_max);
  } else {
    prm.P = static_cast<int>(L_max > 0 ? L_max : S);  // one partition covers every block
    prm.NP = 1;
    prm.L_cap = static_cast<int>(L_max);
  }
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  prm.k_new = k_new;
  prm.v_new = v_new;
  if (H != Hkv)  // (the grouped-query kernel always merges through the workspace)
    return pa::host::launch_grouped(prm, dt, out_dt, D, S, k_new != nullptr, st);
  const bool cluster = partition == 0 && cluster_merge(B, H, prm.NP);
  return pa::host::launch_decode16(prm, dt, out_dt, D, S, k_new != nullptr, cluster,
                                   wide_grid(B, H, prm.NP), st);
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
  if (!(D == 64 || D == 128 || D == 256) || !(S == 8 || S == 16 || S == 32 || S == 64 || S == 128))
    return PA_ERR_INVALID;
  if (!std::isfinite(scale) || !(scale > 0.f)) return PA_ERR_INVALID;
  if (B == 0 || T == 0 || max_q_len == 0) return PA_OK;
  if (!out || !q || !k_cache || !v_cache || !block_tables || !seq_lens || !q_start)
    return PA_ERR_INVALID;
  if (!aligned16(out) || !aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache))
    return PA_ERR_INVALID;
  if (NB == 0 || static_cast<int64_t>(NB) * Hkv * S > INT_MAX) return PA_ERR_INVALID;
  // grid (H, row blocks of up to 256 rows, B): the y and z extents are 16-bit
  if (ceil_div(max_q_len, 128) > 65535 || B > 65535) return PA_ERR_INVALID;
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
  return pa::host::launch_prefill(prm, q, dt, out_dt, D, S, static_cast<cudaStream_t>(stream));
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
  return pa::host::launch_kv_append_fp8(k, v, in_dt, slot_mapping, k_cache, v_cache, k_scale,
                                        v_scale, T, H, D, S, NB, static_cast<cudaStream_t>(stream));
}

// pa_decode_fp8 and pa_decode_append_fp8: k_new / v_new null = plain decode.
// pa_decode_gqa_fp8: Hkv < H (grouped-query heads; no fused append).
static pa_status decode_fp8_impl(void* out, pa_dtype out_dt, const void* q, pa_dtype q_dt,
                                 const void* k_new, const void* v_new, const void* k_cache,
                                 const void* v_cache, float k_scale, float v_scale,
                                 const int32_t* block_tables, int MB, const int32_t* seq_lens,
                                 float scale, int B, int H, int Hkv, int D, int S, int NB,
                                 int partition, int max_seq_len, void* workspace,
                                 size_t ws_bytes, void* stream) {
  if (B < 0 || H <= 0 || NB < 0 || MB < 0) return PA_ERR_INVALID;
  if (Hkv <= 0 || H % Hkv != 0 || (k_new && Hkv != H)) return PA_ERR_INVALID;
  if (!cache_dtype_ok(q_dt) || !out_dtype_ok(out_dt) || !decode_shape_ok(D, S)) return PA_ERR_INVALID;
  if (!std::isfinite(scale)) return PA_ERR_INVALID;
  if (!(std::isfinite(k_scale) && k_scale > 0.f && std::isfinite(v_scale) && v_scale > 0.f))
    return PA_ERR_INVALID;
  if (B > 65535 || H > 65535) return PA_ERR_INVALID;
  const int64_t L_max = static_cast<int64_t>(MB) * S;
  if (L_max > INT_MAX || max_seq_len < 0 || max_seq_len > L_max) return PA_ERR_INVALID;
  int P, NP;
  if (!plan_grouped(B, H, Hkv, S, max_seq_len, partition, &P, &NP)) return PA_ERR_INVALID;
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
  prm.Hkv = Hkv;
  prm.NB = NB;
  if (NP > 1) {
    set_split(prm, workspace, B, H, P, NP, L_max);
  } else {
    prm.P = static_cast<int>(L_max > 0 ? L_max : S);
    prm.NP = 1;
    prm.L_cap = static_cast<int>(L_max);
  }
  if (Hkv != H)  // grouped-query heads: the tensor-core kernel
    return pa::host::launch_grouped_fp8(prm, q_dt, out_dt, D, S,
                                        static_cast<cudaStream_t>(stream));
  const bool append = k_new != nullptr;
  if (append && (!v_new || !aligned16(k_new) || !aligned16(v_new))) return PA_ERR_INVALID;
  prm.k_new = k_new;
  prm.v_new = v_new;
  const bool cluster = partition == 0 && cluster_merge(B, H, prm.NP);
  return pa::host::launch_decode_fp8(prm, q_dt, out_dt, D, S, cluster, wide_grid(B, H, prm.NP),
                                     append, k_scale, static_cast<cudaStream_t>(stream));
}

pa_status pa_decode_fp8(void* out, pa_dtype out_dt, const void* q, pa_dtype q_dt,
                        const void* k_cache, const void* v_cache, float k_scale, float v_scale,
                        const int32_t* block_tables, int MB, const int32_t* seq_lens, float scale,
                        int B, int H, int D, int S, int NB, int partition, int max_seq_len,
                        void* workspace, size_t ws_bytes, void* stream) {
  return decode_fp8_impl(out, out_dt, q, q_dt, nullptr, nullptr, k_cache, v_cache, k_scale,
                         v_scale, block_tables, MB, seq_lens, scale, B, H, H, D, S, NB,
                         partition, max_seq_len, workspace, ws_bytes, stream);
}

pa_status pa_decode_gqa_fp8(void* out, pa_dtype out_dt, const void* q, pa_dtype q_dt,
                            const void* k_cache, const void* v_cache, float k_scale,
                            float v_scale, const int32_t* block_tables, int MB,
                            const int32_t* seq_lens, float scale, int B, int H, int Hkv, int D,
                            int S, int NB, int partition, int max_seq_len, void* workspace,
                            size_t ws_bytes, void* stream) {
  return decode_fp8_impl(out, out_dt, q, q_dt, nullptr, nullptr, k_cache, v_cache, k_scale,
                         v_scale, block_tables, MB, seq_lens, scale, B, H, Hkv, D, S, NB,
                         partition, max_seq_len, workspace, ws_bytes, stream);
}

pa_status pa_decode_append_fp8(void* out, pa_dtype out_dt, const void* q, pa_dtype q_dt,
                               const void* k_new, const void* v_new, void* k_cache,
                               void* v_cache, float k_scale, float v_scale,
                               const int32_t* block_tables, int MB, const int32_t* seq_lens,
                               float scale, int B, int H, int D, int S, int NB, int partition,
                               int max_seq_len, void* workspace, size_t ws_bytes, void* stream) {
  if (B > 0 && (!k_new || !v_new)) return PA_ERR_INVALID;
  return decode_fp8_impl(out, out_dt, q, q_dt, B > 0 ? k_new : nullptr, v_new, k_cache, v_cache,
                         k_scale, v_scale, block_tables, MB, seq_lens, scale, B, H, H, D, S, NB,
                         partition, max_seq_len, workspace, ws_bytes, stream);
}

pa_status pa_get_device_error(void* stream, uint32_t* flags) {
  if (!flags) return PA_ERR_INVALID;
  if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return PA_ERR_CUDA;
  unsigned int v = 0;
  using namespace pa::host;
  if (!take_error_append(&v) || !take_error_decode16(&v) || !take_error_grouped(&v) ||
      !take_error_fp8(&v) || !take_error_prefill(&v))
    return PA_ERR_CUDA;
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

// Device address of g_noalloc_scratch per device, looked up with the device
// current and keyed by the context it was looked up in: a context that is torn
// down and created again (cudaDeviceReset, for one) loads the module again, and
// the array can move. The host-side name of the array is only a stand-in for
// the symbol, never a usable device address.
struct ScratchAddr {
  unsigned long long ctx_id = 0;  // cuCtxGetId of the context the address belongs to
  void* addr = nullptr;
};
std::mutex g_noalloc_mu;
ScratchAddr g_noalloc_addr[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

// The unique id of the current context (0 if the driver does not give one).
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrentFn>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetIdFn>(f);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx ||
      get_id(ctx, &id) != CUDA_SUCCESS)
    return 0;
  return id;
}

}  // namespace

extern "C" size_t pa_noalloc_scratch_bytes(void) { return PA_NOALLOC_SCRATCH_BYTES; }

extern "C" pa_status pa_decode_noalloc(void* out, pa_dtype out_dt, const void* q,
                                       const void* k_cache, const void* v_cache,
                                       const int32_t* block_tables, int MB,
                                       const int32_t* seq_lens, float scale, int B, int H, int D,
                                       int S, int NB, pa_dtype dt, int partition, int max_seq_len,
                                       void* stream) {
  // pa_decode's own checks first, so a bad argument is PA_ERR_INVALID, never PA_ERR_OOM
  int P, NP;
  bool noop;
  const pa_status st = decode_check(out, out_dt, q, k_cache, v_cache, block_tables, MB, seq_lens,
                                    scale, B, H, H, D, S, NB, dt, partition, max_seq_len, &P, &NP,
                                    &noop);
  if (st != PA_OK || noop) return st;
  const size_t need = workspace_for(B, H, D, NP);
  if (need > PA_NOALLOC_SCRATCH_BYTES) return PA_ERR_OOM;  // larger than the static array
  void* scratch = nullptr;
  if (need > 0) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return PA_ERR_CUDA;
    const unsigned long long ctx = current_context_id();
    std::lock_guard<std::mutex> lock(g_noalloc_mu);
    ScratchAddr& a = g_noalloc_addr[dev];
    if (!a.addr || a.ctx_id != ctx || ctx == 0) {
      void* p = nullptr;
      if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return PA_ERR_CUDA;
      a.addr = p;
      a.ctx_id = ctx;
    }
    scratch = a.addr;
  }
  return pa_decode(out, out_dt, q, k_cache, v_cache, block_tables, MB, seq_lens, scale, B, H, D, S,
                   NB, dt, partition, max_seq_len, scratch, PA_NOALLOC_SCRATCH_BYTES, stream);
}
