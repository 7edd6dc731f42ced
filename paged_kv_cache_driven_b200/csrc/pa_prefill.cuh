// Paged prefill attention on the fifth-generation tensor cores.
//
// What it computes ("vLLM KV Cache and PagedAttention Explained", Step 6
// "Prefill and Decode", and the attention formula of its Appendix): request i
// holds seq_lens[i] = L tokens in the paged cache, the last n = q_start[i+1] -
// q_start[i] of them new (already appended). New token j sits at position
// L - n + j and attends, causally, to cache tokens 0 .. L - n + j:
//   out[q_start[i] + j, h] = softmax_t(scale * q . K_t) V_t over those tokens,
// K_t / V_t read through the block table (token t in block
// block_tables[i][t / S], slot t % S), query head h reading KV head h / (H / Hkv).
//
// One CTA per (256 query rows = two 128-row tiles, query head, request), 576
// threads in four roles:
//   warps 0-7, 8-15  softmax for query tile 0 / 1, two warpgroups per tile:
//              warpgroup half h takes keys 64 h .. 64 h + 63 of each key tile
//              and output columns h D / 2 .. of each row; thread r owns row r
//              of its tile (tensor-memory lane r). It reads its half of the
//              scores from tensor memory, meets the other half on an mbarrier
//              to share the row max, keeps the running max / its share of the
//              sum in fp32, writes the weights P back over the scores as 16-bit
//              pairs (bf16 as hi + lo halves, so the weights keep ~16 bits), and
//              rescales its output columns when the reference max moves;
//   warp 16    producer: initialises the barriers, then TMA loads of the two
//              Q tiles and of 128-key K / V tiles, one box per (cache block,
//              64-column block); Q and the first K tile go out before the
//              CTA-wide sync, overlapping the tensor-memory allocation; K and V
//              run two tiles ahead (four for head size 64); lane b reads the
//              table entry of block b of a tile and issues its boxes, so a
//              tile's boxes go out in parallel;
//   warp 17    MMA issuer (lane 0) and tensor-memory owner, also zeroing V rows
//              past the end of the request in the last key tile:
//              S_t = Q_t K^T (both operands K-major in shared memory) and
//              O_t += P_t V (P_t from tensor memory, V an MN-major operand),
//              fp32 accumulators in tensor memory: tile t's S/P in columns
//              256 t .. 256 t + 127, its O in the next 128.
// The two tiles ping-pong: while one tile's softmax runs, the tensor cores
// work on the other tile's products. All shared tiles use the 128-byte swizzle,
// so the TMA boxes land directly in the canonical operand layout. Every wait is
// bounded (about a second); a timeout sets PA_DEVERR_TIMEOUT, stops all roles,
// waits for the copies and MMAs in flight and frees tensor memory.
#pragma once

#include <cuda.h>

#include "pa_device.cuh"
#include "pa_launch.h"
#include "pa_tcgen05.cuh"

namespace pa {

#ifdef PA_PREFILL_TRACE
// Trace build only (libpagedattn_trace.so; the library proper compiles none of
// this): clock64() stamps at the kernel's hand-offs, for the CTAs of query
// head 0 with request < 8 and row block < 8, indexed [CTA][slot][key tile].
// Slots: 31 start, 30 end; producer 25 K(j) issued, 26 V(j) issued; MMA warp
// 24 V(j) landed, 20 + t P(j) of tile t seen, 22 + t its P.V and next S
// issued; softmax half k = 2t + hw: 0 + k scores ready, 4 + k row max taken,
// 8 + k max exchanged, 12 + k P stored, 16 + k output rescaled and fenced.
constexpr int kTraceCtas = 64, kTraceSlots = 32, kTraceTiles = 48;
__device__ long long g_prefill_trace[kTraceCtas][kTraceSlots][kTraceTiles];
#define PA_TRACE(slot, j)                                                       \
  do {                                                                          \
    if (trc >= 0 && (j) < kTraceTiles) g_prefill_trace[trc][slot][j] = clock64(); \
  } while (0)
#else
#define PA_TRACE(slot, j) \
  do {                    \
  } while (0)
#endif


template <int D, bool LO>
struct PrefillTiling {
  static constexpr int BM = 128;              // query rows per tile (MMA M)
  // query tiles per CTA: two that ping-pong; head_dim 256 holds one (its S and
  // O take 384 of the 512 tensor-memory columns, and a second 64 KB query tile
  // would not fit beside the K and V tiles)
  static constexpr int NQT = D == 256 ? 1 : 2;
  static constexpr int BN = 128;              // keys per tile
  // separate K and V rings: S needs K(j + 1) right after P(j) is ready,
  // V(j + 1) only after the next softmax (one stage each at head_dim 256:
  // 64 KB tiles)
  static constexpr int KST = D == 256 ? 1 : (D == 128 ? 2 : 4);  // K stages
  static constexpr int VST = D == 256 ? 1 : (D == 128 ? 2 : 4);  // V stages
  static constexpr int COLB = D / 64;         // 64-element (128-byte) column blocks
  static constexpr int CB_BYTES = 128 * 128;  // one column block of 128 rows
  static constexpr int Q_BYTES = BM * D * 2;  // one query tile
  static constexpr int KV_BYTES = BN * D * 2;
  static constexpr int OFF_K = NQT * Q_BYTES;
  static constexpr int OFF_V = OFF_K + KST * KV_BYTES;
  static constexpr int OFF_XCH = OFF_V + VST * KV_BYTES;  // row-max exchange between halves
  static constexpr int XCH_BYTES = NQT * 2 * 2 * BM * 4;  // [tile][phase parity][half][row]
  static constexpr int OFF_BAR = OFF_XCH + XCH_BYTES;
  // + alignment slack and barriers; at least 120 KB, so that one CTA holds an
  // SM (it allocates all 512 tensor-memory columns)
  static constexpr int SMEM = 1024 + OFF_BAR + 256 > 120 * 1024 ? 1024 + OFF_BAR + 256 : 120 * 1024;
  static constexpr int THREADS = NQT * 256 + 64;  // two softmax warpgroups per tile
  static constexpr uint32_t TMEM_COLS = 512;  // per tile: S/P 128 columns, O D columns
  static_assert(D == 64 || D == 128 || D == 256, "head size 64, 128 or 256");
  // tiles sit 256 columns apart: S (128 columns) then O (D columns)
  static_assert(NQT == 1 ? 128 + D <= 512 : 128 + D <= 256, "tensor-memory columns");
  static_assert(SMEM <= 232448, "shared memory per CTA");
};

// mbarrier wait bounded by time and by the CTA's abort flag.
__device__ __forceinline__ bool wait_or_abort(uint64_t* bar, uint32_t parity,
                                              volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (*abort_flag) return false;
    if (clock64() - t0 > kWaitLimitCycles) {
      *abort_flag = 1;
      raise_error(PA_DEVERR_TIMEOUT);
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ void tma_load_2d_nohint(void* dst, const void* tmap, int x, int y,
                                                   uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

template <typename T>
__device__ __forceinline__ uint32_t pack_pair(float a, float b);
template <>
__device__ __forceinline__ uint32_t pack_pair<__nv_bfloat16>(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}
template <>
__device__ __forceinline__ uint32_t pack_pair<__half>(float a, float b) {
  const __half2 v = __floats2half2_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// The three-input max.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x with the hardware approximation (relative error about 2^-22; 2^-inf = 0).
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

template <typename TO>
__device__ __forceinline__ void store_row32(TO* dst, const float (&v)[32]);
template <>
__device__ __forceinline__ void store_row32<float>(float* dst, const float (&v)[32]) {
#pragma unroll
  for (int k = 0; k < 8; ++k)
    reinterpret_cast<float4*>(dst)[k] = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2],
                                                    v[4 * k + 3]);
}
template <>
__device__ __forceinline__ void store_row32<__nv_bfloat16>(__nv_bfloat16* dst,
                                                           const float (&v)[32]) {
#pragma unroll
  for (int k = 0; k < 4; ++k)
    reinterpret_cast<uint4*>(dst)[k] = make_uint4(
        pack_pair<__nv_bfloat16>(v[8 * k], v[8 * k + 1]),
        pack_pair<__nv_bfloat16>(v[8 * k + 2], v[8 * k + 3]),
        pack_pair<__nv_bfloat16>(v[8 * k + 4], v[8 * k + 5]),
        pack_pair<__nv_bfloat16>(v[8 * k + 6], v[8 * k + 7]));
}
template <>
__device__ __forceinline__ void store_row32<__half>(__half* dst, const float (&v)[32]) {
#pragma unroll
  for (int k = 0; k < 4; ++k)
    reinterpret_cast<uint4*>(dst)[k] =
        make_uint4(pack_pair<__half>(v[8 * k], v[8 * k + 1]),
                   pack_pair<__half>(v[8 * k + 2], v[8 * k + 3]),
                   pack_pair<__half>(v[8 * k + 4], v[8 * k + 5]),
                   pack_pair<__half>(v[8 * k + 6], v[8 * k + 7]));
}

// All 32 lanes wait; false (for every lane) if any lane's wait failed.
__device__ __forceinline__ bool wait_warp(uint64_t* bar, uint32_t parity,
                                          volatile int* abort_flag) {
  const bool ok = wait_or_abort(bar, parity, abort_flag);
  return __all_sync(kFullMask, ok);
}

template <typename T, typename TO, int D, int S>
__global__ void __launch_bounds__(576, 1)
    paged_prefill_kernel(const PrefillParams p, const __grid_constant__ CUtensorMap tmq,
                         const __grid_constant__ CUtensorMap tmk,
                         const __grid_constant__ CUtensorMap tmv) {
  constexpr bool LO = std::is_same<T, __nv_bfloat16>::value;
  using Tl = PrefillTiling<D, LO>;
  constexpr int BPT = Tl::BN / S;  // cache blocks per key tile
  static_assert(S >= 8 && S <= 128 && Tl::BN % S == 0, "block size 8 .. 128, dividing 128");

  const int i = blockIdx.z, h = blockIdx.x;
  const int L = p.seq_lens[i];
  const int q0 = p.q_start[i], q1 = p.q_start[i + 1];
  const int n = q1 - q0;
  if (L < 0 || L > static_cast<int64_t>(p.MB) * S || n < 0 || n > L || q0 < 0 || q1 > p.T ||
      n > p.max_q_len) {
    if (threadIdx.x == 0 && blockIdx.y == 0 && h == 0) raise_error(PA_DEVERR_SEQ_LEN);
    return;
  }
  constexpr int ROWS = Tl::NQT * Tl::BM;
  const int ncta = (n + ROWS - 1) / ROWS;
  const int ct = ncta - 1 - static_cast<int>(blockIdx.y);  // longest first (grid: heads fastest)
  if (ct < 0) return;
  const int row0 = ct * ROWS;
  const int ctx = L - n;  // tokens cached before the first new one
  // key tiles each query tile needs (0: the tile holds no rows of this request)
  int nk[Tl::NQT];
#pragma unroll
  for (int t = 0; t < Tl::NQT; ++t) {
    const int first = row0 + t * Tl::BM;
    nk[t] = first >= n ? 0 : (ctx + min(n, first + Tl::BM) - 1) / Tl::BN + 1;
  }
  int NK = nk[0], nq = 1;  // key tiles of the CTA; query tiles holding rows
#pragma unroll
  for (int t = 1; t < Tl::NQT; ++t) {
    NK = max(NK, nk[t]);
    if (nk[t] > 0) nq = t + 1;
  }
  const int hk = h / (p.H / p.Hkv);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* sm = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  uint8_t* sQ = sm;
  uint8_t* sK = sm + Tl::OFF_K;
  uint8_t* sV = sm + Tl::OFF_V;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sm + Tl::OFF_BAR);
  uint64_t* q_full = bars;
  uint64_t* k_full = bars + 1;                // [KST]
  uint64_t* k_empty = k_full + Tl::KST;       // [KST]
  uint64_t* v_full = k_empty + Tl::KST;       // [VST]
  uint64_t* v_empty = v_full + Tl::VST;       // [VST]
  uint64_t* s_full = v_empty + Tl::VST;       // [NQT]
  uint64_t* p_full = s_full + Tl::NQT;        // [NQT]
  uint64_t* o_done = p_full + Tl::NQT;        // [NQT]
  uint64_t* xch_bar = o_done + Tl::NQT;       // [NQT]: the tile's two halves have posted
  uint64_t* mma_done = xch_bar + Tl::NQT;
  float* xch = reinterpret_cast<float*>(sm + Tl::OFF_XCH);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mma_done + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
#ifdef PA_PREFILL_TRACE
  const int trc = (h == 0 && i < 8 && blockIdx.y < 8) ? i * 8 + blockIdx.y : -1;
  if (threadIdx.x == 0) PA_TRACE(31, 0);
#endif
  constexpr int kProducer = 4 * Tl::NQT * 2, kIssuer = kProducer + 1;  // warps 16, 17
  const int nblk = (L + S - 1) / S;
  const int32_t* table = p.block_tables + static_cast<int64_t>(i) * p.MB;
  // this lane's block id in key tile j (-1: none or invalid)
  auto block_id = [&](int j) {
    const int lb = j * BPT + lane;
    int id = -1;
    if (lane < BPT && lb < nblk) {
      id = table[lb];
      if (id < 0 || id >= p.NB) {
        raise_error(PA_DEVERR_BLOCK_ID);
        id = -1;
      }
    }
    return id;
  };
  // one K or V tile: every lane issues the boxes of its block
  auto load_tile = [&](const CUtensorMap* map, uint8_t* dst, uint64_t* full, int id) {
    const int nvalid = __popc(__ballot_sync(kFullMask, id >= 0));
    if (lane == 0)
      mbar_arrive_expect_tx(full, static_cast<uint32_t>(nvalid) * S * 128 * Tl::COLB);
    __syncwarp();
    if (id >= 0) {
      const int y = (id * p.Hkv + hk) * S;
#pragma unroll
      for (int c = 0; c < Tl::COLB; ++c)
        tma_load_2d_nohint(dst + c * Tl::CB_BYTES + lane * S * 128, map, c * 64, y, full);
    }
  };
  // The producer initialises the barriers and issues Q and the first K tile
  // before the CTA-wide sync, so that their latency overlaps the tensor-memory
  // allocation and the sync.
  int id_v = -1, id_k = -1;
  if (warp == kProducer) {
    if (lane == 0) {
      mbar_init(q_full, 1);
      for (int s = 0; s < Tl::KST; ++s) {
        mbar_init(&k_full[s], 1);
        mbar_init(&k_empty[s], 1);
      }
      for (int s = 0; s < Tl::VST; ++s) {
        mbar_init(&v_full[s], 1);
        mbar_init(&v_empty[s], 1);
      }
      for (int t = 0; t < Tl::NQT; ++t) {
        mbar_init(&s_full[t], 1);
        mbar_init(&p_full[t], 256);
        mbar_init(&o_done[t], 1);
        mbar_init(&xch_bar[t], 256);
      }
      mbar_init(mma_done, 1);
      *abort_flag = 0;
      fence_mbar_init();
    }
    __syncwarp();
    if (lane == 0) {
      mbar_arrive_expect_tx(q_full, nq * Tl::Q_BYTES);
      for (int t = 0; t < nq; ++t)
#pragma unroll
        for (int c = 0; c < Tl::COLB; ++c)
          tc::tma_load_3d(sQ + t * Tl::Q_BYTES + c * Tl::CB_BYTES, &tmq, c * 64, h,
                          q0 + row0 + t * Tl::BM, q_full);
    }
    id_v = block_id(0);
    id_k = id_v;
    load_tile(&tmk, sK, &k_full[0], id_k);
  }
  if (warp == kIssuer) {
    __syncwarp();
    tc::tmem_alloc(tmem_slot, Tl::TMEM_COLS);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = *tmem_slot;
  if (warp == kProducer) {
    // ---------------- producer: lane b loads cache block b of each key tile ----------------
    // K(j + 1) goes out before V(j); block ids are read one tile ahead
    int k_issued = 1, v_issued = 0;
    bool ok = true;
    if (NK > 1) id_k = block_id(1);
    for (int j = 0; j < NK; ++j) {
      if (j + 1 < NK) {
        const int kj = j + 1, st = kj % Tl::KST;
        if (kj >= Tl::KST && !(ok = wait_warp(&k_empty[st], ((kj / Tl::KST) - 1) & 1, abort_flag)))
          break;
        load_tile(&tmk, sK + st * Tl::KV_BYTES, &k_full[st], id_k);
        if (lane == 0) PA_TRACE(25, kj);
        k_issued = kj + 1;
      }
      const int st = j % Tl::VST;
      if (j >= Tl::VST && !(ok = wait_warp(&v_empty[st], ((j / Tl::VST) - 1) & 1, abort_flag)))
        break;
      load_tile(&tmv, sV + st * Tl::KV_BYTES, &v_full[st], id_v);
      if (lane == 0) PA_TRACE(26, j);
      v_issued = j + 1;
      id_v = id_k;
      if (j + 2 < NK) id_k = block_id(j + 2);
    }
    // copies in flight land before the CTA can exit
    if (lane == 0) {
      mbar_wait_bounded(q_full, 0);
      for (int kj = max(k_issued - Tl::KST, 0); kj < k_issued; ++kj)
        mbar_wait_bounded(&k_full[kj % Tl::KST], (kj / Tl::KST) & 1);
      for (int vj = max(v_issued - Tl::VST, 0); vj < v_issued; ++vj)
        mbar_wait_bounded(&v_full[vj % Tl::VST], (vj / Tl::VST) & 1);
    }
    (void)ok;
    __syncwarp();
  } else if (warp == kIssuer) {
    // ---------------- MMA issuer (lane 0), V tail zeroing (whole warp) ----------------
    constexpr int fmt = LO ? 1 : 0;
    constexpr uint32_t idesc_s = tc::instr_desc_f16(fmt, 0, 0, Tl::BM, Tl::BN);
    constexpr uint32_t idesc_o = tc::instr_desc_f16(fmt, 0, 1, Tl::BM, D);
    const uint32_t aQ = smem_u32(sQ), aK = smem_u32(sK), aV = smem_u32(sV);
    auto issue_s = [&](int t, int j) {  // S_t = Q_t K_j^T
      const uint32_t qb = aQ + t * Tl::Q_BYTES;
      const uint32_t kb = aK + (j % Tl::KST) * Tl::KV_BYTES;
#pragma unroll
      for (int s = 0; s < D / 16; ++s) {
        const uint32_t off = (s >> 2) * Tl::CB_BYTES + (s & 3) * 32;
        tc::mma_ss(tmem + t * 256, tc::smem_desc_sw128(qb + off, 16, 1024),
                   tc::smem_desc_sw128(kb + off, 16, 1024), idesc_s, s > 0);
      }
      tc::commit(&s_full[t]);
    };
    bool ok = wait_warp(q_full, 0, abort_flag) && wait_warp(&k_full[0], 0, abort_flag);
    if (ok) {
      tc::fence_after_sync();
      if (lane == 0) {
        for (int t = 0; t < nq; ++t) issue_s(t, 0);
        tc::commit(&k_empty[0]);
      }
    }
    for (int j = 0; ok && j < NK; ++j) {
      const int st = j % Tl::VST;
      ok = wait_warp(&v_full[st], (j / Tl::VST) & 1, abort_flag);
      if (!ok) break;
      if (lane == 0) PA_TRACE(24, j);
      const int kb = j * Tl::BN;
      if (j == NK - 1 && kb + Tl::BN > L) {
        // keys past the end of the request: P is 0 there, and 0 * NaN would not be
        uint8_t* vs = sV + st * Tl::KV_BYTES;
        for (int r = max(L - kb, 0) + lane; r < Tl::BN; r += 32)
#pragma unroll
          for (int c = 0; c < Tl::COLB; ++c)
#pragma unroll
            for (int k = 0; k < 8; ++k)
              reinterpret_cast<uint4*>(vs + c * Tl::CB_BYTES + r * 128)[k] = make_uint4(0, 0, 0, 0);
        tc::fence_proxy_async_smem();
        __syncwarp();
      }
      const uint32_t vb = aV + st * Tl::KV_BYTES;
      for (int t = 0; ok && t < Tl::NQT; ++t) {
        if (j >= nk[t]) continue;
        ok = wait_warp(&p_full[t], j & 1, abort_flag);
        if (!ok) break;
        if (lane == 0) PA_TRACE(20 + t, j);
        tc::fence_after_sync();
        if (lane == 0) {
          const uint32_t tS = tmem + t * 256, tO = tS + 128;
#pragma unroll
          for (int s = 0; s < Tl::BN / 16; ++s) {
            const uint64_t bdesc = tc::smem_desc_sw128(vb + s * 16 * 128, Tl::CB_BYTES, 1024);
            const uint32_t pa = tS + 32 * (s >> 1) + 8 * (s & 1);  // keys 16s .. 16s + 15
            tc::mma_ts(tO, pa, bdesc, idesc_o, j > 0 || s > 0);
            if constexpr (LO) tc::mma_ts(tO, pa + 16, bdesc, idesc_o, true);
          }
          if (j == nk[t] - 1) tc::commit(&o_done[t]);
        }
        if (j + 1 < nk[t]) {
          ok = wait_warp(&k_full[(j + 1) % Tl::KST], ((j + 1) / Tl::KST) & 1, abort_flag);
          if (!ok) break;
          tc::fence_after_sync();
          if (lane == 0) issue_s(t, j + 1);
        }
        if (lane == 0) PA_TRACE(22 + t, j);
      }
      // V(j) and, if any tile read it, K(j + 1) are free once these products finish
      if (ok && lane == 0) {
        tc::commit(&v_empty[st]);
        if (j + 1 < NK) tc::commit(&k_empty[(j + 1) % Tl::KST]);
      }
    }
    // every MMA issued has completed before tensor memory is released
    if (lane == 0) {
      tc::commit(mma_done);
      mbar_wait_bounded(mma_done, 0);
    }
    __syncwarp();
  } else {
    // ---------------- softmax: warps 8t .. 8t + 7 serve query tile t; warpgroup
    // half hw of them takes keys 64 hw .. 64 hw + 63 of each key tile and output
    // columns hw D / 2 .. of each row; thread r of a warpgroup owns row r ----------------
    constexpr int HK = Tl::BN / 2;  // keys per half
    constexpr int HD = D / 2;       // output columns per half
    const int t = warp >> 3;
    const int hw = (warp >> 2) & 1;
    const int r = threadIdx.x & 127;
    const uint32_t lane_base = static_cast<uint32_t>((warp & 3) * 32) << 16;
    const uint32_t tT = tmem + t * 256 + lane_base;
    const uint32_t tS = tT + hw * HK, tO = tT + 128 + hw * HD;
    const int qrow = row0 + t * Tl::BM + r;
    const int lim = min(ctx + qrow, L - 1);  // last key this row sees
    float m = -INFINITY, l = 0.f;  // l: this half's share of the running sum
    bool ok = nk[t] > 0;
    auto slot = [&](int j, int half) { return xch + ((t * 2 + (j & 1)) * 2 + half) * Tl::BM; };
    for (int j = 0; ok && j < nk[t]; ++j) {
      ok = wait_warp(&s_full[t], j & 1, abort_flag);
      if (!ok) break;
      if (r == 0) PA_TRACE(0 + t * 2 + hw, j);
      tc::fence_after_sync();
      const int kb = j * Tl::BN + hw * HK;
      // keys past this row's last one count as -inf (scale > 0, so the order of
      // raw scores is the order of scaled ones)
      const bool diag = kb + HK - 1 > lim;
      float x[HK];
      {
        uint32_t u[HK];
#pragma unroll
        for (int c4 = 0; c4 < HK / 32; ++c4)
          tc::tmem_ld32(tS + c4 * 32, *reinterpret_cast<uint32_t(*)[32]>(&u[c4 * 32]));
        tc::tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < HK; ++c) x[c] = __uint_as_float(u[c]);
        if (diag) {  // only tiles that reach past the row's last key pay for the mask
#pragma unroll
          for (int c = 0; c < HK; ++c) x[c] = kb + c > lim ? -INFINITY : x[c];
        }
      }
      float mx[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
      for (int c = 0; c < HK; c += 2) mx[(c >> 1) & 3] = fmax3(mx[(c >> 1) & 3], x[c], x[c + 1]);
      const float hmax = fmax3(fmaxf(mx[0], mx[1]), mx[2], mx[3]);
      // the row's max over both halves: post this half's, read the other's
      // (slots alternate with the key tile, so a half never overwrites a value
      // the other has not read yet)
      if (r == 0) PA_TRACE(4 + t * 2 + hw, j);
      slot(j, hw)[r] = hmax;
      mbar_arrive(&xch_bar[t]);
      ok = wait_warp(&xch_bar[t], j & 1, abort_flag);
      if (!ok) break;
      if (r == 0) PA_TRACE(8 + t * 2 + hw, j);
      const float tmax = fmaxf(hmax, slot(j, hw ^ 1)[r]) * p.scale_log2;
      // The reference max only moves when the tile max exceeds it by more than
      // 2^8 in weight; the weights stay <= 256, exact in the final ratio. Both
      // halves see the same tile max, so they take the same decision.
      const float m_new = fmaxf(m, tmax);
      const bool grow = m_new > m + 8.f;
      const float m_use = grow ? m_new : m;
      const float alpha = grow ? fast_exp2(m - m_use) : 1.f;
      m = m_use;
      // P over this half's scores, 8 keys at a time: keys 2k, 2k+1 of a 32-key
      // chunk q of the tile as one 16-bit pair in column 32q + k, and for bf16
      // the rounding residue p - bf16(p), itself rounded, in column 32q + 16 + k
      const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
      const float2 nm2 = make_float2(-m_use, -m_use);
      float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
#pragma unroll
      for (int g = 0; g < HK / 8; ++g) {
        float* v = &x[8 * g];
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 tt = ffma2(make_float2(v[2 * e], v[2 * e + 1]), sc2, nm2);
          const float2 pe = make_float2(fast_exp2(tt.x), fast_exp2(tt.y));
          acc[e & 1] = fadd2(acc[e & 1], pe);
          hi[e] = pack_pair<T>(pe.x, pe.y);
          if constexpr (LO) {
            // bf16 pair -> the two fp32 values it holds: exact bit moves
            const float2 hh = make_float2(__uint_as_float(hi[e] << 16),
                                          __uint_as_float(hi[e] & 0xffff0000u));
            lo[e] = pack_pair<T>(pe.x - hh.x, pe.y - hh.y);
          }
        }
        const uint32_t col = 32 * (g >> 2) + 4 * (g & 3);  // within this half's 64 columns
        tc::tmem_st4(tS + col, hi);
        if constexpr (LO) tc::tmem_st4(tS + col + 16, lo);
      }
      if (r == 0) PA_TRACE(12 + t * 2 + hw, j);
      // The product of the previous key tile has completed (the commit that
      // released these scores covers it): rescale this half's output columns
      // of the rows whose max moved.
      if (j > 0 && __any_sync(kFullMask, grow)) {
#pragma unroll 1
        for (int c4 = 0; c4 < HD / 32; ++c4) {
          uint32_t u[32];
          tc::tmem_ld32(tO + c4 * 32, u);
          tc::tmem_wait_ld();
#pragma unroll
          for (int c = 0; c < 32; ++c) u[c] = __float_as_uint(__uint_as_float(u[c]) * alpha);
          tc::tmem_st32(tO + c4 * 32, u);
        }
      }
      l = l * alpha + ((acc[0].x + acc[0].y) + (acc[1].x + acc[1].y));
      tc::tmem_wait_st();
      tc::fence_before_sync();
      if (r == 0) PA_TRACE(16 + t * 2 + hw, j);
      mbar_arrive(&p_full[t]);
    }
    // epilogue: the row's sum over both halves, then O / l -> out (this half's columns)
    if (ok) {
      slot(nk[t], hw)[r] = l;
      mbar_arrive(&xch_bar[t]);
      ok = wait_warp(&xch_bar[t], nk[t] & 1, abort_flag);
    }
    if (ok) ok = wait_warp(&o_done[t], 0, abort_flag);
    if (ok) {
      tc::fence_after_sync();
      const float inv = 1.f / (l + slot(nk[t], hw ^ 1)[r]);
      TO* dst = reinterpret_cast<TO*>(p.out) + (static_cast<int64_t>(q0 + qrow) * p.H + h) * D + hw * HD;
#pragma unroll
      for (int c4 = 0; c4 < HD / 32; ++c4) {
        uint32_t u[32];
        tc::tmem_ld32(tO + c4 * 32, u);
        tc::tmem_wait_ld();
        float v[32];
#pragma unroll
        for (int c = 0; c < 32; ++c) v[c] = __uint_as_float(u[c]) * inv;
        if (qrow < n) store_row32<TO>(dst + c4 * 32, v);
      }
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (threadIdx.x == 0) PA_TRACE(30, 0);
  if (warp == kIssuer) {
    __syncwarp();
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, Tl::TMEM_COLS);
  }
}

}  // namespace pa
