// Grouped-query decode on the tensor cores (paged_decode_gqa_kernel).
//
// What it computes: the decode of pa_decode ("vLLM KV Cache and PagedAttention
// Explained", Appendix) with H query heads sharing Hkv KV heads, query head h
// reading KV head h / (H / Hkv). With G query heads per KV head a unit of 16
// tokens is a small dense contraction, so it runs on the tensor cores. One CTA
// per (partition, KV head, request, chunk of up to 16 query heads):
//   * a producer warp loads each unit's 16 K rows and 16 V rows with tiled TMA
//     copies through tensor maps that view each cache as a 2-D array of
//     D-element rows (row (block * Hkv + head) * S + offset): boxes of 64
//     elements x 16 rows (two boxes of 8 rows from two blocks when S = 8) with
//     the 128-byte swizzle, one lane per box; an NS-stage ring with full /
//     empty barriers, all waits bounded;
//   * NC consumer warps take the units in turn (unit u to warp u % NC, two
//     stages each) and work them transposed -- tokens as the MMA rows, query
//     heads as 8-wide columns -- with mma.sync m16n8k16 (fp32 accumulate):
//     S^T = K Q^T (K by ldmatrix, Q^T kept in registers or in a shared tile),
//     the online softmax per head column (base 2), P^T into the B-operand
//     layout by movmatrix, O^T += V^T P^T (V^T by ldmatrix.trans), P as a
//     16-bit hi + lo pair for bf16; masked tokens are removed by selection in
//     the scores and by zeroing their V^T columns;
//   * the consumers' (m, l, O) merge through shared memory at the end; a
//     single-partition request writes its output, otherwise the partials go to
//     the split-KV workspace for splitkv_reduce_kernel.
#pragma once

#include "pa_decode.cuh"

namespace pa {

template <int D, int EB = 2>
struct GqaTiling {
  static constexpr int ROWS = 16;               // tokens per unit = one MMA k-step of P V
  static constexpr int BOX = 16 * 128;          // one swizzled box: 16 rows x 64 elements
  static constexpr int TILE16 = (D / 64) * BOX; // one K (or V) unit of 16-bit elements
  // as staged: 16-bit tiles as above; E4M3 tiles as 16 unswizzled D-byte rows
  static constexpr int TILE = EB == 2 ? TILE16 : ROWS * D;
  static constexpr int STAGE = 2 * TILE;
  static constexpr int NC = 3;                  // consumer warps; unit u goes to warp u % NC
  static constexpr int NS = 2 * NC;             // two stages per consumer
  // Consumer w takes units w, w + NC, ...; a stage is reused every NS units, so
  // with NS a multiple of NC each stage's units belong to one consumer and it
  // never waits on a stage phase two ahead (which a parity wait cannot tell apart).
  static_assert(NS % NC == 0, "stages must be a multiple of the consumer count");
  static constexpr int SMEM_MERGE = NC * ROWS * (D + 2) * 4;  // reuses the stages at the end
  static constexpr int SMEM_STAGES = NS * STAGE > SMEM_MERGE ? NS * STAGE : SMEM_MERGE;
  // E4M3: each consumer's unit converted to 16-bit K and V tiles (swizzled as
  // TMA would have written them, so the MMA path reads them unchanged)
  static constexpr int SMEM_CONV = EB == 1 ? NC * 2 * TILE16 : 0;
  // + 1024: the stages start on a 1024-byte boundary (the swizzle period)
  static constexpr int QPITCH = (D + 8) * 2;    // the Q tile (when Q is not kept in registers)
  static constexpr int SMEM_Q = ROWS * QPITCH;
  static constexpr int SMEM = 1024 + SMEM_STAGES + SMEM_CONV + SMEM_Q + 2 * NS * 8 + NS * 4;
  static_assert(SMEM_STAGES % 128 == 0, "the converted tiles start on a 128-byte boundary");
};

// The power-of-two exponent qe that brings a query row whose largest magnitude
// is mx below 2^15 (mx * 2^qe < 2^15, clamped to [-100, 100]; 0 for a zero or
// non-finite row): the row times 2^qe then fits f16, exactly up to f16's
// rounding, and the score is divided by 2^qe again.
__device__ __forceinline__ int q_exponent(float mx) {
  int e = 0;
  if (!(mx > 0.f && mx < INFINITY)) return 0;
  frexpf(mx, &e);  // mx = f * 2^e, f in [0.5, 1)
  return max(-100, min(100, 15 - e));
}

// Byte offset of 16-byte chunk cc (0 .. D/8 - 1) of row r (0 .. 15) in a unit tile
// of D/64 boxes, each 16 rows x 128 bytes with the 128-byte swizzle (chunk c of
// row r stored at chunk c ^ (r % 8)).
__device__ __forceinline__ int swz(int r, int cc) {
  return (cc >> 3) * 2048 + r * 128 + (((cc & 7) ^ (r & 7)) << 4);
}

template <typename T>
__device__ __forceinline__ void mma16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1);
template <>
__device__ __forceinline__ void mma16816<__nv_bfloat16>(float (&d)[4], const uint32_t (&a)[4],
                                                        uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
template <>
__device__ __forceinline__ void mma16816<__half>(float (&d)[4], const uint32_t (&a)[4],
                                                 uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}

// Transpose of an 8x8 matrix of 16-bit values held one packed pair per lane in
// the accumulator layout (lane 4g + t: row g, columns 2t, 2t + 1).
__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// Two fp32 -> a packed pair of 16-bit values (low half = first), round to nearest.
template <typename T>
__device__ __forceinline__ uint32_t pack2(float lo, float hi);
template <>
__device__ __forceinline__ uint32_t pack2<__nv_bfloat16>(float lo, float hi) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}
template <>
__device__ __forceinline__ uint32_t pack2<__half>(float lo, float hi) {
  const __half2 v = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&v);
}
// The fp32 value of the low / high 16-bit half of a packed pair.
template <typename T>
__device__ __forceinline__ float2 unpack2(uint32_t x) {
  return Elem<T>::pair(x);
}

// TC: the cache element type, T or E4M3 codes (per-tensor scales: K's folded
// into q_scale, V's applied to the output). Over E4M3 the consumers convert
// each staged unit to f16 tiles and the products run in f16 (E4M3 values are
// f16 values), with q held in f16 after an exact power-of-two scaling per head.
template <typename T, typename TO, int D, int S, bool APPEND, int NHT, typename TC = T>
__global__ void __launch_bounds__((GqaTiling<D, sizeof(TC)>::NC + 1) * 32)
    paged_decode_gqa_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmk,
                            const __grid_constant__ CUtensorMap tmv) {
  constexpr int EB = sizeof(TC);
  static_assert(!APPEND || EB == 2, "no fused append over E4M3 caches here");
  using TM = typename std::conditional<EB == 1, __half, T>::type;  // the MMA operand type
  using Tg = GqaTiling<D, EB>;
  constexpr int ROWS = Tg::ROWS, TILE = Tg::TILE, STAGE = Tg::STAGE;
  constexpr int NS = Tg::NS, NC = Tg::NC;
  constexpr int BR = S < 16 ? S : 16;  // rows per box
  constexpr int SLAB = S * D * EB;
  constexpr int KS = D / 16;  // k-steps of S

  grid_dependents_launch();  // the merge of split requests may be scheduled early
  const int part = blockIdx.x;
  const int G = p.H / p.Hkv;
  const int chunks = (G + 15) / 16;
  const int hk = blockIdx.y / chunks;
  const int c0 = (blockIdx.y % chunks) * 16;  // first query head (within the group) of this CTA
  const int gc = min(16, G - c0);             // query heads served here
  const int i = blockIdx.z;
  const int lane = threadIdx.x & 31;
  const int w = threadIdx.x >> 5;

  // The producer's first table entries assume a whole partition (P / S
  // blocks, clipped to the table's row), so they are requested together with
  // the length; a request's last, partial partition loads them again.
  const int t_beg = part * p.P;
  const int blk0 = t_beg / S;
  const int32_t* trow = p.block_tables + static_cast<int64_t>(i) * p.MB;
  int ids_a = -1, ids_b = -1;
  auto load_ids = [&](int blk1) {
    const int lim = min(blk1, p.MB);
    ids_a = (blk0 + lane < lim) ? __ldg(trow + blk0 + lane) : -1;
    ids_b = (blk0 + 32 + lane < lim) ? __ldg(trow + blk0 + 32 + lane) : -1;
  };
  if (w == NC) load_ids(blk0 + p.P / S);
  int L = __ldg(p.seq_lens + i);
  const bool len_ok = L >= 0 && L <= p.L_cap;
  if (!len_ok) {
    if (threadIdx.x == 0 && part == 0 && blockIdx.y == 0) raise_error(PA_DEVERR_SEQ_LEN);
    L = L < 0 ? 0 : p.L_cap;
  }
  const int nparts = (L + p.P - 1) / p.P;
  if (part > 0 && part >= nparts) return;
  const bool direct = nparts <= 1;

  extern __shared__ __align__(128) uint8_t smem_raw[];
  uint8_t* stages = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint8_t* conv = stages + Tg::SMEM_STAGES;  // E4M3: [NC][K, V] 16-bit tiles
  uint8_t* qtile = conv + Tg::SMEM_CONV;
  uint64_t* full = reinterpret_cast<uint64_t*>(qtile + Tg::SMEM_Q);
  uint64_t* empty = full + NS;
  uint32_t* rowmask = reinterpret_cast<uint32_t*>(empty + NS);  // per stage: rows copied
  if (threadIdx.x == 0) {
#pragma unroll
    for (int k = 0; k < NS; ++k) {
      mbar_init(&full[k], 1);
      mbar_init(&empty[k], 1);
    }
    fence_mbar_init();
  }
  __syncthreads();

  const int t_end = min(t_beg + p.P, L);
  const int nunits = t_end > t_beg ? (t_end - t_beg + ROWS - 1) / ROWS : 0;
  const int64_t block_stride = static_cast<int64_t>(p.Hkv) * SLAB;
  const uint8_t* kbase = static_cast<const uint8_t*>(p.k_cache) + static_cast<int64_t>(hk) * SLAB;
  const uint8_t* vbase = static_cast<const uint8_t*>(p.v_cache) + static_cast<int64_t>(hk) * SLAB;

  if (w == NC) {
    // ---- producer: one lane per box of a unit issues the loads ----
    const uint64_t policy = policy_evict_first();
    const int blk1 = t_end > t_beg ? (t_end + S - 1) / S : blk0;
    if (t_end < t_beg + p.P) load_ids(blk1);  // the last partition: its own run
    int base = 0;
    for (int u = 0; u < nunits; ++u) {
      const int s = u % NS;
      // every lane waits; the warp leaves together if any lane gave up
      if (u >= NS && !__all_sync(kFullMask, mbar_wait_bounded(&empty[s], ((u / NS) - 1) & 1))) {
        if (lane == 0) raise_error(PA_DEVERR_TIMEOUT);
        break;
      }
      const int t0 = t_beg + u * ROWS;
      if (t0 / S - blk0 >= base + 32) {  // slide the id window (a unit spans <= 2 blocks)
        base += 32;
        ids_a = ids_b;
        const int nx = blk0 + base + 32 + lane;
        ids_b = nx < blk1 ? __ldg(trow + nx) : -1;
      }
      const int rel = t0 / S - blk0 - base;  // 0 .. 31
      const int id0 = __shfl_sync(kFullMask, ids_a, rel);
      const int id1a = __shfl_sync(kFullMask, ids_a, (rel + 1) & 31);
      const int id1b = __shfl_sync(kFullMask, ids_b, (rel + 1) & 31);
      // the unit's rows in one box group (S >= 16) or two (S = 8); every lane
      // works out the plan, lane 0 arms the barrier, then one lane per box
      // issues it, so a unit's boxes go out in parallel
      uint32_t okmask = 0, bytes = 0;
      int rows_y[2] = {0, 0};
      bool issue[2] = {false, false};
      constexpr int NH = ROWS / BR;
#pragma unroll
      for (int hh = 0; hh < NH; ++hh) {
        const int th = t0 + hh * BR;
        if (th >= t_end) continue;
        const int id = hh == 0 ? id0 : (rel + 1 < 32 ? id1a : id1b);
        if (static_cast<unsigned>(id) >= static_cast<unsigned>(p.NB)) {
          if (lane == 0) raise_error(PA_DEVERR_BLOCK_ID);
          continue;
        }
        issue[hh] = true;
        rows_y[hh] = (id * p.Hkv + hk) * S + th % S;
        const int nrow = min(BR, t_end - th);
        okmask |= ((1u << nrow) - 1u) << (hh * BR);
        bytes += 2u * BR * D * EB;
      }
      if (lane == 0) {
        rowmask[s] = okmask;
        mbar_arrive_expect_tx(&full[s], bytes);
      }
      __syncwarp();
      if constexpr (EB == 1) {
        // E4M3: one box per (row group, K or V), the rows' whole D bytes
        if (lane < NH * 2) {
          const int hh = lane >> 1, kv = lane & 1;
          if (issue[hh]) {
            uint8_t* dst = stages + s * STAGE + hh * BR * D + kv * TILE;
            tma_load_2d(dst, kv ? &tmv : &tmk, 0, rows_y[hh], &full[s], policy);
          }
        }
      } else {
        constexpr int NBOX = NH * (D / 64) * 2;  // (row group, column block, K or V)
        if (lane < NBOX) {
          const int hh = lane / ((D / 64) * 2), c = (lane >> 1) % (D / 64), kv = lane & 1;
          if (issue[hh]) {
            uint8_t* dst = stages + s * STAGE + c * Tg::BOX + hh * BR * 128 + kv * TILE;
            tma_load_2d(dst, kv ? &tmv : &tmk, c * 64, rows_y[hh], &full[s], policy);
          }
        }
      }
      __syncwarp();
    }
    return;
  }

  // ---- consumers ----
  // The unit is worked transposed, tokens as the MMA rows and query heads as
  // its 8-wide columns, so a group of G <= 8 heads fills the columns instead of
  // padding 16 rows:  S^T[16 tok x 8 heads] = K[16 x D] . Q^T;  then
  // O^T[D x 8 heads] += V^T[D x 16 tok] . P^T.
  const int g = lane >> 2;  // accumulator row (token g and g + 8; d rows of O^T)
  const int t = lane & 3;   // accumulator column pair (heads 2t, 2t + 1 of a column tile)
  // Q^T as the B operand: head (column) g of column tile nt, elements 2t, 2t + 1
  // (b0) and 2t + 8, 2t + 9 (b1) of each k-step. Small groups keep it in
  // registers, loaded once from global memory; otherwise it is a shared tile
  // (rows = heads, zero past gc) read with ldmatrix at every k-step.
  constexpr bool QREG = NHT * KS <= 8;
  uint32_t qb[QREG ? NHT : 1][QREG ? KS : 1][2];
  float qdown[NHT];  // E4M3, Q in registers: 2^-qe of head 8 nt + g
#pragma unroll
  for (int nt = 0; nt < NHT; ++nt) qdown[nt] = 1.f;
  if constexpr (QREG) {
#pragma unroll
    for (int nt = 0; nt < NHT; ++nt) {
      const int row = 8 * nt + g;
      const uint32_t* qrow = reinterpret_cast<const uint32_t*>(
          static_cast<const uint8_t*>(p.q) +
          ((static_cast<int64_t>(i) * p.H + static_cast<int64_t>(hk) * G + c0 +
            min(row, gc - 1)) * D) * 2);
#pragma unroll
      for (int kk = 0; kk < KS; ++kk) {
        qb[nt][kk][0] = row < gc ? __ldg(qrow + kk * 8 + t) : 0u;
        qb[nt][kk][1] = row < gc ? __ldg(qrow + kk * 8 + 4 + t) : 0u;
      }
      if constexpr (EB == 1) {
        // f16 operands: head row's q times 2^qe, its largest element below 2^15
        // (the four lanes t of head g hold the row between them)
        float mx = 0.f;
#pragma unroll
        for (int kk = 0; kk < KS; ++kk)
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const float2 f = unpack2<T>(qb[nt][kk][j]);
            mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
          }
        mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, 2));
        const int qe = q_exponent(mx);
        const float up = ldexpf(1.f, qe);
        qdown[nt] = ldexpf(1.f, -qe);
#pragma unroll
        for (int kk = 0; kk < KS; ++kk)
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            const float2 f = unpack2<T>(qb[nt][kk][j]);
            qb[nt][kk][j] = pack2<__half>(f.x * up, f.y * up);
          }
      }
    }
  } else if constexpr (EB == 1) {
    // the Q tile in f16: 8 threads per head row, each with D / 64 chunks; the
    // row's scale exponent over the 8 (one warp's 8 consecutive lanes), its
    // 2^-qe kept in the row's padding. A warp's four rows of a pass are all in
    // the tile or all past it, so the shuffles see whole warps.
    static_assert(ROWS % 4 == 0, "four head rows per warp and pass");
    const int sub = threadIdx.x & 7;
    constexpr int QC = D / 64;
    for (int row = threadIdx.x >> 3; row < ROWS; row += NC * 4) {
      uint4 val[QC];
      float mx = 0.f;
#pragma unroll
      for (int c = 0; c < QC; ++c) {
        val[c] = make_uint4(0, 0, 0, 0);
        if (row < gc) {
          const int64_t hq = static_cast<int64_t>(hk) * G + c0 + row;
          val[c] = *reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.q) +
                                                   ((static_cast<int64_t>(i) * p.H + hq) * D +
                                                    (sub + 8 * c) * 8) * 2);
        }
        const uint32_t wv[4] = {val[c].x, val[c].y, val[c].z, val[c].w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = unpack2<T>(wv[j]);
          mx = fmaxf(mx, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
      }
#pragma unroll
      for (int off = 1; off < 8; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, off));
      const int qe = q_exponent(mx);
      const float up = ldexpf(1.f, qe);
#pragma unroll
      for (int c = 0; c < QC; ++c) {
        const uint32_t wv[4] = {val[c].x, val[c].y, val[c].z, val[c].w};
        uint32_t hv[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = unpack2<T>(wv[j]);
          hv[j] = pack2<__half>(f.x * up, f.y * up);
        }
        *reinterpret_cast<uint4*>(qtile + row * Tg::QPITCH + (sub + 8 * c) * 16) =
            make_uint4(hv[0], hv[1], hv[2], hv[3]);
      }
      if (sub == 0) *reinterpret_cast<float*>(qtile + row * Tg::QPITCH + D * 2) = ldexpf(1.f, -qe);
    }
    // consumers only: the Q tile is complete before anyone reads it
    asm volatile("bar.sync 1, %0;" ::"n"(NC * 32) : "memory");
  } else {
    for (int idx = threadIdx.x; idx < ROWS * (D / 8); idx += NC * 32) {
      const int row = idx / (D / 8), ch = idx % (D / 8);
      uint4 val = make_uint4(0, 0, 0, 0);
      if (row < gc) {
        const int64_t hq = static_cast<int64_t>(hk) * G + c0 + row;
        val = *reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.q) +
                                              ((static_cast<int64_t>(i) * p.H + hq) * D + ch * 8) * 2);
      }
      *reinterpret_cast<uint4*>(qtile + row * Tg::QPITCH + ch * 16) = val;
    }
    // consumers only: the Q tile is complete before anyone reads it
    asm volatile("bar.sync 1, %0;" ::"n"(NC * 32) : "memory");
  }
  // ldmatrix lane address into the Q tile: head (lane & 7) + 8 (lane >> 4),
  // 8-column half (lane >> 3) & 1 -> r0, r1 = b0, b1 of heads 0-7, r2, r3 of 8-15
  const int q_row = (lane & 7) + 8 * (lane >> 4), q_c8 = ((lane >> 3) & 1) * 8;
  // fused append: the new token's rows, one 16-byte chunk per lane; the warp
  // that consumes the new token's unit patches them in
  const int t_new = L - 1;
  const bool has_new = APPEND && len_ok && L >= 1 && t_new >= t_beg && t_new < t_end &&
                       ((t_new - t_beg) / ROWS) % NC == w;
  uint4 k_chunk = make_uint4(0, 0, 0, 0), v_chunk = make_uint4(0, 0, 0, 0);
  const bool chunk_lane = lane < D / 8;
  if (has_new && chunk_lane) {
    const int64_t off = ((static_cast<int64_t>(i) * p.Hkv + hk) * D + lane * 8) * 2;
    k_chunk = *reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.k_new) + off);
    v_chunk = *reinterpret_cast<const uint4*>(static_cast<const uint8_t*>(p.v_new) + off);
    if (c0 == 0) {  // one CTA per KV head stores the row to the cache
      const int id_new = __ldg(trow + t_new / S);
      if (static_cast<unsigned>(id_new) < static_cast<unsigned>(p.NB)) {
        const int64_t goff = static_cast<int64_t>(id_new) * block_stride +
                             (static_cast<int64_t>(t_new % S) * D + lane * 8) * 2;
        *reinterpret_cast<uint4*>(const_cast<uint8_t*>(kbase) + goff) = k_chunk;
        *reinterpret_cast<uint4*>(const_cast<uint8_t*>(vbase) + goff) = v_chunk;
      }
    }
  }
  __syncwarp();

  constexpr int MT = D / 16;  // 16-row tiles of O^T
  float o[MT][NHT][4];
#pragma unroll
  for (int mt = 0; mt < MT; ++mt)
#pragma unroll
    for (int nt = 0; nt < NHT; ++nt) o[mt][nt][0] = o[mt][nt][1] = o[mt][nt][2] = o[mt][nt][3] = 0.f;
  float m[NHT][2], l[NHT][2];  // per head 8nt + 2t + e: running max (base 2), this lane's sum
#pragma unroll
  for (int nt = 0; nt < NHT; ++nt) m[nt][0] = m[nt][1] = -INFINITY, l[nt][0] = l[nt][1] = 0.f;
  // ldmatrix lane addresses into a token-major 16 x 16 tile, giving the A
  // fragment (rows g / g + 8, k halves 0-7 / 8-15 in r0 .. r3):
  //   K (rows = tokens):            token lane & 15, column half lane >> 4
  //   V^T via .trans (k = tokens):  token (lane & 7) + 8 (lane >> 4), d half (lane >> 3) & 1
  const int k_tok = lane & 15, k_c8 = (lane >> 4) * 8;
  const int v_tok = (lane & 7) + 8 * (lane >> 4), v_c8 = ((lane >> 3) & 1) * 8;

  // E4M3: the score multiplier of head 8 nt + 2t + c (q_scale and 2^-qe)
  float qs[NHT][2];
#pragma unroll
  for (int nt = 0; nt < NHT; ++nt)
#pragma unroll
    for (int c = 0; c < 2; ++c) {
      float down = 1.f;
      if constexpr (EB == 1) {
        if constexpr (QREG)
          down = __shfl_sync(kFullMask, qdown[nt], 4 * (2 * t + c));
        else
          down = *reinterpret_cast<const float*>(qtile + (8 * nt + 2 * t + c) * Tg::QPITCH + D * 2);
      }
      qs[nt][c] = p.q_scale * down;
    }

  for (int k = w; k < nunits; k += NC) {
    const int s = k % NS;
    // every lane waits; the warp leaves together if any lane gave up
    if (!__all_sync(kFullMask, mbar_wait_bounded(&full[s], (k / NS) & 1))) {
      if (lane == 0) raise_error(PA_DEVERR_TIMEOUT);
      break;
    }
    uint8_t* ktile = stages + s * STAGE;
    uint8_t* vtile = ktile + TILE;
    const int t0 = t_beg + k * ROWS;
    uint32_t valid = rowmask[s];
    if constexpr (EB == 1) {
      // E4M3: this consumer converts the unit to f16 tiles of its own (16 codes
      // per chunk, two 16-byte chunks of f16 each), then frees the stage
      uint8_t* kc = conv + w * 2 * Tg::TILE16;
      uint8_t* vc = kc + Tg::TILE16;
#pragma unroll 1
      for (int idx = lane; idx < ROWS * D / 16; idx += 32) {
        const int r = idx / (D / 16), j = idx % (D / 16);
        uint32_t hk2[8], hv2[8];
        e4m3x16_to_h2(ktile + r * D + j * 16, hk2);
        e4m3x16_to_h2(vtile + r * D + j * 16, hv2);
        *reinterpret_cast<uint4*>(kc + swz(r, 2 * j)) = make_uint4(hk2[0], hk2[1], hk2[2], hk2[3]);
        *reinterpret_cast<uint4*>(kc + swz(r, 2 * j + 1)) = make_uint4(hk2[4], hk2[5], hk2[6], hk2[7]);
        *reinterpret_cast<uint4*>(vc + swz(r, 2 * j)) = make_uint4(hv2[0], hv2[1], hv2[2], hv2[3]);
        *reinterpret_cast<uint4*>(vc + swz(r, 2 * j + 1)) = make_uint4(hv2[4], hv2[5], hv2[6], hv2[7]);
      }
      __syncwarp();  // the tiles are written (and the staged codes read) by every lane
      if (lane == 0) mbar_arrive(&empty[s]);
      ktile = kc;
      vtile = vc;
    }
    if (has_new && t_new >= t0 && t_new < t0 + ROWS) {
      const int rnew = t_new - t0;
      if (chunk_lane) {
        *reinterpret_cast<uint4*>(ktile + swz(rnew, lane)) = k_chunk;
        *reinterpret_cast<uint4*>(vtile + swz(rnew, lane)) = v_chunk;
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
    }

    // S^T = K Q^T; even and odd k-steps in separate registers (two MMA chains)
    float sacc[NHT][4], sodd[NHT][4];
#pragma unroll
    for (int nt = 0; nt < NHT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[nt][e] = sodd[nt][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < KS; ++kk) {
      uint32_t a[4];
      ldsm_x4(a, ktile + swz(k_tok, (kk * 16 + k_c8) >> 3));
      if constexpr (QREG) {
#pragma unroll
        for (int nt = 0; nt < NHT; ++nt)
          mma16816<TM>((kk & 1) ? sodd[nt] : sacc[nt], a, qb[nt][kk][0], qb[nt][kk][1]);
      } else {
        uint32_t b[4];
        ldsm_x4(b, qtile + q_row * Tg::QPITCH + (kk * 16 + q_c8) * 2);
#pragma unroll
        for (int nt = 0; nt < NHT; ++nt)
          mma16816<TM>((kk & 1) ? sodd[nt] : sacc[nt], a, b[2 * nt], b[2 * nt + 1]);
      }
    }
    // scores (base 2), masked by selection: element e is token g + 8 (e >> 1),
    // head 8 nt + 2t + (e & 1)
    const bool tok_lo = (valid >> g) & 1u, tok_hi = (valid >> (g + 8)) & 1u;
    uint32_t bhi[NHT][2], blo[NHT][2];
    float al[NHT][2];
    bool any_rescale = false;
#pragma unroll
    for (int nt = 0; nt < NHT; ++nt) {
      float sc[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const bool ok = (e >> 1) ? tok_hi : tok_lo;
        if constexpr (EB == 1)
          sc[e] = ok ? (sacc[nt][e] + sodd[nt][e]) * qs[nt][e & 1] : -INFINITY;
        else
          sc[e] = ok ? (sacc[nt][e] + sodd[nt][e]) * p.q_scale : -INFINITY;
      }
      float pr[4];
#pragma unroll
      for (int c = 0; c < 2; ++c) {  // head 8nt + 2t + c: max over the 16 tokens
        float mx = fmaxf(sc[c], sc[c + 2]);
#pragma unroll
        for (int off = 4; off <= 16; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, off));
        const float mn = fmaxf(m[nt][c], mx);
        // a unit with no valid token for this head keeps its max at -inf
        al[nt][c] = mn == -INFINITY ? 1.f : exp2f(m[nt][c] - mn);
        any_rescale |= al[nt][c] != 1.f;
        pr[c] = sc[c] == -INFINITY ? 0.f : exp2f(sc[c] - mn);
        pr[c + 2] = sc[c + 2] == -INFINITY ? 0.f : exp2f(sc[c + 2] - mn);
        l[nt][c] = l[nt][c] * al[nt][c] + pr[c] + pr[c + 2];
        m[nt][c] = mn;
      }
      // P^T as the B operand: tokens 2t, 2t + 1 (b0) and 2t + 8, 2t + 9 (b1) of
      // head g, by transposing the accumulator-layout pairs. bf16 keeps 8 bits,
      // so P goes in as a hi + lo pair (its rounding drops from 2^-9 to 2^-17);
      // fp16 keeps 11, within the tolerance on its own.
      const uint32_t h0 = pack2<TM>(pr[0], pr[1]), h1 = pack2<TM>(pr[2], pr[3]);
      bhi[nt][0] = movmatrix_trans(h0);
      bhi[nt][1] = movmatrix_trans(h1);
      if (std::is_same<TM, __nv_bfloat16>::value) {
        const float2 f0 = unpack2<TM>(h0), f1 = unpack2<TM>(h1);
        blo[nt][0] = movmatrix_trans(pack2<TM>(pr[0] - f0.x, pr[1] - f0.y));
        blo[nt][1] = movmatrix_trans(pack2<TM>(pr[2] - f1.x, pr[3] - f1.y));
      }
    }
    // once the running max settles most units move no head's max
    if (__any_sync(kFullMask, any_rescale)) {
#pragma unroll
      for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int nt = 0; nt < NHT; ++nt) {
          o[mt][nt][0] *= al[nt][0];
          o[mt][nt][1] *= al[nt][1];
          o[mt][nt][2] *= al[nt][0];
          o[mt][nt][3] *= al[nt][1];
        }
    }
    // V^T as the A operand (ldmatrix.trans of the token-major tile); tokens that
    // were not copied are zeroed in it (0 * NaN would be NaN)
    const bool partial = valid != 0xffffu;
    const uint32_t vm0 = (((valid >> (2 * t)) & 1u) ? 0x0000ffffu : 0u) |
                         (((valid >> (2 * t + 1)) & 1u) ? 0xffff0000u : 0u);
    const uint32_t vm1 = (((valid >> (2 * t + 8)) & 1u) ? 0x0000ffffu : 0u) |
                         (((valid >> (2 * t + 9)) & 1u) ? 0xffff0000u : 0u);
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) {
      uint32_t a[4];
      ldsm_x4_trans(a, vtile + swz(v_tok, (mt * 16 + v_c8) >> 3));
      if (partial) {
        a[0] &= vm0;
        a[1] &= vm0;
        a[2] &= vm1;
        a[3] &= vm1;
      }
#pragma unroll
      for (int nt = 0; nt < NHT; ++nt) {
        mma16816<TM>(o[mt][nt], a, bhi[nt][0], bhi[nt][1]);
        if (std::is_same<TM, __nv_bfloat16>::value)
          mma16816<TM>(o[mt][nt], a, blo[nt][0], blo[nt][1]);
      }
    }
    __syncwarp();
    if constexpr (EB == 2) {
      if (lane == 0) mbar_arrive(&empty[s]);  // (E4M3 freed its stage after converting)
    }
  }

  // head sums over the 8 lanes that share t
#pragma unroll
  for (int nt = 0; nt < NHT; ++nt)
#pragma unroll
    for (int c = 0; c < 2; ++c)
#pragma unroll
      for (int off = 4; off <= 16; off <<= 1)
        l[nt][c] += __shfl_xor_sync(kFullMask, l[nt][c], off);
  // merge the NC consumers' (m, l, O) per head through shared memory (the stages
  // are free: every unit has been consumed once all consumers pass the barrier)
  asm volatile("bar.sync 1, %0;" ::"n"(NC * 32) : "memory");
  float* mg = reinterpret_cast<float*>(stages);  // [NC][ROWS][D + 2]: m, l, O per head
  {
    float* mine = mg + w * ROWS * (D + 2);
#pragma unroll
    for (int nt = 0; nt < NHT; ++nt)
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        float* rowp = mine + (8 * nt + 2 * t + c) * (D + 2);
        if (g == 0) {
          rowp[0] = m[nt][c];
          rowp[1] = l[nt][c];
        }
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          rowp[2 + 16 * mt + g] = o[mt][nt][c];
          rowp[2 + 16 * mt + g + 8] = o[mt][nt][c + 2];
        }
      }
  }
  asm volatile("bar.sync 1, %0;" ::"n"(NC * 32) : "memory");
  // consumer w finishes heads w, w + NC, ...: M = max m, out = sum 2^(m - M) O / sum 2^(m - M) l
  for (int row = w; row < gc; row += NC) {
    float M = -INFINITY;
#pragma unroll
    for (int c = 0; c < NC; ++c) M = fmaxf(M, mg[(c * ROWS + row) * (D + 2)]);
    float wt[NC];
    float lsum = 0.f;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const float mc = mg[(c * ROWS + row) * (D + 2)];
      wt[c] = mc == -INFINITY ? 0.f : exp2f(mc - M);
      lsum = fmaf(wt[c], mg[(c * ROWS + row) * (D + 2) + 1], lsum);
    }
    const int64_t hq = static_cast<int64_t>(hk) * G + c0 + row;
    const int64_t ih = static_cast<int64_t>(i) * p.H + hq;
    for (int d = lane; d < D; d += 32) {
      float a = 0.f;
#pragma unroll
      for (int c = 0; c < NC; ++c) a = fmaf(wt[c], mg[(c * ROWS + row) * (D + 2) + 2 + d], a);
      if constexpr (EB == 1) a *= p.v_scale;
      if (direct) {
        static_cast<TO*>(p.out)[ih * D + d] = to_out<TO>(lsum > 0.f ? a / lsum : 0.f);
      } else {
        p.ws_acc[(ih * p.NP + part) * D + d] = a;
      }
    }
    if (!direct && lane == 0) {
      p.ws_m[ih * p.NP + part] = M;
      p.ws_l[ih * p.NP + part] = lsum;
    }
  }
}

}  // namespace pa
