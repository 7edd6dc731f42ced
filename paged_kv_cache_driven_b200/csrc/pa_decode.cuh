// Paged single-query decode attention for sm_100a: the partition pass and the
// log-sum-exp reduce.
//
// What it computes: "vLLM KV Cache and PagedAttention Explained", "Appendix:
// The Attention Score Formula" -- out = softmax(q K^T * scale) V. The paged form
// described there visits the request's physical blocks in table order; for
// each block it scores the block's keys against the query, rescales the
// running max and sum, and adds the block's weighted values into the
// accumulator. The blocks are read where they are
// ("PagedAttention" card, "Kernel은 무엇이 달라지는가"); long contexts are cut into
// partitions whose partial results a second kernel merges (FlashDecoding, the
// same card, "헷갈리기 쉬운 구분").
//
// Mapping onto the B200 (this is not the pages' shared-memory sketch, which
// names no hardware):
//   * one CTA per (partition, head, request); NW warps split the partition's
//     blocks into contiguous runs; each warp is an independent pipeline.
//   * a warp's block ids are hoisted 32 at a time with one coalesced load and
//     prefetched one chunk ahead, so the dependent table load never stalls
//     the copy stream.
//   * each physical block's K slab and V slab (S x D contiguous, the
//     [Block, Head, Block_Size, Head_D] layout) arrive in shared memory by two
//     1-D bulk async copies (cp.async.bulk, TMA engine, no tensor map needed)
//     on an mbarrier; NS stages per warp keep several blocks in flight.
//   * lane l owns D/32 consecutive elements of q, of every K/V row and of the
//     output accumulator. The S partial dot products of a block are summed
//     across lanes with a transposing butterfly: S values per lane become one
//     finished score per lane in S-1+log2(32/S) shuffles.
//   * the softmax runs in base 2 (q is pre-scaled by scale * log2 e) with an
//     fp32 running max / sum; masked tokens are removed by selection, never by
//     multiplying, so NaN in unused slots cannot leak.
//   * no tensor cores: one query per head is a matrix-vector product.
#pragma once

#include <cuda.h>

#include <type_traits>

#include "pa_device.cuh"

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
};

// Shapes of the partition pass for head_dim D and block_size S.
//   EPL = 8  elements per lane per row fragment (one 16-byte shared load)
//   LPR      lanes per row (D / 8: 8, 16 or 32); RPW = 32 / LPR rows per warp-wide load
//   CR       rows per pipeline unit: CR x D of K and of V (about 4 KB each) is one
//            stage, so the stage size no longer grows with S; a block of S rows
//            is S / CR units
//   NS, NW   stages per warp and warps per CTA: about 64 KB of stages per CTA
template <int D, int S>
struct DecodeTiling {
  static constexpr int EPL = 8;
  static constexpr int LPR = D / EPL;
  static constexpr int RPW = 32 / LPR;
  static constexpr int CR_RAW = 2048 / D;
  static constexpr int CR = CR_RAW < S ? CR_RAW : S;
  static constexpr int NV = CR / RPW;  // rows per lane per unit
  static constexpr int SLAB = S * D * 2;     // one (block, head) slab of K or of V
  static constexpr int UNIT = CR * D * 2;    // one unit of K or of V
  static constexpr int STAGE = 2 * UNIT;
  static constexpr int NS = STAGE <= 4096 ? 4 : 2;
  static constexpr int NW_RAW = 65536 / (NS * STAGE);
  static constexpr int NW = NW_RAW < 1 ? 1 : (NW_RAW > 8 ? 8 : NW_RAW);
  static constexpr int SMEM_PIPE = NW * NS * STAGE;
  static constexpr int SMEM_BARS = NW * NS * 8;
  static constexpr int SMEM_MERGE = NW * (D + 2) * 4;
  static constexpr int SMEM = SMEM_PIPE + SMEM_BARS + SMEM_MERGE;
  static_assert(S % CR == 0 && CR % RPW == 0 && NV >= 1 && NV <= LPR, "bad tiling");
  static_assert(UNIT % 16 == 0, "bulk copies move multiples of 16 bytes");
};

// Finishes NV per-lane partial dot products. Lane l of row group g = l / LPR
// holds, in v[k], its fragment's partial dot of row k * RPW + g. The lanes of a
// group exchange halves of their values (a transposing butterfly) so that each
// value is summed over the group in NV - 1 + log2(LPR / NV) shuffles. On return
// lane l holds the full dot of row (pl / DUP) * RPW + g, pl = l % LPR,
// DUP = LPR / NV; the DUP lanes pl = k * DUP .. k * DUP + DUP - 1 hold row k's.
template <int NV, int LPR>
__device__ __forceinline__ float transpose_reduce(float (&v)[NV], int lane) {
#pragma unroll
  for (int n = NV, off = LPR / 2; n > 1; n >>= 1, off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int j = 0; j < n / 2; ++j) {
      const float send = upper ? v[j] : v[j + n / 2];
      const float keep = upper ? v[j + n / 2] : v[j];
      v[j] = keep + __shfl_xor_sync(kFullMask, send, off);
    }
  }
  float r = v[0];
#pragma unroll
  for (int off = LPR / NV / 2; off >= 1; off >>= 1) r += __shfl_xor_sync(kFullMask, r, off);
  return r;
}

// Raw 16-bit row fragment of 8 elements (16 bytes) for copying K/V rows bit for bit.
struct RawFrag {
  uint4 w;
  __device__ __forceinline__ void load(const void* src) { w = *reinterpret_cast<const uint4*>(src); }
  __device__ __forceinline__ void store(void* dst) const { *reinterpret_cast<uint4*>(dst) = w; }
};

// One CTA per (partition, head, request); NW warps, each an independent
// pipeline over the tokens of a contiguous run of the partition's blocks,
// taken CR rows (one unit) at a time.
//
// APPEND = true fuses the decode step's append: for request i with L >= 1, the
// new token (position L - 1) takes its K/V from k_new / v_new. The warp whose
// run holds that token copies the row into its staged unit once the bulk copy
// has landed (so the scores see it) and stores it to the cache, as
// pa_kv_append would have before the decode.
template <typename T, typename TO, int D, int S, bool APPEND>
__global__ void __launch_bounds__(DecodeTiling<D, S>::NW * 32)
    paged_decode_partition_kernel(const DecodeParams p) {
  using Tl = DecodeTiling<D, S>;
  constexpr int NW = Tl::NW, NS = Tl::NS, SLAB = Tl::SLAB, UNIT = Tl::UNIT, STAGE = Tl::STAGE;
  constexpr int EPL = Tl::EPL, LPR = Tl::LPR, RPW = Tl::RPW, CR = Tl::CR, NV = Tl::NV;
  constexpr int DUP = LPR / NV;  // lanes of a group holding the same row's score

  const int part = blockIdx.x;
  const int h = blockIdx.y;
  const int i = blockIdx.z;
  const int lane = threadIdx.x & 31;
  const int w = threadIdx.x >> 5;
  const int g = lane / LPR;   // row group
  const int pl = lane % LPR;  // position in the row: elements pl * 8 .. pl * 8 + 7

  int L = __ldg(p.seq_lens + i);
  const bool len_ok = L >= 0 && L <= p.L_cap;
  if (!len_ok) {
    if (threadIdx.x == 0 && part == 0 && h == 0) raise_error(PA_DEVERR_SEQ_LEN);
    L = L < 0 ? 0 : p.L_cap;
  }
  const int nparts = (L + p.P - 1) / p.P;
  if (part > 0 && part >= nparts) return;  // nothing here (part 0 writes the L == 0 zeros)
  const bool direct = nparts <= 1;          // the only partition: write the final output

  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Tl::SMEM_PIPE);
  float* merge = reinterpret_cast<float*>(smem + Tl::SMEM_PIPE + Tl::SMEM_BARS);

  if (threadIdx.x == 0) {
#pragma unroll
    for (int k = 0; k < NW * NS; ++k) mbar_init(&bars[k], 1);
    fence_mbar_init();
  }
  __syncthreads();

  // This partition's blocks, split into NW contiguous runs; a warp's tokens are
  // [wb * S, min(we * S, L)), taken CR at a time (units; none is wholly past L).
  const int t_beg = part * p.P;
  const int t_end = min(t_beg + p.P, L);
  const int blk_beg = t_beg / S;
  const int blk_end = t_end > t_beg ? (t_end + S - 1) / S : blk_beg;
  const int nb = blk_end - blk_beg;
  const int wb = blk_beg + static_cast<int>((static_cast<int64_t>(nb) * w) / NW);
  const int we = blk_beg + static_cast<int>((static_cast<int64_t>(nb) * (w + 1)) / NW);
  const int wt0 = wb * S;
  const int wt1 = min(we * S, L);
  const int nunits = wt1 > wt0 ? (wt1 - wt0 + CR - 1) / CR : 0;

  // q fragment, pre-scaled so that scores come out in base-2 units.
  float qf[EPL];
  {
    const T* qp = static_cast<const T*>(p.q) + (static_cast<int64_t>(i) * p.H + h) * D + pl * EPL;
    load_row<T, EPL>(qp, qf);
#pragma unroll
    for (int e = 0; e < EPL; ++e) qf[e] *= p.q_scale;
  }

  uint64_t* bar = bars + w * NS;
  uint8_t* stage0 = smem + w * NS * STAGE;
  const int32_t* trow = p.block_tables + static_cast<int64_t>(i) * p.MB;
  const int hk = h / (p.H / p.Hkv);  // this query head's KV head
  const uint8_t* kbase = static_cast<const uint8_t*>(p.k_cache) + static_cast<int64_t>(hk) * SLAB;
  const uint8_t* vbase = static_cast<const uint8_t*>(p.v_cache) + static_cast<int64_t>(hk) * SLAB;
  const int64_t block_stride = static_cast<int64_t>(p.Hkv) * SLAB;  // bytes per physical block
  const uint64_t policy = policy_evict_first();

  // Fused append: does this warp own the new token?
  const int t_new = L - 1;
  // (a clamped, out-of-range length appends nothing: its position is unknown)
  const bool appender = APPEND && len_ok && L >= 1 && t_new >= wt0 && t_new < wt1;
  RawFrag k_row, v_row;
  int id_new = -1;
  if (appender && g == 0) {
    const int64_t off = ((static_cast<int64_t>(i) * p.Hkv + hk) * D + pl * EPL) * 2;
    k_row.load(static_cast<const uint8_t*>(p.k_new) + off);
    v_row.load(static_cast<const uint8_t*>(p.v_new) + off);
    id_new = __ldg(trow + t_new / S);
  }

  // Block-id prefetch: ids_a holds the table entries of blocks wb + base .. +31,
  // ids_b the next 32.
  int base = 0;
  int ids_a = (wb + lane < we) ? __ldg(trow + wb + lane) : -1;
  int ids_b = (wb + 32 + lane < we) ? __ldg(trow + wb + 32 + lane) : -1;
  uint32_t bad = 0;  // bit s: stage s holds a unit whose block id was out of range
  int issued = 0;

  auto issue_next = [&]() {
    if (issued >= nunits) return;
    const int t0 = wt0 + issued * CR;       // first token of the unit
    const int rb = t0 / S - wb;             // block, relative to the warp's run
    if (rb >= base + 32) {
      base += 32;
      ids_a = ids_b;
      const int nx = wb + base + 32 + lane;
      ids_b = nx < we ? __ldg(trow + nx) : -1;
    }
    const int id = __shfl_sync(kFullMask, ids_a, rb - base);
    const int s = issued % NS;
    const bool ok = static_cast<unsigned>(id) < static_cast<unsigned>(p.NB);
    if (lane == 0) {
      if (ok) {
        mbar_arrive_expect_tx(&bar[s], 2 * UNIT);
        const int64_t off = static_cast<int64_t>(id) * block_stride +
                            static_cast<int64_t>(t0 % S) * D * 2;
        bulk_g2s(stage0 + s * STAGE, kbase + off, UNIT, &bar[s], policy);
        bulk_g2s(stage0 + s * STAGE + UNIT, vbase + off, UNIT, &bar[s], policy);
      } else {
        raise_error(PA_DEVERR_BLOCK_ID);
        mbar_arrive(&bar[s]);  // completes the phase with no data; the unit is skipped
      }
    }
    bad = ok ? (bad & ~(1u << s)) : (bad | (1u << s));
    ++issued;
  };

#pragma unroll
  for (int k = 0; k < NS; ++k) issue_next();

  float m = -INFINITY;  // running max (base-2 units), warp-uniform
  float lsum = 0.f;     // running sum of 2^(s - m); one lane per row counts it
  float acc[EPL];       // this lane's fragment, over the rows of its group
#pragma unroll
  for (int e = 0; e < EPL; ++e) acc[e] = 0.f;
  const int my_row = (pl / DUP) * RPW + g;  // the row whose score this lane ends with

  for (int k = 0; k < nunits; ++k) {
    const int s = k % NS;
    if (!mbar_wait_bounded(&bar[s], (k / NS) & 1)) {
      if (lane == 0) raise_error(PA_DEVERR_TIMEOUT);
      // drain what this warp still has in flight (bounded), then stop
      for (int r = k; r < issued; ++r) mbar_wait_bounded(&bar[r % NS], (r / NS) & 1);
      break;
    }
    if (!((bad >> s) & 1u)) {
      const int t0 = wt0 + k * CR;
      const int nvalid = min(CR, L - t0);
      uint8_t* ks = stage0 + s * STAGE;
      uint8_t* vs = ks + UNIT;
      if (APPEND && appender && t_new >= t0 && t_new < t0 + CR) {
        // the bulk copy brought the old bytes; put the new token's row in both
        // the staged unit and the cache
        if (g == 0) {
          const int64_t row_off = (static_cast<int64_t>(t_new - t0) * D + pl * EPL) * 2;
          k_row.store(ks + row_off);
          v_row.store(vs + row_off);
          const int64_t goff = static_cast<int64_t>(id_new) * block_stride +
                               (static_cast<int64_t>(t_new % S) * D + pl * EPL) * 2;
          k_row.store(const_cast<uint8_t*>(kbase) + goff);
          v_row.store(const_cast<uint8_t*>(vbase) + goff);
          // these generic-proxy writes must be ordered before the next bulk
          // copy (async proxy) that reuses this stage
          asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
        }
        __syncwarp();
      }

      float dot[NV];
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        float kf[EPL];
        load_row<T, EPL>(ks + ((v * RPW + g) * D + pl * EPL) * 2, kf);
        float a = 0.f;
#pragma unroll
        for (int e = 0; e < EPL; ++e) a = fmaf(qf[e], kf[e], a);
        dot[v] = a;
      }
      const float score = transpose_reduce<NV, LPR>(dot, lane);
      const bool valid = my_row < nvalid;
      const float sc = valid ? score : -INFINITY;
      float mb = sc;
#pragma unroll
      for (int off = DUP; off < 32; off <<= 1) mb = fmaxf(mb, __shfl_xor_sync(kFullMask, mb, off));
      const float m_new = fmaxf(m, mb);
      const float alpha = exp2f(m - m_new);
      const float pr = valid ? exp2f(sc - m_new) : 0.f;
      lsum = lsum * alpha + ((pl % DUP) == 0 ? pr : 0.f);
#pragma unroll
      for (int e = 0; e < EPL; ++e) acc[e] *= alpha;
      if (nvalid == CR) {
#pragma unroll
        for (int v = 0; v < NV; ++v) {
          const float pv = __shfl_sync(kFullMask, pr, g * LPR + v * DUP);
          float vf[EPL];
          load_row<T, EPL>(vs + ((v * RPW + g) * D + pl * EPL) * 2, vf);
#pragma unroll
          for (int e = 0; e < EPL; ++e) acc[e] = fmaf(pv, vf[e], acc[e]);
        }
      } else {
        // the request's last unit: rows past nvalid may hold anything (NaN);
        // they are left out by selection, never multiplied by zero
#pragma unroll
        for (int v = 0; v < NV; ++v) {
          if (v * RPW < nvalid) {  // warp-uniform
            const float pv = __shfl_sync(kFullMask, pr, g * LPR + v * DUP);
            const bool row_ok = v * RPW + g < nvalid;
            float vf[EPL];
            load_row<T, EPL>(vs + ((v * RPW + g) * D + pl * EPL) * 2, vf);
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[e] = row_ok ? fmaf(pv, vf[e], acc[e]) : acc[e];
          }
        }
      }
      m = m_new;
    }
    __syncwarp();
    issue_next();
  }

#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) lsum += __shfl_xor_sync(kFullMask, lsum, off);
  // the row groups accumulated disjoint rows of the same fragment: add them up
#pragma unroll
  for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc[e] += __shfl_xor_sync(kFullMask, acc[e], off);
  }

  // Merge the NW warps' (m, l, acc) in shared memory.
  float* m_s = merge;
  float* l_s = merge + NW;
  float* acc_s = merge + 2 * NW;
  if (g == 0) {
#pragma unroll
    for (int e = 0; e < EPL; ++e) acc_s[w * D + pl * EPL + e] = acc[e];
  }
  if (lane == 0) {
    m_s[w] = m;
    l_s[w] = lsum;
  }
  __syncthreads();

  float M = -INFINITY;
#pragma unroll
  for (int u = 0; u < NW; ++u) M = fmaxf(M, m_s[u]);
  float wgt[NW];
  float Ltot = 0.f;
#pragma unroll
  for (int u = 0; u < NW; ++u) {
    wgt[u] = m_s[u] == -INFINITY ? 0.f : exp2f(m_s[u] - M);
    Ltot = fmaf(wgt[u], l_s[u], Ltot);
  }
  const int64_t ih = static_cast<int64_t>(i) * p.H + h;
  for (int d = threadIdx.x; d < D; d += NW * 32) {
    float a = 0.f;
#pragma unroll
    for (int u = 0; u < NW; ++u) a = fmaf(wgt[u], acc_s[u * D + d], a);
    if (direct) {
      const float o = Ltot > 0.f ? a / Ltot : 0.f;
      static_cast<TO*>(p.out)[ih * D + d] = to_out<TO>(o);
    } else {
      p.ws_acc[(ih * p.NP + part) * D + d] = a;
    }
  }
  if (!direct && threadIdx.x == 0) {
    p.ws_m[ih * p.NP + part] = M;
    p.ws_l[ih * p.NP + part] = Ltot;
  }
}

// ---------------------------------------------------------------------------
// Grouped-query decode on the tensor cores.
//
// With G query heads per KV head, a unit of 16 tokens is a small dense
// contraction: S = Q K^T with Q [G x D] and K [16 x D], then O += P V with
// V [16 x D]. One CTA per (partition, KV head, request, chunk of up to 16 query
// heads) has two warps:
//   * the producer loads each unit's 16 K rows and 16 V rows with tiled TMA
//     copies through tensor maps that view each cache as a 2-D array of
//     D-element rows (row (block * Hkv + head) * S + offset): boxes of 64
//     elements x 16 rows (two boxes of 8 rows from two blocks when S = 8), with
//     the 128-byte swizzle, so that the 8 rows an ldmatrix reads fall in 8
//     different bank groups; D / 64 boxes per tile, an NS-stage ring with full /
//     empty barriers, all waits bounded;
//   * NC consumer warps take the units in turn (unit u to warp u % NC, two
//     stages each), each keeping its own running (m, l, O), merged through
//     shared memory at the end; several warps per SM hide the latency of the
//     MMA / softmax dependency chain of one unit. Each consumer keeps Q (rows
//     >= G zero) in shared memory and runs, per unit,
//     mma.sync m16n8k16 (fp32 accumulate): S over D/16 k-steps for the two 8-token
//     halves, the online softmax on the accumulator fragments (row max / sum over
//     each lane quad), and O += P V with P passed, for bf16, as a hi + lo pair,
//     so its rounding (2^-9) does not reach the output (2^-17); fp16 P (2^-11)
//     goes in alone; O stays in registers, D/8 fragments of 16 x 8.
// Tokens past the end or in a skipped block are masked: their scores by
// selection, their V rows by zeroing the fragment halves (rows never copied
// may hold anything, NaN included). The fused append patches the new token's
// rows into the staged unit (one consumer per CTA, so no cross-warp barrier)
// and one CTA per KV head stores them to the cache.
// tcgen05 (M >= 64) would pad an 8-head group eightfold and move the running
// softmax through TMEM; the path is bound by HBM, and m16n8k16 keeps S, P and
// O in registers.
template <int D>
struct GqaTiling {
  static constexpr int ROWS = 16;               // tokens per unit = one MMA k-step of P V
  static constexpr int BOX = 16 * 128;          // one swizzled box: 16 rows x 64 elements
  static constexpr int TILE = (D / 64) * BOX;   // one K (or V) unit
  static constexpr int STAGE = 2 * TILE;
  static constexpr int NC = 4;                  // consumer warps; unit u goes to warp u % NC
  static constexpr int NS = 2 * NC;             // two stages per consumer
  // Consumer w takes units w, w + NC, ...; a stage is reused every NS units, so
  // with NS a multiple of NC each stage's units belong to one consumer and it
  // never waits on a stage phase two ahead (which a parity wait cannot tell apart).
  static_assert(NS % NC == 0, "stages must be a multiple of the consumer count");
  static constexpr int SMEM_MERGE = NC * ROWS * (D + 2) * 4;  // reuses the stages at the end
  static constexpr int SMEM_STAGES = NS * STAGE > SMEM_MERGE ? NS * STAGE : SMEM_MERGE;
  // + 1024: the stages start on a 1024-byte boundary (the swizzle period)
  static constexpr int QPITCH = (D + 8) * 2;    // the Q tile (when Q is not kept in registers)
  static constexpr int SMEM_Q = ROWS * QPITCH;
  static constexpr int SMEM = 1024 + SMEM_STAGES + SMEM_Q + 2 * NS * 8 + NS * 4;
};

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

template <typename T, typename TO, int D, int S, bool APPEND, int NHT>
__global__ void __launch_bounds__((GqaTiling<D>::NC + 1) * 32)
    paged_decode_gqa_kernel(const DecodeParams p, const __grid_constant__ CUtensorMap tmk,
                            const __grid_constant__ CUtensorMap tmv) {
  using Tg = GqaTiling<D>;
  constexpr int ROWS = Tg::ROWS, TILE = Tg::TILE, STAGE = Tg::STAGE;
  constexpr int NS = Tg::NS, NC = Tg::NC;
  constexpr int BR = S < 16 ? S : 16;  // rows per box
  constexpr int SLAB = S * D * 2;
  constexpr int KS = D / 16;  // k-steps of S

  const int part = blockIdx.x;
  const int G = p.H / p.Hkv;
  const int chunks = (G + 15) / 16;
  const int hk = blockIdx.y / chunks;
  const int c0 = (blockIdx.y % chunks) * 16;  // first query head (within the group) of this CTA
  const int gc = min(16, G - c0);             // query heads served here
  const int i = blockIdx.z;
  const int lane = threadIdx.x & 31;
  const int w = threadIdx.x >> 5;

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
  uint8_t* qtile = stages + Tg::SMEM_STAGES;
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

  const int t_beg = part * p.P;
  const int t_end = min(t_beg + p.P, L);
  const int nunits = t_end > t_beg ? (t_end - t_beg + ROWS - 1) / ROWS : 0;
  const int32_t* trow = p.block_tables + static_cast<int64_t>(i) * p.MB;
  const int64_t block_stride = static_cast<int64_t>(p.Hkv) * SLAB;
  const uint8_t* kbase = static_cast<const uint8_t*>(p.k_cache) + static_cast<int64_t>(hk) * SLAB;
  const uint8_t* vbase = static_cast<const uint8_t*>(p.v_cache) + static_cast<int64_t>(hk) * SLAB;

  if (w == NC) {
    // ---- producer: one lane per box of a unit issues the loads ----
    const uint64_t policy = policy_evict_first();
    const int blk0 = t_beg / S;
    const int blk1 = t_end > t_beg ? (t_end + S - 1) / S : blk0;
    int base = 0;
    int ids_a = (blk0 + lane < blk1) ? __ldg(trow + blk0 + lane) : -1;
    int ids_b = (blk0 + 32 + lane < blk1) ? __ldg(trow + blk0 + 32 + lane) : -1;
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
        bytes += 2u * (D / 64) * BR * 128u;
      }
      if (lane == 0) {
        rowmask[s] = okmask;
        mbar_arrive_expect_tx(&full[s], bytes);
      }
      __syncwarp();
      constexpr int NBOX = NH * (D / 64) * 2;  // (row group, column block, K or V)
      if (lane < NBOX) {
        const int hh = lane / ((D / 64) * 2), c = (lane >> 1) % (D / 64), kv = lane & 1;
        if (issue[hh]) {
          uint8_t* dst = stages + s * STAGE + c * Tg::BOX + hh * BR * 128 + kv * TILE;
          tma_load_2d(dst, kv ? &tmv : &tmk, c * 64, rows_y[hh], &full[s], policy);
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
    }
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

  for (int k = w; k < nunits; k += NC) {
    const int s = k % NS;
    if (!mbar_wait_bounded(&full[s], (k / NS) & 1)) {
      if (lane == 0) raise_error(PA_DEVERR_TIMEOUT);
      break;
    }
    uint8_t* ktile = stages + s * STAGE;
    uint8_t* vtile = ktile + TILE;
    const int t0 = t_beg + k * ROWS;
    uint32_t valid = rowmask[s];
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
          mma16816<T>((kk & 1) ? sodd[nt] : sacc[nt], a, qb[nt][kk][0], qb[nt][kk][1]);
      } else {
        uint32_t b[4];
        ldsm_x4(b, qtile + q_row * Tg::QPITCH + (kk * 16 + q_c8) * 2);
#pragma unroll
        for (int nt = 0; nt < NHT; ++nt)
          mma16816<T>((kk & 1) ? sodd[nt] : sacc[nt], a, b[2 * nt], b[2 * nt + 1]);
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
      const uint32_t h0 = pack2<T>(pr[0], pr[1]), h1 = pack2<T>(pr[2], pr[3]);
      bhi[nt][0] = movmatrix_trans(h0);
      bhi[nt][1] = movmatrix_trans(h1);
      if (std::is_same<T, __nv_bfloat16>::value) {
        const float2 f0 = unpack2<T>(h0), f1 = unpack2<T>(h1);
        blo[nt][0] = movmatrix_trans(pack2<T>(pr[0] - f0.x, pr[1] - f0.y));
        blo[nt][1] = movmatrix_trans(pack2<T>(pr[2] - f1.x, pr[3] - f1.y));
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
        mma16816<T>(o[mt][nt], a, bhi[nt][0], bhi[nt][1]);
        if (std::is_same<T, __nv_bfloat16>::value)
          mma16816<T>(o[mt][nt], a, blo[nt][0], blo[nt][1]);
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
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

// Merges the partitions of every (request, head) that has more than one:
//   M = max_p m_p;  out = sum_p 2^(m_p - M) acc_p / sum_p 2^(m_p - M) l_p.
// One warp per (request, head): lanes load the partitions' m and l in parallel
// (32 at a time), then every lane accumulates its D/32 output elements over
// the partitions with the weights broadcast by shuffle.
template <typename TO, int D>
__global__ void __launch_bounds__(128) splitkv_reduce_kernel(const DecodeParams p) {
  constexpr int DL = D / 32;
  const int lane = threadIdx.x & 31;
  const int64_t ih = static_cast<int64_t>(blockIdx.x) * 4 + (threadIdx.x >> 5);
  if (ih >= static_cast<int64_t>(p.B) * p.H) return;
  const int i = static_cast<int>(ih / p.H);
  int L = __ldg(p.seq_lens + i);
  L = L < 0 ? 0 : (L > p.L_cap ? p.L_cap : L);
  const int nparts = (L + p.P - 1) / p.P;
  if (nparts <= 1) return;  // written by the partition pass
  const float* m = p.ws_m + ih * p.NP;
  const float* l = p.ws_l + ih * p.NP;
  const float* acc = p.ws_acc + ih * p.NP * D + lane * DL;

  float M = -INFINITY;
  for (int q = lane; q < nparts; q += 32) M = fmaxf(M, m[q]);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) M = fmaxf(M, __shfl_xor_sync(kFullMask, M, off));

  float lsum = 0.f;
  float a[DL];
#pragma unroll
  for (int e = 0; e < DL; ++e) a[e] = 0.f;
  for (int c = 0; c < nparts; c += 32) {
    const int q = c + lane;
    const float wq = q < nparts ? exp2f(m[q] - M) : 0.f;
    if (q < nparts) lsum = fmaf(wq, l[q], lsum);
    const int n = min(32, nparts - c);
#pragma unroll 4
    for (int r = 0; r < n; ++r) {
      const float w = __shfl_sync(kFullMask, wq, r);
      const float* row = acc + static_cast<int64_t>(c + r) * D;
#pragma unroll
      for (int e = 0; e < DL; e += 2) {
        const float2 v = *reinterpret_cast<const float2*>(row + e);
        a[e] = fmaf(w, v.x, a[e]);
        a[e + 1] = fmaf(w, v.y, a[e + 1]);
      }
    }
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) lsum += __shfl_xor_sync(kFullMask, lsum, off);
  TO* o = static_cast<TO*>(p.out) + ih * D + lane * DL;
#pragma unroll
  for (int e = 0; e < DL; ++e) o[e] = to_out<TO>(lsum > 0.f ? a[e] / lsum : 0.f);
}

}  // namespace pa
