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
#include "pa_launch.h"

namespace pa {


// Shapes of the partition pass for head_dim D, block_size S and EB-byte cache
// elements (2: fp16 / bf16, 1: E4M3).
//   EPL      elements per lane per row fragment (one 16-byte shared load): 16 / EB
//   LPR      lanes per row (D / EPL); RPW = 32 / LPR rows per warp-wide load
//   CR       rows per pipeline unit: CR x D of K and of V (up to 4 KB each) is one
//            stage, so the stage size no longer grows with S; a block of S rows
//            is S / CR units
//   NS, NW   stages per warp and warps per CTA: about 64 KB of stages per CTA.
//            Grids of more than four CTAs per SM (WIDE = false) with units of
//            2 KB or less at head_dim 64 or over E4M3 caches take 32 KB: half
//            the warps, each walking twice the blocks of a partition, so that
//            pipeline fill and drain weigh half as much and twice the CTAs
//            share an SM (head_dim 64 at blocks 8 and 16: 5-12 % faster from
//            batch 32 up; the 13B-shaped E4M3 decode 124 -> 108 us). Smaller
//            grids (WIDE = true, cluster launches among them) keep the wider
//            CTAs, which spread their few CTAs' work over more warps (batch
//            1, head_dim 128, block 8: 14.4 against 17.4 us), and so does
//            16-bit head_dim 128 at block 8 (narrow CTAs: 99 against 89 us at
//            batch 8, 2.441 against 2.476 ms at batch 256).
template <int D, int S, int EB = 2, bool WIDE = false>
struct DecodeTiling {
  static constexpr int EPL = 16 / EB;
  static constexpr int LPR = D / EPL;
  static constexpr int RPW = 32 / LPR;
  static constexpr int CR_RAW = 4096 / (D * EB);
  static constexpr int CR = CR_RAW < S ? CR_RAW : S;
  static constexpr int NV = CR / RPW;  // rows per lane per unit
  static constexpr int SLAB = S * D * EB;    // one (block, head) slab of K or of V
  static constexpr int UNIT = CR * D * EB;   // one unit of K or of V
  static constexpr int STAGE = 2 * UNIT;
  // E4M3 units carry twice the elements per byte, so more warps (two stages
  // each) keep the same bytes in flight with twice the threads to convert them
  static constexpr int NS = (STAGE <= 4096 && EB == 2) ? 4 : 2;
  static constexpr bool NARROW = !WIDE && UNIT <= 2048 && (EB == 1 || D <= 64);
  static constexpr int NW_RAW = (NARROW ? 32768 : 65536) / (NS * STAGE);
  static constexpr int NW = NW_RAW < 1 ? 1 : (NW_RAW > 8 ? 8 : NW_RAW);
  static constexpr int SMEM_PIPE = NW * NS * STAGE;
  static constexpr int SMEM_BARS = NW * NS * 8;
  static constexpr int SMEM_MERGE = NW * (D + 2) * 4;
  static constexpr int SMEM = SMEM_PIPE + SMEM_BARS + SMEM_MERGE;
  // Launched in clusters: partition 0's slots for the (acc, m, l) of up to 8
  // partitions, written by the other CTAs of its cluster.
  static constexpr int SMEM_XCH = 8 * (D + 2) * 4;
  static constexpr int SMEM_CL = SMEM + SMEM_XCH;
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

// A 16-byte row fragment for copying K/V rows bit for bit (8 16-bit elements,
// or 16 E4M3 codes).
struct RawFrag {
  uint4 w;
  __device__ __forceinline__ void load(const void* src) { w = *reinterpret_cast<const uint4*>(src); }
  __device__ __forceinline__ void store(void* dst) const { *reinterpret_cast<uint4*>(dst) = w; }
};

// The E4M3 codes of EL consecutive 16-bit elements (EL = 2, 4 or 8, packed in
// x), each the code of fp32(x / scale) (one correctly rounded division, round
// to nearest even, saturated at 448): the rule of kv_append_fp8_kernel, so the
// fused append stores the same bytes as pa_kv_append_fp8. Codes in element
// order, the first in the lowest byte.
template <typename T, int EL>
__device__ __forceinline__ void quantize_e4m3(const uint32_t (&x)[EL / 2], float scale,
                                              uint32_t (&codes)[(EL + 3) / 4]) {
#pragma unroll
  for (int j = 0; j < (EL + 3) / 4; ++j) codes[j] = 0;
#pragma unroll
  for (int e = 0; e < EL / 2; ++e) {
    const float2 f = Elem<T>::pair(x[e]);
    const uint32_t c = float2_to_e4m3x2(__fdiv_rn(f.x, scale), __fdiv_rn(f.y, scale));
    codes[e / 2] |= c << (16 * (e & 1));
  }
}

// One CTA per (partition, head, request); NW warps, each an independent
// pipeline over the tokens of a contiguous run of the partition's blocks,
// taken CR rows (one unit) at a time.
//
// APPEND = true fuses the decode step's append: for request i with L >= 1, the
// new token (position L - 1) takes its K/V from k_new / v_new. The warp whose
// run holds that token copies the row into its staged unit once the bulk copy
// has landed (so the scores see it) and stores it to the cache, as
// pa_kv_append would have before the decode. Over an E4M3 cache (Prm =
// DecodeParamsQ8) the row is first quantized as pa_kv_append_fp8 does.
//
// TC is the cache element type: T itself, or E4M3 codes with per-tensor
// scales (K's folded into q_scale, V's applied to the accumulated output).
//
// CLUSTER = true: launched in clusters of p.NP CTAs, one per (request, head); partition 0 merges the others' results, which they store
// into its shared memory, instead of the merge kernel reading them from the
// workspace. (A template parameter, so that the plain form's code is not
// touched by it.)
template <typename T, typename TO, int D, int S, bool APPEND, typename TC = T,
          bool CLUSTER = false, typename Prm = DecodeParams, bool WIDE = CLUSTER>
__global__ void __launch_bounds__(DecodeTiling<D, S, sizeof(TC), WIDE>::NW * 32)
    paged_decode_partition_kernel(const Prm p) {
  constexpr int EB = sizeof(TC);
  static_assert(!APPEND || EB == 2 || std::is_same<Prm, DecodeParamsQ8>::value,
                "the fused append over an E4M3 cache needs K's scale");
  static_assert(WIDE || !CLUSTER, "cluster launches take the wide shapes");
  using Tl = DecodeTiling<D, S, EB, WIDE>;
  constexpr int NW = Tl::NW, NS = Tl::NS, SLAB = Tl::SLAB, UNIT = Tl::UNIT, STAGE = Tl::STAGE;
  constexpr int EPL = Tl::EPL, LPR = Tl::LPR, RPW = Tl::RPW, CR = Tl::CR, NV = Tl::NV;
  constexpr int DUP = LPR / NV;  // lanes of a group holding the same row's score

  grid_dependents_launch();  // the merge of split requests may be scheduled early
  // In a cluster launch every thread takes two cluster barriers, whichever
  // path it follows: the first (arrived at here) guarantees that every CTA of
  // the cluster has started before partition 0's shared memory is written, the
  // second that the writes have landed before partition 0 reads them.
  constexpr bool clustered = CLUSTER;
  if constexpr (clustered) cluster_arrive_relaxed();
  const int part = blockIdx.x;  // in a cluster launch, also the CTA's rank
  const int h = blockIdx.y;
  const int i = blockIdx.z;
  const int lane = threadIdx.x & 31;
  const int w = threadIdx.x >> 5;
  if constexpr (APPEND && EB == 1) {
    // the new rows (D 16-bit elements each), wanted by whichever warp turns out
    // to own the new token: have L2 fetch them while the length is read
    // (one KV head per query head here: the row of (i, h); D * 2 bytes, D / 64 lines)
    if (threadIdx.x < D / 64) {
      const int64_t row = ((static_cast<int64_t>(i) * p.H + h) * D) * 2 + threadIdx.x * 128;
      prefetch_l2(static_cast<const uint8_t*>(p.k_new) + row);
      prefetch_l2(static_cast<const uint8_t*>(p.v_new) + row);
    }
  }
  const int g = lane / LPR;   // row group
  const int pl = lane % LPR;  // position in the row: elements pl * EPL .. pl * EPL + EPL - 1

  int L = __ldg(p.seq_lens + i);
  const bool len_ok = L >= 0 && L <= p.L_cap;
  if (!len_ok) {
    if (threadIdx.x == 0 && part == 0 && h == 0) raise_error(PA_DEVERR_SEQ_LEN);
    L = L < 0 ? 0 : p.L_cap;
  }
  const int nparts = (L + p.P - 1) / p.P;
  if (part > 0 && part >= nparts) {  // nothing here (part 0 writes the L == 0 zeros)
    if constexpr (clustered) {
      cluster_wait_acquire();
      cluster_arrive_release();
      cluster_wait_acquire();
    }
    return;
  }
  const bool direct = nparts <= 1;  // the only partition: write the final output

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

  // q fragment, pre-scaled so that scores come out in base-2 units. E4M3 caches
  // take q as f16 pairs instead, exactly scaled by 2^qe so that its largest
  // element is below 2^15 (qe undone on the score): the dot products then run
  // as fp32 accumulations of exact f16 x f16 products straight from the
  // codes' f16 conversion.
  float qf[EPL];
  uint32_t qh[EB == 1 ? EPL / 2 : 1];
  float score_scale = 1.f;
  {
    const T* qp = static_cast<const T*>(p.q) + (static_cast<int64_t>(i) * p.H + h) * D + pl * EPL;
    load_row<T, EPL>(qp, qf);
    if constexpr (EB == 1) {
      float mx = 0.f;
#pragma unroll
      for (int e = 0; e < EPL; ++e) mx = fmaxf(mx, fabsf(qf[e]));
#pragma unroll
      for (int off = 1; off < LPR; off <<= 1) mx = fmaxf(mx, __shfl_xor_sync(kFullMask, mx, off));
      int qe = 0;
      if (mx > 0.f && mx < INFINITY) {
        frexpf(mx, &qe);                      // mx = f * 2^qe, f in [0.5, 1)
        qe = max(-100, min(100, 15 - qe));    // max |q| * 2^qe < 2^15
      }
      const float up = ldexpf(1.f, qe);
      score_scale = p.q_scale * ldexpf(1.f, -qe);
#pragma unroll
      for (int e = 0; e < EPL; e += 2) {
        const __half2 q2 = __floats2half2_rn(qf[e] * up, qf[e + 1] * up);
        qh[e / 2] = *reinterpret_cast<const uint32_t*>(&q2);
      }
    } else {
#pragma unroll
      for (int e = 0; e < EPL; ++e) qf[e] *= p.q_scale;
    }
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
  // E4M3 cache: every lane of the appender warp takes EL = D / 32 elements of
  // the new rows (16-bit), and quantizes and stores them itself
  constexpr int EL = D / 32;
  uint32_t k_raw[EB == 1 ? EL / 2 : 1], v_raw[EB == 1 ? EL / 2 : 1];
  if constexpr (APPEND && EB == 1) {
    if (appender) {
      const int64_t off = ((static_cast<int64_t>(i) * p.Hkv + hk) * D + lane * EL) * 2;
#pragma unroll
      for (int e = 0; e < EL / 2; ++e) {
        k_raw[e] = reinterpret_cast<const uint32_t*>(static_cast<const uint8_t*>(p.k_new) + off)[e];
        v_raw[e] = reinterpret_cast<const uint32_t*>(static_cast<const uint8_t*>(p.v_new) + off)[e];
      }
      id_new = __ldg(trow + t_new / S);
    }
  } else if (appender && g == 0) {
    // the new rows are 16-bit: EPL elements, EPL * 2 bytes, per lane
    const int64_t off = ((static_cast<int64_t>(i) * p.Hkv + hk) * D + pl * EPL) * 2;
    k_row.load(static_cast<const uint8_t*>(p.k_new) + off);
    v_row.load(static_cast<const uint8_t*>(p.v_new) + off);
    id_new = __ldg(trow + t_new / S);
  }
  // E4M3 cache: the new token sits in the appender's last unit. Its codes go to
  // the cache just before that unit's bulk copy is issued (after the warp's
  // earlier copies, so the loads and the quantization overlap their flight),
  // and the copy brings them; the proxy fence orders the generic-proxy stores
  // before lane 0's async-proxy read. The pipeline loop then runs as without
  // the append. (A block id out of range stores nothing; its unit is flagged
  // when issued.)
  const int k_new_unit = appender ? (t_new - wt0) / CR : -1;
  auto store_new_rows = [&]() {
    if constexpr (APPEND && EB == 1) {
      uint32_t kc[(EL + 3) / 4], vc[(EL + 3) / 4];
      quantize_e4m3<T, EL>(k_raw, p.k_scale, kc);
      quantize_e4m3<T, EL>(v_raw, p.v_scale, vc);
      if (static_cast<unsigned>(id_new) < static_cast<unsigned>(p.NB)) {
        const int64_t goff = static_cast<int64_t>(id_new) * block_stride +
                             static_cast<int64_t>(t_new % S) * D + lane * EL;
        uint8_t* kd = const_cast<uint8_t*>(kbase) + goff;
        uint8_t* vd = const_cast<uint8_t*>(vbase) + goff;
        if constexpr (EL == 2) {
          *reinterpret_cast<uint16_t*>(kd) = static_cast<uint16_t>(kc[0]);
          *reinterpret_cast<uint16_t*>(vd) = static_cast<uint16_t>(vc[0]);
        } else if constexpr (EL == 4) {
          *reinterpret_cast<uint32_t*>(kd) = kc[0];
          *reinterpret_cast<uint32_t*>(vd) = vc[0];
        } else {
          *reinterpret_cast<uint2*>(kd) = make_uint2(kc[0], kc[1]);
          *reinterpret_cast<uint2*>(vd) = make_uint2(vc[0], vc[1]);
        }
        asm volatile("fence.proxy.async.global;" ::: "memory");
      }
      __syncwarp();
    }
  };

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
                            static_cast<int64_t>(t0 % S) * D * EB;
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
  for (int k = 0; k < NS; ++k) {
    if constexpr (APPEND && EB == 1) {
      if (issued == k_new_unit) store_new_rows();  // warp-uniform
    }
    issue_next();
  }
  if constexpr (APPEND && EB == 1) {
    if (issued <= k_new_unit) store_new_rows();  // that unit is issued in the loop below
  }

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
      if (APPEND && EB == 2 && appender && t_new >= t0 && t_new < t0 + CR) {
        // the bulk copy brought the old bytes; put the new token's row in both
        // the staged unit and the cache
        if (g == 0) {
          const int64_t row_off = (static_cast<int64_t>(t_new - t0) * D + pl * EPL) * EB;
          k_row.store(ks + row_off);
          v_row.store(vs + row_off);
          const int64_t goff = static_cast<int64_t>(id_new) * block_stride +
                               (static_cast<int64_t>(t_new % S) * D + pl * EPL) * EB;
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
        if constexpr (EB == 1) {  // f16 codes x f16 q, fp32 sums
          uint32_t kh[EPL / 2];
          e4m3x16_to_h2(ks + ((v * RPW + g) * D + pl * EPL), kh);
          float a0 = 0.f, a1 = 0.f;
#pragma unroll
          for (int e = 0; e < EPL / 2; ++e) fma_f16pair_f32(qh[e], kh[e], a0, a1);
          dot[v] = a0 + a1;
        } else {
          float kf[EPL];
          load_cache_row<TC, EPL>(ks + ((v * RPW + g) * D + pl * EPL) * EB, kf);
          float a = 0.f;
#pragma unroll
          for (int e = 0; e < EPL; ++e) a = fmaf(qf[e], kf[e], a);
          dot[v] = a;
        }
      }
      float score = transpose_reduce<NV, LPR>(dot, lane);
      if constexpr (EB == 1) score *= score_scale;
      const bool valid = my_row < nvalid;
      const float sc = valid ? score : -INFINITY;
      float mb = sc;
#pragma unroll
      for (int off = DUP; off < 32; off <<= 1) mb = fmaxf(mb, __shfl_xor_sync(kFullMask, mb, off));
      const float m_new = fmaxf(m, mb);
      const float alpha = exp2f(m - m_new);
      const float pr = valid ? exp2f(sc - m_new) : 0.f;
      lsum = lsum * alpha + ((pl % DUP) == 0 ? pr : 0.f);
      if (m_new != m) {  // warp-uniform; otherwise alpha is exactly 1
#pragma unroll
        for (int e = 0; e < EPL; ++e) acc[e] *= alpha;
      }
      if (nvalid == CR) {
#pragma unroll
        for (int v = 0; v < NV; ++v) {
          const float pv = __shfl_sync(kFullMask, pr, g * LPR + v * DUP);
          if constexpr (EB == 1) {  // the weight as f16 (2^-12 relative), fp32 sums
            uint32_t vh[EPL / 2];
            e4m3x16_to_h2(vs + ((v * RPW + g) * D + pl * EPL), vh);
            const __half2 p2 = __float2half2_rn(pv);
            const uint32_t ph = *reinterpret_cast<const uint32_t*>(&p2);
#pragma unroll
            for (int e = 0; e < EPL / 2; ++e) fma_f16pair_f32(ph, vh[e], acc[2 * e], acc[2 * e + 1]);
          } else {
            float vf[EPL];
            load_cache_row<TC, EPL>(vs + ((v * RPW + g) * D + pl * EPL) * EB, vf);
#pragma unroll
            for (int e = 0; e < EPL; ++e) acc[e] = fmaf(pv, vf[e], acc[e]);
          }
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
            load_cache_row<TC, EPL>(vs + ((v * RPW + g) * D + pl * EPL) * EB, vf);
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
  // Cluster launch: this partition's (acc, m, l) go to its slot in partition
  // 0's shared memory (every CTA of the cluster has started once the first
  // barrier is passed).
  float* xch = reinterpret_cast<float*>(smem + Tl::SMEM);
  uint32_t xrem = 0;
  if constexpr (clustered) {
    cluster_wait_acquire();
    xrem = cluster_map(smem_u32(xch + part * (D + 2)), 0);
  }
  for (int d = threadIdx.x; d < D; d += NW * 32) {
    float a = 0.f;
#pragma unroll
    for (int u = 0; u < NW; ++u) a = fmaf(wgt[u], acc_s[u * D + d], a);
    a *= p.v_scale;
    if (direct) {
      const float o = Ltot > 0.f ? a / Ltot : 0.f;
      static_cast<TO*>(p.out)[ih * D + d] = to_out<TO>(o);
    } else if constexpr (clustered) {
      st_cluster_f32(xrem + d * 4, a);
    } else {
      p.ws_acc[(ih * p.NP + part) * D + d] = a;
    }
  }
  if (!direct && threadIdx.x == 0) {
    if constexpr (clustered) {
      st_cluster_f32(xrem + D * 4, M);
      st_cluster_f32(xrem + (D + 1) * 4, Ltot);
    } else {
      p.ws_m[ih * p.NP + part] = M;
      p.ws_l[ih * p.NP + part] = Ltot;
    }
  }
  if constexpr (clustered) {
    cluster_arrive_release();
    cluster_wait_acquire();
    if (part != 0 || direct) return;
    // Partition 0 merges, with the arithmetic of splitkv_reduce_kernel and in
    // its order, so both ways of merging give the same bits: weights
    // 2^(m_r - M), the weighted l summed as that kernel's shuffle tree sums
    // them, the weighted acc summed over r in order.
    float Mx = -INFINITY;
    for (int r = 0; r < nparts; ++r) Mx = fmaxf(Mx, xch[r * (D + 2) + D]);
    float wr[8], lw[8];
#pragma unroll
    for (int r = 0; r < 8; ++r) {
      wr[r] = r < nparts ? exp2f(xch[r * (D + 2) + D] - Mx) : 0.f;
      lw[r] = r < nparts ? fmaf(wr[r], xch[r * (D + 2) + D + 1], 0.f) : 0.f;
    }
    const float lw_sum =
        ((lw[0] + lw[4]) + (lw[2] + lw[6])) + ((lw[1] + lw[5]) + (lw[3] + lw[7]));
    for (int d = threadIdx.x; d < D; d += NW * 32) {
      float a = 0.f;
      for (int r = 0; r < nparts; ++r) a = fmaf(wr[r], xch[r * (D + 2) + d], a);
      static_cast<TO*>(p.out)[ih * D + d] = to_out<TO>(lw_sum > 0.f ? a / lw_sum : 0.f);
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
  const bool live = ih < static_cast<int64_t>(p.B) * p.H;
  // The lengths are an input of both kernels, not a result of the first, so
  // they are read before the wait.
  int L = live ? __ldg(p.seq_lens + ih / p.H) : 0;
  // Launched as a programmatic dependent of the partition pass: its CTAs may be
  // resident before that pass ends; this waits until the pass has completed
  // and its partials are visible.
  grid_dependency_wait();
  if (!live) return;
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

// Launches the merge of split requests (no-op without a split) on `stream` as a
// programmatic dependent of the partition pass launched just before it, so its
// launch overlaps that pass's last wave instead of following it.
template <typename TO, int D>
inline cudaError_t launch_splitkv_reduce(const DecodeParams& p, cudaStream_t stream) {
  if (p.NP <= 1) return cudaSuccess;
  const int64_t pairs = static_cast<int64_t>(p.B) * p.H;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>((pairs + 3) / 4));
  cfg.blockDim = dim3(128);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, splitkv_reduce_kernel<TO, D>, p);
}

// Launches the partition pass (grid NP x H x B) and the merge: `kern_cl` in
// clusters of NP CTAs that merge among themselves (threads_cl threads, dynamic
// shared memory smem_cl), or `kern` as a plain grid (threads, smem) followed
// by the merge kernel.
template <typename TO, int D, typename Kern, typename Prm>
inline cudaError_t launch_partition_pass(Kern kern, Kern kern_cl, bool cluster, const Prm& p,
                                         int threads, int smem, int threads_cl, int smem_cl,
                                         cudaStream_t stream) {
  const dim3 grid(p.NP, p.H, p.B);
  if (cluster) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(threads_cl);
    cfg.dynamicSmemBytes = smem_cl;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = p.NP;  // one cluster per (request, head)
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern_cl, p);
  }
  kern<<<grid, threads, smem, stream>>>(p);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_splitkv_reduce<TO, D>(p, stream);
}

}  // namespace pa
