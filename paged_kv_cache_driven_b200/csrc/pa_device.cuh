// Device-side building blocks shared by the append and decode kernels:
// the per-device error word, mbarrier / bulk-copy wrappers (inline PTX for
// sm_100a), and 16-bit <-> fp32 conversions.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>
#include <cstdint>

#include "pagedattn.h"

namespace pa {

// One word per device and per translation unit that holds kernels; kernels OR
// PA_DEVERR_* bits into it. take_error_word() (host) reads and clears this
// unit's word; pa_get_device_error() gathers every unit's.
static __device__ unsigned int g_error_word = 0;

__device__ __forceinline__ void raise_error(unsigned int bits) { atomicOr(&g_error_word, bits); }

// Host: ORs this translation unit's error word into *bits and clears it.
static inline bool take_error_word(unsigned int* bits) {
  unsigned int v = 0;
  const unsigned int zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_error_word, sizeof(v)) != cudaSuccess) return false;
  if (cudaMemcpyToSymbol(g_error_word, &zero, sizeof(zero)) != cudaSuccess) return false;
  *bits |= v;
  return true;
}

constexpr unsigned kFullMask = 0xffffffffu;

// About one second at B200 clocks: the bound on every wait for a bulk copy.
constexpr long long kWaitLimitCycles = 2000000000LL;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

// Makes mbarrier initialisation visible to the async proxy (bulk copies).
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Waits for the phase with the given parity to complete; gives up after about
// a second and returns false (the caller flags PA_DEVERR_TIMEOUT).
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitLimitCycles) return false;
  }
  return true;
}

// Programmatic dependent launch: a kernel launched with the programmatic
// stream-serialization attribute may start while the kernel before it on the
// stream still runs; grid_dependency_wait() blocks until that kernel has
// completed and its memory operations are visible. grid_dependents_launch()
// lets the dependent grid be scheduled once every CTA of this grid has issued
// it (or exited).
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void grid_dependents_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// Asks L2 to fetch the 128-byte line at p (no register result, no wait).
__device__ __forceinline__ void prefetch_l2(const void* p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Thread-block clusters. The cluster barrier is split: every thread of every
// CTA of the cluster arrives, then waits until all have arrived (non-.aligned
// forms, so a warp need not be converged). A relaxed arrival orders nothing;
// a release arrival followed by an acquire wait makes the arriving threads'
// earlier shared-memory stores (distributed ones included) visible to the
// waiting threads.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_release() {
  asm volatile("barrier.cluster.arrive.release;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait_acquire() {
  asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
}
// The shared::cluster address of the same shared-memory offset in CTA `rank`
// of this cluster, and a 32-bit store through such an address.
__device__ __forceinline__ uint32_t cluster_map(uint32_t smem_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_cluster_f32(uint32_t addr, float v) {
  asm volatile("st.shared::cluster.f32 [%0], %1;" ::"r"(addr), "f"(v) : "memory");
}

// L2 policy for data read exactly once per step (the KV slabs).
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// One-dimensional bulk copy global -> this CTA's shared memory, completing on
// `bar` with `bytes` of transaction count. Both addresses 16-byte aligned,
// bytes a multiple of 16. No multicast.
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                                         uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
      " [%0], [%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Two-dimensional tiled TMA load global -> this CTA's shared memory through a
// tensor map (in kernel-parameter space), completing on `bar`. x is the
// innermost coordinate; x * element size must be a multiple of 16 bytes. No
// multicast.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, int x, int y,
                                            uint64_t* bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

// Packed pairs of fp32 (one 64-bit register pair, two lanes of work per
// instruction).
__device__ __forceinline__ uint64_t as_u64(float2 a) {
  return static_cast<uint64_t>(__float_as_uint(a.x)) |
         (static_cast<uint64_t>(__float_as_uint(a.y)) << 32);
}
__device__ __forceinline__ float2 as_f2(uint64_t u) {
  return make_float2(__uint_as_float(static_cast<uint32_t>(u)),
                     __uint_as_float(static_cast<uint32_t>(u >> 32)));
}
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(as_u64(a)), "l"(as_u64(b)), "l"(as_u64(c)));
  return as_f2(d);
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(as_u64(a)), "l"(as_u64(b)));
  return as_f2(d);
}
// ---- 16-bit element conversions -------------------------------------------------

template <typename T>
struct Elem;

template <>
struct Elem<__half> {
  __device__ __forceinline__ static float2 pair(uint32_t x) {
    __half2 h;
    *reinterpret_cast<uint32_t*>(&h) = x;
    return __half22float2(h);
  }
  __device__ __forceinline__ static float one(uint16_t x) {
    return __half2float(__ushort_as_half(x));
  }
};

template <>
struct Elem<__nv_bfloat16> {
  // bf16 is the top half of an fp32: widening is a shift / mask, exact.
  __device__ __forceinline__ static float2 pair(uint32_t x) {
    return make_float2(__uint_as_float(x << 16), __uint_as_float(x & 0xffff0000u));
  }
  __device__ __forceinline__ static float one(uint16_t x) {
    return __uint_as_float(static_cast<uint32_t>(x) << 16);
  }
};

// DL consecutive 16-bit elements (DL in {2, 4, 8, 16}) from shared or global
// memory into fp32 registers, with one 4/8/16-byte load (two for 16).
template <typename T, int DL>
__device__ __forceinline__ void load_row(const void* p, float (&f)[DL]) {
  if constexpr (DL == 16) {
    float a[8], b[8];
    load_row<T, 8>(p, a);
    load_row<T, 8>(static_cast<const uint8_t*>(p) + 16, b);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      f[k] = a[k];
      f[8 + k] = b[k];
    }
  } else if constexpr (DL == 2) {
    const uint32_t x = *reinterpret_cast<const uint32_t*>(p);
    const float2 a = Elem<T>::pair(x);
    f[0] = a.x;
    f[1] = a.y;
  } else if constexpr (DL == 4) {
    const uint2 x = *reinterpret_cast<const uint2*>(p);
    const float2 a = Elem<T>::pair(x.x), b = Elem<T>::pair(x.y);
    f[0] = a.x;
    f[1] = a.y;
    f[2] = b.x;
    f[3] = b.y;
  } else {
    static_assert(DL == 8, "DL must be 2, 4 or 8");
    const uint4 x = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 a = Elem<T>::pair(w[k]);
      f[2 * k] = a.x;
      f[2 * k + 1] = a.y;
    }
  }
}

// FP8 E4M3 (cache storage): two codes (low byte first) -> fp32, exactly, through
// the hardware conversion to a pair of binary16 values.
__device__ __forceinline__ float2 e4m3x2_to_float2(uint16_t x) {
  uint32_t h2;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h2) : "h"(x));
  __half2 h;
  *reinterpret_cast<uint32_t*>(&h) = h2;
  return __half22float2(h);
}

// Two fp32 -> two E4M3 codes (lo in the low byte), round to nearest even,
// saturated at +-448.
__device__ __forceinline__ uint16_t float2_to_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// 16 E4M3 codes (one 16-byte fragment) -> 8 f16 pairs, exactly (E4M3 values are
// f16 values).
__device__ __forceinline__ void e4m3x16_to_h2(const void* p, uint32_t (&h)[8]) {
  const uint4 x = *reinterpret_cast<const uint4*>(p);
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h[2 * k]) : "h"(static_cast<uint16_t>(w[k] & 0xffffu)));
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h[2 * k + 1]) : "h"(static_cast<uint16_t>(w[k] >> 16)));
  }
}

// c0 += lo(a) * lo(b), c1 += hi(a) * hi(b): fp32 accumulation of products of
// f16 values (the products are exact in fp32), one mixed-precision FMA each.
__device__ __forceinline__ void fma_f16pair_f32(uint32_t a, uint32_t b, float& c0, float& c1) {
  asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
      "mov.b32 {al, ah}, %2;\n\t"
      "mov.b32 {bl, bh}, %3;\n\t"
      "fma.rn.f32.f16 %0, al, bl, %0;\n\t"
      "fma.rn.f32.f16 %1, ah, bh, %1;\n\t}"
      : "+f"(c0), "+f"(c1)
      : "r"(a), "r"(b));
}

// One row fragment of the cache (16 bytes in shared memory) -> fp32 registers:
// 8 elements of a 16-bit cache, or 16 of an E4M3 cache.
template <typename TC, int EPL>
__device__ __forceinline__ void load_cache_row(const void* p, float (&f)[EPL]) {
  if constexpr (sizeof(TC) == 1) {
    static_assert(EPL == 16, "an E4M3 fragment is 16 codes");
    const uint4 x = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 a = e4m3x2_to_float2(static_cast<uint16_t>(w[k] & 0xffffu));
      const float2 b = e4m3x2_to_float2(static_cast<uint16_t>(w[k] >> 16));
      f[4 * k] = a.x;
      f[4 * k + 1] = a.y;
      f[4 * k + 2] = b.x;
      f[4 * k + 3] = b.y;
    }
  } else {
    load_row<TC, EPL>(p, f);
  }
}

// 8 consecutive 16-bit elements held in a uint4 -> fp32 registers.
template <typename T>
__device__ __forceinline__ void convert_frag(const uint4& x, float (&f)[8]) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 a = Elem<T>::pair(w[k]);
    f[2 * k] = a.x;
    f[2 * k + 1] = a.y;
  }
}

// fp32 -> output element, round to nearest even.
template <typename TO>
__device__ __forceinline__ TO to_out(float x);
template <>
__device__ __forceinline__ float to_out<float>(float x) {
  return x;
}
template <>
__device__ __forceinline__ __half to_out<__half>(float x) {
  return __float2half_rn(x);
}
template <>
__device__ __forceinline__ __nv_bfloat16 to_out<__nv_bfloat16>(float x) {
  return __float2bfloat16_rn(x);
}

}  // namespace pa
