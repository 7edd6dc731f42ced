// Test infrastructure: the CPU oracle for paged single-query decode attention.
//
// Only the tests, the smoke check and the bench's CPU-baseline leg call this
// file; the product path never does. It shares no code, header or constant
// with the CUDA library: every element is decoded here from its IEEE bits, the
// block table is walked with plain integer arithmetic, and the softmax is the
// textbook two-pass form in fp64.
//
// What it computes (the plain definition, which PagedAttention reaches exactly
// because it changes the layout and not the formula):
//   * "vLLM KV Cache and PagedAttention Explained" (hrletsgo.me),
//     "Appendix: The Attention Score Formula": Attention(Q,K,V) =
//     softmax(Q K^T / sqrt(d)) V, evaluated by walking the block table.
//   * "PagedAttention" card (llm-engineer.pages.dev), "OS paging과 같은 발상"
//     and "Kernel은 무엇이 달라지는가": logical block j of a request lives in
//     physical block table[j]; the kernel reads the scattered blocks in place.
//   * "vLLM의 PagedAttention 아키텍처와 GPU 메모리 최적화 원리" (velog.io),
//     section 4: the cache is one 4-D tensor [Block, Head, Block_Size, Head_D],
//     Head_D fastest.
//   * The same card, "헷갈리기 쉬운 구분": FlashDecoding splits long-context
//     decode; oracle_partition_stats gives the per-partition (max, sum, acc)
//     that such a split produces, by definition.
//
// Readings where the pages are silent (each listed in the design notes):
//   * token t of request i sits at physical block table[i][t / S], offset t % S;
//   * the query attends to exactly the first seq_lens[i] cached tokens;
//   * seq_len == 0 gives an all-zero output row;
//   * K and V share the [NB, Hkv, S, D] layout. With as many KV heads as query
//     heads (Hkv == H) this is the pages' multi-head attention; with Hkv < H
//     (grouped-query attention, not on the pages) query head h reads KV head
//     h / (H / Hkv), consecutive query heads sharing one KV head.
//
// Build: g++ -O2 -std=c++17 -shared -fPIC -pthread oracle.cpp -o liboracle.so

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <thread>
#include <vector>

namespace {

// IEEE 754 binary16: 1 sign bit, 5 exponent bits (bias 15), 10 fraction bits.
double decode_binary16(uint16_t bits) {
  const int sign = (bits >> 15) & 1;
  const int expo = (bits >> 10) & 0x1f;
  const int frac = bits & 0x3ff;
  double mag;
  if (expo == 0) {
    mag = std::ldexp(static_cast<double>(frac), -24);  // subnormal: frac * 2^-24
  } else if (expo == 31) {
    mag = frac ? std::numeric_limits<double>::quiet_NaN()
               : std::numeric_limits<double>::infinity();
  } else {
    mag = std::ldexp(static_cast<double>(1024 + frac), expo - 25);
  }
  return sign ? -mag : mag;
}

// bfloat16: the upper 16 bits of an IEEE binary32 (1 sign, 8 exponent bias 127,
// 7 fraction bits).
double decode_bfloat16(uint16_t bits) {
  const int sign = (bits >> 15) & 1;
  const int expo = (bits >> 7) & 0xff;
  const int frac = bits & 0x7f;
  double mag;
  if (expo == 0) {
    mag = std::ldexp(static_cast<double>(frac), -133);  // subnormal: frac * 2^-126 * 2^-7
  } else if (expo == 255) {
    mag = frac ? std::numeric_limits<double>::quiet_NaN()
               : std::numeric_limits<double>::infinity();
  } else {
    mag = std::ldexp(static_cast<double>(128 + frac), expo - 134);
  }
  return sign ? -mag : mag;
}

struct Problem {
  const uint16_t* q;
  const uint16_t* k_cache;
  const uint16_t* v_cache;
  const int32_t* block_tables;
  const int32_t* seq_lens;
  int64_t B, H, D, S, NB, MB;
  double scale;
  int dtype;    // 0 = binary16, 1 = bfloat16
  int64_t Hkv;  // KV heads; query head h reads KV head h / (H / Hkv)
};

double elem(const Problem& p, const uint16_t* base, int64_t idx) {
  return p.dtype == 0 ? decode_binary16(base[idx]) : decode_bfloat16(base[idx]);
}

// Offset of element (token t, dim 0) of request i, query head h, in the cache
// tensor. Returns -1 when the block table names a block outside the pool.
int64_t token_row(const Problem& p, int64_t i, int64_t h, int64_t t) {
  const int64_t logical_block = t / p.S;
  const int64_t offset = t % p.S;
  const int64_t physical_block = p.block_tables[i * p.MB + logical_block];
  if (physical_block < 0 || physical_block >= p.NB) return -1;
  const int64_t kv_head = h / (p.H / p.Hkv);
  return ((physical_block * p.Hkv + kv_head) * p.S + offset) * p.D;
}

// Scores s_t = scale * q . K_t for tokens [t0, t1) of (i, h).
int scores(const Problem& p, int64_t i, int64_t h, int64_t t0, int64_t t1,
           std::vector<double>& s, std::vector<int64_t>& rows) {
  s.assign(static_cast<size_t>(t1 - t0), 0.0);
  rows.assign(static_cast<size_t>(t1 - t0), 0);
  const int64_t qoff = (i * p.H + h) * p.D;
  for (int64_t t = t0; t < t1; ++t) {
    const int64_t row = token_row(p, i, h, t);
    if (row < 0) return 3;
    rows[t - t0] = row;
    double dot = 0.0;
    for (int64_t d = 0; d < p.D; ++d) dot += elem(p, p.q, qoff + d) * elem(p, p.k_cache, row + d);
    s[t - t0] = p.scale * dot;
  }
  return 0;
}

// Full softmax(q K^T * scale) V for one (request, head), two passes over the scores.
int decode_pair(const Problem& p, int64_t i, int64_t h, double* out) {
  const int64_t L = p.seq_lens[i];
  if (L < 0 || L > p.MB * p.S) return 3;
  for (int64_t d = 0; d < p.D; ++d) out[d] = 0.0;
  if (L == 0) return 0;
  std::vector<double> s;
  std::vector<int64_t> rows;
  if (int rc = scores(p, i, h, 0, L, s, rows)) return rc;
  double m = -std::numeric_limits<double>::infinity();
  for (double x : s) m = std::max(m, x);  // pass 1: the maximum
  double z = 0.0;
  for (double x : s) z += std::exp(x - m);  // pass 2: the normaliser
  for (int64_t t = 0; t < L; ++t) {
    const double w = std::exp(s[t] - m) / z;
    for (int64_t d = 0; d < p.D; ++d) out[d] += w * elem(p, p.v_cache, rows[t] + d);
  }
  return 0;
}

// (m, l, acc) of tokens [part*P, min((part+1)*P, L)): the max score, the sum of
// exp(s - m), and the exp(s - m)-weighted sum of V, all unnormalised.
int partition_pair(const Problem& p, int64_t i, int64_t h, int64_t part, int64_t P,
                   double* m_out, double* l_out, double* acc) {
  const int64_t L = p.seq_lens[i];
  if (L < 0 || L > p.MB * p.S) return 3;
  for (int64_t d = 0; d < p.D; ++d) acc[d] = 0.0;
  const int64_t t0 = part * P;
  const int64_t t1 = std::min(L, t0 + P);
  if (t0 >= t1) {
    *m_out = -std::numeric_limits<double>::infinity();
    *l_out = 0.0;
    return 0;
  }
  std::vector<double> s;
  std::vector<int64_t> rows;
  if (int rc = scores(p, i, h, t0, t1, s, rows)) return rc;
  double m = -std::numeric_limits<double>::infinity();
  for (double x : s) m = std::max(m, x);
  double l = 0.0;
  for (int64_t t = t0; t < t1; ++t) {
    const double w = std::exp(s[t - t0] - m);
    l += w;
    for (int64_t d = 0; d < p.D; ++d) acc[d] += w * elem(p, p.v_cache, rows[t - t0] + d);
  }
  *m_out = m;
  *l_out = l;
  return 0;
}

// Runs fn(k) for k in [0, n) on n_threads std::threads; returns the first nonzero code.
template <class Fn>
int parallel_for(int64_t n, int n_threads, Fn fn) {
  if (n_threads <= 0) n_threads = static_cast<int>(std::max(1u, std::thread::hardware_concurrency()));
  n_threads = static_cast<int>(std::min<int64_t>(n_threads, std::max<int64_t>(n, 1)));
  std::atomic<int64_t> next{0};
  std::atomic<int> status{0};
  auto worker = [&]() {
    for (;;) {
      const int64_t k = next.fetch_add(1);
      if (k >= n) break;
      const int rc = fn(k);
      if (rc) {
        int expected = 0;
        status.compare_exchange_strong(expected, rc);
      }
    }
  };
  if (n_threads == 1) {
    worker();
  } else {
    std::vector<std::thread> pool;
    for (int t = 0; t < n_threads; ++t) pool.emplace_back(worker);
    for (auto& th : pool) th.join();
  }
  return status.load();
}

bool valid_problem(const Problem& p) {
  return p.q && p.k_cache && p.v_cache && p.block_tables && p.seq_lens && p.B >= 0 && p.H > 0 &&
         p.D > 0 && p.S > 0 && p.NB >= 0 && p.MB >= 0 && (p.dtype == 0 || p.dtype == 1) &&
         p.Hkv > 0 && p.H % p.Hkv == 0;
}

// FP8 E4M3 (the OCP 8-bit floating-point format, "fn" variant: no infinities):
// sign bit 7, exponent bits 6-3 with bias 7, mantissa bits 2-0. Exponent 0 is
// subnormal (m * 2^-9); exponent 15 with mantissa 7 is NaN; everything else is
// (1 + m / 8) * 2^(e - 7). Not on the pages: a storage format for the paged cache.
double decode_e4m3(uint8_t bits) {
  const int sign = bits >> 7, e = (bits >> 3) & 15, m = bits & 7;
  double v;
  if (e == 15 && m == 7) {
    v = std::numeric_limits<double>::quiet_NaN();
  } else if (e == 0) {
    v = std::ldexp(static_cast<double>(m), -9);
  } else {
    v = std::ldexp(1.0 + m / 8.0, e - 7);
  }
  return sign ? -v : v;
}

}  // namespace

extern "C" {

double oracle_decode_e4m3(uint8_t bits) { return decode_e4m3(bits); }

// Paged decode over an FP8 E4M3 cache with one scale per tensor: K_t = k_scale *
// e4m3(k_cache[...]), V_t likewise; q (16-bit, q_dtype 0 = binary16, 1 = bfloat16)
// [B, H, D]; out[i, h] = softmax_t(scale * q . K_t) V_t over the first seq_lens[i]
// tokens, two-pass in fp64, exactly as oracle_paged_decode with dequantized K/V.
int oracle_paged_decode_fp8(const uint16_t* q, const uint8_t* k_cache, const uint8_t* v_cache,
                            double k_scale, double v_scale, const int32_t* block_tables,
                            const int32_t* seq_lens, int64_t B, int64_t H, int64_t Hkv,
                            int64_t D, int64_t S, int64_t NB, int64_t MB, double scale,
                            int q_dtype, int n_threads, double* out) {
  if (!q || !k_cache || !v_cache || !block_tables || !seq_lens || !out || B < 0 || H <= 0 ||
      Hkv <= 0 || H % Hkv || D <= 0 || S <= 0 || NB < 0 || MB < 0 || (q_dtype != 0 && q_dtype != 1))
    return 1;
  const int64_t G = H / Hkv;
  return parallel_for(B * H, n_threads, [&](int64_t k) {
    const int64_t i = k / H, h = k % H;
    double* o = out + k * D;
    for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
    const int64_t L = seq_lens[i];
    if (L < 0 || L > MB * S) return 3;
    if (L == 0) return 0;
    std::vector<double> sc(static_cast<size_t>(L));
    std::vector<int64_t> rows(static_cast<size_t>(L));
    for (int64_t t = 0; t < L; ++t) {
      const int64_t blk = block_tables[i * MB + t / S];
      if (blk < 0 || blk >= NB) return 3;
      const int64_t row = ((blk * Hkv + h / G) * S + t % S) * D;
      rows[t] = row;
      double dot = 0.0;
      for (int64_t d = 0; d < D; ++d) {
        const uint16_t qb = q[(i * H + h) * D + d];
        const double qv = q_dtype == 0 ? decode_binary16(qb) : decode_bfloat16(qb);
        dot += qv * (k_scale * decode_e4m3(k_cache[row + d]));
      }
      sc[t] = scale * dot;
    }
    double m = -std::numeric_limits<double>::infinity();
    for (double x : sc) m = std::max(m, x);
    double z = 0.0;
    for (double x : sc) z += std::exp(x - m);
    for (int64_t t = 0; t < L; ++t) {
      const double w = std::exp(sc[t] - m) / z;
      for (int64_t d = 0; d < D; ++d) o[d] += w * (v_scale * decode_e4m3(v_cache[rows[t] + d]));
    }
    return 0;
  });
}

// Decodes one 16-bit element (dtype 0 = binary16, 1 = bfloat16) to double.
double oracle_decode16(uint16_t bits, int dtype) {
  return dtype == 0 ? decode_binary16(bits) : decode_bfloat16(bits);
}

// softmax(q K^T * scale) V for each (request, query head) pair, in fp64.
//   q        [B, H, D]        16-bit elements
//   k_cache, v_cache [NB, Hkv, S, D]; Hkv divides H (Hkv == H: one KV head per
//            query head)
//   block_tables [B, MB] int32 (entries past ceil(L/S) are never read)
//   seq_lens [B] int32
//   pairs    optional [n_pairs, 2] int64 (request, head); null = every pair in
//            request-major order
//   out      [n_pairs, D] (or [B, H, D] when pairs is null), fp64
// Returns 0, 1 on a bad argument, 3 when a block id or seq_len is out of range.
int oracle_paged_decode(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                        const int32_t* block_tables, const int32_t* seq_lens, int64_t B, int64_t H,
                        int64_t Hkv, int64_t D, int64_t S, int64_t NB, int64_t MB, double scale,
                        int dtype, const int64_t* pairs, int64_t n_pairs, int n_threads,
                        double* out) {
  const Problem p{q, k_cache, v_cache, block_tables, seq_lens, B, H, D, S, NB, MB, scale, dtype,
                  Hkv};
  if (!valid_problem(p) || !out) return 1;
  const int64_t n = pairs ? n_pairs : B * H;
  for (int64_t k = 0; pairs && k < n; ++k)
    if (pairs[2 * k] < 0 || pairs[2 * k] >= B || pairs[2 * k + 1] < 0 || pairs[2 * k + 1] >= H)
      return 1;
  return parallel_for(n, n_threads, [&](int64_t k) {
    const int64_t i = pairs ? pairs[2 * k] : k / H;
    const int64_t h = pairs ? pairs[2 * k + 1] : k % H;
    return decode_pair(p, i, h, out + k * D);
  });
}

// Per-partition (m, l, acc) of each (request, head) for partitions of P tokens:
//   m [B, H, NP], l [B, H, NP], acc [B, H, NP, D], fp64, natural-log units.
// Partitions past the end of a request hold (-inf, 0, 0).
int oracle_partition_stats(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                           const int32_t* block_tables, const int32_t* seq_lens, int64_t B,
                           int64_t H, int64_t D, int64_t S, int64_t NB, int64_t MB, double scale,
                           int dtype, int64_t P, int64_t NP, int n_threads, double* m, double* l,
                           double* acc) {
  const Problem p{q, k_cache, v_cache, block_tables, seq_lens, B, H, D, S, NB, MB, scale, dtype,
                  H};
  if (!valid_problem(p) || P <= 0 || NP < 0 || !m || !l || !acc) return 1;
  return parallel_for(B * H * NP, n_threads, [&](int64_t k) {
    const int64_t ih = k / NP;
    const int64_t part = k % NP;
    return partition_pair(p, ih / H, ih % H, part, P, m + k, l + k, acc + k * D);
  });
}

// Paged prefill attention, causal ("vLLM KV Cache and PagedAttention
// Explained", 7단계 and Step 6 "Prefill and Decode": all prompt tokens run at
// once; each token attends to the tokens before it and itself). Request i has
// seq_lens[i] tokens in the cache, the last n_i = q_start[i+1] - q_start[i] of
// them new; new token j (absolute position seq_lens[i] - n_i + j) attends to
// cache tokens 0 .. that position. q and out are [q_start[B], H, D]; the
// query rows of request i are q_start[i] .. q_start[i+1) - 1; query head h
// reads KV head h / (H / Hkv).
int oracle_paged_prefill(const uint16_t* q, const uint16_t* k_cache, const uint16_t* v_cache,
                         const int32_t* block_tables, const int32_t* seq_lens,
                         const int32_t* q_start, int64_t B, int64_t H, int64_t Hkv, int64_t D,
                         int64_t S, int64_t NB, int64_t MB, double scale, int dtype,
                         int n_threads, double* out) {
  if (!q_start || !seq_lens || B < 0 || q_start[0] != 0) return 1;
  const int64_t T = q_start[B];
  // one Problem per query row would duplicate q; instead reuse the decode
  // pieces with a per-row length: row t of request i is a decode of length pos+1
  std::vector<int64_t> row_req(static_cast<size_t>(T)), row_pos(static_cast<size_t>(T));
  for (int64_t i = 0; i < B; ++i) {
    const int64_t n = q_start[i + 1] - q_start[i];
    if (n < 0 || n > seq_lens[i] || seq_lens[i] > MB * S) return 1;
    for (int64_t j = 0; j < n; ++j) {
      row_req[q_start[i] + j] = i;
      row_pos[q_start[i] + j] = seq_lens[i] - n + j;
    }
  }
  const Problem p{q, k_cache, v_cache, block_tables, seq_lens, T, H, D, S, NB, MB, scale, dtype, Hkv};
  if (!valid_problem(p) || !out) return 1;
  return parallel_for(T * H, n_threads, [&](int64_t k) {
    const int64_t t = k / H, h = k % H;
    const int64_t i = row_req[t];
    const int64_t L = row_pos[t] + 1;  // tokens this row attends to
    double* o = out + k * D;
    for (int64_t d = 0; d < D; ++d) o[d] = 0.0;
    std::vector<double> sc(static_cast<size_t>(L));
    std::vector<int64_t> rows(static_cast<size_t>(L));
    const int64_t qoff = (t * H + h) * D;
    for (int64_t tt = 0; tt < L; ++tt) {
      const int64_t row = token_row(p, i, h, tt);
      if (row < 0) return 3;
      rows[tt] = row;
      double dot = 0.0;
      for (int64_t d = 0; d < D; ++d) dot += elem(p, q, qoff + d) * elem(p, k_cache, row + d);
      sc[tt] = scale * dot;
    }
    double m = -std::numeric_limits<double>::infinity();
    for (double x : sc) m = std::max(m, x);
    double z = 0.0;
    for (double x : sc) z += std::exp(x - m);
    for (int64_t tt = 0; tt < L; ++tt) {
      const double w = std::exp(sc[tt] - m) / z;
      for (int64_t d = 0; d < D; ++d) o[d] += w * elem(p, v_cache, rows[tt] + d);
    }
    return 0;
  });
}

}  // extern "C"
