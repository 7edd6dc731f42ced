// Host-fed decode step executor: the runtime around the decode kernels for a
// batch whose per-step inputs arrive in host memory.
//
// "vLLM KV Cache and PagedAttention Explained", 7단계 "전체 흐름 요약" and Step 8:
// every decode step grows each running request by one token (a new block at a
// block boundary), writes the new token's K/V into the cache and attends over
// the cached tokens. The worker side of that step ("PagedAttention" card,
// "vLLM에서의 위치": the worker turns block tables into device tensors) is
// what this file does, natively: one call per step runs the host allocator,
// uploads q/k/v and the tables, launches the decode and downloads the result,
// with the transfers of neighbouring steps overlapped with the kernels:
//
//   host   : pa_prepare_step -> staging set n % depth (once its upload of step n - depth landed)
//   up     : wait compute(n - depth); upload q|k|v, tables|lengths (| slots); record up(n)
//   compute: wait up(n), down(n - depth); pa_decode_append (or pa_kv_append + pa_decode);
//            record compute(n)
//   down   : wait compute(n); download out(n); record down(n)
//
// Uploads and downloads go on two streams of their own (and so on the two copy
// engines): on one shared stream the upload of step n would queue behind the
// download of step n - 1, which waits for step n - 1's kernels, and every step
// would pay compute + download + upload in series.
//
// The executor owns its staging: pinned host and device buffers allocated at
// creation and freed at destruction. Every copy is one cudaMemcpyAsync.

#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstring>
#include <new>
#include <vector>

#include "pagedattn.h"

namespace {

struct Set {
  int64_t* h_slots = nullptr;
  int32_t* h_meta = nullptr;  // tables [B, MB] then lengths [B]
  void* h_out = nullptr;
  void* d_qkv = nullptr;      // q, k, v [3, B, H, D]
  int64_t* d_slots = nullptr;
  int32_t* d_meta = nullptr;
  void* d_out = nullptr;
  cudaEvent_t ev_up = nullptr, ev_compute = nullptr, ev_down = nullptr;
  int64_t step = -1;          // the step whose data this set holds
};

size_t elem_size(pa_dtype dt) { return dt == PA_F32 ? 4 : 2; }

}  // namespace

struct pa_stepper {
  pa_alloc* alloc = nullptr;
  int B = 0, H = 0, D = 0, S = 0, NB = 0, MB = 0, max_len = 0, partition = 0;
  bool fused = true;
  pa_dtype dt = PA_BF16, out_dt = PA_BF16;
  void* k_cache = nullptr;
  void* v_cache = nullptr;
  float scale = 0.f;
  cudaStream_t compute = nullptr, up = nullptr, down = nullptr;
  void* ws = nullptr;
  size_t ws_bytes = 0;
  std::vector<Set> sets;
  int64_t n = 0;

  size_t qkv_bytes() const { return 3ull * B * H * D * elem_size(dt); }
  size_t meta_bytes() const { return (static_cast<size_t>(B) * MB + B) * sizeof(int32_t); }
  size_t out_bytes() const { return static_cast<size_t>(B) * H * D * elem_size(out_dt); }
};

namespace {

void release(pa_stepper* s) {
  for (Set& t : s->sets) {
    cudaFreeHost(t.h_slots);
    cudaFreeHost(t.h_meta);
    cudaFreeHost(t.h_out);
    cudaFree(t.d_qkv);
    cudaFree(t.d_slots);
    cudaFree(t.d_meta);
    cudaFree(t.d_out);
    if (t.ev_up) cudaEventDestroy(t.ev_up);
    if (t.ev_compute) cudaEventDestroy(t.ev_compute);
    if (t.ev_down) cudaEventDestroy(t.ev_down);
  }
  cudaFree(s->ws);
  if (s->up) cudaStreamDestroy(s->up);
  if (s->down) cudaStreamDestroy(s->down);
  delete s;
}

}  // namespace

extern "C" {

pa_status pa_stepper_create(pa_alloc* alloc, void* k_cache, void* v_cache, int B, int H, int D,
                            int S, int NB, int MB, pa_dtype dt, pa_dtype out_dt, float scale,
                            int max_len, int partition, int fused, int depth,
                            void* compute_stream, pa_stepper** out) {
  if (!out) return PA_ERR_INVALID;
  *out = nullptr;
  if (!alloc || !k_cache || !v_cache || B <= 0 || H <= 0 || NB <= 0 || MB <= 0 || depth < 1 ||
      depth > 8 || max_len < 0 || max_len > static_cast<int64_t>(MB) * S)
    return PA_ERR_INVALID;
  if ((dt != PA_F16 && dt != PA_BF16) || (out_dt != PA_F16 && out_dt != PA_BF16 && out_dt != PA_F32))
    return PA_ERR_INVALID;
  int P = 0, NP = 0;
  if (pa_decode_plan(B, H, D, S, max_len, partition, &P, &NP) != PA_OK) return PA_ERR_INVALID;
  pa_stepper* s = new (std::nothrow) pa_stepper;
  if (!s) return PA_ERR_OOM;
  s->alloc = alloc;
  s->B = B, s->H = H, s->D = D, s->S = S, s->NB = NB, s->MB = MB;
  s->max_len = max_len, s->partition = partition, s->fused = fused != 0;
  s->dt = dt, s->out_dt = out_dt, s->k_cache = k_cache, s->v_cache = v_cache, s->scale = scale;
  s->compute = static_cast<cudaStream_t>(compute_stream);
  bool ok = cudaStreamCreateWithFlags(&s->up, cudaStreamNonBlocking) == cudaSuccess &&
            cudaStreamCreateWithFlags(&s->down, cudaStreamNonBlocking) == cudaSuccess;
  s->ws_bytes = pa_decode_workspace_bytes(B, H, D, S, max_len, partition);
  if (ok && s->ws_bytes) ok = cudaMalloc(&s->ws, s->ws_bytes) == cudaSuccess;
  s->sets.resize(static_cast<size_t>(depth));
  for (Set& t : s->sets) {
    if (!ok) break;
    ok = cudaMallocHost(reinterpret_cast<void**>(&t.h_slots), sizeof(int64_t) * B) == cudaSuccess &&
         cudaMallocHost(reinterpret_cast<void**>(&t.h_meta), s->meta_bytes()) == cudaSuccess &&
         cudaMallocHost(&t.h_out, s->out_bytes()) == cudaSuccess &&
         cudaMalloc(&t.d_qkv, s->qkv_bytes()) == cudaSuccess &&
         cudaMalloc(reinterpret_cast<void**>(&t.d_slots), sizeof(int64_t) * B) == cudaSuccess &&
         cudaMalloc(reinterpret_cast<void**>(&t.d_meta), s->meta_bytes()) == cudaSuccess &&
         cudaMalloc(&t.d_out, s->out_bytes()) == cudaSuccess &&
         cudaEventCreateWithFlags(&t.ev_up, cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&t.ev_compute, cudaEventDisableTiming) == cudaSuccess &&
         cudaEventCreateWithFlags(&t.ev_down, cudaEventDisableTiming) == cudaSuccess;
  }
  if (!ok) {
    release(s);
    return PA_ERR_CUDA;
  }
  *out = s;
  return PA_OK;
}

void pa_stepper_destroy(pa_stepper* s) {
  if (!s) return;
  if (s->up) cudaStreamSynchronize(s->up);
  if (s->down) cudaStreamSynchronize(s->down);
  cudaStreamSynchronize(s->compute);
  release(s);
}

pa_status pa_stepper_step(pa_stepper* s, const int64_t* seq_ids, const void* h_qkv,
                          int64_t* step_out, int* max_len_out) {
  if (!s || !seq_ids || !h_qkv) return PA_ERR_INVALID;
  Set& t = s->sets[static_cast<size_t>(s->n % static_cast<int64_t>(s->sets.size()))];
  if (t.step >= 0 && cudaEventSynchronize(t.ev_up) != cudaSuccess) return PA_ERR_CUDA;
  const int B = s->B, MB = s->MB;
  // refuse before anything changes if a request would outgrow the sized workspace
  for (int k = 0; k < B; ++k) {
    int len = 0;
    if (pa_status st = pa_seq_len(s->alloc, seq_ids[k], &len)) return st;
    if (len + 1 > s->max_len) return PA_ERR_OUT_OF_RANGE;
  }
  int32_t* h_tables = t.h_meta;
  int32_t* h_lens = t.h_meta + static_cast<size_t>(B) * MB;
  if (pa_status st = pa_prepare_step(s->alloc, seq_ids, B, 1, MB, t.h_slots, h_tables, h_lens))
    return st;
  int max_len = 0;
  for (int k = 0; k < B; ++k) max_len = std::max(max_len, h_lens[k]);
  bool ok = true;
  if (t.step >= 0) ok = cudaStreamWaitEvent(s->up, t.ev_compute, 0) == cudaSuccess;
  ok = ok && cudaMemcpyAsync(t.d_qkv, h_qkv, s->qkv_bytes(), cudaMemcpyHostToDevice, s->up) ==
                 cudaSuccess;
  ok = ok && cudaMemcpyAsync(t.d_meta, t.h_meta, s->meta_bytes(), cudaMemcpyHostToDevice,
                             s->up) == cudaSuccess;
  if (!s->fused)
    ok = ok && cudaMemcpyAsync(t.d_slots, t.h_slots, sizeof(int64_t) * B, cudaMemcpyHostToDevice,
                               s->up) == cudaSuccess;
  ok = ok && cudaEventRecord(t.ev_up, s->up) == cudaSuccess;
  ok = ok && cudaStreamWaitEvent(s->compute, t.ev_up, 0) == cudaSuccess;
  // the kernels overwrite this set's device output: its previous download must be done
  if (t.step >= 0) ok = ok && cudaStreamWaitEvent(s->compute, t.ev_down, 0) == cudaSuccess;
  if (!ok) return PA_ERR_CUDA;
  const size_t plane = static_cast<size_t>(B) * s->H * s->D * elem_size(s->dt);
  uint8_t* qkv = static_cast<uint8_t*>(t.d_qkv);
  const int32_t* d_tables = t.d_meta;
  const int32_t* d_lens = t.d_meta + static_cast<size_t>(B) * MB;
  pa_status st;
  if (s->fused) {
    st = pa_decode_append(t.d_out, s->out_dt, qkv, qkv + plane, qkv + 2 * plane, s->k_cache,
                          s->v_cache, d_tables, MB, d_lens, s->scale, B, s->H, s->D, s->S, s->NB,
                          s->dt, s->partition, max_len, s->ws, s->ws_bytes, s->compute);
  } else {
    st = pa_kv_append(qkv + plane, qkv + 2 * plane, t.d_slots, s->k_cache, s->v_cache, B, s->H,
                      s->D, s->S, s->NB, s->dt, s->compute);
    if (st == PA_OK)
      st = pa_decode(t.d_out, s->out_dt, qkv, s->k_cache, s->v_cache, d_tables, MB, d_lens,
                     s->scale, B, s->H, s->D, s->S, s->NB, s->dt, s->partition, max_len, s->ws,
                     s->ws_bytes, s->compute);
  }
  if (st != PA_OK) return st;
  ok = cudaEventRecord(t.ev_compute, s->compute) == cudaSuccess &&
       cudaStreamWaitEvent(s->down, t.ev_compute, 0) == cudaSuccess &&
       cudaMemcpyAsync(t.h_out, t.d_out, s->out_bytes(), cudaMemcpyDeviceToHost, s->down) ==
           cudaSuccess &&
       cudaEventRecord(t.ev_down, s->down) == cudaSuccess;
  if (!ok) return PA_ERR_CUDA;
  t.step = s->n;
  if (step_out) *step_out = s->n;
  if (max_len_out) *max_len_out = max_len;
  ++s->n;
  return PA_OK;
}

pa_status pa_stepper_output(pa_stepper* s, int64_t step, const void** host_out) {
  if (!s || !host_out || step < 0) return PA_ERR_INVALID;
  const Set& t = s->sets[static_cast<size_t>(step % static_cast<int64_t>(s->sets.size()))];
  if (t.step != step) return PA_ERR_OUT_OF_RANGE;  // not issued yet, or already overwritten
  if (cudaEventSynchronize(t.ev_down) != cudaSuccess) return PA_ERR_CUDA;
  *host_out = t.h_out;
  return PA_OK;
}

pa_status pa_stepper_drain(pa_stepper* s) {
  if (!s) return PA_ERR_INVALID;
  for (const Set& t : s->sets)
    if (t.step >= 0 && cudaStreamWaitEvent(s->compute, t.ev_down, 0) != cudaSuccess)
      return PA_ERR_CUDA;
  return PA_OK;
}

}  // extern "C"
