/*
 * pagedattn.h -- C ABI of libpagedattn.so: a paged KV cache for single-query
 * decode attention on NVIDIA B200 (sm_100a).
 *
 * The pages this follows:
 *   [card]   "PagedAttention" (llm-engineer.pages.dev, LLM inference / vLLM path)
 *   [vllm]   "vLLM KV Cache and PagedAttention Explained" (hrletsgo.me)
 *   [velog]  "vLLM의 PagedAttention 아키텍처와 GPU 메모리 최적화 원리" (velog.io, @min_tech)
 *
 * Cache layout ([velog] section 4): K and V are each one tensor
 *   [NB, H, S, D] = [num_blocks, num_heads, block_size, head_dim], D fastest,
 * so the S x D slab of one (block, head) is contiguous. Token t of a request
 * lives in physical block block_table[t / S] at offset t % S ([card]
 * "OS paging과 같은 발상"; [vllm] Step 5 "PagedAttention in vLLM"). A slot is
 * the integer block * S + offset ([vllm] Step 6 "Decode": "slot 6 of block 42").
 *
 * Conventions for every call:
 *   - Errors are return codes; nothing throws across the ABI. Arguments are
 *     validated on the host before anything is launched; a rejected call
 *     launches nothing and changes nothing.
 *   - Device calls take device pointers owned by the caller and enqueue work
 *     on `stream` (a cudaStream_t; NULL = the legacy default stream). They do
 *     not synchronise. They allocate no device memory.
 *   - Device-side range checks are always on: a block id outside [0, NB), a
 *     seq_len outside [0, MB * S] or a slot at or past NB * S is never
 *     dereferenced; the kernel skips it and sets a per-device error word that
 *     pa_get_device_error() reads and clears.
 *   - The host allocator is not thread-safe: one caller thread per pa_alloc.
 */
#ifndef PAGEDATTN_H
#define PAGEDATTN_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID = 1,      /* bad argument: null pointer, bad size, misalignment, unknown id */
  PA_ERR_OOM = 2,          /* the block pool cannot satisfy a grow; state unchanged */
  PA_ERR_OUT_OF_RANGE = 3, /* an index past an allocated range (or a device range check fired) */
  PA_ERR_CUDA = 4          /* a CUDA launch or copy failed */
} pa_status;

typedef enum { PA_F16 = 0, PA_BF16 = 1, PA_F32 = 2 } pa_dtype; /* PA_F32 only for decode output */

/* Bits of the device error word (pa_get_device_error). */
#define PA_DEVERR_BLOCK_ID 0x1u /* a block table entry outside [0, NB) was skipped */
#define PA_DEVERR_SEQ_LEN 0x2u  /* a seq_len outside [0, MB * S] was clamped */
#define PA_DEVERR_SLOT 0x4u     /* an append slot at or past NB * S was skipped */
#define PA_DEVERR_TIMEOUT 0x8u  /* a pipeline wait gave up after about one second */

/* Human-readable name of a status code (static storage). */
const char* pa_status_string(pa_status s);

/* ABI version of this library (major * 100 + minor). */
int pa_version(void);

/* ---------------------------------------------------------------------------
 * KV append: the slot_mapping scatter.
 * [vllm] Step 6 "Decode" / Step 7 item 5: the new token's K/V is stored in its
 * slot (slot 6 of block 42); Step 6 "Prefill": K1..K6/V1..V6 written to the cache.
 *
 *   k, v          [T, H, D] new tokens' keys and values, dtype `dt`, contiguous
 *   slot_mapping  [T] int64; token t goes to block slot/S, offset slot%S for
 *                 every head; a negative slot skips the token (padding). Slots
 *                 in one call must be distinct (duplicates: one of the writes wins)
 *   k_cache, v_cache  [NB, H, S, D], dtype `dt`, written in place
 *   dt            PA_F16 or PA_BF16
 * Requires D % 8 == 0 and 16-byte aligned k, v, k_cache, v_cache. T == 0 is a
 * no-op. Bit-exact copy: no arithmetic touches the values.
 * ------------------------------------------------------------------------- */
pa_status pa_kv_append(const void* k, const void* v, const int64_t* slot_mapping, void* k_cache,
                       void* v_cache, int T, int H, int D, int S, int NB, pa_dtype dt,
                       void* stream);

/* ---------------------------------------------------------------------------
 * Paged decode attention.
 * [vllm] "Appendix: The Attention Score Formula": out = softmax(q K^T * scale) V
 * for one query per (request, head), computed by walking the request's block
 * table and reading each physical block in place, with a running softmax
 * ([card] "Kernel은 무엇이 달라지는가": no gather into a contiguous tensor).
 * Long contexts are split into partitions of `partition` tokens whose partial
 * results are merged by a log-sum-exp reduce ([card] "헷갈리기 쉬운 구분":
 * FlashDecoding).
 *
 *   out           [B, H, D], dtype out_dt (PA_F32, PA_F16 or PA_BF16). fp16/bf16
 *                 output is the round-to-nearest-even of the fp32 result
 *   q             [B, H, D], dtype dt
 *   k_cache, v_cache [NB, H, S, D], dtype dt
 *   block_tables  [B, MB] int32; entries past ceil(seq_lens[i] / S) are never read
 *   seq_lens      [B] int32 on the device; request i attends to exactly its first
 *                 seq_lens[i] cached tokens; 0 gives an all-zero output row
 *   scale         multiplies q . k (1/sqrt(D) for the pages' formula)
 *   dt            PA_F16 or PA_BF16; D in {64, 128, 256}; S in {8, 16, 32}
 *   partition     0 = choose automatically, -1 = never split, > 0 = split into
 *                 partitions of this many tokens (a multiple of S)
 *   max_seq_len   a host-side upper bound on seq_lens (sizes the grid); must be
 *                 <= MB * S. Requests longer than it are clamped and flagged
 *   workspace     device scratch of ws_bytes >= pa_decode_workspace_bytes(...)
 *                 for the same arguments; may be NULL when that size is 0. It
 *                 needs no initialisation and may be reused by later calls of
 *                 any shape, but calls whose work overlaps on the GPU need
 *                 workspaces of their own. The library keeps no pointer to it
 *                 after the call's work ends
 * Requires 16-byte aligned q, k_cache, v_cache, out and workspace.
 * How a split is merged: an automatic split (partition = 0) into 2, 4 or 8
 * partitions whose grid (B * H * partitions CTAs) fits within two CTAs per SM
 * runs as thread-block clusters, one per (request, head), and partition 0
 * merges the others' results through distributed shared memory: the workspace
 * is still required but left untouched. Every other split leaves per-partition
 * results in the workspace (layout below) for a merge kernel. Both merges do
 * the same arithmetic in the same order: the output bits do not depend on
 * which one ran.
 * pa_decode_workspace_bytes: the workspace any decode entry point needs for
 * these arguments (H the query heads), the grouped-query plans of every Hkv
 * included (pa_decode_plan_grouped); 0 when nothing splits or the arguments
 * are bad.
 * ------------------------------------------------------------------------- */
size_t pa_decode_workspace_bytes(int B, int H, int D, int S, int max_seq_len, int partition);

/* The partition length (tokens) and the number of partitions pa_decode will use
 * for these arguments on the current device; *partition_tokens = 0 and
 * *num_partitions = 1 mean a single pass with no workspace. The automatic choice
 * (partition = 0) depends on B * H and the device's SM count: call this and
 * pa_decode_workspace_bytes with the device current that pa_decode will run on.
 * Automatic: 512-token partitions, halved (down to 64 tokens) while the grid
 * has fewer CTAs than the device has SMs, or for contexts of 32K tokens and
 * more doubled (up to 2048) while the grid keeps 8 CTAs per SM; a resulting
 * count of 3, 5, 6 or 7 is
 * then re-cut to the next (else the previous) power of two when that grid fits
 * within two CTAs per SM, so that the split merges inside clusters. */
pa_status pa_decode_plan(int B, int H, int D, int S, int max_seq_len, int partition,
                         int* partition_tokens, int* num_partitions);

/* The plan of pa_decode_gqa / pa_decode_gqa_fp8 with Hkv KV heads (H a multiple
 * of Hkv; Hkv == H gives pa_decode_plan). Their partition pass has
 * B * Hkv * ceil(H / Hkv / 16) CTAs per partition, so an automatic plan whose
 * 512-token grid holds at most two CTAs per SM halves the partitions (down to
 * 128 tokens, multiples of S) while the grid stays within that bound; other
 * grids take pa_decode_plan's choice. pa_decode_workspace_bytes(B, H, ...)
 * covers this plan for every Hkv. PA_ERR_INVALID for bad arguments. */
pa_status pa_decode_plan_grouped(int B, int H, int Hkv, int D, int S, int max_seq_len,
                                 int partition, int* partition_tokens, int* num_partitions);

pa_status pa_decode(void* out, pa_dtype out_dt, const void* q, const void* k_cache,
                    const void* v_cache, const int32_t* block_tables, int MB,
                    const int32_t* seq_lens, float scale, int B, int H, int D, int S, int NB,
                    pa_dtype dt, int partition, int max_seq_len, void* workspace,
                    size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * One decode step in one launch: append, then attend.
 * [vllm] 7단계 "전체 흐름 요약" and Step 6 "Decode": in every decode step the new
 * token's K/V is added to the cache and attention reads the cached K/V. For each
 * request i with L = seq_lens[i] >= 1, k_new[i] and v_new[i] ([B, H, D], dtype
 * dt) are written to the cache at token position L - 1 (physical block
 * block_tables[i][(L-1)/S], offset (L-1)%S), and out[i] is the attention over
 * the first L tokens, the new one included. The result, cache and output, is
 * bit for bit that of pa_kv_append with those slots followed by pa_decode with
 * the same arguments, with one launch fewer. Arguments are pa_decode's plus
 * k_new and v_new (16-byte aligned); the cache is written.
 * ------------------------------------------------------------------------- */
pa_status pa_decode_append(void* out, pa_dtype out_dt, const void* q, const void* k_new,
                           const void* v_new, void* k_cache, void* v_cache,
                           const int32_t* block_tables, int MB, const int32_t* seq_lens,
                           float scale, int B, int H, int D, int S, int NB, pa_dtype dt,
                           int partition, int max_seq_len, void* workspace, size_t ws_bytes,
                           void* stream);

/* ---------------------------------------------------------------------------
 * FP8 E4M3 KV cache (not on the pages, which keep K/V in 16-bit; a storage
 * extension that halves the bytes decode reads). The caches are [NB, H, S, D]
 * uint8 arrays of E4M3 codes ("fn" variant: sign bit 7, exponent bits 6-3 with
 * bias 7, mantissa bits 2-0, no infinities, largest magnitude 448), one fp32
 * scale per tensor: K = k_scale * e4m3(code), V = v_scale * e4m3(code).
 *
 * pa_kv_append_fp8: the slot_mapping scatter of pa_kv_append, storing each
 * element of k / v ([T, H, D], in_dt F16 or BF16, 16-byte aligned) as the code
 * of fp32(x / scale) -- one correctly rounded fp32 division, then round to
 * nearest even, magnitudes past 448 saturated. D a multiple of 16; scales
 * finite and > 0. Slots and errors as pa_kv_append.
 * ------------------------------------------------------------------------- */
pa_status pa_kv_append_fp8(const void* k, const void* v, pa_dtype in_dt,
                           const int64_t* slot_mapping, void* k_cache, void* v_cache,
                           float k_scale, float v_scale, int T, int H, int D, int S, int NB,
                           void* stream);

/* pa_decode over E4M3 caches: q [B, H, D] (q_dt F16 or BF16), out as pa_decode;
 * out[i, h] = softmax_t(scale * q . K_t) V_t with K_t, V_t dequantized as above
 * (k_scale is folded into the scores, v_scale into the output). D, S,
 * partition, workspace (pa_decode_workspace_bytes) and errors as pa_decode; one
 * KV head per query head. */
pa_status pa_decode_fp8(void* out, pa_dtype out_dt, const void* q, pa_dtype q_dt,
                        const void* k_cache, const void* v_cache, float k_scale, float v_scale,
                        const int32_t* block_tables, int MB, const int32_t* seq_lens, float scale,
                        int B, int H, int D, int S, int NB, int partition, int max_seq_len,
                        void* workspace, size_t ws_bytes, void* stream);

/* One decode step over E4M3 caches in one launch: pa_kv_append_fp8 of the new
 * tokens' rows, then pa_decode_fp8 ([vllm] 7단계 "전체 흐름 요약": the new token's
 * K/V is added to the cache, then attention reads the cache). For each request
 * i with L = seq_lens[i] >= 1, k_new[i] and v_new[i] ([B, H, D], dtype q_dt,
 * 16-byte aligned) are quantized with k_scale / v_scale as pa_kv_append_fp8
 * does and written at token position L - 1 (block block_tables[i][(L-1)/S],
 * offset (L-1)%S), and the attention over the request's L tokens sees them.
 * The output and the cache bytes are those of pa_kv_append_fp8 followed by
 * pa_decode_fp8, bit for bit. Other arguments, workspace and errors as
 * pa_decode_fp8; a request whose length is out of range appends nothing. */
pa_status pa_decode_append_fp8(void* out, pa_dtype out_dt, const void* q, pa_dtype q_dt,
                               const void* k_new, const void* v_new, void* k_cache,
                               void* v_cache, float k_scale, float v_scale,
                               const int32_t* block_tables, int MB, const int32_t* seq_lens,
                               float scale, int B, int H, int D, int S, int NB, int partition,
                               int max_seq_len, void* workspace, size_t ws_bytes, void* stream);

/* pa_decode_fp8 with grouped-query heads: H query heads share Hkv KV heads
 * (H % Hkv == 0), query head h reading KV head h / (H / Hkv) of the E4M3 caches
 * [NB, Hkv, S, D]. The products run on the tensor cores in f16 (E4M3 values
 * are f16 values; each query head is held in f16 after an exact power-of-two
 * scaling that keeps its largest element below 2^15, undone on its scores),
 * with fp32 accumulation; the softmax weights enter P.V as f16. Hkv == H is
 * pa_decode_fp8. Other arguments, workspace (pa_decode_workspace_bytes with H
 * the query heads) and errors as pa_decode_fp8; no fused append. */
pa_status pa_decode_gqa_fp8(void* out, pa_dtype out_dt, const void* q, pa_dtype q_dt,
                            const void* k_cache, const void* v_cache, float k_scale,
                            float v_scale, const int32_t* block_tables, int MB,
                            const int32_t* seq_lens, float scale, int B, int H, int Hkv, int D,
                            int S, int NB, int partition, int max_seq_len, void* workspace,
                            size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------
 * Paged prefill attention ("vLLM KV Cache and PagedAttention Explained", Step 6
 * "Prefill and Decode": every prompt token is processed at once, and each one
 * attends to the tokens before it and to itself; the attention formula of its
 * Appendix). Request i holds L = seq_lens[i] tokens in the cache, of which the
 * last n = q_start[i+1] - q_start[i] are new and already appended (for example
 * by pa_kv_append); the first L - n are context cached earlier (a plain prompt
 * has none). New token j of request i sits at position L - n + j and
 *   out[q_start[i] + j, h] = softmax_t(scale * q[q_start[i] + j, h] . K_t) V_t
 * over cache tokens t = 0 .. L - n + j, read through block_tables[i] as in
 * pa_decode; query head h reads KV head h / (H / Hkv).
 *
 * out        [T, H, D] device, out_dt (F32, F16, BF16), 16-byte aligned.
 * q          [T, H, D] device, dt (F16 or BF16), 16-byte aligned; the rows of
 *            all requests packed back to back.
 * k_cache,   [NB, Hkv, S, D] device, dt, 16-byte aligned; read only.
 * v_cache
 * block_tables [B, MB] int32 device; seq_lens [B] int32 device.
 * q_start    [B + 1] int32 device: q_start[0] = 0, non-decreasing, q_start[B] = T.
 * T          rows of q and out (host copy of q_start[B]).
 * max_q_len  host bound on q_start[i+1] - q_start[i]; sets the launch grid
 *            (at most 65535 * 128 = 8,388,480)
 * D          64, 128 or 256 (256: one 128-row query tile per CTA instead of two);
 *            S one of 8, 16, 32, 64, 128; NB * Hkv * S <= 2^31 - 1.
 * scale      finite and > 0 (the usual 1 / sqrt(D)).
 * The contraction runs on the tensor cores with fp32 accumulation; for bf16
 * the softmax weights enter the second product as two bf16 terms (value and
 * rounding residue), for f16 as one f16 term.
 * Errors: PA_ERR_INVALID for bad sizes, dtypes, null or misaligned pointers
 * (nothing launched); B, T or max_q_len of 0 is a no-op. On the device, a
 * request whose seq_lens/q_start are inconsistent (n < 0, n > L, L > MB * S,
 * rows outside [0, T), n > max_q_len) is skipped with PA_DEVERR_SEQ_LEN, a table
 * entry outside [0, NB) is skipped with PA_DEVERR_BLOCK_ID (that request's
 * output is then undefined), and a wait that exceeds about a second sets
 * PA_DEVERR_TIMEOUT; see pa_get_device_error. Asynchronous on `stream`.
 * ------------------------------------------------------------------------- */
pa_status pa_prefill(void* out, pa_dtype out_dt, const void* q, const void* k_cache,
                     const void* v_cache, const int32_t* block_tables, int MB,
                     const int32_t* seq_lens, const int32_t* q_start, float scale, int B, int H,
                     int Hkv, int D, int S, int NB, pa_dtype dt, int T, int max_q_len,
                     void* stream);

/* ---------------------------------------------------------------------------
 * Grouped-query decode (not on the pages, which have one KV head per query
 * head): the cache holds Hkv KV heads, [NB, Hkv, S, D]; q and out hold H query
 * heads, H a multiple of Hkv, and query head h reads KV head h / (H / Hkv)
 * (consecutive query heads share a KV head). For H > Hkv one CTA serves up to
 * 16 query heads of a KV head from one staged copy of each K/V unit (on the
 * tensor cores), so every K/V byte is read from HBM once per group of up to 16
 * heads. k_new, v_new
 * ([B, Hkv, D]) are optional together: when given, the step's new token is
 * appended at position seq_lens[i] - 1 first, exactly as pa_decode_append.
 * Everything else (dtypes, D, S, partition, workspace sized by
 * pa_decode_workspace_bytes(B, H, ...) with H the query heads, errors) is as
 * pa_decode, except that the automatic plan is pa_decode_plan_grouped's.
 * H == Hkv gives pa_decode / pa_decode_append bit for bit.
 * ------------------------------------------------------------------------- */
pa_status pa_decode_gqa(void* out, pa_dtype out_dt, const void* q, const void* k_new,
                        const void* v_new, void* k_cache, void* v_cache,
                        const int32_t* block_tables, int MB, const int32_t* seq_lens, float scale,
                        int B, int H, int Hkv, int D, int S, int NB, pa_dtype dt, int partition,
                        int max_seq_len, void* workspace, size_t ws_bytes, void* stream);

/* Split-KV workspace layout, for tests that inspect the partition pass
 * (NP = number of partitions, n = B*H*NP, all fp32, offsets in bytes from
 * `workspace`):
 *   m   [B, H, NP] at 0                 max of scale * q.k * log2(e) (base-2 units)
 *   l   [B, H, NP] at n*4               sum of 2^(s - m) over the partition
 *   acc [B, H, NP, D] at align256(n*8)  sum of 2^(s - m) * V, unnormalised
 * Only partitions p < ceil(seq_lens[i] / partition) of requests with more than
 * one partition are written; a second kernel, launched so that it can start
 * while the first finishes, merges them by log-sum-exp ([card] "헷갈리기 쉬운
 * 구분"). Everything the merge reads is written by the same call, so the
 * workspace needs no initialisation. (A split merged inside clusters, see
 * pa_decode, writes none of it.) */

/* ---------------------------------------------------------------------------
 * Decode without any caller-provided scratch. This entry point has no
 * counterpart on the pages: it exists for callers that cannot allocate device
 * memory themselves, such as a plugin whose host framework owns every device
 * allocation and offers it no allocator, or a serving process that fixes its
 * device-memory budget at start-up and must not call cudaMalloc afterwards
 * (an allocation at run time can synchronise the device and stall other
 * streams). It behaves exactly like pa_decode, with the same arguments minus
 * the workspace: the split-KV partials go to a static device array of
 * PA_NOALLOC_SCRATCH_BYTES that the library holds on every GPU that loads it,
 * until the process exits. The call allocates nothing.
 *   - The first call on a device that needs the array looks up its device
 *     address (cudaGetSymbolAddress) with the device current, and again
 *     whenever the device's context has changed (after a cudaDeviceReset);
 *     make that first call before any stream capture on the device.
 *   - Arguments are checked as pa_decode checks them, first: a bad argument
 *     returns PA_ERR_INVALID whatever the size of the split.
 *   - A call whose split needs more scratch than the array holds (see
 *     pa_decode_workspace_bytes) returns PA_ERR_OOM and launches nothing.
 *   - Every call shares the one array and leaves its partials there; nothing
 *     in it needs to start at zero (each call writes every partial it reads).
 *     Calls whose work overlaps on the GPU (other streams, other threads)
 *     race on the array: order them on one stream or serialise them.
 * ------------------------------------------------------------------------- */
#define PA_NOALLOC_SCRATCH_BYTES (16u << 20)

/* The size of that array as compiled into the library (PA_NOALLOC_SCRATCH_BYTES). */
size_t pa_noalloc_scratch_bytes(void);

pa_status pa_decode_noalloc(void* out, pa_dtype out_dt, const void* q, const void* k_cache,
                            const void* v_cache, const int32_t* block_tables, int MB,
                            const int32_t* seq_lens, float scale, int B, int H, int D, int S,
                            int NB, pa_dtype dt, int partition, int max_seq_len, void* stream);

/* Reads and clears the device error word of the current device after
 * synchronising `stream`. *flags receives PA_DEVERR_* bits (0 = clean).
 * Returns PA_OK, or PA_ERR_CUDA if the read failed. */
pa_status pa_get_device_error(void* stream, uint32_t* flags);

/* ---------------------------------------------------------------------------
 * Host block allocator ([vllm] 5단계, Step 5-8; [card] "무엇이 좋아지는가").
 * A pool of NB physical blocks of S tokens. Each sequence owns a block table
 * that grows on demand (ceil(len / S) blocks; a new block when the length
 * crosses a block boundary) and returns its blocks to the pool when freed.
 * The free list is a LIFO stack: growth pops ids one at a time and appends them
 * in pop order; a freed sequence pushes its ids back in logical order, so they
 * are the first handed out again. The library owns the state.
 * ------------------------------------------------------------------------- */
typedef struct pa_alloc pa_alloc;

/* initial_order: NULL, or a permutation of [0, NB) listing the order in which
 * ids are first handed out (NULL = 0, 1, 2, ...). Shuffling is the caller's
 * choice: pass a shuffled order. */
pa_status pa_alloc_create(int NB, int S, const int32_t* initial_order, pa_alloc** out);
void pa_alloc_destroy(pa_alloc* a);

/* Creates seq_id if unknown, then grows it to new_len tokens (new_len >= its
 * current length, else PA_ERR_INVALID). PA_ERR_OOM if the pool is short: the
 * state is then unchanged (an unknown seq_id is not created). */
pa_status pa_seq_grow(pa_alloc* a, int64_t seq_id, int new_len);

/* Returns every block of seq_id to the pool and forgets seq_id. */
pa_status pa_seq_free(pa_alloc* a, int64_t seq_id);

/* Current length (tokens) of seq_id. */
pa_status pa_seq_len(const pa_alloc* a, int64_t seq_id, int* len);

/* Copies seq_id's block table (logical order) into dst[0..cap); *n receives
 * its length. PA_ERR_OUT_OF_RANGE if cap is too small (nothing copied). */
pa_status pa_seq_block_table(const pa_alloc* a, int64_t seq_id, int32_t* dst, int cap, int* n);

/* Prefix sharing ([vllm] Step 9 "Safe Sharing with Copy-on-Write"): child
 * starts as parent's copy (same length, same physical blocks, every block's
 * reference count + 1). Blocks return to the pool when their count reaches 0.
 * When a sequence grows past its length while its last block is partly filled
 * and named by another table too, pa_seq_grow / pa_prepare_step first give it
 * a private block: a free block is taken, the (shared, private) pair is queued,
 * the sequence's table entry is repointed; the other tables keep the original.
 * The caller must copy the queued pairs on the device (pa_copy_blocks) before
 * the append that writes the new token. PA_ERR_INVALID if parent is unknown or
 * child exists. */
pa_status pa_seq_fork(pa_alloc* a, int64_t parent, int64_t child);

/* Moves the queued copy-on-write pairs, oldest first, into src_dst [cap, 2]
 * (int32: source block, destination block) and clears the queue; *n receives
 * the count. PA_ERR_OUT_OF_RANGE (nothing taken) if cap is too small. */
pa_status pa_alloc_take_copies(pa_alloc* a, int32_t* src_dst, int cap, int* n);

/* Copies the reference count of every block into dst[0..NB) (0 = free). */
pa_status pa_alloc_refcounts(const pa_alloc* a, int32_t* dst, int cap);

/* Device half of copy-on-write: for each of the n pairs in src_dst (device
 * int32 [n, 2]), copies physical block src to block dst in both caches, every
 * head, bit for bit. Destinations must be distinct and not sources of other
 * pairs. Ids outside [0, NB) are skipped and flagged (PA_DEVERR_BLOCK_ID).
 * Requires D % 8 == 0 and 16-byte aligned caches. */
pa_status pa_copy_blocks(void* k_cache, void* v_cache, const int32_t* src_dst, int n, int H,
                         int S, int D, int NB, pa_dtype dt, void* stream);

/* Host slot mapping: for each sequence k, tokens start_pos[k] .. start_pos[k]
 * + n_tok[k] - 1 are written to dst in order, as table[pos / S] * S + pos % S.
 * dst holds sum(n_tok) entries. PA_ERR_OUT_OF_RANGE if a position is not yet
 * allocated (grow first). */
pa_status pa_build_slot_mapping(const pa_alloc* a, const int64_t* seq_ids, const int* start_pos,
                                const int* n_tok, int n_seq, int64_t* dst);

/* Host-side check of a slot mapping before pa_kv_append / pa_kv_append_fp8
 * (which do not detect duplicates; with two tokens on one slot one write
 * wins): slots [T] host int64, n_slots = NB * S. Returns PA_OK if every
 * non-negative slot is below n_slots and no slot appears twice (negative
 * entries are padding); PA_ERR_OUT_OF_RANGE for a slot >= n_slots,
 * PA_ERR_INVALID for a repeated slot or bad arguments; *first_bad (optional)
 * receives the index of the offending entry (for a repeat, the later one). */
pa_status pa_check_slots(const int64_t* slots, int64_t T, int64_t n_slots, int64_t* first_bad);

/* Host block tables [n_seq, MB] int32, padded with -1. PA_ERR_OUT_OF_RANGE if
 * a table has more than MB blocks. */
pa_status pa_build_block_tables(const pa_alloc* a, const int64_t* seq_ids, int n_seq, int MB,
                                int32_t* dst);

/* One decode step's host work for n_seq sequences in one call: grows each
 * sequence by n_new tokens (all-or-nothing: on PA_ERR_OOM nothing changes),
 * then writes the new tokens' slots (dst_slots [n_seq * n_new], sequence-major),
 * the padded block tables (dst_tables [n_seq, MB]) and the new lengths
 * (dst_lens [n_seq]). Any of the three outputs may be NULL to skip it. */
pa_status pa_prepare_step(pa_alloc* a, const int64_t* seq_ids, int n_seq, int n_new, int MB,
                          int64_t* dst_slots, int32_t* dst_tables, int32_t* dst_lens);

/* Pool statistics: free blocks, tokens held (sum of lengths) and empty slots in
 * held blocks (the tail waste of [vllm] Step 5 "Why Waste Stays Below 4%"),
 * counted per sequence (a shared block counts once per table naming it). */
pa_status pa_alloc_stats(const pa_alloc* a, int* free_blocks, int64_t* used_slots,
                         int64_t* wasted_slots);

/* Copies the free list, bottom of the stack first (the last entry is handed out
 * next), into dst[0..cap); *n receives its length. For bit-exact tests. */
pa_status pa_alloc_dump(const pa_alloc* a, int32_t* free_list, int cap, int* n);

/* ---------------------------------------------------------------------------
 * Host-fed decode step executor ([vllm] 7단계 "전체 흐름 요약", Step 8; [card]
 * "vLLM에서의 위치": the worker turns the scheduler's block tables into device
 * tensors each step). For a fixed batch of B running sequences whose per-step
 * q, k, v arrive in host memory, one pa_stepper_step call grows every sequence
 * by one token on the allocator (pa_prepare_step), uploads q|k|v and the
 * tables and lengths, runs the decode with the append, and downloads the
 * output. Transfers go on the executor's own copy stream and every staging
 * buffer is `depth` sets deep, so a step's transfers overlap its neighbours'
 * kernels. Unlike the calls above, the executor allocates: at creation it
 * takes pinned host memory and device memory for its staging (depth sets of
 * q|k|v, tables, lengths, output, plus the split-KV workspace) and a CUDA
 * stream; pa_stepper_destroy releases them. Not thread-safe.
 * ------------------------------------------------------------------------- */
typedef struct pa_stepper pa_stepper;

/* k_cache, v_cache [NB, H, S, D] (dtype dt) and the allocator `alloc` stay
 * owned by the caller and must outlive the executor. max_len bounds every
 * sequence length the executor will decode (sizes the workspace; <= MB * S).
 * fused != 0 uses pa_decode_append, 0 uses pa_kv_append + pa_decode. depth in
 * [1, 8]. compute_stream: the stream the kernels run on (NULL = legacy). */
pa_status pa_stepper_create(pa_alloc* alloc, void* k_cache, void* v_cache, int B, int H, int D,
                            int S, int NB, int MB, pa_dtype dt, pa_dtype out_dt, float scale,
                            int max_len, int partition, int fused, int depth,
                            void* compute_stream, pa_stepper** out);
void pa_stepper_destroy(pa_stepper* s);

/* Enqueues one step for seq_ids[0..B) (each must exist in the allocator and
 * grows by one token). h_qkv: host memory (pinned, for the copy to overlap)
 * holding q, k, v as [3, B, H, D], read by the upload; it must stay unchanged
 * until the step's upload has run, i.e. until the next call that reuses the
 * step's staging set (depth steps later) returns, or pa_stepper_output.
 * *step_out receives the step's number, *max_len_out its longest sequence.
 * PA_ERR_OUT_OF_RANGE (nothing changed) if a sequence would exceed max_len. */
pa_status pa_stepper_step(pa_stepper* s, const int64_t* seq_ids, const void* h_qkv,
                          int64_t* step_out, int* max_len_out);

/* Waits for step `step`'s download and returns the host address of its output
 * [B, H, D] (dtype out_dt), valid until the call that reuses its staging set.
 * PA_ERR_OUT_OF_RANGE if that step is not among the last `depth` steps. */
pa_status pa_stepper_output(pa_stepper* s, int64_t step, const void** host_out);

/* Makes the compute stream wait for every outstanding download. */
pa_status pa_stepper_drain(pa_stepper* s);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDATTN_H */
