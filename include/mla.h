/*
 * mla.h — C ABI of the B200 (sm_100a) paged latent-attention library.
 *
 * The operation (page "mstar.engine.resources.attn.flashinfer_mla": module
 * description, FlashInferMLAWrapper.plan / .run, FlashInferMLAManager.run):
 *
 *   The cache holds one latent row per token, [ckv (kv_lora_rank = 512) | kpe (64)],
 *   bf16, in pages of `page_size` tokens: cache[num_pages][page_size][576].
 *   Row b of a batch names its pages by kv_indices[kv_indptr[b] .. kv_indptr[b+1]);
 *   its last page holds last_page_len[b] tokens, so it has
 *       k_b = (n_b - 1) * page_size + last_page_len[b]   keys   (0 if n_b == 0).
 *   Its query tokens are t in [qo_indptr[b], qo_indptr[b+1]), q_b of them, each
 *   with H heads of absorbed query q_nope[t][h][512] (already multiplied by W_UK)
 *   and rope query q_pe[t][h][64] (used as given: the library rotates nothing).
 *   For query i of row b (0-based) and causal = 1, the visible keys are
 *       j < vis = clamp(k_b - q_b + i + 1, 0, k_b)
 *   (queries aligned to the END of the keys: page
 *   "mstar.engine.resources.attn.ragged.wrappers", PrefixedPrefillWrapper);
 *   with causal = 0, vis = k_b.
 *       s_j  = sm_scale * (q_nope[t][h] . ckv_j + q_pe[t][h] . kpe_j)
 *       lse  = ln sum_{j<vis} exp(s_j)                 (natural log)
 *       out  = sum_{j<vis} exp(s_j - lse) * ckv_j      (latent space, 512 wide)
 *   A query with vis == 0 gets out = 0 and lse = -inf.
 *   out is bf16 [T][H][512] (round to nearest even), lse is fp32 [T][H].
 *
 * Threading and streams: a plan belongs to the CUDA device that was current when it
 * was made; call mla_run with that device current.  Calls on one plan must not
 * overlap on the host.  Every function returns a status code; nothing throws,
 * traps or aborts.
 */
#ifndef PAGED_MLA_B200_H
#define PAGED_MLA_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MLA_OK = 0,
  MLA_ERR_INVALID_ARGUMENT = 1, /* bad pointer, size, index table or alignment      */
  MLA_ERR_UNSUPPORTED = 2,      /* shape outside mla_supports()                     */
  MLA_ERR_CUDA = 3,             /* a CUDA runtime/driver call failed                */
  MLA_ERR_OUT_OF_MEMORY = 4,    /* device or pinned host allocation failed          */
  MLA_ERR_DEVICE_TIMEOUT = 5    /* a bounded wait inside a kernel gave up           */
} mla_status;

/* Geometry and scale (page "mstar.engine.resources.attn.flashinfer_mla",
 * FlashInferMLAWrapper constructor: num_qo_heads, kv_lora_rank, qk_rope_head_dim,
 * page_size, max_num_pages, sm_scale — the scale of the ORIGINAL 192-wide head,
 * 192 ** -0.5 for the DeepSeek shape). */
typedef struct {
  int32_t num_heads;    /* H: local query heads; 16, 32, 64 or 128                 */
  int32_t kv_lora_rank; /* ckv width; must be 512                                  */
  int32_t rope_dim;     /* kpe width; must be 64                                   */
  int32_t page_size;    /* tokens per page; 16, 32, 64 or 128                      */
  int32_t num_pages;    /* pages in the cache pool (cache.shape[0]) , >= 1         */
  float sm_scale;       /* softmax scale applied to q.k; finite and > 0            */
} mla_dims;

/* Optional planning knobs; pass NULL for the defaults (all zero). */
typedef struct {
  int32_t split_keys;       /* 0: automatic split-KV; > 0: cut every key range into
                               chunks of this many keys (a multiple of MLA_KEY_TILE);
                               < 0: never split                                       */
  int32_t num_sms;          /* 0: query the device; > 0: plan for this many SMs       */
  uint64_t wait_timeout_ns; /* bound on every in-kernel wait; 0: 4 seconds            */
  int32_t debug_flags;      /* bit 0 (MLA_DEBUG_DROP_FIRST_KV_LOAD): the kernel never
                               loads its first key chunk, so the wait on it runs out and
                               the run reports MLA_ERR_DEVICE_TIMEOUT (tests the
                               timeout path without faulting anything)                */
  int32_t host_only;        /* 1: build the work lists on the host only, touching no
                               CUDA API (for inspecting a plan on a machine without a
                               GPU); such a plan can be described but not run         */
} mla_plan_options;

/* Keys per tile of the attention kernel: work items start on multiples of it. */
#define MLA_KEY_TILE 64

#define MLA_DEBUG_DROP_FIRST_KV_LOAD 1
#define MLA_DEBUG_KERNEL_TIMING 2 /* bit 1: mla_run records CUDA events around each of its
                                     launches (see mla_plan_kernel_times)              */

/* Counts describing a plan (for callers that size buffers, and for tests). */
typedef struct {
  int32_t batch;           /* rows B                                                  */
  int32_t total_tokens;    /* T = qo_indptr[B]                                        */
  int32_t num_work;        /* attention work items (one CTA pair each)                */
  int32_t num_merge;       /* query tiles whose keys were split                       */
  int32_t num_partials;    /* partial results the merge kernel combines               */
  int32_t num_sms;         /* SMs the plan was balanced for                           */
  int64_t workspace_bytes; /* plan-owned split-KV workspace                           */
} mla_plan_info;

typedef struct mla_plan_s* mla_plan_t; /* opaque ("immutable and opaque to runner":
                                          FlashInferMLAManager.plan)                 */

/* 1 if the library runs this shape on sm_100a, else 0.  The pages' kernel is
 * specialised to ckv 512 with kpe 0 or 64 (flashinfer_mla_supports); this library
 * implements kpe 64 only, H in {16, 32, 64, 128}, page_size in {16, 32, 64, 128}. */
int mla_supports(int kv_lora_rank, int rope_dim, int num_heads, int page_size);

/* Build a plan for one step (FlashInferMLAWrapper.plan: "inputs may be CPU tensors").
 *   qo_indptr     host int32 [batch + 1]; [0] == 0, nondecreasing
 *   kv_indptr     host int32 [batch + 1]; [0] == 0, nondecreasing
 *   kv_indices    host int32 [kv_indptr[batch]]; each in [0, num_pages); repeats are
 *                 allowed (rows sharing a prefix name the same pages)
 *   last_page_len host int32 [batch]; in [1, page_size] for a row with pages, ignored
 *                 (any value in [0, page_size]) for a row without
 *   causal        0 or 1
 *   stream        cudaStream_t (may be NULL) for the plan's uploads
 *   opts          NULL or knobs above
 *   out_plan      receives the plan
 * The library copies every host array; the caller may reuse them on return.  The plan
 * owns its device work lists, page table copy, split-KV workspace, status word and
 * pinned staging, so plans never share a staging buffer (the double-buffering hazard
 * described for FlashInferMLAManager.force_double_buffer cannot arise).
 * Errors: INVALID_ARGUMENT (bad tables or NULL), UNSUPPORTED (shape), OUT_OF_MEMORY,
 * CUDA.  On error *out_plan is NULL and nothing leaks. */
mla_status mla_plan(const mla_dims* dims, int32_t batch, const int32_t* qo_indptr,
                    const int32_t* kv_indptr, const int32_t* kv_indices,
                    const int32_t* last_page_len, int32_t causal, void* stream,
                    const mla_plan_options* opts, mla_plan_t* out_plan);

/* Run the attention of a plan (FlashInferMLAWrapper.run).
 *   q_nope  device bf16 [T][H][512], contiguous, 16-byte aligned
 *   q_pe    device bf16 [T][H][64], contiguous, 16-byte aligned
 *   cache   device bf16 [num_pages][page_size][576], contiguous, 16-byte aligned
 *   out     device bf16 [T][H][512], contiguous, 16-byte aligned (written)
 *   lse     device fp32 [T][H] or NULL (written when non-NULL)
 *   stream  cudaStream_t (may be NULL)
 * Enqueues one attention launch, plus one merge launch when the plan split keys.
 * Allocates nothing and never synchronises.  The caller keeps every buffer alive
 * until the stream has passed the work.  Errors: INVALID_ARGUMENT (NULL or misaligned
 * pointer), CUDA (launch failure).  In-kernel timeouts are reported by
 * mla_plan_check. */
mla_status mla_run(mla_plan_t plan, const void* q_nope, const void* q_pe, const void* cache,
                   void* out, float* lse, void* stream);

/* Wait for the plan's last run to finish and report (then clear) its device status
 * word: MLA_OK, or MLA_ERR_DEVICE_TIMEOUT when an in-kernel wait gave up. */
mla_status mla_plan_check(mla_plan_t plan);

/* Counts of a plan. */
mla_status mla_plan_get_info(mla_plan_t plan, mla_plan_info* info);

/* Copy the plan's bookkeeping to host arrays (each may be NULL):
 *   kv_len [batch]                      keys per row, k_b
 *   work   [num_work * MLA_WORK_FIELDS] one record per work item:
 *     { q_row0, n_rows, page_base, kv_len, key_begin, key_end, diag_base, partial }
 *     q_row0 = first (token * H + head) row of the 128-row query tile; n_rows valid
 *     rows; page_base = kv_indptr of the row; keys [key_begin, key_end) of the tile;
 *     row r of the tile sees keys < clamp(diag_base + r / H + 1, 0, kv_len);
 *     partial = -1 (written straight to out/lse) or the workspace slot.
 *   merge  [num_merge * MLA_MERGE_FIELDS] { q_row0, n_rows, first_partial, n_partials } */
#define MLA_WORK_FIELDS 8
#define MLA_MERGE_FIELDS 4
mla_status mla_plan_describe(mla_plan_t plan, int32_t* kv_len, int32_t* work, int32_t* merge);

/* Kernel durations of the plan's most recent runs, for plans made with
 * MLA_DEBUG_KERNEL_TIMING: each mla_run records events on its stream before the
 * attention launch, between the attention and merge launches, and after the merge.
 * Waits for the last run, then writes up to `capacity` entries, oldest first (the plan
 * keeps the last 256 runs): attn_ms[i] = attention kernel time, merge_ms[i] = merge
 * kernel time (0 when the plan has no split).  *count receives the number written.
 * Errors: INVALID_ARGUMENT (NULL, or a plan made without the flag), CUDA. */
mla_status mla_plan_kernel_times(mla_plan_t plan, int32_t capacity, float* attn_ms, float* merge_ms,
                                 int32_t* count);

/* Plan and run one step without allocating any memory (no paper counterpart: this is a
 * library-level entry point, not part of the method).
 *
 * For callers that cannot allocate when they run attention: serving processes whose
 * memory manager has handed all of HBM to its own pools and forbids other allocations,
 * plug-in hosts that give the library no allocator, and latency-critical loops where a
 * cudaMalloc/cudaFree could synchronise the device.  mla_plan allocates; this call does
 * not (no cudaMalloc, cudaFree or pinned allocation, and no heap use while planning).
 *
 * Arguments are those of mla_plan (host tables, copied during the call) followed by
 * those of mla_run (device tensors, same layouts and alignment rules).  Planning uses a
 * fixed split rule instead of mla_plan's balancing search, so the split points may
 * differ from mla_run's; results agree within floating-point tolerance.
 *
 * All device scratch (status word, work list, page-table copy, split-KV partials) lives
 * in one 16 MiB array compiled into the library; every GPU that loads the library holds
 * it until the process exits.  Limits: kv_indptr[batch] <= 524288 page ids and at most
 * 16384 query tiles (a tile is 128 / H tokens of one row); larger steps return
 * MLA_ERR_INVALID_ARGUMENT.  Long key ranges are split only while the array has room
 * for their partial results (at least 32 tiles' worth); the rest run unsplit.
 *
 * The first call on a device looks up the array's device address (and the SM count)
 * with that device current; make that first call before any stream capture.  Every call
 * shares the one array (and static host buffers), so calls must not overlap, on the host
 * or on the GPU: issue them from one thread, on one stream, or synchronise in between.
 * In-kernel wait timeouts are recorded in the array's status word, which is not
 * reported back; use mla_plan/mla_run/mla_plan_check where that matters.
 * Errors: INVALID_ARGUMENT (bad tables or pointers, or beyond the limits above),
 * UNSUPPORTED (shape), CUDA. */
mla_status mla_run_noalloc(const mla_dims* dims, int32_t batch, const int32_t* qo_indptr,
                           const int32_t* kv_indptr, const int32_t* kv_indices,
                           const int32_t* last_page_len, int32_t causal, const void* q_nope,
                           const void* q_pe, const void* cache, void* out, float* lse, void* stream);

/* Wait for the plan's last run, then free everything it owns.  NULL is a no-op. */
void mla_plan_destroy(mla_plan_t plan);

/* Static string for a status code. */
const char* mla_status_string(mla_status status);

#ifdef __cplusplus
}
#endif

#endif /* PAGED_MLA_B200_H */
