/*
 * mla.h — C ABI of the B200 (sm_100a) paged latent-attention library.
 *
 * The operation (page "mstar.engine.resources.attn.flashinfer_mla": module
 * description, FlashInferMLAWrapper.plan / .run, FlashInferMLAManager.run):
 *
 *   The cache holds one latent row per token, [ckv (kv_lora_rank = 512) | kpe (rope_dim
 *   = 64, or 0)], bf16, in pages of `page_size` tokens: cache[num_pages][page_size][D],
 *   D = 512 + rope_dim (576 for the DeepSeek shape).
 *   Row b of a batch names its pages by kv_indices[kv_indptr[b] .. kv_indptr[b+1]);
 *   its last page holds last_page_len[b] tokens, so it has
 *       k_b = (n_b - 1) * page_size + last_page_len[b]   keys   (0 if n_b == 0).
 *   Its query tokens are t in [qo_indptr[b], qo_indptr[b+1]), q_b of them, each
 *   with H heads of absorbed query q_nope[t][h][512] (already multiplied by W_UK)
 *   and rope query q_pe[t][h][rope_dim] (used as given: the library rotates nothing).
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
  int32_t rope_dim;     /* kpe width: 64, or 0 (no rope part: q_pe is not read)   */
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
  /* Graph bucket (FlashInferMLAWrapper: use_cuda_graph with a batch_size fixed for the
   * wrapper's life; base page: captured_page_capacity).  When graph_max_tokens > 0 the
   * plan is a GRAPH PLAN: its device buffers and the launch shapes of mla_run and
   * mla_append_kv are fixed for a bucket of at most graph_max_batch rows,
   * graph_max_tokens query tokens and graph_max_page_ids page ids, so that a CUDA graph
   * captured around mla_run replays correctly after mla_plan_update has re-planned the
   * plan in place for another step of the bucket.  Unused launch slots are empty work
   * items that return at once.  Every per-token buffer given to a graph plan (q_nope,
   * q_pe, out, lse, kv_new) holds graph_max_tokens tokens; a step's T tokens are its
   * first T.  All three bounds must be > 0 together.                                  */
  int32_t graph_max_batch;
  int32_t graph_max_tokens;
  int32_t graph_max_page_ids;
  /* 1: a CONTEXT-ONLY plan (FlashInferMLAManager.kv_len_buf): each row's queries attend
   * only the row's stored context, keys j < c_b = k_b - q_b, all of which precede every
   * query, so no causal mask applies; mla_plan_describe's kv_len reports c_b.  The page
   * tables still cover the step's own q_b entries (mla_append_kv writes them at
   * positions c_b + i).  Requires k_b >= q_b on every row.  The caller merges the
   * result with an attention over the step's own tokens (mla_merge_state).          */
  int32_t context_only;
  /* 1: SHARED-PREFIX CASCADE.  Consecutive rows whose page lists begin with the same
   * page ids (base page: captured_page_capacity, "rows that matched one cached prefix
   * all name its pages") attend that shared prefix together: one work item per 128
   * query rows of the whole group covers the prefix keys, its partial results are
   * merged by log-sum-exp with each row's own suffix.  Applies where the shared prefix
   * spans at least MLA_KEY_TILE keys, every query of the group sees all of it, and one
   * prefix tile packs the query tiles of two or more rows (H * q_b <= 64): with 128
   * heads a token already fills a tile, so a prefix tile would only add a merge.     */
  int32_t cascade;
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
  int64_t workspace_bytes; /* split-KV workspace in use                               */
  int32_t num_merge_refs;  /* entries of the merge reference list                     */
  int32_t num_cascade;     /* work items that attend a shared prefix for a row group  */
  int32_t graph;           /* 1 for a graph plan                                      */
  int32_t work_capacity;   /* launch slots of the attention grid (num_work unless a
                              graph plan)                                             */
} mla_plan_info;

typedef struct mla_plan_s* mla_plan_t; /* opaque ("immutable and opaque to runner":
                                          FlashInferMLAManager.plan)                 */

/* 1 if the library runs this shape on sm_100a, else 0.  The pages' kernel is
 * specialised to ckv 512 with kpe 0 or 64 (flashinfer_mla_supports); so is this
 * library, with H in {16, 32, 64, 128} and page_size in {16, 32, 64, 128}. */
int mla_supports(int kv_lora_rank, int rope_dim, int num_heads, int page_size);

/* Build a plan for one step (FlashInferMLAWrapper.plan: "inputs may be CPU tensors").
 *   qo_indptr     host int32 [batch + 1]; [0] == 0, nondecreasing
 *   kv_indptr     host int32 [batch + 1]; [0] == 0, nondecreasing
 *   kv_indices    host int32 [kv_indptr[batch]]; each in [0, num_pages); repeats are
 *                 allowed (rows sharing a prefix name the same pages)
 *   last_page_len host int32 [batch]; in [1, page_size] for a row with pages, ignored
 *                 (any value in [0, page_size]) for a row without
 *   causal        0 or 1
 *   stream        cudaStream_t (may be NULL) for the plan's uploads; a run on another
 *                 stream must be ordered after them by the caller (an event recorded
 *                 on `stream` after this call, or after later work of `stream`)
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
 *   q_pe    device bf16 [T][H][64], contiguous, 16-byte aligned (NULL allowed when
 *           rope_dim is 0: it is not read)
 *   cache   device bf16 [num_pages][page_size][512 + rope_dim], contiguous, 16-byte
 *           aligned
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
 * word: MLA_OK, or MLA_ERR_DEVICE_TIMEOUT when an in-kernel wait gave up.  The kernel
 * that records the first error also writes it to a host-mapped copy, which this call
 * reads: no device-to-host copy, so it waits for the plan's launches only, not for
 * copies other streams have queued. */
mla_status mla_plan_check(mla_plan_t plan);

/* Counts of a plan. */
mla_status mla_plan_get_info(mla_plan_t plan, mla_plan_info* info);

/* Copy the plan's bookkeeping to host arrays (each may be NULL):
 *   kv_len [batch]                      keys per row: k_b, or c_b = k_b - q_b for a
 *                                       context-only plan
 *   work   [num_work * MLA_WORK_FIELDS] one record per work item:
 *     { q_row0, n_rows, page_base, kv_len, key_begin, key_end, diag_base, partial }
 *     q_row0 = first (token * H + head) row of the query tile, n_rows its rows (at most
 *     128; a cascade item's rows may span several batch rows of one group, every other
 *     item's lie in one row); page_base = the kv_indptr entry whose pages the item
 *     reads; kv_len = keys addressable from there; keys [key_begin, key_end);
 *     row r of the tile sees keys < clamp(diag_base + r / H + 1, 0, kv_len);
 *     partial = -1 (written straight to out/lse) or the first workspace row of the
 *     item's partial result (its row r lands in workspace row partial + r).
 *   merge  [num_merge * MLA_MERGE_FIELDS] { q_row0, n_rows, first_ref, n_refs }: output
 *     rows [q_row0, q_row0 + n_rows) combine the n_refs partial results whose row 0 is
 *     workspace row refs[first_ref + i].
 *   refs   [num_merge_refs]             the merge reference list. */
#define MLA_WORK_FIELDS 8
#define MLA_MERGE_FIELDS 4
mla_status mla_plan_describe(mla_plan_t plan, int32_t* kv_len, int32_t* work, int32_t* merge, int32_t* refs);

/* Re-plan a plan for another step, in place (base page: PlanCacheKey, "when it is
 * unchanged between steps the re-plan is skippable"; FlashInferMLAWrapper.plan).
 * Arguments as for mla_plan; dims, causal and options stay those of the plan.
 *   *reused (may be NULL) receives 1 when the tables equal those of the plan's current
 *   step (same batch, qo_indptr, kv_indptr, kv_indices and last_page_len): nothing is
 *   planned or uploaded.  Otherwise 0: the plan is rebuilt and its device lists are
 *   rewritten by an upload enqueued on `stream`, so runs enqueued on that stream
 *   before the call see the old step and runs after it the new one.
 * A graph plan keeps every device address and launch shape: a CUDA graph that captured
 * mla_run (or mla_append_kv) on it replays the new step.  The step must fit the bucket
 * (batch, tokens and page ids within the graph bounds), else INVALID_ARGUMENT and the
 * plan is unchanged.  Other plans may grow their buffers (waiting for their last run
 * first when they do).  The host staging is double-buffered: the call waits only for
 * the upload of two updates ago, so the host may run one step ahead of the GPU
 * (FlashInferMLAManager.force_double_buffer describes the race this avoids).  It must
 * not be called while `stream` is being captured into a graph (the upload belongs to
 * the moment of re-planning, not to every replay): INVALID_ARGUMENT.
 * Errors: INVALID_ARGUMENT, OUT_OF_MEMORY, CUDA; on error the plan still describes and
 * runs its previous step. */
mla_status mla_plan_update(mla_plan_t plan, int32_t batch, const int32_t* qo_indptr, const int32_t* kv_indptr,
                           const int32_t* kv_indices, const int32_t* last_page_len, void* stream,
                           int32_t* reused);

/* Write the step's latent rows into their cache slots (base page: AttentionManager
 * .requires_kv_write, "a layer must write this step's K/V through the KV resource
 * before calling run").  Token i of row b (t = qo_indptr[b] + i) is key position
 * k_b - q_b + i of its row, i.e. slot (k_b - q_b + i) mod page_size of page
 * kv_indices[kv_indptr[b] + (k_b - q_b + i) / page_size]:
 *   kv_new  device bf16 [T][512 + rope_dim] ([ckv | kpe] per token), contiguous,
 *           16-byte aligned
 *   cache   device bf16 [num_pages][page_size][512 + rope_dim] (written at those slots
 *           only)
 * One launch, no allocation, no synchronisation.  Where several tokens name the same
 * slot (a page listed twice), the latest of them (highest t) is the one written: the
 * plan gives the earlier ones no destination, so no two writes race on a slot.
 * Errors: INVALID_ARGUMENT (NULL
 * or misaligned pointer, or a row with q_b > k_b, whose tokens have no slots), CUDA. */
mla_status mla_append_kv(mla_plan_t plan, const void* kv_new, void* cache, void* stream);

/* mla_append_kv followed by mla_run, as one enqueue: the attention launch is a
 * programmatic dependent of the append launch, so its set-up (barriers, tensor memory,
 * query tiles) overlaps the append and only its key loads wait for the append's
 * writes.  Arguments and errors as for the two calls. */
mla_status mla_run_append(mla_plan_t plan, const void* q_nope, const void* q_pe, const void* kv_new, void* cache,
                          void* out, float* lse, void* stream);

/* Merge two attention states over disjoint key sets by their log-sum-exps
 * (FlashInferMLAManager.run: "the natural log-sum-exp of the scores ... for merging with
 * another key segment"):
 *   M = max(lse_a, lse_b);  w_x = exp(lse_x - M);
 *   out = (w_a out_a + w_b out_b) / (w_a + w_b);  lse = M + ln(w_a + w_b)
 * with a state whose lse is -inf contributing nothing (both -inf: out = 0, lse = -inf).
 *   out_a, out_b, out   device bf16 [rows][512], 16-byte aligned (out may alias either)
 *   lse_a, lse_b        device fp32 [rows]
 *   lse                 device fp32 [rows] or NULL
 * Errors: INVALID_ARGUMENT (NULL or misaligned pointer, rows < 0), CUDA. */
mla_status mla_merge_state(const void* out_a, const float* lse_a, const void* out_b, const float* lse_b, void* out,
                           float* lse, int64_t rows, void* stream);

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
 * those of mla_run (device tensors, same layouts and alignment rules).  Planning follows
 * mla_plan's split rule within the fixed scratch below (long rows beyond its room run
 * unsplit), so the split points may differ from mla_run's; results agree within
 * floating-point tolerance.  No graph, context-only or cascade options.
 *
 * All device scratch (status word, work list, page-table copy, split-KV partials) lives
 * in one 16 MiB array compiled into the library; every GPU that loads the library holds
 * it until the process exits.  Limits: kv_indptr[batch] <= 524288 page ids and at most
 * 16384 query tiles (a tile is 128 / H tokens of one row); larger steps return
 * MLA_ERR_INVALID_ARGUMENT.  Long key ranges are split only while the array has room
 * for their partial results (at least 32 tiles' worth); the rest run unsplit.
 *
 * The first call on a device looks up the array's device address (and the SM count)
 * with that device current.  Every call shares the one array (and static host
 * buffers), so calls must not overlap, on the host or on the GPU: issue them from one
 * thread, on one stream, or synchronise in between.  The call cannot be captured into a
 * CUDA graph (its uploads read static host buffers at enqueue time): on a capturing
 * stream it returns MLA_ERR_UNSUPPORTED and enqueues nothing.
 *   status_out  device int32 or NULL.  When given, it receives the call's device status
 *               once the stream has passed the call: 0, or MLA_ERR_DEVICE_TIMEOUT in its
 *               low byte when an in-kernel wait gave up (the bits above name the wait).
 *               Read it after synchronising; the call only writes it.
 * Errors: INVALID_ARGUMENT (bad tables or pointers, or beyond the limits above),
 * UNSUPPORTED (shape, or a capturing stream), CUDA. */
mla_status mla_run_noalloc(const mla_dims* dims, int32_t batch, const int32_t* qo_indptr,
                           const int32_t* kv_indptr, const int32_t* kv_indices,
                           const int32_t* last_page_len, int32_t causal, const void* q_nope,
                           const void* q_pe, const void* cache, void* out, float* lse, void* stream,
                           int32_t* status_out);

/* Wait for the plan's last run, then free everything it owns.  NULL is a no-op. */
void mla_plan_destroy(mla_plan_t plan);

/* Static string for a status code. */
const char* mla_status_string(mla_status status);

#ifdef __cplusplus
}
#endif

#endif /* PAGED_MLA_B200_H */
