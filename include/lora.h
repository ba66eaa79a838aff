/*
 * liblora — heterogeneous-batch LoRA adapter branch on one B200 (sm_100a).
 *
 * Computes, for every token t of a batch whose adapter id is i = ids[t]:
 *
 *     Y[t, :] += (alpha_i / r_i) * (X[t, :] A_i) B_i
 *
 * with A_i [d_in x r_i] and B_i [r_i x d_out] taken from a paged GPU pool.
 * Page "Multi-LoRA Serving in Production" (llms.blog), section "The
 * Mathematical Anatomy of Heterogeneous Batches", gives the formula and the
 * per-sequence adapters; section "Segmented Gather Matrix-Vector
 * Multiplication (SGMV)" gives the shrink (v = x A) and the scaled expand
 * (y += (alpha/r) v B) steps and the grouping of tokens by adapter; sections
 * "Multi-Size Batched Gather Kernels (MBGMV and MBGMM)" and "Unified Paging
 * Architecture" give mixed ranks without padding to the maximum rank and
 * weights gathered from non-contiguous pages through physical page indices.
 *
 * Conventions for every call below
 *  - Return value: LORA_OK (0) or a negative LORA_ERR_* code.  A call that
 *    returns an error has enqueued no work.
 *  - Every compute call is asynchronous on the given stream and does no
 *    host synchronisation.  Pointers named *_dev, and X, Y, V, ids, ranks,
 *    scales, page_table and ws, are device pointers; everything else is host.
 *  - The library's kernels let the next kernel on the stream start its
 *    preamble early (programmatic dependent launch).  ranks, scales and
 *    page_table are slot state and may be read in that preamble, before the
 *    kernels ahead on the stream have finished; every other input is read
 *    only after they have.  So a kernel that writes ranks, scales or
 *    page_table must not itself let its dependents start early (ordinary
 *    kernels do not).
 *  - bf16 data is passed as uint16_t bit patterns.  Matrices are row-major.
 *  - Inputs are never modified, except Y (updated in place) and the outputs
 *    named in each call.
 *  - The device error word err_dev (may be NULL) receives an OR of
 *    LORA_DEV_ERR_* bits.  A token whose id is outside [-1, S) or names an
 *    empty slot (rank 0) is skipped: its Y row is left untouched.  id = -1
 *    means "base model only" and is not an error.  Kernels never trap.
 *  - Scratch space comes from the caller's workspace (ws, ws_bytes).  The one
 *    exception is lora_apply_noalloc, for callers that cannot allocate: its
 *    plan lives in a fixed static device array of the library
 *    (LORA_NOALLOC_SCRATCH_BYTES per GPU that loads the library, held until
 *    the process exits).  No call allocates device memory.
 *  - Host threads: calls may come from several threads.  A pool's free list,
 *    a slot cache and the options are guarded inside the library; a
 *    workspace, an error word and the device tables belong to whoever passes
 *    them, and calls that share one must be ordered on one stream.
 */
#ifndef LORA_H_
#define LORA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *lora_stream_t;      /* a cudaStream_t; NULL = legacy default stream */
typedef struct lora_pool_s *lora_pool_t;        /* opaque host handle of one page pool */

/* Host return codes. */
#define LORA_OK                  0
#define LORA_ERR_INVALID_ARG    -1   /* NULL pointer, negative size, misaligned buffer, unknown option */
#define LORA_ERR_BAD_RANK       -2   /* rank outside [1, LORA_MAX_RANK] */
#define LORA_ERR_WIDTH_MISMATCH -3   /* pool row width differs from d_in / d_out */
#define LORA_ERR_POOL_OOM       -4   /* not enough free pages */
#define LORA_ERR_BAD_SLOT       -5   /* slot outside [0, num_slots), or page id not free / out of range */
#define LORA_ERR_CUDA           -6   /* a CUDA runtime call failed; see lora_last_cuda_error() */
#define LORA_ERR_WORKSPACE      -7   /* ws is NULL or ws_bytes < lora_workspace_size(...) */
#define LORA_ERR_TOO_LARGE      -8   /* lora_apply_noalloc: T or num_slots beyond its fixed scratch */
#define LORA_ERR_ALL_PINNED     -9   /* slot cache: every slot is held by a running batch */

/* Device error word bits. */
#define LORA_DEV_ERR_BAD_ID      1   /* some id < -1 or id >= num_slots */
#define LORA_DEV_ERR_EMPTY_SLOT  2   /* some id names a slot with rank 0 */
#define LORA_DEV_ERR_TIMEOUT     4   /* a kernel's bounded wait ran out (results of that call are undefined) */
#define LORA_DEV_ERR_BAD_PAGE    8   /* a used slot's rank exceeds 64 or its page table names a page outside the
                                        pool; its tokens are skipped */

/* Fixed geometry. */
#define LORA_PAGE_ROWS            16   /* rank-rows per page */
#define LORA_MAX_RANK             64
#define LORA_MAX_PAGES_PER_MATRIX 4    /* LORA_MAX_RANK / LORA_PAGE_ROWS */
#define LORA_MAX_JOB_TOKENS       16   /* most tokens one gather job serves (one weight read) */
#define LORA_MAX_PROJECTIONS      8    /* most projections one lora_apply_multi call updates */
#define LORA_MAX_SLOTS            4096

/* ------------------------------------------------------------------------ */
/* Page pool (page "Multi-LoRA Serving in Production", section "Unified     */
/* Paging Architecture": fixed-size physical pages, adapter weights sliced  */
/* along the rank dimension, logical page tables naming physical pages).   */
/* ------------------------------------------------------------------------ */

/* Wrap caller-owned device memory dev_buf[bytes] as a pool of pages of
 * page_rows (must be LORA_PAGE_ROWS) rows of `width` bf16 values each.
 * num_pages = bytes / (page_rows * width * 2).  dev_buf must be 256-byte
 * aligned and width a positive multiple of 8, at most 2^24.  The caller keeps ownership of
 * dev_buf and must keep it alive until lora_pool_destroy; the library owns
 * the host-side free list.  Physical row p*page_rows + j of the pool is the
 * bf16 row at dev_buf + (p*page_rows + j) * width * 2 bytes. */
int lora_pool_create(void *dev_buf, size_t bytes, int width, int page_rows, lora_pool_t *out);

/* Free the host handle (not the device memory).  NULL is accepted. */
int lora_pool_destroy(lora_pool_t pool);

/* Pages currently free / in total; -1 for a NULL handle. */
int lora_pool_free_pages(lora_pool_t pool);
int lora_pool_num_pages(lora_pool_t pool);

/* Unified paging: the pool's pages also serve a second tenant of the same
 * memory, such as KV-cache blocks (16 token vectors of `width` values per
 * page).  Page "Multi-LoRA Serving in Production", section "Unified Paging
 * Architecture": all dynamic memory outside the base model is one pool of
 * fixed-size physical pages that holds KV-cache tensors and adapter weights
 * alike, so memory moves between the two as traffic changes with no external
 * fragmentation; page "Multi-LoRA Serving Architecture ... (2026)", section
 * "S-LoRA unified paging".  Adapter loads and these calls draw on one free
 * list.
 *
 * lora_pool_alloc_pages takes n free pages and writes their ids to ids_out
 * (host, n entries); LORA_ERR_POOL_OOM (nothing taken) when fewer are free.
 * Page p is rows [16 p, 16 p + 16) of the pool, owned by the caller until it
 * is returned; the library never reads or writes it. */
int lora_pool_alloc_pages(lora_pool_t pool, int n, int32_t *ids_out);

/* Return pages taken by lora_pool_alloc_pages (ids: host, n entries).  All or
 * nothing: LORA_ERR_BAD_SLOT if an id is out of range, repeated, free, or
 * held by an adapter. */
int lora_pool_free_page_list(lora_pool_t pool, const int32_t *ids, int n);

/* Pages held by adapters and by lora_pool_alloc_pages (host outputs). */
int lora_pool_usage(lora_pool_t pool, int *adapter_pages, int *other_pages);

/* Load adapter (A, B) of rank `rank` into slot `slot` of the page table
 * page_table_dev [num_slots][2][LORA_MAX_PAGES_PER_MATRIX] (int32; matrix 0 =
 * A, 1 = B; unused entries are written as -1).
 *  a_t  : A transposed, [rank][d_in] bf16 (row k = column k of A), d_in = pa's width
 *  b    : B, [rank][d_out] bf16, d_out = pb's width
 *  a_t and b may be host (pinned or pageable) or device pointers.
 * ceil(rank/16) pages are taken from each pool's free list, or, when
 * page_ids (host, [2][LORA_MAX_PAGES_PER_MATRIX]) is not NULL, exactly those
 * pages (which must be free).  The rows are copied with cudaMemcpyAsync on
 * `stream` (page "Multi-LoRA Serving in Production", section "Asynchronous
 * Prefetching and Request Queuing"); the unused rows of a partly filled last
 * page are zeroed.  The slot's page-table row, scale_dev[slot] = alpha/rank
 * (fp32) and rank_dev[slot] = rank are written on the same stream.
 * The slot must be empty (load into an occupied slot returns
 * LORA_ERR_BAD_SLOT; evict it first).  Validation (page "Multi-LoRA
 * Serving Architecture ... (2026)", section "Trade-offs, Gotchas": validate
 * shape and rank before admission): rank in [1, 64] else LORA_ERR_BAD_RANK.
 * The pools record which pages belong to (page_table_dev, slot). */
int lora_pool_load(lora_pool_t pa, lora_pool_t pb, int slot, int num_slots, int rank, float alpha,
                   const uint16_t *a_t, const uint16_t *b, const int32_t *page_ids,
                   int32_t *page_table_dev, float *scale_dev, int32_t *rank_dev,
                   lora_stream_t stream);

/* Return the pages of (page_table_dev, slot) to the free lists and mark the
 * slot empty on the device (rank 0, scale 0, page entries -1) on `stream`.
 * Page "LoRA Adapters at Serve Time with vLLM Multi-LoRA", section "The
 * Inference Mechanism: A Worked Scenario", step "Eviction": a resident
 * adapter is swapped out to make room; page "Multi-LoRA Serving in
 * Production", section "Unified Paging Architecture": its pages go back to
 * the shared pool.
 * Pages are reused in stream order: a later load on the same stream is safe;
 * a caller using several streams must order them itself. */
int lora_pool_evict(lora_pool_t pa, lora_pool_t pb, int slot, int num_slots,
                    int32_t *page_table_dev, float *scale_dev, int32_t *rank_dev,
                    lora_stream_t stream);

/* Copy rank-row k of matrix m (0 = A^T, 1 = B) of a loaded slot back into
 * out_dev (device, width bf16) by resolving the page table on the device:
 * physical row = page_table[slot][m][k / 16] * 16 + k % 16 (used to verify
 * the paging round trip). */
int lora_pool_read_row(lora_pool_t pool, const int32_t *page_table_dev, int num_slots, int slot,
                       int m, int k, uint16_t *out_dev, lora_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Compute                                                                  */
/* ------------------------------------------------------------------------ */

/* Bytes of workspace the calls below need for T tokens and num_slots slots. */
size_t lora_workspace_size(int T, int num_slots);

/* Group tokens by adapter slot (page "Multi-LoRA Serving in Production",
 * section SGMV: requests are grouped by their target adapter), stably, and
 * store the plan of the batch in ws:
 *   perm   [T]    tokens with a valid adapter, by slot ascending, then by
 *                 token index; entries past the number of valid tokens are
 *                 left untouched
 *   seg_start [S+1]  tokens of slot i are perm[seg_start[i] .. seg_start[i+1])
 * plus the work lists of the two compute paths.  When perm_out / seg_start_out
 * (device) are not NULL the two arrays are also written there.
 * Tokens with id -1 are dropped; invalid ids are dropped and flagged in err_dev.
 * ranks: [num_slots] int32 (0 = empty slot).  The plan stays valid in ws for
 * lora_apply_planned until ws is reused; it depends on ids, ranks, T,
 * num_slots and the LORA_OPT_* values at the time of the call. */
int lora_plan(const int32_t *ids, int T, const int32_t *ranks, int num_slots,
              int32_t *perm_out, int32_t *seg_start_out,
              void *ws, size_t ws_bytes, int32_t *err_dev, lora_stream_t stream);

/* Shrink: V[t, k] = sum_j X[t, j] A_i[j, k] for k < r_i, fp32 accumulate.
 * Page "Multi-LoRA Serving in Production", section "Segmented Gather
 * Matrix-Vector Multiplication (SGMV)": the first of the two steps projects
 * each token onto its own adapter's rank-r_i space (v = x A).
 *   X [T][d_in] bf16, V [T][LORA_MAX_RANK] fp32 (columns >= r_i and rows of
 *   tokens without a valid adapter are left untouched).  pa's width must be d_in. */
int lora_shrink(const uint16_t *X, int T, int d_in, const int32_t *ids, int num_slots,
                const int32_t *ranks, const int32_t *page_table, lora_pool_t pa,
                float *V, void *ws, size_t ws_bytes, int32_t *err_dev, lora_stream_t stream);

/* Expand-add: Y[t, c] += s_i * sum_{k < r_i} V[t, k] B_i[k, c], fp32.
 * Page "Multi-LoRA Serving in Production", section "Segmented Gather
 * Matrix-Vector Multiplication (SGMV)": the second step expands v back to the
 * output width through B, scales it by alpha/r and adds it to the base
 * output.
 *   V [T][LORA_MAX_RANK] fp32, Y [T][d_out] fp32 in place, scales [num_slots]
 *   fp32 (alpha_i / r_i).  pb's width must be d_out.  The product runs on the
 *   tensor cores with each V value split into a bf16 high part and a bf16
 *   low part (about 16 significant bits of V), fp32 accumulation. */
int lora_expand_add(const float *V, float *Y, int T, int d_out, const int32_t *ids, int num_slots,
                    const int32_t *ranks, const float *scales, const int32_t *page_table,
                    lora_pool_t pb, void *ws, size_t ws_bytes, int32_t *err_dev,
                    lora_stream_t stream);

/* lora_expand_add into a column block of a wider output: row t of the block
 * starts at Y + t * ldy (ldy >= d_out, a multiple of 4; Y 16-byte aligned),
 * and only its first d_out columns are updated.  Page "Multi-LoRA Serving in
 * Production", section "S-LoRA TP Communication Optimization": for small
 * ranks a row-parallel layer splits B by columns and exchanges the rank-r
 * vector v; each rank then adds s v B_k into its own column block of the
 * partial output before the layer's all-reduce.  LORA_ERR_INVALID_ARG for a
 * bad ldy; otherwise as lora_expand_add. */
int lora_expand_add_strided(const float *V, float *Y, int ldy, int T, int d_out, const int32_t *ids, int num_slots,
                            const int32_t *ranks, const float *scales, const int32_t *page_table, lora_pool_t pb,
                            void *ws, size_t ws_bytes, int32_t *err_dev, lora_stream_t stream);

/* Fused shrink + expand-add: Y[t] += s_i (X[t] A_i) B_i for every token.
 *   X [T][d_in] bf16, Y [T][d_out] fp32 (holds Y_base = X W0 on entry, computed
 *   by the caller; page "Multi-LoRA Serving Architecture ... (2026)", section
 *   "Heterogeneous batching: the core compute trick": the base GEMM runs once
 *   on the whole batch and the two branches are added).
 * Segments shorter than the long-segment threshold take the gather
 * (MBGMV-style) kernels; longer ones take the tensor-core (MBGMM-style)
 * tiles.  The result does not depend on the token order. */
int lora_apply(const uint16_t *X, float *Y, int T, int d_in, int d_out, const int32_t *ids,
               int num_slots, const int32_t *ranks, const float *scales,
               const int32_t *page_table, lora_pool_t pa, lora_pool_t pb,
               void *ws, size_t ws_bytes, int32_t *err_dev, lora_stream_t stream);

/* The compute half of lora_apply: Y[t] += s_i (X[t] A_i) B_i using the plan
 * that lora_plan left in ws for this batch (same T, num_slots, ranks and
 * options).  A model applies one plan to all of its adapted layers: a token's
 * adapter slot is the same in every layer, only the pools, page tables and
 * scales differ.  Launches only the compute kernels. */
/* The compute half of lora_apply over the plan that lora_plan (or an earlier
 * apply call on the same batch) left in ws: a model plans once per batch (a
 * token's adapter is the same in every layer) and calls this for every
 * adapted projection.  Arguments, layouts and errors as lora_apply without
 * ids.  Ordering: the library's kernels let the next kernel on the stream
 * start before they finish and release it only after their own wait, so when
 * the plan was not the library's last launch on this stream, this call reads
 * the plan and starts loading adapter pages before it waits for the kernel
 * ahead (X and Y are read only after that wait).  Plain launches, events and
 * CUDA graphs keep this safe; a caller's own kernel launched between lora_plan
 * and this call with programmatic dependent launch that releases its
 * dependents before its own wait does not. */
int lora_apply_planned(const uint16_t *X, float *Y, int T, int d_in, int d_out, int num_slots,
                       const int32_t *ranks, const float *scales, const int32_t *page_table,
                       lora_pool_t pa, lora_pool_t pb, void *ws, size_t ws_bytes,
                       int32_t *err_dev, lora_stream_t stream);

/* One adapted projection of lora_apply_multi: its output Y [T][d_out] fp32
 * (in place, 16-byte aligned), its slot tables (ranks, scales, page_table as
 * for lora_apply) and its pools (pa of width d_in, pb of width d_out). */
typedef struct {
    float *Y;
    int d_out;
    const int32_t *ranks;
    const float *scales;
    const int32_t *page_table;
    lora_pool_t pa;
    lora_pool_t pb;
} lora_projection_t;

/* Several projections that read the same X, in one call: for every
 * projection p and token t, Y_p[t] += s_{p,i} (X[t] A_{p,i}) B_{p,i}.
 * Page "Multi-LoRA Serving Architecture ... (2026)", section "The memory
 * arithmetic that makes it work": an all-linear adapter has A and B for each
 * of a layer's seven projections (query, key and value read the same input,
 * as do gate and up), each with its own output width.
 *   projs: host array of num_projs (1..LORA_MAX_PROJECTIONS) projections;
 *   the library reads it during the call only.  All share X, T, d_in, ids,
 *   num_slots and one plan (made with projs[0].ranks: the error bits and the
 *   tokens dropped follow projection 0; a slot that is empty in another
 *   projection is skipped there).  Short segments of every projection are
 *   handled by one gather launch (on the split gather path: a shrink and an
 *   expand launch per projection); long runs by one tile launch for all
 *   projections (one projection: a tile shrink and a tile expand launch).  ws as for lora_apply (lora_workspace_size(T, num_slots)).
 * Each projection's result is bit-identical to lora_apply on that projection
 * alone.  Errors: as lora_apply, checked for every projection before any
 * work is enqueued; LORA_ERR_INVALID_ARG for num_projs out of range. */
int lora_apply_multi(const uint16_t *X, int T, int d_in, const int32_t *ids, int num_slots,
                     const lora_projection_t *projs, int num_projs, void *ws, size_t ws_bytes,
                     int32_t *err_dev, lora_stream_t stream);

/* The compute half of lora_apply_multi over the plan that lora_plan (or an
 * earlier apply call on this batch) left in ws, as lora_apply_planned is for
 * lora_apply: a model plans once per batch and applies every group of
 * projections that share an input.  Same arguments and errors as
 * lora_apply_multi without ids; launches only the compute kernels. */
int lora_apply_multi_planned(const uint16_t *X, int T, int d_in, int num_slots,
                             const lora_projection_t *projs, int num_projs, void *ws, size_t ws_bytes,
                             int32_t *err_dev, lora_stream_t stream);

/* lora_apply without a workspace argument, for callers that cannot allocate
 * device memory: e.g. a plug-in inside a host framework that owns all device
 * memory through its own pool and forbids outside allocations, or a
 * latency-critical serving loop that must not call cudaMalloc/cudaFree
 * because they can synchronise the device.  The pages describe no such call;
 * it has no counterpart there.
 *
 * Same arguments, result and error-word behaviour as lora_apply, minus
 * (ws, ws_bytes).  The segment plan lives in one fixed scratch array of
 * LORA_NOALLOC_SCRATCH_BYTES that is a static __device__ variable of the
 * library: every GPU that loads the library holds it until the process exits,
 * and the library itself never calls cudaMalloc, cudaFree or any allocating
 * routine.  Limits: T <= LORA_NOALLOC_MAX_TOKENS and num_slots <=
 * LORA_MAX_SLOTS; larger sizes return LORA_ERR_TOO_LARGE before any work is
 * enqueued.  The first call on a device looks up the scratch's device
 * address (cudaGetSymbolAddress) with that device current; make that first
 * call before any stream capture.  The address is kept for the process's
 * life and belongs to the device's primary context: after cudaDeviceReset on
 * a device, do not call lora_apply_noalloc on that device again.  All calls share the one array (it keeps the
 * last call's contents; each call writes everything it reads, so nothing needs
 * clearing), so calls whose kernels overlap on the GPU - on different streams
 * or from different host threads without ordering - race and give undefined
 * results: order them on one stream. */
#define LORA_NOALLOC_MAX_TOKENS    32768
#define LORA_NOALLOC_SCRATCH_BYTES 2162688   /* 2 MiB + 64 KiB: the plan of 32768 tokens and 4096 slots */
int lora_apply_noalloc(const uint16_t *X, float *Y, int T, int d_in, int d_out, const int32_t *ids,
                       int num_slots, const int32_t *ranks, const float *scales,
                       const int32_t *page_table, lora_pool_t pa, lora_pool_t pb,
                       int32_t *err_dev, lora_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Slot manager (host bookkeeping of which adapter lives in which slot)       */
/* ------------------------------------------------------------------------ */
/* Page "LoRA Adapters at Serve Time with vLLM Multi-LoRA", section "The
 * Inference Mechanism: A Worked Scenario", step "Eviction": when every slot is
 * taken the least recently used adapter is swapped out; page "Multi-LoRA
 * Serving Architecture ... (2026)", section "An adapter-cache LRU simulator":
 * an LRU over a fixed slot count judged by its hit rate, where in a batching
 * engine the slots hold the running batch's adapters (here: pinned slots).
 * The manager is host-only and thread-safe; it never touches device memory:
 * on a miss the caller evicts the returned key's pages and loads the new
 * adapter into the returned slot with lora_pool_evict / lora_pool_load, on the
 * stream of its choice (a second stream overlaps the load with compute). */
typedef struct lora_slot_cache_s *lora_slot_cache_t;

/* num_slots in [1, LORA_MAX_SLOTS], all initially empty. */
int lora_slot_cache_create(int num_slots, lora_slot_cache_t *out);
int lora_slot_cache_destroy(lora_slot_cache_t c);

/* Make adapter `key` (>= 0, the caller's id) resident and most recently used.
 *   *hit_out = 1: it already was, in *slot_out.
 *   *hit_out = 0: it now owns *slot_out: the lowest-numbered never-used slot,
 *   else the most recently emptied one, else the least recently used slot
 *   whose pin count is 0; *evicted_key_out is the key that slot held (-1 if
 *   none).  The caller must load the adapter before a batch uses the slot.
 * pin != 0 adds one to the slot's pin count (a running batch uses it).
 * Errors: LORA_ERR_ALL_PINNED when a miss finds every slot pinned (nothing
 * changes); LORA_ERR_INVALID_ARG for key < 0 or NULL outputs. */
int lora_slot_cache_acquire(lora_slot_cache_t c, int64_t key, int pin, int *slot_out, int *hit_out,
                            int64_t *evicted_key_out);

/* Drop one pin of `slot` (the batch that used it finished).  LORA_ERR_BAD_SLOT
 * for a slot out of range, LORA_ERR_INVALID_ARG when it holds no pin. */
int lora_slot_cache_unpin(lora_slot_cache_t c, int slot);

/* Mark `slot` empty (its adapter was evicted by the caller); it is the next
 * slot a miss takes.  LORA_ERR_ALL_PINNED if the slot is pinned. */
int lora_slot_cache_invalidate(lora_slot_cache_t c, int slot);

/* Slot of `key`, or -1, without touching the recency order. */
int lora_slot_cache_lookup(lora_slot_cache_t c, int64_t key, int *slot_out);

/* Counters since creation: acquire hits, misses, and misses that evicted. */
int lora_slot_cache_stats(lora_slot_cache_t c, int64_t *hits, int64_t *misses, int64_t *evictions);

/* ------------------------------------------------------------------------ */
/* Options and diagnostics (process-wide)                                   */
/* ------------------------------------------------------------------------ */

#define LORA_OPT_LONG_SEGMENT   1   /* runs of >= this many consecutive tokens of one slot use the tensor-core path
                                        (default 128, one full tile; 0 = never) */
#define LORA_OPT_DECODE_JOB_TOKENS 2 /* max tokens per gather job: the short tokens of a slot are split into
                                        jobs of at most this many, each reading the weights once
                                        (1..LORA_MAX_JOB_TOKENS, default LORA_MAX_JOB_TOKENS) */

#define LORA_OPT_GATHER_PATH    3   /* kernels for short segments in lora_apply, lora_apply_planned and the
                                        multi-projection calls: LORA_GATHER_AUTO (default), LORA_GATHER_CLUSTER
                                        or LORA_GATHER_SPLIT; every choice gives bit-identical results */
#define LORA_GATHER_AUTO        0   /* the library picks by the call's shape: the split pair for one projection
                                        with num_slots >= 256 and T >= 64 (many distinct adapters likely),
                                        the cluster kernel otherwise */
#define LORA_GATHER_CLUSTER     1   /* one kernel: 4-CTA clusters exchange the shrink partials on chip */
#define LORA_GATHER_SPLIT       2   /* a shrink kernel writes per-quarter partials to the workspace, an expand
                                        kernel adds them and updates Y; one pair per projection */
#define LORA_OPT_PLAN_KERNEL    4   /* the plan's kernel: LORA_PLAN_AUTO (default) or LORA_PLAN_GENERAL; both
                                        write the same plan, bit for bit */
#define LORA_PLAN_AUTO          0   /* one warp for batches of at most 256 tokens, 128 slots and no long runs,
                                        the block-wide kernel otherwise */
#define LORA_PLAN_GENERAL       1   /* always the block-wide kernel */

int lora_set_option(int key, int value);
int lora_get_option(int key);

/* Message of the last CUDA error seen by this library (static string). */
const char *lora_last_cuda_error(void);

/* Number of kernels launched by the last lora_apply / lora_shrink /
 * lora_expand_add / lora_plan call on the calling host thread. */
int lora_last_launch_count(void);

#ifdef __cplusplus
}
#endif
#endif /* LORA_H_ */
