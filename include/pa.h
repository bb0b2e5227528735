/*
 * pa.h -- C ABI of the prefix-aware decode-attention library (libpa.so).
 *
 * The library computes batched single-token decode attention
 *     out[b][h] = softmax(q[b][h] . K_b^T / sqrt(d)) V_b
 * for B requests over a paged bf16 KV cache whose requests share prefixes.
 * Sources: the PAT review ("PAT: Accelerating LLM Decoding via Prefix-Aware
 * Attention with Resource Efficient Multi-Tile Kernel", section 三 核心公式 for the
 * formula, Pack-Forward-merge 范式 for the three stages), and the short-term
 * memory page (技术原理: each request's own token is appended to its KV before
 * it attends; PagedAttention for the paged cache).
 *
 * The three stages map to calls:
 *   pack     pa_plan_create   host: tree-structured block table, profit model,
 *                             split of long nodes, tile-class selection
 *            pa_plan_upload   async H2D copy of the plan into the workspace
 *   forward  pa_forward       device: partial attention per (node, kv head,
 *                             query tile, key range) into fp32 partials
 *   merge    pa_merge         device: log-sum-exp combine of each (request,
 *                             head)'s partials into bf16 out and fp32 lse
 *
 * Memory ownership: the caller allocates and owns every device buffer (q, the
 * pools, the workspace, out, lse).  The library owns only the host-side plan
 * object; a plan keeps no device pointer past the call that received it.
 * Device calls are asynchronous on the stream given.  Nothing throws across
 * this ABI; every call returns a pa_status.
 *
 * Tensor layouts (row-major, contiguous, bf16 = IEEE bfloat16 bit patterns):
 *   q       bf16 [B][Hq][D]
 *   k_pool  bf16 [num_pages][Hkv][P][D]     (v_pool alike); 16-byte aligned
 *   out     bf16 [B][Hq][D]                 round-to-nearest-even
 *   lse     fp32 [B][Hq]                    natural log of sum exp(scaled logits)
 *   block_table int32 [B][max_pages] (host); kv_lens int32 [B] (host)
 * Query head h reads kv head h / (Hq / Hkv).  Token t of request b is slot
 * t % P of page block_table[b][t / P]; entries past ceil(kv_len/P) are ignored.
 */
#ifndef PA_H_
#define PA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  PA_OK = 0,
  PA_ERR_INVALID = 1,     /* bad argument: page id, kv_len, shape */
  PA_ERR_UNSUPPORTED = 2, /* valid but not built: head_dim, GQA ratio, page size */
  PA_ERR_NOMEM = 3,       /* host allocation failed, or workspace too small */
  PA_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed */
  PA_ERR_TIMEOUT = 5,     /* a device-side bounded wait gave up (recorded in the workspace) */
  PA_ERR_DEVICE = 6       /* a device-side check failed (recorded in the workspace) */
} pa_status;

/* pa_config.flags */
#define PA_PLAN_NO_SHARING (1u << 0)   /* query-centric: inline every shared node (baseline mode) */
#define PA_PLAN_ALWAYS_SHARE (1u << 1) /* keep every shared node shared, whatever the profit model says */
#define PA_PLAN_DEBUG_CHECKS (1u << 2) /* device-side index checks; failures set PA_ERR_DEVICE */
#define PA_PLAN_KEEP_PACK (1u << 3)    /* keep the pack result in the plan, for pa_plan_advance */
#define PA_PLAN_FAULT_DROP_LOAD (1u << 8) /* tests only: forward skips one KV load, so its bounded
                                             wait must expire and record PA_ERR_TIMEOUT */

typedef struct {
  int32_t num_q_heads;      /* Hq */
  int32_t num_kv_heads;     /* Hkv; Hq / Hkv must be 1, 2, 4 or 8 */
  int32_t head_dim;         /* D: 64 or 128 */
  int32_t page_size;        /* P: 16 */
  float softmax_scale;      /* 0 selects 1/sqrt(head_dim) */
  int32_t num_sms;          /* 0: query the current device (148 on B200 if none) */
  int32_t max_chunk_tokens; /* 0: heuristic; else upper bound on tokens per forward work unit
                               (rounded down to a multiple of page_size, at least one page) */
  uint32_t flags;           /* PA_PLAN_* */
  int32_t wait_timeout_us;  /* device bounded-wait limit; 0 selects 2,000,000 (2 s) */
} pa_config;

typedef struct pa_plan pa_plan; /* opaque, host-owned */

typedef struct {
  int32_t batch;
  int32_t num_nodes;        /* non-empty nodes of the tree block table */
  int32_t num_shared_nodes; /* nodes with two or more requests */
  int32_t num_kept_shared;  /* shared nodes the profit model kept shared (not inlined) */
  int32_t num_items;        /* node items (a node x query tile) */
  int32_t num_segments;     /* forward work units (item x kv head x key range) */
  int32_t num_segments_simt;/* units on the CUDA-core class (one request, G rows) */
  int32_t num_segments_mma; /* units on the tensor-core class (two or more requests) */
  int32_t num_partial_rows; /* partial result rows per kv head group (each holds G rows) */
  int32_t simt_warps;       /* CUDA-core class warps of the forward launch */
  int32_t mma_ctas;         /* tensor-core class CTAs of the forward launch (one per SM) */
  int32_t num_tail_pairs;   /* (request, kv head) pairs merged by the tail merge launch */
  int64_t unique_tokens;    /* tokens of distinct tree nodes (each shared page once) */
  int64_t naive_tokens;     /* sum of kv_lens (query-centric reads) */
  int64_t read_tokens;      /* tokens the plan reads from the pools (per kv head) */
  int64_t unique_kv_bytes;  /* unique_tokens * 2 * Hkv * D * 2 */
  int64_t read_kv_bytes;    /* read_tokens * 2 * Hkv * D * 2 */
  uint64_t workspace_bytes; /* device workspace the caller must provide */
  uint64_t image_bytes;     /* bytes pa_plan_upload copies to the device */
  double plan_us;           /* host time spent in pa_plan_create or pa_plan_advance */
} pa_plan_stats;

/*
 * Pack: build a plan for one decode batch (host only; no device call).
 * Source: the PAT review, section 三, Pack-Forward-merge 范式 item 1 (group the
 * queries of a batch into CTA work by shared prefix, with a profit-model
 * heuristic) and Pack Scheduler 工作流, Figure 7 (the tree-structured block
 * table; packing scheme 1 keeps a parent node apart from its leaves, scheme 2
 * folds it into them); item 2 of the same list for the tile selector and the
 * split of long KV that the plan also fixes.
 *   cfg               head configuration and planner options (copied)
 *   batch             B >= 1
 *   kv_lens           host int32[B], each in [1, max_pages * page_size]
 *   block_table       host int32[B][max_pages], row-major; the first
 *                     ceil(kv_lens[b] / page_size) entries of row b must be in
 *                     [0, num_pages_in_pool)
 *   num_pages_in_pool size of the pools' first dimension
 *   out               receives the new plan (NULL on error)
 * Two requests share a page when their rows hold the same page id at the same
 * position after an identical prefix (prefix caching).  A shared page is
 * packed as shared (read once for all its requests) where it is full for all
 * of them; a page that is the last, partial page of some of the requests that
 * hold it (the queries of one session sharing its partial last page, or a
 * request continuing in a page another one ends in) is read by each of those
 * requests in its own item.  Inputs are read
 * during the call only.
 */
pa_status pa_plan_create(const pa_config *cfg, int32_t batch, const int32_t *kv_lens,
                         const int32_t *block_table, int32_t max_pages, int32_t num_pages_in_pool,
                         pa_plan **out);

/*
 * Pack for the next decode step of the same batch, from the previous step's
 * plan instead of a new walk of the block table (PAT review, section 六,
 * overhead analysis, Figure 16: the pack scheduler runs at every decode step;
 * here its tree is carried over from one step to the next).
 *   prev              a plan made with PA_PLAN_KEEP_PACK (by pa_plan_create or
 *                     by this call); not modified
 *   kv_lens, block_table, max_pages, num_pages_in_pool
 *                     as for pa_plan_create, for the same batch
 *   out               receives the new plan (NULL on error); it keeps its pack
 *                     result, so it can be advanced in turn
 * The caller asserts that the first ceil(prev_kv_len / page_size) entries of
 * every row are the ones the previous plan was made from: the tree of shared
 * nodes is reused as it was, and only each request's own tail grows (its one-
 * request item takes the new tokens and pages; a request that ended exactly at
 * the end of a shared node gets a new one-request item).  New page ids are
 * range-checked.  A request whose kv_len shrank, or a smaller pool, makes the
 * call plan from scratch (same result as pa_plan_create with prev's config).
 * New pages that several requests share are read once per request (no new
 * sharing is found; the next full pa_plan_create finds it).
 * Errors: PA_ERR_INVALID for a prev without a kept pack result, a different
 * batch size, or inputs pa_plan_create would reject.
 */
pa_status pa_plan_advance(const pa_plan *prev, const int32_t *kv_lens, const int32_t *block_table,
                          int32_t max_pages, int32_t num_pages_in_pool, pa_plan **out);

/*
 * Pack for chunks of new tokens appended to sessions (prefix-aware grouped
 * prefill of stateful sessions).  Source: the stateful-streaming summary
 * ("Attention Once Is All You Need", 方法拆解: a session's KV cache persists
 * and is advanced as new data arrives; the scheduler groups the prefill of the
 * sessions prefix-aware) and the short-term-memory page (技术原理: a token's K
 * and V are appended before it attends, so each new token sees the context and
 * the chunk up to itself).
 *   n_sessions        S >= 1
 *   ctx_lens          host int32[S]: tokens of session s before its chunk (>= 0)
 *   chunk_lens        host int32[S]: new tokens of session s (>= 1)
 *   block_table       host int32[S][max_pages]: session s's pages, covering its
 *                     ctx_lens[s] + chunk_lens[s] tokens (K and V of the chunk
 *                     already written there)
 * The plan has one row per new token, sessions in order and each chunk in
 * token order: row i of session s attends over tokens 0 .. ctx_lens[s] + i of
 * the session.  q, out and lse of pa_forward / pa_merge / pa_attend are then
 * [sum(chunk_lens)][Hq][D] (lse [rows][Hq]).  The rows of a session share the
 * context's full pages, so the pack stage reads those once for all of a
 * session's rows (chunk x G rows on the tensor cores); the chunk's own pages
 * are read per row up to its position.  Errors as pa_plan_create.
 */
pa_status pa_plan_create_append(const pa_config *cfg, int32_t n_sessions, const int32_t *ctx_lens,
                                const int32_t *chunk_lens, const int32_t *block_table, int32_t max_pages,
                                int32_t num_pages_in_pool, pa_plan **out);

/* Device workspace size in bytes for this plan (256-byte aligned buffer required).
 * The workspace holds the plan image and the forward stage's fp32 partial
 * results (the intermediate results the PAT review's Merge stage combines). */
pa_status pa_plan_workspace_size(const pa_plan *plan, size_t *bytes);

/*
 * Copy the plan (item, segment and page tables, and a zeroed status word) into
 * the caller's device workspace, asynchronously on `stream` (cudaStream_t).
 * This is the hand-over from the host pack stage to the device forward stage
 * of the PAT review's Pack-Forward-merge 范式 (section 三).
 * The image is first copied into a library-owned pinned staging buffer (a
 * small pool reused once each copy has completed), so the call does not wait
 * for earlier work on the stream and the plan may be destroyed right after it
 * returns.  bytes must be at least pa_plan_workspace_size; the workspace must
 * be 256-byte aligned.
 */
pa_status pa_plan_upload(const pa_plan *plan, void *d_workspace, size_t bytes, void *stream);

/*
 * Forward: partial attention of every planned work unit into the workspace's
 * fp32 partial buffers.  Source: the PAT review, section 三, Forward 阶段
 * (multi-tile kernels, a runtime tile selector per CTA, multi-stream execution
 * and long-KV splitting) and Figure 3 (decode attention as two GEMVs, q.K^T
 * and p.V, fed by a tiling pipeline from global memory).  q, k_pool, v_pool are device pointers in the layouts
 * above; k_pool and v_pool must be 16-byte aligned.  Needs a prior
 * pa_plan_upload to the same workspace (ordered before on the stream).
 * Asynchronous on `stream`; launch failures return PA_ERR_CUDA.
 */
pa_status pa_forward(const pa_plan *plan, const void *q, const void *k_pool, const void *v_pool,
                     void *d_workspace, void *stream);

/*
 * Merge: log-sum-exp combine of the partials of every (request, head) into
 * out (bf16 [B][Hq][D], round-to-nearest-even) and lse (fp32 [B][Hq]; may be
 * NULL).  Asynchronous on `stream`, ordered after pa_forward.  Source: the PAT
 * review, section 三, Merge 阶段 (a light online-softmax kernel that combines
 * each query's intermediate results across CTAs).
 */
pa_status pa_merge(const pa_plan *plan, void *d_workspace, void *out, float *lse, void *stream);

/*
 * Merge into fp32 instead of bf16: out is fp32 [B][Hq][D] (not rounded), lse
 * fp32 [B][Hq] (may be NULL).  This is the per-rank result of context
 * parallelism, which pa_merge_rows combines after the ranks' rows have been
 * gathered; otherwise as pa_merge (the PAT review's Merge 阶段, section 三).
 */
pa_status pa_merge_f32(const pa_plan *plan, void *d_workspace, float *out, float *lse, void *stream);

/*
 * Merge of attention rows gathered from several parts of the KV (context
 * parallelism: each part is one rank's result over its slice of every
 * request's pages).  The combine is the merge stage's log-sum-exp rule (the
 * PAT review, section 三, Merge 阶段), taken over the parts in order:
 *   lse[b][h] = log sum_p e^{lse_p}, out[b][h] = sum_p e^{lse_p - lse} o_p.
 *   n_parts, rows_per_part
 *                     parts of the gather, each padded to rows_per_part rows
 *   batch, num_q_heads, head_dim
 *                     B, Hq, D (64 or 128) of the whole batch
 *   d_part_req        device int32 [n_parts][rows_per_part]: the request of
 *                     each row, ascending within a part, -1 for padding rows
 *                     (which must come last)
 *   d_part_o          device fp32 [n_parts][rows_per_part][Hq][D] (pa_merge_f32
 *                     of each part), 16-byte aligned
 *   d_part_lse        device fp32 [n_parts][rows_per_part][Hq]
 *   out               device bf16 [B][Hq][D] (round-to-nearest-even), lse fp32
 *                     [B][Hq] (may be NULL); a request in no part gets zeros
 *                     and lse = -inf
 * Asynchronous on `stream`; errors PA_ERR_INVALID / PA_ERR_UNSUPPORTED before
 * anything is enqueued, PA_ERR_CUDA on a launch failure.
 */
pa_status pa_merge_rows(int32_t n_parts, int32_t rows_per_part, int32_t batch, int32_t num_q_heads,
                        int32_t head_dim, const int32_t *d_part_req, const float *d_part_o, const float *d_part_lse,
                        void *out, float *lse, void *stream);

/*
 * Forward with the merge fused into it (one launch): the warp that writes the
 * last partial row of a (request, kv head) pair merges that pair into out and
 * lse (the PAT review's Forward and Merge stages, section 三, in one pass).  Same results as pa_forward + pa_merge, bit for bit.  The arrival
 * counters it uses are left at zero, so the uploaded plan can be run again.
 */
pa_status pa_attend(const pa_plan *plan, const void *q, const void *k_pool, const void *v_pool,
                    void *d_workspace, void *out, float *lse, void *stream);

/*
 * Read the device status word of the workspace (synchronises `stream`).
 * *out = PA_OK, PA_ERR_TIMEOUT or PA_ERR_DEVICE.  The word is cleared by the
 * next pa_plan_upload.  d_workspace == NULL reads the word of the static
 * workspace of pa_attend_noalloc instead (the status of the last call made
 * there, by any plan).  The pages have no counterpart of this call: it
 * reports the device-side bounded waits and checks of this library.
 */
pa_status pa_get_device_status(const pa_plan *plan, const void *d_workspace, void *stream, pa_status *out);

/* Counters of the plan (host only). */
pa_status pa_plan_get_stats(const pa_plan *plan, pa_plan_stats *out);

/*
 * Copy the host image that pa_plan_upload sends (stats.image_bytes bytes) into
 * dst (host memory).  Its layout is described by pa_image_layout below; tests
 * use it to execute a plan on the CPU.
 */
pa_status pa_plan_host_image(const pa_plan *plan, void *dst, size_t bytes);

/*
 * Profiling hook: up to four cudaEvent_t handles (owned by the caller) that
 * the device calls record on their stream around each launch:
 *   events[0], events[1]  before / after the forward launch (pa_forward, pa_attend)
 *   events[2], events[3]  before / after the merge launch (pa_merge)
 * NULL entries are skipped; n = 0 turns the hook off.  The events must stay
 * valid while the plan uses them.
 */
pa_status pa_plan_set_profile_events(pa_plan *plan, void *const *events, int32_t n);

/*
 * One decode step in one call: pa_plan_create, the upload of the plan image and
 * pa_attend (forward with the merge fused) on `stream`.  Source: the PAT review,
 * section 六, 开销分析 and Figure 16 (the pack scheduler runs at every decode
 * step of the serving system, beside the attention kernels).
 *   d_workspace, workspace_bytes
 *                     caller-owned device buffer for the partial rows; must
 *                     cover pa_plan_workspace_size of a plan of the same batch
 *   d_images, images_bytes
 *                     caller-owned device buffer (256-byte aligned) for the
 *                     plan images; its two halves are used alternately, so a
 *                     plan whose image exceeds images_bytes / 2 (rounded down
 *                     to 256 bytes) is refused with PA_ERR_NOMEM
 * The image is copied into the next half on a stream of the library's own (the
 * library keeps one copy stream and four events per device, and no device
 * memory): the copy for step k+1 runs while the kernels of step k do, and
 * `stream` waits for it (an event) before its launches.  An image of at most
 * 16 KiB is copied on `stream` itself instead (in stream order, with fewer
 * host calls).  A half is refilled only after the launches that read it have
 * completed.  The device status word
 * of the step is in its half: read it with pa_get_device_status on the plan
 * returned through plan_out, before two more pa_decode_step calls refill that
 * half.  pa_plan_upload (or pa_attend_noalloc) of that plan makes it refer to
 * the new copy instead.
 * profile_events: NULL, or four cudaEvent_t as for pa_plan_set_profile_events.
 * plan_out: NULL (the plan is released before returning; its upload has
 * already been staged) or receives the plan, which the caller then releases.
 */
pa_status pa_decode_step(const pa_config *cfg, int32_t batch, const int32_t *kv_lens, const int32_t *block_table,
                         int32_t max_pages, int32_t num_pages_in_pool, const void *q, const void *k_pool,
                         const void *v_pool, void *d_workspace, size_t workspace_bytes, void *d_images,
                         size_t images_bytes, void *out, float *lse, void *const *profile_events, void *stream,
                         pa_plan **plan_out);

/*
 * pa_attend without a caller workspace, for callers that cannot allocate
 * device memory where they run attention (inside a memory pool that forbids
 * further allocation, an allocator-free runtime, a hook that must not touch
 * the caching allocator).  The pages this library implements have no
 * counterpart of this call; it is a deployment convenience.
 *   The workspace is one static device array of 24 MiB, held by every GPU
 *   that loads the library until the process exits.  A plan whose
 *   pa_plan_workspace_size exceeds 24 MiB is refused with PA_ERR_NOMEM before
 *   anything is enqueued.
 *   Each call copies the plan image (status word and arrival counters at zero)
 *   into the array with cudaMemcpyAsync from the plan's host memory, then runs
 *   the fused forward there.  It calls no cudaMalloc, cudaFree, pinned-memory
 *   allocator or other allocating routine.
 *   Every call shares the one array and leaves the last call's contents in it:
 *   calls that overlap on the GPU (other streams, other threads) race and
 *   must be ordered by the caller.
 *   The first call on a device looks up the array's device address (with that
 *   device current); make that first call before any stream capture.
 * Returns as pa_attend.  The device status word of the call is in the shared
 * array: pa_get_device_status(plan, NULL, stream, &st) reads it (until the
 * next call overwrites it).
 */
pa_status pa_attend_noalloc(const pa_plan *plan, const void *q, const void *k_pool, const void *v_pool, void *out,
                            float *lse, void *stream);

/* Release a plan (NULL is ignored). */
void pa_plan_destroy(pa_plan *plan);

/* Static description of a status code. */
const char *pa_status_string(pa_status s);

/*
 * Layout of the uploaded image and the workspace.  All offsets are bytes from
 * the workspace base and are multiples of 256.
 *
 *   header      pa_image_header
 *   nodes       pa_item[num_items]            a node (or its query tile)
 *   segs        pa_seg[num_segments]          SIMT segments first, then MMA
 *   pages       int32[num_page_entries]       page ids, per item
 *   queries     int32[num_query_entries]      request ids, per item
 *   seg_prows   int32[num_query_entries_mma]  partial row of each (MMA seg, query)
 *   mma_segs    int32[2]                      {0, num_segments_mma}: the tensor-core work units,
 *                                             longest first; CTA c starts with unit c, and the
 *                                             CTAs take the rest one at a time from the counter
 *                                             mma_next of the header
 *   counters    int32[B * Hkv]                arrival counters of the fused merge (zero)
 *   warp_segs   int32[simt_warps + 1]         SIMT warp w runs segs [warp_segs[w], warp_segs[w+1])
 *   prow_off    int32[B * Hkv + 1]            partial rows of (b, g) are
 *                                             [prow_off[b*Hkv+g], prow_off[b*Hkv+g+1])
 *   tail_pairs  int32[num_tail_pairs]         b*Hkv+g of every pair merged by the tail merge
 *                                             launch (tensor-core rows only, or mode 3), ascending
 *   mix_pairs   int32[num_mix_pairs][2]       {b*Hkv+g, its number of SIMT rows} of the pairs
 *                                             with both SIMT and tensor-core rows (mode 2); entry
 *                                             k is SIMT warp (k mod simt_warps)'s to count once
 *                                             the tensor-core launch has finished; {-1, -1}:
 *                                             no pair
 *   partial_lse fp32[num_partial_rows][G]     (workspace only, not uploaded)
 *   partial_o   fp32[num_partial_rows][G][D]  (workspace only, not uploaded)
 */
typedef struct {
  int32_t page_off;  /* into pages: this item's page ids */
  int32_t n_tokens;  /* valid tokens of the item, from slot 0 of its first page */
  int32_t n_queries; /* requests in the item; rows = n_queries * G */
  int32_t query_off; /* into queries */
} pa_item;

typedef struct {
  int32_t item;       /* index into nodes */
  int32_t kv_head;    /* kv head g */
  int32_t page_begin; /* first page of the run, index within the item's pages */
  int32_t n_tokens;   /* valid tokens of the run (its pages are ceil(n_tokens / P)) */
  int32_t prow;       /* SIMT: the partial row written; MMA: index into seg_prows */
  int32_t query;      /* SIMT: the request; MMA: the item's query_off (its requests are
                       * queries[query .. query + sole)) */
  int32_t sole;       /* SIMT: how the fused path combines this partial row of (query, kv_head).
                       * Bits 0-1, the mode: 0: arrival counter, the last of the pair's SIMT
                       * rows merges the pair; 1: it is the pair's only partial row and goes
                       * straight to the output; 2: the pair also has tensor-core rows: its
                       * counter also takes one arrival from the SIMT warp that the pair's
                       * mix_pairs entry names, made after that warp's own work once the
                       * tensor-core launch has finished, and whichever arrival is the last
                       * merges the pair; 3: the pair also has tensor-core rows and is
                       * merged by the tail merge launch (plans with more than 3 such pairs
                       * per SIMT warp).  Bits 2-31: the pair's number of SIMT partial
                       * rows.  MMA segments: the item's n_queries (the tile has sole * G
                       * rows). */
  int32_t page_start; /* index into pages of the run's first page (item page_off + page_begin) */
} pa_seg;

typedef struct {
  uint32_t magic;   /* 0x50414231 */
  int32_t status;   /* device status word (pa_status), 0 after upload */
  int32_t fault_a;  /* where a device check or wait failed (diagnostics) */
  int32_t fault_b;
  int32_t batch, num_q_heads, num_kv_heads, head_dim, page_size;
  int32_t num_items, num_segments, num_segments_simt, num_segments_mma, simt_warps;
  int32_t num_partial_rows, mma_ctas;
  int32_t num_tail_pairs; /* pairs merged by the tail launch of pa_attend / pa_decode_step */
  int32_t mma_next;       /* takes of tensor-core work units from the counter so far in the
                             running launch (units past each CTA's first): 0 after upload,
                             and back at 0 after every launch that completes (after a
                             device-side error, upload the plan again) */
  int32_t num_mix_pairs;  /* entries of mix_pairs */
  int32_t simt_warps_per_cta; /* SIMT warps of a CTA of the small-row launch (6 or 8): warp w runs
                                 in CTA w / simt_warps_per_cta */
  uint64_t off_nodes, off_segs, off_pages, off_queries, off_seg_prows, off_mma_segs, off_counters, off_warp_segs,
      off_prow_off, off_tail_pairs, off_mix_pairs;
  uint64_t off_partial_lse, off_partial_o, image_bytes, workspace_bytes;
} pa_image_header;

#ifdef __cplusplus
}
#endif

#endif /* PA_H_ */
