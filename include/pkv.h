/*
 * pkv.h - C ABI of the B200 paged GQA decode-attention library (libpkv.so).
 *
 * One decode step: every sequence ("row") i of a batch has one new query
 * token with H_q query heads and N_i cached tokens whose keys and values live
 * in a paged pool.  G = H_q / H_kv query heads share each KV head; query head
 * hq reads KV head floor(hq / G).  For each (row, query head):
 *
 *     out = softmax(scale * q . K^T) V     over the row's N_i cached tokens,
 *
 * with K and V read straight through the block table, never repacked:
 * token t of row i is slot t mod P of physical page block_table[i][t / P].
 * Sources: "PersistentKV: Page-Aware Decode Scheduling for Long-Context LLM
 * Serving on Commodity GPUs" (gist.science explainer, "PKV" below), Technical
 * summary > Methodology > 1 "Native block-table decode engine" (GQA grouping,
 * layout without repacking); "Chapter 8 - Next-generation KV cache management"
 * (actionbridge.io), section 8.1 (block table = logical block -> physical block).
 *
 * Conventions for every function:
 *  - The return value is a pkv_status; nothing else reports errors.
 *  - Device memory is allocated by the caller (e.g. PyTorch) and owned by the
 *    caller; the library allocates no device memory at run time (the scratch
 *    of pkv_paged_decode_noalloc is a fixed array in the library image) and
 *    touches no caller buffer after a call returns (a small host-side cache
 *    of encoded TMA descriptors is keyed by pool address and shape).  Host
 *    functions are pure and thread-safe.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  Device work is queued on it asynchronously unless stated.
 *  - Sizes are element counts unless the name ends in _bytes.
 *  - The fast path supports bf16 q/K/V/out, page_size 16, head_dim 64 or 128,
 *    1 <= G <= 16, pools 16-byte aligned with head_dim contiguous and token,
 *    head and page strides that are multiples of 8 elements.  Anything else
 *    returns PKV_ERR_UNSUPPORTED.
 */
#ifndef PKV_H
#define PKV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define PKV_API __attribute__((visibility("default")))
#else
#define PKV_API
#endif

/* Status codes. */
typedef enum {
    PKV_OK = 0,
    PKV_ERR_INVALID = -1,      /* an argument is malformed (null pointer, negative size, bad table) */
    PKV_ERR_UNSUPPORTED = -2,  /* well formed but outside the fast path (see above) */
    PKV_ERR_CAPACITY = -3,     /* a caller buffer (items, workspace, staging) is too small */
    PKV_ERR_CUDA = -4,         /* a CUDA runtime call or kernel launch failed */
    PKV_ERR_TIMEOUT = -5,      /* a device-side wait gave up (reported by pkv_workspace_status) */
    PKV_ERR_DEVICE_INPUT = -6  /* the kernel met an out-of-range seq_len, page id or work item
                                  (reported by pkv_workspace_status); it clamped and went on */
} pkv_status;

/* Execution paths [PKV, Methodology 2 "Calibrated adaptive policy"]. */
typedef enum {
    PKV_NO_SPLIT = 0,   /* one block per (row, KV head) covers the whole row; no merge */
    PKV_SPLIT_S = 1,    /* rectangular grid (row, KV head, split); empty splits write the neutral state */
    PKV_WORK_QUEUE = 2, /* 1D grid over the compact queue of non-empty (row, KV head, chunk) items */
    PKV_BALANCED = 3    /* the compact queue cut into equal page shares for a fixed grid of T blocks
                           (one wave on the GPU): each block streams its items back to back */
} pkv_mode;

/* pkv_plan.flags / pkv_policy_rule.flags */
#define PKV_FLAG_SEPARATE_MERGE 1 /* merge partial states in a second kernel instead of in the
                                     last block that finishes a (row, KV head) */
#define PKV_FLAG_NO_PDL 2         /* launch without programmatic dependent launch (by default the
                                     kernels may be scheduled while the previous kernel on the
                                     stream finishes; they wait for it before any memory access) */
#define PKV_FLAG_DEEP_RING 4      /* split kernel with a 12-page shared-memory ring (two blocks per
                                     SM) instead of 8 pages (three blocks per SM): more bytes in
                                     flight per block, for grids of about two blocks per SM */
#define PKV_FLAG_PDL_EARLY 16     /* the caller promises that the kernel queued right before this call
                                     writes neither seq_lens, block_table, the queue nor any K/V page
                                     except each row's last one: the split kernel then reads those and
                                     starts copying pages before waiting for that kernel (it still
                                     waits before q, a row's last page and any write).  Ignored by the
                                     balanced mode, which always waits first. */
#define PKV_FLAG_CLUSTER_MERGE 8  /* SPLIT_S with S <= 16 only: the S blocks of each (row, KV head)
                                     run as one thread-block cluster and merge their states through
                                     distributed shared memory (no partial states in the workspace,
                                     no merge launch); other modes return PKV_ERR_UNSUPPORTED */
#define PKV_FLAG_SHARED_PREFIX 64 /* WORK_QUEUE only, plan {2, U, C, flags}: items / indptr hold the
                                     prefix-sharing queue of pkv_build_prefix_queue at chunk C and U is its
                                     unit count: one block per unit stages the unit's shared pages once
                                     for all its members (always with the 12-page ring, as if
                                     PKV_FLAG_DEEP_RING were set).  n_items = the item count.  Not with
                                     PKV_FLAG_DEVICE_FILL or PKV_FLAG_PDL_EARLY (PKV_ERR_UNSUPPORTED) */
#define PKV_FLAG_DEVICE_FILL 32   /* WORK_QUEUE only, plan {2, T, 0, flags}: no queue is passed; every
                                     block derives its own item of the compact queue whose chunk fills
                                     one wave of T blocks (the fill rule of pkv_select_policy) from the
                                     device seq_lens, so one plan, or one captured CUDA graph, serves any
                                     lengths without host planning or a builder kernel.  items / indptr
                                     may be NULL; n_items (the grid) must be >= max(T, B * H_kv); B <=
                                     1024; not with PKV_FLAG_SEPARATE_MERGE (PKV_ERR_UNSUPPORTED) */

/* Problem shape and pool layout.  Pool element (page, kv_head, slot, d) of
 * k_pool / v_pool lives at  page*kv_stride_page + kv_head*kv_stride_head +
 * slot*kv_stride_token + d  (elements).  The default "HND" pool
 * [num_pool_pages][H_kv][page_size][head_dim] has strides
 * (H_kv*P*D, P*D, D); an "NHD" pool [pages][P][H_kv][D] has (P*H_kv*D, D, H_kv*D).
 * K and V share these strides, and either pool may be a view into a larger
 * cache: the halves of one combined [pages][2][H_kv][P][D] cache (page stride
 * 2*H_kv*P*D, V at K + H_kv*P*D elements), rows padded past D, pages holding
 * more heads.  Nothing outside the addressed elements is read. */
typedef struct {
    int32_t B;                  /* rows (sequences) in the batch, >= 0 */
    int32_t H_q;                /* query heads, a multiple of H_kv */
    int32_t H_kv;               /* KV heads */
    int32_t head_dim;           /* D */
    int32_t page_size;          /* P, tokens per page */
    int32_t max_pages_per_seq;  /* columns of block_table; every N_i <= max_pages_per_seq * P */
    int32_t num_pool_pages;     /* pages in each pool; block-table entries lie in [0, num_pool_pages) */
    int32_t reserved;           /* 0 */
    int64_t kv_stride_page;
    int64_t kv_stride_head;
    int64_t kv_stride_token;
} pkv_shape;

/* The chosen execution plan (16 bytes, compared bit-exactly by the tests).
 *   NO_SPLIT:    {0, 1, 0, flags}
 *   SPLIT_S:     {1, S', C, flags}  C = ceil(pages_max / S), S' = ceil(pages_max / C)
 *   WORK_QUEUE:  {2, S', C, flags}  C from the rule,        S' = ceil(pages_max / C)
 *                {2, T, 0, flags}   with PKV_FLAG_DEVICE_FILL: the fill budget T, C found on the device
 *                {2, U, C, flags}   with PKV_FLAG_SHARED_PREFIX: U units of the prefix-sharing queue
 *   BALANCED:    {3, T, 0, flags}   T blocks from the rule's num_splits
 * where pages_max = ceil(N_max / P).  S' is the most chunks any row needs. */
typedef struct {
    int32_t mode;
    int32_t num_splits;
    int32_t chunk_pages;
    int32_t flags;
} pkv_plan;

/* One work item: tokens [tok_begin, tok_end) of (row, kv_head).  tok_begin is
 * a multiple of the page size; an item with tok_begin == tok_end exists only
 * for a row with N_i = 0 (it writes that row's zero output). */
typedef struct {
    int32_t row;
    int32_t kv_head;
    int32_t tok_begin;
    int32_t tok_end;
} pkv_work_item;

/* One row of a policy table: batches with b_lo <= B < b_hi and
 * nmax_lo <= N_max < nmax_hi take this rule's plan.  The first matching rule
 * wins; no match means NO_SPLIT.  Use INT32_MAX for an open upper end. */
typedef struct {
    int32_t b_lo, b_hi;
    int32_t nmax_lo, nmax_hi;
    int32_t mode;         /* pkv_mode */
    int32_t num_splits;   /* SPLIT_S: requested S >= 1; BALANCED: blocks T >= 1;
                             WORK_QUEUE with chunk_pages = 0: the item budget T >= 1 */
    int32_t chunk_pages;  /* WORK_QUEUE: chunk size C >= 1 in pages, or 0: the smallest C
                             whose queue has at most T = num_splits items (one wave of T
                             blocks), or ceil(N_max / P) when one item per (row, KV head)
                             already exceeds T */
    int32_t flags;        /* PKV_FLAG_* */
} pkv_policy_rule;

/* Scheduler workload counters of one step [PKV, Key contributions:
 * "scheduler-induced workload counters"; Results: launch fan-out and
 * merge-state traffic].  All in units of the name (bytes or counts). */
typedef struct {
    int64_t launches;           /* kernel launches of the step */
    int64_t work_items;         /* blocks of the attention kernel */
    int64_t empty_items;        /* blocks that only write a neutral state or a zero row */
    int64_t merge_state_bytes;  /* partial states written and read back: 2*slots*G*(D+2)*4
                                   over every (row, KV head) with more than one slot */
    int64_t kv_bytes;           /* K+V of the valid tokens: sum_i N_i * H_kv * 2 * D * 2 */
    int64_t kv_bytes_streamed;  /* K+V of whole pages: sum_i ceil(N_i/P) * P * H_kv * 2 * D * 2 */
    int64_t q_bytes;            /* B * H_q * D * 2 */
    int64_t out_bytes;          /* B * H_q * D * 2 */
    int64_t queue_bytes;        /* WORK_QUEUE: 16 * items + 4 * (B*H_kv + 1) sent to the device */
    int64_t bucket_launches;    /* exact-length bucketing: 2 * distinct non-zero N_i */
} pkv_counters;

/* Library version string (static storage). */
PKV_API const char *pkv_version(void);

/* Human-readable name of a status code (static storage). */
PKV_API const char *pkv_status_string(int status);

/* Copy the built-in policy table (calibrated on B200 with seed 20260622) into
 * rules[0 .. capacity).  *n_rules receives its length; PKV_ERR_CAPACITY if
 * capacity is smaller (rules may then be NULL to query the length). */
PKV_API int pkv_default_policy(pkv_policy_rule *rules, int32_t capacity, int32_t *n_rules);

/* Pick the plan for a batch from (B, N_max) [PKV, Methodology 2 "Calibrated
 * adaptive policy": B = 1 long context -> split with length buckets, B >= 8
 * -> compact work queue, otherwise the single kernel; Results, B = 4 boundary].
 * seq_lens_host: host int32[shape->B]; rules: n_rules rows, or NULL for the
 * built-in table.  Pure host function; writes *plan (see pkv_plan).
 * PKV_ERR_INVALID on a negative length, a rule with an unknown mode,
 * num_splits < 1 in a SPLIT_S rule or chunk_pages < 1 in a WORK_QUEUE rule. */
PKV_API int pkv_select_policy(const int32_t *seq_lens_host, const pkv_shape *shape,
                              const pkv_policy_rule *rules, int32_t n_rules, pkv_plan *plan);

/* Number of items pkv_build_work_queue emits:
 *   H_kv * sum_i max(1, ceil(ceil(N_i / P) / chunk_pages)). */
PKV_API int pkv_work_queue_size(const int32_t *seq_lens_host, const pkv_shape *shape,
                                int32_t chunk_pages, int32_t *n_items);

/* Build the compact work queue [PKV, Methodology 1 "Compact work queue" and
 * "Row-local bounds"]: one item per (row, KV head, chunk) whose token range is
 * non-empty, in lexicographic (row, kv_head, chunk) order; chunk c covers
 * tokens [c*C*P, min((c+1)*C*P, N_i)) with C = chunk_pages, so bounds follow
 * each row's real length.  indptr (host int32[B*H_kv + 1]) receives the first
 * item of each (row, kv_head) pair, indptr[B*H_kv] = *n_items.  items: host
 * array of `capacity` entries; PKV_ERR_CAPACITY (with *n_items set to the
 * size needed) if it is too small.  Pure host function. */
PKV_API int pkv_build_work_queue(const int32_t *seq_lens_host, const pkv_shape *shape,
                                 int32_t chunk_pages, pkv_work_item *items, int32_t capacity,
                                 int32_t *indptr, int32_t *n_items);

/* Number of items pkv_build_balanced_queue emits for n_blocks blocks. */
PKV_API int pkv_balanced_queue_size(const int32_t *seq_lens_host, const pkv_shape *shape,
                                    int32_t n_blocks, int32_t *n_items);

/* Build the balanced work queue [PKV, Methodology 1 "Compact work queue",
 * "Row-local bounds"; cut for a fixed grid].  The (row, KV head) pairs are
 * laid end to end in lexicographic order, ceil(N_i / P) pages each; of the U
 * pages in total, block b (T = n_blocks) owns pages
 * [floor(b*U/T), floor((b+1)*U/T)).  Each maximal run of one pair's pages
 * inside one block's share is an item {row, kv_head, tok_begin, tok_end}
 * (page-aligned begin, end clipped to N_i); a row with N_i = 0 gets one empty
 * item per head.  Items are in lexicographic order.  indptr (host int32,
 * B*H_kv + 1 + n_blocks + 1 entries) receives the pair offsets as in
 * pkv_build_work_queue, followed by the block offsets: block b owns items
 * indptr[B*H_kv + 1 + b] .. indptr[B*H_kv + 2 + b].  Capacity errors as in
 * pkv_build_work_queue. */
PKV_API int pkv_build_balanced_queue(const int32_t *seq_lens_host, const pkv_shape *shape,
                                     int32_t n_blocks, pkv_work_item *items, int32_t capacity,
                                     int32_t *indptr, int32_t *n_items);

/* Items pkv_build_balanced_queue can emit for any lengths of this shape:
 * B*H_kv + n_blocks (an upper bound; the exact count is
 * pkv_balanced_queue_size).  Sizes the buffers of the device-side builder. */
PKV_API int pkv_balanced_queue_capacity(const pkv_shape *shape, int32_t n_blocks, int32_t *capacity);

/* The balanced queue built on the device from device-resident lengths,
 * bit-identical to pkv_build_balanced_queue for the same lengths, so that a
 * decode step whose lengths change on the device (a replayed CUDA graph)
 * needs no host planning.  There is no counterpart on the pages beyond the
 * queue itself [PKV, Methodology 1 "Compact work queue"]; this is the
 * device-side builder the queue invites.
 *   seq_lens   device int32 [B] (read after the kernel queued before on
 *              `stream` completes); a length outside [0, max_pages_per_seq * P]
 *              is clamped and sets the seq_len bit in `workspace`'s error word
 *   items      device, >= pkv_balanced_queue_capacity() entries; entries past
 *              the real count are left untouched
 *   indptr     device int32, B*H_kv + 1 + n_blocks + 1 entries: pair offsets,
 *              then block offsets, as pkv_build_balanced_queue
 *   workspace  the workspace of the decode call that will read the queue
 *              (its error word)
 * Then call pkv_paged_decode with a BALANCED plan of num_splits = n_blocks,
 * the same items / indptr and n_items = the capacity (the workspace sized for
 * that many items).  Asynchronous on `stream`, one kernel (one block of
 * threads), capturable in a CUDA graph.  B must be <= 4096
 * (PKV_ERR_UNSUPPORTED otherwise); capacity below the bound returns
 * PKV_ERR_CAPACITY before anything is queued. */
PKV_API int pkv_build_balanced_queue_device(const int32_t *seq_lens, const pkv_shape *shape,
                                            int32_t n_blocks, pkv_work_item *items, int32_t capacity,
                                            int32_t *indptr, void *workspace, void *stream);

/* Items the compact queue filling one wave of n_blocks blocks can hold for
 * any lengths of this shape: max(n_blocks, B*H_kv). */
PKV_API int pkv_fill_queue_capacity(const pkv_shape *shape, int32_t n_blocks, int32_t *capacity);

/* The compact queue whose chunk fills one wave of T = n_blocks blocks, built
 * on the device from device-resident lengths: the chunk C is the one
 * pkv_select_policy picks for a WORK_QUEUE rule with chunk_pages = 0 and
 * num_splits = T, and items / indptr (B*H_kv + 1 entries: pair offsets, the
 * last one the item count) equal pkv_build_work_queue's at that C.  The
 * device-side counterpart of the fill rule [PKV, Methodology 1 "Compact work
 * queue"; the rule itself is this library's].  Arguments, errors, limits and
 * capturability as pkv_build_balanced_queue_device; capacity >=
 * pkv_fill_queue_capacity().  Then call pkv_paged_decode with a WORK_QUEUE
 * plan (any chunk_pages >= 1: the items carry their token ranges), the same
 * items / indptr and n_items = the capacity: the grid has that many blocks
 * and those past the device-side count return at once. */
PKV_API int pkv_build_fill_queue_device(const int32_t *seq_lens, const pkv_shape *shape, int32_t n_blocks,
                                        pkv_work_item *items, int32_t capacity, int32_t *indptr,
                                        void *workspace, void *stream);

/* Sizes of the prefix-sharing queue (pkv_build_prefix_queue): *n_items
 * items and *n_units units. */
PKV_API int pkv_prefix_queue_size(const int32_t *seq_lens_host, const int32_t *block_table_host,
                                  const pkv_shape *shape, int32_t chunk_pages, int32_t max_members,
                                  int32_t *n_items, int32_t *n_units);

/* The compact work queue that stages shared prefix pages once for several
 * rows ["Chapter 8 - Next-generation KV cache management" (actionbridge.io),
 * 8.1: reference-counted block sharing, best-of-8 over one prompt; 8.3:
 * prefix caches, whose sharers hold the same physical blocks; PKV,
 * Methodology 1 "Compact work queue", "Row-local bounds"].
 *  - Sharing groups: rows with at least one full page and the same first
 *    physical page in block_table_host (host int32 [B][max_pages_per_seq]);
 *    the lowest row leads.  A group's shared length L is the number of
 *    leading entries every member has in common with the leader, counting
 *    only pages that are full in every member.  Groups of one row or with
 *    L = 0 are dropped.
 *  - Items, in lexicographic (row, kv_head) order with pair offsets as in
 *    pkv_build_work_queue: a grouped row's [0, L*P) is cut into chunks of C
 *    = chunk_pages pages from 0, then [L*P, N_i) into chunks of C pages from
 *    L*P; other rows as pkv_build_work_queue.
 *  - Units (the blocks of the decode grid): for each group, KV head and
 *    shared chunk, the members' items in row order, in runs of at most
 *    max_members; every other item is a unit of its own; units ordered by
 *    their first member.  A unit's members read the same pages, staged once.
 * indptr (host int32, indptr_capacity >= B*H_kv + 1 + n_units + 1 + n_items
 * entries) receives the pair offsets, then the unit offsets (n_units + 1),
 * then the members' item indices unit by unit.  Decode with a WORK_QUEUE plan
 * carrying PKV_FLAG_SHARED_PREFIX, n_items = the item count (the workspace
 * sized for that many items); max_members * G must be <= 16.  Capacity
 * errors as pkv_build_work_queue; PKV_ERR_INVALID for a length past the
 * table.  Pure host function. */
PKV_API int pkv_build_prefix_queue(const int32_t *seq_lens_host, const int32_t *block_table_host,
                                   const pkv_shape *shape, int32_t chunk_pages, int32_t max_members,
                                   pkv_work_item *items, int32_t capacity, int32_t *indptr,
                                   int32_t indptr_capacity, int32_t *n_items, int32_t *n_units);

/* Closed-form workload counters of `plan` on this batch (host, pure). */
PKV_API int pkv_plan_counters(const int32_t *seq_lens_host, const pkv_shape *shape,
                              const pkv_plan *plan, pkv_counters *counters);

/* Device workspace that pkv_paged_decode needs for this shape and plan
 * (n_items: WORK_QUEUE / BALANCED queue length, ignored otherwise).  The workspace holds
 * a device error word, one completion counter per (row, KV head) pair and the
 * fp32 partial states (m, l, acc) of every split. */
PKV_API int pkv_workspace_bytes(const pkv_shape *shape, const pkv_plan *plan, int32_t n_items,
                                size_t *bytes);

/* Zero a workspace on `stream` (queued memset).  A workspace must be zeroed
 * once before its first use; every successful decode leaves it zeroed again,
 * so later calls need no memset.  Also clears a recorded device error. */
PKV_API int pkv_workspace_init(void *workspace, size_t workspace_bytes, void *stream);

/* Self-test of the device-side failure detection: every wait of the kernels
 * on an mbarrier is bounded, and a wait that runs out sets the timeout bit in
 * the workspace's error word instead of hanging.  This queues one small
 * kernel on `stream` that waits on an mbarrier no thread ever arrives at;
 * after limit_us microseconds (1 .. 1000000) the wait gives up and records
 * the timeout, which pkv_workspace_status then reports as PKV_ERR_TIMEOUT
 * (clear it with pkv_workspace_init).  No kernel of a decode runs. */
PKV_API int pkv_selftest_wait_timeout(void *workspace, size_t workspace_bytes, uint32_t limit_us,
                                      void *stream);

/* Synchronize `stream`, then read the workspace's device error word:
 * PKV_OK, PKV_ERR_TIMEOUT or PKV_ERR_DEVICE_INPUT (also stored in
 * *device_error when not NULL, as the raw bit mask: 1 timeout, 2 seq_len out
 * of range, 4 page id out of range, 8 malformed work item). */
PKV_API int pkv_workspace_status(const void *workspace, void *stream, int32_t *device_error);

/* One decode step on the GPU.  All pointers but `shape`, `plan` are device
 * pointers:
 *   q            bf16 [B][H_q][D], contiguous
 *   k_pool       bf16 pool, layout from `shape` (never repacked, only read)
 *   v_pool       bf16 pool, same layout as k_pool
 *   block_table  int32 [B][max_pages_per_seq]; entries past a row's last page are never read
 *   seq_lens     int32 [B]; N_i in [0, max_pages_per_seq * P]
 *   out          bf16 [B][H_q][D], contiguous; fully overwritten (rows with N_i = 0 get zeros)
 *   items,indptr WORK_QUEUE / BALANCED: the queue from pkv_build_work_queue or
 *                pkv_build_balanced_queue (indptr with its block offsets), copied to the device
 *   workspace    >= pkv_workspace_bytes(), zeroed once (pkv_workspace_init)
 * page_size must equal shape->page_size; scale multiplies the logits.
 * The split kernel streams whole K/V pages through the block table into
 * shared memory (TMA, multi-stage), computes each split's partial softmax
 * state on the tensor cores, and the exact merge of the splits runs in the
 * last block to finish each (row, KV head) [PKV, Methodology 1 "Sequence
 * splitting": "a separate merge kernel combines the states exactly"] or,
 * with PKV_FLAG_SEPARATE_MERGE, in a second kernel.  Results are
 * deterministic: the merge order is fixed (ascending split index).
 * Asynchronous on `stream`; a workspace must not be shared by calls that may
 * run at the same time.  Returns PKV_ERR_CUDA if a launch fails; errors the
 * kernels detect on device data are read back with pkv_workspace_status. */
PKV_API int pkv_paged_decode(const void *q, const void *k_pool, const void *v_pool,
                             const int32_t *block_table, const int32_t *seq_lens, int32_t page_size,
                             float scale, void *out, const pkv_shape *shape, const pkv_plan *plan,
                             const pkv_work_item *items, const int32_t *indptr, int32_t n_items,
                             void *workspace, size_t workspace_bytes, void *stream);

/* Scratch bytes held inside the library for pkv_paged_decode_noalloc. */
#define PKV_NOALLOC_SCRATCH_BYTES ((size_t)16 << 20)

/* pkv_paged_decode for callers that cannot allocate device memory.  The
 * paper has no counterpart; this is a convenience of this library.
 * Some callers cannot call cudaMalloc at the point where they decode: a
 * plugin inside a host framework that owns every device allocation and
 * hands out no scratch, a deployment that must run in a fixed, pre-sized
 * memory budget, or a latency-critical loop that cannot afford the device
 * synchronization an allocation may cause.  They pass the same inputs and
 * output as pkv_paged_decode but no workspace: the error word, completion
 * counters and partial softmax states live in a 16 MiB array compiled into
 * the library (PKV_NOALLOC_SCRATCH_BYTES; every GPU that loads the library
 * holds it until the process exits).  The call allocates nothing: no
 * cudaMalloc, no cudaFree, no allocating library routine.
 *  - A plan whose workspace (pkv_workspace_bytes) exceeds the array returns
 *    PKV_ERR_CAPACITY before anything is queued.
 *  - The first call in a CUDA context looks up the array's device address
 *    with cudaGetSymbolAddress (the device current) and caches it for that
 *    context; make that first call before any stream capture.  After
 *    cudaDeviceReset the cached address may be stale: reload the library.
 *  - A call that passes every argument check queues a memset that zeroes the
 *    error word and the counters, then the kernels; a rejected call queues
 *    nothing.  The array keeps the last call's contents otherwise.
 *  - All calls share the one array: calls that may overlap on the GPU (two
 *    streams, two threads) race and corrupt each other's results.  Order
 *    them on one stream.
 *  - Errors the kernels detect on device data are read back with
 *    pkv_noalloc_status.
 * Other arguments, layouts and return codes as pkv_paged_decode. */
PKV_API int pkv_paged_decode_noalloc(const void *q, const void *k_pool, const void *v_pool,
                                     const int32_t *block_table, const int32_t *seq_lens,
                                     int32_t page_size, float scale, void *out, const pkv_shape *shape,
                                     const pkv_plan *plan, const pkv_work_item *items,
                                     const int32_t *indptr, int32_t n_items, void *stream);

/* pkv_workspace_status for the scratch of pkv_paged_decode_noalloc:
 * synchronize `stream`, then read the error word the last no-alloc call left
 * (PKV_OK, PKV_ERR_TIMEOUT or PKV_ERR_DEVICE_INPUT; the raw bit mask in
 * *device_error when not NULL).  Allocates nothing.  The paper has no
 * counterpart. */
PKV_API int pkv_noalloc_status(void *stream, int32_t *device_error);

/* Sizes of the caller buffers pkv_decode_host needs for this batch and
 * policy table (rules NULL = built-in): *device_bytes of device memory and
 * *host_bytes of host staging memory (page-locked memory makes the copies
 * asynchronous; pageable memory also works). */
PKV_API int pkv_decode_host_bytes(const int32_t *seq_lens_host, const pkv_shape *shape,
                                  const pkv_policy_rule *rules, int32_t n_rules,
                                  size_t *device_bytes, size_t *host_bytes);

/* One synchronous decode step from host buffers, the way a serving loop
 * calls it [PKV, Methodology 3 "Evaluation protocol": synchronized wall time
 * including host planning]: pick the plan (pkv_select_policy), build its
 * queue into host_staging (pkv_build_work_queue or pkv_build_balanced_queue),
 * move q, seq_lens, block_table, the queue and the zeroed completion
 * counters and error word host->device in ONE copy, run pkv_paged_decode,
 * move the error word and out device->host in ONE copy and synchronize
 * `stream`.  q, block_table and out larger than 64 KiB each get a copy of
 * their own instead of travelling through the staging buffer.  When out_host
 * and host_staging are page-locked (mapped into the device's address space,
 * as all page-locked memory is under unified addressing) the kernels write
 * out straight into out_host and report device errors as flag words in
 * host_staging, so the step moves its result without a device->host copy;
 * pageable buffers take the packed device->host copy.  q_host,
 * block_table_host, seq_lens_host, out_host are host pointers with the
 * layouts of pkv_paged_decode; k_pool / v_pool are device pools (the cache
 * stays resident on the device).  An untimed call whose q, block table, out
 * and staging all qualify for the paths above (page-locked, q and the table
 * inside the staging image) and that needs the same copy and launches as the
 * calling thread's previous call (same buffers, pools, scale, shape, plan and
 * queue length; new contents are fine) is captured as a CUDA graph, and the
 * thread's later calls with the same needs replay it: one graph launch per
 * step instead of a copy and the kernel launches.  A step that cannot be
 * captured runs as before.  device_buffer must be 256-byte aligned
 * (PKV_ERR_UNSUPPORTED otherwise); it needs no zeroing.  The plan used is
 * written to *plan_out when not NULL.  Returns the device error status like
 * pkv_workspace_status when the kernels ran. */
PKV_API int pkv_decode_host(const void *q_host, const int32_t *block_table_host,
                            const int32_t *seq_lens_host, void *out_host, const void *k_pool,
                            const void *v_pool, float scale, const pkv_shape *shape,
                            const pkv_policy_rule *rules, int32_t n_rules, void *device_buffer,
                            size_t device_buffer_bytes, void *host_staging,
                            size_t host_staging_bytes, void *stream, pkv_plan *plan_out);

/* Where the time of one pkv_decode_host call goes (pkv_decode_host_timed).
 * Host parts from a monotonic host clock, device parts from CUDA events
 * recorded on the call's stream around the copies and the kernels. */
typedef struct {
    double host_plan_us;     /* policy, queue and the upload image written into host_staging */
    double host_enqueue_us;  /* the copies and the kernel launches queued on the stream */
    double host_wait_us;     /* cudaStreamSynchronize, from the last enqueue until it returned */
    double host_unpack_us;   /* out and the error word read back from host_staging */
    double dev_h2d_us;       /* device time of the host->device copies */
    double dev_kernel_us;    /* device time of the decode kernels */
    double dev_d2h_us;       /* device time of the device->host copies (none when out is page-locked) */
    double host_events_us;   /* reading the events back: the measurement's own cost, not the step's */
} pkv_host_timing;

/* pkv_decode_host that also reports where its time went into *timing (when
 * not NULL; the events it records add a little device time of their own, and
 * a timed call always queues its copy and launches itself, never a graph).
 * Arguments and return codes as pkv_decode_host [PKV, Methodology 3
 * "Evaluation protocol": synchronized wall time including host planning]. */
PKV_API int pkv_decode_host_timed(const void *q_host, const int32_t *block_table_host,
                                  const int32_t *seq_lens_host, void *out_host, const void *k_pool,
                                  const void *v_pool, float scale, const pkv_shape *shape,
                                  const pkv_policy_rule *rules, int32_t n_rules, void *device_buffer,
                                  size_t device_buffer_bytes, void *host_staging, size_t host_staging_bytes,
                                  void *stream, pkv_plan *plan_out, pkv_host_timing *timing);

/* The arguments of pkv_decode_host as one parameter block, for a serving
 * loop that issues the same call every step (same buffers, new contents):
 * the caller fills the block once and passes its address each step, which
 * spares a foreign-function binding the marshalling of sixteen arguments per
 * call.  Every field means what the argument of the same name of
 * pkv_decode_host_timed means; the block is read, never written, and the
 * caller owns it. */
typedef struct {
    const void *q_host;
    const int32_t *block_table_host;
    const int32_t *seq_lens_host;
    void *out_host;
    const void *k_pool;
    const void *v_pool;
    float scale;
    const pkv_shape *shape;
    const pkv_policy_rule *rules;
    int32_t n_rules;
    void *device_buffer;
    size_t device_buffer_bytes;
    void *host_staging;
    size_t host_staging_bytes;
    void *stream;
    pkv_plan *plan_out;
    pkv_host_timing *timing; /* NULL, or where pkv_decode_host_timed reports its time */
} pkv_host_call;

/* How many pkv_decode_host calls of the calling thread replayed a captured
 * graph of their step (see pkv_decode_host). */
PKV_API int64_t pkv_decode_host_replays(void);

/* pkv_decode_host_timed(call->q_host, ..., call->plan_out, call->timing):
 * the same step, the same return codes; PKV_ERR_INVALID when call is NULL
 * [PKV, Methodology 3 "Evaluation protocol": synchronized wall time
 * including host planning]. */
PKV_API int pkv_decode_host_call(const pkv_host_call *call);

#ifdef __cplusplus
}
#endif

#endif /* PKV_H */
