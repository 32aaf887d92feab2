/*
 * fca.h -- C ABI of libfca_b200.so: Forest Cascade Attention (FCA) decode on
 * NVIDIA B200 (sm_100a).
 *
 * The method ("ZoRRo Inference & Forest Cascade Attention", sections
 * "Overview" and "Core Mechanism"): for one decode step of a batch whose paged
 * KV caches share prefixes,
 *   1. discover the groups of requests that share a KV-cache prefix
 *      (fca_plan);
 *   2. run one grouped pass over each group's shared prefix blocks, so each
 *      such block is read once per group instead of once per request;
 *   3. run one pass per request over its own (suffix) blocks;
 *   4. reduce the partial results by their log-sum-exp weights
 *      (steps 2-4: fca_decode).
 * The output equals standard softmax attention over each request's whole
 * sequence.
 *
 * Cache layout ("PagedAttention vs. RadixAttention", "How PagedAttention
 * Works", steps 1-2 and 4): K and V are bf16 [num_blocks][block_size]
 * [num_kv_heads][head_dim], row-major; a request's block table row maps its
 * logical block j to a physical block id.  Two requests share a block when
 * their tables hold the same physical id at the same logical index.  Only
 * FULL blocks (j < seq_len / block_size) are shareable; a partly filled block
 * is treated as private to each request that references it (copy-on-write).
 *
 * Conventions for every call:
 *   - Pointers marked DEVICE are CUDA device pointers on the current device;
 *     HOST pointers are ordinary host memory.  The caller owns every buffer it
 *     passes in; the library owns only what a plan handle holds.
 *   - A plan belongs to the device that was current when it was built.  Calls
 *     that take a plan run on that device (made current for the call, the
 *     caller's current device restored on return); their buffers and stream
 *     must belong to it.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Calls that
 *     take a stream are asynchronous on it unless stated otherwise.
 *   - Functions return fca_status; nothing throws, traps or aborts across the
 *     ABI.  On an error return no output has been written unless stated.
 *   - Query head h reads KV head h / (num_q_heads / num_kv_heads).
 *   - lse is the natural-log log-sum-exp of the scaled scores, fp32.
 */
#ifndef FCA_H_
#define FCA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fca_status {
    FCA_OK = 0,
    FCA_ERR_INVALID_ARG = 1,   /* bad shape, null pointer, seq_len out of range */
    FCA_ERR_BAD_BLOCK_ID = 2,  /* a referenced table entry is outside [0, num_blocks) */
    FCA_ERR_UNSUPPORTED = 3,   /* valid input this build does not handle (e.g. head_dim) */
    FCA_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed */
    FCA_ERR_OOM = 5,           /* device allocation failed */
    FCA_ERR_DEVICE_FLAG = 6,   /* a kernel reported an internal error (bounded wait ran out) */
    FCA_ERR_TOO_LARGE = 7      /* fca_paged_decode_static: the problem exceeds its fixed scratch */
} fca_status;

/* Opaque plan: the group forest, per-request suffix starts, the work lists of
 * the three passes and the device workspace they need.  Library-owned; free
 * with fca_plan_destroy.  A plan stays valid for every layer whose caches use
 * the same block tables and shapes; q/k/v pointers are bound per decode. */
typedef struct fca_plan_s *fca_plan_t;

/* Plan options.  Pass NULL for the defaults. */
typedef struct fca_plan_opts {
    int32_t min_group_size;    /* groups need at least this many requests (>= 2; default 2) */
    int32_t min_shared_blocks; /* a group shorter than this many blocks is folded into the
                                  group below it or into its members' suffixes (>= 1; default 1) */
    int32_t split_tokens;      /* split-KV chunk length in tokens, multiple of 64;
                                  0 = automatic */
    int32_t flags;             /* FCA_PLAN_* bits */
    int32_t min_saved_blocks;  /* a group is used only if (members - 1) x its length in
                                  blocks -- the block reads sharing it saves -- reaches
                                  this; otherwise it is folded like a short group
                                  (>= 0; default 32, 0 = use every shared prefix).  The
                                  reading here of FCA's automatic activation ("ZoRRo
                                  Inference & Forest Cascade Attention", "How It
                                  Works"): groups too small to pay for their own
                                  grouped-pass work are read by their members' own
                                  passes instead. */
} fca_plan_opts;

/* Build a plan with no groups: every request reads its whole table in its own
 * pass.  fca_decode on such a plan is the flat (non-cascaded) paged decode. */
#define FCA_PLAN_FLAT 1u

/* Let fca_plan_update run without synchronising the host: the plan reserves,
 * when it is built, own-pass room for the longest request the tables can hold
 * (each request's table width past its shared blocks, in chunks of at least
 * 512 tokens, or split_tokens when set), and each update is checked, sized
 * and applied on the device.  See fca_plan_update for what changes. */
#define FCA_PLAN_ASYNC_UPDATE 2u

/* Default options (min_group_size 2, min_shared_blocks 1, split auto, flags 0,
 * min_saved_blocks 32). */
void fca_plan_opts_default(fca_plan_opts *opts /* HOST, out */);

/*
 * fca_plan -- group discovery ("Core Mechanism" step 1) and work-list build.
 *
 *   block_tables  DEVICE int32 [num_requests][max_blocks]; entries at
 *                 j >= ceil(seq_len / block_size) are ignored.
 *   seq_lens      DEVICE int32 [num_requests]; each in [1, max_blocks*block_size].
 *   block_size    tokens per block; this build supports 16.
 *   num_blocks    physical blocks in the caches (ids must be in [0, num_blocks)).
 *   num_q_heads, num_kv_heads  num_q_heads % num_kv_heads == 0,
 *                 num_q_heads / num_kv_heads <= 16.
 *   head_dim      64 or 128.
 *   out_plan      HOST, out: the new plan (NULL on error).
 *
 * Runs GPU kernels on `stream`, then synchronises the stream once to read back
 * the sizes of the forest and work lists and allocates the plan's device
 * workspace.  Plans allocate, in stream order on `stream`, from a memory pool
 * the library creates per device on first use and never trims: memory that
 * destroyed plans return stays in the pool (at most the largest total of
 * plans alive at once) and makes the next plan's allocation free of page
 * mapping.  The input buffers may be reused once it returns.
 * Errors: FCA_ERR_INVALID_ARG (shapes, a seq_len out of range),
 * FCA_ERR_BAD_BLOCK_ID (a referenced id out of range), FCA_ERR_UNSUPPORTED,
 * FCA_ERR_CUDA, FCA_ERR_OOM.  num_requests <= 16384, max_blocks <= 1 << 20.
 */
fca_status fca_plan(const int32_t *block_tables, int32_t max_blocks, const int32_t *seq_lens,
                    int32_t num_requests, int32_t block_size, int32_t num_blocks,
                    int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                    const fca_plan_opts *opts, fca_plan_t *out_plan, void *stream);

/*
 * fca_plan_update -- the plan for the next decode step of the same batch,
 * without group discovery.  Between decode steps a request's table only grows
 * (new blocks for its new tokens, written by that request alone), so the
 * forest of shared prefixes stays what it was; only the requests' own ranges
 * and the work lists of the per-request pass change.  Groups are not
 * rediscovered: blocks shared for the first time after the plan was built are
 * read by each request's own pass (still exact, just not deduplicated) until
 * a fresh fca_plan.
 *
 *   block_tables, max_blocks, seq_lens, num_requests  as for fca_plan; the
 *                 same num_requests and max_blocks as the plan (else
 *                 FCA_ERR_INVALID_ARG).  Each request's first suffix_start
 *                 blocks (the ones its groups read) must be unchanged and its
 *                 seq_len must still cover them.
 *
 * The plan's tables, lengths and own-pass work lists are rewritten on
 * `stream`: call it on the stream the plan's decodes use, after the decode
 * of the previous step has been queued there.
 *
 * Synchronises `stream` once (the new sizes), like fca_plan; may take more
 * memory from the plan pool if the own work outgrew the plan.
 *
 * A plan built with FCA_PLAN_ASYNC_UPDATE is updated without any host
 * synchronisation: the checks below run on the device, a refused update
 * leaves the plan as it was and records kErrUpdateRefused (32) in the plan's
 * device status (fca_check_device_status), and the function returns FCA_OK
 * as soon as the work is queued; block_tables and seq_lens must stay valid
 * until `stream` has run it.  fca_plan_get_stats then keeps describing the
 * plan as built.  Errors (synchronous plans):
 * FCA_ERR_INVALID_ARG (a shared entry changed, a length no longer covers the
 * shared blocks or is out of range, another table shape), FCA_ERR_BAD_BLOCK_ID,
 * FCA_ERR_UNSUPPORTED (more partial rows than the planner indexes),
 * FCA_ERR_OOM, FCA_ERR_CUDA.  After any of them but FCA_ERR_CUDA the plan is
 * left as it was; after FCA_ERR_CUDA destroy it.  Not part of the
 * method's steps: it is "Core Mechanism" step 1 carried over from one decode
 * step to the next.
 */
fca_status fca_plan_update(fca_plan_t plan, const int32_t *block_tables, int32_t max_blocks,
                           const int32_t *seq_lens, int32_t num_requests, void *stream);

/*
 * fca_decode -- steps 2-4 of "Core Mechanism": the grouped prefix pass, the
 * per-request suffix pass and the log-sum-exp merge, for one layer.
 *
 *   q        DEVICE bf16 [num_requests][num_q_heads][head_dim], 16-byte aligned.
 *   k_cache, v_cache  DEVICE bf16 [num_blocks][block_size][num_kv_heads][head_dim],
 *            16-byte aligned.
 *   out      DEVICE bf16 [num_requests][num_q_heads][head_dim] (round to nearest even).
 *   lse      DEVICE fp32 [num_requests][num_q_heads], or NULL to skip.
 *   scale    multiplier of q.k (normally 1/sqrt(head_dim)); positive and finite,
 *            else FCA_ERR_INVALID_ARG.
 *
 * Asynchronous on `stream`, three kernels in order.  When the plan has both
 * grouped and per-request work, the two passes share the SMs: the grouped
 * pass takes its share, and the per-request pass (launched with programmatic
 * stream serialization) starts on the other SMs as soon as the grouped pass
 * runs, then takes over each SM the grouped pass gives up; it ends after the
 * grouped pass, and the merge follows it.  Uses the plan's workspace, so
 * decodes that share a plan must be ordered on one stream.  A kernel that
 * detects an internal error records it in the plan; read it with
 * fca_check_device_status.
 */
fca_status fca_decode(const void *q, const void *k_cache, const void *v_cache, fca_plan_t plan,
                      void *out, float *lse, float scale, void *stream);

/*
 * fca_flat_decode -- the flat paged decode baseline: standard split-KV
 * attention of every request over its whole table, same kernels and merge.
 * `plan` must have been built with FCA_PLAN_FLAT (else FCA_ERR_INVALID_ARG).
 * Arguments as fca_decode.
 */
fca_status fca_flat_decode(const void *q, const void *k_cache, const void *v_cache,
                           fca_plan_t plan, void *out, float *lse, float scale, void *stream);

/*
 * The three passes of fca_decode as separate calls, in the order fca_decode
 * runs them: fca_prefix_pass (grouped pass over shared prefix blocks, no-op
 * for a flat plan or a plan without groups), fca_suffix_pass (per-request
 * pass over own blocks) and fca_merge_pass (log-sum-exp reduction into out
 * and lse).  Each runs on every SM.  Running the three in order on one
 * stream gives exactly the result of fca_decode (every work item writes its
 * own partial rows, whichever SM runs it); they exist so that each kernel can
 * be timed alone.  The first two write only the plan's partial buffers.
 * Arguments as fca_decode.
 */
fca_status fca_prefix_pass(const void *q, const void *k_cache, const void *v_cache, fca_plan_t plan,
                           float scale, void *stream);
fca_status fca_suffix_pass(const void *q, const void *k_cache, const void *v_cache, fca_plan_t plan,
                           float scale, void *stream);
fca_status fca_merge_pass(fca_plan_t plan, void *out, float *lse, void *stream);

/* Sizes and byte counts of a plan (HOST struct, filled synchronously): of the
 * plan as built or last updated synchronously (a plan built with
 * FCA_PLAN_ASYNC_UPDATE keeps the figures of the plan as built). */
typedef struct fca_plan_stats {
    int32_t num_requests, num_groups, max_depth, num_q_heads, num_kv_heads, head_dim;
    int32_t split_tokens;           /* chunk target of the per-request pass */
    int32_t prefix_split_tokens;    /* chunk target of the grouped pass */
    int32_t prefix_items, suffix_items;   /* work items of the two passes */
    int64_t num_partials;           /* partial (o, lse) rows written per decode */
    int64_t unique_kv_tokens;       /* each referenced physical block once, its valid tokens */
    int64_t unique_kv_bytes;        /* unique_kv_tokens * num_kv_heads * head_dim * 2 * 2 */
    int64_t flat_kv_bytes;          /* sum of seq_len * num_kv_heads * head_dim * 2 * 2 */
    int64_t fca_kv_bytes;           /* KV bytes the FCA passes read (prefix once per group) */
    int64_t prefix_kv_bytes;        /* of which the grouped pass reads */
    int64_t suffix_kv_bytes;        /* of which the per-request pass reads */
    int64_t workspace_bytes;        /* device bytes the plan holds */
} fca_plan_stats;

fca_status fca_plan_get_stats(fca_plan_t plan, fca_plan_stats *stats /* HOST, out */);

/*
 * fca_plan_export -- copy the canonical forest to HOST buffers (synchronous).
 * Canonical order: groups by (first block ascending, smallest member
 * ascending); members of a group ascending; parent as an index in that order
 * (-1 for a root).  Group g reads blocks [a[g], b[g]) of its members' tables;
 * its members are members[member_off[g] .. member_off[g] + n_members[g]).
 * suffix_start[r] is the first block of request r's own pass (the b of its
 * deepest group, else 0).  Any output pointer may be NULL.  Capacities:
 * num_groups entries for the group arrays, the total member count for
 * members, num_requests for suffix_start (see fca_plan_get_stats and
 * fca_plan_member_count).
 */
fca_status fca_plan_export(fca_plan_t plan, int32_t *a, int32_t *b, int32_t *parent,
                           int32_t *member_off, int32_t *n_members, int32_t *members,
                           int32_t *suffix_start);

/* Total member entries over all groups (HOST out). */
fca_status fca_plan_member_count(fca_plan_t plan, int64_t *count);

/* Free a plan (synchronises the device first); its device workspace goes
 * back to the library's plan pool.  NULL is ok. */
fca_status fca_plan_destroy(fca_plan_t plan);

/*
 * Read and clear the plan's device error word after the work queued on
 * `stream` finishes (synchronises the stream).  *code (HOST, may be NULL)
 * receives the raw word: 0 = no error.  Returns FCA_ERR_DEVICE_FLAG when the
 * word was non-zero.
 */
fca_status fca_check_device_status(fca_plan_t plan, void *stream, int32_t *code);

/*
 * fca_selftest_wait_timeout -- check that a wait which runs out ends in a
 * status, not a hang.  Every spin-wait of this library's kernels is bounded
 * by 1 s of wall-clock time; when the bound is reached the kernel records
 * bit 1 in a device error word and returns.  This call runs one
 * single-thread kernel whose wait, through the same bounded wait, is for a
 * barrier phase that nothing completes, and copies the error word it
 * recorded into *out_word (HOST): bit 1 set means the wait gave up as
 * designed.  Takes about 1 s; synchronises `stream`; uses the current
 * device.  Returns FCA_OK when the kernel ran, FCA_ERR_INVALID_ARG for a
 * NULL out_word, FCA_ERR_OOM / FCA_ERR_CUDA when a CUDA call failed.  Not a
 * step of the method: a diagnostic of its failure detection.
 */
fca_status fca_selftest_wait_timeout(void *stream, int32_t *out_word);

/*
 * fca_paged_decode_static -- the flat paged decode of fca_flat_decode
 * (standard split-KV attention of every request over its whole block table,
 * then the log-sum-exp merge) in one call that allocates nothing.  This entry
 * has no counterpart in the method's description; it is for callers that
 * cannot allocate device memory at decode time: an engine whose device memory is all handed out by its own
 * pool, or code that must not call the CUDA allocator while it records a
 * stream.  It needs no plan; it does not share prefix blocks.
 *
 * Memory: the work list and the partial results live in one fixed device
 * array of this library, 64 MiB (FCA_STATIC_SCRATCH_BYTES) on each device,
 * set aside by the CUDA runtime when it loads the library's kernels there.
 * The call itself makes no cudaMalloc, cudaFree or other allocating call:
 * it issues one cudaMemsetAsync of 16 bytes and three kernels on `stream`.
 * The first call on a device looks the array's address up
 * (cudaGetSymbolAddress), which may load the library's kernels on that
 * device; make that first call before any stream capture.  The address is
 * kept for the life of the process: do not call this entry point on a device
 * after cudaDeviceReset (or another release of its primary context) in the
 * same process, since the array may then sit elsewhere.
 * q, k_cache, v_cache, block_tables, seq_lens, out, lse and dev_status must
 * all be on the current device.
 *
 * What must start at zero: the array's three work counters, which the call
 * zeroes itself on `stream` before its kernels; and *dev_status, which the
 * caller zeroes.
 *
 * Concurrency: every call on a device uses the same array.  Calls must be
 * ordered (one stream, or events between streams); two calls in flight at
 * once on one device race and both results are undefined.
 *
 *   q, k_cache, v_cache, out, lse, scale  as fca_decode.
 *   block_tables  DEVICE int32 [num_requests][max_blocks], 4-byte aligned.
 *   seq_lens      DEVICE int32 [num_requests]; each in [1, max_blocks * 16].
 *   num_blocks    physical blocks in each cache (block size 16).
 *   dev_status    DEVICE int32, or NULL: the kernels OR error bits into it:
 *                 1 a bounded wait ran out, 2 a work item failed its range
 *                 check, 8 a seq_len out of range, 16 a used block id out of
 *                 [0, num_blocks).  A request with a bad length or id is
 *                 skipped (its out rows are 0, its lse -inf).  With NULL the
 *                 bits are dropped.
 *
 * Returns FCA_ERR_INVALID_ARG (null or misaligned pointer, bad shape),
 * FCA_ERR_UNSUPPORTED (head_dim not 64 or 128, more than 16 query heads per
 * KV head), FCA_ERR_TOO_LARGE when num_requests x num_q_heads partial rows
 * of one split each, plus the work list, exceed the array (about
 * num_requests * num_q_heads * (head_dim + 1) * 4 + num_requests *
 * num_kv_heads * 32 bytes must stay under 64 MiB; e.g. up to 3900 requests
 * at 32 query heads of head_dim 128), FCA_ERR_CUDA.  num_requests == 0 is a
 * no-op.  Asynchronous on `stream`.
 */
#define FCA_STATIC_SCRATCH_BYTES (64u << 20)
fca_status fca_paged_decode_static(const void *q, const void *k_cache, const void *v_cache,
                                   const int32_t *block_tables, int32_t max_blocks,
                                   const int32_t *seq_lens, int32_t num_requests, int32_t num_blocks,
                                   int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                   void *out, float *lse, float scale, int32_t *dev_status,
                                   void *stream);

/* Text of the last CUDA error a call of this library met on the calling
 * thread ("no error" if none); valid until the next failing call. */
const char *fca_last_cuda_error(void);

/* Static description of a status code. */
const char *fca_status_string(fca_status status);

/* Library version string, e.g. "fca_b200 0.1.0 sm_100a". */
const char *fca_version(void);

#ifdef __cplusplus
}
#endif

#endif /* FCA_H_ */
