/*
 * libpagedattn -- one-token batched decode attention read directly from a
 * paged KV cache, and the per-step KV append that feeds it (NVIDIA B200,
 * sm_100a).
 *
 * The operations follow the pages on mini vLLM-style engines:
 *   - paged storage: per layer, K and V tensors shaped
 *     [num_blocks, block_size, Hkv, D] in token-before-head (NHD) order, one
 *     fixed-size physical block per block-table entry (BareLLM README, cache
 *     section and "Cache layers" bullets);
 *   - address translation: position t of request b lives in physical block
 *     block_tables[b][t / block_size] at row t % block_size (BareLLM README,
 *     cache section; Nano-vLLM overview, "Kernmodul: Sequence");
 *   - decode: for every request and query head, softmax(q . K^T * scale) . V
 *     over that request's own context length, for MHA, GQA and MQA
 *     (BareLLM README feature list), computed with a running max and sum
 *     (MinivLLM review, engine layout section; LLAISYS self-attention bullet)
 *     and, for long contexts, split over context partitions whose partial
 *     results are combined by log-sum-exp;
 *   - append: PagedKVCache's logical-to-physical write of each request's new
 *     token (BareLLM README component list).
 *
 * Conventions for every entry point:
 *   - All device pointers are caller-owned; the library never allocates,
 *     frees or synchronises inside pa_kv_append / pa_decode.  Work is queued
 *     on `stream` (a cudaStream_t; NULL = the legacy default stream).
 *   - Errors are returned as pa_status; nothing throws across the ABI.
 *     pa_last_error_message() gives a one-line reason for the last non-OK
 *     status returned on the calling host thread.
 *   - Value tensors (q, k/v cache, k/v new, out) have dtype s->dtype and must
 *     be 16-byte aligned.  Index tensors are int32.
 *   - Nothing falls back silently: shapes outside the supported set return
 *     PA_ERR_UNSUPPORTED.
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
    PA_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, inconsistent shape or plan */
    PA_ERR_UNSUPPORTED = 2,  /* a valid shape this build does not implement */
    PA_ERR_CUDA = 3,         /* a CUDA runtime call or kernel launch failed */
    PA_ERR_WORKSPACE = 4     /* workspace missing or smaller than the plan needs */
} pa_status;

typedef enum { PA_DTYPE_F32 = 0, PA_DTYPE_BF16 = 1, PA_DTYPE_F16 = 2 } pa_dtype;

/* Bits of the device error word (see pa_get_device_error).  Kernels never
 * trap: an out-of-range index is recorded here and the access is skipped. */
#define PA_DEVERR_BLOCK_ID    0x1  /* a block-table entry outside [0, num_blocks) */
#define PA_DEVERR_CONTEXT_LEN 0x2  /* context_lens[b] < 0 or > max_blocks_per_seq*block_size */
#define PA_DEVERR_TIMEOUT     0x4  /* a pipeline wait gave up (internal error) */
#define PA_DEVERR_WORKSPACE   0x8  /* more partitions than the plan provided for */
#define PA_DEVERR_SLOT        0x10 /* an append slot >= num_blocks*block_size */
#define PA_DEVERR_SMEM        0x20 /* dynamic shared memory not 1024-byte aligned (internal error) */

/* Problem shape.  B requests, Hq query heads, Hkv KV heads (Hq % Hkv == 0;
 * query head h reads KV head h / (Hq/Hkv)), head dim D, block_size tokens per
 * physical block, num_blocks blocks in the pool, max_blocks_per_seq columns
 * in the block table. */
typedef struct {
    int32_t B, Hq, Hkv, D;
    int32_t block_size, num_blocks, max_blocks_per_seq;
    int32_t dtype; /* pa_dtype */
} pa_shape;

/* How a decode call splits its work (filled by pa_plan; treat as opaque). */
typedef enum {
    PA_SPLIT_BALANCED = 0, /* persistent CTAs, equal token share each, split anywhere */
    PA_SPLIT_FIXED = 1     /* fixed partitions of partition_tokens tokens per request */
} pa_split_mode;

typedef struct {
    int32_t mode;             /* pa_split_mode */
    int32_t partition_tokens; /* PA_SPLIT_FIXED: tokens per partition */
    int32_t num_ctas;         /* persistent CTAs launched */
    int32_t tile_tokens;      /* tokens staged per pipeline stage */
    int32_t stages;           /* pipeline depth */
    int32_t head_group;       /* KV heads handled per work item */
    int32_t heads_per_unit;   /* query heads one warp carries */
    int32_t units_per_warp;
    int32_t warps_per_unit;   /* >1: a warp team splits the tokens of one unit */
    int32_t max_context_len;  /* the longest context the plan was made for */
    int32_t smem_bytes;
    int32_t dynamic_share;    /* PA_SPLIT_BALANCED: share of each request's tiles handed out
                                 at run time to whichever CTA is free, in 1/256.  pa_plan
                                 sets 0; a caller may set 1..64 when B <= 512 (the
                                 workspace is sized for 64) */
    int32_t flags;            /* PA_PLAN_* bits; pa_plan sets 0, a caller may set them */
    int32_t split_merge;      /* 1: the pieces of split requests are combined by a second grid
                                 launched behind the decode grid (one CTA per request and query
                                 head), chosen when the CTAs outnumber the (request, KV head
                                 group) pairs 8 to 1, so that each request is spread over many
                                 CTAs; 0: the CTA that delivers a request's last piece does it */
    int64_t max_slots;        /* partial-result slots in the workspace */
    pa_shape shape;           /* the shape this plan was made for */
    size_t workspace_bytes;   /* bytes pa_decode needs at `workspace` */
} pa_plan_t;

/* pa_plan_t.flags.  By default a decode grid launched behind another grid on
 * the same stream (programmatic dependent launch) reads context_lens and the
 * block table as they are while that grid still runs, plans its work from
 * them and pulls its first K/V blocks into L2.  Once that grid has
 * completed it reads both again and keeps the plan only if nothing changed
 * (otherwise it plans again), so the result never depends on the early
 * reads.  PA_PLAN_NO_SPECULATION turns the early reads off (useful when the
 * preceding kernel rewrites the metadata every step).  PA_PLAN_TEST_MISGUESS
 * makes every early guess wrong, so that the plan-again path runs (for
 * tests; slower).  PA_PLAN_TEST_STALL is for tests of the failure path only:
 * the first CTA publishes its first piece but never fills a pipeline stage
 * for it, so its consumers' bounded wait (about 2 s) gives up, records
 * PA_DEVERR_TIMEOUT and the whole CTA leaves cleanly (no copy outstanding);
 * the output is then undefined and the workspace must be re-initialised. */
#define PA_PLAN_NO_SPECULATION 0x1
#define PA_PLAN_TEST_MISGUESS  0x2
#define PA_PLAN_TEST_STALL     0x4

/* Library version: major*10000 + minor*100 + patch. */
int32_t pa_version(void);

const char *pa_status_str(pa_status st);

/* One-line reason for the last non-OK status on this host thread ("" if none). */
const char *pa_last_error_message(void);

/*
 * KV append (BareLLM README: PagedKVCache's logical-to-physical writes).
 * For each i < s->B with slot = slot_mapping[i] >= 0:
 *     k_cache[slot / block_size][slot % block_size][:][:] = k_new[i][:][:]
 * and the same for V; slot < 0 skips request i.
 *   k_new, v_new : device, [B, Hkv, D], dtype s->dtype
 *   slot_mapping : device, [B] int32, slot = physical_block*block_size + row
 *   k_cache, v_cache : device, [num_blocks, block_size, Hkv, D], updated in place
 *   device_error : device int32 or NULL; a slot >= num_blocks*block_size is
 *                  skipped and, if non-NULL, PA_DEVERR_SLOT is OR-ed in.
 * Non-negative slots must be distinct (two writes to one slot race).
 * Only s->B, Hkv, D, block_size, num_blocks and dtype are read from s.
 */
pa_status pa_kv_append(const void *k_new, const void *v_new, const int32_t *slot_mapping, void *k_cache,
                       void *v_cache, const pa_shape *s, int32_t *device_error, void *stream);

/*
 * Host-only planner (no device work, no allocation): the "host-side partition
 * planner" of the problem statement, here sized for a persistent grid.
 *   max_context_len : the largest context_lens[b] any later call will pass
 *                     (at most max_blocks_per_seq*block_size); recorded in
 *                     the plan.
 *   partition_tokens: 0 = PA_SPLIT_BALANCED (persistent CTAs with an equal
 *                     share of all requests' tokens each); > 0 =
 *                     PA_SPLIT_FIXED with partitions of that many tokens (a
 *                     multiple of 16), dealt to the CTAs in equal shares of
 *                     whole partitions; the partitions of a request that one
 *                     CTA takes are combined as they stream, the others by
 *                     log-sum-exp; >= max_context_len gives one partition per
 *                     request (no split).
 *   num_sms         : SM count to size the grid for; 0 = query the current
 *                     CUDA device.
 * The workspace holds one partial result per (request, CTA) pair that can
 * share a request, so its size does not depend on the context lengths.
 * Returns PA_ERR_UNSUPPORTED for shapes the kernels do not cover:
 * D not in {64, 128}; block_size not a power of two in [16, 256]; a GQA
 * group Hq/Hkv that is not a power of two <= 64; more query heads than one
 * CTA can carry.
 */
pa_status pa_plan(const pa_shape *s, int32_t max_context_len, int32_t partition_tokens, int32_t num_sms,
                  pa_plan_t *plan_out);

/* Bytes of device workspace pa_decode needs for `plan` (== plan->workspace_bytes).
 * The size follows from the plan alone (the planner fixes it from the shape,
 * the partition size and the CTA count), not from the context lengths. */
size_t pa_decode_workspace_size(const pa_plan_t *plan);

/* Zero a workspace before its first pa_decode.  A call that completes
 * leaves the workspace ready for the next one; a call that recorded
 * PA_DEVERR_TIMEOUT (a CTA gave up part-way) may leave its merge counters
 * set, so re-initialise the workspace after such an error.  Queued on
 * `stream`. */
pa_status pa_workspace_init(void *workspace, size_t workspace_bytes, void *stream);

/*
 * Decode attention over the paged cache.
 *   q            : device, [B, Hq, D] (NHD), dtype s->dtype
 *   k_cache/v_cache : device, [num_blocks, block_size, Hkv, D]
 *   block_tables : device, [B, max_blocks_per_seq] int32; entries past
 *                  ceil(context_lens[b]/block_size) are never read
 *   context_lens : device, [B] int32, tokens of request b (0 gives out = 0)
 *   scale        : softmax scale (typically 1/sqrt(D))
 *   out          : device, [B, Hq, D], dtype s->dtype (fp32 results rounded
 *                  to nearest-even for bf16)
 *   plan         : from pa_plan for the same *s; a plan whose fields differ
 *                  from what pa_plan gives for the shape, max_context_len,
 *                  partition size and CTA count it records is rejected with
 *                  PA_ERR_INVALID_ARG (only dynamic_share and flags are the
 *                  caller's to change)
 *   workspace    : device, >= plan->workspace_bytes, 256-byte aligned,
 *                  zeroed once by pa_workspace_init; holds partial results,
 *                  merge counters and the device error word.  Two calls that
 *                  overlap on the GPU must not share a workspace.
 * out[b][h] = sum_t softmax_t(scale * q[b][h] . K[t]) V[t], t < context_lens[b],
 * with K[t], V[t] the rows of KV head h / (Hq/Hkv) found through the table.
 */
pa_status pa_decode(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
                    const int32_t *context_lens, float scale, void *out, const pa_shape *s,
                    const pa_plan_t *plan, void *workspace, size_t workspace_bytes, void *stream);

/*
 * One decode step: pa_kv_append followed by pa_decode on the same stream,
 * the decode grid launched as a programmatic dependent of the append grid so
 * that its prologue (lengths, block table, q) overlaps the append; every K/V
 * row is read only after the append grid has completed.  Arguments as in the
 * two calls; the append's slot errors land in the workspace error word.
 * Requires that nothing but the append writes q, block_tables and
 * context_lens between the two launches (true by construction here).
 */
pa_status pa_kv_append_decode(const void *k_new, const void *v_new, const int32_t *slot_mapping, const void *q,
                              void *k_cache, void *v_cache, const int32_t *block_tables,
                              const int32_t *context_lens, float scale, void *out, const pa_shape *s,
                              const pa_plan_t *plan, void *workspace, size_t workspace_bytes, void *stream);

/*
 * pa_decode for callers that cannot allocate device memory: a caller whose
 * host framework owns every device allocation and gives it none, or code
 * that runs where cudaMalloc is not allowed.  It takes no workspace; it uses
 * a 16 MiB array compiled into the library instead (every GPU that loads
 * the library holds it until the process exits).  There is no counterpart
 * of this call in the pages: it only changes where the scratch lives.
 *   Arguments as in pa_decode, minus workspace and workspace_bytes.
 *   plan->workspace_bytes above 16 MiB returns PA_ERR_WORKSPACE.  Every
 *   argument is checked before anything is queued.
 *   Allocates nothing: no cudaMalloc, no cudaFree, no allocating library call.
 *   The first call on a device looks up the array's device address for that
 *   device (with it current); make that first call before any stream capture.
 *   Every call first zeroes the array's merge counters (one cudaMemsetAsync
 *   on `stream`); the array's error word is not cleared by it: it gathers the
 *   index errors of all calls until pa_no_alloc_device_error reads it.
 *   All calls share the one array: two calls that overlap on the GPU race.
 */
pa_status pa_decode_no_alloc(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
                             const int32_t *context_lens, float scale, void *out, const pa_shape *s,
                             const pa_plan_t *plan, void *stream);

/*
 * Chunked prefill over the paged cache (the step before decode: a request's
 * new tokens attend to its cached history and to each other, causally; the
 * MinivLLM review's prefill path, read straight from the pages).
 *
 * Host-only planner.  s->B is the number of requests; max_new_tokens bounds
 * query_start[b+1] - query_start[b] for every later call.  Supported: bf16
 * and fp16; D in {64, 128}; block_size a power of two in [16, 256]; a GQA
 * group Hq/Hkv that is a power of two <= 128.
 */
typedef struct {
    int32_t q_tile;          /* new tokens per query tile (q_tile * Hq/Hkv rows); a CTA takes two */
    int32_t kv_tile;         /* keys per pipeline stage */
    int32_t stages;
    int32_t num_qtiles;      /* CTA tiles (two query tiles) per request the grid covers */
    int32_t max_new_tokens;
    int32_t smem_bytes;
    pa_shape shape;
} pa_prefill_plan_t;

pa_status pa_prefill_plan(const pa_shape *s, int32_t max_new_tokens, pa_prefill_plan_t *plan_out);

/*
 * Prefill attention.  Request b owns rows query_start[b] .. query_start[b+1]-1
 * of q and out: its n_b new tokens, the last n_b of its context_lens[b]
 * positions, whose K/V must already be in the cache (pa_kv_append with one
 * row per new token: a shape whose B is the number of new tokens).  New
 * token j of request b sits at position context_lens[b] - n_b + j and
 * attends to positions 0 .. that position:
 *     out[row][h] = sum_{t <= pos} softmax_t(scale * q[row][h] . K[t]) V[t].
 *   q, out       : device, [T, Hq, D], T = query_start[B], dtype s->dtype
 *   query_start  : device, [B + 1] int32, query_start[0] = 0, non-decreasing
 *   context_lens : device, [B] int32 (history + new tokens)
 *   block_tables, k_cache, v_cache : as for pa_decode
 *   device_error : device int32 or NULL; a request with a length outside
 *                  [0, max_blocks_per_seq*block_size], more new tokens than
 *                  its length or than the plan covers is skipped and sets
 *                  PA_DEVERR_CONTEXT_LEN; a bad block id sets PA_DEVERR_BLOCK_ID.
 * No workspace; nothing is allocated.  Queued on `stream`.
 */
pa_status pa_prefill(const void *q, const void *k_cache, const void *v_cache, const int32_t *block_tables,
                     const int32_t *context_lens, const int32_t *query_start, float scale, void *out,
                     const pa_shape *s, const pa_prefill_plan_t *plan, int32_t *device_error, void *stream);

/* Copy the device error word of `workspace` to *err_out (synchronises
 * `stream`; not for the hot path).  clear != 0 resets it to 0 afterwards.
 * The word is the first four bytes of the workspace: pa_kv_append may be
 * given the same workspace pointer as its device_error. */
pa_status pa_get_device_error(void *workspace, int32_t clear, int32_t *err_out, void *stream);

/* The error word of pa_decode_no_alloc's built-in array on the current
 * device, as pa_get_device_error does for a workspace: the PA_DEVERR_* bits
 * of every pa_decode_no_alloc call since the word was last cleared
 * (synchronises `stream`; clear != 0 resets it afterwards).  Allocates
 * nothing.  No counterpart in the pages. */
pa_status pa_no_alloc_device_error(int32_t clear, int32_t *err_out, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* PAGEDATTN_H */
