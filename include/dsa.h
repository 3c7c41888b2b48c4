/*
 * dsa.h -- C ABI of libdsa.so: the prefill hot path of DeepSeek Sparse
 * Attention (DSA) on NVIDIA B200 (sm_100a).
 *
 * The path has three stages per query token t of a prefill chunk:
 *
 *   1. Lightning-indexer scores over every causally visible cached key s,
 *        I[t,s] = sum_h w[t,h] * ReLU(q_idx[t,h,:] . k_idx[s,:]),
 *      ReLU per indexer head before the signed head weight; one indexer key
 *      per position shared by all indexer heads.
 *      (mlx-lm PR #1997, "GLM prefill now attends only to the keys its indexer
 *      picks", section "How it works": the indexer scores each query against
 *      every key with 32 heads and keeps the top-k keys per query.)
 *   2. Exact top-k selection per query without an L x N score tensor in
 *      memory: a pruned candidate write-back that still returns the exact
 *      top-k (LiteTopK, arXiv 2607.11976, Abstract).  Ties go to the smaller
 *      key index.  The result is an int32 [L, topk] index tensor, each row in
 *      ascending key order, -1 where a query sees fewer than topk keys
 *      (llama.cpp PR #25917, discussion: sparse index mask, -1 = masked).
 *   3. Absorbed-MLA attention over only the gathered keys: each key is the
 *      576-wide joined cache row (512 latent + 64 rope), one gathered block is
 *      shared by all heads, the value is the 512-wide latent part
 *      (mlx-lm PR #1997, "How it works").
 *
 * Conventions for every entry point
 *   - Query t of a chunk sits at position q_pos0 + t and sees keys 0..q_pos0+t
 *     (inclusive causality, position == key index).  0 <= q_pos0, q_pos0+L <= N.
 *   - All tensor arguments are DEVICE pointers to row-major buffers owned by
 *     the caller, contiguous except for the row strides of the key caches
 *     (ldk, ldkv); the library allocates no device memory and keeps no state
 *     between calls (dsa_indexer_topk_noalloc's fixed scratch aside).
 *     Pointers must be 16-byte aligned.
 *   - bf16 / fp8 buffers are passed as raw bits (uint16 / uint8 storage).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream) and keep its order with the caller's other work.  The
 *     library's own kernels use programmatic dependent launch: each may be
 *     scheduled while its predecessor in the stream finishes, but waits for
 *     that predecessor to complete before it touches memory.  Argument errors
 *     are returned before anything is launched; a failed launch returns
 *     DSA_ERR_CUDA.  Device-side conditions (a wait that timed out, an
 *     out-of-range index) are recorded in the workspace's status word and read
 *     back with dsa_workspace_status(), which plays the role of an explicit
 *     check: every entry point clears the word when it starts (it never
 *     synchronises to look at the previous call's word), so read it after a
 *     call and before the next call on the same workspace.
 *   - No function aborts the process or throws across the ABI.
 */
#ifndef DSA_H_
#define DSA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1, /* bad pointer, size or shape */
  DSA_ERR_UNSUPPORTED = 2, /* valid but not implemented (e.g. H_I, D_I, topk) */
  DSA_ERR_WORKSPACE = 3,   /* workspace missing or too small */
  DSA_ERR_CUDA = 4,        /* a CUDA runtime / driver call failed */
  DSA_ERR_INTERNAL = 5     /* device status word reports a failure */
} dsa_status_t;

typedef enum {
  DSA_BF16 = 0,    /* bfloat16 */
  DSA_FP8_E4M3 = 1 /* OCP FP8 E4M3FN, unit scale */
} dsa_dtype_t;

typedef struct CUstream_st *dsa_stream_t; /* same type as cudaStream_t */

/* Version of this ABI (incremented on incompatible change). */
int dsa_version(void);

/* Human-readable name of a status code (static string, never NULL). */
const char *dsa_status_string(dsa_status_t status);

/* Message of the CUDA error behind the calling thread's most recent
 * DSA_ERR_CUDA (static string, never NULL; "no CUDA error recorded" if none). */
const char *dsa_last_error_string(void);

/*
 * Workspace (bytes) that dsa_indexer_topk needs for these sizes.  A larger
 * buffer is fine.  A smaller one that still holds the fixed part shrinks the
 * per-query candidate capacity; queries whose candidates do not fit are then
 * resolved by the exact fallback (slower, same result).  The fixed part holds
 * one N-score row per CTA of the exact fallback, one CTA per SM of the
 * current device (at least 16, at most one per query of a block), so the size
 * depends on the device queried.  Returns 0 for invalid sizes.
 */
size_t dsa_indexer_topk_workspace(int L, int N, int H_I, int D_I, int topk, dsa_dtype_t dtype);

/*
 * Stages 1+2: lightning-indexer scores and exact top-k per query.
 *
 *   q_idx      [L, H_I, D_I]  indexer queries, dtype bits
 *   k_idx      [N, D_I]       indexer key cache, dtype bits; rows ldk elements
 *                             apart (ldk = 0: D_I, contiguous; otherwise
 *                             ldk >= D_I and every row 16-byte aligned, e.g. a
 *                             padded cache or the leading columns of a wider
 *                             buffer; the padding is never read)
 *   w          [L, H_I]       fp32 head weights (signed)
 *   topk_idx   [L, topk]      out: int32 selected keys, ascending, -1 padded
 *   topk_score [L, topk]      out (optional, may be NULL): fp32 indexer score
 *                             of each selected key, -inf for padding
 *   workspace                 device scratch, workspace_bytes long
 *
 * Supported: D_I = 128 with H_I in {8, 16, 32} (bf16 or fp8), D_I = 64 with
 * H_I in {4, 32} (bf16); 1 <= topk <= 4096.  Queries are processed in blocks of
 * up to 1,024 (mlx-lm PR #1997, "How it works": long chunks split into query
 * blocks); the result does not depend on the blocking: every score is computed
 * by the same tensor-core instruction sequence wherever the query falls, the
 * queries the threshold sample misjudges included.
 */
dsa_status_t dsa_indexer_topk(const void *q_idx, const void *k_idx, int64_t ldk, const float *w,
                              dsa_dtype_t dtype, int L, int N, int H_I, int D_I, int q_pos0, int topk,
                              int32_t *topk_idx, float *topk_score, void *workspace, size_t workspace_bytes,
                              dsa_stream_t stream);

/*
 * dsa_indexer_topk with general visibility carried by an index mask instead of
 * the causal triangle (llama.cpp PR #25917, discussion: causality applied to
 * the indices, so that a unified cache holding several sequences, or a
 * non-triangular mask, can be expressed per query).  Query t sees exactly the
 * keys s with key_lo[t] <= s < key_hi[t]; its top-k is taken among them, with
 * -1 padding when the range holds fewer than topk keys (an empty range
 * selects nothing).  Everything else as dsa_indexer_topk.
 *
 *   key_lo, key_hi [L] int32, device, 4-byte aligned; 0 <= key_lo[t] <=
 *                  key_hi[t] <= N.  A range that breaks this is treated as
 *                  empty and flags the device status word (bit 1, see
 *                  dsa_workspace_status).
 *
 * Packed sequences (batched prefill): with several sequences stored one after
 * another in the cache, query t of the sequence starting at key b sees
 * [b, its own position + 1).  Workspace: dsa_indexer_topk_workspace.
 */
dsa_status_t dsa_indexer_topk_ranges(const void *q_idx, const void *k_idx, int64_t ldk, const float *w,
                                     dsa_dtype_t dtype, int L, int N, int H_I, int D_I, const int32_t *key_lo,
                                     const int32_t *key_hi, int topk, int32_t *topk_idx, float *topk_score,
                                     void *workspace, size_t workspace_bytes, dsa_stream_t stream);

/*
 * dsa_indexer_topk for callers that cannot allocate device memory: code that
 * owns no allocator (an inference runtime whose memory is planned once up
 * front and hands kernels only their inputs and outputs), or a process whose
 * device memory is already fully reserved by others.  Same arguments and
 * results as dsa_indexer_topk, minus the workspace: the scratch is one fixed
 * 16 MiB device array inside libdsa.so (every GPU that loads the library holds
 * it until the process exits).  The pages describe no counterpart; this is a
 * property of this library only.
 *
 *   - Limit: problems whose scratch exceeds 16 MiB at 64-query blocks are
 *     rejected with DSA_ERR_WORKSPACE before anything is launched (with
 *     top-k <= 2048 that admits N up to about 180,000 cached keys; calls of
 *     fewer than 16 queries hold fewer fallback score rows and admit more).
 *   - The first call on each device (each CUDA context: again after a device
 *     reset) looks up the array's device address with cudaGetSymbolAddress,
 *     a synchronous runtime query.
 *   - No cudaMalloc or cudaFree, and no allocating library call, is made.
 *   - Every call on a device shares the one array, which keeps the previous
 *     call's contents; the call clears what must start at zero.  Calls that
 *     overlap on the GPU (two streams, two host threads) race on the array
 *     and must be serialised by the caller.
 *   - Device-side conditions land in the array's status word; read them with
 *     dsa_indexer_topk_noalloc_status.
 */
dsa_status_t dsa_indexer_topk_noalloc(const void *q_idx, const void *k_idx, int64_t ldk, const float *w,
                                      dsa_dtype_t dtype, int L, int N, int H_I, int D_I, int q_pos0, int topk,
                                      int32_t *topk_idx, float *topk_score, dsa_stream_t stream);

/*
 * Status of the fixed scratch of dsa_indexer_topk_noalloc on the current
 * device: synchronises `stream`, reads the array's status word (bits as in
 * dsa_workspace_status) into *flags and returns DSA_OK when it is zero,
 * DSA_ERR_INTERNAL when it is not, DSA_ERR_CUDA on a CUDA error.  Like the
 * workspace's word, it describes the most recent dsa_indexer_topk_noalloc call
 * on the device, which clears it when it starts.  The pages have no
 * counterpart.
 */
dsa_status_t dsa_indexer_topk_noalloc_status(dsa_stream_t stream, unsigned *flags);

/* Workspace (bytes) for dsa_sparse_mla_prefill: the status word, plus the
 * union buffers of packed attention (H <= 32) or the fp32 partial results of
 * split-key attention (chunks with few queries), whichever is larger; the
 * size depends on the current device's SM count.  A smaller workspace (at
 * least the status word) is accepted: the call then runs neither packed nor
 * split, with the same results up to rounding. */
size_t dsa_sparse_mla_workspace(int L, int H, int topk);

/*
 * Stage 3: sparse absorbed-MLA attention.
 *
 *   q        [L, H, 576]  bf16: per head 512 latent then 64 rope columns
 *   kv       [N, 576]     bf16 joined cache: 512 latent then 64 rope columns;
 *                         rows ldkv elements apart (0: 576, contiguous;
 *                         otherwise ldkv >= 576 with 16-byte aligned rows)
 *   topk_idx [L, topk]    int32 keys per query; -1 entries are skipped; any
 *                         order; values >= N are skipped and flagged
 *   out      [L, H, 512]  out: bf16 attention output
 *   lse      [L, H]       out (optional, may be NULL): fp32 natural-log
 *                         log-sum-exp of the scaled logits, -inf if no key
 *
 *   z_j = scale * (q_lat . kv_lat[i_j] + q_rope . k_rope[i_j]);
 *   out = sum_j softmax(z)_j * kv_lat[i_j]    (fp32 accumulate, bf16 out)
 *
 * Supported: any H >= 1 (processed in groups of 64 heads), topk >= 1.
 *
 * Scheduling (results are the same up to fp32 rounding order):
 *   - H <= 32 and many queries: neighbouring queries whose selections share
 *     most keys are packed into one CTA over the union of their keys;
 *   - L * ceil(H / 64) below half the SM count (decode-like chunks): each
 *     query's selection is split into up to 16 shares of at least 128 keys,
 *     attended by separate CTAs and merged by their log-sum-exp (a second
 *     kernel).  The choice depends on L, H and topk only, never on a caller's
 *     query blocking.
 */
dsa_status_t dsa_sparse_mla_prefill(const void *q, const void *kv, int64_t ldkv, const int32_t *topk_idx, int L,
                                    int N, int H, int topk, float scale, void *out, float *lse, void *workspace,
                                    size_t workspace_bytes, dsa_stream_t stream);

/* Workspace (bytes) for dsa_prefill_chunk with these sizes (query_block <= 0
 * selects 1,024; rounded up as dsa_prefill_chunk does). */
size_t dsa_prefill_chunk_workspace(int L, int N, int H_I, int D_I, int H, int topk, int query_block,
                                   dsa_dtype_t dtype, int want_topk_out);

/*
 * All three stages for one prefill chunk, query block by query block
 * (query_block <= 0 selects 1,024 queries per block; a block size is rounded
 * up to a whole number of the indexer's query groups, 256 / H_I queries, e.g.
 * 8 at H_I = 32).  Selections and outputs are bit-identical for every blocking.
 *
 *   q_idx, k_idx, ldk, w, dtype, H_I, D_I : as dsa_indexer_topk
 *   q, kv, ldkv, H, scale                 : as dsa_sparse_mla_prefill
 *   topk_idx_out [L, topk]           : optional (may be NULL) selected keys;
 *                                      when NULL they live in the workspace
 *   out [L, H, 512], lse [L, H]      : as dsa_sparse_mla_prefill (lse optional)
 *
 * want_topk_out of the workspace query must be 0 when topk_idx_out is NULL.
 */
dsa_status_t dsa_prefill_chunk(const void *q_idx, const void *k_idx, int64_t ldk, const float *w,
                               dsa_dtype_t dtype, const void *q, const void *kv, int64_t ldkv, int L, int N, int H_I,
                               int D_I, int H, int q_pos0, int topk, float scale, int query_block,
                               int32_t *topk_idx_out, void *out, float *lse, void *workspace, size_t workspace_bytes,
                               dsa_stream_t stream);

/*
 * dsa_prefill_chunk with general visibility: query t sees keys key_lo[t] <=
 * s < key_hi[t] (as dsa_indexer_topk_ranges) instead of the causal prefix
 * from q_pos0.  Workspace: dsa_prefill_chunk_workspace.
 */
dsa_status_t dsa_prefill_chunk_ranges(const void *q_idx, const void *k_idx, int64_t ldk, const float *w,
                                      dsa_dtype_t dtype, const void *q, const void *kv, int64_t ldkv, int L, int N,
                                      int H_I, int D_I, int H, const int32_t *key_lo, const int32_t *key_hi, int topk,
                                      float scale, int query_block, int32_t *topk_idx_out, void *out, float *lse,
                                      void *workspace, size_t workspace_bytes, dsa_stream_t stream);

/*
 * dsa_prefill_chunk, additionally recording CUDA events on `stream` between
 * its stages (a profiling aid; the computation is identical).  `events` holds
 * n_events >= 7 * ceil(L / query_block) cudaEvent_t handles; for query block b,
 * events[7b + 0..6] are recorded before the pilot pass, after the pilot pass,
 * after the threshold kernel, after the main indexer pass, after the
 * selection, after the exact fallback and after the attention kernel.  A NULL
 * handle leaves that boundary unmarked (an event between two kernels keeps the
 * second from launching before the first completes).
 */
dsa_status_t dsa_prefill_chunk_profiled(const void *q_idx, const void *k_idx, int64_t ldk, const float *w,
                                        dsa_dtype_t dtype, const void *q, const void *kv, int64_t ldkv, int L, int N,
                                        int H_I, int D_I, int H, int q_pos0, int topk, float scale, int query_block,
                                        int32_t *topk_idx_out, void *out, float *lse, void *workspace,
                                        size_t workspace_bytes, dsa_stream_t stream, void *const *events,
                                        int n_events);

/*
 * Diagnostic with no counterpart in the method: exercises the bounded-wait
 * error path that every kernel of this library takes when a wait on another
 * role (or another block of the pipeline) never completes.  Clears the
 * workspace's status word, then launches one thread that waits on an mbarrier
 * nothing arrives on; after limit_ms (1..2000) it gives up and sets bit 0
 * (timeout) of the status word, the context staying usable.  Read the result
 * with dsa_workspace_status (expect DSA_ERR_INTERNAL with bit 0 set).
 *   workspace: any workspace of this library (>= its 256-byte header).
 */
dsa_status_t dsa_selftest_wait_timeout(void *workspace, size_t workspace_bytes, unsigned limit_ms,
                                       dsa_stream_t stream);

/*
 * Synchronise `stream`, read the device status word at the start of a
 * workspace used by the calls above and store it in *flags (bit 0: a wait
 * timed out, bit 1: an index outside [0, N) reached the attention stage,
 * bit 2: an internal selection count mismatch).  Returns DSA_OK when the word
 * is zero, DSA_ERR_INTERNAL when it is not, DSA_ERR_CUDA on a CUDA error.
 * Every entry point clears the word when it starts, so the word describes the
 * most recent call on this workspace: this is the explicit check of that call.
 */
dsa_status_t dsa_workspace_status(const void *workspace, dsa_stream_t stream, unsigned *flags);

/* Selection totals of the most recent dsa_indexer_topk* / dsa_prefill_chunk*
 * call on a workspace, over all its query blocks (cleared when a call starts). */
typedef struct {
  unsigned long long candidates; /* candidate keys written back (above the sample threshold), all queries */
  unsigned queries;              /* queries selected */
  unsigned fallback_queries;     /* queries the threshold sample misjudged, resolved by the exact fallback */
  unsigned max_candidates;       /* largest candidate count of one query */
  unsigned reserved;
} dsa_selection_stats_t;

/*
 * Diagnostic with no counterpart in the method: synchronise `stream` and copy
 * the selection totals above from `workspace` (DSA_ERR_INVALID_ARG for NULL
 * pointers, DSA_ERR_CUDA on a CUDA error).  LiteTopK (arXiv 2607.11976,
 * Abstract) writes back only promising candidates; these totals show how many.
 */
dsa_status_t dsa_workspace_selection_stats(const void *workspace, dsa_stream_t stream,
                                           dsa_selection_stats_t *stats);

#ifdef __cplusplus
}
#endif

#endif /* DSA_H_ */
