// dsa_internal.h -- declarations shared by the library's translation units
// (kernel argument blocks and launchers).  Not part of the public C ABI.
#pragma once
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

namespace dsa {

// Launch a kernel of this library on `stream` with programmatic stream
// serialisation: the grid may be scheduled while the previous kernel in the
// stream is still running.  Every kernel of the library starts with
// pdl_wait_and_release() (ptx.cuh), which blocks until all prerequisite grids
// have completed and their memory is visible, so the ordering seen by the
// kernel's code is exactly that of a plain launch; only the launch latency
// overlaps the predecessor's tail.
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                                 Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...);
}

// Arguments of one indexer launch (one query block).
struct IndexerArgs {
  const float *w;                 // [Lb, H_I] head weights of the block's queries
  const unsigned *tau;            // [Lb] threshold score keys (EMIT mode; 0 = keep all)
  float *dense;                   // [Lb, dense_ld] sample scores (PILOT mode)
  unsigned long long *cand;       // [Lb, cap] candidate keys (EMIT mode)
  int *cand_count;                // [Lb] candidates seen (may exceed cap)
  unsigned *status;               // device status word
  int dense_ld;
  int cap;
  int Lb;                         // queries in the block
  int q_pos0;                     // position of the block's first query
  int n_keys;                     // rows of the key tensor map (PILOT: samples, EMIT: N)
  int q_row0;                     // first row of the block in the [L*H_I, D_I] query tensor map
  int total_tiles;                // sum over query groups of their 128-key tiles
  int pilot;                      // 1 = PILOT mode
  // FALLBACK mode: the CTAs take the queries of fb_list[0 .. fb_counters[0])
  // (fb_counters[1] hands out jobs), score every visible key of the query into
  // a dense row of `dense` (dense_ld = N floats per row) and select its exact
  // top-k into topk_idx / topk_score.  With at least as many CTAs as queries,
  // a query's key tiles are split into gridDim.x / count chunks, one job each,
  // into row = the query's position in fb_list, and the CTA that completes its
  // last chunk (fb_done counts them) selects; otherwise a job is a whole query
  // and a CTA uses its own row blockIdx.x.
  const int *fb_list;             // [Lb] queries of the block, as positions tl
  int *fb_counters;               // [0] = count, [1] = next
  int *fb_done;                   // [Lb] chunks done per fallback query (zeroed by the selection)
  int32_t *topk_idx;              // [Lb, topk] rows of the block's queries
  float *topk_score;              // [Lb, topk] or nullptr
  int topk;
  // Per-query key ranges (general causality; nullptr = causal, query tl sees
  // keys <= q_pos0 + tl): query tl of the block sees keys key_lo[tl] <=
  // s < key_hi[tl].  Then group g covers the 128-key tiles grp_tile0[g] ..
  // grp_tile0[g] + grp_start[g+1] - grp_start[g] - 1, and grp_start[G] is
  // the total (total_tiles is ignored).
  const int *key_lo, *key_hi;     // [Lb] clamped ranges
  const int *grp_tile0;           // [G]
  const int *grp_start;           // [G + 1] exclusive prefix of the groups' tile counts
};

// Clamp the block's ranges into [0, N] (flagging bad ones) and plan the
// indexer's per-group tile windows.
struct RangePlanArgs {
  const int32_t *lo_in, *hi_in;   // [Lb] caller's ranges of the block's queries
  int *lo, *hi;                   // [Lb] clamped (an invalid or empty range becomes lo = hi)
  int *grp_tile0, *grp_start;     // as IndexerArgs
  unsigned *status;
  int Lb, QG, N;
};
cudaError_t launch_range_plan(const RangePlanArgs &a, cudaStream_t stream);
cudaError_t launch_wait_timeout_probe(unsigned *status, unsigned long long limit_ns, cudaStream_t stream);

// Modes of the indexer kernel: every visible score compared with the query's
// threshold (EMIT), dense scores of a key sample (PILOT), or the exact
// fallback for the queries the selection could not resolve (FALLBACK).
enum IndexerMode : int { kIdxEmit = 0, kIdxPilot = 1, kIdxFallback = 2 };

cudaError_t launch_indexer(const CUtensorMap &tq, const CUtensorMap &tk, const IndexerArgs &a, int D_I, int H_I,
                           bool fp8, IndexerMode mode, int grid, cudaStream_t stream);
bool indexer_supported(int D_I, int H_I, bool fp8);
int indexer_queries_per_group(int H_I);

// Selection totals of one call, accumulated by the selection kernel over all
// query blocks (in the workspace header; layout of dsa_selection_stats_t).
struct SelectionStats {
  unsigned long long candidates;  // candidate keys found over all queries (before the capacity cut)
  unsigned queries;               // queries selected
  unsigned fallback_queries;      // queries resolved by the exact fallback
  unsigned max_candidates;        // largest candidate count of one query
  unsigned pad;
};

// Threshold / selection stage.
struct SelectArgs {
  const float *dense;             // [Lb, dense_ld] pilot sample scores, or nullptr
  unsigned *tau;                  // [Lb] threshold score keys
  const unsigned long long *cand; // [Lb, cap]
  int *cand_count;                // [Lb]
  int *fb_list;                   // [Lb] queries that need the exact fallback
  int *fb_counters;               // [0] = count, [1] = next
  int *fb_done;                   // [Lb] chunk counters of the fallback queries (zeroed here)
  unsigned *status;
  SelectionStats *stats;          // totals over the call (workspace header)
  int32_t *topk_idx;              // [L, topk] whole chunk
  float *topk_score;              // [L, topk] or nullptr
  int dense_ld, n_samples, cap;
  const int *key_lo, *key_hi;     // [Lb] clamped per-query ranges, or nullptr (causal)
  int sample_stride;              // with ranges: pilot sample i is key i * sample_stride
  int t0, Lb, q_pos0;             // block: first query (chunk row), size, position of first query
  int N, topk;
};

cudaError_t launch_threshold(const SelectArgs &a, cudaStream_t stream);
cudaError_t launch_select(const SelectArgs &a, cudaStream_t stream);

// Sparse absorbed-MLA attention.
struct MlaArgs {
  const uint16_t *q;              // [L, H, 576] bf16 bits: per head 512 latent then 64 rope
  const int32_t *topk_idx;        // [L, topk]
  const void *kv;                 // [N, 576] bf16 joined cache, rows kv_ld elements apart
  long long kv_ld;
  uint16_t *out;                  // [L, H, 512] bf16 bits
  float *lse;                     // [L, H] or nullptr
  unsigned *status;
  int L, N, H, topk;
  int t0, Lq;                     // queries [t0, t0 + Lq) of the chunk in this launch
  float scale_log2;               // softmax scale * log2(e)
  // Packed mode (G >= 2 queries of H <= 32 heads share one 64-row tile): the
  // union of the pack's selections and, per union key, which queries chose it.
  const int32_t *ukeys;           // [npacks, umax] ascending union keys
  const unsigned long long *qmask;  // [npacks, umax / 64, 64]: word j of tile i = keys of tile i chosen by query j
  const int *ucount;              // [npacks]
  int G, umax;
  // Optional work list: CTA i serves item list[i] (a pack in packed mode, a
  // query in unpacked mode) and CTAs with i >= *list_count exit at once.
  const int *list;
  const int *list_count;
  // Split-key mode (unpacked, nsplit > 1): CTA z of a query takes its z-th
  // share of the selection and writes a partial result; a combine kernel
  // merges the shares by their log-sum-exp.
  int nsplit;
  float *part_o;                  // [Lq, H, nsplit, 512] normalised partial outputs
  float *part_lse;                // [Lq, H, nsplit] natural-log LSE of each share (-inf if empty)
};

// Union of each pack's G index rows with membership masks (packed attention).
struct PackArgs {
  const int32_t *topk_idx;        // [L, topk]
  int32_t *ukeys;
  unsigned long long *qmask;      // [npacks, umax / 64, 64] per tile and query: which keys it chose
  int *ucount;
  int *plist, *pcount;            // packs worth packing (union small enough)
  int *slist, *scount;            // queries of the other packs, served one per CTA
  unsigned *status;
  int t0, Lq, G, topk, umax, N;
  float max_union_ratio;          // pack when |union| <= ratio * sum of the members' selections
};

cudaError_t launch_pack_plan(const PackArgs &a, cudaStream_t stream);

cudaError_t launch_sparse_mla(const MlaArgs &a, bool packed, cudaStream_t stream);
cudaError_t launch_mla_combine(const MlaArgs &a, cudaStream_t stream);

}  // namespace dsa
