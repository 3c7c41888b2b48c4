// api.cu -- the C ABI of libdsa.so (declared in include/dsa.h): argument
// checks, workspace carving, TMA descriptor encoding and the per-query-block
// launch sequence of the DSA prefill path.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>

#include "dsa.h"
#include "dsa_internal.h"

namespace {

using namespace dsa;

constexpr int kDefaultQueryBlock = 1024;  // mlx-lm PR #1997: query blocks of 1,024
constexpr int kSamples = 4096;            // strided key sample per query block
constexpr int kFallbackSlots = 16;        // CTAs of the exact fallback: at least this many (exactly, without a workspace)
constexpr int kMinCap = 8192;             // default candidate capacity per query
constexpr int kMaxTopk = 4096;
constexpr size_t kHeaderBytes = 256;      // status word, fallback counters, selection totals
constexpr size_t kStatsOffset = 32;       // selection totals in the header
static_assert(sizeof(dsa::SelectionStats) == sizeof(dsa_selection_stats_t), "stats layout");

// The CUDA error behind the calling thread's last DSA_ERR_CUDA (cudaSuccess if none).
thread_local cudaError_t t_last_cuda_error = cudaSuccess;

// True on success; otherwise remembers the error for dsa_last_error_string().
bool cuda_ok(cudaError_t e) {
  if (e == cudaSuccess) return true;
  t_last_cuda_error = e;
  return false;
}

size_t align256(size_t x) { return (x + 255) & ~static_cast<size_t>(255); }
bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  // The driver entry point is looked up once; it carries no per-call state.
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2D tiled map: `rows` rows of `inner` elements, `pitch` bytes apart; box of
// box_inner x box_rows elements, 128-byte swizzle, zero fill out of bounds.
bool make_map_2d(CUtensorMap *m, const void *base, CUtensorMapDataType dt, uint64_t inner, uint64_t rows,
                 uint64_t pitch, uint32_t box_inner, uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {inner, rows};
  const cuuint64_t strides[1] = {pitch};
  const cuuint32_t box[2] = {box_inner, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  std::memset(m, 0, sizeof(*m));
  return fn(m, dt, 2, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

int default_cap(int topk) { return std::max(kMinCap, 4 * topk); }

// Queries per block: the caller's query_block (<= 0: 1,024), rounded up to a
// whole number of indexer query groups (256 / H_I queries share one tensor-core
// tile), at most L.  Every query then sits in the same group tile, at the same
// column, whatever the blocking, so its scores -- and its selection -- do not
// depend on the blocking.
int query_block_size(int L, int query_block, int H_I) {
  const int qg = (H_I > 0 && 256 % H_I == 0) ? 256 / H_I : 1;
  long long qb = query_block > 0 ? query_block : kDefaultQueryBlock;
  qb = (qb + qg - 1) / qg * qg;
  return static_cast<int>(std::min<long long>(L, qb));
}

// CTAs of the exact fallback: one per SM (at least kFallbackSlots), so that
// many fallback queries are rescored at once and a few are split over all
// of them.  Its dense score rows: one per CTA, but never more than a block
// has queries (a query's chunks share its row).
int fallback_ctas() { return std::max(kFallbackSlots, sm_count()); }
size_t fallback_rows(int QB, int fb_ctas) { return static_cast<size_t>(std::max(1, std::min(QB, fb_ctas))); }

// Fixed part of the indexer workspace (everything but the candidate lists).
size_t idx_fixed_bytes(int QB, int N, int fb_ctas) {
  return kHeaderBytes + 6 * align256(static_cast<size_t>(QB) * 4) + 2 * align256((QB + 2) * sizeof(int)) +
         align256(static_cast<size_t>(QB) * kSamples * 4) + align256(fallback_rows(QB, fb_ctas) * N * 4);
}

struct IdxWorkspace {
  unsigned *status;
  int *fb_counters;
  SelectionStats *stats;
  unsigned *tau;
  int *cand_count;
  int *fb_list;
  int *fb_done;
  float *dense;
  float *fb_scratch;
  unsigned long long *cand;
  int *rlo, *rhi;                 // [QB] clamped per-query key ranges (ranges mode)
  int *grp_tile0, *grp_start;     // per-group tile windows (ranges mode)
  int cap;
  int fb_ctas;                    // CTAs of the exact fallback (fb_scratch holds fallback_rows rows)
};

bool carve_idx_ws(void *ws, size_t bytes, int QB, int N, int fb_ctas, IdxWorkspace *o) {
  const size_t fixed = idx_fixed_bytes(QB, N, fb_ctas);
  o->fb_ctas = fb_ctas;
  if (ws == nullptr || bytes < fixed + static_cast<size_t>(QB) * 8) return false;
  uint8_t *p = static_cast<uint8_t *>(ws);
  o->status = reinterpret_cast<unsigned *>(p);
  o->fb_counters = reinterpret_cast<int *>(p + 16);
  o->stats = reinterpret_cast<SelectionStats *>(p + kStatsOffset);
  p += kHeaderBytes;
  o->tau = reinterpret_cast<unsigned *>(p);
  p += align256(static_cast<size_t>(QB) * 4);
  o->cand_count = reinterpret_cast<int *>(p);
  p += align256(static_cast<size_t>(QB) * 4);
  o->fb_list = reinterpret_cast<int *>(p);
  p += align256(static_cast<size_t>(QB) * 4);
  o->fb_done = reinterpret_cast<int *>(p);
  p += align256(static_cast<size_t>(QB) * 4);
  o->rlo = reinterpret_cast<int *>(p);
  p += align256(static_cast<size_t>(QB) * 4);
  o->rhi = reinterpret_cast<int *>(p);
  p += align256(static_cast<size_t>(QB) * 4);
  o->grp_tile0 = reinterpret_cast<int *>(p);
  p += align256((QB + 2) * sizeof(int));
  o->grp_start = reinterpret_cast<int *>(p);
  p += align256((QB + 2) * sizeof(int));
  o->dense = reinterpret_cast<float *>(p);
  p += align256(static_cast<size_t>(QB) * kSamples * 4);
  o->fb_scratch = reinterpret_cast<float *>(p);
  p += align256(fallback_rows(QB, fb_ctas) * N * 4);
  o->cand = reinterpret_cast<unsigned long long *>(p);
  const size_t room = (bytes - fixed) / (static_cast<size_t>(QB) * 8);
  o->cap = static_cast<int>(std::min<size_t>(room, 1u << 30));
  return o->cap >= 1;
}

struct IndexerProblem {
  const void *q_idx, *k_idx;
  const float *w;
  bool fp8;
  int L, N, H_I, D_I, q_pos0, topk;
  int32_t *topk_idx;
  float *topk_score;
  // Per-query key ranges (device, [L]; nullptr = causal from q_pos0).
  const int32_t *key_lo = nullptr, *key_hi = nullptr;
  long long ldk = 0;              // k_idx row stride in elements (0 = D_I, contiguous)
  long long key_ld() const { return ldk > 0 ? ldk : D_I; }
};

dsa_status_t check_indexer_args(const IndexerProblem &p) {
  if (p.q_idx == nullptr || p.k_idx == nullptr || p.w == nullptr || p.topk_idx == nullptr)
    return DSA_ERR_INVALID_ARG;
  if (!aligned16(p.q_idx) || !aligned16(p.k_idx) || !aligned16(p.w) || !aligned16(p.topk_idx))
    return DSA_ERR_INVALID_ARG;
  if (p.topk_score != nullptr && !aligned16(p.topk_score)) return DSA_ERR_INVALID_ARG;
  if (p.L <= 0 || p.N <= 0 || p.H_I <= 0 || p.D_I <= 0 || p.topk <= 0) return DSA_ERR_INVALID_ARG;
  if ((p.key_lo == nullptr) != (p.key_hi == nullptr)) return DSA_ERR_INVALID_ARG;
  if (p.key_lo == nullptr) {
    if (p.q_pos0 < 0 || static_cast<long long>(p.q_pos0) + p.L > p.N) return DSA_ERR_INVALID_ARG;
  } else if (!aligned4(p.key_lo) || !aligned4(p.key_hi)) {
    return DSA_ERR_INVALID_ARG;
  }
  if (p.topk > kMaxTopk) return DSA_ERR_UNSUPPORTED;
  if (!indexer_supported(p.D_I, p.H_I, p.fp8)) return DSA_ERR_UNSUPPORTED;
  // k_idx rows may be padded: stride >= D_I, and every row 16-byte aligned (TMA)
  if (p.ldk < 0 || (p.ldk > 0 && p.ldk < p.D_I)) return DSA_ERR_INVALID_ARG;
  if ((p.key_ld() * (p.fp8 ? 1 : 2)) % 16 != 0) return DSA_ERR_INVALID_ARG;
  return DSA_OK;
}

// Stages 1+2 for queries [t0, t0 + Lb) of the chunk.
// Record ev[i] on the stream when profiling events were supplied.
bool mark(cudaEvent_t *ev, int i, cudaStream_t stream) {
  return ev == nullptr || ev[i] == nullptr || cuda_ok(cudaEventRecord(ev[i], stream));
}

// ev (optional): 6 events recorded before the pilot, after the pilot, after the
// threshold, after the main indexer pass, after the selection, after the fallback.
dsa_status_t run_indexer_block(const IndexerProblem &p, const CUtensorMap &tq, const CUtensorMap &tk,
                               const IdxWorkspace &ws, int t0, int Lb, cudaStream_t stream,
                               cudaEvent_t *ev = nullptr) {
  const int QG = indexer_queries_per_group(p.H_I);
  const int G = (Lb + QG - 1) / QG;
  const int q_pos0 = p.q_pos0 + t0;
  const int sms = std::max(1, sm_count());
  const long long esz = p.fp8 ? 1 : 2;
  const long long row_bytes = p.key_ld() * esz;  // k_idx row pitch

  IndexerArgs ia{};
  ia.w = p.w + static_cast<long long>(t0) * p.H_I;
  ia.tau = ws.tau;
  ia.dense = ws.dense;
  ia.cand = ws.cand;
  ia.cand_count = ws.cand_count;
  ia.status = ws.status;
  ia.cap = ws.cap;
  ia.Lb = Lb;
  ia.q_pos0 = q_pos0;
  ia.q_row0 = t0 * p.H_I;

  const bool ranges = p.key_lo != nullptr;
  if (!mark(ev, 0, stream)) return DSA_ERR_CUDA;
  if (ranges) {
    // Clamp the block's ranges and plan the indexer's per-group key windows.
    RangePlanArgs ra{};
    ra.lo_in = p.key_lo + t0;
    ra.hi_in = p.key_hi + t0;
    ra.lo = ws.rlo;
    ra.hi = ws.rhi;
    ra.grp_tile0 = ws.grp_tile0;
    ra.grp_start = ws.grp_start;
    ra.status = ws.status;
    ra.Lb = Lb;
    ra.QG = QG;
    ra.N = p.N;
    if (!cuda_ok(launch_range_plan(ra, stream))) return DSA_ERR_CUDA;
    ia.key_lo = ws.rlo;
    ia.key_hi = ws.rhi;
    ia.grp_tile0 = ws.grp_tile0;
    ia.grp_start = ws.grp_start;
  }
  // The pilot samples the keys a query can see: with ranges (unknown on the
  // host) it samples the whole cache and each query uses the samples inside
  // its own range.
  const long long sampled = ranges ? p.N : static_cast<long long>(q_pos0) + 1;
  const bool pilot = ranges ? p.N > ws.cap : static_cast<long long>(q_pos0) + Lb > ws.cap;
  int n_samples = 0;
  long long stride = 1;
  if (pilot) {
    n_samples = static_cast<int>(std::min<long long>(kSamples, sampled));
    stride = sampled / n_samples;
    CUtensorMap ts;
    const CUtensorMapDataType dt = p.fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    if (!make_map_2d(&ts, p.k_idx, dt, p.D_I, n_samples, stride * row_bytes, 128 / esz, 128)) return DSA_ERR_CUDA;
    IndexerArgs pa = ia;
    pa.pilot = 1;
    pa.dense_ld = n_samples;
    pa.n_keys = n_samples;
    pa.total_tiles = G * ((n_samples + 127) / 128);
    if (!cuda_ok(launch_indexer(tq, ts, pa, p.D_I, p.H_I, p.fp8, kIdxPilot, std::min(sms, pa.total_tiles), stream)))
      return DSA_ERR_CUDA;
  }

  SelectArgs sa{};
  sa.dense = pilot ? ws.dense : nullptr;
  sa.tau = ws.tau;
  sa.cand = ws.cand;
  sa.cand_count = ws.cand_count;
  sa.fb_list = ws.fb_list;
  sa.fb_counters = ws.fb_counters;
  sa.fb_done = ws.fb_done;
  sa.status = ws.status;
  sa.stats = ws.stats;
  sa.topk_idx = p.topk_idx;
  sa.topk_score = p.topk_score;
  sa.dense_ld = n_samples;
  sa.n_samples = n_samples;
  sa.cap = ws.cap;
  sa.t0 = t0;
  sa.Lb = Lb;
  sa.q_pos0 = q_pos0;
  sa.key_lo = ranges ? ws.rlo : nullptr;
  sa.key_hi = ranges ? ws.rhi : nullptr;
  sa.sample_stride = static_cast<int>(stride);
  sa.N = p.N;
  sa.topk = p.topk;
  if (!mark(ev, 1, stream)) return DSA_ERR_CUDA;
  if (!cuda_ok(launch_threshold(sa, stream))) return DSA_ERR_CUDA;
  if (!mark(ev, 2, stream)) return DSA_ERR_CUDA;

  IndexerArgs ea = ia;
  ea.pilot = 0;
  ea.n_keys = p.N;
  long long total = 0;
  if (ranges) {
    total = static_cast<long long>(G) * ((p.N + 127) / 128);  // an upper bound; the kernel reads the plan
  } else {
    for (int g = 0; g < G; ++g) {
      const int last = std::min(Lb, (g + 1) * QG);
      const long long keys = std::min<long long>(p.N, static_cast<long long>(q_pos0) + last);
      total += (keys + 127) / 128;
    }
  }
  if (total > (1ll << 30)) return DSA_ERR_UNSUPPORTED;
  ea.total_tiles = static_cast<int>(total);
  if (!cuda_ok(launch_indexer(tq, tk, ea, p.D_I, p.H_I, p.fp8, kIdxEmit,
                              static_cast<int>(std::min<long long>(sms, total)), stream)))
    return DSA_ERR_CUDA;
  if (!mark(ev, 3, stream)) return DSA_ERR_CUDA;
  if (!cuda_ok(launch_select(sa, stream))) return DSA_ERR_CUDA;
  if (!mark(ev, 4, stream)) return DSA_ERR_CUDA;
  // Exact fallback for the queries the selection handed over: the indexer
  // kernel rescores each of them over all its visible keys with the main
  // pass's arithmetic (same group tile, same key tiles) into a dense row and
  // selects from it.  With no such query its CTAs exit at once.
  IndexerArgs fa = ea;
  fa.dense = ws.fb_scratch;
  fa.dense_ld = p.N;
  fa.fb_list = ws.fb_list;
  fa.fb_counters = ws.fb_counters;
  fa.fb_done = ws.fb_done;
  fa.topk_idx = p.topk_idx + static_cast<long long>(t0) * p.topk;
  fa.topk_score = p.topk_score ? p.topk_score + static_cast<long long>(t0) * p.topk : nullptr;
  fa.topk = p.topk;
  if (!cuda_ok(launch_indexer(tq, tk, fa, p.D_I, p.H_I, p.fp8, kIdxFallback, ws.fb_ctas, stream)))
    return DSA_ERR_CUDA;
  if (!mark(ev, 5, stream)) return DSA_ERR_CUDA;
  return DSA_OK;
}

bool make_indexer_maps(const IndexerProblem &p, CUtensorMap *tq, CUtensorMap *tk) {
  const CUtensorMapDataType dt = p.fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const uint32_t esz = p.fp8 ? 1 : 2;
  const uint64_t row_bytes = static_cast<uint64_t>(p.D_I) * esz;
  return make_map_2d(tq, p.q_idx, dt, p.D_I, static_cast<uint64_t>(p.L) * p.H_I, row_bytes, 128 / esz, 256) &&
         make_map_2d(tk, p.k_idx, dt, p.D_I, p.N, static_cast<uint64_t>(p.key_ld()) * esz, 128 / esz, 128);
}

struct MlaProblem {
  const void *q, *kv;
  const int32_t *topk_idx;
  int L, N, H, topk;
  float scale;
  void *out;
  float *lse;
  long long ldkv = 0;             // kv row stride in elements (0 = 576, contiguous)
  long long kv_ld() const { return ldkv > 0 ? ldkv : 576; }
};

dsa_status_t check_mla_args(const MlaProblem &p) {
  if (p.q == nullptr || p.kv == nullptr || p.topk_idx == nullptr || p.out == nullptr) return DSA_ERR_INVALID_ARG;
  if (!aligned16(p.q) || !aligned16(p.kv) || !aligned16(p.topk_idx) || !aligned16(p.out))
    return DSA_ERR_INVALID_ARG;
  if (p.lse != nullptr && !aligned16(p.lse)) return DSA_ERR_INVALID_ARG;
  if (p.L <= 0 || p.N <= 0 || p.H <= 0 || p.topk <= 0) return DSA_ERR_INVALID_ARG;
  if (!std::isfinite(p.scale)) return DSA_ERR_INVALID_ARG;
  // kv rows may be padded: stride >= 576 elements, every row 16-byte aligned (16-byte copies)
  if (p.ldkv < 0 || (p.ldkv > 0 && p.ldkv < 576) || (p.kv_ld() * 2) % 16 != 0) return DSA_ERR_INVALID_ARG;
  if (static_cast<long long>(p.L) * p.H >= (1ll << 31)) return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

// ---- query packing for the attention stage (LiteDSA-style candidate reuse)
constexpr int kPackMaxEntries = 8192;  // G * topk selection entries per pack (bounds the union)
constexpr float kMaxUnionRatio = 0.75f; // pack when the union is at most 75% of the members' keys

// Queries packed per CTA: with H <= 32 heads a 64-row tile has room for
// 64 / H queries, and packing them over the union of their selections never
// adds tensor work (the rows were idle) while shared keys are gathered once.
// Capped so the attention grid still covers the GPU at least twice.  Decided
// from the whole chunk's L (never a query block's) and rounded down to a power
// of two, so that packs, which start at a block's first query, are the same
// for every blocking (blocks are whole multiples of 8 queries).
int pack_group(int H, int topk, int L, int N) {
  if (H <= 0 || topk <= 0) return 1;
  if (H > 32 || N > 800 * 1024) return 1;  // the pack plan's key bitmap must fit in shared memory
  int G = std::min(64 / H, 8);  // the attention kernel tracks up to 8 queries per CTA
  G = std::min(G, kPackMaxEntries / topk);
  G = std::min(G, std::max(1, L / (2 * std::max(1, sm_count()))));
  G = std::max(G, 1);
  while (G & (G - 1)) G &= G - 1;  // largest power of two <= G
  return G;
}

// Union buffers for up to Lq queries packed G at a time (any G).
size_t union_bytes(int Lq, int topk) {
  // packs * (G * topk rounded up to whole 64-key tiles), for any G
  const size_t slots = static_cast<size_t>(Lq + 64) * topk + static_cast<size_t>(Lq + 1) * 64;
  return align256(slots * 4) + align256(slots * 8) + 3 * align256(static_cast<size_t>(Lq) * 4) + 256;
}

// Split-key attention: when a chunk has too few (query, 64-head group) items
// to occupy the GPU (decode-like shapes), each query's selection is divided
// among up to 16 CTAs of at least two 64-key tiles each, and the shares are
// merged by their log-sum-exp.  Decided from the whole chunk's L, never from
// a query block's size, so that results do not depend on the blocking.
int mla_splits(int L, int H, int topk) {
  const int items = L * ((H + 63) / 64);
  const int sms = std::max(1, sm_count());
  if (items <= 0 || 2 * items > sms) return 1;
  return std::max(1, std::min({16, (topk + 127) / 128, sms / items}));
}

// Partial results of a block of Lq queries with ns shares each.
size_t split_bytes(int Lq, int H, int ns) {
  if (Lq <= 0 || ns <= 1) return 0;
  const size_t rows = static_cast<size_t>(Lq) * H * ns;
  return align256(rows * 512 * 4) + align256(rows * 4);
}

// Scratch of the attention stage beyond the status header: the union buffers
// of packed attention or the partial results of split-key attention (the two
// never occur in the same block: packing needs many queries, splitting few).
struct UnionWorkspace {
  void *base = nullptr;
  size_t bytes = 0;
};

// Attention scratch for an L-query chunk run in blocks of QB: the larger of
// the packing unions (H <= 32) and the split-key partials of either block size.
size_t attention_scratch_bytes(int L, int QB, int H, int topk) {
  const size_t b = H <= 32 ? union_bytes(QB, topk) : 0;
  return std::max(b, split_bytes(std::min(L, QB), H, mla_splits(L, H, topk)));
}

dsa_status_t run_mla_block(const MlaProblem &p, unsigned *status, int t0, int Lq, cudaStream_t stream,
                           UnionWorkspace uw = UnionWorkspace()) {
  // p.L is the whole chunk's query count (see mla_splits).
  MlaArgs a{};
  a.q = static_cast<const uint16_t *>(p.q);
  a.topk_idx = p.topk_idx;
  a.kv = p.kv;
  a.kv_ld = p.kv_ld();
  a.out = static_cast<uint16_t *>(p.out);
  a.lse = p.lse;
  a.status = status;
  a.L = p.L;
  a.N = p.N;
  a.H = p.H;
  a.topk = p.topk;
  a.t0 = t0;
  a.Lq = Lq;
  a.scale_log2 = p.scale * 1.4426950408889634f;
  a.G = 1;
  a.nsplit = 1;
  const int ns = mla_splits(p.L, p.H, p.topk);
  if (ns > 1 && uw.base != nullptr && uw.bytes >= split_bytes(Lq, p.H, ns)) {
    const size_t rows = static_cast<size_t>(Lq) * p.H * ns;
    a.nsplit = ns;
    a.part_o = static_cast<float *>(uw.base);
    a.part_lse = reinterpret_cast<float *>(static_cast<uint8_t *>(uw.base) + align256(rows * 512 * 4));
    if (!cuda_ok(launch_sparse_mla(a, false, stream))) return DSA_ERR_CUDA;
    return cuda_ok(launch_mla_combine(a, stream)) ? DSA_OK : DSA_ERR_CUDA;
  }
  const int G = pack_group(p.H, p.topk, p.L, p.N);
  if (G >= 2 && uw.base != nullptr && uw.bytes >= union_bytes(Lq, p.topk)) {
    const int npacks = (Lq + G - 1) / G;
    const int umax = (G * p.topk + 63) / 64 * 64;  // whole 64-key tiles
    const size_t slots = static_cast<size_t>(npacks) * umax;
    uint8_t *b = static_cast<uint8_t *>(uw.base);
    PackArgs pa{};
    pa.topk_idx = p.topk_idx;
    pa.ukeys = reinterpret_cast<int32_t *>(b);
    pa.qmask = reinterpret_cast<unsigned long long *>(b + align256(slots * 4));
    uint8_t *c = b + align256(slots * 4) + align256(slots * 8);
    pa.ucount = reinterpret_cast<int *>(c);
    pa.plist = reinterpret_cast<int *>(c + align256(static_cast<size_t>(Lq) * 4));
    pa.slist = reinterpret_cast<int *>(c + 2 * align256(static_cast<size_t>(Lq) * 4));
    int *counters = reinterpret_cast<int *>(c + 3 * align256(static_cast<size_t>(Lq) * 4));
    pa.pcount = counters;
    pa.scount = counters + 1;
    pa.max_union_ratio = kMaxUnionRatio;
    pa.status = status;
    if (!cuda_ok(cudaMemsetAsync(counters, 0, 2 * sizeof(int), stream))) return DSA_ERR_CUDA;
    pa.t0 = t0;
    pa.Lq = Lq;
    pa.G = G;
    pa.topk = p.topk;
    pa.umax = umax;
    pa.N = p.N;
    if (!cuda_ok(launch_pack_plan(pa, stream))) return DSA_ERR_CUDA;
    a.G = G;
    a.umax = umax;
    a.ukeys = pa.ukeys;
    a.qmask = pa.qmask;
    a.ucount = pa.ucount;
    a.list = pa.plist;
    a.list_count = pa.pcount;
    if (!cuda_ok(launch_sparse_mla(a, true, stream))) return DSA_ERR_CUDA;
    MlaArgs single = a;
    single.G = 1;
    single.list = pa.slist;
    single.list_count = pa.scount;
    return cuda_ok(launch_sparse_mla(single, false, stream)) ? DSA_OK : DSA_ERR_CUDA;
  }
  return cuda_ok(launch_sparse_mla(a, false, stream)) ? DSA_OK : DSA_ERR_CUDA;
}

}  // namespace

extern "C" {

int dsa_version(void) { return 1; }

const char *dsa_last_error_string(void) {
  return t_last_cuda_error == cudaSuccess ? "no CUDA error recorded" : cudaGetErrorString(t_last_cuda_error);
}

const char *dsa_status_string(dsa_status_t s) {
  switch (s) {
    case DSA_OK: return "DSA_OK";
    case DSA_ERR_INVALID_ARG: return "DSA_ERR_INVALID_ARG: bad pointer, size or shape";
    case DSA_ERR_UNSUPPORTED: return "DSA_ERR_UNSUPPORTED: valid but unsupported shape or type";
    case DSA_ERR_WORKSPACE: return "DSA_ERR_WORKSPACE: workspace missing or too small";
    case DSA_ERR_CUDA: return "DSA_ERR_CUDA: a CUDA call failed";
    case DSA_ERR_INTERNAL: return "DSA_ERR_INTERNAL: device status word reports a failure";
  }
  return "unknown dsa_status_t";
}

size_t dsa_indexer_topk_workspace(int L, int N, int H_I, int D_I, int topk, dsa_dtype_t dtype) {
  if (L <= 0 || N <= 0 || H_I <= 0 || D_I <= 0 || topk <= 0) return 0;
  (void)dtype;
  const int QB = query_block_size(L, 0, H_I);
  return idx_fixed_bytes(QB, N, fallback_ctas()) + align256(static_cast<size_t>(QB) * default_cap(topk) * 8);
}

}  // extern "C"

namespace {

dsa_status_t indexer_topk_impl(const void *q_idx, const void *k_idx, int64_t ldk, const float *w, dsa_dtype_t dtype,
                               int L, int N, int H_I, int D_I, int q_pos0, const int32_t *key_lo,
                               const int32_t *key_hi, int topk, int32_t *topk_idx, float *topk_score, void *workspace,
                               size_t workspace_bytes, dsa_stream_t stream_) {
  if (dtype != DSA_BF16 && dtype != DSA_FP8_E4M3) return DSA_ERR_INVALID_ARG;
  IndexerProblem p{q_idx, k_idx, w, dtype == DSA_FP8_E4M3, L, N, H_I, D_I, q_pos0, topk, topk_idx, topk_score};
  p.key_lo = key_lo;
  p.key_hi = key_hi;
  p.ldk = ldk;
  dsa_status_t st = check_indexer_args(p);
  if (st != DSA_OK) return st;
  const int QB = query_block_size(L, 0, H_I);
  IdxWorkspace ws;
  if (!carve_idx_ws(workspace, workspace_bytes, QB, N, fallback_ctas(), &ws)) return DSA_ERR_WORKSPACE;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  CUtensorMap tq, tk;
  if (!make_indexer_maps(p, &tq, &tk)) return DSA_ERR_CUDA;
  if (!cuda_ok(cudaMemsetAsync(ws.status, 0, kHeaderBytes, stream))) return DSA_ERR_CUDA;
  for (int t0 = 0; t0 < L; t0 += QB) {
    st = run_indexer_block(p, tq, tk, ws, t0, std::min(QB, L - t0), stream);
    if (st != DSA_OK) return st;
  }
  return DSA_OK;
}

}  // namespace

extern "C" {

dsa_status_t dsa_indexer_topk(const void *q_idx, const void *k_idx, int64_t ldk, const float *w, dsa_dtype_t dtype,
                              int L, int N, int H_I, int D_I, int q_pos0, int topk, int32_t *topk_idx,
                              float *topk_score, void *workspace, size_t workspace_bytes, dsa_stream_t stream) {
  return indexer_topk_impl(q_idx, k_idx, ldk, w, dtype, L, N, H_I, D_I, q_pos0, nullptr, nullptr, topk, topk_idx,
                           topk_score, workspace, workspace_bytes, stream);
}

dsa_status_t dsa_indexer_topk_ranges(const void *q_idx, const void *k_idx, int64_t ldk, const float *w,
                                     dsa_dtype_t dtype, int L, int N, int H_I, int D_I, const int32_t *key_lo,
                                     const int32_t *key_hi, int topk, int32_t *topk_idx, float *topk_score,
                                     void *workspace, size_t workspace_bytes, dsa_stream_t stream) {
  if (key_lo == nullptr || key_hi == nullptr) return DSA_ERR_INVALID_ARG;
  return indexer_topk_impl(q_idx, k_idx, ldk, w, dtype, L, N, H_I, D_I, 0, key_lo, key_hi, topk, topk_idx,
                           topk_score, workspace, workspace_bytes, stream);
}

size_t dsa_sparse_mla_workspace(int L, int H, int topk) {
  if (L <= 0 || H <= 0 || topk <= 0) return 0;
  return kHeaderBytes + attention_scratch_bytes(L, L, H, topk);
}

dsa_status_t dsa_sparse_mla_prefill(const void *q, const void *kv, int64_t ldkv, const int32_t *topk_idx, int L,
                                    int N, int H, int topk, float scale, void *out, float *lse, void *workspace,
                                    size_t workspace_bytes, dsa_stream_t stream_) {
  MlaProblem p{q, kv, topk_idx, L, N, H, topk, scale, out, lse};
  p.ldkv = ldkv;
  dsa_status_t st = check_mla_args(p);
  if (st != DSA_OK) return st;
  if (workspace == nullptr || workspace_bytes < kHeaderBytes) return DSA_ERR_WORKSPACE;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  unsigned *status = static_cast<unsigned *>(workspace);
  if (!cuda_ok(cudaMemsetAsync(status, 0, kHeaderBytes, stream))) return DSA_ERR_CUDA;
  UnionWorkspace uw;
  uw.base = static_cast<uint8_t *>(workspace) + kHeaderBytes;
  uw.bytes = workspace_bytes - kHeaderBytes;
  return run_mla_block(p, status, 0, L, stream, uw);
}

size_t dsa_prefill_chunk_workspace(int L, int N, int H_I, int D_I, int H, int topk, int query_block,
                                   dsa_dtype_t dtype, int want_topk_out) {
  if (L <= 0 || N <= 0 || H_I <= 0 || D_I <= 0 || H <= 0 || topk <= 0) return 0;
  (void)dtype;
  const int QB = query_block_size(L, query_block, H_I);
  size_t bytes = idx_fixed_bytes(QB, N, fallback_ctas()) + align256(static_cast<size_t>(QB) * default_cap(topk) * 8);
  if (!want_topk_out) bytes += align256(static_cast<size_t>(QB) * topk * 4);
  const size_t extra = attention_scratch_bytes(L, QB, H, topk);
  if (extra > 0) bytes += extra + 256;
  return bytes;
}

}  // extern "C"

namespace {

dsa_status_t prefill_chunk_impl(const void *q_idx, const void *k_idx, int64_t ldk, const float *w, dsa_dtype_t dtype,
                                const void *q, const void *kv, int64_t ldkv, int L, int N, int H_I, int D_I, int H,
                                int q_pos0, const int32_t *key_lo, const int32_t *key_hi, int topk, float scale,
                                int query_block, int32_t *topk_idx_out, void *out, float *lse, void *workspace,
                                size_t workspace_bytes, dsa_stream_t stream_, cudaEvent_t *events, int n_events) {
  if (dtype != DSA_BF16 && dtype != DSA_FP8_E4M3) return DSA_ERR_INVALID_ARG;
  // Sizes first: the scratch planning below divides by them.
  if (L <= 0 || N <= 0 || H_I <= 0 || D_I <= 0 || H <= 0 || topk <= 0) return DSA_ERR_INVALID_ARG;
  const int QB = query_block_size(L, query_block, H_I);
  // Selected keys: the caller's buffer, or a block-sized region at the end of the workspace.
  size_t idx_bytes = workspace_bytes;
  int32_t *block_idx = nullptr;
  if (topk_idx_out == nullptr) {
    const size_t need = align256(static_cast<size_t>(QB) * topk * 4);
    if (workspace == nullptr || workspace_bytes < need) return DSA_ERR_WORKSPACE;
    idx_bytes = (workspace_bytes - need) & ~static_cast<size_t>(255);
    block_idx = reinterpret_cast<int32_t *>(static_cast<uint8_t *>(workspace) + idx_bytes);
  }
  // Attention scratch (packed-attention unions or split-key partials), below the selected keys.
  UnionWorkspace uw;
  const size_t ub = attention_scratch_bytes(L, QB, H, topk);
  const size_t idx_need =
      idx_fixed_bytes(QB, N, fallback_ctas()) + align256(static_cast<size_t>(QB) * default_cap(topk) * 8);
  if (ub > 0 && workspace != nullptr && idx_bytes >= ub + idx_need) {
    const size_t off = (idx_bytes - ub) & ~static_cast<size_t>(255);
    uw.base = static_cast<uint8_t *>(workspace) + off;
    uw.bytes = idx_bytes - off;
    idx_bytes = off;
  }
  IndexerProblem ip{q_idx, k_idx, w, dtype == DSA_FP8_E4M3, L, N, H_I, D_I, q_pos0, topk,
                    topk_idx_out ? topk_idx_out : block_idx, nullptr};
  ip.key_lo = key_lo;
  ip.key_hi = key_hi;
  ip.ldk = ldk;
  dsa_status_t st = check_indexer_args(ip);
  if (st != DSA_OK) return st;
  MlaProblem mp{q, kv, ip.topk_idx, L, N, H, topk, scale, out, lse};
  mp.ldkv = ldkv;
  st = check_mla_args(mp);
  if (st != DSA_OK) return st;
  IdxWorkspace ws;
  if (!carve_idx_ws(workspace, idx_bytes, QB, N, fallback_ctas(), &ws)) return DSA_ERR_WORKSPACE;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  CUtensorMap tq, tk;
  if (!make_indexer_maps(ip, &tq, &tk)) return DSA_ERR_CUDA;
  const int nblocks = (L + QB - 1) / QB;
  if (events != nullptr && n_events < 7 * nblocks) return DSA_ERR_INVALID_ARG;
  if (!cuda_ok(cudaMemsetAsync(ws.status, 0, kHeaderBytes, stream))) return DSA_ERR_CUDA;
  for (int t0 = 0; t0 < L; t0 += QB) {
    const int Lb = std::min(QB, L - t0);
    cudaEvent_t *ev = events ? events + 7 * (t0 / QB) : nullptr;
    IndexerProblem bp = ip;
    MlaProblem bm = mp;
    if (block_idx != nullptr) {
      // The block's indices land at rows [0, Lb) of the workspace buffer.
      bp.topk_idx = block_idx - static_cast<long long>(t0) * topk;
      bm.topk_idx = bp.topk_idx;
    }
    st = run_indexer_block(bp, tq, tk, ws, t0, Lb, stream, ev);
    if (st != DSA_OK) return st;
    st = run_mla_block(bm, ws.status, t0, Lb, stream, uw);
    if (st != DSA_OK) return st;
    if (!mark(ev, 6, stream)) return DSA_ERR_CUDA;
  }
  return DSA_OK;
}

}  // namespace

extern "C" {

dsa_status_t dsa_prefill_chunk(const void *q_idx, const void *k_idx, int64_t ldk, const float *w, dsa_dtype_t dtype,
                               const void *q, const void *kv, int64_t ldkv, int L, int N, int H_I, int D_I, int H,
                               int q_pos0, int topk, float scale, int query_block, int32_t *topk_idx_out, void *out,
                               float *lse, void *workspace, size_t workspace_bytes, dsa_stream_t stream) {
  return prefill_chunk_impl(q_idx, k_idx, ldk, w, dtype, q, kv, ldkv, L, N, H_I, D_I, H, q_pos0, nullptr, nullptr,
                            topk, scale, query_block, topk_idx_out, out, lse, workspace, workspace_bytes, stream,
                            nullptr, 0);
}

dsa_status_t dsa_prefill_chunk_ranges(const void *q_idx, const void *k_idx, int64_t ldk, const float *w,
                                      dsa_dtype_t dtype, const void *q, const void *kv, int64_t ldkv, int L, int N,
                                      int H_I, int D_I, int H, const int32_t *key_lo, const int32_t *key_hi, int topk,
                                      float scale, int query_block, int32_t *topk_idx_out, void *out, float *lse,
                                      void *workspace, size_t workspace_bytes, dsa_stream_t stream) {
  if (key_lo == nullptr || key_hi == nullptr) return DSA_ERR_INVALID_ARG;
  return prefill_chunk_impl(q_idx, k_idx, ldk, w, dtype, q, kv, ldkv, L, N, H_I, D_I, H, 0, key_lo, key_hi, topk,
                            scale, query_block, topk_idx_out, out, lse, workspace, workspace_bytes, stream, nullptr,
                            0);
}

dsa_status_t dsa_prefill_chunk_profiled(const void *q_idx, const void *k_idx, int64_t ldk, const float *w,
                                        dsa_dtype_t dtype, const void *q, const void *kv, int64_t ldkv, int L, int N,
                                        int H_I, int D_I, int H, int q_pos0, int topk, float scale, int query_block,
                                        int32_t *topk_idx_out, void *out, float *lse, void *workspace,
                                        size_t workspace_bytes, dsa_stream_t stream, void *const *events,
                                        int n_events) {
  if (events == nullptr) return DSA_ERR_INVALID_ARG;
  return prefill_chunk_impl(q_idx, k_idx, ldk, w, dtype, q, kv, ldkv, L, N, H_I, D_I, H, q_pos0, nullptr, nullptr,
                            topk, scale, query_block, topk_idx_out, out, lse, workspace, workspace_bytes, stream,
                            reinterpret_cast<cudaEvent_t *>(const_cast<void **>(events)), n_events);
}

dsa_status_t dsa_selftest_wait_timeout(void *workspace, size_t workspace_bytes, unsigned limit_ms,
                                       dsa_stream_t stream_) {
  if (workspace == nullptr || workspace_bytes < kHeaderBytes) return DSA_ERR_WORKSPACE;
  if (limit_ms == 0 || limit_ms > 2000) return DSA_ERR_INVALID_ARG;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  unsigned *status = static_cast<unsigned *>(workspace);
  if (!cuda_ok(cudaMemsetAsync(status, 0, kHeaderBytes, stream))) return DSA_ERR_CUDA;
  return cuda_ok(launch_wait_timeout_probe(status, static_cast<unsigned long long>(limit_ms) * 1000000ull, stream))
             ? DSA_OK
             : DSA_ERR_CUDA;
}

dsa_status_t dsa_workspace_selection_stats(const void *workspace, dsa_stream_t stream_,
                                           dsa_selection_stats_t *stats) {
  if (workspace == nullptr || stats == nullptr) return DSA_ERR_INVALID_ARG;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  if (!cuda_ok(cudaStreamSynchronize(stream))) return DSA_ERR_CUDA;
  if (!cuda_ok(cudaMemcpy(stats, static_cast<const uint8_t *>(workspace) + kStatsOffset, sizeof(*stats),
                          cudaMemcpyDeviceToHost)))
    return DSA_ERR_CUDA;
  return DSA_OK;
}

dsa_status_t dsa_workspace_status(const void *workspace, dsa_stream_t stream_, unsigned *flags) {
  if (workspace == nullptr || flags == nullptr) return DSA_ERR_INVALID_ARG;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  unsigned v = 0;
  if (!cuda_ok(cudaStreamSynchronize(stream))) return DSA_ERR_CUDA;
  if (!cuda_ok(cudaMemcpy(&v, workspace, sizeof(v), cudaMemcpyDeviceToHost))) return DSA_ERR_CUDA;
  *flags = v;
  return v == 0 ? DSA_OK : DSA_ERR_INTERNAL;
}

}  // extern "C"

// ---------------------------------------------------------------------------
// dsa_indexer_topk_noalloc: the indexer top-k for callers that cannot allocate
// device memory (see include/dsa.h).  Its scratch is this file-scope device
// array, held by every GPU that loads the library until the process exits.
// Host code cannot use the array's name as a device address: the address is
// looked up with cudaGetSymbolAddress, with the device current, the first time
// a device (more exactly, a CUDA context on it) is used, and passed on.
// ---------------------------------------------------------------------------
#include <mutex>

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB
constexpr int kNoAllocQueryBlock = 64;                      // queries per block in the fixed scratch
constexpr int kNoAllocMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Identity of the calling thread's current CUDA context (0 if there is none
// or the driver cannot tell).  A device reset or a re-created primary context
// gets a new identity, and the library's module -- with the array -- may then
// sit elsewhere, so the cached address is keyed on it.
unsigned long long current_context_id() {
  typedef CUresult (*GetCurrentFn)(CUcontext *);
  typedef CUresult (*GetIdFn)(CUcontext, unsigned long long *);
  static GetCurrentFn get_current = nullptr;
  static GetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetCurrent", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrentFn>(p);
    p = nullptr;
    if (cudaGetDriverEntryPointByVersion("cuCtxGetId", &p, 12000, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetIdFn>(p);
  });
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current == nullptr || get_id == nullptr || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

struct NoAllocEntry {
  void *addr = nullptr;
  unsigned long long ctx_id = 0;
};
std::mutex g_noalloc_mutex;
NoAllocEntry g_noalloc[kNoAllocMaxDevices];

// Device address of the scratch array in the current device's context.  The
// lookup runs on the first call in a context (and on every call if the
// context's identity cannot be read).
dsa_status_t noalloc_scratch(void **out) {
  int dev = 0;
  if (!cuda_ok(cudaGetDevice(&dev))) return DSA_ERR_CUDA;
  if (dev < 0 || dev >= kNoAllocMaxDevices) return DSA_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_noalloc_mutex);
  NoAllocEntry &e = g_noalloc[dev];
  const unsigned long long id = current_context_id();
  if (e.addr == nullptr || id == 0 || id != e.ctx_id) {
    void *p = nullptr;
    if (!cuda_ok(cudaGetSymbolAddress(&p, g_noalloc_scratch))) return DSA_ERR_CUDA;
    e.addr = p;
    e.ctx_id = current_context_id();  // the lookup may have created the context
  }
  *out = e.addr;
  return DSA_OK;
}

}  // namespace

extern "C" dsa_status_t dsa_indexer_topk_noalloc(const void *q_idx, const void *k_idx, int64_t ldk, const float *w,
                                                 dsa_dtype_t dtype, int L, int N, int H_I, int D_I, int q_pos0,
                                                 int topk, int32_t *topk_idx, float *topk_score,
                                                 dsa_stream_t stream_) {
  if (dtype != DSA_BF16 && dtype != DSA_FP8_E4M3) return DSA_ERR_INVALID_ARG;
  IndexerProblem p{q_idx, k_idx, w, dtype == DSA_FP8_E4M3, L, N, H_I, D_I, q_pos0, topk, topk_idx, topk_score};
  p.ldk = ldk;
  dsa_status_t st = check_indexer_args(p);
  if (st != DSA_OK) return st;
  const int QB = query_block_size(L, kNoAllocQueryBlock, H_I);
  // Too large for the fixed scratch: refuse before touching the device.
  if (idx_fixed_bytes(QB, N, kFallbackSlots) + static_cast<size_t>(QB) * default_cap(topk) * 8 > kNoAllocScratchBytes)
    return DSA_ERR_WORKSPACE;
  void *scratch = nullptr;
  st = noalloc_scratch(&scratch);
  if (st != DSA_OK) return st;
  IdxWorkspace ws;
  if (!carve_idx_ws(scratch, kNoAllocScratchBytes, QB, N, kFallbackSlots, &ws)) return DSA_ERR_WORKSPACE;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  CUtensorMap tq, tk;
  if (!make_indexer_maps(p, &tq, &tk)) return DSA_ERR_CUDA;
  // The array keeps the previous call's contents: clear the status word and
  // the fallback counters; every other region is rewritten before it is read.
  if (!cuda_ok(cudaMemsetAsync(ws.status, 0, kHeaderBytes, stream))) return DSA_ERR_CUDA;
  for (int t0 = 0; t0 < L; t0 += QB) {
    st = run_indexer_block(p, tq, tk, ws, t0, std::min(QB, L - t0), stream);
    if (st != DSA_OK) return st;
  }
  return DSA_OK;
}

extern "C" dsa_status_t dsa_indexer_topk_noalloc_status(dsa_stream_t stream_, unsigned *flags) {
  if (flags == nullptr) return DSA_ERR_INVALID_ARG;
  void *scratch = nullptr;
  const dsa_status_t st = noalloc_scratch(&scratch);
  if (st != DSA_OK) return st;
  cudaStream_t stream = reinterpret_cast<cudaStream_t>(stream_);
  unsigned v = 0;
  if (!cuda_ok(cudaStreamSynchronize(stream))) return DSA_ERR_CUDA;
  if (!cuda_ok(cudaMemcpy(&v, scratch, sizeof(v), cudaMemcpyDeviceToHost))) return DSA_ERR_CUDA;
  *flags = v;
  return v == 0 ? DSA_OK : DSA_ERR_INTERNAL;
}
