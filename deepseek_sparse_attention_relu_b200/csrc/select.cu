// select.cu -- exact top-k selection from the indexer's pruned candidates.
//
// LiteTopK (arXiv 2607.11976, Abstract) keeps a tight approximate threshold
// from a small sample, writes back only the candidates above it, and still
// returns the exact top-k.  The B200 version here has three steps per query
// block:
//   1. threshold_kernel: from the indexer's dense scores of a strided key
//      sample, pick the r-th best sample score as the query's threshold, with r
//      chosen so that, by the order statistics of a uniform sample, at least
//      topk visible keys lie above it with a 5-sigma margin.
//   2. select_kernel: if the query's candidate list holds at least topk keys and
//      did not overflow, it contains the exact top-k (every key scoring at
//      least the threshold was written).  A block-wide MSB-first radix select on
//      64-bit keys (order-preserving score bits << 32 | ~key index) finds the
//      k-th best; the winners are emitted in ascending key order with -1
//      padding (the int32 index-mask convention of llama.cpp PR #25917,
//      discussion).  Equal scores go to the smaller index.
//   3. the exact fallback: any query the sample misjudged (too few or too
//      many candidates) is rescored over all its visible keys by the indexer
//      kernel itself (FALLBACK mode, indexer.cu), with the same tensor-core
//      arithmetic as the main pass, and selected exactly from the dense row;
//      so neither the sample nor the query blocking can change a selection.
#include <cuda_runtime.h>

#include <cmath>

#include "dsa_internal.h"
#include "ptx.cuh"
#include "select_common.cuh"

namespace dsa {

constexpr int kSelThreads = 512;

// ------------------------------------------------------------------ threshold
constexpr int kMaxSamples = 4096;

// 1,024 queries per block and seven CTAs per SM (register and shared-memory
// budgets sized for it) make the launch a single wave on 148 SMs.
__global__ void __launch_bounds__(256, 7) threshold_kernel(SelectArgs a) {
  pdl_wait_and_release();
  __shared__ unsigned hist[256];
  __shared__ unsigned misc[4];
  __shared__ unsigned keys[kMaxSamples];  // the query's sample scores as order-preserving keys
  const int tl = blockIdx.x;
  if (threadIdx.x == 0) {
    a.cand_count[tl] = 0;
    if (tl == 0) {
      a.fb_counters[0] = 0;
      a.fb_counters[1] = 0;
    }
  }
  // Visible keys [lo, lo + nvis) and the pilot samples [i0, i0 + ns) among them.
  int lo = 0, nvis = a.q_pos0 + tl + 1, i0 = 0, ns = a.n_samples;
  if (a.key_lo != nullptr) {
    lo = a.key_lo[tl];
    nvis = a.key_hi[tl] - lo;
    const int st = max(1, a.sample_stride);
    i0 = min(a.n_samples, (lo + st - 1) / st);
    ns = min(a.n_samples, (a.key_hi[tl] + st - 1) / st) - i0;
  }
  const int need = min(a.topk, nvis);
  unsigned tau = 0u;  // key 0: every score passes
  if (a.dense != nullptr && nvis > a.cap && ns > 0) {
    const double z = 5.0;
    const double x = static_cast<double>(need) * ns / nvis;
    const double rt = z / 2.0 + sqrt(z * z / 4.0 + x);
    const double rd = ceil(rt * rt);
    if (rd < ns) {
      const int r = static_cast<int>(rd);
      const float *row = a.dense + static_cast<long long>(tl) * a.dense_ld + i0;
      for (int i = threadIdx.x; i < ns; i += blockDim.x) keys[i] = float_order_key(row[i]);
      __syncthreads();
      unsigned prefix, mask;
      block_radix_select<unsigned>([&](int i) { return keys[i]; }, ns, r, prefix, mask, hist, misc);
      tau = prefix;
    }
  }
  if (threadIdx.x == 0) a.tau[tl] = tau;
}

// Bitonic sort of n (power of two) 64-bit values in shared memory, ascending.
__device__ void block_bitonic_sort(unsigned long long *v, int n) {
  for (int k = 2; k <= n; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = threadIdx.x; i < n; i += blockDim.x) {
        const int p = i ^ j;
        if (p > i) {
          const bool up = (i & k) == 0;
          const unsigned long long x = v[i], y = v[p];
          if ((x > y) == up) {
            v[i] = y;
            v[p] = x;
          }
        }
      }
      __syncthreads();
    }
  }
}

// ------------------------------------------------------------------ select
// Shared memory of the selection kernel, sized per launch so that several of
// its CTAs share an SM: up to kSmemCand candidates are staged (a longer list is
// read from L2), then a region that holds either the bitmap over the visible
// keys (ascending output) or the sort buffer of the selected pairs.
constexpr int kSmemCand = 6144;
constexpr int kBitmapMaxKeys = 262144;  // the bitmap path covers caches up to this many keys

int select_stage_cap(const SelectArgs &a) { return min(a.cap, kSmemCand); }
int select_region_bytes(const SelectArgs &a) {
  int npow = 1;
  while (npow < a.topk) npow <<= 1;
  const int bitmap = a.N <= kBitmapMaxKeys ? (a.N + 31) / 32 * 4 : 0;
  return max(bitmap, npow * 8);
}

__global__ void __launch_bounds__(kSelThreads) select_kernel(SelectArgs a) {
  pdl_wait_and_release();
  extern __shared__ __align__(16) unsigned char sel_smem[];
  unsigned long long *cs = reinterpret_cast<unsigned long long *>(sel_smem);         // staged candidates
  const int stage_cap = min(a.cap, kSmemCand);
  unsigned char *region = sel_smem + static_cast<size_t>(stage_cap) * 8;  // bitmap or sort buffer
  __shared__ unsigned hist[256];
  __shared__ unsigned misc[4];
  __shared__ int warp_tot[kSelThreads / 32];
  __shared__ int total, nsel;
  const int tl = blockIdx.x;
  const int t = a.t0 + tl;
  const int lo = a.key_lo != nullptr ? a.key_lo[tl] : 0;  // visible keys [lo, lo + nvis)
  const int nvis = a.key_lo != nullptr ? a.key_hi[tl] - lo : a.q_pos0 + tl + 1;
  const int need = min(a.topk, nvis);
  const int count = a.cand_count[tl];
  const bool fallback = count > a.cap || count < need;
  if (threadIdx.x == 0 && a.stats != nullptr) {
    atomicAdd(&a.stats->candidates, static_cast<unsigned long long>(count));
    atomicAdd(&a.stats->queries, 1u);
    atomicMax(&a.stats->max_candidates, static_cast<unsigned>(count));
    if (fallback) atomicAdd(&a.stats->fallback_queries, 1u);
  }
  if (fallback) {
    if (threadIdx.x == 0) {
      const int pos = atomicAdd(&a.fb_counters[0], 1);
      a.fb_list[pos] = tl;
      a.fb_done[pos] = 0;
    }
    return;
  }
  const unsigned long long *cand = a.cand + static_cast<long long>(tl) * a.cap;
  const bool staged = count <= stage_cap;
  if (staged) {
    for (int i = threadIdx.x; i < count; i += blockDim.x) cs[i] = cand[i];
    __syncthreads();
  }
  auto fetch = [&](int i) { return staged ? cs[i] : cand[i]; };
  unsigned long long prefix = 0, mask = 0;
  if (count > need) block_radix_select<unsigned long long>(fetch, count, need, prefix, mask, hist, misc);
  int32_t *out = a.topk_idx + static_cast<long long>(t) * a.topk;
  float *osc = a.topk_score ? a.topk_score + static_cast<long long>(t) * a.topk : nullptr;

  // (the region holds a bitmap over [lo, lo + nvis) whenever N <= kBitmapMaxKeys, since nvis <= N)
  if (osc == nullptr && a.N <= kBitmapMaxKeys) {
    // Winners -> bitmap over key indices -> ordered compaction (ascending keys).
    unsigned *bitmap = reinterpret_cast<unsigned *>(region);
    const int nwords = (nvis + 31) >> 5;
    for (int i = threadIdx.x; i < nwords; i += blockDim.x) bitmap[i] = 0u;
    __syncthreads();
    for (int i = threadIdx.x; i < count; i += blockDim.x) {
      const unsigned long long k = fetch(i);
      if (k >= prefix) {
        const unsigned idx = ~static_cast<unsigned>(k & 0xFFFFFFFFull) - static_cast<unsigned>(lo);
        atomicOr(&bitmap[idx >> 5], 1u << (idx & 31));
      }
    }
    __syncthreads();
    const int per = (nwords + blockDim.x - 1) / blockDim.x;
    const int w0 = threadIdx.x * per, w1 = min(nwords, w0 + per);
    int mine = 0;
    for (int wd = w0; wd < w1; ++wd) mine += __popc(bitmap[wd]);
    int pos = block_exclusive_scan(mine, warp_tot, &total);
    for (int wd = w0; wd < w1; ++wd) {
      unsigned bits = bitmap[wd];
      while (bits) {
        const int b = __ffs(bits) - 1;
        bits &= bits - 1;
        if (pos < need) out[pos] = lo + wd * 32 + b;
        ++pos;
      }
    }
    if (threadIdx.x == 0 && total != need) atomicOr(a.status, DEV_OVERFLOW);
    for (int j = need + threadIdx.x; j < a.topk; j += blockDim.x) out[j] = -1;
    return;
  }

  // Scores requested (or a very long cache): bitonic sort of (index, score key) pairs.
  unsigned long long *sortbuf = reinterpret_cast<unsigned long long *>(region);
  if (threadIdx.x == 0) nsel = 0;
  int npow = 1;
  while (npow < need) npow <<= 1;
  for (int i = threadIdx.x; i < npow; i += blockDim.x) sortbuf[i] = ~0ull;
  __syncthreads();
  for (int i = threadIdx.x; i < count; i += blockDim.x) {
    const unsigned long long k = fetch(i);
    if (k >= prefix) {
      const int p = atomicAdd(&nsel, 1);
      const unsigned idx = ~static_cast<unsigned>(k & 0xFFFFFFFFull);
      if (p < npow) sortbuf[p] = (static_cast<unsigned long long>(idx) << 32) | (k >> 32);
    }
  }
  __syncthreads();
  if (nsel != need) {
    if (threadIdx.x == 0) atomicOr(a.status, DEV_OVERFLOW);
  }
  block_bitonic_sort(sortbuf, npow);
  for (int j = threadIdx.x; j < a.topk; j += blockDim.x) {
    if (j < need) {
      const unsigned long long v = sortbuf[j];
      out[j] = static_cast<int32_t>(v >> 32);
      if (osc) osc[j] = order_key_float(static_cast<unsigned>(v & 0xFFFFFFFFull));
    } else {
      out[j] = -1;
      if (osc) osc[j] = -INFINITY;
    }
  }
}

// ------------------------------------------------------------------ wait self-test
// The bounded-wait path of every kernel, exercised on purpose: one thread
// waits on an mbarrier that nothing arrives on, gives up after limit_ns and
// records DEV_TIMEOUT, exactly as a kernel whose producer stalled would.
__global__ void wait_timeout_probe_kernel(unsigned *status, unsigned long long limit_ns) {
  pdl_wait_and_release();
  __shared__ uint64_t never;
  if (threadIdx.x != 0) return;
  mbar_init(&never, 1);
  fence_mbar_init();
  if (!mbar_wait_limit(&never, 0u, nullptr, limit_ns)) atomicOr(status, DEV_TIMEOUT);
}

cudaError_t launch_wait_timeout_probe(unsigned *status, unsigned long long limit_ns, cudaStream_t stream) {
  return launch_kernel(wait_timeout_probe_kernel, dim3(1), dim3(32), 0, stream, status, limit_ns);
}

// ------------------------------------------------------------------ range plan
// Per-query key ranges: clamp each into [0, N] (a range with lo < 0, hi > N
// or lo > hi is flagged and made empty), then give every query group the
// window of 128-key tiles that covers its queries' non-empty ranges, and the
// exclusive prefix of the windows' sizes for the indexer's work split.
__global__ void __launch_bounds__(128) range_plan_kernel(RangePlanArgs a) {
  pdl_wait_and_release();
  __shared__ int cnt_s[128];
  const int G = (a.Lb + a.QG - 1) / a.QG;
  for (int t = threadIdx.x; t < a.Lb; t += blockDim.x) {
    int lo = a.lo_in[t], hi = a.hi_in[t];
    if (lo < 0 || hi > a.N || lo > hi) {
      atomicOr(a.status, DEV_BAD_INDEX);
      lo = hi = 0;
    }
    a.lo[t] = lo;
    a.hi[t] = hi;
  }
  __syncthreads();
  const int g = threadIdx.x;
  int n = 0, t0 = 0;
  if (g < G) {
    int mn = a.N, mx = 0;
    for (int t = g * a.QG; t < min(a.Lb, (g + 1) * a.QG); ++t) {
      if (a.lo[t] < a.hi[t]) {
        mn = min(mn, a.lo[t]);
        mx = max(mx, a.hi[t]);
      }
    }
    if (mx > mn) {
      t0 = mn / 128;
      n = (mx + 127) / 128 - t0;
    }
    a.grp_tile0[g] = t0;
  }
  cnt_s[threadIdx.x] = n;
  __syncthreads();
  if (threadIdx.x == 0) {
    int acc = 0;
    for (int i = 0; i < G; ++i) {
      a.grp_start[i] = acc;
      acc += cnt_s[i];
    }
    a.grp_start[G] = acc;
  }
}

cudaError_t launch_range_plan(const RangePlanArgs &a, cudaStream_t stream) {
  if ((a.Lb + a.QG - 1) / a.QG > 128) return cudaErrorInvalidValue;
  return launch_kernel(range_plan_kernel, dim3(1), dim3(128), 0, stream, a);
}

// ------------------------------------------------------------------ pack plan
// LiteDSA (arXiv 2607.11976, Abstract) packs neighbouring queries' candidate
// sets for joint computation and masks each query's scores to its own set.
// One CTA per pack of G consecutive queries: mark every selected key in a
// shared bitmap over key indices, number the marked keys in ascending order
// (per-word prefix popcounts give any key's rank in O(1)), and record for
// every 64-key tile of that union which keys each query chose.  The pack is
// packed only if the union is small enough and its rows are clean (unique,
// in-range keys); otherwise its queries are handed to the unpacked kernel.
constexpr int kPackThreads = 1024;

__global__ void __launch_bounds__(kPackThreads) pack_plan_kernel(PackArgs a) {
  pdl_wait_and_release();
  extern __shared__ unsigned pk_words[];  // bitmap [nwords], then exclusive prefix counts [nwords]
  __shared__ int warp_tot[kPackThreads / 32];
  __shared__ int total, nvalid_s, bad_s;
  __shared__ int qcount[64];
  const int nwords = (a.N + 31) >> 5;
  unsigned *bm = pk_words;
  unsigned *pre = pk_words + nwords;
  const int p = blockIdx.x;
  const int q0 = a.t0 + p * a.G;
  const int nq = min(a.G, a.t0 + a.Lq - q0);
  const int n = nq * a.topk;
  const int32_t *rows = a.topk_idx + static_cast<long long>(q0) * a.topk;
  for (int w = threadIdx.x; w < nwords; w += blockDim.x) bm[w] = 0u;
  if (threadIdx.x < 64) qcount[threadIdx.x] = 0;
  if (threadIdx.x == 0) { nvalid_s = 0; bad_s = 0; }
  __syncthreads();
  int valid = 0, bad = 0;
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    const int key = rows[e];
    if (key >= 0 && key < a.N) {
      atomicOr(&bm[key >> 5], 1u << (key & 31));
      ++valid;
    } else if (key != -1) {
      ++bad;
    }
  }
  if (valid) atomicAdd(&nvalid_s, valid);
  if (bad) atomicAdd(&bad_s, bad);
  __syncthreads();
  const int per = (nwords + blockDim.x - 1) / blockDim.x;
  const int w0 = threadIdx.x * per, w1 = min(nwords, w0 + per);
  int mine = 0;
  for (int w = w0; w < w1; ++w) mine += __popc(bm[w]);
  int base = block_exclusive_scan(mine, warp_tot, &total);
  for (int w = w0; w < w1; ++w) {
    pre[w] = base;
    base += __popc(bm[w]);
  }
  const int nu = min(total, a.umax);
  const int ntiles = (nu + 63) / 64;
  unsigned long long *qm = a.qmask + static_cast<long long>(p) * a.umax;
  for (int i = threadIdx.x; i < ntiles * 64; i += blockDim.x) qm[i] = 0ull;
  __syncthreads();
  // Union keys in ascending order, and each query's membership bits.
  int32_t *uk = a.ukeys + static_cast<long long>(p) * a.umax;
  for (int w = w0; w < w1; ++w) {
    unsigned bits = bm[w];
    int u = pre[w];
    while (bits) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1;
      if (u < a.umax) uk[u] = w * 32 + b;
      ++u;
    }
  }
  for (int e = threadIdx.x; e < n; e += blockDim.x) {
    const int key = rows[e];
    if (key < 0 || key >= a.N) continue;
    const int j = e / a.topk;
    const int u = pre[key >> 5] + __popc(bm[key >> 5] & ((1u << (key & 31)) - 1u));
    if (u < a.umax) {
      const unsigned long long bit = 1ull << (u & 63);
      const unsigned long long old = atomicOr(&qm[(u >> 6) * 64 + j], bit);
      if (!(old & bit)) atomicAdd(&qcount[j], 1);  // a repeated key of one query sets no new bit
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    int unique = 0;
    for (int j = 0; j < nq; ++j) unique += qcount[j];
    const bool clean = bad_s == 0 && unique == nvalid_s && total <= a.umax;
    const bool pack = clean && static_cast<float>(total) <= a.max_union_ratio * nvalid_s;
    a.ucount[p] = nu;
    if (pack) {
      a.plist[atomicAdd(a.pcount, 1)] = p;
    } else {
      const int b = atomicAdd(a.scount, nq);
      for (int j = 0; j < nq; ++j) a.slist[b + j] = p * a.G + j;
    }
  }
}

cudaError_t launch_pack_plan(const PackArgs &a, cudaStream_t stream) {
  const int npacks = (a.Lq + a.G - 1) / a.G;
  const int smem = ((a.N + 31) / 32) * 8;
  if (smem > 200 * 1024 || a.G > 64) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(pack_plan_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_kernel(pack_plan_kernel, dim3(npacks), dim3(kPackThreads), smem, stream, a);
}

cudaError_t launch_threshold(const SelectArgs &a, cudaStream_t stream) {
  return launch_kernel(threshold_kernel, dim3(a.Lb), dim3(256), 0, stream, a);
}

cudaError_t launch_select(const SelectArgs &a, cudaStream_t stream) {
  const int smem = select_stage_cap(a) * 8 + select_region_bytes(a);
  cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  return launch_kernel(select_kernel, dim3(a.Lb), dim3(kSelThreads), smem, stream, a);
}


}  // namespace dsa
