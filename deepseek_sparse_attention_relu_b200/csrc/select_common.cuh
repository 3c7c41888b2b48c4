// select_common.cuh -- block-wide selection helpers shared by the selection
// kernels (select.cu) and the exact fallback pass of the indexer kernel
// (indexer.cu): an MSB-first radix select on order-preserving keys, a block
// prefix sum, and the exact top-k of one dense score row.
#pragma once
#include <cstdint>

#include "ptx.cuh"

namespace dsa {

// Block-wide MSB-first radix select.  Among n unique keys (fetch(i), i < n) find
// (prefix, mask) such that exactly `need` keys satisfy (key & mask) >= prefix,
// i.e. key >= prefix.  1 <= need <= n.  Every thread of the block must call it.
// UNROLL > 1 keeps that many keys per thread in flight in the histogram passes
// (for keys read from global memory).
template <typename KeyT, int UNROLL = 1, typename Fetch>
__device__ void block_radix_select(Fetch fetch, int n, int need, KeyT &prefix_out, KeyT &mask_out,
                                   unsigned *hist, unsigned *misc) {
  constexpr int BITS = sizeof(KeyT) * 8;
  KeyT prefix = 0, mask = 0;
  unsigned remaining = static_cast<unsigned>(need);
  for (int shift = BITS - 8; shift >= 0; shift -= 8) {
    for (int b = threadIdx.x; b < 256; b += blockDim.x) hist[b] = 0;
    __syncthreads();
    const int bd = static_cast<int>(blockDim.x);
    int i = threadIdx.x;
    if constexpr (UNROLL > 1) {
      for (; i + (UNROLL - 1) * bd < n; i += UNROLL * bd) {
        KeyT kk[UNROLL];
#pragma unroll
        for (int u = 0; u < UNROLL; ++u) kk[u] = fetch(i + u * bd);
#pragma unroll
        for (int u = 0; u < UNROLL; ++u)
          if ((kk[u] & mask) == prefix) atomicAdd(&hist[static_cast<unsigned>(kk[u] >> shift) & 255u], 1u);
      }
    }
    for (; i < n; i += bd) {
      const KeyT k = fetch(i);
      if ((k & mask) == prefix) atomicAdd(&hist[static_cast<unsigned>(k >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (threadIdx.x < 32) {
      const int lane = threadIdx.x;
      unsigned local = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) local += hist[255 - 8 * lane - j];
      unsigned incl = local;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const unsigned o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      const unsigned excl = incl - local;
      if (excl < remaining && remaining <= incl) {
        unsigned c = excl;
        for (int j = 0; j < 8; ++j) {
          const int bin = 255 - 8 * lane - j;
          if (c + hist[bin] >= remaining) {
            misc[0] = static_cast<unsigned>(bin);
            misc[1] = remaining - c;
            misc[2] = hist[bin];
            break;
          }
          c += hist[bin];
        }
      }
    }
    __syncthreads();
    const unsigned chosen = misc[0];
    remaining = misc[1];
    const unsigned cnt = misc[2];
    prefix |= static_cast<KeyT>(chosen) << shift;
    mask |= static_cast<KeyT>(0xFF) << shift;
    __syncthreads();
    if (cnt == remaining) break;
  }
  prefix_out = prefix;
  mask_out = mask;
}

// Exclusive prefix sum of one int per thread over the block (blockDim.x <= 1024).
__device__ __forceinline__ int block_exclusive_scan(int v, int *warp_tot, int *total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = (blockDim.x + 31) >> 5;
  int incl = v;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) warp_tot[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int t = lane < nwarps ? warp_tot[lane] : 0;
    int ti = t;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xffffffffu, ti, off);
      if (lane >= off) ti += o;
    }
    if (lane < nwarps) warp_tot[lane] = ti - t;
    if (lane == 31) *total = ti;
  }
  __syncthreads();
  return warp_tot[warp] + incl - v;
}

// Shared-memory scratch of select_dense_row (any block size up to 1,024 threads).
struct DenseSelectSmem {
  unsigned hist[256];
  unsigned misc[4];
  int warp_tot[32];
  int total;
};

// Exact top-k of one query from its dense score row: scores[j] is the score of
// key lo + j, j < nvis.  The `need` best under (score desc, key asc) are
// written to out[0 .. need) in ascending key order (with their scores to osc
// when it is not null), then -1 (and -inf) up to topk.  Every thread of the
// block must call it; a count that does not come out at `need` sets
// DEV_OVERFLOW.  The row is read from L2 (other CTAs may have written parts
// of it), with coalesced loads and eight keys per thread in flight.  When the
// caller lends `bitmap_words` words of idle shared memory that cover the row,
// the winners are marked in a bitmap and compacted warp by warp in key order;
// otherwise each thread compacts a contiguous run of keys.
__device__ __forceinline__ void select_dense_row(const float *scores, int lo, int nvis, int need, int topk,
                                                 int32_t *out, float *osc, unsigned *status, DenseSelectSmem *sm,
                                                 unsigned *bitmap = nullptr, int bitmap_words = 0) {
  auto key_of = [&](int j) {
    return (static_cast<unsigned long long>(float_order_key(__ldcg(scores + j))) << 32) |
           static_cast<unsigned>(~static_cast<unsigned>(lo + j));
  };
  unsigned long long prefix = 0, mask = 0;
  if (nvis > need) block_radix_select<unsigned long long, 8>(key_of, nvis, need, prefix, mask, sm->hist, sm->misc);
  const int nwords = (nvis + 31) >> 5;
  if (bitmap != nullptr && nwords <= bitmap_words) {
    const int bd = static_cast<int>(blockDim.x), tid = static_cast<int>(threadIdx.x);
    for (int wd = tid; wd < nwords; wd += bd) bitmap[wd] = 0u;
    __syncthreads();
    int j = tid;
    for (; j + 7 * bd < nvis; j += 8 * bd) {
      unsigned long long kk[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) kk[u] = key_of(j + u * bd);
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int jj = j + u * bd;
        if (kk[u] >= prefix) atomicOr(&bitmap[jj >> 5], 1u << (jj & 31));
      }
    }
    for (; j < nvis; j += bd)
      if (key_of(j) >= prefix) atomicOr(&bitmap[j >> 5], 1u << (j & 31));
    __syncthreads();
    // Each warp compacts a contiguous run of words, 32 at a time (lane l takes
    // word w0 + l): its base from a block scan of the warp totals, each word's
    // offset from a warp scan.
    const int lane = tid & 31, warp = tid >> 5, nw = bd >> 5;
    const int chunk = (nwords + nw - 1) / nw;
    const int cw0 = min(nwords, warp * chunk), cw1 = min(nwords, cw0 + chunk);
    int wcount = 0;
    for (int wd = cw0 + lane; wd < cw1; wd += 32) wcount += __popc(bitmap[wd]);
#pragma unroll
    for (int off = 16; off >= 1; off >>= 1) wcount += __shfl_xor_sync(0xffffffffu, wcount, off);
    int base = block_exclusive_scan(lane == 0 ? wcount : 0, sm->warp_tot, &sm->total);
    base = __shfl_sync(0xffffffffu, base, 0);
    for (int w0 = cw0; w0 < cw1; w0 += 32) {
      const int wd = w0 + lane;
      unsigned bits = wd < cw1 ? bitmap[wd] : 0u;
      const int c = __popc(bits);
      int incl = c;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int o = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += o;
      }
      int pos = base + incl - c;
      while (bits) {
        const int b = __ffs(bits) - 1;
        bits &= bits - 1;
        if (pos < need) {
          out[pos] = lo + wd * 32 + b;
          if (osc) osc[pos] = __ldcg(scores + wd * 32 + b);
        }
        ++pos;
      }
      base += __shfl_sync(0xffffffffu, incl, 31);
    }
  } else {
    // Ordered compaction: each thread takes a contiguous run of keys, so the
    // block prefix sum of the per-thread counts gives every winner its slot.
    const int per = (nvis + blockDim.x - 1) / blockDim.x;
    const int j0 = threadIdx.x * per, j1 = min(nvis, j0 + per);
    int mine = 0;
#pragma unroll 4
    for (int j = j0; j < j1; ++j) mine += key_of(j) >= prefix ? 1 : 0;
    int pos = block_exclusive_scan(mine, sm->warp_tot, &sm->total);
    for (int j = j0; j < j1; ++j) {
      if (key_of(j) >= prefix) {
        if (pos < need) {
          out[pos] = lo + j;
          if (osc) osc[pos] = __ldcg(scores + j);
        }
        ++pos;
      }
    }
  }
  if (threadIdx.x == 0 && sm->total != need) atomicOr(status, DEV_OVERFLOW);
  for (int j = need + threadIdx.x; j < topk; j += blockDim.x) {
    out[j] = -1;
    if (osc) osc[j] = -INFINITY;
  }
}

}  // namespace dsa
