// indexer.cu -- lightning-indexer scoring on the 5th-generation tensor cores.
//
// For one block of queries the kernel computes, for every (query t, visible
// key s) pair,
//     I[t,s] = sum_h w[t,h] * max(0, q_idx[t,h,:] . k_idx[s,:])
// (the DeepSeek Sparse Attention lightning indexer: 32 ReLU-gated, weighted
// heads over one shared indexer key per position; mlx-lm PR #1997 "GLM prefill
// now attends only to the keys its indexer picks", section "How it works"),
// and never writes the L x N score matrix: the ReLU / head-weight reduction is
// fused into the accumulator epilogue and each score is either
//   * PILOT mode: written densely for a strided sample of the keys (the small
//     sample that LiteTopK, arXiv 2607.11976 Abstract, uses to estimate each
//     query's score range), or
//   * EMIT mode: compared with the query's threshold and, when it passes,
//     appended to that query's candidate list, so that only keys able to
//     reach the top-k are stored (LiteTopK Abstract).
//
// Tile shape (swap-AB): A = 128 keys x D_I (UMMA M = 128), B = a group of
// 256 / H_I queries x H_I heads = 256 rows x D_I (UMMA N = 256), K = D_I.
// Each TMEM lane then holds one key.  Warp roles: warp 0 TMA producer, warp 1
// MMA issuer and TMEM owner, warps 2..17 epilogue (four per TMEM lane quarter,
// each taking 64 of the 256 accumulator columns).  The accumulator is
// double-buffered (2 x 256 columns) so the epilogue of tile i overlaps the MMA
// of tile i+1.  With H_I a multiple of 8 the epilogue reads the accumulator in
// 16-lane x 256-bit pieces: a thread then sees four keys but only a quarter of
// the heads, so its head weights (16 values) stay in registers for the whole
// query group instead of being re-read from shared memory every tile (per-lane
// shared loads of the weights had kept the load/store unit's register
// write-back busy 60% of the time), and four partial sums per score are added
// across the thread quad with two shuffles.
#include <cuda_runtime.h>

#include "dsa_internal.h"
#include "ptx.cuh"
#include "select_common.cuh"

namespace dsa {

template <int DI, int HI, bool FP8>
struct IdxCfg {
  static constexpr int ESZ = FP8 ? 1 : 2;
  static constexpr int ROW_BYTES = DI * ESZ;
  static constexpr int ATOMS = ROW_BYTES / 128;  // 128-byte swizzle atoms along K
  static constexpr int ATOM_ELEMS = 128 / ESZ;
  static constexpr int KSTEP = FP8 ? 32 : 16;  // K of one tcgen05.mma
  static constexpr int KSTEPS_PER_ATOM = ATOM_ELEMS / KSTEP;
  static constexpr int BM = 128;  // keys per tile
  static constexpr int BN = 256;  // query-head rows per group
  static constexpr int QG = BN / HI;
  static constexpr int K_TILE = BM * ROW_BYTES;
  static constexpr int Q_TILE = BN * ROW_BYTES;
  static constexpr int EPI_WARPS = 16;                   // four per TMEM lane quarter
  static constexpr int THREADS = 64 + EPI_WARPS * 32;
  static constexpr int COLS = BN / 4;                     // accumulator columns per epilogue warp
  static constexpr int QH = QG / 4;                       // queries per epilogue warp
  static constexpr int SB = (128 / QH) < 32 ? 32 : (128 / QH);  // staged candidates per (warp, query)
  static constexpr int STG_BYTES = EPI_WARPS * QH * SB * 8;
  static constexpr int SMEM_BUDGET = 224 * 1024;
  static constexpr int FIXED = Q_TILE + STG_BYTES + 2 * EPI_WARPS * COLS * 4 + 2048;
  static constexpr int STAGES_FIT = (SMEM_BUDGET - FIXED) / K_TILE;
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  // shared memory carve-up (offsets from a 1024-aligned base)
  static constexpr int OFF_Q = 0;
  static constexpr int OFF_K = OFF_Q + Q_TILE;
  static constexpr int OFF_STG = OFF_K + STAGES * K_TILE;        // [EPI_WARPS][QH][SB] candidate keys
  static constexpr int OFF_W = OFF_STG + STG_BYTES;               // [EPI_WARPS][COLS] floats
  static constexpr int OFF_TAU = OFF_W + EPI_WARPS * COLS * 4;    // [EPI_WARPS][QH] float thresholds
  static constexpr int OFF_BAR = OFF_TAU + EPI_WARPS * COLS * 4;  // mbarriers
  static constexpr int NBAR = 2 * STAGES + 2 + 4 + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;     // tmem addr, abort flag, counters
  static constexpr int SMEM_BYTES = OFF_MISC + 64 + 1024;  // + alignment slack
  static_assert(STAGES >= 3, "not enough shared memory for the key pipeline");
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(ROW_BYTES % 128 == 0, "indexer rows must be whole 128-byte atoms");
  static_assert(HI % 4 == 0, "head weights are read four at a time");
  static_assert(QG * HI == BN, "H_I must divide 256");
  static_assert(QH * HI == COLS && COLS % 32 == 0, "each epilogue warp covers whole queries");
};

union F2U {
  float2 f;
  unsigned long long u;
};

// Two independent fp32 FMAs in one instruction: {a.x*b.x + c.x, a.y*b.y + c.y}, round to nearest.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  F2U x, y, z, r;
  x.f = a;
  y.f = b;
  z.f = c;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r.u) : "l"(x.u), "l"(y.u), "l"(z.u));
  return r.f;
}

__device__ __forceinline__ float2 relu2(uint32_t a, uint32_t b) {
  return make_float2(fmaxf(__uint_as_float(a), 0.0f), fmaxf(__uint_as_float(b), 0.0f));
}

// Threshold key -> float: a score s passes iff s >= threshold_float(key).  Key 0
// (and anything at or below the key of -inf) passes every finite score.
__device__ __forceinline__ float threshold_float(unsigned key) {
  return key < 0x00800000u ? -INFINITY : order_key_float(key);
}

// Per-group number of 128-key tiles.  RANGES: per-query key ranges (the
// planned windows); otherwise the causal prefix (or, in PILOT mode, all samples).
template <bool RANGES>
__device__ __forceinline__ int idx_group_tiles(const IndexerArgs &a, int g, int QG) {
  if (RANGES) return a.grp_start[g + 1] - a.grp_start[g];
  int keys;
  if (a.pilot) {
    keys = a.n_keys;
  } else {
    int last = min(a.Lb, (g + 1) * QG);  // queries [g*QG, last) ; positions up to q_pos0 + last - 1
    keys = min(a.n_keys, a.q_pos0 + last);
  }
  return (keys + 127) / 128;
}

// First 128-key tile of group g (per-query ranges only; 0 otherwise).
template <bool RANGES>
__device__ __forceinline__ int idx_group_tile0(const IndexerArgs &a, int g) {
  return RANGES ? a.grp_tile0[g] : 0;
}

// Tile range of this CTA in the linearised (group, key tile) space.  `key0`
// is the first key of the current tile.
struct TileCursor {
  int g, tile, ntiles_g, left, tile0;
  __device__ __forceinline__ int key0() const { return (tile0 + tile) * 128; }
};

template <bool RANGES>
__device__ __forceinline__ TileCursor idx_cursor_begin(const IndexerArgs &a, int QG) {
  const int G = (a.Lb + QG - 1) / QG;
  const long long T = RANGES ? a.grp_start[G] : a.total_tiles;
  const long long u0 = T * blockIdx.x / gridDim.x;
  const long long u1 = T * (blockIdx.x + 1) / gridDim.x;
  TileCursor c;
  c.left = static_cast<int>(u1 - u0);
  c.g = 0;
  c.tile = 0;
  c.ntiles_g = 0;
  c.tile0 = 0;
  if (c.left <= 0) {
    c.left = 0;
    return c;
  }
  // u0 < T, so the walk stops at a group that has tiles (empty groups are passed over).
  long long acc = 0;
  int g = 0;
  int nt = idx_group_tiles<RANGES>(a, 0, QG);
  while (acc + nt <= u0) {
    acc += nt;
    ++g;
    nt = idx_group_tiles<RANGES>(a, g, QG);
  }
  c.g = g;
  c.tile = static_cast<int>(u0 - acc);
  c.ntiles_g = nt;
  c.tile0 = idx_group_tile0<RANGES>(a, g);
  return c;
}

template <bool RANGES>
__device__ __forceinline__ void idx_cursor_next(TileCursor &c, const IndexerArgs &a, int QG) {
  --c.left;
  if (++c.tile == c.ntiles_g) {
    c.tile = 0;
    if (c.left <= 0) return;  // nothing follows; do not look past the last group
    // tiles remain, so a later group has some
    do {
      ++c.g;
      c.ntiles_g = idx_group_tiles<RANGES>(a, c.g, QG);
    } while (c.ntiles_g == 0);
    c.tile0 = idx_group_tile0<RANGES>(a, c.g);
  }
}

// Tiles of one fallback job: every 128-key tile holding a visible key of query
// tl (its clamped range, or its causal prefix), within the query's group.  The
// tiles sit at the same 128-key boundaries, and the query at the same column
// of the same group tile, as in the main pass, so its scores come out
// bit-identical to the main pass's.
template <bool RANGES>
__device__ __forceinline__ TileCursor idx_cursor_job(const IndexerArgs &a, int tl, int QG, int &lo, int &hi) {
  lo = RANGES ? a.key_lo[tl] : 0;
  hi = RANGES ? a.key_hi[tl] : min(a.n_keys, a.q_pos0 + tl + 1);
  TileCursor c;
  c.g = tl / QG;
  c.tile = 0;
  c.tile0 = lo / 128;
  c.ntiles_g = hi > lo ? (hi - 1) / 128 - lo / 128 + 1 : 0;
  c.left = c.ntiles_g;
  return c;
}

template <int DI, int HI, bool FP8, int MODE, bool RANGES>
__global__ void __launch_bounds__(IdxCfg<DI, HI, FP8>::THREADS, 1)
    indexer_kernel(const __grid_constant__ CUtensorMap tmap_q, const __grid_constant__ CUtensorMap tmap_k,
                   IndexerArgs a) {
  pdl_wait_and_release();
  using C = IdxCfg<DI, HI, FP8>;
  constexpr bool PILOT = MODE == kIdxPilot;
  constexpr bool FB = MODE == kIdxFallback;
  // No query to rescore (the usual case): leave before any set-up.  The count
  // was written by the selection kernel, which has completed.
  if (FB && *reinterpret_cast<volatile int *>(&a.fb_counters[0]) == 0) return;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *q_s = smem + C::OFF_Q;
  uint8_t *k_s = smem + C::OFF_K;
  float *w_s = reinterpret_cast<float *>(smem + C::OFF_W);
  float *tau_s = reinterpret_cast<float *>(smem + C::OFF_TAU);
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
  uint64_t *full = bars;                    // [STAGES] TMA -> MMA
  uint64_t *empty = bars + C::STAGES;       // [STAGES] MMA -> TMA
  uint64_t *q_full = bars + 2 * C::STAGES;  // query tile landed
  uint64_t *q_empty = q_full + 1;           // MMA done with the query tile
  uint64_t *acc_full = q_full + 2;          // [2] MMA -> epilogue
  uint64_t *acc_empty = q_full + 4;         // [2] epilogue -> MMA
  uint64_t *drain = q_full + 6;             // MMA drain on abort
  unsigned *tmem_slot = reinterpret_cast<unsigned *>(smem + C::OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 8);
  volatile int *job_s = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 12);  // FALLBACK: current query
  // FALLBACK: [0] score row, [1] chunk, [2] chunks per query, [3] position in fb_list, [4] select flag
  volatile int *job_meta = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 16);

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int i = 0; i < C::STAGES; ++i) {
      mbar_init(&full[i], 1);
      mbar_init(&empty[i], 1);
    }
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], C::EPI_WARPS);
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tensormap(&tmap_q);
    prefetch_tensormap(&tmap_k);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const unsigned tmem_base = *tmem_slot;

  // ---- role state; it carries over from one fallback job to the next (the
  // other modes make a single pass over the CTA's share of the tiles).
  // TMA producer (warp 0, lane 0)
  int p_stage = 0, p_issued = 0, p_q_issued = 0;
  unsigned p_phase = 0, p_qphase = 0;
  bool p_ok = true;
  // MMA issuer (warp 1)
  int m_stage = 0, m_acc = 0;
  unsigned m_phase = 0, m_acc_phase = 0, m_qphase = 0;
  bool m_ok = true;
  // epilogue (warps 2..17)
  const int ew = warp - 2;          // 0..15
  const int quarter = warp & 3;     // TMEM lane quarter this warp may access
  const int slot = ew >> 2;         // which 64 accumulator columns
  constexpr int QH = C::QH;         // queries per warp
  constexpr int SB = C::SB;
  int e_acc = 0, e_prev_g = -1;
  unsigned e_acc_phase = 0;
  bool e_ok = true;
  const unsigned lane_mask_lt = (1u << lane) - 1u;
  float *w_w = w_s + ew * C::COLS;   // this warp's head weights: [QH queries][HI]
  float *tau_w = tau_s + ew * C::COLS;
  int *lo_w = reinterpret_cast<int *>(tau_w + QH);      // per-query key ranges (ranges mode)
  int *hi_w = reinterpret_cast<int *>(tau_w + 2 * QH);
  static_assert(3 * C::QH <= C::COLS, "thresholds and ranges share the per-warp slot");
  unsigned long long *stg = reinterpret_cast<unsigned long long *>(smem + C::OFF_STG) + ew * QH * SB;
  int cnt[QH];                   // staged candidates per query (warp-uniform)
  // Indexer heads in whole 8-column blocks: 16-lane accumulator loads with the
  // warp's head weights held in registers for the whole query group.
  constexpr bool QUAD = (HI % 8) == 0;
  const int c4 = lane & 3, r4 = lane >> 2;
  float2 wreg[QH][HI / 8 > 0 ? HI / 8 : 1];
#pragma unroll
  for (int qq = 0; qq < QH; ++qq) cnt[qq] = 0;

  // Move a query's staged candidates to its global list: one atomic per batch.
  auto flush = [&](int qq, int gq) {
    const int n = cnt[qq];
    if (n == 0) return;
    const int tl = gq * C::QG + slot * QH + qq;
    __syncwarp();
    int base = 0;
    if (lane == 0) base = atomicAdd(&a.cand_count[tl], n);
    base = __shfl_sync(0xffffffffu, base, 0);
    for (int i = lane; i < n; i += 32) {
      const int pos = base + i;
      if (pos < a.cap) a.cand[static_cast<long long>(tl) * a.cap + pos] = stg[qq * SB + i];
    }
    __syncwarp();
    cnt[qq] = 0;
  };

  for (int round = 0;; ++round) {
    // ---- the tiles of this round: the CTA's share of the block (one round),
    // or one fallback query at a time.
    TileCursor c;
    int job_tl = -1, job_lo = 0, job_hi = 0, job_row = 0, job_cpq = 1, job_pos = 0;
    if constexpr (FB) {
      if (threadIdx.x == 0) {
        int j = -1;
        if (!*abort_flag) {
          // Fewer queries than CTAs: each query's tiles are split into
          // gridDim.x / count chunks (one job each) so that all CTAs work.
          const int nfb = *reinterpret_cast<volatile int *>(&a.fb_counters[0]);  // >= 1 here
          const int cpq = nfb < static_cast<int>(gridDim.x) ? static_cast<int>(gridDim.x) / nfb : 1;
          const int n = atomicAdd(&a.fb_counters[1], 1);
          if (n < nfb * cpq) {
            const int pos = n / cpq;
            j = a.fb_list[pos];
            job_meta[0] = cpq > 1 ? pos : static_cast<int>(blockIdx.x);
            job_meta[1] = n - pos * cpq;
            job_meta[2] = cpq;
            job_meta[3] = pos;
          }
        }
        *job_s = j;
      }
      __syncthreads();
      job_tl = *job_s;
      if (job_tl < 0) break;
      job_row = job_meta[0];
      job_cpq = job_meta[2];
      job_pos = job_meta[3];
      c = idx_cursor_job<RANGES>(a, job_tl, C::QG, job_lo, job_hi);
      if (job_cpq > 1) {  // this job's share of the query's tiles
        const int per = (c.ntiles_g + job_cpq - 1) / job_cpq;
        const int first = min(c.ntiles_g, job_meta[1] * per);
        const int len = min(per, c.ntiles_g - first);
        c.tile0 += first;
        c.ntiles_g = len;
        c.left = len;
      }
      e_prev_g = -1;  // every job loads its group's weights afresh
    } else {
      if (round > 0) break;
      c = idx_cursor_begin<RANGES>(a, C::QG);
    }

    if (warp == 0) {
      // ---------------------------------------------------------- TMA producer
      if (lane == 0 && p_ok) {
        int prev_g = -1;
        while (c.left > 0) {
          if (c.g != prev_g) {
            if (p_q_issued > 0) {
              if (!mbar_wait(q_empty, p_qphase, abort_flag)) { p_ok = false; break; }
              p_qphase ^= 1u;
            }
            mbar_arrive_expect_tx(q_full, C::Q_TILE);
            for (int at = 0; at < C::ATOMS; ++at)
              tma_load_2d(q_s + at * C::BN * 128, &tmap_q, q_full, at * C::ATOM_ELEMS, a.q_row0 + c.g * C::BN);
            ++p_q_issued;
            prev_g = c.g;
          }
          if (!mbar_wait(&empty[p_stage], p_phase ^ 1u, abort_flag)) { p_ok = false; break; }
          mbar_arrive_expect_tx(&full[p_stage], C::K_TILE);
          for (int at = 0; at < C::ATOMS; ++at)
            tma_load_2d(k_s + p_stage * C::K_TILE + at * C::BM * 128, &tmap_k, &full[p_stage], at * C::ATOM_ELEMS,
                        c.key0());
          ++p_issued;
          if (++p_stage == C::STAGES) { p_stage = 0; p_phase ^= 1u; }
          idx_cursor_next<RANGES>(c, a, C::QG);
        }
        if (!p_ok) {
          atomicOr(a.status, DEV_TIMEOUT);
          *abort_flag = 1;
        }
      }
    } else if (warp == 1) {
      // ---------------------------------------------------------- MMA issuer
      constexpr unsigned idesc = make_idesc(C::BM, C::BN, FP8 ? 0u : 1u, 0u, 0u);
      int prev_g = -1;
      while (m_ok && c.left > 0) {
        const int g = c.g;
        if (g != prev_g) {
          if (!mbar_wait(q_full, m_qphase, abort_flag)) { m_ok = false; break; }
          m_qphase ^= 1u;
          prev_g = g;
        }
        if (!mbar_wait(&full[m_stage], m_phase, abort_flag)) { m_ok = false; break; }
        if (!mbar_wait(&acc_empty[m_acc], m_acc_phase ^ 1u, abort_flag)) { m_ok = false; break; }
        tc_fence_after();
        TileCursor nx = c;
        idx_cursor_next<RANGES>(nx, a, C::QG);
        const bool last_of_group = (nx.left == 0) || (nx.g != g);
        if (lane == 0) {
          const unsigned d_tmem = tmem_base + m_acc * 256;
          const uint64_t a0 = smem_desc_sw128(smem_u32(k_s + m_stage * C::K_TILE), 16, 1024);
          const uint64_t b0 = smem_desc_sw128(smem_u32(q_s), 16, 1024);
#pragma unroll
          for (int at = 0; at < C::ATOMS; ++at) {
#pragma unroll
            for (int ks = 0; ks < C::KSTEPS_PER_ATOM; ++ks) {
              // offsets go into the start-address field (address >> 4), which cannot carry
              const uint64_t ad = a0 + static_cast<uint64_t>((at * C::BM * 128 + ks * 32) >> 4);
              const uint64_t bd = b0 + static_cast<uint64_t>((at * C::BN * 128 + ks * 32) >> 4);
              const unsigned accum = (at | ks) ? 1u : 0u;
              if (FP8)
                mma_fp8_ss(d_tmem, ad, bd, idesc, accum);
              else
                mma_bf16_ss(d_tmem, ad, bd, idesc, accum);
            }
          }
          tc_commit(&empty[m_stage]);
          tc_commit(&acc_full[m_acc]);
          if (last_of_group) tc_commit(q_empty);
        }
        __syncwarp();
        if (++m_stage == C::STAGES) { m_stage = 0; m_phase ^= 1u; }
        if (++m_acc == 2) { m_acc = 0; m_acc_phase ^= 1u; }
        c = nx;
      }
      if (!m_ok && lane == 0) {
        atomicOr(a.status, DEV_TIMEOUT);
        *abort_flag = 1;
      }
    } else {
      // ---------------------------------------------------------- epilogue
      while (e_ok && c.left > 0) {
        const int g = c.g;
        if (g != e_prev_g) {
          if (!PILOT && !FB && e_prev_g >= 0) {
#pragma unroll
            for (int qq = 0; qq < QH; ++qq) flush(qq, e_prev_g);
          }
          // Each warp stages the head weights / thresholds of its own queries
          // (no cross-warp barrier, so an aborting warp cannot strand the others).
          __syncwarp();
          if constexpr (QUAD) {
#pragma unroll
            for (int qq = 0; qq < QH; ++qq) {
              const int tl = g * C::QG + slot * QH + qq;
#pragma unroll
              for (int hp = 0; hp < HI / 8; ++hp) {
                const long long o = static_cast<long long>(tl) * HI + 8 * hp + 2 * c4;
                wreg[qq][hp] = (tl < a.Lb) ? make_float2(a.w[o], a.w[o + 1]) : make_float2(0.0f, 0.0f);
              }
            }
          } else {
            for (int j = lane; j < C::COLS; j += 32) {
              const int tl = g * C::QG + slot * QH + j / HI;
              w_w[j] = (tl < a.Lb) ? a.w[static_cast<long long>(g * C::QG + slot * QH) * HI + j] : 0.0f;
            }
          }
          if (!PILOT && !FB) {
            for (int j = lane; j < QH; j += 32) {
              const int tl = g * C::QG + slot * QH + j;
              tau_w[j] = (tl < a.Lb) ? threshold_float(a.tau[tl]) : INFINITY;
              if (RANGES) {
                lo_w[j] = (tl < a.Lb) ? a.key_lo[tl] : 0;
                hi_w[j] = (tl < a.Lb) ? a.key_hi[tl] : 0;
              }
            }
          }
          __syncwarp();
          e_prev_g = g;
        }
        if (!mbar_wait(&acc_full[e_acc], e_acc_phase, abort_flag)) { e_ok = false; break; }
        tc_fence_after();
        const unsigned taddr =
            tmem_base + (static_cast<unsigned>(quarter * 32) << 16) + e_acc * 256 + slot * C::COLS;
        // Score of (query qq of this warp, key): dense write (pilot), the
        // fallback query's dense row, or threshold test and staging (main
        // pass).  Called by all 32 lanes together.
        auto emit = [&](int qq, int key, float score) {
          const int tl = g * C::QG + slot * QH + qq;  // query within the block
          if (PILOT) {
            if (tl < a.Lb && key < a.n_keys) a.dense[static_cast<long long>(tl) * a.dense_ld + key] = score;
          } else if (FB) {
            if (tl == job_tl && key >= job_lo && key < job_hi)
              a.dense[static_cast<long long>(job_row) * a.dense_ld + (key - job_lo)] = score;
          } else {
            const bool vis = RANGES ? (key >= lo_w[qq] && key < hi_w[qq]) : (key <= a.q_pos0 + tl);
            const bool pass = (tl < a.Lb) && vis && (score >= tau_w[qq]);
            const unsigned m = __ballot_sync(0xffffffffu, pass);
            if (m) {
              const int n = __popc(m);
              if (cnt[qq] + n > SB) flush(qq, g);
              if (pass) {
                const unsigned long long k64 = (static_cast<unsigned long long>(float_order_key(score)) << 32) |
                                               static_cast<unsigned>(~static_cast<unsigned>(key));
                stg[qq * SB + cnt[qq] + __popc(m & lane_mask_lt)] = k64;
              }
              cnt[qq] += n;
            }
          }
        };
        if constexpr (QUAD) {
          // 16-lane loads: this thread sees keys r4, r4 + 8, r4 + 16, r4 + 24 of the
          // warp's 32 and, in every 8-column block, the two heads 2*c4, 2*c4 + 1.
          // Its partial sums over those heads are added across the four threads
          // of its quad; the thread ends with key r4 + 8*c4 for every query.
          const int key = c.key0() + quarter * 32 + r4 + 8 * c4;
          constexpr int NQ = 32 / HI;  // queries per 32-column chunk
#pragma unroll
          for (int ch = 0; ch < C::COLS / 32; ++ch) {
            uint32_t va[16], vb[16];
            tmem_ld_16x256b_x4(taddr + ch * 32, va);
            tmem_ld_16x256b_x4(taddr + (16u << 16) + ch * 32, vb);
            tmem_ld_wait();
            if (ch == C::COLS / 32 - 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&acc_empty[e_acc]);
            }
            float2 pa[NQ][4];
#pragma unroll
            for (int qc = 0; qc < NQ; ++qc)
#pragma unroll
              for (int kk = 0; kk < 4; ++kk) pa[qc][kk] = make_float2(0.0f, 0.0f);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int qc = (8 * j) / HI;
              const float2 wv = wreg[ch * NQ + qc][((8 * j) % HI) / 8];
              pa[qc][0] = ffma2(wv, relu2(va[4 * j], va[4 * j + 1]), pa[qc][0]);
              pa[qc][1] = ffma2(wv, relu2(va[4 * j + 2], va[4 * j + 3]), pa[qc][1]);
              pa[qc][2] = ffma2(wv, relu2(vb[4 * j], vb[4 * j + 1]), pa[qc][2]);
              pa[qc][3] = ffma2(wv, relu2(vb[4 * j + 2], vb[4 * j + 3]), pa[qc][3]);
            }
#pragma unroll
            for (int qc = 0; qc < NQ; ++qc) {
              // Reduce-scatter over the quad: lane bit 1 picks keys {0,1} or {2,3},
              // lane bit 0 one of the pair.  Every thread adds the same four
              // partials in the same tree, ((p0 + p2) + (p1 + p3)).
              const float v0 = pa[qc][0].x + pa[qc][0].y, v1 = pa[qc][1].x + pa[qc][1].y;
              const float v2 = pa[qc][2].x + pa[qc][2].y, v3 = pa[qc][3].x + pa[qc][3].y;
              const bool b1 = (c4 & 2) != 0, b0 = (c4 & 1) != 0;
              float k0 = b1 ? v2 : v0, k1 = b1 ? v3 : v1;
              k0 += __shfl_xor_sync(0xffffffffu, b1 ? v0 : v2, 2);
              k1 += __shfl_xor_sync(0xffffffffu, b1 ? v1 : v3, 2);
              float score = b0 ? k1 : k0;
              score += __shfl_xor_sync(0xffffffffu, b0 ? k0 : k1, 1);
              emit(ch * NQ + qc, key, score);
            }
          }
        } else {
          const int key = c.key0() + quarter * 32 + lane;
          // One 32-column chunk of the accumulator at a time (keeps the live
          // register set small); the buffer goes back to the MMA warp after the
          // last chunk has been read.
#pragma unroll
          for (int ch = 0; ch < C::COLS / 32; ++ch) {
            uint32_t vc[32];
            tmem_ld_32x32b_x32(taddr + ch * 32, vc);
            tmem_ld_wait();
            if (ch == C::COLS / 32 - 1) {
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&acc_empty[e_acc]);
            }
#pragma unroll
            for (int qq = ch * 32 / HI; qq < (ch + 1) * 32 / HI; ++qq) {
              const float4 *wq = reinterpret_cast<const float4 *>(w_w + qq * HI);
              float2 acc0 = make_float2(0.0f, 0.0f), acc1 = make_float2(0.0f, 0.0f);
#pragma unroll
              for (int h4 = 0; h4 < HI / 4; ++h4) {
                const float4 w4 = wq[h4];
                const int col = qq * HI + 4 * h4;
                const float r0 = fmaxf(__uint_as_float(vc[(col + 0) % 32]), 0.0f);
                const float r1 = fmaxf(__uint_as_float(vc[(col + 1) % 32]), 0.0f);
                const float r2 = fmaxf(__uint_as_float(vc[(col + 2) % 32]), 0.0f);
                const float r3 = fmaxf(__uint_as_float(vc[(col + 3) % 32]), 0.0f);
                acc0 = ffma2(make_float2(w4.x, w4.y), make_float2(r0, r1), acc0);
                acc1 = ffma2(make_float2(w4.z, w4.w), make_float2(r2, r3), acc1);
              }
              emit(qq, key, (acc0.x + acc1.x) + (acc0.y + acc1.y));
            }
          }
        }
        if (++e_acc == 2) { e_acc = 0; e_acc_phase ^= 1u; }
        idx_cursor_next<RANGES>(c, a, C::QG);
      }
      if (!e_ok) {
        if (lane == 0) atomicOr(a.status, DEV_TIMEOUT);
        *abort_flag = 1;
      }
    }

    if constexpr (FB) {
      // The job's scores are written (every epilogue write precedes the
      // fence and the barrier).  A whole query: the CTA selects its exact
      // top-k from the row.  A chunk: the CTA that completes the query's last
      // chunk does, once every chunk's scores are visible.
      __threadfence();
      __syncthreads();
      bool select_now = true;
      if (job_cpq > 1) {
        if (threadIdx.x == 0) {
          const int done = atomicAdd(&a.fb_done[job_pos], 1);
          __threadfence();
          job_meta[4] = done == job_cpq - 1 ? 1 : 0;
        }
        __syncthreads();
        select_now = job_meta[4] != 0;
      }
      if (select_now && !*abort_flag) {
        const int need = min(a.topk, job_hi - job_lo);
        DenseSelectSmem *sm = reinterpret_cast<DenseSelectSmem *>(smem + C::OFF_STG);
        select_dense_row(a.dense + static_cast<long long>(job_row) * a.dense_ld, job_lo, job_hi - job_lo, need,
                         a.topk, a.topk_idx + static_cast<long long>(job_tl) * a.topk,
                         a.topk_score ? a.topk_score + static_cast<long long>(job_tl) * a.topk : nullptr, a.status,
                         sm, reinterpret_cast<unsigned *>(smem + C::OFF_Q), C::OFF_STG / 4);  // query + key stages are idle
      }
    }
  }

  if (warp == 0 && lane == 0) {
    // Never leave with copies in flight.  Only the last STAGES issued tiles can
    // still be landing, and each of them is the final use of its stage, so the
    // phase parity below is unambiguous (an older phase of a reused stage would
    // alias the current, never-completing one).
    bool drained = true;
    for (int i = (p_issued > C::STAGES ? p_issued - C::STAGES : 0); i < p_issued; ++i)
      drained &= mbar_wait(&full[i % C::STAGES], (i / C::STAGES) & 1u, nullptr);
    if (p_q_issued > 0) drained &= mbar_wait(q_full, static_cast<unsigned>(p_q_issued - 1) & 1u, nullptr);
    if (!drained) atomicOr(a.status, DEV_TIMEOUT);
  } else if (warp == 1) {
    // Drain: every MMA this warp issued must finish before TMEM is released.
    if (lane == 0) {
      tc_commit(drain);
      if (!mbar_wait(drain, 0u, nullptr)) atomicOr(a.status, DEV_TIMEOUT);
    }
    __syncwarp();
  } else if (warp >= 2) {
    if (e_ok && !PILOT && !FB && e_prev_g >= 0) {
#pragma unroll
      for (int qq = 0; qq < QH; ++qq) flush(qq, e_prev_g);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

template <int DI, int HI, bool FP8, int MODE, bool RANGES>
static cudaError_t launch_indexer_t(const CUtensorMap &tq, const CUtensorMap &tk, const IndexerArgs &a, int grid,
                                    cudaStream_t stream) {
  using C = IdxCfg<DI, HI, FP8>;
  auto kern = indexer_kernel<DI, HI, FP8, MODE, RANGES>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  return launch_kernel(kern, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, stream, tq, tk, a);
}

int indexer_queries_per_group(int H_I) { return 256 / H_I; }

template <int DI, int HI, bool FP8>
static cudaError_t launch_indexer_mode(const CUtensorMap &tq, const CUtensorMap &tk, const IndexerArgs &a,
                                       IndexerMode mode, int grid, cudaStream_t stream) {
  const bool ranges = a.key_lo != nullptr;
  switch (mode) {
    case kIdxPilot: return launch_indexer_t<DI, HI, FP8, kIdxPilot, false>(tq, tk, a, grid, stream);
    case kIdxEmit:
      return ranges ? launch_indexer_t<DI, HI, FP8, kIdxEmit, true>(tq, tk, a, grid, stream)
                    : launch_indexer_t<DI, HI, FP8, kIdxEmit, false>(tq, tk, a, grid, stream);
    case kIdxFallback:
      return ranges ? launch_indexer_t<DI, HI, FP8, kIdxFallback, true>(tq, tk, a, grid, stream)
                    : launch_indexer_t<DI, HI, FP8, kIdxFallback, false>(tq, tk, a, grid, stream);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_indexer(const CUtensorMap &tq, const CUtensorMap &tk, const IndexerArgs &a, int D_I, int H_I,
                           bool fp8, IndexerMode mode, int grid, cudaStream_t stream) {
#define DSA_IDX_CASE(DI_, HI_, FP8_) \
  if (D_I == DI_ && H_I == HI_ && fp8 == FP8_) return launch_indexer_mode<DI_, HI_, FP8_>(tq, tk, a, mode, grid, stream);
  DSA_IDX_CASE(128, 32, false)
  DSA_IDX_CASE(128, 32, true)
  DSA_IDX_CASE(64, 4, false)
  DSA_IDX_CASE(64, 32, false)
  DSA_IDX_CASE(128, 16, false)
  DSA_IDX_CASE(128, 16, true)
  DSA_IDX_CASE(128, 8, false)
  DSA_IDX_CASE(128, 8, true)
#undef DSA_IDX_CASE
  return cudaErrorInvalidValue;
}

bool indexer_supported(int D_I, int H_I, bool fp8) {
  if (fp8) return D_I == 128 && (H_I == 32 || H_I == 16 || H_I == 8);
  if (D_I == 128) return H_I == 32 || H_I == 16 || H_I == 8;
  if (D_I == 64) return H_I == 32 || H_I == 4;
  return false;
}

}  // namespace dsa
