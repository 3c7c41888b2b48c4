// mla.cu -- sparse absorbed-MLA attention over each query's selected keys.
//
// mlx-lm PR #1997 ("GLM prefill now attends only to the keys its indexer
// picks", section "How it works"): each cached position holds a single key of
// 576 values (512 latent followed by 64 rope); a query's selected rows are
// fetched once for all of its heads; the heads attend in latent space with
// the key projection absorbed into the query, as in decode.  The work per
// chunk therefore grows with L * top-k rather than L * N.  For query t and
// head h:
//     z_j = scale * (q_lat[t,h] . kv_lat[i_j] + q_rope[t,h] . k_rope[i_j])
//     out[t,h] = sum_j softmax(z)_j * kv_lat[i_j]          (512 wide)
// Index -1 marks a skipped entry (llama.cpp PR #25917, discussion).
//
// B200 mapping.  One CTA per (query, group of 64 heads).  Q lives in tensor
// memory for the whole CTA: its 64 x 576 bf16 rows arrive by bulk copies in
// the still idle second stage and the softmax warps move them into tensor
// memory once, and S = Q K^T reads its A operand from there, so shared
// memory holds only gathered keys (two 108 KB stages of 96-key tiles; the
// packed variant uses three 72 KB stages of 64 keys) and the S MMAs read only
// the key tile from it.  Per tile:
//   * eleven producer warps gather the tile's selected rows with 16-byte
//     cp.async copies straight into the 128-byte-swizzled UMMA operand
//     layout, two rows x 256 bytes per warp instruction, with asynchronous
//     per-lane arrivals; a tensor-map gather (tile::gather4) was measured to
//     issue too slowly for 1,152-byte rows;
//   * S = Q K^T on tcgen05 (M = 64 heads, N = 96 keys, K = 576), fp32 in TMEM;
//   * softmax warps read S from TMEM (two lanes per head row, 48 key columns
//     each), keep a running max (rescaling the output only when the max grows
//     by more than 2^8) and write P (bf16) in the UMMA layout into the rope
//     chunk of the tile's own stage (dead once S is done), so P is buffered
//     with the stages at no extra shared memory;
//   * O += P V on tcgen05 (M = 64, N = 2 x 256 latent columns, K = 96 keys),
//     V read in place from the gathered tile as an MN-major operand; it
//     commits per 32-key group, and the producers refill each group of the
//     stage as soon as its MMAs are done.
// The producers also pull the next tile's rows from HBM into L2
// (prefetch.global.L2) while the current tile's copies land, and the MMA warp
// polls its barriers with the non-suspending mbarrier.test_wait.  Split-key
// mode (chunks with few queries, e.g. decode): CTA z of a query attends its
// z-th share of the selection and writes a normalised fp32 partial and its
// log-sum-exp; mla_combine_kernel merges the shares.
// TMEM (M = 64 operands occupy one 16-lane half of each 32-lane quarter):
// lanes 0-15 hold Q (columns 0-287, two bf16 per column) and the two S buffers
// (from column 288); lanes 16-31 hold O (columns 0-511).  Warp roles: warp 0
// MMA issuer / TMEM owner, warps 1-11 gather producers (all of them fill every
// tile), warps 12-15 Q load, softmax and output.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "dsa_internal.h"
#include "ptx.cuh"

namespace dsa {
namespace mla {

constexpr int HT = 64;           // heads per CTA (UMMA M)
constexpr int DIM = 576;         // joined key width
constexpr int LAT = 512;         // value width
constexpr int ATOMS = DIM / 64;  // 128-byte column atoms
constexpr int N_PROD = 11;       // gather producer warps
constexpr int WARP_PROD0 = 1, WARP_SOFT0 = WARP_PROD0 + N_PROD;
constexpr int THREADS = 32 * (WARP_SOFT0 + 4);
// Tensor memory (512 columns; M = 64 operands use one half of each 32-lane
// quarter): lanes 0-15 hold Q as the A operand of S = Q K^T (576 bf16, two per
// column: columns 0-287) and the two S buffers (from column 288); lanes 16-31
// hold O (columns 0-511, one per latent dimension).
constexpr unsigned Q_COL = 0;
constexpr unsigned S_COL = 288;
constexpr unsigned O_LANE = 16u << 16;
constexpr float kRescaleLog2 = 8.0f;

// Per-variant tiling.  Unpacked: 96-key tiles in two stages (an S MMA of
// N = 96 costs about what one of N = 64 does, so S = Q K^T takes a third fewer
// MMA instructions per key).  Packed (H <= 32): 64-key tiles in three stages,
// matching the pack plan's 64-key union tiles and membership masks.
template <bool PACKED>
struct MlaCfg {
  static constexpr int BK = PACKED ? 64 : 96;          // keys per tile (N of S = Q K^T)
  static constexpr int STAGES = PACKED ? 3 : 2;
  static constexpr int ATOM_BYTES = BK * 128;          // BK rows x 128 B
  static constexpr int KV_BYTES = ATOMS * ATOM_BYTES;
  static constexpr int ROPE_OFF = 8 * ATOM_BYTES;      // a stage's rope chunk; holds P once S of its tile is done
  static constexpr int NC = BK / 2;                    // key columns per softmax thread (two threads per row)
  static constexpr int PPW = (BK / 2 + N_PROD - 1) / N_PROD;  // 2-row groups per producer warp
  static constexpr int GPW = (BK / 4 + N_PROD - 1) / N_PROD;  // 4-row groups per producer warp
  static constexpr int OFF_KV = 0;
  // Q is staged through shared memory once, from stage 1 on (idle until the
  // second tile's gather): one 1,152-byte row every Q_PITCH bytes, so that the
  // 16-byte reads of eight consecutive rows fall in distinct banks.
  static constexpr int Q_PITCH = DIM * 2 + 16;
  static constexpr int OFF_QSTAGE = OFF_KV + KV_BYTES;
  static constexpr int OFF_BAR = OFF_KV + STAGES * KV_BYTES;
  // O += P V of a tile frees its stage in 32-key row groups (P of a group
  // lies in the group's own rope rows), so the next gather into the stage
  // starts while the later groups are still being multiplied.
  static constexpr int NG = BK / 32;
  static constexpr int NBAR = 1 + 4 * STAGES + 2 + 2 + 1 + 1 + NG * STAGES;
  static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
  static constexpr int OFF_VALID = OFF_MISC + 64;      // [STAGES][N_PROD][2] key validity words (128 keys max)
  static constexpr int OFF_MEMB = OFF_VALID + STAGES * N_PROD * 16;  // [STAGES][64] per-query key masks (packed)
  static constexpr int SMEM_BYTES = OFF_MEMB + STAGES * 64 * 8 + 1024;
  static_assert(SMEM_BYTES <= 227 * 1024, "shared memory budget");
  static_assert(S_COL + 2 * BK <= 512, "tensor memory budget");
  static_assert(OFF_QSTAGE + HT * Q_PITCH <= OFF_BAR, "Q staging area");
  static_assert(BK % 32 == 0 && BK <= 128, "tile width");
};

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// PACKED: the CTA serves G consecutive queries of H <= 32 heads (rows
// j*H .. j*H+H-1 of the 64-row tile belong to query j) over the union of their
// selections; a union key counts for row r only if query r / H chose it.
template <bool PACKED>
__global__ void __launch_bounds__(THREADS, 1) sparse_mla_kernel(MlaArgs a) {
  pdl_wait_and_release();
  using C = MlaCfg<PACKED>;
  constexpr int BK = C::BK, STAGES = C::STAGES, ATOM_BYTES = C::ATOM_BYTES, KV_BYTES = C::KV_BYTES;
  constexpr int ROPE_OFF = C::ROPE_OFF, NC = C::NC, PPW = C::PPW, GPW = C::GPW;
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *kv_s = smem + C::OFF_KV;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + C::OFF_BAR);
  uint64_t *q_full = bars;                     // Q written into tensor memory (one arrival per softmax warp)
  uint64_t *kv_full = bars + 1;                // [STAGES]
  uint64_t *kv_empty = bars + 1 + STAGES;      // [STAGES]
  uint64_t *valid_full = bars + 1 + 2 * STAGES;  // [STAGES] validity words of the stage's tile published
  uint64_t *s_full = bars + 1 + 3 * STAGES;    // [2]
  uint64_t *s_free = s_full + 2;               // [2]
  // [STAGES] P of the stage's tile written.  One barrier per stage: the
  // softmax may finish two tiles before the MMA warp looks, and with a single
  // barrier the parity of a phase two ahead would read as "not yet".
  uint64_t *p_full = s_full + 4;
  uint64_t *drain = p_full + STAGES;
  uint64_t *q_copied = drain + 1;              // Q rows landed in the staging area (transaction bytes)
  uint64_t *grp_free = q_copied + 1;           // [STAGES][NG] O += P V done with the stage's 32-key row group
  unsigned *tmem_slot = reinterpret_cast<unsigned *>(smem + C::OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + C::OFF_MISC + 4);
  unsigned long long *valid_s = reinterpret_cast<unsigned long long *>(smem + C::OFF_VALID);  // [STAGES][N_PROD][2]
  unsigned long long *memb_s = reinterpret_cast<unsigned long long *>(smem + C::OFF_MEMB);    // [STAGES][64]

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  int item = blockIdx.x;  // the query (or pack) this CTA serves
  if (a.list != nullptr) {
    if (static_cast<int>(blockIdx.x) >= *a.list_count) return;
    item = a.list[blockIdx.x];
  }
  const int t = a.t0 + item * (PACKED ? a.G : 1);  // first query of this CTA
  const int hg = blockIdx.y;
  const int nq = PACKED ? min(a.G, a.t0 + a.Lq - t) : 1;  // queries served
  // Keys this CTA walks: the query's selection (or its share of it in
  // split-key mode), or the pack's union.
  int nkeys = PACKED ? a.ucount[item] : a.topk;
  const int32_t *keys = PACKED ? a.ukeys + static_cast<long long>(item) * a.umax
                               : a.topk_idx + static_cast<long long>(t) * a.topk;
  const bool split_mode = !PACKED && a.nsplit > 1;
  const int split = blockIdx.z;
  if (split_mode) {
    const int per = ((nkeys + BK - 1) / BK + a.nsplit - 1) / a.nsplit * BK;  // whole tiles per share
    const int k0 = split * per;
    keys += k0;
    nkeys = max(0, min(nkeys - k0, per));
  }
  const unsigned long long *qmask = PACKED ? a.qmask + static_cast<long long>(item) * a.umax : nullptr;
  const int ntiles = max(1, (nkeys + BK - 1) / BK);
  // Output rows of the 64-row tile: global row out_row0 + r for r < row_limit.
  const long long out_row0 = static_cast<long long>(t) * a.H + (PACKED ? 0 : hg * HT);
  const int row_limit = PACKED ? nq * a.H : min(HT, a.H - hg * HT);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 4);
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&kv_full[i], N_PROD * 32);  // one asynchronous arrival per producer lane
      mbar_init(&kv_empty[i], 1);
      mbar_init(&valid_full[i], N_PROD);
      mbar_init(&p_full[i], 4);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
    }
    mbar_init(drain, 1);
    mbar_init(q_copied, 1);
    for (int i = 0; i < STAGES * C::NG; ++i) mbar_init(&grp_free[i], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 0) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const unsigned tmem = *tmem_slot;
  const unsigned s_col = tmem + S_COL;                 // S buffers (lanes 0-15 of each quarter)
  const unsigned o_lat0 = tmem + O_LANE;               // O, latent dims 0-255 (lanes 16-31)
  const unsigned o_lat1 = tmem + O_LANE + 256;         // O, latent dims 256-511

  if (warp >= WARP_PROD0 && warp < WARP_SOFT0) {
    // ------------------------------------------------------------ gather producers
    // All producer warps fill every tile (tile j goes to stage j % STAGES).
    // The latent chunks go in pairs: a warp instruction moves 2 rows x 256
    // bytes (lane / 16 picks the row, lane / 8 % 2 the chunk of the pair, lane
    // % 8 the 16-byte piece), which gathers about twice as fast as 4 rows x
    // 128 bytes; the rope chunk goes 4 rows x 128 bytes.  Producer warp pw
    // takes row pairs and row quads pw + N_PROD i.  Each lane's arrival on
    // the stage's barrier fires when its copies land, so the producers never
    // block on data and keep many rows in flight.
    const int pw = warp - WARP_PROD0;
    const int u = lane & 7;
    const int sub2 = lane >> 4, seg = (lane >> 3) & 1;  // pair mapping
    const int sub4 = lane >> 3;                         // quad mapping
    bool ok = true;
    auto key_at = [&](int j, int r) -> int {
      const int pos = j * BK + r;
      return (j < ntiles && pos < nkeys) ? keys[pos] : -1;
    };
    auto load_keys = [&](int j, int (&kp)[PPW], int (&kq)[GPW]) {
#pragma unroll
      for (int i = 0; i < PPW; ++i) {
        const int grp = pw + N_PROD * i;
        kp[i] = grp < BK / 2 ? key_at(j, 2 * grp + sub2) : -1;
      }
#pragma unroll
      for (int i = 0; i < GPW; ++i) {
        const int grp = pw + N_PROD * i;
        kq[i] = grp < BK / 4 ? key_at(j, 4 * grp + sub4) : -1;
      }
    };
    // Packed mode: lane q < G of producer warp 0 carries query q's 64-bit key mask of the tile.
    auto load_mask = [&](int j) -> unsigned long long {
      return (PACKED && pw == 0 && lane < nq && j < ntiles) ? qmask[static_cast<long long>(j) * 64 + lane] : 0ull;
    };
    auto row_offset = [&](int v) -> long long {  // invalid entries read row 0 (their scores are masked)
      return static_cast<long long>((v >= 0 && v < a.N) ? v : 0) * a.kv_ld * 2;
    };
    const uint8_t *kv = static_cast<const uint8_t *>(a.kv);
    // Index registers run one tile ahead.
    int kp[PPW], kq[GPW], kp_n[PPW], kq_n[GPW];
    unsigned long long cm = 0ull, cm_n = 0ull;
    load_keys(0, kp, kq);
    cm = load_mask(0);
    for (int j = 0; j < ntiles; ++j) {
      load_keys(j + 1, kp_n, kq_n);
      cm_n = load_mask(j + 1);
      const int st = j % STAGES;
      unsigned long long vlo = 0, vhi = 0;  // validity of tile rows 0-63, 64-127
#pragma unroll
      for (int i = 0; i < GPW; ++i) {
        const int v = kq[i];
        if (u == 0 && (v >= a.N || v < -1)) atomicOr(a.status, DEV_BAD_INDEX);
        const int grp = pw + N_PROD * i;
        if (grp < BK / 4 && v >= 0 && v < a.N) {
          const int bit = 4 * grp + sub4;
          if (bit < 64) vlo |= 1ull << bit; else vhi |= 1ull << (bit - 64);
        }
      }
      vlo |= __shfl_xor_sync(0xffffffffu, vlo, 8);
      vlo |= __shfl_xor_sync(0xffffffffu, vlo, 16);
      vhi |= __shfl_xor_sync(0xffffffffu, vhi, 8);
      vhi |= __shfl_xor_sync(0xffffffffu, vhi, 16);
      // Stage 1 on holds the staged Q rows until they are in tensor memory.
      if (j == 1 && !mbar_wait(q_full, 0u, abort_flag)) { ok = false; break; }
      // Row group g (keys 32g .. 32g + 31) of the stage is refilled as soon as
      // O += P V of the stage's previous tile is done with it.
      const unsigned stage_base = smem_u32(kv_s + st * KV_BYTES);
#pragma unroll
      for (int g = 0; g < C::NG; ++g) {
        if (!mbar_wait(&grp_free[st * C::NG + g], ((j / STAGES) & 1) ^ 1u, abort_flag)) { ok = false; break; }
        if (g == 0) {
          // The stage's previous tile has been consumed (its softmax included).
          if (PACKED && pw == 0 && lane < nq) memb_s[st * 64 + lane] = cm;
          __syncwarp();
          if (lane == 0) {
            valid_s[(st * N_PROD + pw) * 2] = vlo;
            valid_s[(st * N_PROD + pw) * 2 + 1] = vhi;
            mbar_arrive(&valid_full[st]);
          }
        }
#pragma unroll
        for (int pr = 0; pr < 4; ++pr) {
          const int c = 2 * pr + seg;
#pragma unroll
          for (int i = 0; i < PPW; ++i) {
            const int grp = pw + N_PROD * i;  // row pair
            const int r = 2 * grp + sub2;
            if (grp >= 16 * g && grp < 16 * g + 16 && r < BK)
              cp_async_16(stage_base + c * ATOM_BYTES + r * 128 + ((u ^ (r & 7)) << 4),
                          kv + row_offset(kp[i]) + c * 128 + u * 16);
          }
        }
#pragma unroll
        for (int i = 0; i < GPW; ++i) {
          const int grp = pw + N_PROD * i;  // row quad
          const int r = 4 * grp + sub4;
          if (grp >= 8 * g && grp < 8 * g + 8 && r < BK)
            cp_async_16(stage_base + 8 * ATOM_BYTES + r * 128 + ((u ^ (r & 7)) << 4),
                        kv + row_offset(kq[i]) + 8 * 128 + u * 16);
        }
      }
      if (!ok) break;
      cp_async_arrive_noinc(&kv_full[st]);
      // Pull the next tile's rows from HBM into L2 now; its gather starts only
      // once its stage is consumed.
#pragma unroll
      for (int i = 0; i < GPW; ++i) {
        const int v = kq_n[i];
        if (v >= 0 && v < a.N) {
          const uint8_t *row = kv + row_offset(v);
          prefetch_l2_line(row + u * 128);
          if (u == 0) prefetch_l2_line(row + 8 * 128);
        }
      }
#pragma unroll
      for (int i = 0; i < PPW; ++i) kp[i] = kp_n[i];
#pragma unroll
      for (int i = 0; i < GPW; ++i) kq[i] = kq_n[i];
      cm = cm_n;
    }
    cp_async_wait_all();  // never leave with copies in flight
    if (!ok) {
      if (lane == 0) atomicOr(a.status, DEV_TIMEOUT);
      *abort_flag = 1;
    }
    __syncwarp();
  } else if (warp == 0) {
    // ------------------------------------------------------------ MMA issuer
    constexpr unsigned idesc_qk = make_idesc(HT, BK, 1u, 0u, 0u);   // S = Q K^T, Q from TMEM, K K-major
    constexpr unsigned idesc_pv = make_idesc(HT, 256, 1u, 0u, 1u);  // O += P V, V MN-major
    bool ok = mbar_wait(q_full, 0u, abort_flag);
    tc_fence_after();
    // Descriptors of stage 0; a stage's operands sit KV_BYTES further on,
    // added to the start-address field (address >> 4; shared addresses stay
    // below 2^18, so the 14-bit field never carries).
    const uint64_t k_desc0 = smem_desc_sw128(smem_u32(kv_s), 16, 1024);
    const uint64_t v_desc0 = smem_desc_sw128(smem_u32(kv_s), ATOM_BYTES, 1024);
    // P (A of O += P V) in the no-swizzle core-matrix layout, key-chunk major:
    // the 8-row x 16-byte core matrix (row group rg, 8-key chunk kc) sits at
    // kc * 1024 + rg * 128, so the P of keys 32g .. 32g + 31 fills exactly the
    // rope rows of those keys (the rope chunk is dead once S = Q K^T is done).
    const uint64_t p_desc0 = smem_desc_noswz(smem_u32(kv_s + ROPE_OFF), 1024, 128);
    auto issue_pv = [&](int jj) {
      const int s = jj % STAGES;
      const uint64_t so = static_cast<uint64_t>((s * KV_BYTES) >> 4);
#pragma unroll
      for (int g = 0; g < C::NG; ++g) {
#pragma unroll
        for (int ks = 2 * g; ks < 2 * g + 2; ++ks) {
          const unsigned acc = (jj > 0 || ks > 0) ? 1u : 0u;
          mma_bf16_ss(o_lat0, p_desc0 + so + ((ks * 2048) >> 4), v_desc0 + so + ((ks * 2048) >> 4), idesc_pv, acc);
          mma_bf16_ss(o_lat1, p_desc0 + so + ((ks * 2048) >> 4),
                      v_desc0 + so + ((4 * ATOM_BYTES + ks * 2048) >> 4), idesc_pv, acc);
        }
        tc_commit(&grp_free[s * C::NG + g]);  // this group's V rows and P are read
      }
      tc_commit(&kv_empty[s]);
    };
    // Event-driven issue: O += P V for tile np as soon as its P is written (it
    // frees a gather stage), otherwise S = Q K^T for tile nq once its keys have
    // landed and its S buffer is free.  Lane 0 polls, the warp follows.
    int nq = 0, np = 0;
    bool idle = false;
    unsigned long long t_idle = 0;
    unsigned spins = 0;
    while (ok && np < ntiles) {
      int action = 0;
      if (lane == 0) {
        if (np < nq && mbar_test_wait(&p_full[np % STAGES], (np / STAGES) & 1u))
          action = 1;
        else if (nq < ntiles && mbar_test_wait(&kv_full[nq % STAGES], (nq / STAGES) & 1u) &&
                 mbar_test_wait(&s_free[nq & 1], ((nq >> 1) & 1u) ^ 1u))
          action = 2;
        // the gathered rows were written through the generic proxy
        if (action == 2) fence_proxy_async_smem();
      }
      action = __shfl_sync(0xffffffffu, action, 0);
      if (action == 1) {
        tc_fence_after();
        if (lane == 0) issue_pv(np);
        __syncwarp();
        ++np;
        idle = false;
      } else if (action == 2) {
        tc_fence_after();
        if (lane == 0) {
          const int st = nq % STAGES;
          const uint64_t kd = k_desc0 + static_cast<uint64_t>((st * KV_BYTES) >> 4);
          const unsigned s_tmem = s_col + (nq & 1) * BK;
#pragma unroll
          for (int at = 0; at < ATOMS; ++at) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              const uint64_t off = static_cast<uint64_t>((at * ATOM_BYTES + ks * 32) >> 4);
              mma_bf16_ts(s_tmem, tmem + Q_COL + at * 32 + ks * 8, kd + off, idesc_qk, (at | ks) ? 1u : 0u);
            }
          }
          tc_commit(&s_full[nq & 1]);
        }
        __syncwarp();
        ++nq;
        idle = false;
      } else if (!idle) {
        idle = true;
        t_idle = globaltimer();
        spins = 0;
      } else if ((++spins & 63u) == 0) {
        if (*abort_flag || globaltimer() - t_idle > kWaitLimitNs) ok = false;
      }
    }
    if (!ok) {
      if (lane == 0) atomicOr(a.status, DEV_TIMEOUT);
      *abort_flag = 1;
    }
    if (lane == 0) {
      tc_commit(drain);
      if (!mbar_wait(drain, 0u, nullptr)) atomicOr(a.status, DEV_TIMEOUT);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ Q load, softmax, output
    const int quarter = warp & 3;
    const int r16 = lane & 15;
    const int row = quarter * 16 + r16;  // head within the CTA's group
    const unsigned lane_base = static_cast<unsigned>(quarter * 32) << 16;
    const int half = lane >> 4;          // which 32 of each 64 columns this thread's 16x32bx2 accesses cover
    bool ok = true;
    {
      // Q rows into tensor memory as the A operand of S = Q K^T, through the
      // staging area: one bulk copy per valid row (two warps issue them), then
      // row `row` goes to lane quarter*32 + r16, dims 2c and 2c + 1 in column
      // c.  Thread halves take alternate 64-dim runs of the row (the 16x32bx2
      // store pairs them); rows past the tile's last valid row are zero.
      const unsigned qstage = smem_u32(smem + C::OFF_QSTAGE);
      if (warp == WARP_SOFT0 && lane == 0) mbar_arrive_expect_tx(q_copied, static_cast<unsigned>(row_limit) * DIM * 2);
      if (warp < WARP_SOFT0 + 2) {
        const int qr = (warp - WARP_SOFT0) * 32 + lane;
        if (qr < row_limit)
          bulk_copy_g2s(qstage + qr * C::Q_PITCH, a.q + (out_row0 + qr) * DIM, DIM * 2, q_copied);
      }
      ok = mbar_wait(q_copied, 0u, abort_flag);
      if (!ok) *abort_flag = 1;
      const bool qv = ok && row < row_limit;
      const uint8_t *src = smem + C::OFF_QSTAGE + row * C::Q_PITCH;
      const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll 1
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t r[32];
        const int e0 = 128 * ch + 64 * half;  // first dim of this thread's run
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const uint4 v = qv ? *reinterpret_cast<const uint4 *>(src + (e0 + 8 * k) * 2) : z4;
          r[4 * k] = v.x;
          r[4 * k + 1] = v.y;
          r[4 * k + 2] = v.z;
          r[4 * k + 3] = v.w;
        }
        tmem_st_16x32bx2_x32(tmem + lane_base + Q_COL + 64 * ch, r);
      }
      {
        uint32_t r[16];
        const int e0 = 512 + 32 * half;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint4 v = qv ? *reinterpret_cast<const uint4 *>(src + (e0 + 8 * k) * 2) : z4;
          r[4 * k] = v.x;
          r[4 * k + 1] = v.y;
          r[4 * k + 2] = v.z;
          r[4 * k + 3] = v.w;
        }
        tmem_st_16x32bx2_x16(tmem + lane_base + Q_COL + 256, r);
      }
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(q_full);
    }
    float m_used = -INFINITY, l = 0.0f, l_exact = 0.0f;  // l: sum of the bf16 P used; l_exact: fp32 sum for the LSE
    // This thread's NC of the tile's BK key columns: [32 half, 32 half + 32)
    // and, for 96-key tiles, also [64 + 16 half, 64 + 16 half + 16) (TMEM
    // half-split loads whose second half sits one load width further on).
    const int c0 = half * 32;
    for (int j = 0; ok && j < ntiles; ++j) {
      const int sb = j & 1;
      const int st = j % STAGES;
      if (!mbar_wait(&s_full[sb], (j >> 1) & 1u, abort_flag)) { ok = false; break; }
      tc_fence_after();
      if (!mbar_wait(&valid_full[st], (j / STAGES) & 1u, abort_flag)) { ok = false; break; }
      uint32_t sv[NC];
      tmem_ld_16x32bx2_x32_split<32>(s_col + lane_base + sb * BK, sv);
      if constexpr (NC == 48) tmem_ld_16x32bx2_x16_split<16>(s_col + lane_base + sb * BK + 64, sv + 32);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[sb]);
      unsigned long long vbits;  // bit c: this thread's c-th key column holds a valid key
      if (PACKED) {
        // keys of this tile that the row's own query chose
        const int qj = row / a.H;
        vbits = qj < nq ? (memb_s[st * 64 + qj] >> c0) : 0ull;
      } else {
        unsigned long long lo = 0ull, hi = 0ull;
#pragma unroll
        for (int w = 0; w < N_PROD; ++w) {
          lo |= valid_s[(st * N_PROD + w) * 2];
          hi |= valid_s[(st * N_PROD + w) * 2 + 1];
        }
        vbits = ((lo >> c0) & 0xFFFFFFFFull) | (((hi >> (16 * half)) & 0xFFFFull) << 32);
      }
      // Logits in the log2 domain, z = S * scale * log2(e) (packed multiplies);
      // skipped or padding entries -inf, masked only in a tile that has any.
      float z[NC];
      {
        const float2 sc2 = make_float2(a.scale_log2, a.scale_log2);
#pragma unroll
        for (int c = 0; c < NC; c += 2) {
          const float2 zz = fmul2(make_float2(__uint_as_float(sv[c]), __uint_as_float(sv[c + 1])), sc2);
          z[c] = zz.x;
          z[c + 1] = zz.y;
        }
      }
      constexpr unsigned long long kAllCols = (1ull << NC) - 1ull;  // NC <= 48
      if (!__all_sync(0xffffffffu, (vbits & kAllCols) == kAllCols)) {
#pragma unroll
        for (int c = 0; c < NC; ++c) z[c] = ((vbits >> c) & 1ull) ? z[c] : -INFINITY;
      }
      float tmax = -INFINITY;
#pragma unroll
      for (int c = 0; c < NC; c += 2) tmax = fmax3(tmax, z[c], z[c + 1]);
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));  // whole row (both halves)
      const float m_old = m_used;
      bool rescale = false;
      if (tmax > m_used + kRescaleLog2 || (m_used == -INFINITY && tmax > -INFINITY)) {
        rescale = (m_used != -INFINITY) && (j > 0);
        m_used = tmax;
      }
      // P in bf16, rounded once; the normaliser sums the rounded values (two
      // packed partial sums; the fp32 sum of the unrounded values feeds the
      // LSE).  A row with no valid key yet has m = -inf and z = -inf: subtract
      // 0 so that exp2 gives 0.
      uint32_t pk[NC / 2];
      const float m_sub = (m_used == -INFINITY) ? 0.0f : m_used;
      const float2 m2 = make_float2(m_sub, m_sub);
      float2 tsum2 = make_float2(0.0f, 0.0f), texact2 = make_float2(0.0f, 0.0f);
#pragma unroll
      for (int c = 0; c < NC; c += 2) {
        const float2 d = fsub2(make_float2(z[c], z[c + 1]), m2);
        const float p0 = fast_exp2(d.x), p1 = fast_exp2(d.y);
        const __nv_bfloat162 b = __floats2bfloat162_rn(p0, p1);
        tsum2 = fadd2(tsum2, __bfloat1622float2(b));
        texact2 = fadd2(texact2, make_float2(p0, p1));
        pk[c >> 1] = *reinterpret_cast<const uint32_t *>(&b);
      }
      float tsum = tsum2.x + tsum2.y, tsum_exact = texact2.x + texact2.y;
      tsum += __shfl_xor_sync(0xffffffffu, tsum, 16);
      tsum_exact += __shfl_xor_sync(0xffffffffu, tsum_exact, 16);
      const float alpha = rescale ? fast_exp2(m_old - m_used) : 1.0f;
      l = l * alpha + tsum;
      l_exact = l_exact * alpha + tsum_exact;
      // Rescale O when the running max moved: both halves of a row (lanes r16
      // and r16 + 16) take 32 of every 64 columns of the row's O (same
      // alpha).  O is idle once O += P V of the previous tile is done.
      if (__any_sync(0xffffffffu, rescale)) {
        if (!mbar_wait(&kv_empty[(j - 1) % STAGES], ((j - 1) / STAGES) & 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
#pragma unroll 1
        for (int ch = 0; ch < 8; ++ch) {
          uint32_t ov[32];
          tmem_ld_16x32bx2_x32(o_lat0 + lane_base + ch * 64, ov);
          tmem_ld_wait();
          if (rescale) {
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
          }
          tmem_st_16x32bx2_x32(o_lat0 + lane_base + ch * 64, ov);
        }
        tmem_st_wait();
      }
      {
        // P of tile j goes into the rope chunk of its own stage (dead after S = Q K^T)
        uint8_t *pbase = kv_s + st * KV_BYTES + ROPE_OFF;
#pragma unroll
        for (int ch = 0; ch < NC / 8; ++ch) {
          const uint4 v = make_uint4(pk[ch * 4 + 0], pk[ch * 4 + 1], pk[ch * 4 + 2], pk[ch * 4 + 3]);
          const int k = ch < 4 ? 4 * half + ch : 8 + 2 * half + (ch - 4);  // 8-key chunk of the tile
          // core matrix (row / 8, k) at k * 1024 + (row / 8) * 128, row row % 8 within it
          *reinterpret_cast<uint4 *>(pbase + k * 1024 + row * 16) = v;
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[st]);
    }
    if (ok) ok = mbar_wait(&kv_empty[(ntiles - 1) % STAGES], ((ntiles - 1) / STAGES) & 1u, abort_flag);
    if (!ok) {
      if (lane == 0) atomicOr(a.status, DEV_TIMEOUT);
      *abort_flag = 1;
    } else {
      tc_fence_after();
      const float inv = l > 0.0f ? 1.0f / l : 0.0f;  // both halves of a row hold the row's l
      const bool has_row = row < row_limit;
      uint16_t *orow = a.out + (out_row0 + row) * LAT;
      // split-key mode: this share's normalised fp32 output row
      const long long prow_idx = (static_cast<long long>(t - a.t0) * a.H + hg * HT + row) * a.nsplit + split;
      float *porow = split_mode ? a.part_o + prow_idx * LAT : nullptr;
      // Normalise, convert and store 64 output columns of the row per step;
      // the next step's tensor-memory load is in flight meanwhile.
      // Rows are 1,024 bytes and each thread's 32 dims start 64-byte aligned:
      // 32-byte stores work whenever the output itself is 32-byte aligned.
      const bool out32 = (reinterpret_cast<uintptr_t>(a.out) & 31u) == 0;
      auto emit = [&](int ch, const uint32_t (&ov)[32]) {
        const int d0 = 64 * ch + c0;  // this thread's 32 latent dims
        if (has_row && split_mode) {
          float4 *dst = reinterpret_cast<float4 *>(porow + d0);
#pragma unroll
          for (int e = 0; e < 8; ++e)
            dst[e] = make_float4(__uint_as_float(ov[4 * e]) * inv, __uint_as_float(ov[4 * e + 1]) * inv,
                                 __uint_as_float(ov[4 * e + 2]) * inv, __uint_as_float(ov[4 * e + 3]) * inv);
        } else if (has_row) {
          uint32_t pkd[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const __nv_bfloat162 b =
                __floats2bfloat162_rn(__uint_as_float(ov[2 * e]) * inv, __uint_as_float(ov[2 * e + 1]) * inv);
            pkd[e] = *reinterpret_cast<const uint32_t *>(&b);
          }
          if (out32) {  // two 32-byte stores: whole 32-byte sectors, half the store requests
            st_global_v8(orow + d0, pkd);
            st_global_v8(orow + d0 + 16, pkd + 8);
          } else {
            uint4 *dst = reinterpret_cast<uint4 *>(orow + d0);
#pragma unroll
            for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pkd[4 * e], pkd[4 * e + 1], pkd[4 * e + 2], pkd[4 * e + 3]);
          }
        }
      };
      uint32_t ova[32], ovb[32];
      tmem_ld_16x32bx2_x32(o_lat0 + lane_base, ova);
      tmem_ld_wait();
      reg_fence(ova);
#pragma unroll 1
      for (int ch = 0; ch < 8; ch += 2) {
        tmem_ld_16x32bx2_x32(o_lat0 + lane_base + (ch + 1) * 64, ovb);
        emit(ch, ova);
        tmem_ld_wait();
        reg_fence(ovb);
        if (ch + 2 < 8) tmem_ld_16x32bx2_x32(o_lat0 + lane_base + (ch + 2) * 64, ova);
        emit(ch + 1, ovb);
        tmem_ld_wait();
        reg_fence(ova);
      }
      const float row_lse = l_exact > 0.0f ? (m_used + log2f(l_exact)) * 0.69314718055994530942f : -INFINITY;
      if (lane < 16 && has_row && split_mode) {
        a.part_lse[prow_idx] = row_lse;
      } else if (lane < 16 && has_row && a.lse != nullptr) {
        a.lse[out_row0 + row] = row_lse;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Merge the key shares of split-key mode: one warp per (query, head) row.
// With per-share log-sum-exps lse_s and normalised outputs o_s, the row's
// lse = log sum_s exp(lse_s) and out = sum_s exp(lse_s - lse) o_s, which is
// the softmax over the union of the shares (they are disjoint).
__global__ void __launch_bounds__(256) mla_combine_kernel(MlaArgs a) {
  pdl_wait_and_release();
  const int lane = threadIdx.x % 32;
  const long long rowg = (static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x) / 32;
  if (rowg >= static_cast<long long>(a.Lq) * a.H) return;
  const float *ls = a.part_lse + rowg * a.nsplit;
  const float my = lane < a.nsplit ? ls[lane] : -INFINITY;
  float m = my;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  float wgt = (m == -INFINITY || my == -INFINITY) ? 0.0f : __expf(my - m);
  float sum = wgt;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float inv = sum > 0.0f ? 1.0f / sum : 0.0f;
  // lane d16 accumulates dims [16 d16, 16 d16 + 16)
  float acc[16];
#pragma unroll
  for (int e = 0; e < 16; ++e) acc[e] = 0.0f;
  // Four shares' loads in flight at a time (the shares are added in order;
  // an empty share has weight 0 and its row, which may hold anything, is skipped).
  for (int sp0 = 0; sp0 < a.nsplit; sp0 += 4) {
    float4 v[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int sp = min(sp0 + j, a.nsplit - 1);
      const float4 *src = reinterpret_cast<const float4 *>(a.part_o + (rowg * a.nsplit + sp) * LAT + lane * 16);
#pragma unroll
      for (int e = 0; e < 4; ++e) v[j][e] = src[e];
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float ws = __shfl_sync(0xffffffffu, wgt, sp0 + j) * inv;  // lanes >= nsplit carry weight 0
      if (sp0 + j >= a.nsplit || ws == 0.0f) continue;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        acc[4 * e] += ws * v[j][e].x;
        acc[4 * e + 1] += ws * v[j][e].y;
        acc[4 * e + 2] += ws * v[j][e].z;
        acc[4 * e + 3] += ws * v[j][e].w;
      }
    }
  }
  const long long orow = (static_cast<long long>(a.t0) * a.H + rowg) * LAT + lane * 16;
  uint32_t pk[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(acc[2 * e], acc[2 * e + 1]);
    pk[e] = *reinterpret_cast<const uint32_t *>(&b);
  }
  uint4 *dst = reinterpret_cast<uint4 *>(a.out + orow);
  dst[0] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
  dst[1] = make_uint4(pk[4], pk[5], pk[6], pk[7]);
  if (lane == 0 && a.lse != nullptr)
    a.lse[static_cast<long long>(a.t0) * a.H + rowg] = sum > 0.0f ? m + logf(sum) : -INFINITY;
}

}  // namespace mla

cudaError_t launch_mla_combine(const MlaArgs &a, cudaStream_t stream) {
  const long long rows = static_cast<long long>(a.Lq) * a.H;
  const int blocks = static_cast<int>((rows * 32 + 255) / 256);
  return launch_kernel(mla::mla_combine_kernel, dim3(blocks), dim3(256), 0, stream, a);
}

cudaError_t launch_sparse_mla(const MlaArgs &a, bool packed, cudaStream_t stream) {
  auto kern = packed ? mla::sparse_mla_kernel<true> : mla::sparse_mla_kernel<false>;
  const int smem = packed ? mla::MlaCfg<true>::SMEM_BYTES : mla::MlaCfg<false>::SMEM_BYTES;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  dim3 grid(packed ? (a.Lq + a.G - 1) / a.G : a.Lq, packed ? 1 : (a.H + mla::HT - 1) / mla::HT,
            packed ? 1 : max(1, a.nsplit));
  return launch_kernel(kern, grid, dim3(mla::THREADS), smem, stream, a);
}

}  // namespace dsa
