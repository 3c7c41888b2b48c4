// mla.cu -- sparse absorbed-MLA attention over each query's selected keys.
//
// mlx-lm PR #1997 ("GLM prefill now attends only to the keys its indexer
// picks", section "How it works"): the latent and rope caches are joined into
// one 576-wide key per position, the top-k rows a query picked are gathered
// once and shared by all its heads, and attention runs in the absorbed latent
// space, so a chunk costs L * top-k instead of L * N.  For query t and head h:
//     z_j = scale * (q_lat[t,h] . kv_lat[i_j] + q_rope[t,h] . k_rope[i_j])
//     out[t,h] = sum_j softmax(z)_j * kv_lat[i_j]          (512 wide)
// Index -1 marks a skipped entry (llama.cpp PR #25917, discussion).
//
// B200 mapping.  One CTA per (query, group of 64 heads).  Per 64-key tile:
//   * two producer warps, one per stage, gather the 64 selected rows with
//     16-byte cp.async copies (each 8-lane group moves one 128-byte row
//     segment, coalesced) straight into the 128-byte-swizzled UMMA operand
//     layout; a tensor-map gather (tile::gather4) was measured to issue too
//     slowly for 1,152-byte rows;
//   * S = Q K^T on tcgen05 (M = 64 heads, N = 64 keys, K = 576), fp32 in TMEM;
//   * softmax warps read S from TMEM (two lanes per head row, 32 key columns
//     each), keep a running max (rescaling the output only when the max grows
//     by more than 2^8) and write P (bf16) to shared memory in the UMMA layout;
//   * O += P V on tcgen05 (M = 64, N = 2 x 256 latent columns, K = 64 keys),
//     V read in place from the gathered tile as an MN-major operand.
// TMEM: the two 64 x 256 fp32 halves of O sit in the two half-subpartitions
// (lanes 0-15 and 16-31 of each 32-lane quarter) of columns 0-255, the two S
// buffers in columns 256-383.  Warp roles: warps 0 and 6 gather producers
// (stage 0 / stage 1), warp 1 MMA issuer / TMEM owner, warps 2-5 softmax and
// output.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "dsa_internal.h"
#include "ptx.cuh"

namespace dsa {
namespace mla {

constexpr int HT = 64;           // heads per CTA (UMMA M)
constexpr int BK = 64;           // keys per tile
constexpr int DIM = 576;         // joined key width
constexpr int LAT = 512;         // value width
constexpr int ATOMS = DIM / 64;  // 128-byte column atoms
constexpr int ATOM_BYTES = 64 * 128;  // 64 rows x 128 B
constexpr int Q_BYTES = ATOMS * ATOM_BYTES;
constexpr int KV_BYTES = ATOMS * ATOM_BYTES;
constexpr int P_BYTES = HT * BK * 2;
constexpr int STAGES = 2;
constexpr int THREADS = 224;
constexpr int OFF_Q = 0;
constexpr int OFF_KV = OFF_Q + Q_BYTES;
constexpr int OFF_P = OFF_KV + STAGES * KV_BYTES;
constexpr int OFF_BAR = OFF_P + P_BYTES;
constexpr int NBAR = 1 + 2 * STAGES + 4 + 2 + 1;
constexpr int OFF_MISC = OFF_BAR + NBAR * 8;
constexpr int OFF_MEMB = OFF_MISC + 64;             // [STAGES][64] per-query key masks (packed mode)
constexpr int SMEM_BYTES = OFF_MEMB + STAGES * BK * 8 + 1024;
constexpr float kRescaleLog2 = 8.0f;

__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// PACKED: the CTA serves G consecutive queries of H <= 32 heads (rows
// j*H .. j*H+H-1 of the 64-row tile belong to query j) over the union of their
// selections; a union key counts for row r only if query r / H chose it.
template <bool PACKED>
__global__ void __launch_bounds__(THREADS, 1)
    sparse_mla_kernel(const __grid_constant__ CUtensorMap tmap_q, MlaArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t *q_s = smem + OFF_Q;
  uint8_t *kv_s = smem + OFF_KV;
  uint8_t *p_s = smem + OFF_P;
  uint64_t *bars = reinterpret_cast<uint64_t *>(smem + OFF_BAR);
  uint64_t *q_full = bars;
  uint64_t *kv_full = bars + 1;           // [2]
  uint64_t *kv_empty = bars + 3;          // [2]
  uint64_t *s_full = bars + 5;            // [2]
  uint64_t *s_free = bars + 7;            // [2]
  uint64_t *p_full = bars + 9;
  uint64_t *p_free = bars + 10;
  uint64_t *drain = bars + 11;
  unsigned *tmem_slot = reinterpret_cast<unsigned *>(smem + OFF_MISC);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + OFF_MISC + 4);
  unsigned long long *valid_s = reinterpret_cast<unsigned long long *>(smem + OFF_MISC + 8);  // [2]
  unsigned long long *memb_s = reinterpret_cast<unsigned long long *>(smem + OFF_MEMB);       // [2][BK]

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
  // Keys this CTA walks: the query's selection, or the pack's union.
  const int nkeys = PACKED ? a.ucount[item] : a.topk;
  const int32_t *keys = PACKED ? a.ukeys + static_cast<long long>(item) * a.umax
                               : a.topk_idx + static_cast<long long>(t) * a.topk;
  const unsigned long long *qmask = PACKED ? a.qmask + static_cast<long long>(item) * a.umax : nullptr;
  const int ntiles = max(1, (nkeys + BK - 1) / BK);
  // Output rows of the 64-row tile: global row out_row0 + r for r < row_limit.
  const long long out_row0 = static_cast<long long>(t) * a.H + (PACKED ? 0 : hg * HT);
  const int row_limit = PACKED ? nq * a.H : min(HT, a.H - hg * HT);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
    }
    mbar_init(p_full, 4);
    mbar_init(p_free, 1);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) prefetch_tensormap(&tmap_q);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const unsigned tmem = *tmem_slot;
  const unsigned o_lo = tmem;                          // lanes 0-15 of each quarter, cols 0-255
  const unsigned o_hi = tmem + (16u << 16);            // lanes 16-31 of each quarter, cols 0-255
  const unsigned s_col = tmem + 256;                   // S buffers: cols 256-319, 320-383

  if (warp == 0 || warp == 6) {
    // ------------------------------------------------------------ gather producers
    // Producer p owns stage p and fills tiles p, p + 2, p + 4, ...  Lane l moves
    // the 16-byte column chunk (l % 8) of rows 4g + l / 8 (g = 0..15) for all
    // 9 column atoms: every 8-lane group reads one whole 128-byte segment.
    const int p = warp == 0 ? 0 : 1;
    const int r = lane >> 3, c8 = lane & 7;
    bool ok = true;
    if (p == 0 && lane == 0) {
      mbar_arrive_expect_tx(q_full, Q_BYTES);
      const int row0 = t * a.H + hg * HT;
      for (int at = 0; at < ATOMS; ++at) tma_load_2d(q_s + at * ATOM_BYTES, &tmap_q, q_full, at * 64, row0);
    }
    auto load_idx = [&](int j, int (&v)[16]) {
#pragma unroll
      for (int g = 0; g < 16; ++g) {
        const int pos = j * BK + 4 * g + r;
        v[g] = (j < ntiles && pos < nkeys) ? keys[pos] : -1;
      }
    };
    const uint8_t *kv = static_cast<const uint8_t *>(a.kv);
    const unsigned stage_base = smem_u32(kv_s + p * KV_BYTES);
    // Packed mode: lane j < G also carries query j's 64-bit key mask of the tile.
    auto load_mask = [&](int j) -> unsigned long long {
      return (PACKED && lane < nq && j < ntiles) ? qmask[static_cast<long long>(j) * 64 + lane] : 0ull;
    };
    int cur[16], nxt[16];
    unsigned long long cur_m = 0ull, nxt_m = 0ull;
    load_idx(p, cur);
    cur_m = load_mask(p);
    for (int j = p; j < ntiles; j += 2) {
      load_idx(j + 2, nxt);
      nxt_m = load_mask(j + 2);
      if (!mbar_wait(&kv_empty[p], ((j >> 1) & 1) ^ 1u, abort_flag)) { ok = false; break; }
      unsigned long long vbits = 0;
      if (PACKED && lane < nq) memb_s[p * BK + lane] = cur_m;
#pragma unroll
      for (int g = 0; g < 16; ++g) {
        const int v = cur[g];
        const bool good = v >= 0 && v < a.N;
        if (c8 == 0 && (v >= a.N || v < -1)) atomicOr(a.status, DEV_BAD_INDEX);
        vbits |= static_cast<unsigned long long>(good ? 1u : 0u) << (4 * g + r);
        const int row = good ? v : 0;
        const int key = 4 * g + r;
        const uint8_t *src = kv + static_cast<long long>(row) * (DIM * 2) + c8 * 16;
        const unsigned dst = stage_base + key * 128 + ((c8 ^ (key & 7)) << 4);
#pragma unroll
        for (int at = 0; at < ATOMS; ++at) cp_async_16(dst + at * ATOM_BYTES, src + at * 128);
      }
      cp_async_wait_all();
      fence_proxy_async_smem();
      vbits |= __shfl_xor_sync(0xffffffffu, vbits, 8);
      vbits |= __shfl_xor_sync(0xffffffffu, vbits, 16);
      __syncwarp();
      if (lane == 0) {
        valid_s[p] = vbits;
        mbar_arrive(&kv_full[p]);
      }
#pragma unroll
      for (int g = 0; g < 16; ++g) cur[g] = nxt[g];
      cur_m = nxt_m;
    }
    cp_async_wait_all();  // never leave with copies in flight
    if (!ok) {
      if (lane == 0) atomicOr(a.status, DEV_TIMEOUT);
      *abort_flag = 1;
    }
    if (p == 0 && lane == 0 && !mbar_wait(q_full, 0u, nullptr)) atomicOr(a.status, DEV_TIMEOUT);
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    constexpr unsigned idesc_qk = make_idesc(HT, BK, 1u, 0u, 0u);   // S = Q K^T, both K-major
    constexpr unsigned idesc_pv = make_idesc(HT, 256, 1u, 0u, 1u);  // O += P V, V MN-major
    bool ok = mbar_wait(q_full, 0u, abort_flag);
    // Descriptors are built once; an operand offset is added to the start
    // address field (address >> 4; shared addresses stay below 2^18, so the
    // 14-bit field never carries).
    const uint64_t q_desc = smem_desc_sw128(smem_u32(q_s), 16, 1024);
    const uint64_t p_desc = smem_desc_sw128(smem_u32(p_s), 16, 1024);
    const uint64_t k_desc[2] = {smem_desc_sw128(smem_u32(kv_s), 16, 1024),
                                smem_desc_sw128(smem_u32(kv_s + KV_BYTES), 16, 1024)};
    const uint64_t v_desc[2] = {smem_desc_sw128(smem_u32(kv_s), ATOM_BYTES, 1024),
                                smem_desc_sw128(smem_u32(kv_s + KV_BYTES), ATOM_BYTES, 1024)};
    auto issue_pv = [&](int jj) {
      const uint64_t vd = v_desc[jj & 1];
#pragma unroll
      for (int ks = 0; ks < BK / 16; ++ks) {
        const unsigned acc = (jj > 0 || ks > 0) ? 1u : 0u;
        mma_bf16_ss(o_lo, p_desc + ((ks * 32) >> 4), vd + ((ks * 2048) >> 4), idesc_pv, acc);
        mma_bf16_ss(o_hi, p_desc + ((ks * 32) >> 4), vd + ((4 * ATOM_BYTES + ks * 2048) >> 4), idesc_pv, acc);
      }
      tc_commit(&kv_empty[jj & 1]);
      tc_commit(p_free);
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
        if (np < nq && mbar_try_wait(p_full, np & 1u))
          action = 1;
        else if (nq < ntiles && mbar_try_wait(&kv_full[nq & 1], (nq >> 1) & 1u) &&
                 mbar_try_wait(&s_free[nq & 1], ((nq >> 1) & 1u) ^ 1u))
          action = 2;
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
          const int st = nq & 1;
          const uint64_t kd = k_desc[st];
          const unsigned s_tmem = s_col + st * 64;
#pragma unroll
          for (int at = 0; at < ATOMS; ++at) {
#pragma unroll
            for (int ks = 0; ks < 4; ++ks) {
              const uint64_t off = static_cast<uint64_t>((at * ATOM_BYTES + ks * 32) >> 4);
              mma_bf16_ss(s_tmem, q_desc + off, kd + off, idesc_qk, (at | ks) ? 1u : 0u);
            }
          }
          tc_commit(&s_full[st]);
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
    // ------------------------------------------------------------ softmax + output
    const int quarter = warp & 3;
    const int r16 = lane & 15;
    const int row = quarter * 16 + r16;  // head within the CTA's group
    const unsigned lane_base = static_cast<unsigned>(quarter * 32) << 16;
    float m_used = -INFINITY, l = 0.0f, l_exact = 0.0f;  // l: sum of the bf16 P used; l_exact: fp32 sum for the LSE
    bool ok = true;
    const int c0 = (lane >> 4) * 32;  // this thread's 32 of the tile's 64 key columns
    for (int j = 0; j < ntiles; ++j) {
      const int sb = j & 1;
      if (!mbar_wait(&s_full[sb], (j >> 1) & 1u, abort_flag)) { ok = false; break; }
      tc_fence_after();
      uint32_t sv[32];
      tmem_ld_16x32bx2_x32(s_col + lane_base + sb * 64, sv);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[sb]);
      unsigned vbits;
      if (PACKED) {
        // keys of this tile that the row's own query chose
        const int qj = row / a.H;
        vbits = qj < nq ? static_cast<unsigned>(memb_s[(j & 1) * BK + qj] >> c0) : 0u;
      } else {
        vbits = static_cast<unsigned>(valid_s[j & 1] >> c0);
      }
      float z[32];
      float tmax = -INFINITY;
#pragma unroll
      for (int c = 0; c < 32; ++c) {
        z[c] = ((vbits >> c) & 1u) ? __uint_as_float(sv[c]) * a.scale_log2 : -INFINITY;
        tmax = fmaxf(tmax, z[c]);
      }
      tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));  // whole row (both halves)
      const float m_old = m_used;
      bool rescale = false;
      if (tmax > m_used + kRescaleLog2 || (m_used == -INFINITY && tmax > -INFINITY)) {
        rescale = (m_used != -INFINITY) && (j > 0);
        m_used = tmax;
      }
      // P in bf16, rounded once; the normaliser sums the rounded values.
      uint32_t pk[16];
      float tsum = 0.0f, tsum_exact = 0.0f;
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        const float p0 = (m_used == -INFINITY) ? 0.0f : fast_exp2(z[c] - m_used);
        const float p1 = (m_used == -INFINITY) ? 0.0f : fast_exp2(z[c + 1] - m_used);
        const __nv_bfloat162 b = __floats2bfloat162_rn(p0, p1);
        const float2 br = __bfloat1622float2(b);
        tsum += br.x + br.y;
        tsum_exact += p0 + p1;
        pk[c >> 1] = *reinterpret_cast<const uint32_t *>(&b);
      }
      tsum += __shfl_xor_sync(0xffffffffu, tsum, 16);
      tsum_exact += __shfl_xor_sync(0xffffffffu, tsum_exact, 16);
      const float alpha = rescale ? fast_exp2(m_old - m_used) : 1.0f;
      l = l * alpha + tsum;
      l_exact = l_exact * alpha + tsum_exact;
      if (j > 0) {
        if (!mbar_wait(p_free, (j - 1) & 1u, abort_flag)) { ok = false; break; }
        tc_fence_after();
      }
      // Rescale O when the running max moved: lanes 0-15 own the O_lo rows and
      // lanes 16-31 the O_hi rows of the same heads (same alpha).
      if (__any_sync(0xffffffffu, rescale)) {
        const unsigned obase = o_lo + lane_base;  // one 32x32b access: O_lo rows then O_hi rows
#pragma unroll 1
        for (int ch = 0; ch < 8; ++ch) {
          uint32_t ov[32];
          tmem_ld_32x32b_x32(obase + ch * 32, ov);
          tmem_ld_wait();
          if (rescale) {
#pragma unroll
            for (int e = 0; e < 32; ++e) ov[e] = __float_as_uint(__uint_as_float(ov[e]) * alpha);
          }
          tmem_st_32x32b_x32(obase + ch * 32, ov);
        }
        tmem_st_wait();
      }
      {
        uint8_t *prow = p_s + row * 128;
        const int cbase = c0 >> 3;  // first 16-byte chunk of this thread's 32 columns
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          const uint4 v = make_uint4(pk[ch * 4 + 0], pk[ch * 4 + 1], pk[ch * 4 + 2], pk[ch * 4 + 3]);
          *reinterpret_cast<uint4 *>(prow + (((cbase + ch) ^ (row & 7)) << 4)) = v;
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(p_full);
    }
    if (ok) ok = mbar_wait(p_free, (ntiles - 1) & 1u, abort_flag);
    if (!ok) {
      if (lane == 0) atomicOr(a.status, DEV_TIMEOUT);
      *abort_flag = 1;
    } else {
      tc_fence_after();
      const float inv = l > 0.0f ? 1.0f / l : 0.0f;  // both halves of a row hold the row's l
      const bool has_row = row < row_limit;
      const int dim0 = lane < 16 ? 0 : 256;
      uint16_t *orow = a.out + (out_row0 + row) * LAT + dim0;
#pragma unroll 1
      for (int ch = 0; ch < 8; ++ch) {
        uint32_t ov[32];
        tmem_ld_32x32b_x32(o_lo + lane_base + ch * 32, ov);
        tmem_ld_wait();
        if (has_row) {
          uint32_t pkd[16];
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const __nv_bfloat162 b =
                __floats2bfloat162_rn(__uint_as_float(ov[2 * e]) * inv, __uint_as_float(ov[2 * e + 1]) * inv);
            pkd[e] = *reinterpret_cast<const uint32_t *>(&b);
          }
          uint4 *dst = reinterpret_cast<uint4 *>(orow + ch * 32);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pkd[4 * e], pkd[4 * e + 1], pkd[4 * e + 2], pkd[4 * e + 3]);
        }
      }
      if (lane < 16 && has_row && a.lse != nullptr) {
        a.lse[out_row0 + row] =
            l_exact > 0.0f ? (m_used + log2f(l_exact)) * 0.69314718055994530942f : -INFINITY;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace mla

cudaError_t launch_sparse_mla(const CUtensorMap &tq, const MlaArgs &a, bool packed, cudaStream_t stream) {
  auto kern = packed ? mla::sparse_mla_kernel<true> : mla::sparse_mla_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, mla::SMEM_BYTES);
  if (e != cudaSuccess) return e;
  dim3 grid(packed ? (a.Lq + a.G - 1) / a.G : a.Lq, packed ? 1 : (a.H + mla::HT - 1) / mla::HT);
  kern<<<grid, mla::THREADS, mla::SMEM_BYTES, stream>>>(tq, a);
  return cudaGetLastError();
}

}  // namespace dsa
