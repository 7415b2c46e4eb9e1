// Causal GQA attention on the 5th-generation tensor cores (tcgen05), for head
// dim 128 and sequences of at most 512 positions (the 8B and 32B workloads of
// the streamed trainer).  Forward: one CTA per (128-query tile, query head,
// sequence).  Backward: a dQ kernel per query tile and a dK/dV kernel per key
// chunk (below), each the sole owner of its outputs (no atomics).
//
//   S_j = Q K_j^T              tcgen05, fp32 in TMEM, 128 columns per 128-key chunk j
//   P   = exp2(S*c - max)      exact two-pass softmax over the whole row (all of S
//                               fits TMEM: 4 chunks x 128 columns), P in bf16 in
//                               shared memory, 128-byte swizzled K-major
//   O   = sum_j P_j V_j         tcgen05 into TMEM columns 0-127 (chunk 0's scores
//                               are consumed before the first product lands)
//   o   = O / l, lse = (max + log2 l) / log2(e)
//
// Layouts as the mma.sync kernels: q, o [B, S, Hq, 128]; k, v [B, S, Hkv, 128];
// lse [B, Hq, S].  Query head h reads kv head h / (Hq / Hkv).  K and V arrive
// through a two-slot TMA ring (K chunks, then V chunks).  Warp 0: TMA; warp 1:
// TMEM owner and MMA issuer; warps 2-5: softmax and epilogue, one query row
// per thread (TMEM lane = row).  Every wait is bounded; no atomics.
#include "common.cuh"
#include "host_common.h"

namespace lsq {
namespace atc {

constexpr int D = 128;           // head dim
constexpr int BQ = 128;          // query rows per CTA
constexpr int BC = 128;          // keys per chunk
constexpr int MAXC = 4;          // chunks: sequences of at most 512
constexpr int TILE = BQ * D * 2; // 128 x 128 bf16 tile: two 64-column 128B-swizzled halves of 16 KB
constexpr int HALF = TILE / 2;
constexpr int OFF_Q = 0;
constexpr int OFF_RING = OFF_Q + TILE;
constexpr int OFF_P = OFF_RING + 2 * TILE;
constexpr int OFF_BAR = OFF_P + MAXC * TILE;
constexpr int NBAR = 1 + 2 + 2 + 1 + MAXC + 1;  // qfull, rfull[2], rempty[2], sfull, pready[4], ofull
constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
constexpr int NTHREADS = 192;
constexpr float LOG2E = 1.4426950408889634f;
static_assert(SMEM_BYTES <= 232448, "shared memory");

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// smem descriptor of a K-major operand tile (rows x 128 elements as two
// 64-element 128B-swizzled halves) at k-step kk (16 elements)
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t base, int kk) {
  return smem_desc(base + (kk >> 2) * HALF + (kk & 3) * 32, 16, 1024, 2);
}

__global__ void __launch_bounds__(NTHREADS, 1) attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                                                                  const __grid_constant__ CUtensorMap kmap,
                                                                  const __grid_constant__ CUtensorMap vmap,
                                                                  __nv_bfloat16* __restrict__ o,
                                                                  float* __restrict__ lse, int S, int Hq, int Hkv,
                                                                  float scale_log2) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* qfull = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* rfull = qfull + 1;
  uint64_t* rempty = rfull + 2;
  uint64_t* sfull = rempty + 2;
  uint64_t* pready = sfull + 1;
  uint64_t* ofull = pready + MAXC;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + OFF_MISC);

  const int nt = (S + BQ - 1) / BQ;
  const int t = nt - 1 - (int)blockIdx.x;  // longest causal tiles first
  const int h = blockIdx.y, b = blockIdx.z;
  const int hk = h / (Hq / Hkv);
  const int q0 = t * BQ;
  const int nc = t + 1;  // key chunks at or before this query tile
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(qfull, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&rfull[i], 1);
      mbar_init(&rempty[i], 1);
    }
    mbar_init(sfull, 1);
    for (int j = 0; j < MAXC; ++j) mbar_init(&pready[j], 4);  // one arrival per softmax warp
    mbar_init(ofull, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 0) {
    if (lane == 0) {
      const int row0 = b * S;
      mbar_arrive_expect_tx(qfull, (uint32_t)TILE);
      tma_load_2d(smem + OFF_Q, &qmap, qfull, h * D, row0 + q0);
      tma_load_2d(smem + OFF_Q + HALF, &qmap, qfull, h * D + 64, row0 + q0);
      for (int it = 0; it < 2 * nc; ++it) {  // K chunks 0..nc-1, then V chunks 0..nc-1
        const int slot = it & 1;
        const uint32_t ph = (uint32_t)(it >> 1) & 1u;
        if (!mbar_wait(&rempty[slot], ph ^ 1u, 461)) break;
        const int j = it < nc ? it : it - nc;
        const CUtensorMap* m = it < nc ? &kmap : &vmap;
        uint8_t* dst = smem + OFF_RING + slot * TILE;
        mbar_arrive_expect_tx(&rfull[slot], (uint32_t)TILE);
        tma_load_2d(dst, m, &rfull[slot], hk * D, row0 + j * BC);
        tma_load_2d(dst + HALF, m, &rfull[slot], hk * D + 64, row0 + j * BC);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = mbar_wait(qfull, 0, 561);
      if (ok) tc_fence_after();
      const uint32_t qb = smem_u32(smem + OFF_Q);
      const uint32_t id_s = idesc_bf16(BQ, BC, 0, 0);  // Q K^T: both K-major
      const uint32_t id_o = idesc_bf16(BQ, D, 0, 1);   // P V: P K-major, V MN-major
      for (int j = 0; ok && j < nc; ++j) {
        const int slot = j & 1;
        if (!mbar_wait(&rfull[slot], (uint32_t)(j >> 1) & 1u, 562)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t kb = smem_u32(smem + OFF_RING + slot * TILE);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          tc_mma(tmem + (uint32_t)(j * BC), desc_kmajor(qb, kk), desc_kmajor(kb, kk), id_s, kk != 0);
        tc_commit(&rempty[slot]);
      }
      if (ok) tc_commit(sfull);
      for (int j = 0; ok && j < nc; ++j) {
        const int it = nc + j, slot = it & 1;
        if (!mbar_wait(&rfull[slot], (uint32_t)(it >> 1) & 1u, 563) || !mbar_wait(&pready[j], 0, 564)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t pb = smem_u32(smem + OFF_P + j * TILE);
        const uint32_t vb = smem_u32(smem + OFF_RING + slot * TILE);
#pragma unroll
        for (int kk = 0; kk < BC / 16; ++kk)
          tc_mma(tmem, desc_kmajor(pb, kk), smem_desc(vb + kk * 2048, HALF, 1024, 2), id_o, (j | kk) != 0);
        tc_commit(&rempty[slot]);
      }
      tc_commit(ofull);  // also drains what was issued if a wait gave up
      if (!ok) mbar_wait(ofull, 0, 565);
    }
  } else {
    // softmax and epilogue: one query row per thread
    const int qd = warp & 3;
    const int r = qd * 32 + lane;
    const int qi = q0 + r;
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
    bool ok = __all_sync(0xffffffffu, mbar_wait(sfull, 0, 761));
    float m = -INFINITY, l = 0.0f;
    if (ok) {
      tc_fence_after();
      for (int j = 0; j < nc; ++j) {
        for (int c4 = 0; c4 < BC / 32; ++c4) {
          float v[32];
          tmem_ld32(tmem + lane_base + (uint32_t)(j * BC + c4 * 32), v);
          tc_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int kj = j * BC + c4 * 32 + e;
            if (kj <= qi && kj < S) m = fmaxf(m, v[e] * scale_log2);
          }
        }
      }
      for (int j = 0; j < nc; ++j) {
        const uint32_t pbase = smem_u32(smem + OFF_P + j * TILE) + r * 128;
        for (int c4 = 0; c4 < BC / 32; ++c4) {
          float v[32];
          tmem_ld32(tmem + lane_base + (uint32_t)(j * BC + c4 * 32), v);
          tc_wait_ld();
          uint32_t w[16];
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            const int kj = j * BC + c4 * 32 + e;
            const float p0 = (kj <= qi && kj < S) ? exp2f(v[e] * scale_log2 - m) : 0.0f;
            const float p1 = (kj + 1 <= qi && kj + 1 < S) ? exp2f(v[e + 1] * scale_log2 - m) : 0.0f;
            l += p0 + p1;
            w[e / 2] = pack_bf16x2(p0, p1);
          }
          // keys c4*32 .. +31 of this chunk: half c4 >> 1, 16-byte units (c4 & 1) * 4 .. + 3
          const uint32_t hbase = pbase + (uint32_t)(c4 >> 1) * HALF;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int unit = (c4 & 1) * 4 + u;
            st_shared_v4(hbase + ((uint32_t)(unit ^ (r & 7)) << 4), w[4 * u], w[4 * u + 1], w[4 * u + 2],
                         w[4 * u + 3]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&pready[j]);
      }
      ok = __all_sync(0xffffffffu, mbar_wait(ofull, 0, 762));
    }
    if (ok) {
      tc_fence_after();
      const float inv = 1.0f / l;
      __nv_bfloat16* orow = o + (((int64_t)b * S + qi) * Hq + h) * D;
      for (int c4 = 0; c4 < D / 32; ++c4) {
        float v[32];
        tmem_ld32(tmem + lane_base + (uint32_t)(c4 * 32), v);
        tc_wait_ld();
        if (qi < S) {
#pragma unroll
          for (int u = 0; u < 4; ++u)
            *reinterpret_cast<uint4*>(orow + c4 * 32 + u * 8) =
                make_uint4(pack_bf16x2(v[8 * u] * inv, v[8 * u + 1] * inv),
                           pack_bf16x2(v[8 * u + 2] * inv, v[8 * u + 3] * inv),
                           pack_bf16x2(v[8 * u + 4] * inv, v[8 * u + 5] * inv),
                           pack_bf16x2(v[8 * u + 6] * inv, v[8 * u + 7] * inv));
        }
      }
      if (qi < S) lse[((int64_t)b * Hq + h) * S + qi] = (m + log2f(l)) / LOG2E;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ================================================================ backward
// dQ: one CTA per (128-query tile, query head, sequence); per key chunk j <= tile:
//   S = Q K_j^T, dP = dO V_j^T (TMEM), dS = P (dP - Dvec) in bf16 (shared
//   memory, K-major), dQ += dS K_j (TMEM); dq = dQ / sqrt(D).
constexpr int Q_OFF_Q = 0;
constexpr int Q_OFF_DO = Q_OFF_Q + TILE;
constexpr int Q_OFF_RING = Q_OFF_DO + TILE;  // 2 slots of [K_j | V_j]
constexpr int Q_OFF_DS = Q_OFF_RING + 4 * TILE;
constexpr int Q_OFF_BAR = Q_OFF_DS + TILE;
constexpr int Q_NBAR = 1 + 2 + 2 + 1 + 1 + 1 + 1;  // qfull, rfull[2], rempty[2], sfull, dsready, dsfree, dqfull
constexpr int Q_OFF_MISC = Q_OFF_BAR + 8 * Q_NBAR;
constexpr int Q_SMEM = Q_OFF_MISC + 16 + 1024;
static_assert(Q_SMEM <= 232448, "shared memory");

__global__ void __launch_bounds__(NTHREADS, 1) attn_dq_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                                                                 const __grid_constant__ CUtensorMap kmap,
                                                                 const __grid_constant__ CUtensorMap vmap,
                                                                 const __grid_constant__ CUtensorMap domap,
                                                                 const float* __restrict__ lse,
                                                                 const float* __restrict__ dvec,
                                                                 __nv_bfloat16* __restrict__ dq, int S, int Hq,
                                                                 int Hkv, float scale, float scale_log2) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* qfull = reinterpret_cast<uint64_t*>(smem + Q_OFF_BAR);
  uint64_t* rfull = qfull + 1;
  uint64_t* rempty = rfull + 2;
  uint64_t* sfull = rempty + 2;
  uint64_t* dsready = sfull + 1;
  uint64_t* dsfree = dsready + 1;
  uint64_t* dqfull = dsfree + 1;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + Q_OFF_MISC);

  const int nt = (S + BQ - 1) / BQ;
  const int t = nt - 1 - (int)blockIdx.x;
  const int h = blockIdx.y, b = blockIdx.z;
  const int hk = h / (Hq / Hkv);
  const int q0 = t * BQ;
  const int nc = t + 1;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr uint32_t T_S = 0, T_DP = 128, T_DQ = 256;

  if (threadIdx.x == 0) {
    mbar_init(qfull, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&rfull[i], 1);
      mbar_init(&rempty[i], 1);
    }
    mbar_init(sfull, 1);
    mbar_init(dsready, 4);
    mbar_init(dsfree, 1);
    mbar_init(dqfull, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 0) {
    if (lane == 0) {
      const int row0 = b * S;
      mbar_arrive_expect_tx(qfull, 2u * TILE);
      tma_load_2d(smem + Q_OFF_Q, &qmap, qfull, h * D, row0 + q0);
      tma_load_2d(smem + Q_OFF_Q + HALF, &qmap, qfull, h * D + 64, row0 + q0);
      tma_load_2d(smem + Q_OFF_DO, &domap, qfull, h * D, row0 + q0);
      tma_load_2d(smem + Q_OFF_DO + HALF, &domap, qfull, h * D + 64, row0 + q0);
      for (int j = 0; j < nc; ++j) {
        const int slot = j & 1;
        if (!mbar_wait(&rempty[slot], ((uint32_t)(j >> 1) & 1u) ^ 1u, 471)) break;
        uint8_t* dst = smem + Q_OFF_RING + slot * 2 * TILE;
        mbar_arrive_expect_tx(&rfull[slot], 2u * TILE);
        tma_load_2d(dst, &kmap, &rfull[slot], hk * D, row0 + j * BC);
        tma_load_2d(dst + HALF, &kmap, &rfull[slot], hk * D + 64, row0 + j * BC);
        tma_load_2d(dst + TILE, &vmap, &rfull[slot], hk * D, row0 + j * BC);
        tma_load_2d(dst + TILE + HALF, &vmap, &rfull[slot], hk * D + 64, row0 + j * BC);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = mbar_wait(qfull, 0, 571);
      const uint32_t qb = smem_u32(smem + Q_OFF_Q), dob = smem_u32(smem + Q_OFF_DO);
      const uint32_t dsb = smem_u32(smem + Q_OFF_DS);
      const uint32_t id_k = idesc_bf16(BQ, BC, 0, 0);  // S, dP: both operands K-major
      const uint32_t id_q = idesc_bf16(BQ, D, 0, 1);   // dS K: K MN-major
      for (int j = 0; ok && j < nc; ++j) {
        const int slot = j & 1;
        if (!mbar_wait(&rfull[slot], (uint32_t)(j >> 1) & 1u, 572)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t kb = smem_u32(smem + Q_OFF_RING + slot * 2 * TILE), vb = kb + TILE;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          tc_mma(tmem + T_S, desc_kmajor(qb, kk), desc_kmajor(kb, kk), id_k, kk != 0);
          tc_mma(tmem + T_DP, desc_kmajor(dob, kk), desc_kmajor(vb, kk), id_k, kk != 0);
        }
        tc_commit(sfull);
        if (!mbar_wait(dsready, (uint32_t)j & 1u, 573)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BC / 16; ++kk)
          tc_mma(tmem + T_DQ, desc_kmajor(dsb, kk), smem_desc(kb + kk * 2048, HALF, 1024, 2), id_q, (j | kk) != 0);
        tc_commit(dsfree);
        tc_commit(&rempty[slot]);
      }
      tc_commit(dqfull);
      if (!ok) mbar_wait(dqfull, 0, 574);
    }
  } else {
    const int qd = warp & 3;
    const int r = qd * 32 + lane;
    const int qi = q0 + r;
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
    const int64_t ri = ((int64_t)b * Hq + h) * S + (qi < S ? qi : 0);
    const float lse2 = lse[ri] * LOG2E, dv = dvec[ri];
    bool ok = true;
    for (int j = 0; ok && j < nc; ++j) {
      if (!__all_sync(0xffffffffu, mbar_wait(sfull, (uint32_t)j & 1u, 771))) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (j > 0 && !__all_sync(0xffffffffu, mbar_wait(dsfree, (uint32_t)(j - 1) & 1u, 772))) {
        ok = false;
        break;
      }
      const uint32_t rbase = smem_u32(smem + Q_OFF_DS) + r * 128;
      for (int c4 = 0; c4 < BC / 32; ++c4) {
        float sv[32], pv[32];
        tmem_ld32(tmem + lane_base + T_S + (uint32_t)(c4 * 32), sv);
        tmem_ld32(tmem + lane_base + T_DP + (uint32_t)(c4 * 32), pv);
        tc_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int kj = j * BC + c4 * 32 + e;
          const bool ok0 = kj <= qi && kj < S && qi < S, ok1 = kj + 1 <= qi && kj + 1 < S && qi < S;
          const float p0 = ok0 ? exp2f(sv[e] * scale_log2 - lse2) : 0.0f;
          const float p1 = ok1 ? exp2f(sv[e + 1] * scale_log2 - lse2) : 0.0f;
          w[e / 2] = pack_bf16x2(p0 * (pv[e] - dv), p1 * (pv[e + 1] - dv));
        }
        const uint32_t hbase = rbase + (uint32_t)(c4 >> 1) * HALF;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int unit = (c4 & 1) * 4 + u;
          st_shared_v4(hbase + ((uint32_t)(unit ^ (r & 7)) << 4), w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(dsready);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(dqfull, 0, 773))) {
      tc_fence_after();
      __nv_bfloat16* row = dq + (((int64_t)b * S + qi) * Hq + h) * D;
      for (int c4 = 0; c4 < D / 32; ++c4) {
        float v[32];
        tmem_ld32(tmem + lane_base + T_DQ + (uint32_t)(c4 * 32), v);
        tc_wait_ld();
        if (qi < S) {
#pragma unroll
          for (int u = 0; u < 4; ++u)
            *reinterpret_cast<uint4*>(row + c4 * 32 + u * 8) =
                make_uint4(pack_bf16x2(v[8 * u] * scale, v[8 * u + 1] * scale),
                           pack_bf16x2(v[8 * u + 2] * scale, v[8 * u + 3] * scale),
                           pack_bf16x2(v[8 * u + 4] * scale, v[8 * u + 5] * scale),
                           pack_bf16x2(v[8 * u + 6] * scale, v[8 * u + 7] * scale));
        }
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

// dK, dV: one CTA per (128-key chunk, kv head, sequence); loops over the group's
// query heads and the 128-query tiles at or after the chunk:
//   S^T = K Q_i^T, dP^T = V dO_i^T (TMEM), P^T and dS^T = P^T (dP^T - Dvec) in
//   bf16 (shared memory), dV += P^T dO_i, dK += dS^T Q_i (TMEM);
//   dk = dK / sqrt(D), dv = dV.
constexpr int K_OFF_K = 0;
constexpr int K_OFF_V = K_OFF_K + TILE;
constexpr int K_OFF_Q = K_OFF_V + TILE;
constexpr int K_OFF_DO = K_OFF_Q + TILE;
constexpr int K_OFF_P = K_OFF_DO + TILE;
constexpr int K_OFF_DS = K_OFF_P + TILE;
constexpr int K_OFF_BAR = K_OFF_DS + TILE;
constexpr int K_NBAR = 1 + 1 + 1 + 1 + 1 + 1;  // kvfull, qfull, qempty, sfull, psready, done
constexpr int K_OFF_MISC = K_OFF_BAR + 8 * K_NBAR;
constexpr int K_SMEM = K_OFF_MISC + 16 + 1024;
static_assert(K_SMEM <= 232448, "shared memory");

__global__ void __launch_bounds__(NTHREADS, 1) attn_dkv_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                                                                  const __grid_constant__ CUtensorMap kmap,
                                                                  const __grid_constant__ CUtensorMap vmap,
                                                                  const __grid_constant__ CUtensorMap domap,
                                                                  const float* __restrict__ lse,
                                                                  const float* __restrict__ dvec,
                                                                  __nv_bfloat16* __restrict__ dk,
                                                                  __nv_bfloat16* __restrict__ dv_out, int S, int Hq,
                                                                  int Hkv, float scale, float scale_log2) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* kvfull = reinterpret_cast<uint64_t*>(smem + K_OFF_BAR);
  uint64_t* qfull = kvfull + 1;
  uint64_t* qempty = qfull + 1;
  uint64_t* sfull = qempty + 1;
  uint64_t* psready = sfull + 1;
  uint64_t* done = psready + 1;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + K_OFF_MISC);

  const int nt = (S + BQ - 1) / BQ;
  const int jc = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int group = Hq / Hkv;
  const int k0 = jc * BC;
  const int nq = nt - jc;            // query tiles at or after the chunk
  const int items = group * nq;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr uint32_t T_S = 0, T_DP = 128, T_DV = 256, T_DK = 384;

  if (threadIdx.x == 0) {
    mbar_init(kvfull, 1);
    mbar_init(qfull, 1);
    mbar_init(qempty, 1);
    mbar_init(sfull, 1);
    mbar_init(psready, 4);
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 0) {
    if (lane == 0) {
      const int row0 = b * S;
      mbar_arrive_expect_tx(kvfull, 2u * TILE);
      tma_load_2d(smem + K_OFF_K, &kmap, kvfull, hk * D, row0 + k0);
      tma_load_2d(smem + K_OFF_K + HALF, &kmap, kvfull, hk * D + 64, row0 + k0);
      tma_load_2d(smem + K_OFF_V, &vmap, kvfull, hk * D, row0 + k0);
      tma_load_2d(smem + K_OFF_V + HALF, &vmap, kvfull, hk * D + 64, row0 + k0);
      for (int it = 0; it < items; ++it) {
        if (!mbar_wait(qempty, ((uint32_t)it & 1u) ^ 1u, 481)) break;
        const int h = hk * group + it / nq, qs = k0 + (it % nq) * BQ;
        mbar_arrive_expect_tx(qfull, 2u * TILE);
        tma_load_2d(smem + K_OFF_Q, &qmap, qfull, h * D, row0 + qs);
        tma_load_2d(smem + K_OFF_Q + HALF, &qmap, qfull, h * D + 64, row0 + qs);
        tma_load_2d(smem + K_OFF_DO, &domap, qfull, h * D, row0 + qs);
        tma_load_2d(smem + K_OFF_DO + HALF, &domap, qfull, h * D + 64, row0 + qs);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = mbar_wait(kvfull, 0, 581);
      const uint32_t kb = smem_u32(smem + K_OFF_K), vb = smem_u32(smem + K_OFF_V);
      const uint32_t qb = smem_u32(smem + K_OFF_Q), dob = smem_u32(smem + K_OFF_DO);
      const uint32_t pb = smem_u32(smem + K_OFF_P), dsb = smem_u32(smem + K_OFF_DS);
      const uint32_t id_k = idesc_bf16(BC, BQ, 0, 0);  // S^T, dP^T: both K-major
      const uint32_t id_m = idesc_bf16(BC, D, 0, 1);   // P^T dO, dS^T Q: dO / Q MN-major
      for (int it = 0; ok && it < items; ++it) {
        if (!mbar_wait(qfull, (uint32_t)it & 1u, 582)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          tc_mma(tmem + T_S, desc_kmajor(kb, kk), desc_kmajor(qb, kk), id_k, kk != 0);
          tc_mma(tmem + T_DP, desc_kmajor(vb, kk), desc_kmajor(dob, kk), id_k, kk != 0);
        }
        tc_commit(sfull);
        if (!mbar_wait(psready, (uint32_t)it & 1u, 583)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < BQ / 16; ++kk) {
          tc_mma(tmem + T_DV, desc_kmajor(pb, kk), smem_desc(dob + kk * 2048, HALF, 1024, 2), id_m, (it | kk) != 0);
          tc_mma(tmem + T_DK, desc_kmajor(dsb, kk), smem_desc(qb + kk * 2048, HALF, 1024, 2), id_m, (it | kk) != 0);
        }
        tc_commit(qempty);
      }
      tc_commit(done);
      if (!ok) mbar_wait(done, 0, 584);
    }
  } else {
    const int qd = warp & 3;
    const int r = qd * 32 + lane;  // key row of the chunk
    const int kj = k0 + r;
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
    bool ok = true;
    for (int it = 0; ok && it < items; ++it) {
      const int h = hk * group + it / nq, qs = k0 + (it % nq) * BQ;
      if (!__all_sync(0xffffffffu, mbar_wait(sfull, (uint32_t)it & 1u, 781))) {
        ok = false;
        break;
      }
      tc_fence_after();
      // the previous item's P^T / dS^T (and lse2 / Dvec rows) are free once its dV / dK products are done
      if (it > 0 && !__all_sync(0xffffffffu, mbar_wait(qempty, (uint32_t)(it - 1) & 1u, 782))) {
        ok = false;
        break;
      }
      const uint32_t prow = smem_u32(smem + K_OFF_P) + r * 128, drow = smem_u32(smem + K_OFF_DS) + r * 128;
      for (int c4 = 0; c4 < BQ / 32; ++c4) {
        float sv[32], pv[32];
        tmem_ld32(tmem + lane_base + T_S + (uint32_t)(c4 * 32), sv);
        tmem_ld32(tmem + lane_base + T_DP + (uint32_t)(c4 * 32), pv);
        // lse and Dvec of these 32 queries: lane l loads query l, shuffles broadcast
        const int qown = qs + c4 * 32 + lane;
        const int64_t rown = ((int64_t)b * Hq + h) * S + (qown < S ? qown : 0);
        const float l2own = lse[rown] * LOG2E, dvown = dvec[rown];
        tc_wait_ld();
        uint32_t wp[16], wd[16];
#pragma unroll
        for (int e = 0; e < 32; e += 2) {
          const int qi = qs + c4 * 32 + e;
          const float l20 = __shfl_sync(0xffffffffu, l2own, e), l21 = __shfl_sync(0xffffffffu, l2own, e + 1);
          const float d0 = __shfl_sync(0xffffffffu, dvown, e), d1 = __shfl_sync(0xffffffffu, dvown, e + 1);
          const bool ok0 = kj <= qi && qi < S && kj < S, ok1 = kj <= qi + 1 && qi + 1 < S && kj < S;
          const float p0 = ok0 ? exp2f(sv[e] * scale_log2 - l20) : 0.0f;
          const float p1 = ok1 ? exp2f(sv[e + 1] * scale_log2 - l21) : 0.0f;
          wp[e / 2] = pack_bf16x2(p0, p1);
          wd[e / 2] = pack_bf16x2(p0 * (pv[e] - d0), p1 * (pv[e + 1] - d1));
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const uint32_t off = (uint32_t)(c4 >> 1) * HALF + ((uint32_t)(((c4 & 1) * 4 + u) ^ (r & 7)) << 4);
          st_shared_v4(prow + off, wp[4 * u], wp[4 * u + 1], wp[4 * u + 2], wp[4 * u + 3]);
          st_shared_v4(drow + off, wd[4 * u], wd[4 * u + 1], wd[4 * u + 2], wd[4 * u + 3]);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(psready);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(done, 0, 783))) {
      tc_fence_after();
      const int64_t off = (((int64_t)b * S + kj) * Hkv + hk) * D;
      for (int c4 = 0; c4 < D / 32; ++c4) {
        float a[32], c[32];
        tmem_ld32(tmem + lane_base + T_DK + (uint32_t)(c4 * 32), a);
        tmem_ld32(tmem + lane_base + T_DV + (uint32_t)(c4 * 32), c);
        tc_wait_ld();
        if (kj < S) {
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            *reinterpret_cast<uint4*>(dk + off + c4 * 32 + u * 8) =
                make_uint4(pack_bf16x2(a[8 * u] * scale, a[8 * u + 1] * scale),
                           pack_bf16x2(a[8 * u + 2] * scale, a[8 * u + 3] * scale),
                           pack_bf16x2(a[8 * u + 4] * scale, a[8 * u + 5] * scale),
                           pack_bf16x2(a[8 * u + 6] * scale, a[8 * u + 7] * scale));
            *reinterpret_cast<uint4*>(dv_out + off + c4 * 32 + u * 8) =
                make_uint4(pack_bf16x2(c[8 * u], c[8 * u + 1]), pack_bf16x2(c[8 * u + 2], c[8 * u + 3]),
                           pack_bf16x2(c[8 * u + 4], c[8 * u + 5]), pack_bf16x2(c[8 * u + 6], c[8 * u + 7]));
          }
        }
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

static lsq_status tmap_heads(CUtensorMap* m, const void* base, int64_t rows, int64_t heads) {
  return encode_tmap_2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, (uint64_t)(heads * D), (uint64_t)rows,
                        (uint64_t)(heads * D * 2), 64, BQ, CU_TENSOR_MAP_SWIZZLE_128B);
}

// true when the tcgen05 path serves this shape
bool fwd_supported(int64_t S, int64_t hd) { return hd == D && S >= 1 && S <= MAXC * BC; }

lsq_status run_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int S, int Hq, int Hkv,
                   cudaStream_t st) {
  static int cfg[64];
  int dev = 0;
  LSQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev >= 0 && dev < 64 && !cfg[dev]) {
    LSQ_CUDA_TRY(cudaFuncSetAttribute(attn_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES));
    cfg[dev] = 1;
  }
  CUtensorMap qm, km, vm;
  lsq_status s;
  const int64_t rows = (int64_t)B * S;
  if ((s = tmap_heads(&qm, q, rows, Hq)) != LSQ_OK) return s;
  if ((s = tmap_heads(&km, k, rows, Hkv)) != LSQ_OK) return s;
  if ((s = tmap_heads(&vm, v, rows, Hkv)) != LSQ_OK) return s;
  const float sl = LOG2E / sqrtf((float)D);
  attn_fwd_tc_kernel<<<dim3((S + BQ - 1) / BQ, Hq, B), NTHREADS, SMEM_BYTES, st>>>(
      qm, km, vm, static_cast<__nv_bfloat16*>(o), lse, S, Hq, Hkv, sl);
  LSQ_LAUNCH_CHECK("attn_fwd_tc_kernel");
  return LSQ_OK;
}

bool bwd_supported(int64_t S, int64_t hd) { return fwd_supported(S, hd); }

lsq_status run_bwd(const void* q, const void* k, const void* v, const void* d_o, const float* lse, const float* dvec,
                   void* dq, void* dk, void* dv, int B, int S, int Hq, int Hkv, cudaStream_t st) {
  static int cfg[64];
  int dev = 0;
  LSQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev >= 0 && dev < 64 && !cfg[dev]) {
    LSQ_CUDA_TRY(cudaFuncSetAttribute(attn_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Q_SMEM));
    LSQ_CUDA_TRY(cudaFuncSetAttribute(attn_dkv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, K_SMEM));
    cfg[dev] = 1;
  }
  CUtensorMap qm, km, vm, dom;
  lsq_status s;
  const int64_t rows = (int64_t)B * S;
  if ((s = tmap_heads(&qm, q, rows, Hq)) != LSQ_OK) return s;
  if ((s = tmap_heads(&km, k, rows, Hkv)) != LSQ_OK) return s;
  if ((s = tmap_heads(&vm, v, rows, Hkv)) != LSQ_OK) return s;
  if ((s = tmap_heads(&dom, d_o, rows, Hq)) != LSQ_OK) return s;
  const float scale = 1.0f / sqrtf((float)D), sl = LOG2E * scale;
  const int nt = (S + BQ - 1) / BQ;
  attn_dq_tc_kernel<<<dim3(nt, Hq, B), NTHREADS, Q_SMEM, st>>>(qm, km, vm, dom, lse, dvec,
                                                               static_cast<__nv_bfloat16*>(dq), S, Hq, Hkv, scale, sl);
  LSQ_LAUNCH_CHECK("attn_dq_tc_kernel");
  attn_dkv_tc_kernel<<<dim3(nt, Hkv, B), NTHREADS, K_SMEM, st>>>(qm, km, vm, dom, lse, dvec,
                                                                 static_cast<__nv_bfloat16*>(dk),
                                                                 static_cast<__nv_bfloat16*>(dv), S, Hq, Hkv, scale,
                                                                 sl);
  LSQ_LAUNCH_CHECK("attn_dkv_tc_kernel");
  return LSQ_OK;
}

}  // namespace atc
}  // namespace lsq
