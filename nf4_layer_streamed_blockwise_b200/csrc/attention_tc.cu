// Causal GQA attention on the 5th-generation tensor cores (tcgen05), for head
// dim 128 and sequences of at most 512 positions (the 8B and 32B workloads of
// the streamed trainer).  Forward: one CTA per (query head, sequence, 128-query
// tile), two per SM, online softmax over 64-key chunks (below).  Backward: a
// dQ kernel per query tile and a dK/dV kernel per key chunk (with a GQA group
// of two or more, a two-CTA cluster per chunk), each the sole owner of its
// outputs (no atomics).  Every grid puts the causal tile index slowest and
// reversed, so the longest tiles of all heads start first.
//
// Layouts as the mma.sync kernels: q, o [B, S, Hq, 128]; k, v [B, S, Hkv, 128];
// lse [B, Hq, S].  Query head h reads kv head h / (Hq / Hkv).  Operands are
// staged by TMA with the 128-byte swizzle; every wait is bounded.
#include "common.cuh"
#include "host_common.h"

namespace lsq {
namespace atc {

constexpr int D = 128;           // head dim
constexpr int BQ = 128;          // query rows per CTA
constexpr int BC = 128;          // keys per backward chunk
constexpr int MAXC = 4;          // 128-key chunks: sequences of at most 512
constexpr int TILE = BQ * D * 2; // 128 x 128 bf16 tile: two 64-column 128B-swizzled halves of 16 KB
constexpr int HALF = TILE / 2;
constexpr float LOG2E = 1.4426950408889634f;
constexpr int EW = 16;                     // backward element-wise warps: four per TMEM lane quarter

constexpr int SUB = 64;                     // keys per forward chunk, rows per backward sub-item
constexpr int ST = SUB * D * 2;             // 64 x 128 bf16 tile: two 64-column halves of 8 KB
constexpr int SHALF = ST / 2;
constexpr int PT = BC * SUB * 2;            // 128 x 64 bf16 operand (one 128-byte swizzled column block)

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

// 2^x in one special-function instruction (relative error about 2^-22, far
// below the bf16 rounding of the probabilities); 0 for very negative x
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// smem descriptor of a K-major operand tile (rows x 128 elements as two
// 64-element 128B-swizzled halves) at k-step kk (16 elements)
__device__ __forceinline__ uint64_t desc_kmajor(uint32_t base, int kk) {
  return smem_desc(base + (kk >> 2) * HALF + (kk & 3) * 32, 16, 1024, 2);
}
// K-major 128-row x 64-element operand at k-step kk (16 elements)
__device__ __forceinline__ uint64_t desc_k64(uint32_t base, int kk) { return smem_desc(base + kk * 32, 16, 1024, 2); }
// K-major 64-row x 128-element operand (two 64-element halves of 8 KB) at k-step kk
__device__ __forceinline__ uint64_t desc_sub_kmajor(uint32_t base, int kk) {
  return smem_desc(base + (kk >> 2) * SHALF + (kk & 3) * 32, 16, 1024, 2);
}
// MN-major 64-row (K) x 128-column (N) operand: N halves 8 KB apart, 16 rows per k-step
__device__ __forceinline__ uint64_t desc_sub_mnmajor(uint32_t base, int kk) {
  return smem_desc(base + kk * 2048, SHALF, 1024, 2);
}

// ================================================================ forward
// One CTA per (query head, sequence, 128-query tile), two CTAs per SM: while
// one CTA's softmax warps turn scores into probabilities, the other's products
// run on the tensor core.  Online softmax over 64-key chunks j:
//
//   S_j = Q K_j^T                 tcgen05 into one of two 64-column score buffers
//   m   = running row max          (scaled to log2 units); kept while a chunk's
//                                  max exceeds it by at most 8, so P_j <= 2^8 and
//                                  O is rescaled only when the max jumps further
//   P_j = exp2(S_j c - m)         bf16, written over K_j in its ring slot (the
//                                  score product has read it)
//   O  += P_j V_j                  tcgen05 into TMEM columns 0-127; l += rowsum P_j
//   o   = O / l, lse = (m + log2 l) / log2(e)
//
// TMEM: O in columns 0-127, the score buffers in 128-191 and 192-255 (256 of
// the SM's 512 per CTA).  Shared memory: Q (32 KB) and a five-slot ring of
// 64-row K / V tiles (16 KB each), about 113 KB.  Warp 0: TMA (Q, then K_0, K_1,
// and per chunk j: V_j, K_{j+2}, the order the products consume them); warp 1:
// TMEM owner and MMA issuer (S_0, S_1, then per chunk: P_j V_j, S_{j+2}); warps
// 2-5: softmax and epilogue, one query row per thread (TMEM lane = row).  Every
// wait is bounded; no atomics.
constexpr int FR = 5;                             // ring slots
constexpr int F_OFF_Q = 0;
constexpr int F_OFF_RING = F_OFF_Q + TILE;
constexpr int F_OFF_BAR = F_OFF_RING + FR * ST;
// qfull, rfull[FR], rempty[FR], sfull[2], pready[2], pvdone, drain
constexpr int F_NBAR = 1 + 2 * FR + 2 + 2 + 1 + 1;
constexpr int F_OFF_MISC = F_OFF_BAR + 8 * F_NBAR;
constexpr int SMEM_BYTES = F_OFF_MISC + 16;
constexpr int FWD_THREADS = 32 * 6;
constexpr uint32_t F_T_O = 0, F_T_S = 128;       // TMEM columns
constexpr float RESCALE_LOG2 = 8.0f;              // P_j <= 2^8 between rescales
// two CTAs per SM: 228 KB of shared memory, 1 KB of it reserved per CTA.  The tiles need 1024-byte
// alignment for the 128-byte swizzle and there is no room to round the base up: the kernel checks it
static_assert(2 * (SMEM_BYTES + 1024) <= 233472, "two CTAs per SM");

// ring position of K_j and V_j in the load order K_0, K_1, V_0, K_2, V_1, K_3, ..., V_{n-1}
__device__ __forceinline__ int fwd_kidx(int j) { return j < 2 ? j : 2 * j - 1; }
__device__ __forceinline__ int fwd_vidx(int j, int n) { return j == n - 1 ? 2 * n - 1 : 2 + 2 * j; }

__global__ void __launch_bounds__(FWD_THREADS, 2) attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                                                                     const __grid_constant__ CUtensorMap kmap64,
                                                                     const __grid_constant__ CUtensorMap vmap64,
                                                                     __nv_bfloat16* __restrict__ o,
                                                                     float* __restrict__ lse, int S, int Hq, int Hkv,
                                                                     float scale_log2) {
  extern __shared__ __align__(1024) uint8_t smem[];
  uint64_t* qfull = reinterpret_cast<uint64_t*>(smem + F_OFF_BAR);
  uint64_t* rfull = qfull + 1;
  uint64_t* rempty = rfull + FR;
  uint64_t* sfull = rempty + FR;    // [2]: score buffer b holds S_j (j % 2 == b)
  uint64_t* pready = sfull + 2;     // [2]: P_j written, S_j read, O rescaled (one arrival per softmax warp)
  uint64_t* pvdone = pready + 2;    // one phase per chunk: P_j V_j (and everything before it) done
  uint64_t* drain = pvdone + 1;     // error path: every product issued so far has completed
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + F_OFF_MISC);
  if (smem_u32(smem) & 1023u) {     // uniform over the CTA: nothing was started
    if (threadIdx.x == 0) report(LSQ_EINVAL, 560);
    return;
  }

  const int nt = (S + BQ - 1) / BQ;
  // grid (head, sequence, query tile), tiles reversed: every head's longest causal tile is dispatched
  // before any shorter one
  const int t = nt - 1 - (int)blockIdx.z;
  const int h = blockIdx.x, b = blockIdx.y;
  const int hk = h / (Hq / Hkv);
  const int q0 = t * BQ;
  const int n = (min(q0 + BQ, S) + SUB - 1) / SUB;  // 64-key chunks at or before the tile's last row
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    mbar_init(qfull, 1);
    for (int i = 0; i < FR; ++i) {
      mbar_init(&rfull[i], 1);
      mbar_init(&rempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sfull[i], 1);
      mbar_init(&pready[i], 4);
    }
    mbar_init(pvdone, 1);
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, 256);
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
      tma_load_2d(smem + F_OFF_Q, &qmap, qfull, h * D, row0 + q0);
      tma_load_2d(smem + F_OFF_Q + HALF, &qmap, qfull, h * D + 64, row0 + q0);
      int idx = 0;
      bool ok = true;
      auto load = [&](const CUtensorMap* m, int chunk) {
        const int slot = idx % FR;
        if (!ok || !mbar_wait(&rempty[slot], ((uint32_t)(idx / FR) & 1u) ^ 1u, 461)) {
          ok = false;
          return;
        }
        uint8_t* dst = smem + F_OFF_RING + slot * ST;
        mbar_arrive_expect_tx(&rfull[slot], (uint32_t)ST);
        tma_load_2d(dst, m, &rfull[slot], hk * D, row0 + chunk * SUB);
        tma_load_2d(dst + SHALF, m, &rfull[slot], hk * D + 64, row0 + chunk * SUB);
        ++idx;
      };
      load(&kmap64, 0);
      if (n > 1) load(&kmap64, 1);
      for (int j = 0; j < n; ++j) {
        load(&vmap64, j);
        if (j + 2 < n) load(&kmap64, j + 2);
      }
      // no load may land after the CTA has gone: wait for the last one in each slot
      for (int i = max(0, idx - FR); i < idx; ++i) mbar_wait(&rfull[i % FR], (uint32_t)(i / FR) & 1u, 462);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = mbar_wait(qfull, 0, 561);
      const uint32_t qb = smem_u32(smem + F_OFF_Q);
      const uint32_t id_s = idesc_bf16(BQ, SUB, 0, 0);  // Q K^T: both K-major
      const uint32_t id_o = idesc_bf16(BQ, D, 0, 1);    // P V: P K-major, V MN-major
      auto score = [&](int j) {                          // S_j into buffer j % 2
        const int c = fwd_kidx(j), slot = c % FR;
        if (!ok || !mbar_wait(&rfull[slot], (uint32_t)(c / FR) & 1u, 562)) {
          ok = false;
          return;
        }
        tc_fence_after();
        const uint32_t kb = smem_u32(smem + F_OFF_RING + slot * ST);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          tc_mma(tmem + F_T_S + (uint32_t)((j & 1) * SUB), desc_kmajor(qb, kk), desc_sub_kmajor(kb, kk), id_s,
                 kk != 0);
        tc_commit(&sfull[j & 1]);
      };
      if (ok) tc_fence_after();
      score(0);
      if (n > 1) score(1);
      for (int j = 0; ok && j < n; ++j) {
        const int c = fwd_vidx(j, n), vslot = c % FR, kslot = fwd_kidx(j) % FR;
        if (!mbar_wait(&pready[j & 1], (uint32_t)(j >> 1) & 1u, 563) ||
            !mbar_wait(&rfull[vslot], (uint32_t)(c / FR) & 1u, 564)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t pb = smem_u32(smem + F_OFF_RING + kslot * ST);  // P_j, written over K_j
        const uint32_t vb = smem_u32(smem + F_OFF_RING + vslot * ST);
#pragma unroll
        for (int kk = 0; kk < SUB / 16; ++kk)
          tc_mma(tmem + F_T_O, desc_k64(pb, kk), desc_sub_mnmajor(vb, kk), id_o, (j | kk) != 0);
        tc_commit(pvdone);
        tc_commit(&rempty[kslot]);
        tc_commit(&rempty[vslot]);
        if (j + 2 < n) score(j + 2);
      }
      if (!ok) {  // let every product issued so far finish before TMEM is released
        tc_commit(drain);
        mbar_wait(drain, 0, 565);
      }
    }
  } else {
    // softmax and epilogue: one query row per thread
    const int quad = warp & 3;
    const int r = quad * 32 + lane;
    const int qi = q0 + r;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    float m = -INFINITY, l = 0.0f;
    bool ok = true;
    for (int j = 0; j < n; ++j) {
      const int bb = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&sfull[bb], (uint32_t)(j >> 1) & 1u, 761))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float s[64];
      {
        float lo[32], hi[32];
        tmem_ld32(tmem + lane_base + F_T_S + (uint32_t)(bb * SUB), lo);
        tmem_ld32(tmem + lane_base + F_T_S + (uint32_t)(bb * SUB + 32), hi);
        tc_wait_ld();
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          s[e] = lo[e];
          s[32 + e] = hi[e];
        }
      }
      const int k0 = j * SUB;
      const bool full = k0 + SUB - 1 <= q0 && k0 + SUB <= S;  // every key of the chunk is visible to every row
      if (!full) {
#pragma unroll
        for (int e = 0; e < 64; ++e)
          if (k0 + e > qi || k0 + e >= S) s[e] = -INFINITY;
      }
      float mxa = fmaxf(s[0], s[1]), mxb = fmaxf(s[2], s[3]);
#pragma unroll
      for (int e = 4; e < 64; e += 4) {
        mxa = max3(mxa, s[e], s[e + 1]);
        mxb = max3(mxb, s[e + 2], s[e + 3]);
      }
      const float mc = fmaxf(mxa, mxb) * scale_log2;  // the scale is positive: max of scaled = scaled max
      const bool need = mc > m + RESCALE_LOG2;
      // P_{j-1} V_{j-1} is done before O is rescaled or P_j may be consumed
      if (j > 0 && !__all_sync(0xffffffffu, mbar_wait(pvdone, (uint32_t)(j - 1) & 1u, 762))) {
        ok = false;
        break;
      }
      if (j > 0 && __any_sync(0xffffffffu, need)) {
        tc_fence_after();
        const float alpha = need ? ex2(m - mc) : 1.0f;
        l *= alpha;
#pragma unroll 1
        for (int c = 0; c < D / 32; ++c) {
          float v[32];
          tmem_ld32(tmem + lane_base + F_T_O + (uint32_t)(c * 32), v);
          tc_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] *= alpha;
          tmem_st32(tmem + lane_base + F_T_O + (uint32_t)(c * 32), v);
        }
        tc_wait_st();
      }
      if (need) m = mc;
      // p = 2^(s c - m), two columns per instruction but for the exponentials
      uint32_t w[32];
      const uint64_t c2 = f2(scale_log2, scale_log2), nm2 = f2(-m, -m);
      uint64_t la = f2(0.0f, 0.0f), lb = la;
#pragma unroll
      for (int e = 0; e < 64; e += 4) {
        const float2 xa = f2split(fma2(f2(s[e], s[e + 1]), c2, nm2));
        const float2 xb = f2split(fma2(f2(s[e + 2], s[e + 3]), c2, nm2));
        const uint64_t pa = f2(ex2(xa.x), ex2(xa.y)), pb = f2(ex2(xb.x), ex2(xb.y));
        la = add2(la, pa);
        lb = add2(lb, pb);
        w[e / 2] = pack_bf16x2(pa);
        w[e / 2 + 1] = pack_bf16x2(pb);
      }
      const float2 ls = f2split(add2(la, lb));
      l += ls.x + ls.y;
      // P_j over K_j (its score product completed before sfull): 128-byte rows, 16-byte units swizzled
      const uint32_t prow = smem_u32(smem + F_OFF_RING + (fwd_kidx(j) % FR) * ST) + r * 128;
#pragma unroll
      for (int u = 0; u < 8; ++u)
        st_shared_v4(prow + ((uint32_t)(u ^ (r & 7)) << 4), w[4 * u], w[4 * u + 1], w[4 * u + 2], w[4 * u + 3]);
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&pready[bb]);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(pvdone, (uint32_t)(n - 1) & 1u, 763))) {
      tc_fence_after();
      const float inv = 1.0f / l;
      __nv_bfloat16* orow = o + (((int64_t)b * S + qi) * Hq + h) * D;
#pragma unroll 1
      for (int c = 0; c < D / 32; ++c) {
        float v[32];
        tmem_ld32(tmem + lane_base + F_T_O + (uint32_t)(c * 32), v);
        tc_wait_ld();
        if (qi < S) {
#pragma unroll
          for (int u = 0; u < 4; ++u)
            *reinterpret_cast<uint4*>(orow + c * 32 + u * 8) =
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
    tmem_dealloc(tmem, 256);
  }
}

// ================================================================ backward
// Both backward kernels work through a list of 64-row sub-items with two
// score accumulators in TMEM, so that the element-wise step of sub-item i
// (sixteen warps) overlaps the
// score products of sub-item i+1 and the accumulating products of i-1:
//
//   MMA issue order:  S(0)  S(1) A(0)  S(2) A(1)  ...  A(n-1)
//   element-wise:           E(0)       E(1)      ...
//
// where S(i) writes score buffer i % 2 (after E(i-2) has read it), E(i) turns
// it into bf16 operands in shared-memory buffer i % 2 (after A(i-2) has read
// it) and A(i) accumulates from them.  A three-stage TMA ring feeds the 64-row
// operand tiles.  Warp 0: TMA; warp 1: TMEM owner and MMA issuer; warps 2-17:
// element-wise and epilogue, four per TMEM lane quarter, 16 columns each (four
// warps per SM sub-partition hide the TMEM, exp and shuffle latencies).
constexpr int NRING = 3;
constexpr int CW = SUB / (EW / 4);           // columns per element-wise warp
constexpr int BWD_THREADS = 32 * (2 + EW);

// CW bf16 values (CW / 2 pairs) of row r into a 128-row x 64-column swizzled
// operand: the row's 16-byte units part * CW / 8 onwards
__device__ __forceinline__ void store_row_units(uint32_t row_base, int r, int part, const uint32_t (&w)[CW / 2]) {
#pragma unroll
  for (int u = 0; u < CW / 8; ++u)
    st_shared_v4(row_base + ((uint32_t)((part * (CW / 8) + u) ^ (r & 7)) << 4), w[4 * u], w[4 * u + 1],
                 w[4 * u + 2], w[4 * u + 3]);
}

// dx1 = g1 c + g2 s, dx2 = g2 c - g1 s (the transpose of rotate-half RoPE) for 16
// column pairs (i, i + 64) of a head, g = f * accumulator; the angle of pair i is
// pos * inv[i] (inv: the frequencies i..i+15), its cosine and sine from rope_cs;
// writes columns i.. at dst and i + 64.. at dst + 64
__device__ __forceinline__ void rope_t_store(__nv_bfloat16* dst, const float (&g1)[16], const float (&g2)[16],
                                             const float* __restrict__ inv, float pos, float f) {
  float o1[16], o2[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) {
    const float2 t = rope_cs(pos * __ldg(inv + i));
    const float a = g1[i] * f, b = g2[i] * f;
    o1[i] = a * t.x + b * t.y;
    o2[i] = b * t.x - a * t.y;
  }
#pragma unroll
  for (int u = 0; u < 2; ++u) {
    *reinterpret_cast<uint4*>(dst + 8 * u) =
        make_uint4(pack_bf16x2(o1[8 * u], o1[8 * u + 1]), pack_bf16x2(o1[8 * u + 2], o1[8 * u + 3]),
                   pack_bf16x2(o1[8 * u + 4], o1[8 * u + 5]), pack_bf16x2(o1[8 * u + 6], o1[8 * u + 7]));
    *reinterpret_cast<uint4*>(dst + 64 + 8 * u) =
        make_uint4(pack_bf16x2(o2[8 * u], o2[8 * u + 1]), pack_bf16x2(o2[8 * u + 2], o2[8 * u + 3]),
                   pack_bf16x2(o2[8 * u + 4], o2[8 * u + 5]), pack_bf16x2(o2[8 * u + 6], o2[8 * u + 7]));
  }
}

// ---------------------------------------------------------------- dQ
// One CTA per (128-query tile, head, sequence); sub-items = 64-key slices of
// the keys at or before the tile:  S = Q K_j^T, dP = dO V_j^T (TMEM), dS =
// P (dP - D) (bf16, shared memory), dQ += dS K_j (TMEM); dq = dQ / sqrt(D).
constexpr int Q_OFF_Q = 0;
constexpr int Q_OFF_DO = Q_OFF_Q + TILE;
constexpr int Q_OFF_RING = Q_OFF_DO + TILE;        // stage s: K at +s*2*ST, V at +s*2*ST + ST
constexpr int Q_OFF_DS = Q_OFF_RING + NRING * 2 * ST;  // buffer b at +b*PT
constexpr int Q_OFF_BAR = Q_OFF_DS + 2 * PT;
// qfull, rfull[3], rempty[3], sfull[2], tfree[2], dsready[2], dsfree[2], done
constexpr int Q_NBAR = 1 + 3 + 3 + 2 + 2 + 2 + 2 + 1;
constexpr int Q_OFF_MISC = Q_OFF_BAR + 8 * Q_NBAR;
constexpr int Q_SMEM = Q_OFF_MISC + 16 + 1024;
static_assert(Q_SMEM <= 232448, "shared memory");

__global__ void __launch_bounds__(BWD_THREADS, 1) attn_dq_tc_kernel(const __grid_constant__ CUtensorMap qmap,
                                                                    const __grid_constant__ CUtensorMap kmap64,
                                                                    const __grid_constant__ CUtensorMap vmap64,
                                                                    const __grid_constant__ CUtensorMap domap,
                                                                    const float4* __restrict__ stats, int Sp,
                                                                    __nv_bfloat16* __restrict__ dq, int S, int Hq,
                                                                    int Hkv, float scale, float scale_log2,
                                                                    const float2* __restrict__ rope) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* qfull = reinterpret_cast<uint64_t*>(smem + Q_OFF_BAR);
  uint64_t* rfull = qfull + 1;
  uint64_t* rempty = rfull + NRING;
  uint64_t* sfull = rempty + NRING;
  uint64_t* tfree = sfull + 2;
  uint64_t* dsready = tfree + 2;
  uint64_t* dsfree = dsready + 2;
  uint64_t* done = dsfree + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + Q_OFF_MISC);

  const int nt = (S + BQ - 1) / BQ;
  // grid (head, sequence, query tile), tiles reversed: every head's longest causal tile is dispatched
  // before any shorter one
  const int t = nt - 1 - (int)blockIdx.z;
  const int h = blockIdx.x, b = blockIdx.y;
  const int hk = h / (Hq / Hkv);
  const int q0 = t * BQ;
  const int nkeys = min(q0 + BQ, S);
  const int nsub = (nkeys + SUB - 1) / SUB;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr uint32_t T_S = 0, T_DP = 128, T_DQ = 256;

  if (threadIdx.x == 0) {
    mbar_init(qfull, 1);
    for (int i = 0; i < NRING; ++i) {
      mbar_init(&rfull[i], 1);
      mbar_init(&rempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sfull[i], 1);
      mbar_init(&tfree[i], EW);
      mbar_init(&dsready[i], EW);
      mbar_init(&dsfree[i], 1);
    }
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
      mbar_arrive_expect_tx(qfull, 2u * TILE);
      tma_load_2d(smem + Q_OFF_Q, &qmap, qfull, h * D, row0 + q0);
      tma_load_2d(smem + Q_OFF_Q + HALF, &qmap, qfull, h * D + 64, row0 + q0);
      tma_load_2d(smem + Q_OFF_DO, &domap, qfull, h * D, row0 + q0);
      tma_load_2d(smem + Q_OFF_DO + HALF, &domap, qfull, h * D + 64, row0 + q0);
      for (int j = 0; j < nsub; ++j) {
        const int s = j % NRING;
        if (!mbar_wait(&rempty[s], ((uint32_t)(j / NRING) & 1u) ^ 1u, 471)) break;
        uint8_t* dst = smem + Q_OFF_RING + s * 2 * ST;
        mbar_arrive_expect_tx(&rfull[s], 2u * ST);
        tma_load_2d(dst, &kmap64, &rfull[s], hk * D, row0 + j * SUB);
        tma_load_2d(dst + SHALF, &kmap64, &rfull[s], hk * D + 64, row0 + j * SUB);
        tma_load_2d(dst + ST, &vmap64, &rfull[s], hk * D, row0 + j * SUB);
        tma_load_2d(dst + ST + SHALF, &vmap64, &rfull[s], hk * D + 64, row0 + j * SUB);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = mbar_wait(qfull, 0, 571);
      const uint32_t qb = smem_u32(smem + Q_OFF_Q), dob = smem_u32(smem + Q_OFF_DO);
      const uint32_t id_s = idesc_bf16(BQ, SUB, 0, 0);  // S, dP: both operands K-major
      const uint32_t id_q = idesc_bf16(BQ, D, 0, 1);    // dS K: K MN-major
      for (int j = 0; ok && j <= nsub; ++j) {
        if (j < nsub) {
          const int s = j % NRING, bb = j & 1;
          if (!mbar_wait(&rfull[s], (uint32_t)(j / NRING) & 1u, 572) ||
              (j >= 2 && !mbar_wait(&tfree[bb], (uint32_t)((j - 2) >> 1) & 1u, 573))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t kb = smem_u32(smem + Q_OFF_RING + s * 2 * ST), vb = kb + ST;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            tc_mma(tmem + T_S + bb * SUB, desc_kmajor(qb, kk), desc_sub_kmajor(kb, kk), id_s, kk != 0);
            tc_mma(tmem + T_DP + bb * SUB, desc_kmajor(dob, kk), desc_sub_kmajor(vb, kk), id_s, kk != 0);
          }
          tc_commit(&sfull[bb]);
        }
        if (j >= 1) {
          const int p = j - 1, ps = p % NRING, pb = p & 1;
          if (!mbar_wait(&dsready[pb], (uint32_t)(p >> 1) & 1u, 574)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t dsb = smem_u32(smem + Q_OFF_DS + pb * PT);
          const uint32_t kb = smem_u32(smem + Q_OFF_RING + ps * 2 * ST);
#pragma unroll
          for (int kk = 0; kk < SUB / 16; ++kk)
            tc_mma(tmem + T_DQ, desc_k64(dsb, kk), desc_sub_mnmajor(kb, kk), id_q, (p | kk) != 0);
          tc_commit(&dsfree[pb]);
          tc_commit(&rempty[ps]);
        }
      }
      tc_commit(done);  // also drains what was issued if a wait gave up
      if (!ok) mbar_wait(done, 0, 575);
    }
  } else {
    const int quad = warp & 3, part = (warp - 2) >> 2;
    const int r = quad * 32 + lane;  // query row of the tile
    const int qi = q0 + r;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    // this row's -lse (log2 units) and -D from the statistics table
    const int64_t pr = ((int64_t)b * Hq + h) * Sp + (qi < S ? qi : 0);
    const float4 st = stats[pr >> 1];
    const float nl2 = (pr & 1) ? st.y : st.x, nd = (pr & 1) ? st.w : st.z;
    const uint64_t c2 = f2(scale_log2, scale_log2), nl22 = f2(nl2, nl2), nd2 = f2(nd, nd);
    bool ok = true;
    for (int j = 0; ok && j < nsub; ++j) {
      const int bb = j & 1;
      if (!__all_sync(0xffffffffu, mbar_wait(&sfull[bb], (uint32_t)(j >> 1) & 1u, 771))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sv[CW], pv[CW];
      tmem_ld16(tmem + lane_base + T_S + bb * SUB + part * CW, sv);
      tmem_ld16(tmem + lane_base + T_DP + bb * SUB + part * CW, pv);
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tfree[bb]);
      // P = 2^(s c - lse), dS = P (dP - D), two columns per instruction but for the exponentials
      uint32_t w[CW / 2];
      const bool nomask = (j + 1) * SUB <= q0 && q0 + BQ <= S;  // keys all before the tile, rows inside S
#pragma unroll
      for (int e = 0; e < CW; e += 2) {
        const float2 x = f2split(fma2(f2(sv[e], sv[e + 1]), c2, nl22));
        float p0 = ex2(x.x), p1 = ex2(x.y);
        if (!nomask) {
          const int kj = j * SUB + part * CW + e;
          p0 = (kj <= qi && kj < S && qi < S) ? p0 : 0.0f;
          p1 = (kj + 1 <= qi && kj + 1 < S && qi < S) ? p1 : 0.0f;
        }
        w[e / 2] = pack_bf16x2(mul2(f2(p0, p1), add2(f2(pv[e], pv[e + 1]), nd2)));
      }
      // buffer bb was read by the dQ product of sub-item j - 2
      if (j >= 2 && !__all_sync(0xffffffffu, mbar_wait(&dsfree[bb], (uint32_t)((j - 2) >> 1) & 1u, 772))) {
        ok = false;
        break;
      }
      store_row_units(smem_u32(smem + Q_OFF_DS + bb * PT) + r * 128, r, part, w);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&dsready[bb]);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(done, 0, 773))) {
      tc_fence_after();
      __nv_bfloat16* row = dq + (((int64_t)b * S + qi) * Hq + h) * D;
      if (rope) {
        // the transpose of the forward's RoPE, on the fp32 gradient before its one rounding:
        // this warp takes columns [16 part, 16 part + 16) and their partners 64 further on
        float x1[16], x2[16];
        tmem_ld16(tmem + lane_base + T_DQ + (uint32_t)(part * 16), x1);
        tmem_ld16(tmem + lane_base + T_DQ + (uint32_t)(64 + part * 16), x2);
        tc_wait_ld();
        if (qi < S)
          rope_t_store(row + part * 16, x1, x2, reinterpret_cast<const float*>(rope) + (int64_t)S * D + part * 16,
                       (float)qi, scale);
      } else {
        const int c4 = part;  // 32 of the 128 output columns per warp
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

// ---------------------------------------------------------------- dK, dV
// One CTA per (128-key chunk, kv head, sequence); sub-items = (query head of
// the group, 64 queries at or after the chunk):  S^T = K Q_i^T, dP^T = V dO_i^T
// (TMEM), P^T and dS^T = P^T (dP^T - D) (bf16, shared memory), dV += P^T dO_i,
// dK += dS^T Q_i (TMEM); dk = dK / sqrt(D), dv = dV.
// With split = 2 (a GQA group of two or more query heads) the two CTAs of a
// cluster take half of the group's heads each; both park their dK / dV
// accumulators in their shared memory and each adds half of the rows of the
// two through distributed shared memory, rank 0's partial first (the same
// order in both CTAs).  The first key chunk's CTAs, which bound the kernel's
// time, then have half as many sub-items.
__device__ __forceinline__ uint32_t dsmem_addr(const void* p, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_u32(p)), "r"(rank));
  return r;
}
__device__ __forceinline__ float4 ld_dsmem4(uint32_t caddr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(caddr)
               : "memory");
  return v;
}
__device__ __forceinline__ void cluster_barrier() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
constexpr int PSTRIDE = 132;  // floats per parked row: 33 x 16 bytes, conflict-free float4 stores
constexpr int K_OFF_K = 0;
constexpr int K_OFF_V = K_OFF_K + TILE;
constexpr int K_OFF_RING = K_OFF_V + TILE;          // stage s: Q at +s*2*ST, dO at +s*2*ST + ST
constexpr int K_OFF_P = K_OFF_RING + NRING * 2 * ST;  // buffer b: P^T at +b*2*PT, dS^T at +b*2*PT + PT
constexpr int K_OFF_BAR = K_OFF_P + 2 * 2 * PT;
// kvfull, qfull[3], qempty[3], sfull[2], tfree[2], psready[2], pfree[2], done
constexpr int K_NBAR = 1 + 3 + 3 + 2 + 2 + 2 + 2 + 1;
constexpr int K_OFF_MISC = K_OFF_BAR + 8 * K_NBAR;
constexpr int K_SMEM = K_OFF_MISC + 16 + 1024;
static_assert(K_SMEM <= 232448, "shared memory");
static_assert(2 * BC * PSTRIDE * 4 <= K_OFF_BAR, "parked dK / dV partials stay below the barriers");

__global__ void __launch_bounds__(BWD_THREADS, 1) attn_dkv_tc_kernel(const __grid_constant__ CUtensorMap qmap64,
                                                                     const __grid_constant__ CUtensorMap kmap,
                                                                     const __grid_constant__ CUtensorMap vmap,
                                                                     const __grid_constant__ CUtensorMap domap64,
                                                                     const float4* __restrict__ stats, int Sp,
                                                                     __nv_bfloat16* __restrict__ dk,
                                                                     __nv_bfloat16* __restrict__ dv_out, int S, int Hq,
                                                                     int Hkv, float scale, float scale_log2, int split,
                                                                     const float2* __restrict__ rope) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* kvfull = reinterpret_cast<uint64_t*>(smem + K_OFF_BAR);
  uint64_t* qfull = kvfull + 1;
  uint64_t* qempty = qfull + NRING;
  uint64_t* sfull = qempty + NRING;
  uint64_t* tfree = sfull + 2;
  uint64_t* psready = tfree + 2;
  uint64_t* pfree = psready + 2;
  uint64_t* done = pfree + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + K_OFF_MISC);

  // grid (kv head x split, sequence, key chunk): the chunks with the most sub-items (the first ones) are
  // dispatched first, the short ones fill in behind them
  const int jc = blockIdx.z, b = blockIdx.y;
  const int hk = (int)blockIdx.x / split, half = (int)blockIdx.x % split;  // half = cluster rank when split
  const int group = Hq / Hkv;
  const int gh = (group + split - 1) / split;  // query heads of the first half
  const int h_begin = hk * group + half * gh, nheads = half == 0 ? gh : group - gh;
  const int k0 = jc * BC;
  const int nsub = (S - k0 + SUB - 1) / SUB;  // 64-query slices at or after the chunk, per head
  const int items = nheads * nsub;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr uint32_t T_S = 0, T_DP = 128, T_DV = 256, T_DK = 384;

  if (threadIdx.x == 0) {
    mbar_init(kvfull, 1);
    for (int i = 0; i < NRING; ++i) {
      mbar_init(&qfull[i], 1);
      mbar_init(&qempty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&sfull[i], 1);
      mbar_init(&tfree[i], EW);
      mbar_init(&psready[i], EW);
      mbar_init(&pfree[i], 1);
    }
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
        const int s = it % NRING;
        if (!mbar_wait(&qempty[s], ((uint32_t)(it / NRING) & 1u) ^ 1u, 481)) break;
        const int h = h_begin + it / nsub, qs = k0 + (it % nsub) * SUB;
        uint8_t* dst = smem + K_OFF_RING + s * 2 * ST;
        mbar_arrive_expect_tx(&qfull[s], 2u * ST);
        tma_load_2d(dst, &qmap64, &qfull[s], h * D, row0 + qs);
        tma_load_2d(dst + SHALF, &qmap64, &qfull[s], h * D + 64, row0 + qs);
        tma_load_2d(dst + ST, &domap64, &qfull[s], h * D, row0 + qs);
        tma_load_2d(dst + ST + SHALF, &domap64, &qfull[s], h * D + 64, row0 + qs);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = mbar_wait(kvfull, 0, 581);
      const uint32_t kb = smem_u32(smem + K_OFF_K), vb = smem_u32(smem + K_OFF_V);
      const uint32_t id_s = idesc_bf16(BC, SUB, 0, 0);  // S^T, dP^T: both K-major
      const uint32_t id_m = idesc_bf16(BC, D, 0, 1);    // P^T dO, dS^T Q: dO / Q MN-major
      for (int it = 0; ok && it <= items; ++it) {
        if (it < items) {
          const int s = it % NRING, bb = it & 1;
          if (!mbar_wait(&qfull[s], (uint32_t)(it / NRING) & 1u, 582) ||
              (it >= 2 && !mbar_wait(&tfree[bb], (uint32_t)((it - 2) >> 1) & 1u, 583))) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t qb = smem_u32(smem + K_OFF_RING + s * 2 * ST), dob = qb + ST;
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            tc_mma(tmem + T_S + bb * SUB, desc_kmajor(kb, kk), desc_sub_kmajor(qb, kk), id_s, kk != 0);
            tc_mma(tmem + T_DP + bb * SUB, desc_kmajor(vb, kk), desc_sub_kmajor(dob, kk), id_s, kk != 0);
          }
          tc_commit(&sfull[bb]);
        }
        if (it >= 1) {
          const int p = it - 1, ps = p % NRING, pb = p & 1;
          if (!mbar_wait(&psready[pb], (uint32_t)(p >> 1) & 1u, 584)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t pbase = smem_u32(smem + K_OFF_P + pb * 2 * PT), dsbase = pbase + PT;
          const uint32_t qb = smem_u32(smem + K_OFF_RING + ps * 2 * ST), dob = qb + ST;
#pragma unroll
          for (int kk = 0; kk < SUB / 16; ++kk) {
            tc_mma(tmem + T_DV, desc_k64(pbase, kk), desc_sub_mnmajor(dob, kk), id_m, (p | kk) != 0);
            tc_mma(tmem + T_DK, desc_k64(dsbase, kk), desc_sub_mnmajor(qb, kk), id_m, (p | kk) != 0);
          }
          tc_commit(&pfree[pb]);
          tc_commit(&qempty[ps]);
        }
      }
      tc_commit(done);
      if (!ok) mbar_wait(done, 0, 585);
    }
  } else {
    const int quad = warp & 3, part = (warp - 2) >> 2;
    const int r = quad * 32 + lane;  // key row of the chunk
    const int kj = k0 + r;
    const uint32_t lane_base = (uint32_t)(quad * 32) << 16;
    const uint64_t c2 = f2(scale_log2, scale_log2);
    bool ok = true;
    for (int it = 0; ok && it < items; ++it) {
      const int bb = it & 1;
      const int qs = k0 + (it % nsub) * SUB;
      // -lse (log2 units) and -D of this warp's CW queries, two queries per float4 of the statistics
      // table (the same 16-byte loads in every lane), issued before the wait for the scores
      float4 st[CW / 2];
      {
        const float4* src = stats + ((((int64_t)b * Hq + h_begin + it / nsub) * Sp + qs + part * CW) >> 1);
#pragma unroll
        for (int u = 0; u < CW / 2; ++u) st[u] = __ldg(src + u);
      }
      if (!__all_sync(0xffffffffu, mbar_wait(&sfull[bb], (uint32_t)(it >> 1) & 1u, 781))) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sv[CW], pv[CW];
      tmem_ld16(tmem + lane_base + T_S + bb * SUB + part * CW, sv);
      tmem_ld16(tmem + lane_base + T_DP + bb * SUB + part * CW, pv);
      tc_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tfree[bb]);
      // P^T = 2^(s c - lse), dS^T = P^T (dP^T - D), two columns (queries) per instruction but for the
      // exponentials
      uint32_t wp[CW / 2], wd[CW / 2];
      const bool nomask = qs >= k0 + BC && qs + SUB <= S && k0 + BC <= S;  // every query after every key
#pragma unroll
      for (int e = 0; e < CW; e += 2) {
        const float4 t = st[e / 2];
        const float2 x = f2split(fma2(f2(sv[e], sv[e + 1]), c2, f2(t.x, t.y)));
        float p0 = ex2(x.x), p1 = ex2(x.y);
        if (!nomask) {
          const int qi = qs + part * CW + e;
          p0 = (kj <= qi && qi < S && kj < S) ? p0 : 0.0f;
          p1 = (kj <= qi + 1 && qi + 1 < S && kj < S) ? p1 : 0.0f;
        }
        const uint64_t p = f2(p0, p1);
        wp[e / 2] = pack_bf16x2(p);
        wd[e / 2] = pack_bf16x2(mul2(p, add2(f2(pv[e], pv[e + 1]), f2(t.z, t.w))));
      }
      // buffer bb was read by the dV / dK products of sub-item it - 2
      if (it >= 2 && !__all_sync(0xffffffffu, mbar_wait(&pfree[bb], (uint32_t)((it - 2) >> 1) & 1u, 782))) {
        ok = false;
        break;
      }
      const uint32_t prow = smem_u32(smem + K_OFF_P + bb * 2 * PT) + r * 128;
      store_row_units(prow, r, part, wp);
      store_row_units(prow + PT, r, part, wd);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&psready[bb]);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(done, 0, 783)) && split > 1) {
      // park this CTA's partial dK / dV (fp32) in its shared memory, free now that every product is done
      tc_fence_after();
      float* pk = reinterpret_cast<float*>(smem) + (size_t)r * PSTRIDE + part * 32;
      float* pv = pk + BC * PSTRIDE;
      float a[32], c[32];
      tmem_ld32(tmem + lane_base + T_DK + (uint32_t)(part * 32), a);
      tmem_ld32(tmem + lane_base + T_DV + (uint32_t)(part * 32), c);
      tc_wait_ld();
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        reinterpret_cast<float4*>(pk)[u] = make_float4(a[4 * u], a[4 * u + 1], a[4 * u + 2], a[4 * u + 3]);
        reinterpret_cast<float4*>(pv)[u] = make_float4(c[4 * u], c[4 * u + 1], c[4 * u + 2], c[4 * u + 3]);
      }
    } else if (ok && split == 1) {
      tc_fence_after();
      const int64_t off = (((int64_t)b * S + kj) * Hkv + hk) * D;
      if (rope) {
        // dK with the transpose of the forward's RoPE (columns 16 part.. and 64 further on), dV as it is
        float x1[16], x2[16], c[32];
        tmem_ld16(tmem + lane_base + T_DK + (uint32_t)(part * 16), x1);
        tmem_ld16(tmem + lane_base + T_DK + (uint32_t)(64 + part * 16), x2);
        tmem_ld32(tmem + lane_base + T_DV + (uint32_t)(part * 32), c);
        tc_wait_ld();
        if (kj < S) {
          rope_t_store(dk + off + part * 16, x1, x2, reinterpret_cast<const float*>(rope) + (int64_t)S * D + part * 16,
                       (float)kj, scale);
#pragma unroll
          for (int u = 0; u < 4; ++u)
            *reinterpret_cast<uint4*>(dv_out + off + part * 32 + u * 8) =
                make_uint4(pack_bf16x2(c[8 * u], c[8 * u + 1]), pack_bf16x2(c[8 * u + 2], c[8 * u + 3]),
                           pack_bf16x2(c[8 * u + 4], c[8 * u + 5]), pack_bf16x2(c[8 * u + 6], c[8 * u + 7]));
        }
      } else {
        const int c4 = part;  // 32 of the 128 output columns per warp
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
  if (split > 1) {
    // rank q adds rows [64 q, 64 q + 64) of both partials, rank 0's first, and writes dK, dV
    cluster_barrier();
    const float* pk0 = reinterpret_cast<const float*>(smem);
    for (int e = (int)threadIdx.x; e < (BC / 2) * 2 * (D / 4); e += blockDim.x) {
      const int t = e / ((BC / 2) * (D / 4));              // 0: dK, 1: dV
      const int rr = (e / (D / 4)) % (BC / 2) + half * (BC / 2), c4 = e % (D / 4);
      if (rope && t == 0 && c4 >= D / 8) continue;         // with RoPE each dK unit below D/2 takes its partner
      const int kr = k0 + rr;
      auto sum4 = [&](int col) {                           // both CTAs' partials of 4 columns, rank 0's first
        const float* loc = pk0 + (size_t)t * BC * PSTRIDE + (size_t)rr * PSTRIDE + col;
        const float4 mine = *reinterpret_cast<const float4*>(loc);
        const float4 peer = ld_dsmem4(dsmem_addr(loc, (uint32_t)(half ^ 1)));
        const float4 lo = half == 0 ? mine : peer, hi = half == 0 ? peer : mine;
        return make_float4(lo.x + hi.x, lo.y + hi.y, lo.z + hi.z, lo.w + hi.w);
      };
      const float4 a = sum4(c4 * 4);
      __nv_bfloat16* dst = (t == 0 ? dk : dv_out) + (((int64_t)b * S + kr) * Hkv + hk) * D + c4 * 4;
      if (rope && t == 0) {
        const float4 g = sum4(c4 * 4 + D / 2);
        const float a_[4] = {a.x * scale, a.y * scale, a.z * scale, a.w * scale};
        const float g_[4] = {g.x * scale, g.y * scale, g.z * scale, g.w * scale};
        float o1[4], o2[4];
        const float* inv = reinterpret_cast<const float*>(rope) + (int64_t)S * D + c4 * 4;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 tq = rope_cs((float)kr * __ldg(inv + j));
          o1[j] = a_[j] * tq.x + g_[j] * tq.y;
          o2[j] = g_[j] * tq.x - a_[j] * tq.y;
        }
        if (kr < S) {
          *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(o1[0], o1[1]), pack_bf16x2(o1[2], o1[3]));
          *reinterpret_cast<uint2*>(dst + D / 2) = make_uint2(pack_bf16x2(o2[0], o2[1]), pack_bf16x2(o2[2], o2[3]));
        }
        continue;
      }
      const float f = t == 0 ? scale : 1.0f;
      if (kr < S)
        *reinterpret_cast<uint2*>(dst) = make_uint2(pack_bf16x2(a.x * f, a.y * f), pack_bf16x2(a.z * f, a.w * f));
    }
    cluster_barrier();  // the peer has read this CTA's partials
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Row statistics for the backward kernels: per (sequence b, query head h, position q) -lse in log2
// units and -D (D = rowsum(dO o), fp32, summed as the plain kernels sum it), stored as one float4
// {-l2[q], -l2[q+1], -D[q], -D[q+1]} per even q, so that the dK/dV kernel reads two queries' values
// with one 16-byte load and feeds them to the paired fp32 arithmetic as they are.  Each (b, h) row of
// the table holds Sp positions (S rounded up to 64, zeros past S): every 64-query slice reads inside
// it, and what it reads past S is finite.  16 lanes per row, 8 of its 128 columns each.
__global__ void __launch_bounds__(256) rowstats_kernel(const __nv_bfloat16* __restrict__ o,
                                                       const __nv_bfloat16* __restrict__ d_o,
                                                       const float* __restrict__ lse, float* __restrict__ stats, int B,
                                                       int S, int Sp, int Hq) {
  const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t w = t >> 4;  // row of [B][Sp][Hq]
  const int part = (int)(t & 15);
  const int64_t rows = (int64_t)B * Sp * Hq;
  const int h = (int)(w % Hq);
  const int q = (int)((w / Hq) % Sp);
  const int b = (int)(w / ((int64_t)Hq * Sp));
  const bool live = w < rows && q < S;
  float sum = 0.0f;
  if (live) {
    const int64_t row = ((int64_t)b * S + q) * Hq + h;
    const uint4 av = *reinterpret_cast<const uint4*>(o + row * D + part * 8);
    const uint4 gv = *reinterpret_cast<const uint4*>(d_o + row * D + part * 8);
    const uint32_t a[4] = {av.x, av.y, av.z, av.w}, g[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      sum = fmaf(bf16lo(a[k]), bf16lo(g[k]), sum);
      sum = fmaf(bf16hi(a[k]), bf16hi(g[k]), sum);
    }
  }
  for (int off = 8; off; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);  // the row's 16 lanes
  if (w < rows && part == 0) {
    const int64_t pr = ((int64_t)b * Hq + h) * Sp + q;
    float* dst = stats + (pr >> 1) * 4 + (pr & 1);
    dst[0] = live ? -lse[((int64_t)b * Hq + h) * S + q] * LOG2E : 0.0f;
    dst[2] = live ? -sum : 0.0f;
  }
}

size_t bwd_stats_bytes(int64_t B, int64_t S, int64_t Hq) { return (size_t)(B * Hq * ((S + SUB - 1) / SUB * SUB)) * 8; }

static lsq_status tmap_heads(CUtensorMap* m, const void* base, int64_t rows, int64_t heads, int box_rows = BQ) {
  return encode_tmap_2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, (uint64_t)(heads * D), (uint64_t)rows,
                        (uint64_t)(heads * D * 2), 64, (uint32_t)box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
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
  if ((s = tmap_heads(&km, k, rows, Hkv, SUB)) != LSQ_OK) return s;
  if ((s = tmap_heads(&vm, v, rows, Hkv, SUB)) != LSQ_OK) return s;
  const float sl = LOG2E / sqrtf((float)D);
  attn_fwd_tc_kernel<<<dim3(Hq, B, (S + BQ - 1) / BQ), FWD_THREADS, SMEM_BYTES, st>>>(
      qm, km, vm, static_cast<__nv_bfloat16*>(o), lse, S, Hq, Hkv, sl);
  LSQ_LAUNCH_CHECK("attn_fwd_tc_kernel");
  return LSQ_OK;
}

bool bwd_supported(int64_t S, int64_t hd) { return fwd_supported(S, hd); }

lsq_status run_bwd(const void* q, const void* k, const void* v, const void* o, const void* d_o, const float* lse,
                   void* ws, void* dq, void* dk, void* dv, int B, int S, int Hq, int Hkv, cudaStream_t st,
                   const float* rope_table) {
  const float2* rope = reinterpret_cast<const float2*>(rope_table);
  static int cfg[64];
  int dev = 0;
  LSQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev >= 0 && dev < 64 && !cfg[dev]) {
    LSQ_CUDA_TRY(cudaFuncSetAttribute(attn_dq_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, Q_SMEM));
    LSQ_CUDA_TRY(cudaFuncSetAttribute(attn_dkv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, K_SMEM));
    cfg[dev] = 1;
  }
  CUtensorMap qm, km, vm, dom, qm64, km64, vm64, dom64;
  lsq_status s;
  const int64_t rows = (int64_t)B * S;
  if ((s = tmap_heads(&qm, q, rows, Hq)) != LSQ_OK) return s;
  if ((s = tmap_heads(&km, k, rows, Hkv)) != LSQ_OK) return s;
  if ((s = tmap_heads(&vm, v, rows, Hkv)) != LSQ_OK) return s;
  if ((s = tmap_heads(&dom, d_o, rows, Hq)) != LSQ_OK) return s;
  if ((s = tmap_heads(&qm64, q, rows, Hq, SUB)) != LSQ_OK) return s;
  if ((s = tmap_heads(&km64, k, rows, Hkv, SUB)) != LSQ_OK) return s;
  if ((s = tmap_heads(&vm64, v, rows, Hkv, SUB)) != LSQ_OK) return s;
  if ((s = tmap_heads(&dom64, d_o, rows, Hq, SUB)) != LSQ_OK) return s;
  const float scale = 1.0f / sqrtf((float)D), sl = LOG2E * scale;
  const int nt = (S + BQ - 1) / BQ;
  const int Sp = (S + SUB - 1) / SUB * SUB;
  const int64_t srows = (int64_t)B * Sp * Hq;
  rowstats_kernel<<<(unsigned)((srows * 16 + 255) / 256), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(o), static_cast<const __nv_bfloat16*>(d_o), lse, static_cast<float*>(ws), B,
      S, Sp, Hq);
  LSQ_LAUNCH_CHECK("attention rowstats_kernel");
  const float4* stats = static_cast<const float4*>(ws);
  attn_dq_tc_kernel<<<dim3(Hq, B, nt), BWD_THREADS, Q_SMEM, st>>>(qm, km64, vm64, dom, stats, Sp,
                                                                  static_cast<__nv_bfloat16*>(dq), S, Hq, Hkv, scale,
                                                                  sl, rope);
  LSQ_LAUNCH_CHECK("attn_dq_tc_kernel");
  const int split = Hq / Hkv >= 2 ? 2 : 1;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(Hkv * split, B, nt);
  lc.blockDim = dim3(BWD_THREADS);
  lc.dynamicSmemBytes = K_SMEM;
  lc.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = (unsigned)split;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  LSQ_CUDA_TRY(cudaLaunchKernelEx(&lc, attn_dkv_tc_kernel, qm64, km, vm, dom64, stats, Sp,
                                  static_cast<__nv_bfloat16*>(dk), static_cast<__nv_bfloat16*>(dv), S, Hq, Hkv, scale,
                                  sl, split, rope));
  return LSQ_OK;
}

}  // namespace atc
}  // namespace lsq
