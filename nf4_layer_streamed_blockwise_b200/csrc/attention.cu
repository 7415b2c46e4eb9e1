// Causal GQA attention for the decoder layers (Llama / Qwen), forward and
// backward, flash-style: scores stay in registers, softmax is online in fp32,
// operands go through the tensor cores as bf16 (mma.sync m16n8k16, fp32
// accumulate).  These serve every shape; at head dim 128 and up to 512
// positions the forward and backward run on the tcgen05 kernels of
// attention_tc.cu instead.
//
// Layouts: q, o [B, S, Hq, D]; k, v [B, S, Hkv, D]; lse [B, Hq, S] (natural
// log of the sum of exp of the scaled scores).  Query head h reads kv head
// h / (Hq / Hkv).  Scale 1/sqrt(D).
// Backward is deterministic: dQ and (dK, dV) are separate kernels that each
// own their outputs; the GQA sum over query heads runs in a fixed order.
#include <algorithm>

#include "common.cuh"
#include "host_common.h"

namespace lsq {
namespace attn {

constexpr float LOG2E = 1.4426950408889634f;

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma16816(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Tiles in shared memory: rows of D bf16 padded by 8 elements (16 bytes) so
// that the eight row addresses of an ldmatrix hit distinct banks.
template <int D>
struct Tile {
  static constexpr int LD = D + 8;  // elements per smem row
};

// copy `rows` rows (positions p0.. of head h) of a [B,S,H,D] tensor into smem
template <int D>
__device__ __forceinline__ void load_tile(__nv_bfloat16* s, const __nv_bfloat16* g, int b, int p0, int rows, int S,
                                          int H, int h, int nthreads) {
  constexpr int C = D / 8;
  for (int idx = threadIdx.x; idx < rows * C; idx += nthreads) {
    const int r = idx / C, c = idx % C;
    const int p = p0 + r;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (p < S) v = *reinterpret_cast<const uint4*>(g + (((int64_t)b * S + p) * H + h) * D + c * 8);
    *reinterpret_cast<uint4*>(s + r * Tile<D>::LD + c * 8) = v;
  }
}

// the same copy with cp.async (16-byte chunks, rows past S zero-filled); the
// caller commits the group
template <int D>
__device__ __forceinline__ void load_tile_async(__nv_bfloat16* s, const __nv_bfloat16* g, int b, int p0, int rows,
                                                int S, int H, int h, int nthreads) {
  constexpr int C = D / 8;
  for (int idx = threadIdx.x; idx < rows * C; idx += nthreads) {
    const int r = idx / C, c = idx % C;
    const int p = p0 + r;
    const bool v = p < S;
    const __nv_bfloat16* src = v ? g + (((int64_t)b * S + p) * H + h) * D + c * 8 : g;
    const uint32_t dst = smem_u32(s + r * Tile<D>::LD + c * 8);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(v ? 16 : 0) : "memory");
  }
}
__device__ __forceinline__ void cp_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// A fragment (16 x 16, rows r0.., cols c0..) of a row-major smem tile
template <int D>
__device__ __forceinline__ void frag_a(const __nv_bfloat16* s, int r0, int c0, uint32_t* a) {
  const int i = threadIdx.x & 31;
  const int r = r0 + (i & 7) + ((i >> 3) & 1) * 8, c = c0 + (i >> 4) * 8;
  ldsm_x4(smem_u32(s + r * Tile<D>::LD + c), a[0], a[1], a[2], a[3]);
}
// B fragments of two n-blocks where B[k][n] = T[n][k] (T rows = n): rows n0..n0+15, cols k0..k0+15
template <int D>
__device__ __forceinline__ void frag_b_rows_n(const __nv_bfloat16* s, int n0, int k0, uint32_t* b) {
  const int i = threadIdx.x & 31;
  const int r = n0 + (i & 7) + (i >> 4) * 8, c = k0 + ((i >> 3) & 1) * 8;
  ldsm_x4(smem_u32(s + r * Tile<D>::LD + c), b[0], b[1], b[2], b[3]);
}
// B fragments of two n-blocks where B[k][n] = T[k][n] (T rows = k): rows k0..k0+15, cols n0..n0+15
template <int D>
__device__ __forceinline__ void frag_b_rows_k(const __nv_bfloat16* s, int k0, int n0, uint32_t* b) {
  const int i = threadIdx.x & 31;
  const int r = k0 + (i & 7) + ((i >> 3) & 1) * 8, c = n0 + (i >> 4) * 8;
  ldsm_x4_t(smem_u32(s + r * Tile<D>::LD + c), b[0], b[1], b[2], b[3]);
}

// accumulator fragments (16 x 64 as 8 n-blocks) -> bf16 A fragments (4 k-steps)
__device__ __forceinline__ void acc_to_a(const float (*acc)[4], int kk, uint32_t* a) {
  a[0] = pack_bf16x2(acc[2 * kk][0], acc[2 * kk][1]);
  a[1] = pack_bf16x2(acc[2 * kk][2], acc[2 * kk][3]);
  a[2] = pack_bf16x2(acc[2 * kk + 1][0], acc[2 * kk + 1][1]);
  a[3] = pack_bf16x2(acc[2 * kk + 1][2], acc[2 * kk + 1][3]);
}

constexpr int BQ = 64;  // query rows per CTA (4 warps x 16)
constexpr int BKV = 64; // keys per step

// ---------------------------------------------------------------- forward
template <int D>
__global__ void __launch_bounds__(128) fwd_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                                                  const __nv_bfloat16* __restrict__ v, __nv_bfloat16* __restrict__ o,
                                                  float* __restrict__ lse, int S, int Hq, int Hkv, float scale_log2) {
  extern __shared__ __align__(16) uint8_t smem[];
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* sKb = sQ + BQ * Tile<D>::LD;        // 2 buffers of K
  __nv_bfloat16* sVb = sKb + 2 * BKV * Tile<D>::LD;  // 2 buffers of V
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int hk = h / (Hq / Hkv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = qb * BQ;
  const int nkb = (min(q0 + BQ, S) + BKV - 1) / BKV;
  load_tile_async<D>(sQ, q, b, q0, BQ, S, Hq, h, 128);
  load_tile_async<D>(sKb, k, b, 0, BKV, S, Hkv, hk, 128);
  load_tile_async<D>(sVb, v, b, 0, BKV, S, Hkv, hk, 128);
  cp_commit();
  uint32_t qf[D / 16][4];

  float oacc[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.0f;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.0f, 0.0f};
  const int qi0 = q0 + warp * 16 + (lane >> 2);  // rows qi0 and qi0 + 8

  for (int kb = 0; kb < nkb; ++kb) {
    // prefetch the next key/value tile into the other buffer
    if (kb + 1 < nkb) {
      const int nb = (kb + 1) & 1;
      load_tile_async<D>(sKb + nb * BKV * Tile<D>::LD, k, b, (kb + 1) * BKV, BKV, S, Hkv, hk, 128);
      load_tile_async<D>(sVb + nb * BKV * Tile<D>::LD, v, b, (kb + 1) * BKV, BKV, S, Hkv, hk, 128);
      cp_commit();
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    if (kb == 0) {
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) frag_a<D>(sQ, warp * 16, ks * 16, qf[ks]);
    }
    const __nv_bfloat16* sK = sKb + (kb & 1) * BKV * Tile<D>::LD;
    const __nv_bfloat16* sV = sVb + (kb & 1) * BKV * Tile<D>::LD;
    float sacc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i) sacc[i][0] = sacc[i][1] = sacc[i][2] = sacc[i][3] = 0.0f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t bb[4];
        frag_b_rows_n<D>(sK, np * 16, ks * 16, bb);
        mma16816(sacc[2 * np], qf[ks], bb[0], bb[1]);
        mma16816(sacc[2 * np + 1], qf[ks], bb[2], bb[3]);
      }
    }
    // scale (base 2), causal + length mask, online softmax
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int kj = kb * BKV + nb * 8 + (lane & 3) * 2 + (e & 1);
        const int qi = qi0 + (e >> 1) * 8;
        float sv = sacc[nb][e] * scale_log2;
        if (kj > qi || kj >= S) sv = -INFINITY;
        sacc[nb][e] = sv;
        mx[e >> 1] = fmaxf(mx[e >> 1], sv);
      }
    }
    float corr[2];
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 1));
      mx[r] = fmaxf(mx[r], __shfl_xor_sync(0xffffffffu, mx[r], 2));
      const float mnew = fmaxf(mrow[r], mx[r]);
      corr[r] = (mrow[r] == -INFINITY) ? 0.0f : exp2f(mrow[r] - mnew);
      mrow[r] = mnew;
      lrow[r] *= corr[r];
    }
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = e >> 1;
        const float p = (sacc[nb][e] == -INFINITY) ? 0.0f : exp2f(sacc[nb][e] - mrow[r]);
        sacc[nb][e] = p;
        lrow[r] += p;
      }
    }
#pragma unroll
    for (int i = 0; i < D / 8; ++i) {
      oacc[i][0] *= corr[0];
      oacc[i][1] *= corr[0];
      oacc[i][2] *= corr[1];
      oacc[i][3] *= corr[1];
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t a[4];
      acc_to_a(sacc, kk, a);
#pragma unroll
      for (int dp = 0; dp < D / 16; ++dp) {
        uint32_t bb[4];
        frag_b_rows_k<D>(sV, kk * 16, dp * 16, bb);
        mma16816(oacc[2 * dp], a, bb[0], bb[1]);
        mma16816(oacc[2 * dp + 1], a, bb[2], bb[3]);
      }
    }
    __syncthreads();  // this buffer is refilled by the prefetch two iterations on
  }
  // normalise and store
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 1);
    lrow[r] += __shfl_xor_sync(0xffffffffu, lrow[r], 2);
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int qi = qi0 + r * 8;
    if (qi >= S) continue;
    const float inv = 1.0f / lrow[r];
    __nv_bfloat16* orow = o + (((int64_t)b * S + qi) * Hq + h) * D;
#pragma unroll
    for (int nb = 0; nb < D / 8; ++nb) {
      const int c = nb * 8 + (lane & 3) * 2;
      *reinterpret_cast<uint32_t*>(orow + c) = pack_bf16x2(oacc[nb][2 * r] * inv, oacc[nb][2 * r + 1] * inv);
    }
    if ((lane & 3) == 0) lse[((int64_t)b * Hq + h) * S + qi] = (mrow[r] + log2f(lrow[r])) / LOG2E;
  }
}

// ---------------------------------------------------------------- backward
// Dvec[b, h, i] = sum_d dO[b, i, h, d] * O[b, i, h, d]
// D / 8 lanes per (b, i, h) row (D = 64 or 128: 8 or 16 lanes, a power of two
// that divides the warp), each on one 16-byte chunk of both rows
__global__ void __launch_bounds__(256) dvec_kernel(const __nv_bfloat16* __restrict__ o, const __nv_bfloat16* __restrict__ d_o,
                                                   float* __restrict__ dvec, int64_t rows, int S, int Hq, int D) {
  const int lpr = D / 8;
  const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t w = t / lpr;
  const int part = (int)(t % lpr);
  float s = 0.0f;
  if (w < rows) {
    const uint4 av = *reinterpret_cast<const uint4*>(o + w * D + part * 8);
    const uint4 gv = *reinterpret_cast<const uint4*>(d_o + w * D + part * 8);
    const uint32_t a[4] = {av.x, av.y, av.z, av.w}, g[4] = {gv.x, gv.y, gv.z, gv.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      s = fmaf(bf16lo(a[k]), bf16lo(g[k]), s);
      s = fmaf(bf16hi(a[k]), bf16hi(g[k]), s);
    }
  }
  for (int off = lpr / 2; off; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);  // within the row's lanes
  if (w < rows && part == 0) {
    const int64_t h = w % Hq, bi = w / Hq, i = bi % S, b = bi / S;
    dvec[(b * Hq + h) * S + i] = s;
  }
}

// dQ: one CTA per (query block, q head, batch); loops over key blocks.
template <int D>
__global__ void __launch_bounds__(128) dq_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                                                 const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ d_o,
                                                 const float* __restrict__ lse, const float* __restrict__ dvec,
                                                 __nv_bfloat16* __restrict__ dq, int S, int Hq, int Hkv, float scale,
                                                 float scale_log2) {
  extern __shared__ __align__(16) uint8_t smem[];
  __nv_bfloat16* sQ = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* sdO = sQ + BQ * Tile<D>::LD;
  __nv_bfloat16* sKb = sdO + BQ * Tile<D>::LD;       // 2 buffers of K
  __nv_bfloat16* sVb = sKb + 2 * BKV * Tile<D>::LD;  // 2 buffers of V
  const int qb = blockIdx.x, h = blockIdx.y, b = blockIdx.z;
  const int hk = h / (Hq / Hkv);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int q0 = qb * BQ;
  const int nkb = (min(q0 + BQ, S) + BKV - 1) / BKV;
  load_tile_async<D>(sQ, q, b, q0, BQ, S, Hq, h, 128);
  load_tile_async<D>(sdO, d_o, b, q0, BQ, S, Hq, h, 128);
  load_tile_async<D>(sKb, k, b, 0, BKV, S, Hkv, hk, 128);
  load_tile_async<D>(sVb, v, b, 0, BKV, S, Hkv, hk, 128);
  cp_commit();
  const int qi0 = q0 + warp * 16 + (lane >> 2);
  float lse2[2], dv[2];
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int qi = qi0 + r * 8;
    const int64_t idx = ((int64_t)b * Hq + h) * S + (qi < S ? qi : 0);
    lse2[r] = lse[idx] * LOG2E;
    dv[r] = dvec[idx];
  }
  float dqacc[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i) dqacc[i][0] = dqacc[i][1] = dqacc[i][2] = dqacc[i][3] = 0.0f;
  for (int kb = 0; kb < nkb; ++kb) {
    if (kb + 1 < nkb) {
      const int nb = (kb + 1) & 1;
      load_tile_async<D>(sKb + nb * BKV * Tile<D>::LD, k, b, (kb + 1) * BKV, BKV, S, Hkv, hk, 128);
      load_tile_async<D>(sVb + nb * BKV * Tile<D>::LD, v, b, (kb + 1) * BKV, BKV, S, Hkv, hk, 128);
      cp_commit();
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    const __nv_bfloat16* sK = sKb + (kb & 1) * BKV * Tile<D>::LD;
    const __nv_bfloat16* sV = sVb + (kb & 1) * BKV * Tile<D>::LD;
    float sacc[8][4], pacc[8][4];
#pragma unroll
    for (int i = 0; i < 8; ++i)
#pragma unroll
      for (int e = 0; e < 4; ++e) sacc[i][e] = pacc[i][e] = 0.0f;
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t qa[4], da[4];
      frag_a<D>(sQ, warp * 16, ks * 16, qa);
      frag_a<D>(sdO, warp * 16, ks * 16, da);
#pragma unroll
      for (int np = 0; np < 4; ++np) {
        uint32_t bk[4], bv[4];
        frag_b_rows_n<D>(sK, np * 16, ks * 16, bk);
        frag_b_rows_n<D>(sV, np * 16, ks * 16, bv);
        mma16816(sacc[2 * np], qa, bk[0], bk[1]);
        mma16816(sacc[2 * np + 1], qa, bk[2], bk[3]);
        mma16816(pacc[2 * np], da, bv[0], bv[1]);       // dP = dO V^T
        mma16816(pacc[2 * np + 1], da, bv[2], bv[3]);
      }
    }
    // dS = P * (dP - Dvec)
#pragma unroll
    for (int nb = 0; nb < 8; ++nb) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int kj = kb * BKV + nb * 8 + (lane & 3) * 2 + (e & 1);
        const int r = e >> 1;
        const int qi = qi0 + r * 8;
        const float p = (kj > qi || kj >= S || qi >= S) ? 0.0f : exp2f(sacc[nb][e] * scale_log2 - lse2[r]);
        sacc[nb][e] = p * (pacc[nb][e] - dv[r]);
      }
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      uint32_t a[4];
      acc_to_a(sacc, kk, a);
#pragma unroll
      for (int dp = 0; dp < D / 16; ++dp) {
        uint32_t bb[4];
        frag_b_rows_k<D>(sK, kk * 16, dp * 16, bb);  // dQ += dS K
        mma16816(dqacc[2 * dp], a, bb[0], bb[1]);
        mma16816(dqacc[2 * dp + 1], a, bb[2], bb[3]);
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int qi = qi0 + r * 8;
    if (qi >= S) continue;
    __nv_bfloat16* row = dq + (((int64_t)b * S + qi) * Hq + h) * D;
#pragma unroll
    for (int nb = 0; nb < D / 8; ++nb) {
      const int c = nb * 8 + (lane & 3) * 2;
      *reinterpret_cast<uint32_t*>(row + c) = pack_bf16x2(dqacc[nb][2 * r] * scale, dqacc[nb][2 * r + 1] * scale);
    }
  }
}

constexpr int BQ2 = 32;  // query rows per step in the dK/dV kernel

// dK, dV: one CTA per (key block, kv head, batch); loops over the group's
// query heads and the query blocks at or after the key block.
template <int D>
__global__ void __launch_bounds__(128) dkv_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ k,
                                                  const __nv_bfloat16* __restrict__ v, const __nv_bfloat16* __restrict__ d_o,
                                                  const float* __restrict__ lse, const float* __restrict__ dvec,
                                                  __nv_bfloat16* __restrict__ dk, __nv_bfloat16* __restrict__ dv_out,
                                                  int S, int Hq, int Hkv, float scale, float scale_log2) {
  extern __shared__ __align__(16) uint8_t smem[];
  __nv_bfloat16* sK = reinterpret_cast<__nv_bfloat16*>(smem);
  __nv_bfloat16* sV = sK + BKV * Tile<D>::LD;
  __nv_bfloat16* sQb = sV + BKV * Tile<D>::LD;        // 2 buffers of Q
  __nv_bfloat16* sdOb = sQb + 2 * BQ2 * Tile<D>::LD;  // 2 buffers of dO
  float* sLb = reinterpret_cast<float*>(sdOb + 2 * BQ2 * Tile<D>::LD);
  float* sDb = sLb + 2 * BQ2;
  const int kb = blockIdx.x, hk = blockIdx.y, b = blockIdx.z;
  const int group = Hq / Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k0 = kb * BKV;
  const int nq = (S - k0 + BQ2 - 1) / BQ2;  // query blocks at or after the key block, per head
  const int total = group * nq;
  auto issue = [&](int it, int buf) {
    const int h = hk * group + it / nq, qs = k0 + (it % nq) * BQ2;
    load_tile_async<D>(sQb + buf * BQ2 * Tile<D>::LD, q, b, qs, BQ2, S, Hq, h, 128);
    load_tile_async<D>(sdOb + buf * BQ2 * Tile<D>::LD, d_o, b, qs, BQ2, S, Hq, h, 128);
    cp_commit();
    if (threadIdx.x < BQ2) {
      const int qi = qs + threadIdx.x;
      const int64_t idx = ((int64_t)b * Hq + h) * S + (qi < S ? qi : 0);
      sLb[buf * BQ2 + threadIdx.x] = lse[idx] * LOG2E;
      sDb[buf * BQ2 + threadIdx.x] = dvec[idx];
    }
  };
  load_tile_async<D>(sK, k, b, k0, BKV, S, Hkv, hk, 128);
  load_tile_async<D>(sV, v, b, k0, BKV, S, Hkv, hk, 128);
  cp_commit();
  if (total > 0) issue(0, 0);
  float dkacc[D / 8][4], dvacc[D / 8][4];
#pragma unroll
  for (int i = 0; i < D / 8; ++i)
#pragma unroll
    for (int e = 0; e < 4; ++e) dkacc[i][e] = dvacc[i][e] = 0.0f;
  const int kj0 = k0 + warp * 16 + (lane >> 2);  // this thread's key rows kj0, kj0 + 8
  for (int it = 0; it < total; ++it) {
    const int buf = it & 1;
    const int qs = k0 + (it % nq) * BQ2;
    if (it + 1 < total) {
      issue(it + 1, buf ^ 1);
      cp_wait<1>();
    } else {
      cp_wait<0>();
    }
    __syncthreads();
    const __nv_bfloat16* sQ = sQb + buf * BQ2 * Tile<D>::LD;
    const __nv_bfloat16* sdO = sdOb + buf * BQ2 * Tile<D>::LD;
    const float* sL = sLb + buf * BQ2;
    const float* sD = sDb + buf * BQ2;
    {
      // S^T (16 keys x 32 queries) and dP^T = V dO^T
      float st[4][4], dpt[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int e = 0; e < 4; ++e) st[i][e] = dpt[i][e] = 0.0f;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        uint32_t ka[4], va[4];
        frag_a<D>(sK, warp * 16, ks * 16, ka);
        frag_a<D>(sV, warp * 16, ks * 16, va);
#pragma unroll
        for (int np = 0; np < 2; ++np) {
          uint32_t bq[4], bd[4];
          frag_b_rows_n<D>(sQ, np * 16, ks * 16, bq);
          frag_b_rows_n<D>(sdO, np * 16, ks * 16, bd);
          mma16816(st[2 * np], ka, bq[0], bq[1]);
          mma16816(st[2 * np + 1], ka, bq[2], bq[3]);
          mma16816(dpt[2 * np], va, bd[0], bd[1]);
          mma16816(dpt[2 * np + 1], va, bd[2], bd[3]);
        }
      }
      // P^T and dS^T
#pragma unroll
      for (int nb = 0; nb < 4; ++nb) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int ql = nb * 8 + (lane & 3) * 2 + (e & 1);
          const int qi = qs + ql;
          const int kj = kj0 + (e >> 1) * 8;
          const float p = (qi < kj || qi >= S || kj >= S) ? 0.0f : exp2f(st[nb][e] * scale_log2 - sL[ql]);
          st[nb][e] = p;
          dpt[nb][e] = p * (dpt[nb][e] - sD[ql]);
        }
      }
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        uint32_t pa[4], sa[4];
        acc_to_a(st, kk, pa);
        acc_to_a(dpt, kk, sa);
#pragma unroll
        for (int dp = 0; dp < D / 16; ++dp) {
          uint32_t bd[4], bq[4];
          frag_b_rows_k<D>(sdO, kk * 16, dp * 16, bd);  // dV += P^T dO
          frag_b_rows_k<D>(sQ, kk * 16, dp * 16, bq);   // dK += dS^T Q
          mma16816(dvacc[2 * dp], pa, bd[0], bd[1]);
          mma16816(dvacc[2 * dp + 1], pa, bd[2], bd[3]);
          mma16816(dkacc[2 * dp], sa, bq[0], bq[1]);
          mma16816(dkacc[2 * dp + 1], sa, bq[2], bq[3]);
        }
      }
    }
    __syncthreads();
  }
#pragma unroll
  for (int r = 0; r < 2; ++r) {
    const int kj = kj0 + r * 8;
    if (kj >= S) continue;
    const int64_t off = (((int64_t)b * S + kj) * Hkv + hk) * D;
#pragma unroll
    for (int nb = 0; nb < D / 8; ++nb) {
      const int c = nb * 8 + (lane & 3) * 2;
      *reinterpret_cast<uint32_t*>(dk + off + c) = pack_bf16x2(dkacc[nb][2 * r] * scale, dkacc[nb][2 * r + 1] * scale);
      *reinterpret_cast<uint32_t*>(dv_out + off + c) = pack_bf16x2(dvacc[nb][2 * r], dvacc[nb][2 * r + 1]);
    }
  }
}

template <int D>
static lsq_status run_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int B, int S, int Hq,
                          int Hkv, cudaStream_t st) {
  const size_t smem = (size_t)(BQ + 4 * BKV) * Tile<D>::LD * 2;
  static int cfg[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (!cfg[dev]) {
    LSQ_CUDA_TRY(cudaFuncSetAttribute(fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem));
    cfg[dev] = 1;
  }
  dim3 grid((S + BQ - 1) / BQ, Hq, B);
  const float sl = LOG2E / sqrtf((float)D);
  fwd_kernel<D><<<grid, 128, smem, st>>>((const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v,
                                         (__nv_bfloat16*)o, lse, S, Hq, Hkv, sl);
  LSQ_LAUNCH_CHECK("attention fwd_kernel");
  return LSQ_OK;
}

template <int D>
static lsq_status run_bwd(const void* q, const void* k, const void* v, const void* d_o, const float* lse,
                          const float* dvec, void* dq, void* dk, void* dv, int B, int S, int Hq, int Hkv,
                          cudaStream_t st) {
  const size_t smem_q = (size_t)(2 * BQ + 4 * BKV) * Tile<D>::LD * 2;
  const size_t smem_kv = (size_t)(2 * BKV + 4 * BQ2) * Tile<D>::LD * 2 + 4 * BQ2 * sizeof(float);
  static int cfg[64];
  int dev = 0;
  cudaGetDevice(&dev);
  if (!cfg[dev]) {
    LSQ_CUDA_TRY(cudaFuncSetAttribute(dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_q));
    LSQ_CUDA_TRY(cudaFuncSetAttribute(dkv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem_kv));
    cfg[dev] = 1;
  }
  const float scale = 1.0f / sqrtf((float)D);
  const float sl = LOG2E * scale;
  dq_kernel<D><<<dim3((S + BQ - 1) / BQ, Hq, B), 128, smem_q, st>>>(
      (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, (const __nv_bfloat16*)d_o, lse, dvec,
      (__nv_bfloat16*)dq, S, Hq, Hkv, scale, sl);
  LSQ_LAUNCH_CHECK("attention dq_kernel");
  dkv_kernel<D><<<dim3((S + BKV - 1) / BKV, Hkv, B), 128, smem_kv, st>>>(
      (const __nv_bfloat16*)q, (const __nv_bfloat16*)k, (const __nv_bfloat16*)v, (const __nv_bfloat16*)d_o, lse, dvec,
      (__nv_bfloat16*)dk, (__nv_bfloat16*)dv, S, Hq, Hkv, scale, sl);
  LSQ_LAUNCH_CHECK("attention dkv_kernel");
  return LSQ_OK;
}

static lsq_status check_args(const char* who, int64_t B, int64_t S, int64_t Hq, int64_t Hkv, int64_t D) {
  if (B < 1 || S < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv != 0 || S > (1 << 20) || B * S * Hq > (1ll << 31))
    return fail(LSQ_EINVAL, "%s: bad shape (B=%lld S=%lld Hq=%lld Hkv=%lld)", who, (long long)B, (long long)S,
                (long long)Hq, (long long)Hkv);
  if (D != 64 && D != 128) return fail(LSQ_EUNSUPPORTED, "%s: head dim %lld (supported: 64, 128)", who, (long long)D);
  return check_device();
}

}  // namespace attn
}  // namespace lsq

using namespace lsq;
using namespace lsq::attn;

extern "C" lsq_status lsq_attention_fwd(const void* q, const void* k, const void* v, void* o, float* lse, int64_t batch,
                                        int64_t seq, int64_t hq, int64_t hkv, int64_t hd, lsq_cuda_stream stream) {
  if (!q || !k || !v || !o || !lse) return fail(LSQ_EINVAL, "lsq_attention_fwd: NULL argument");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16))
    return fail(LSQ_EINVAL, "lsq_attention_fwd: alignment");
  lsq_status st = check_args("lsq_attention_fwd", batch, seq, hq, hkv, hd);
  if (st != LSQ_OK) return st;
  // head dim 128 at up to 512 positions: the tcgen05 kernel (attention_tc.cu)
  if (atc::fwd_supported(seq, hd))
    return atc::run_fwd(q, k, v, o, lse, (int)batch, (int)seq, (int)hq, (int)hkv, (cudaStream_t)stream);
  if (hd == 64) return run_fwd<64>(q, k, v, o, lse, (int)batch, (int)seq, (int)hq, (int)hkv, (cudaStream_t)stream);
  return run_fwd<128>(q, k, v, o, lse, (int)batch, (int)seq, (int)hq, (int)hkv, (cudaStream_t)stream);
}

extern "C" size_t lsq_attention_bwd_workspace_size(int64_t batch, int64_t seq, int64_t hq) {
  // the plain kernels' D [B, Hq, S] in fp32, or the tcgen05 kernels' row statistics table
  const size_t plain = (size_t)(batch * seq * hq > 0 ? batch * seq * hq : 1) * sizeof(float);
  const size_t tc = batch > 0 && seq > 0 && hq > 0 ? atc::bwd_stats_bytes(batch, seq, hq) : 0;
  return (std::max(plain, tc) + 255) / 256 * 256;
}

namespace lsq {
namespace ops {
lsq_status rope_from_table(void* x, const float* table, int64_t batch, int64_t seq, int64_t heads, int64_t hd,
                           int inverse, cudaStream_t stream);
}
}  // namespace lsq

extern "C" lsq_status lsq_attention_bwd_ex(const void* q, const void* k, const void* v, const void* o, const float* lse,
                                           const void* d_o, void* dq, void* dk, void* dv, int64_t batch, int64_t seq,
                                           int64_t hq, int64_t hkv, int64_t hd, const float* rope_table,
                                           void* workspace, size_t workspace_bytes, lsq_cuda_stream stream) {
  if (!q || !k || !v || !o || !lse || !d_o || !dq || !dk || !dv || !workspace)
    return fail(LSQ_EINVAL, "lsq_attention_bwd: NULL argument");
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) || !aligned(d_o, 16) ||
      !aligned(dq, 16) || !aligned(dk, 16) || !aligned(dv, 16) || (rope_table && !aligned(rope_table, 16)))
    return fail(LSQ_EINVAL, "lsq_attention_bwd: alignment");
  lsq_status st = check_args("lsq_attention_bwd", batch, seq, hq, hkv, hd);
  if (st != LSQ_OK) return st;
  if (workspace_bytes < lsq_attention_bwd_workspace_size(batch, seq, hq) || !aligned(workspace, 16))
    return fail(LSQ_EINVAL, "lsq_attention_bwd: workspace too small or not 16-byte aligned");
  const cudaStream_t cs = (cudaStream_t)stream;
  // the tcgen05 kernels form their row statistics themselves and apply the RoPE transpose in their
  // epilogues; the others take D from the pass below and leave RoPE to a pass after them
  if (atc::bwd_supported(seq, hd))
    return atc::run_bwd(q, k, v, o, d_o, lse, workspace, dq, dk, dv, (int)batch, (int)seq, (int)hq, (int)hkv, cs,
                        rope_table);
  float* dvec = static_cast<float*>(workspace);
  const int64_t rows = batch * seq * hq;
  dvec_kernel<<<(unsigned)((rows * (hd / 8) + 255) / 256), 256, 0, cs>>>((const __nv_bfloat16*)o, (const __nv_bfloat16*)d_o,
                                                                  dvec, rows, (int)seq, (int)hq, (int)hd);
  LSQ_LAUNCH_CHECK("attention dvec_kernel");
  st = hd == 64 ? run_bwd<64>(q, k, v, d_o, lse, dvec, dq, dk, dv, (int)batch, (int)seq, (int)hq, (int)hkv, cs)
                : run_bwd<128>(q, k, v, d_o, lse, dvec, dq, dk, dv, (int)batch, (int)seq, (int)hq, (int)hkv, cs);
  if (st != LSQ_OK || !rope_table) return st;
  if ((st = ops::rope_from_table(dq, rope_table, batch, seq, hq, hd, 1, cs)) != LSQ_OK) return st;
  return ops::rope_from_table(dk, rope_table, batch, seq, hkv, hd, 1, cs);
}

extern "C" lsq_status lsq_attention_bwd(const void* q, const void* k, const void* v, const void* o, const float* lse,
                                        const void* d_o, void* dq, void* dk, void* dv, int64_t batch, int64_t seq,
                                        int64_t hq, int64_t hkv, int64_t hd, void* workspace, size_t workspace_bytes,
                                        lsq_cuda_stream stream) {
  return lsq_attention_bwd_ex(q, k, v, o, lse, d_o, dq, dk, dv, batch, seq, hq, hkv, hd, nullptr, workspace,
                              workspace_bytes, stream);
}
