// Fused NF4-dequant GEMMs with the LoRA path, sm_100a (tcgen05 + TMEM + TMA).
//
//   FWD: Y = residual + X deq(W)^T + s (X A^T) B^T,  U = X A^T
//   DX : dX = sum_seg dY_seg deq(W_seg) + s sum_seg G_seg A_seg,  G_seg = dY_seg B_seg
//
// One CTA computes a 256 x BN output tile (BN = 128 or 192) as two 128-row
// halves that share one dequantised weight tile per stage: the NF4 decode work
// per tensor-core FLOP is half that of a 128-row tile.  Contraction blocks of
// 64; NST shared-memory stages.
//
// Warp roles:
//   0-3        epilogue warpgroup (TMEM lanes 0-127; both halves)
//   4          TMA producer: activation tile (256 rows, 128-byte swizzle),
//              packed NF4 codes, and (FWD) the LoRA-down tile
//   5          MMA issuer + TMEM owner
//   6 ..       BN/16 dequantiser warps: two threads per 64-element NF4 block per
//              stage, each writing half of one 128-byte row of the swizzled
//              bf16 operand
// The rank-r down product rides in the same MMA as the base GEMM: the LoRA
// operand tile sits right after the weight tile in shared memory, so one MMA
// per half (N = BN + LW) reads the activation slice once and writes
// [acc | U] (FWD, LW = rp: A's rows appended to W's) or [dX | G] (DX, LW = 64:
// each segment's B in its own rank-padded column range, so the segments' G
// stay apart).  TMEM columns of half h: [h*NW, h*NW + BN) accumulator,
// [h*NW + BN, h*NW + NW) the rank-r product; NW = BN + LW, 2*NW <= 512.
//
// The LoRA-up product runs on the tensor cores: after the main loop the
// epilogue writes s*U (or s*G) as bf16 into shared memory and the MMA warp adds
// (sU) B^T (or (sG) A) into the same accumulators (K = KE), so the output is
// rounded to bf16 once.  Every wait is bounded (common.cuh); there are no
// atomics, so results do not depend on timing or buffer addresses.
#include "common.cuh"
#include "host_common.h"

namespace lsq {
namespace nf4g {

enum Mode { FWD = 0, DX = 1 };

constexpr int BM = 256, HM = 128, BK = 64, NST = 3;
constexpr int KE_MAX = 64;
constexpr int A_BYTES = BM * BK * 2;  // 32 KB

template <int BN>
struct Cfg {
  static constexpr int DQ_WARPS = BN / 16;  // two threads per 64-element NF4 block
  static constexpr int NTHREADS = (6 + DQ_WARPS) * 32;
  static constexpr int W_BYTES = BN * BK * 2;             // dequantised weight tile
  static constexpr int B_BYTES = W_BYTES + KE_MAX * BK * 2;  // + LoRA operand tile (<= 64 x 64)
  static constexpr int C_BYTES = BN * BK / 2;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + NST * A_BYTES;
  static constexpr int OFF_C = OFF_B + NST * B_BYTES;
  static constexpr int OFF_BAR = OFF_C + NST * C_BYTES;
  // epilogue LoRA operands, aliased onto the stages (used after the main loop)
  static constexpr int OFF_UE = 0;                          // 2 x [128 x KE] bf16
  static constexpr int OFF_BE = 2 * HM * KE_MAX * 2;        // [BN x KE] bf16
  static_assert(OFF_BE + BN * KE_MAX * 2 <= OFF_C, "epilogue operands must fit the stage buffers");
  static constexpr int NBAR = 3 * NST + 4;
  static constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;
  static constexpr int BYTES = OFF_MISC + 128 + 1024;
  static_assert(BYTES <= 232448, "shared memory");
};

struct Seg {
  const float* absmax;
  const __nv_bfloat16* la;   // LoRA A [r, K_in]
  const __nv_bfloat16* lb;   // LoRA B [n, r]
  const __nv_bfloat16* lat;  // DX: A^T [K_in, rp], columns >= r zero
  __nv_bfloat16* y;          // FWD output [M, n]
  const __nv_bfloat16* res;  // FWD residual [M, n] or null
  float* uo;                 // U (FWD) or G (DX) [M, r] or null
  int n;                     // rows of W
  int first;                 // FWD: first n-tile of the segment; DX: first contraction block
};

struct Params {
  Seg seg[3];
  int nseg;
  int M, K;     // K = k_in
  int r, rp;
  float s;
  float cb[16];
  __nv_bfloat16* dx;  // DX output [M, K] or null
  int nkb;
};

struct Maps {
  CUtensorMap a[3];  // FWD: x; DX: dy of each segment (box 64 x 256 rows, 128B swizzle)
  CUtensorMap c[3];  // packed codes of each segment
  CUtensorMap l[3];  // LoRA operand of the main loop: FWD A [r, K] (box 64 x rp rows);
                     // DX rank-padded B [n, 64] (box 64 x 64 rows)
};

__device__ __forceinline__ int seg_of_block(const Params& p, int i) {
  int sg = 0;
  while (sg + 1 < p.nseg && i >= p.seg[sg + 1].first) ++sg;
  return sg;
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void st_shared_u16(uint32_t addr, uint16_t v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(addr), "h"(v) : "memory");
}

// eight codes (one 32-bit word; first element = high nibble of byte 0) -> eight bf16
__device__ __forceinline__ uint4 dq8(uint32_t w, float a, const float* cb) {
  uint4 o;
  o.x = pack_bf16x2(__fmul_rn(cb[(w >> 4) & 15], a), __fmul_rn(cb[w & 15], a));
  o.y = pack_bf16x2(__fmul_rn(cb[(w >> 12) & 15], a), __fmul_rn(cb[(w >> 8) & 15], a));
  o.z = pack_bf16x2(__fmul_rn(cb[(w >> 20) & 15], a), __fmul_rn(cb[(w >> 16) & 15], a));
  o.w = pack_bf16x2(__fmul_rn(cb[(w >> 28) & 15], a), __fmul_rn(cb[(w >> 24) & 15], a));
  return o;
}

// half of an NF4 block (32 values, 16 code bytes) -> 16-byte chunks
// half*4 .. half*4+3 of one 128-byte row of a 128B-swizzled tile
__device__ __forceinline__ void store_half_row(uint32_t row_addr, int row, int half, uint4 c, float a,
                                               const float* cb) {
  const uint32_t w[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
  for (int q = 0; q < 4; ++q)
    st_shared_v4(row_addr + ((uint32_t)((half * 4 + q) ^ (row & 7)) << 4), dq8(w[q], a, cb));
}

template <int MODE, int BN>
__global__ void __launch_bounds__(Cfg<BN>::NTHREADS, 1) nf4_gemm_kernel(const __grid_constant__ Maps maps,
                                                                         const __grid_constant__ Params p) {
  using C = Cfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* empty = full + NST;
  uint64_t* cfull = empty + NST;
  uint64_t* ufull = cfull + NST;
  uint64_t* lready = ufull + 1;
  uint64_t* afull = ufull + 2;
  uint64_t* drain = ufull + 3;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  float* s_cb = reinterpret_cast<float*>(smem + C::OFF_MISC + 16);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * BM;
  int seg = 0, tile = blockIdx.x;
  if (MODE == FWD) {
    while (seg + 1 < p.nseg && (int)blockIdx.x >= p.seg[seg + 1].first) ++seg;
    tile = blockIdx.x - p.seg[seg].first;
  }
  const int n0 = tile * BN;  // FWD: output column in the segment; DX: k_in column
  const bool lora = p.rp > 0;
  const int KE = (MODE == DX) ? p.nseg * p.rp : p.rp;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1 + C::DQ_WARPS);
      mbar_init(&empty[s], 1);
      mbar_init(&cfull[s], 1);
    }
    mbar_init(ufull, 1);
    mbar_init(lready, 1);
    mbar_init(afull, 1);
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (threadIdx.x < 16) s_cb[threadIdx.x] = p.cb[threadIdx.x];
  if (warp == 5) {
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 4) {
    // ---------------------------------------------------------------- TMA producer
    if (lane == 0) {
      for (int i = 0; i < p.nkb; ++i) {
        const int s = i % NST;
        const uint32_t ph = (uint32_t)(i / NST) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, 411)) break;
        uint8_t* a_dst = smem + C::OFF_A + s * A_BYTES;
        uint8_t* c_dst = smem + C::OFF_C + s * C::C_BYTES;
        const uint32_t lbytes = lora ? (MODE == DX ? 64u * 128u : (uint32_t)p.rp * 128u) : 0u;
        mbar_arrive_expect_tx(&full[s], (uint32_t)A_BYTES + lbytes);
        uint8_t* l_dst = smem + C::OFF_B + s * C::B_BYTES + C::W_BYTES;
        mbar_arrive_expect_tx(&cfull[s], (uint32_t)C::C_BYTES);
        if (MODE == DX) {
          const int sg = seg_of_block(p, i);
          const int nb = i - p.seg[sg].first;
          tma_load_2d(a_dst, &maps.a[sg], &full[s], nb * BK, m0);
          tma_load_2d(c_dst, &maps.c[sg], &cfull[s], n0 / 2, nb * BK);
          if (lora) tma_load_2d(l_dst, &maps.l[sg], &full[s], 0, nb * BK);
        } else {
          tma_load_2d(a_dst, &maps.a[0], &full[s], i * BK, m0);
          tma_load_2d(c_dst, &maps.c[seg], &cfull[s], i * (BK / 2), n0);
          if (lora) tma_load_2d(l_dst, &maps.l[seg], &full[s], i * BK, 0);
        }
      }
    }
  } else if (warp == 5) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const int LW = lora ? (MODE == DX ? 64 : p.rp) : 0;  // LoRA columns appended to the weight tile
      const int NW = BN + LW;
      const uint32_t id_main = idesc_bf16(HM, NW, 0, MODE == DX ? 1 : 0);
      const uint32_t id_ep = idesc_bf16(HM, BN, 0, 0);
      bool ok = true;
      for (int i = 0; i < p.nkb; ++i) {
        const int s = i % NST;
        const uint32_t ph = (uint32_t)(i / NST) & 1u;
        if (!mbar_wait(&full[s], ph, 511)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_base = smem_u32(smem + C::OFF_A + s * A_BYTES);
        const uint32_t b_base = smem_u32(smem + C::OFF_B + s * C::B_BYTES);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t bd = (MODE == DX) ? smem_desc(b_base + kk * 2048, 8192, 1024, 2)
                                           : smem_desc(b_base + kk * 32, 16, 1024, 2);
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint64_t ad = smem_desc(a_base + h * (HM * 128) + kk * 32, 16, 1024, 2);
            tc_mma(tmem + h * NW, ad, bd, id_main, (i | kk) != 0);
          }
        }
        tc_commit(&empty[s]);
      }
      if (ok) {
        tc_commit(ufull);
        if (lora) {
          if (mbar_wait(lready, 0, 512)) {
            tc_fence_after();
            const uint32_t be = smem_u32(smem + C::OFF_BE);
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const uint32_t ue = smem_u32(smem + C::OFF_UE + h * HM * KE_MAX * 2);
              for (int kk = 0; kk < KE / 16; ++kk)
                tc_mma(tmem + h * NW, smem_desc(ue + kk * 256, 128, KE * 16, 0),
                       smem_desc(be + kk * 256, 128, KE * 16, 0), id_ep, 1);
            }
            tc_commit(afull);
          } else {
            ok = false;
          }
        }
      }
      if (!ok) {
        tc_commit(drain);
        mbar_wait(drain, 0, 513);
      }
    }
  } else if (warp >= 6) {
    // ---------------------------------------------------------------- NF4 dequantisers
    const int t = threadIdx.x - 6 * 32;  // 0 .. 2*BN-1
    const int KB = p.K / 64;
    if (MODE == FWD) {
      // thread -> (row, half): consecutive lanes read consecutive 16-byte code
      // chunks and write conflict-free swizzled chunks
      const int row = t >> 1, half = t & 1;
      const Seg& sg = p.seg[seg];
      const int n = n0 + row;
      const bool valid = n < sg.n;
      const float* arow = sg.absmax + (int64_t)(valid ? n : 0) * KB;
      const bool vec = (KB % 4) == 0;
      float4 acur = make_float4(0.f, 0.f, 0.f, 0.f), anext = acur;
      float s0 = 0.f, s1 = 0.f, s2 = 0.f;
      if (valid) {
        if (vec) {
          acur = __ldg(reinterpret_cast<const float4*>(arow));
          if (KB > 4) anext = __ldg(reinterpret_cast<const float4*>(arow + 4));
        } else {
          s0 = __ldg(arow);
          if (KB > 1) s1 = __ldg(arow + 1);
          if (KB > 2) s2 = __ldg(arow + 2);
        }
      }
      for (int i = 0; i < p.nkb; ++i) {
        const int s = i % NST;
        const uint32_t ph = (uint32_t)(i / NST) & 1u;
        const int q = i & 3;
        const float a = vec ? (q == 0 ? acur.x : q == 1 ? acur.y : q == 2 ? acur.z : acur.w) : s0;
        if (!mbar_wait(&cfull[s], ph, 611)) break;
        const uint4 c = *reinterpret_cast<const uint4*>(smem + C::OFF_C + s * C::C_BYTES + t * 16);
        store_half_row(smem_u32(smem + C::OFF_B + s * C::B_BYTES) + row * 128, row, half, c, valid ? a : 0.0f, s_cb);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[s]);
        if (valid) {
          if (vec) {
            if (q == 3) {
              acur = anext;
              if (i + 5 < KB) anext = __ldg(reinterpret_cast<const float4*>(arow + i + 5));
            }
          } else {
            s0 = s1;
            s1 = s2;
            if (i + 3 < KB) s2 = __ldg(arow + i + 3);
          }
        }
      }
    } else {
      // DX stage tile: 64 contraction rows (n) x BN output columns (k) = 64 x BN/64
      // blocks; thread -> (k chunk, row, half) so that the 8 lanes of each
      // store phase write 8 different swizzled chunks of 4 rows of one chunk
      const int kc = t >> 7, nl = (t & 127) >> 1, half = t & 1;
      const int kcol = n0 + kc * 64;
      auto absmax_of = [&](int i) {
        const int sgi = seg_of_block(p, i);
        const Seg& sg = p.seg[sgi];
        const int nrow = (i - sg.first) * BK + nl;
        return (nrow < sg.n && kcol < p.K) ? __ldg(sg.absmax + (int64_t)nrow * KB + kcol / 64) : 0.0f;
      };
      float a_nx = p.nkb > 0 ? absmax_of(0) : 0.0f;
      for (int i = 0; i < p.nkb; ++i) {
        const int s = i % NST;
        const uint32_t ph = (uint32_t)(i / NST) & 1u;
        const float a = a_nx;
        if (i + 1 < p.nkb) a_nx = absmax_of(i + 1);
        if (!mbar_wait(&cfull[s], ph, 612)) break;
        const uint4 c =
            *reinterpret_cast<const uint4*>(smem + C::OFF_C + s * C::C_BYTES + nl * (BN / 2) + kc * 32 + half * 16);
        store_half_row(smem_u32(smem + C::OFF_B + s * C::B_BYTES) + kc * 8192 + nl * 128, nl, half, c, a, s_cb);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&full[s]);
      }
    }
  } else {
    // ---------------------------------------------------------------- epilogue (warps 0-3)
    const int e = threadIdx.x;  // TMEM lane = row of each half
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const int NW = BN + (lora ? (MODE == DX ? 64 : p.rp) : 0);
    bool ok = mbar_wait(ufull, 0, 711);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) tc_fence_after();
    if (ok && lora) {
      // LoRA-up operand sBe [BN rows x KE], no-swizzle K-major:
      //   FWD: B[n0 + row, j];  DX: A_seg[j, n0 + row] at column seg*rp + j
      const uint32_t be = smem_u32(smem + C::OFF_BE);
      for (int row = e; row < BN; row += 128) {
        for (int jc = 0; jc < KE / 8; ++jc) {
          uint4 w = make_uint4(0, 0, 0, 0);
          if (MODE == FWD) {
            const int n = n0 + row, j0 = jc * 8;
            if (n < p.seg[seg].n && j0 < p.r) {
              const __nv_bfloat16* src = p.seg[seg].lb + (int64_t)n * p.r + j0;
              if ((p.r & 7) == 0) {
                w = __ldg(reinterpret_cast<const uint4*>(src));
              } else {
                float v[8];
#pragma unroll
                for (int q = 0; q < 8; ++q) v[q] = (j0 + q < p.r) ? __bfloat162float(src[q]) : 0.0f;
                w = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]), pack_bf16x2(v[4], v[5]),
                               pack_bf16x2(v[6], v[7]));
              }
            }
          } else {
            const int sg = (jc * 8) / p.rp, jj = (jc * 8) % p.rp, k = n0 + row;
            if (k < p.K) w = __ldg(reinterpret_cast<const uint4*>(p.seg[sg].lat + (int64_t)k * p.rp + jj));
          }
          st_shared_v4(be + (row >> 3) * (KE * 16) + jc * 128 + (row & 7) * 16, w);
        }
      }
      // s * U (or s * G) as bf16, one operand per half
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int m = m0 + h * HM + e;
        const uint32_t ue = smem_u32(smem + C::OFF_UE + h * HM * KE_MAX * 2);
        for (int c = 0; c < KE / 16; ++c) {
          float v[16];
          tmem_ld16(tmem + lane_base + h * NW + BN + c * 16, v);
          tc_wait_ld();
          if (m < p.M) {
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const int j = c * 16 + q;
              if (MODE == FWD) {
                if (tile == 0 && p.seg[seg].uo && j < p.r) p.seg[seg].uo[(int64_t)m * p.r + j] = v[q];
              } else {
                const int sg = j / p.rp, jj = j % p.rp;
                if (blockIdx.x == 0 && p.seg[sg].uo && jj < p.r) p.seg[sg].uo[(int64_t)m * p.r + jj] = v[q];
              }
            }
          }
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            uint4 o;
            o.x = pack_bf16x2(v[hh * 8 + 0] * p.s, v[hh * 8 + 1] * p.s);
            o.y = pack_bf16x2(v[hh * 8 + 2] * p.s, v[hh * 8 + 3] * p.s);
            o.z = pack_bf16x2(v[hh * 8 + 4] * p.s, v[hh * 8 + 5] * p.s);
            o.w = pack_bf16x2(v[hh * 8 + 6] * p.s, v[hh * 8 + 7] * p.s);
            st_shared_v4(ue + (e >> 3) * (KE * 16) + (c * 2 + hh) * 128 + (e & 7) * 16, o);
          }
        }
      }
      fence_proxy_async_smem();
      named_bar_sync(1, 128);
      if (e == 0) mbar_arrive(lready);
      ok = mbar_wait(afull, 0, 712);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) tc_fence_after();
    }
    if (ok) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int m = m0 + h * HM + e;
        for (int c = 0; c < BN / 32; ++c) {
          float v[32];
          tmem_ld32(tmem + lane_base + h * NW + c * 32, v);
          tc_wait_ld();
          if (m >= p.M) continue;
#pragma unroll
          for (int gq = 0; gq < 4; ++gq) {
            const int col = n0 + c * 32 + gq * 8;
            float* x = v + gq * 8;
            if (MODE == FWD) {
              const Seg& sg = p.seg[seg];
              if (col >= sg.n) continue;
              const int64_t off = (int64_t)m * sg.n + col;
              if (sg.res) {
                const uint4 rv = *reinterpret_cast<const uint4*>(sg.res + off);
                x[0] += bf16lo(rv.x); x[1] += bf16hi(rv.x);
                x[2] += bf16lo(rv.y); x[3] += bf16hi(rv.y);
                x[4] += bf16lo(rv.z); x[5] += bf16hi(rv.z);
                x[6] += bf16lo(rv.w); x[7] += bf16hi(rv.w);
              }
              *reinterpret_cast<uint4*>(sg.y + off) = make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]),
                                                                 pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
            } else {
              if (col >= p.K || p.dx == nullptr) continue;
              *reinterpret_cast<uint4*>(p.dx + (int64_t)m * p.K + col) =
                  make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                             pack_bf16x2(x[6], x[7]));
            }
          }
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int MODE, int BN>
static lsq_status launch(const Maps& maps, const Params& p, dim3 grid, cudaStream_t stream) {
  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    LSQ_CUDA_TRY(cudaFuncSetAttribute(nf4_gemm_kernel<MODE, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      Cfg<BN>::BYTES));
    configured[dev] = 1;
  }
  nf4_gemm_kernel<MODE, BN><<<grid, Cfg<BN>::NTHREADS, Cfg<BN>::BYTES, stream>>>(maps, p);
  LSQ_LAUNCH_CHECK("nf4_gemm_kernel");
  return LSQ_OK;
}

// N-tile width: the one whose wave count on the SMs times tile width is smaller
// (ties to the wider tile, which re-reads the activation tile less often).
static int pick_bn(const int64_t* ns, int nseg, int64_t M, bool lora_ok192) {
  const int64_t mt = (M + BM - 1) / BM;
  const int sms = num_sms();
  int64_t best = -1;
  int bn_best = 192;
  for (int bn : {192, 128}) {
    if (bn == 192 && !lora_ok192) continue;
    int64_t tiles = 0;
    for (int i = 0; i < nseg; ++i) tiles += (ns[i] + bn - 1) / bn;
    const int64_t waves = (tiles * mt + sms - 1) / sms;
    const int64_t cost = waves * bn;
    if (best < 0 || cost < best) {
      best = cost;
      bn_best = bn;
    }
  }
  return bn_best;
}

static void fill_cb(Params& p) {
  const float* cb = codebook();
  for (int i = 0; i < 16; ++i) p.cb[i] = cb[i];
}

}  // namespace nf4g
}  // namespace lsq

namespace lsq {
namespace tc {
using namespace lsq::nf4g;

static lsq_status nf4_checks(int64_t M, int64_t K, int32_t r, const char* who) {
  lsq_status st = check_device();
  if (st != LSQ_OK) return st;
  if (M < 1 || M > (1 << 30)) return fail(LSQ_EINVAL, "%s: M out of range (%lld)", who, (long long)M);
  if (K < 64 || K % 64 != 0 || K > (1 << 30))
    return fail(LSQ_EINVAL, "%s: k_in must be a positive multiple of 64 (got %lld)", who, (long long)K);
  if (r < 0 || r > 64) return fail(LSQ_EINVAL, "%s: LoRA rank must be in [0, 64] (got %d)", who, r);
  return LSQ_OK;
}

static lsq_status check_weight(const lsq_nf4_weight& w, int64_t K, const char* who) {
  if (!w.codes || !w.absmax) return fail(LSQ_EINVAL, "%s: NULL weight pointer", who);
  if (w.k_in != K) return fail(LSQ_EINVAL, "%s: k_in mismatch (%lld vs %lld)", who, (long long)w.k_in, (long long)K);
  if (w.n_out < 8 || w.n_out % 8 != 0 || w.n_out > (1 << 30))
    return fail(LSQ_EINVAL, "%s: n_out must be a positive multiple of 8 (got %lld)", who, (long long)w.n_out);
  if (!aligned(w.codes, 16) || !aligned(w.absmax, 4))
    return fail(LSQ_EINVAL, "%s: codes must be 16-byte and absmax 4-byte aligned", who);
  return LSQ_OK;
}

lsq_status launch_dx(int nseg, const lsq_nf4_weight* W, const void* const* dy, int64_t M,
                     const __nv_bfloat16* const* Bp, const __nv_bfloat16* const* At, int r, float s, void* dx,
                     float* const* g_out, cudaStream_t stream) {
  const int64_t K = W[0].k_in;
  Params p;
  memset(&p, 0, sizeof(p));
  p.nseg = nseg;
  p.M = (int)M;
  p.K = (int)K;
  p.r = r;
  p.rp = r > 0 ? (r + 15) / 16 * 16 : 0;
  p.s = s;
  p.dx = static_cast<__nv_bfloat16*>(dx);
  fill_cb(p);
  if (nseg * p.rp > KE_MAX) return fail(LSQ_EUNSUPPORTED, "lsq_nf4_lora_bwd: nseg * round16(r) must be <= 64");
  const int64_t kk[1] = {K};
  const int BN = pick_bn(kk, 1, M, true);
  Maps maps;
  memset(&maps, 0, sizeof(maps));
  int blocks = 0;
  lsq_status st;
  for (int i = 0; i < nseg; ++i) {
    Seg& g = p.seg[i];
    g.absmax = W[i].absmax;
    g.lat = r > 0 ? At[i] : nullptr;
    g.uo = r > 0 ? g_out[i] : nullptr;
    g.n = (int)W[i].n_out;
    g.first = blocks;
    blocks += (int)((W[i].n_out + BK - 1) / BK);
    if ((st = encode_tmap_2d(&maps.a[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dy[i], W[i].n_out, M, W[i].n_out * 2, BK,
                             BM, CU_TENSOR_MAP_SWIZZLE_128B)) != LSQ_OK)
      return st;
    if ((st = encode_tmap_2d(&maps.c[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, W[i].codes, K / 2, W[i].n_out, K / 2, BN / 2,
                             BK, CU_TENSOR_MAP_SWIZZLE_NONE)) != LSQ_OK)
      return st;
    if (r > 0 && (st = encode_tmap_2d(&maps.l[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, Bp[i], 64, W[i].n_out, 64 * 2,
                                      64, BK, CU_TENSOR_MAP_SWIZZLE_128B)) != LSQ_OK)
      return st;
  }
  p.nkb = blocks;
  dim3 grid((unsigned)((K + BN - 1) / BN), (unsigned)((M + BM - 1) / BM));
  if (BN == 192) return launch<DX, 192>(maps, p, grid, stream);
  return launch<DX, 128>(maps, p, grid, stream);
}

}  // namespace tc
}  // namespace lsq

extern "C" lsq_status lsq_nf4_lora_fwd_multi(int32_t nseg, const lsq_nf4_weight* W, const void* x, int64_t M,
                                             const void* const* A, const void* const* B, int32_t r, float s,
                                             const void* const* residual, void* const* y, float* const* u_out,
                                             lsq_cuda_stream stream) {
  using namespace lsq;
  using namespace lsq::nf4g;
  const char* who = "lsq_nf4_lora_fwd";
  if (nseg < 1 || nseg > 3) return fail(LSQ_EINVAL, "%s: 1..3 segments (got %d)", who, nseg);
  if (!W || !x || !y) return fail(LSQ_EINVAL, "%s: NULL argument", who);
  const int64_t K = W[0].k_in;
  lsq_status st = tc::nf4_checks(M, K, r, who);
  if (st != LSQ_OK) return st;
  if (!aligned(x, 16)) return fail(LSQ_EINVAL, "%s: x must be 16-byte aligned", who);
  Params p;
  memset(&p, 0, sizeof(p));
  p.nseg = nseg;
  p.M = (int)M;
  p.K = (int)K;
  p.r = r;
  p.rp = r > 0 ? (r + 15) / 16 * 16 : 0;
  p.s = s;
  p.nkb = (int)(K / BK);
  fill_cb(p);
  int64_t ns[3];
  for (int i = 0; i < nseg; ++i) {
    if ((st = tc::check_weight(W[i], K, who)) != LSQ_OK) return st;
    ns[i] = W[i].n_out;
  }
  const int BN = pick_bn(ns, nseg, M, true);
  Maps maps;
  memset(&maps, 0, sizeof(maps));
  if ((st = encode_tmap_2d(&maps.a[0], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, K, M, K * 2, BK, BM,
                           CU_TENSOR_MAP_SWIZZLE_128B)) != LSQ_OK)
    return st;
  int tiles = 0;
  for (int i = 0; i < nseg; ++i) {
    if (!y[i] || !aligned(y[i], 16)) return fail(LSQ_EINVAL, "%s: y[%d] NULL or not 16-byte aligned", who, i);
    const void* res = residual ? residual[i] : nullptr;
    if (res && !aligned(res, 16)) return fail(LSQ_EINVAL, "%s: residual must be 16-byte aligned", who);
    if (r > 0) {
      if (!A || !B || !A[i] || !B[i]) return fail(LSQ_EINVAL, "%s: LoRA A/B NULL with r > 0", who);
      if (!aligned(A[i], 16) || !aligned(B[i], 2)) return fail(LSQ_EINVAL, "%s: LoRA A must be 16-byte aligned", who);
    }
    Seg& g = p.seg[i];
    g.absmax = W[i].absmax;
    g.la = r > 0 ? static_cast<const __nv_bfloat16*>(A[i]) : nullptr;
    g.lb = r > 0 ? static_cast<const __nv_bfloat16*>(B[i]) : nullptr;
    g.y = static_cast<__nv_bfloat16*>(y[i]);
    g.res = static_cast<const __nv_bfloat16*>(res);
    g.uo = (u_out && r > 0) ? u_out[i] : nullptr;
    g.n = (int)W[i].n_out;
    g.first = tiles;
    tiles += (int)((W[i].n_out + BN - 1) / BN);
    if ((st = encode_tmap_2d(&maps.c[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, W[i].codes, K / 2, W[i].n_out, K / 2, BK / 2,
                             BN, CU_TENSOR_MAP_SWIZZLE_NONE)) != LSQ_OK)
      return st;
    if (r > 0 && (st = encode_tmap_2d(&maps.l[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A[i], K, r, K * 2, BK, p.rp,
                                      CU_TENSOR_MAP_SWIZZLE_128B)) != LSQ_OK)
      return st;
  }
  dim3 grid(tiles, (unsigned)((M + BM - 1) / BM));
  if (BN == 192) return launch<FWD, 192>(maps, p, grid, (cudaStream_t)stream);
  return launch<FWD, 128>(maps, p, grid, (cudaStream_t)stream);
}

extern "C" lsq_status lsq_nf4_lora_fwd(const lsq_nf4_weight* W, const void* x, int64_t M, const void* A,
                                       const void* B, int32_t r, float s, const void* residual, void* y,
                                       float* u_out, lsq_cuda_stream stream) {
  const void* a[1] = {A};
  const void* b[1] = {B};
  const void* res[1] = {residual};
  void* yy[1] = {y};
  float* uu[1] = {u_out};
  return lsq_nf4_lora_fwd_multi(1, W, x, M, a, b, r, s, res, yy, uu, stream);
}
