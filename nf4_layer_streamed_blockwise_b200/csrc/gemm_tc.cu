// Tensor-core GEMMs of the streamed NF4-LoRA path on sm_100a (tcgen05 + TMEM).
//
//   NF4_FWD : Y = residual + X deq(W)^T + s (X A^T) B^T,  U = X A^T
//   NF4_DX  : dX = sum_seg dY_seg deq(W_seg) + s sum_seg G_seg A_seg,  G_seg = dY_seg B_seg
//   DENSE_NT: out = a b^T      (lm_head forward, b = [N, K])
//   DENSE_NN: out = a b        (lm_head input gradient, b = [K, N])
//
// One CTA computes a 128 x 256 output tile; contraction blocks of 64.
// Warp roles (14 warps):
//   0-3   epilogue warpgroup: TMEM -> registers -> global; also the LoRA
//         epilogue operands (s*U or s*G as bf16, and B or A^T) in smem
//   4     TMA producer (activation tiles; the bf16 weight tiles of DENSE_*)
//   5     MMA issuer (one thread) + TMEM owner
//   6-13  NF4 dequantisers: packed codes + absmax -> bf16 tile in the 128-byte
//         swizzled canonical layout the tensor core reads (K-major for the
//         forward, MN-major for dX), plus the LoRA operand of the main loop
// Pipeline: NST shared-memory stages; full[s] completes when TMA bytes landed
// and every dequant warp arrived; empty[s] is armed by tcgen05.commit once the
// MMAs reading stage s retire.  The accumulator (fp32, 256 TMEM columns) and
// the rank-r product U or G (up to 64 more columns) live in TMEM.
// All waits are bounded (common.cuh); nothing here uses atomics, so every
// result is deterministic and independent of buffer addresses.
#include "common.cuh"
#include "host_common.h"

namespace lsq {
namespace tc {

enum Mode { NF4_FWD = 0, NF4_DX = 1, DENSE_NT = 2, DENSE_NN = 3 };

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int NTHREADS = 448;
constexpr int TMA_WARP = 4, MMA_WARP = 5, DQ_WARP0 = 6;
constexpr int KE_MAX = 64;  // columns of the rank-r products held in TMEM
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int L_BYTES = KE_MAX * BK * 2;   // LoRA operand of the main loop (rp rows x 64)
constexpr int C_BYTES = BN * BK / 2;       // packed NF4 codes of one stage (8 KB)
constexpr int UE_BYTES = BM * KE_MAX * 2;
constexpr int BE_BYTES = BN * KE_MAX * 2;
constexpr uint32_t TMEM_COLS = 512;

// Shared memory.  The epilogue's LoRA operands (UE, BE) alias the activation
// stages: they are written only after every main-loop MMA has retired.
template <int MODE>
struct Layout {
  static constexpr bool NF4 = (MODE == NF4_FWD || MODE == NF4_DX);
  static constexpr int NST = NF4 ? 3 : 4;
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + NST * A_BYTES;
  static constexpr int OFF_C = OFF_B + NST * B_BYTES;
  static constexpr int OFF_L = OFF_C + (NF4 ? NST * C_BYTES : 0);
  static constexpr int OFF_BAR = OFF_L + (NF4 ? NST * L_BYTES : 0);
  static constexpr int OFF_UE = OFF_A;
  static constexpr int OFF_BE = OFF_A + UE_BYTES;
  static_assert(!NF4 || UE_BYTES + BE_BYTES <= NST * (A_BYTES + B_BYTES), "epilogue operands must fit the stages");
  static constexpr int NBAR = 3 * NST + 4;
  static constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;
  static constexpr int BYTES = OFF_MISC + 128 + 1024;  // + alignment slack
};

struct Seg {
  const uint8_t* codes;
  const float* absmax;
  const __nv_bfloat16* la;   // LoRA A [r, K_in]
  const __nv_bfloat16* lb;   // LoRA B [n, r]
  __nv_bfloat16* y;          // forward output [M, n]
  const __nv_bfloat16* res;  // forward residual [M, n] or null
  float* uo;                 // U (forward) or G (dX) [M, r] or null
  int n;                     // rows of W (forward: output columns; dX: contraction length)
  int first;                 // forward: first n-tile of the segment; dX: first contraction block
};

struct Params {
  Seg seg[3];
  int nseg;
  int M, K, N;  // K: k_in (NF4) or contraction (dense); N: dense output columns
  int r, rp;    // LoRA rank and its padding to a multiple of 16 (0: no LoRA)
  float s;
  float cb[16];
  void* out;    // NF4_DX: dx [M, K] bf16 (may be null); DENSE: [M, N]
  int out_f32;
  int nkb;      // contraction blocks
};

struct Maps {
  CUtensorMap a[3];  // activation (forward: x; dX: dy of each segment)
  CUtensorMap b;     // dense: bf16 weight
  CUtensorMap c[3];  // NF4: packed codes of each segment (uint8 [n, K/2])
  CUtensorMap l[3];  // forward: LoRA A of each segment (bf16 [r, K], box rp rows)
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

// four packed code bytes -> eight bf16 (first element of a byte = high nibble)
__device__ __forceinline__ uint32_t dq_pair(uint32_t byte, float a, const float* cb) {
  return pack_bf16x2(__fmul_rn(cb[(byte >> 4) & 15], a), __fmul_rn(cb[byte & 15], a));
}
__device__ __forceinline__ uint4 dq8(uint32_t w, float a, const float* cb) {
  uint4 o;
  o.x = dq_pair(w & 0xFF, a, cb);
  o.y = dq_pair((w >> 8) & 0xFF, a, cb);
  o.z = dq_pair((w >> 16) & 0xFF, a, cb);
  o.w = dq_pair(w >> 24, a, cb);
  return o;
}

// 64 dequantised values (one NF4 block) -> one 128-byte row of a 128B-swizzled
// tile; `row` is the row index inside its 1024-byte swizzle atom group.
__device__ __forceinline__ void store_block_row(uint32_t row_addr, int row, uint4 c0, uint4 c1, float a,
                                                const float* cb) {
  const uint32_t w[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
#pragma unroll
  for (int j = 0; j < 8; ++j) st_shared_v4(row_addr + ((uint32_t)(j ^ (row & 7)) << 4), dq8(w[j], a, cb));
}

template <int MODE>
__global__ void __launch_bounds__(NTHREADS, 1) gemm_kernel(const __grid_constant__ Maps maps,
                                                           const __grid_constant__ Params p) {
  using L = Layout<MODE>;
  constexpr int NST = L::NST;
  constexpr bool NF4 = L::NF4;
  constexpr int B_MN = (MODE == NF4_DX || MODE == DENSE_NN) ? 1 : 0;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::OFF_BAR);
  uint64_t* empty = full + NST;
  uint64_t* cfull = empty + NST;  // packed codes of stage s landed (NF4)
  uint64_t* ufull = cfull + NST;
  uint64_t* lready = ufull + 1;
  uint64_t* afull = ufull + 2;
  uint64_t* drain = ufull + 3;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + L::OFF_MISC);
  float* s_cb = reinterpret_cast<float*>(smem + L::OFF_MISC + 16);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.y * BM;
  int seg = 0;
  int tile = blockIdx.x;
  if (MODE == NF4_FWD) {
    while (seg + 1 < p.nseg && (int)blockIdx.x >= p.seg[seg + 1].first) ++seg;
    tile = blockIdx.x - p.seg[seg].first;
  }
  const int n0 = tile * BN;  // forward: column in the segment; dX: k_in column; dense: column
  const bool lora = NF4 && p.rp > 0;
  const int KE = (MODE == NF4_DX) ? p.nseg * p.rp : p.rp;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1 + (NF4 ? 8 : 0));
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
  if (warp == MMA_WARP) {
    tmem_alloc(s_tmem, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == TMA_WARP) {
    // ------------------------------------------------------------ TMA producer
    // per stage: the activation tile, the bf16 weight tile (dense) or the
    // packed NF4 codes (into their own buffer, signalled on cfull[s]) and, in
    // the forward, the LoRA-down tile A[0:rp, k-block] (rows >= r read as 0).
    if (lane == 0) {
      tma_prefetch_desc(&maps.a[0]);
      for (int i = 0; i < p.nkb; ++i) {
        const int s = i % NST;
        const uint32_t ph = (uint32_t)(i / NST) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, 401)) break;
        uint8_t* a_dst = smem + L::OFF_A + s * A_BYTES;
        uint8_t* b_dst = smem + L::OFF_B + s * B_BYTES;
        uint32_t bytes = A_BYTES;
        if (!NF4) bytes += B_BYTES;
        if (MODE == NF4_FWD && lora) bytes += p.rp * 128;
        mbar_arrive_expect_tx(&full[s], bytes);
        if (MODE == NF4_DX) {
          const int sg = seg_of_block(p, i);
          const int nb = i - p.seg[sg].first;
          tma_load_2d(a_dst, &maps.a[sg], &full[s], nb * BK, m0);
          mbar_arrive_expect_tx(&cfull[s], C_BYTES);
          tma_load_2d(smem + L::OFF_C + s * C_BYTES, &maps.c[sg], &cfull[s], n0 / 2, nb * BK);
        } else {
          tma_load_2d(a_dst, &maps.a[0], &full[s], i * BK, m0);
        }
        if (MODE == NF4_FWD) {
          mbar_arrive_expect_tx(&cfull[s], C_BYTES);
          tma_load_2d(smem + L::OFF_C + s * C_BYTES, &maps.c[seg], &cfull[s], i * (BK / 2), n0);
          if (lora) tma_load_2d(smem + L::OFF_L + s * L_BYTES, &maps.l[seg], &full[s], i * BK, 0);
        }
        if (MODE == DENSE_NT) tma_load_2d(b_dst, &maps.b, &full[s], i * BK, n0);
        if (MODE == DENSE_NN) {
#pragma unroll
          for (int c = 0; c < BN / 64; ++c) tma_load_2d(b_dst + c * 8192, &maps.b, &full[s], n0 + c * 64, i * BK);
        }
      }
    }
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_main = idesc_bf16(BM, BN, 0, B_MN);
      const uint32_t id_lora = idesc_bf16(BM, p.rp > 0 ? p.rp : 16, 0, 0);
      const uint32_t id_ep = idesc_bf16(BM, BN, 0, 0);
      bool ok = true;
      for (int i = 0; i < p.nkb; ++i) {
        const int s = i % NST;
        const uint32_t ph = (uint32_t)(i / NST) & 1u;
        if (!mbar_wait(&full[s], ph, 501)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_base = smem_u32(smem + L::OFF_A + s * A_BYTES);
        const uint32_t b_base = smem_u32(smem + L::OFF_B + s * B_BYTES);
        uint32_t ucol = BN;
        bool first = (i == 0);
        if (MODE == NF4_DX) {
          const int sg = seg_of_block(p, i);
          ucol = BN + sg * p.rp;
          first = (i == p.seg[sg].first);
        }
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t ad = smem_desc(a_base + kk * 32, 16, 1024, 2);
          const uint64_t bd = B_MN ? smem_desc(b_base + kk * 2048, 8192, 1024, 2)
                                   : smem_desc(b_base + kk * 32, 16, 1024, 2);
          tc_mma(tmem, ad, bd, id_main, (i | kk) != 0);
          if (lora) {
            const uint32_t l_base = smem_u32(smem + L::OFF_L + s * L_BYTES);
            tc_mma(tmem + ucol, ad, smem_desc(l_base + kk * 32, 16, 1024, 2), id_lora, !(first && kk == 0));
          }
        }
        tc_commit(&empty[s]);
      }
      if (ok) {
        tc_commit(ufull);
        if (lora) {
          if (mbar_wait(lready, 0, 502)) {
            tc_fence_after();
            const uint32_t ue = smem_u32(smem + L::OFF_UE), be = smem_u32(smem + L::OFF_BE);
            for (int kk = 0; kk < KE / 16; ++kk)
              tc_mma(tmem, smem_desc(ue + kk * 256, 128, KE * 16, 0), smem_desc(be + kk * 256, 128, KE * 16, 0), id_ep,
                     1);
            tc_commit(afull);
          } else {
            ok = false;
          }
        }
      }
      if (!ok) {  // let every issued MMA retire before TMEM is released
        tc_commit(drain);
        mbar_wait(drain, 0, 503);
      }
    }
  } else if (warp >= DQ_WARP0) {
    // ------------------------------------------------------------ NF4 dequantisers
    // Each thread turns one 64-element NF4 block per stage (32 code bytes from
    // the TMA-filled codes tile, one absmax from registers, fetched ahead) into
    // one 128-byte row of the swizzled bf16 operand tile.
    if (NF4) {
      const int t = threadIdx.x - DQ_WARP0 * 32;  // 0..255
      const int KB = p.K / 64;
      if (MODE == NF4_FWD) {
        const Seg& sg = p.seg[seg];
        const int n = n0 + t;
        const bool valid = n < sg.n;
        const float* arow = sg.absmax + (int64_t)(valid ? n : 0) * KB;
        // absmax: four blocks per 16-byte load when rows are 16-byte aligned,
        // one group fetched ahead; else a 2-deep scalar prefetch
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
          float a;
          if (vec) {
            const int q = i & 3;
            a = q == 0 ? acur.x : q == 1 ? acur.y : q == 2 ? acur.z : acur.w;
          } else {
            a = s0;
          }
          if (!mbar_wait(&cfull[s], ph, 601)) break;
          const uint8_t* crow = smem + L::OFF_C + s * C_BYTES + t * 32;
          const uint4 c0 = *reinterpret_cast<const uint4*>(crow);
          const uint4 c1 = *reinterpret_cast<const uint4*>(crow + 16);
          store_block_row(smem_u32(smem + L::OFF_B + s * B_BYTES) + t * 128, t, c0, c1, valid ? a : 0.0f, s_cb);
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&full[s]);
          if (valid) {
            if (vec) {
              if ((i & 3) == 3) {
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
      } else {  // NF4_DX: tile = 64 contraction rows (n) x 256 output columns (k)
        const int nl = t >> 2, kc = t & 3;
        const int kcol = n0 + kc * 64;
        const int jq = p.rp / 4;  // LoRA B^T values per thread (rp <= 64 -> <= 16)
        const int bn = t & 63, bj0 = (t >> 6) * jq;
        float a_nx = 0.f;
        uint16_t bl_nx[16];
        // fetch absmax and the LoRA operand of contraction block i
        auto fetch = [&](int i, float& a, uint16_t* bl) {
          const int sgi = seg_of_block(p, i);
          const Seg& sg = p.seg[sgi];
          const int nrow = (i - sg.first) * BK + nl;
          a = (nrow < sg.n && kcol < p.K) ? __ldg(sg.absmax + (int64_t)nrow * KB + kcol / 64) : 0.0f;
          if (lora) {
            const int brow = (i - sg.first) * BK + bn;
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const int j = bj0 + q;
              bl[q] = 0;
              if (q < jq && j < p.r && brow < sg.n)
                bl[q] = __ldg(reinterpret_cast<const unsigned short*>(sg.lb) + (int64_t)brow * p.r + j);
            }
          }
        };
        if (p.nkb > 0) fetch(0, a_nx, bl_nx);
        for (int i = 0; i < p.nkb; ++i) {
          const int s = i % NST;
          const uint32_t ph = (uint32_t)(i / NST) & 1u;
          const float a = a_nx;
          uint16_t bl[16];
#pragma unroll
          for (int q = 0; q < 16; ++q) bl[q] = bl_nx[q];
          if (i + 1 < p.nkb) fetch(i + 1, a_nx, bl_nx);
          if (!mbar_wait(&cfull[s], ph, 602)) break;
          const uint8_t* crow = smem + L::OFF_C + s * C_BYTES + nl * 128 + kc * 32;
          const uint4 c0 = *reinterpret_cast<const uint4*>(crow);
          const uint4 c1 = *reinterpret_cast<const uint4*>(crow + 16);
          store_block_row(smem_u32(smem + L::OFF_B + s * B_BYTES) + kc * 8192 + nl * 128, nl, c0, c1, a, s_cb);
          if (lora) {
            const uint32_t lbase = smem_u32(smem + L::OFF_L + s * L_BYTES);
#pragma unroll
            for (int q = 0; q < 16; ++q) {
              const int j = bj0 + q;
              if (q < jq)
                st_shared_u16(lbase + j * 128 + ((uint32_t)((bn >> 3) ^ (j & 7)) << 4) + (bn & 7) * 2, bl[q]);
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) mbar_arrive(&full[s]);
        }
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue (warps 0-3)
    const int e = threadIdx.x;  // accumulator row / TMEM lane
    const int m = m0 + e;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    bool ok = mbar_wait(ufull, 0, 701);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) tc_fence_after();
    if (ok && lora) {
      // Every main-loop MMA has retired: the stage buffers are free and hold
      // the epilogue's LoRA operands now (no-swizzle K-major):
      //   sBe [BN rows x KE]: forward B[n0 + row, j]; dX A_seg[j, n0 + row] at column seg*rp + j
      //   sUe [128 rows x KE]: s*U (forward) or s*G (dX) as bf16
      const uint32_t be = smem_u32(smem + L::OFF_BE);
      for (int row = e; row < BN; row += 128) {
        for (int jc = 0; jc < KE / 8; ++jc) {
          uint32_t w[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            float v2[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              const int j = jc * 8 + q * 2 + h;
              float v = 0.0f;
              if (MODE == NF4_FWD) {
                const int n = n0 + row;
                if (j < p.r && n < p.seg[seg].n) v = __bfloat162float(p.seg[seg].lb[(int64_t)n * p.r + j]);
              } else {
                const int sg = j / p.rp, jj = j % p.rp, k = n0 + row;
                if (jj < p.r && k < p.K) v = __bfloat162float(p.seg[sg].la[(int64_t)jj * p.K + k]);
              }
              v2[h] = v;
            }
            w[q] = pack_bf16x2(v2[0], v2[1]);
          }
          st_shared_v4(be + (row >> 3) * (KE * 16) + jc * 128 + (row & 7) * 16, make_uint4(w[0], w[1], w[2], w[3]));
        }
      }
      const uint32_t ue = smem_u32(smem + L::OFF_UE);
      for (int c = 0; c < KE / 16; ++c) {
        float v[16];
        tmem_ld16(tmem + lane_base + BN + c * 16, v);
        tc_wait_ld();
        if (m < p.M) {
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const int j = c * 16 + q;
            if (MODE == NF4_FWD) {
              if (tile == 0 && p.seg[seg].uo && j < p.r) p.seg[seg].uo[(int64_t)m * p.r + j] = v[q];
            } else {
              const int sg = j / p.rp, jj = j % p.rp;
              if (blockIdx.x == 0 && p.seg[sg].uo && jj < p.r) p.seg[sg].uo[(int64_t)m * p.r + jj] = v[q];
            }
          }
        }
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint4 o;
          o.x = pack_bf16x2(v[h * 8 + 0] * p.s, v[h * 8 + 1] * p.s);
          o.y = pack_bf16x2(v[h * 8 + 2] * p.s, v[h * 8 + 3] * p.s);
          o.z = pack_bf16x2(v[h * 8 + 4] * p.s, v[h * 8 + 5] * p.s);
          o.w = pack_bf16x2(v[h * 8 + 6] * p.s, v[h * 8 + 7] * p.s);
          st_shared_v4(ue + (e >> 3) * (KE * 16) + (c * 2 + h) * 128 + (e & 7) * 16, o);
        }
      }
      fence_proxy_async_smem();
      named_bar_sync(1, 128);
      if (e == 0) mbar_arrive(lready);
      ok = mbar_wait(afull, 0, 702);
      ok = __all_sync(0xffffffffu, ok);
      if (ok) tc_fence_after();
    }
    if (ok) {
      for (int c = 0; c < BN / 32; ++c) {
        float v[32];
        tmem_ld32(tmem + lane_base + c * 32, v);
        tc_wait_ld();
        if (m >= p.M) continue;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int col = n0 + c * 32 + g * 8;
          float* x = v + g * 8;
          if (MODE == NF4_FWD) {
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
            const int ncols = (MODE == NF4_DX) ? p.K : p.N;
            if (col >= ncols || p.out == nullptr) continue;
            const int64_t off = (int64_t)m * ncols + col;
            if (p.out_f32) {
              float4* o = reinterpret_cast<float4*>(static_cast<float*>(p.out) + off);
              o[0] = make_float4(x[0], x[1], x[2], x[3]);
              o[1] = make_float4(x[4], x[5], x[6], x[7]);
            } else {
              *reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(p.out) + off) =
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
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem, TMEM_COLS);
  }
}

template <int MODE>
static lsq_status launch(const Maps& maps, const Params& p, dim3 grid, cudaStream_t stream) {
  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    LSQ_CUDA_TRY(cudaFuncSetAttribute(gemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      Layout<MODE>::BYTES));
    configured[dev] = 1;
  }
  gemm_kernel<MODE><<<grid, NTHREADS, Layout<MODE>::BYTES, stream>>>(maps, p);
  LSQ_LAUNCH_CHECK("gemm_kernel");
  return LSQ_OK;
}

static void fill_cb(Params& p) {
  const float* cb = codebook();
  for (int i = 0; i < 16; ++i) p.cb[i] = cb[i];
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

static lsq_status common_checks(int64_t M, int64_t K, int32_t r, const char* who) {
  lsq_status st = check_device();
  if (st != LSQ_OK) return st;
  if (M < 1 || M > (1 << 30)) return fail(LSQ_EINVAL, "%s: M out of range (%lld)", who, (long long)M);
  if (K < 64 || K % 64 != 0 || K > (1 << 30))
    return fail(LSQ_EINVAL, "%s: k_in must be a positive multiple of 64 (got %lld)", who, (long long)K);
  if (r < 0 || r > 64) return fail(LSQ_EINVAL, "%s: LoRA rank must be in [0, 64] (got %d)", who, r);
  return LSQ_OK;
}

}  // namespace tc
}  // namespace lsq

using namespace lsq;
using namespace lsq::tc;

extern "C" lsq_status lsq_nf4_lora_fwd_multi(int32_t nseg, const lsq_nf4_weight* W, const void* x, int64_t M,
                                             const void* const* A, const void* const* B, int32_t r, float s,
                                             const void* const* residual, void* const* y, float* const* u_out,
                                             lsq_cuda_stream stream) {
  const char* who = "lsq_nf4_lora_fwd";
  if (nseg < 1 || nseg > 3) return fail(LSQ_EINVAL, "%s: 1..3 segments (got %d)", who, nseg);
  if (!W || !x || !y) return fail(LSQ_EINVAL, "%s: NULL argument", who);
  const int64_t K = W[0].k_in;
  lsq_status st = common_checks(M, K, r, who);
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
  int tiles = 0;
  for (int i = 0; i < nseg; ++i) {
    if ((st = check_weight(W[i], K, who)) != LSQ_OK) return st;
    if (!y[i] || !aligned(y[i], 16)) return fail(LSQ_EINVAL, "%s: y[%d] NULL or not 16-byte aligned", who, i);
    const void* res = residual ? residual[i] : nullptr;
    if (res && !aligned(res, 16)) return fail(LSQ_EINVAL, "%s: residual must be 16-byte aligned", who);
    if (r > 0) {
      if (!A || !B || !A[i] || !B[i]) return fail(LSQ_EINVAL, "%s: LoRA A/B NULL with r > 0", who);
      if (!aligned(A[i], 16) || !aligned(B[i], 2)) return fail(LSQ_EINVAL, "%s: LoRA A must be 16-byte aligned", who);
    }
    Seg& g = p.seg[i];
    g.codes = W[i].codes;
    g.absmax = W[i].absmax;
    g.la = r > 0 ? static_cast<const __nv_bfloat16*>(A[i]) : nullptr;
    g.lb = r > 0 ? static_cast<const __nv_bfloat16*>(B[i]) : nullptr;
    g.y = static_cast<__nv_bfloat16*>(y[i]);
    g.res = static_cast<const __nv_bfloat16*>(res);
    g.uo = (u_out && r > 0) ? u_out[i] : nullptr;
    g.n = (int)W[i].n_out;
    g.first = tiles;
    tiles += (int)((W[i].n_out + BN - 1) / BN);
  }
  Maps maps;
  memset(&maps, 0, sizeof(maps));
  if ((st = encode_tmap_2d(&maps.a[0], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, x, K, M, K * 2, BK, BM,
                           CU_TENSOR_MAP_SWIZZLE_128B)) != LSQ_OK)
    return st;
  for (int i = 0; i < nseg; ++i) {
    // packed codes: rows of K/2 bytes, one stage = 256 rows x 32 bytes
    if ((st = encode_tmap_2d(&maps.c[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, W[i].codes, K / 2, W[i].n_out, K / 2,
                             BK / 2, BN, CU_TENSOR_MAP_SWIZZLE_NONE)) != LSQ_OK)
      return st;
    // LoRA A [r, K]: one stage = rp rows x 64 columns; rows r..rp-1 read as zero
    if (r > 0 && (st = encode_tmap_2d(&maps.l[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A[i], K, r, K * 2, BK, p.rp,
                                      CU_TENSOR_MAP_SWIZZLE_128B)) != LSQ_OK)
      return st;
  }
  dim3 grid(tiles, (unsigned)((M + BM - 1) / BM));
  return launch<NF4_FWD>(maps, p, grid, (cudaStream_t)stream);
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

// dX kernel: shared by lsq_nf4_lora_bwd*; writes G_seg into g_out[seg] ([M, r] fp32)
namespace lsq {
namespace tc {
lsq_status launch_dx(int nseg, const lsq_nf4_weight* W, const void* const* dy, int64_t M, const void* const* A,
                     const void* const* B, int r, float s, void* dx, float* const* g_out, cudaStream_t stream) {
  const int64_t K = W[0].k_in;
  Params p;
  memset(&p, 0, sizeof(p));
  p.nseg = nseg;
  p.M = (int)M;
  p.K = (int)K;
  p.r = r;
  p.rp = r > 0 ? (r + 15) / 16 * 16 : 0;
  p.s = s;
  p.out = dx;
  fill_cb(p);
  if (nseg * p.rp > KE_MAX) return fail(LSQ_EUNSUPPORTED, "lsq_nf4_lora_bwd: nseg * round16(r) must be <= 64");
  Maps maps;
  memset(&maps, 0, sizeof(maps));
  int blocks = 0;
  lsq_status st;
  for (int i = 0; i < nseg; ++i) {
    Seg& g = p.seg[i];
    g.codes = W[i].codes;
    g.absmax = W[i].absmax;
    g.la = r > 0 ? static_cast<const __nv_bfloat16*>(A[i]) : nullptr;
    g.lb = r > 0 ? static_cast<const __nv_bfloat16*>(B[i]) : nullptr;
    g.uo = r > 0 ? g_out[i] : nullptr;
    g.n = (int)W[i].n_out;
    g.first = blocks;
    blocks += (int)((W[i].n_out + BK - 1) / BK);
    if ((st = encode_tmap_2d(&maps.a[i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, dy[i], W[i].n_out, M, W[i].n_out * 2, BK,
                             BM, CU_TENSOR_MAP_SWIZZLE_128B)) != LSQ_OK)
      return st;
    // packed codes: one stage = 64 rows (contraction) x 128 bytes (256 output columns)
    if ((st = encode_tmap_2d(&maps.c[i], CU_TENSOR_MAP_DATA_TYPE_UINT8, W[i].codes, K / 2, W[i].n_out, K / 2,
                             BN / 2, BK, CU_TENSOR_MAP_SWIZZLE_NONE)) != LSQ_OK)
      return st;
  }
  p.nkb = blocks;
  dim3 grid((unsigned)((K + BN - 1) / BN), (unsigned)((M + BM - 1) / BM));
  return launch<NF4_DX>(maps, p, grid, stream);
}
}  // namespace tc
}  // namespace lsq

extern "C" lsq_status lsq_dense_gemm(const void* a, const void* b, void* out, int64_t M, int64_t N, int64_t K,
                                     int32_t trans_b, int32_t out_f32, lsq_cuda_stream stream) {
  const char* who = "lsq_dense_gemm";
  if (!a || !b || !out) return fail(LSQ_EINVAL, "%s: NULL argument", who);
  lsq_status st = check_device();
  if (st != LSQ_OK) return st;
  if (M < 1 || M > (1 << 30)) return fail(LSQ_EINVAL, "%s: M out of range (%lld)", who, (long long)M);
  if (K < 8 || K % 8 != 0 || K > (1 << 30))
    return fail(LSQ_EINVAL, "%s: K must be a positive multiple of 8 (got %lld)", who, (long long)K);
  if (N < 8 || N % 8 != 0 || N > (1 << 30)) return fail(LSQ_EINVAL, "%s: N must be a positive multiple of 8", who);
  if (!aligned(a, 16) || !aligned(b, 16) || !aligned(out, 16))
    return fail(LSQ_EINVAL, "%s: operands must be 16-byte aligned", who);
  Params p;
  memset(&p, 0, sizeof(p));
  p.nseg = 1;
  p.M = (int)M;
  p.K = (int)K;
  p.N = (int)N;
  p.out = out;
  p.out_f32 = out_f32 ? 1 : 0;
  p.nkb = (int)((K + BK - 1) / BK);  // the K tail reads as zeros (TMA out-of-bounds fill)
  Maps maps;
  memset(&maps, 0, sizeof(maps));
  if ((st = encode_tmap_2d(&maps.a[0], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a, K, M, K * 2, BK, BM,
                           CU_TENSOR_MAP_SWIZZLE_128B)) != LSQ_OK)
    return st;
  dim3 grid((unsigned)((N + BN - 1) / BN), (unsigned)((M + BM - 1) / BM));
  if (!trans_b) {
    if ((st = encode_tmap_2d(&maps.b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, b, K, N, K * 2, BK, BN,
                             CU_TENSOR_MAP_SWIZZLE_128B)) != LSQ_OK)
      return st;
    return launch<DENSE_NT>(maps, p, grid, (cudaStream_t)stream);
  }
  if ((st = encode_tmap_2d(&maps.b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, b, N, K, N * 2, 64, BK,
                           CU_TENSOR_MAP_SWIZZLE_128B)) != LSQ_OK)
    return st;
  return launch<DENSE_NN>(maps, p, grid, (cudaStream_t)stream);
}
