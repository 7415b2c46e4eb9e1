// Dense bf16 GEMMs for the resident, unquantised lm_head, sm_100a (tcgen05 +
// TMEM + TMA):
//   NT: out = a b^T      (logits = h E^T, b = [N, K])
//   NN: out = a b        (input gradient dh = dlogits E, b = [K, N])
//
// One CTA computes a 128 x 256 output tile; contraction blocks of 64, 4
// shared-memory stages filled by TMA (128-byte swizzle; for NN the weight
// tile is loaded as four 64-column boxes in the MN-major canonical layout).
// The row-tile index varies fastest across the grid, so the CTAs that share a
// 256-row slice of the weight run together and read it from DRAM once (for
// the logits, E [V, d] is 1 GB: with the column index fastest each slice came
// back from DRAM once per row tile, 16 times at 2048 tokens).
// Warps 0-3: epilogue (TMEM -> registers -> global, fp32 or bf16); warp 4:
// TMA producer; warp 5: MMA issuer + TMEM owner.  Bounded waits; no atomics.
//
// Chunked use (the lm_head streamed in vocabulary chunks): the operands and
// the output may be column blocks of wider row-major tensors (row strides
// lda, ldo), and a contraction can be split into consecutive K ranges: the
// call for a later range starts from the fp32 accumulator the earlier ranges
// left (acc_in), which the epilogue warps write into TMEM before the first
// MMA.  TMEM then holds exactly what an uninterrupted contraction holds at
// that point of its K loop, so with ranges cut at multiples of 64 the result
// is bit-identical to one call over the whole K.
#include "common.cuh"
#include "host_common.h"

namespace lsq {
namespace dense {

constexpr int BM = 128, BN = 256, BK = 64, NST = 4;
constexpr int NTHREADS = 192;
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + NST * A_BYTES;
constexpr int OFF_BAR = OFF_B + NST * B_BYTES;
constexpr int NBAR = 2 * NST + 3;
constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;
constexpr int BYTES = OFF_MISC + 64 + 1024;

struct Params {
  int M, N, K, nkb;
  void* out;
  int64_t ldo;            // output row stride (elements)
  const float* acc_in;    // fp32 accumulator to start from (row stride ldo), or null
  int out_f32;
};

struct Maps {
  CUtensorMap a, b;
};

template <int NN>
__global__ void __launch_bounds__(NTHREADS, 1) dense_gemm_kernel(const __grid_constant__ Maps maps,
                                                                 const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* empty = full + NST;
  uint64_t* afull = empty + NST;
  uint64_t* drain = afull + 1;
  uint64_t* ainit = drain + 1;  // the epilogue warps have written acc_in into TMEM
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * BM, n0 = blockIdx.y * BN;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(afull, 1);
    mbar_init(drain, 1);
    mbar_init(ainit, 4);
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(s_tmem, 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 4) {
    if (lane == 0) {
      for (int i = 0; i < p.nkb; ++i) {
        const int s = i % NST;
        const uint32_t ph = (uint32_t)(i / NST) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, 421)) break;
        uint8_t* b_dst = smem + OFF_B + s * B_BYTES;
        mbar_arrive_expect_tx(&full[s], (uint32_t)(A_BYTES + B_BYTES));
        tma_load_2d(smem + OFF_A + s * A_BYTES, &maps.a, &full[s], i * BK, m0);
        if (!NN) {
          tma_load_2d(b_dst, &maps.b, &full[s], i * BK, n0);
        } else {
#pragma unroll
          for (int c = 0; c < BN / 64; ++c) tma_load_2d(b_dst + c * 8192, &maps.b, &full[s], n0 + c * 64, i * BK);
        }
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      const uint32_t id = idesc_bf16(BM, BN, 0, NN);
      bool ok = true;
      if (p.acc_in) {
        ok = mbar_wait(ainit, 0, 523);
        tc_fence_after();
      }
      for (int i = 0; ok && i < p.nkb; ++i) {
        const int s = i % NST;
        const uint32_t ph = (uint32_t)(i / NST) & 1u;
        if (!mbar_wait(&full[s], ph, 521)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_base = smem_u32(smem + OFF_A + s * A_BYTES);
        const uint32_t b_base = smem_u32(smem + OFF_B + s * B_BYTES);
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          const uint64_t bd = NN ? smem_desc(b_base + kk * 2048, 8192, 1024, 2) : smem_desc(b_base + kk * 32, 16, 1024, 2);
          tc_mma(tmem, smem_desc(a_base + kk * 32, 16, 1024, 2), bd, id, p.acc_in != nullptr || (i | kk) != 0);
        }
        tc_commit(&empty[s]);
      }
      if (ok) {
        tc_commit(afull);
      } else {
        tc_commit(drain);
        mbar_wait(drain, 0, 522);
      }
    }
  } else {
    const int e = threadIdx.x;
    const int m = m0 + e;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    if (p.acc_in) {  // this row's accumulator so far -> TMEM (zeros outside the matrix)
      for (int c = 0; c < BN / 32; ++c) {
        float v[32];
#pragma unroll
        for (int g = 0; g < 8; ++g) {
          const int col = n0 + c * 32 + g * 4;
          float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
          if (m < p.M && col < p.N) x = *reinterpret_cast<const float4*>(p.acc_in + (int64_t)m * p.ldo + col);
          v[4 * g] = x.x;
          v[4 * g + 1] = x.y;
          v[4 * g + 2] = x.z;
          v[4 * g + 3] = x.w;
        }
        tmem_st32(tmem + lane_base + c * 32, v);
      }
      tc_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(ainit);
    }
    bool ok = mbar_wait(afull, 0, 721);
    ok = __all_sync(0xffffffffu, ok);
    if (ok) {
      tc_fence_after();
      for (int c = 0; c < BN / 32; ++c) {
        float v[32];
        tmem_ld32(tmem + lane_base + c * 32, v);
        tc_wait_ld();
        if (m >= p.M) continue;
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          const int col = n0 + c * 32 + g * 8;
          if (col >= p.N) continue;
          const float* x = v + g * 8;
          const int64_t off = (int64_t)m * p.ldo + col;
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

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// ---------------------------------------------------------------- persistent form
// Without acc_in the tiles go to a persistent grid (one CTA per SM, tile t, t + G, ... with the row
// tile fastest, as above) whose two TMEM accumulators (2 x 256 columns) alternate, so the epilogue
// of one tile runs under the products of the next.  The epilogue stages each warp's 32 rows x 32
// columns in shared memory (two buffers per warp; fp32 rows of 128 bytes in the 128-byte swizzle,
// bf16 rows of 64 bytes in the 64-byte one) and one lane stores the box with TMA, so the output
// leaves as whole lines; the accumulator goes back to the MMA issuer once its last columns are in
// registers.
constexpr int PSTG = 2;  // staging buffers per epilogue warp
template <int F32>
struct PCfg {
  static constexpr int STG = 32 * 32 * (F32 ? 4 : 2);
  static constexpr int OFF_STG = OFF_B + NST * B_BYTES;
  static constexpr int OFF_PBAR = OFF_STG + 4 * PSTG * STG;
  static constexpr int NPBAR = 2 * NST + 4;  // full, empty, tfull[2], tempty[2]
  static constexpr int OFF_PMISC = OFF_PBAR + 8 * NPBAR;
  static constexpr int PBYTES = OFF_PMISC + 64 + 1024;
  static_assert(PBYTES <= 232448, "shared memory");
};

__device__ __forceinline__ void sts_v4(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void wait_ld_dep(float (&v)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+f"(v[0]), "+f"(v[1]), "+f"(v[2]), "+f"(v[3]), "+f"(v[4]), "+f"(v[5]), "+f"(v[6]), "+f"(v[7]),
                 "+f"(v[8]), "+f"(v[9]), "+f"(v[10]), "+f"(v[11]), "+f"(v[12]), "+f"(v[13]), "+f"(v[14]),
                 "+f"(v[15]), "+f"(v[16]), "+f"(v[17]), "+f"(v[18]), "+f"(v[19]), "+f"(v[20]), "+f"(v[21]),
                 "+f"(v[22]), "+f"(v[23]), "+f"(v[24]), "+f"(v[25]), "+f"(v[26]), "+f"(v[27]), "+f"(v[28]),
                 "+f"(v[29]), "+f"(v[30]), "+f"(v[31])
               :
               : "memory");
}
// one lane's row of a 32 x 32 output chunk into its staged row at s_row: fp32 as eight 16-byte
// pieces, piece q at (q ^ (row % 8)) * 16; bf16 as four, piece q at (q ^ (row / 2 % 4)) * 16
template <int F32>
__device__ __forceinline__ void stage_row(const float (&v)[32], uint32_t s_row, int lane) {
  if (F32) {
#pragma unroll
    for (int q = 0; q < 8; ++q)
      sts_v4(s_row + ((uint32_t)(q ^ (lane & 7)) << 4),
             make_uint4(__float_as_uint(v[4 * q]), __float_as_uint(v[4 * q + 1]), __float_as_uint(v[4 * q + 2]),
                        __float_as_uint(v[4 * q + 3])));
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q)
      sts_v4(s_row + ((uint32_t)(q ^ ((lane >> 1) & 3)) << 4),
             make_uint4(pack_bf16x2(v[8 * q], v[8 * q + 1]), pack_bf16x2(v[8 * q + 2], v[8 * q + 3]),
                        pack_bf16x2(v[8 * q + 4], v[8 * q + 5]), pack_bf16x2(v[8 * q + 6], v[8 * q + 7])));
  }
}

struct PMaps {
  CUtensorMap a, b, out;  // out: [M, N] with row stride ldo, box 32 x 32 (swizzle as staged)
};

template <int NN, int F32>
__global__ void __launch_bounds__(NTHREADS, 1) dense_pgemm_kernel(const __grid_constant__ PMaps maps,
                                                                  const __grid_constant__ Params p) {
  using C = PCfg<F32>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::OFF_PBAR);
  uint64_t* empty = full + NST;
  uint64_t* tfull = empty + NST;
  uint64_t* tempty = tfull + 2;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + C::OFF_PMISC);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntm = (p.M + BM - 1) / BM, ntn = (p.N + BN - 1) / BN, tiles = ntm * ntn;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 1);
    }
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 4) {
    if (lane == 0) {
      uint32_t g = 0;
      bool ok = true;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x) {
        const int m0 = (t % ntm) * BM, n0 = (t / ntm) * BN;
        for (int i = 0; i < p.nkb; ++i, ++g) {
          const int s = (int)(g % NST);
          const uint32_t ph = (g / NST) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, 425)) {
            ok = false;
            break;
          }
          uint8_t* b_dst = smem + OFF_B + s * B_BYTES;
          mbar_arrive_expect_tx(&full[s], (uint32_t)(A_BYTES + B_BYTES));
          tma_load_2d(smem + OFF_A + s * A_BYTES, &maps.a, &full[s], i * BK, m0);
          if (!NN) {
            tma_load_2d(b_dst, &maps.b, &full[s], i * BK, n0);
          } else {
#pragma unroll
            for (int c = 0; c < BN / 64; ++c) tma_load_2d(b_dst + c * 8192, &maps.b, &full[s], n0 + c * 64, i * BK);
          }
        }
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      const uint32_t id = idesc_bf16(BM, BN, 0, NN);
      uint32_t g = 0;
      bool ok = true;
      int j = 0;
      for (int t = blockIdx.x; ok && t < tiles; t += gridDim.x, ++j) {
        const int buf = j & 1;
        if (!mbar_wait(&tempty[buf], ((uint32_t)(j >> 1) & 1u) ^ 1u, 526)) break;
        tc_fence_after();
        const uint32_t d = tmem + (uint32_t)(buf * BN);
        for (int i = 0; i < p.nkb; ++i, ++g) {
          const int s = (int)(g % NST);
          const uint32_t ph = (g / NST) & 1u;
          if (!mbar_wait(&full[s], ph, 527)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + OFF_A + s * A_BYTES);
          const uint32_t b_base = smem_u32(smem + OFF_B + s * B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t bd =
                NN ? smem_desc(b_base + kk * 2048, 8192, 1024, 2) : smem_desc(b_base + kk * 32, 16, 1024, 2);
            tc_mma(d, smem_desc(a_base + kk * 32, 16, 1024, 2), bd, id, (i | kk) != 0);
          }
          tc_commit(&empty[s]);
        }
        tc_commit(&tfull[buf]);  // also when a wait gave up: the epilogue is not left waiting
      }
    }
  } else {
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    uint8_t* stg = smem + C::OFF_STG + warp * PSTG * C::STG;
    int j = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++j) {
      const int m0 = (t % ntm) * BM, n0 = (t / ntm) * BN;
      const int buf = j & 1;
      const int row = m0 + warp * 32;  // the warp's first row
      if (!__all_sync(0xffffffffu, mbar_wait(&tfull[buf], (uint32_t)(j >> 1) & 1u, 726))) break;
      tc_fence_after();
      const int cvalid = min(BN / 32, (p.N - n0 + 31) / 32);
      for (int c = 0; c < cvalid; c += 2) {
        // chunk c + 1 < BN / 32 always exists in TMEM; past N it is loaded but not stored
        float va[32], vb[32];
        tmem_ld32(tmem + lane_base + (uint32_t)(buf * BN + c * 32), va);
        tmem_ld32(tmem + lane_base + (uint32_t)(buf * BN + (c + 1) * 32), vb);
        if (lane == 0) bulk_wait_read<0>();  // the last stores have read both buffers
        __syncwarp();
        wait_ld_dep(va);
        wait_ld_dep(vb);
        if (c + 2 >= cvalid) {  // the accumulator is in registers: hand it back
          tc_fence_before();
          named_bar_sync(1, 128);
          if (threadIdx.x == 0) mbar_arrive(&tempty[buf]);
        }
        if (row >= p.M) continue;  // warp-uniform
        const bool two = c + 1 < cvalid;
        const uint32_t s0 = smem_u32(stg) + (uint32_t)lane * (F32 ? 128 : 64);
        stage_row<F32>(va, s0, lane);
        if (two) stage_row<F32>(vb, s0 + C::STG, lane);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          tma_store_2d(&maps.out, stg, n0 + c * 32, row);
          if (two) tma_store_2d(&maps.out, stg + C::STG, n0 + (c + 1) * 32, row);
          bulk_commit();
        }
      }
    }
    if (lane == 0) bulk_wait_all();  // the staged stores are written before the CTA exits
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int NN, int F32>
static lsq_status launch_p(const PMaps& maps, const Params& p, cudaStream_t stream) {
  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    LSQ_CUDA_TRY(cudaFuncSetAttribute(dense_pgemm_kernel<NN, F32>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      PCfg<F32>::PBYTES));
    configured[dev] = 1;
  }
  const int64_t tiles = (int64_t)((p.M + BM - 1) / BM) * ((p.N + BN - 1) / BN);
  const int grid = (int)std::min<int64_t>(tiles, (int64_t)num_sms());
  dense_pgemm_kernel<NN, F32><<<grid, NTHREADS, PCfg<F32>::PBYTES, stream>>>(maps, p);
  LSQ_LAUNCH_CHECK("dense_pgemm_kernel");
  return LSQ_OK;
}

template <int NN>
static lsq_status launch(const Maps& maps, const Params& p, dim3 grid, cudaStream_t stream) {
  static int configured[64] = {0};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    LSQ_CUDA_TRY(cudaFuncSetAttribute(dense_gemm_kernel<NN>, cudaFuncAttributeMaxDynamicSharedMemorySize, BYTES));
    configured[dev] = 1;
  }
  dense_gemm_kernel<NN><<<grid, NTHREADS, BYTES, stream>>>(maps, p);
  LSQ_LAUNCH_CHECK("dense_gemm_kernel");
  return LSQ_OK;
}

}  // namespace dense
}  // namespace lsq

extern "C" lsq_status lsq_dense_gemm_ex(const void* a, int64_t lda, const void* b, void* out, int64_t ldo,
                                        const float* acc_in, int64_t M, int64_t N, int64_t K, int32_t trans_b,
                                        int32_t out_f32, lsq_cuda_stream stream) {
  using namespace lsq;
  using namespace lsq::dense;
  const char* who = "lsq_dense_gemm";
  if (!a || !b || !out) return fail(LSQ_EINVAL, "%s: NULL argument", who);
  lsq_status st = check_device();
  if (st != LSQ_OK) return st;
  if (M < 1 || M > (1 << 30)) return fail(LSQ_EINVAL, "%s: M out of range (%lld)", who, (long long)M);
  if (K < 8 || K % 8 != 0 || K > (1 << 30))
    return fail(LSQ_EINVAL, "%s: K must be a positive multiple of 8 (got %lld)", who, (long long)K);
  if (N < 8 || N % 8 != 0 || N > (1 << 30)) return fail(LSQ_EINVAL, "%s: N must be a positive multiple of 8", who);
  if (lda < K || lda % 8 != 0 || ldo < N || ldo % 8 != 0 || lda > (1ll << 31) || ldo > (1ll << 31))
    return fail(LSQ_EINVAL, "%s: lda >= K and ldo >= N, multiples of 8 (got %lld, %lld)", who, (long long)lda,
                (long long)ldo);
  if (!aligned(a, 16) || !aligned(b, 16) || !aligned(out, 16) || (acc_in && !aligned(acc_in, 16)))
    return fail(LSQ_EINVAL, "%s: operands must be 16-byte aligned", who);
  Params p;
  p.M = (int)M;
  p.N = (int)N;
  p.K = (int)K;
  p.nkb = (int)((K + BK - 1) / BK);  // the K tail reads as zeros (TMA out-of-bounds fill)
  p.out = out;
  p.ldo = ldo;
  p.acc_in = acc_in;
  p.out_f32 = out_f32 ? 1 : 0;
  Maps maps;
  memset(&maps, 0, sizeof(maps));
  if ((st = encode_tmap_2d(&maps.a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, a, K, M, lda * 2, BK, BM,
                           CU_TENSOR_MAP_SWIZZLE_128B)) != LSQ_OK)
    return st;
  if (!acc_in) {  // the persistent form (two accumulators, staged TMA stores)
    PMaps pm;
    memset(&pm, 0, sizeof(pm));
    pm.a = maps.a;
    if (!trans_b) {
      if ((st = encode_tmap_2d(&pm.b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, b, K, N, K * 2, BK, BN,
                               CU_TENSOR_MAP_SWIZZLE_128B)) != LSQ_OK)
        return st;
    } else if ((st = encode_tmap_2d(&pm.b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, b, N, K, N * 2, 64, BK,
                                    CU_TENSOR_MAP_SWIZZLE_128B)) != LSQ_OK) {
      return st;
    }
    if (out_f32) {
      if ((st = encode_tmap_2d(&pm.out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, out, N, M, ldo * 4, 32, 32,
                               CU_TENSOR_MAP_SWIZZLE_128B)) != LSQ_OK)
        return st;
      return trans_b ? launch_p<1, 1>(pm, p, (cudaStream_t)stream) : launch_p<0, 1>(pm, p, (cudaStream_t)stream);
    }
    if ((st = encode_tmap_2d(&pm.out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, out, N, M, ldo * 2, 32, 32,
                             CU_TENSOR_MAP_SWIZZLE_64B)) != LSQ_OK)
      return st;
    return trans_b ? launch_p<1, 0>(pm, p, (cudaStream_t)stream) : launch_p<0, 0>(pm, p, (cudaStream_t)stream);
  }
  if ((N + BN - 1) / BN > 65535) return fail(LSQ_EINVAL, "%s: N too large for the grid", who);
  dim3 grid((unsigned)((M + BM - 1) / BM), (unsigned)((N + BN - 1) / BN));
  if (!trans_b) {
    if ((st = encode_tmap_2d(&maps.b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, b, K, N, K * 2, BK, BN,
                             CU_TENSOR_MAP_SWIZZLE_128B)) != LSQ_OK)
      return st;
    return launch<0>(maps, p, grid, (cudaStream_t)stream);
  }
  if ((st = encode_tmap_2d(&maps.b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, b, N, K, N * 2, 64, BK,
                           CU_TENSOR_MAP_SWIZZLE_128B)) != LSQ_OK)
    return st;
  return launch<1>(maps, p, grid, (cudaStream_t)stream);
}

extern "C" lsq_status lsq_dense_gemm(const void* a, const void* b, void* out, int64_t M, int64_t N, int64_t K,
                                     int32_t trans_b, int32_t out_f32, lsq_cuda_stream stream) {
  return lsq_dense_gemm_ex(a, K, b, out, N, nullptr, M, N, K, trans_b, out_f32, stream);
}
