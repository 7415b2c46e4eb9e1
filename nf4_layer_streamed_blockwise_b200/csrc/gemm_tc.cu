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
