// Backward of the fused NF4-LoRA linear:
//   s*G = s [dY_seg B_seg]                      (split-K tensor-core kernel, gemm_nf4.cu)
//   dX = sum_seg dY_seg deq(W_seg) + (s G) A    (SM-pair tensor-core kernel, gemm_nf4.cu)
//   dA_seg = (s G_seg)^T X,  dB_seg = dY_seg^T (s U_seg)      (here)
// dA of every segment is one product X^T [s G_1 | s G_2 | ...] with N = 64
// columns (the segments' ranks side by side, zero-padded), dB of segment q is
// dY_q^T (s U_q) with N = 64: tensor-core GEMMs over the M token rows, both
// operands read "MN-major" straight from their row-major tensors by TMA.  The
// token range is split across CTAs; a second kernel adds the fp32 partials in
// a fixed order (no atomics, results bit-identical run to run) and writes the
// gradients in their own layouts (dA [r, k_in], dB [n_out, r]), overwriting or
// adding.  s*G and s*U are bf16, the tensor cores' input type.
#include <algorithm>

#include "common.cuh"
#include "host_common.h"

namespace lsq {
namespace lg {

constexpr int BM = 128;    // output rows per CTA (k for dA, n for dB)
constexpr int BN = 64;     // output columns (ranks, zero-padded)
constexpr int BKT = 64;    // token rows per stage
constexpr int NST = 4;
constexpr int A_BYTES = BM * BKT * 2;  // two 64-row MN chunks, 16 KB
constexpr int B_BYTES = BN * BKT * 2;  // 8 KB
constexpr int OFF_A = 0;
constexpr int OFF_B = OFF_A + NST * A_BYTES;
constexpr int OFF_BAR = OFF_B + NST * B_BYTES;
constexpr int NBAR = 2 * NST + 1;
constexpr int OFF_MISC = OFF_BAR + 8 * NBAR;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
constexpr int NTHREADS = 192;
constexpr int TARGET_CTAS = 296;
constexpr int MAXP = 4;  // dA + up to three dB

struct Prob {
  float* part;  // [splits][rows][64]
  int rows;     // k_in (dA) or n_out of the segment (dB)
  int first;    // first 128-row tile of this problem in the grid
};
struct Params {
  Prob pr[MAXP];
  int nprob, M, kbps, splits;
};
struct Maps {
  CUtensorMap a[MAXP];  // token-major activation side: x [M, k_in] or dy_q [M, n_q] (box 64 x 64 rows)
  CUtensorMap b[MAXP];  // token-major rank side: s*G or s*U_q [M, 64] (box 64 x 64 rows)
};

__global__ void __launch_bounds__(NTHREADS, 1) lora_grad_kernel(const __grid_constant__ Maps maps,
                                                                const __grid_constant__ Params p) {
  int pi = 0;
  while (pi + 1 < p.nprob && (int)blockIdx.x >= p.pr[pi + 1].first) ++pi;
  const Prob& P = p.pr[pi];
  const int r0 = ((int)blockIdx.x - P.first) * BM;
  const int split = blockIdx.y;
  const int nblk = (p.M + BKT - 1) / BKT;
  const int kb0 = split * p.kbps;
  const int nk = min(nblk, kb0 + p.kbps) - kb0;  // >= 1: splits = ceil(nblk / kbps)

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* empty = full + NST;
  uint64_t* done = empty + NST;
  uint32_t* s_tmem = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(done, 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(s_tmem, 64);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *s_tmem;

  if (warp == 0) {
    if (lane == 0) {
      for (int i = 0; i < nk; ++i) {
        const int s = i % NST;
        const uint32_t ph = (uint32_t)(i / NST) & 1u;
        if (!mbar_wait(&empty[s], ph ^ 1u, 451)) break;
        mbar_arrive_expect_tx(&full[s], (uint32_t)(A_BYTES + B_BYTES));
        const int y = (kb0 + i) * BKT;
        uint8_t* a = smem + OFF_A + s * A_BYTES;
        tma_load_2d(a, &maps.a[pi], &full[s], r0, y);
        tma_load_2d(a + A_BYTES / 2, &maps.a[pi], &full[s], r0 + 64, y);
        tma_load_2d(smem + OFF_B + s * B_BYTES, &maps.b[pi], &full[s], 0, y);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t id = idesc_bf16(BM, BN, 1, 1);  // both operands MN-major (contiguous along rows / ranks)
      bool ok = true;
      for (int i = 0; i < nk; ++i) {
        const int s = i % NST;
        const uint32_t ph = (uint32_t)(i / NST) & 1u;
        if (!mbar_wait(&full[s], ph, 551)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a = smem_u32(smem + OFF_A + s * A_BYTES);
        const uint32_t b = smem_u32(smem + OFF_B + s * B_BYTES);
#pragma unroll
        for (int kk = 0; kk < BKT / 16; ++kk)  // 16 tokens = 16 rows of 128 bytes
          tc_mma(tmem, smem_desc(a + kk * 2048, A_BYTES / 2, 1024, 2), smem_desc(b + kk * 2048, B_BYTES, 1024, 2),
                 id, (i | kk) != 0);
        tc_commit(&empty[s]);
      }
      tc_commit(done);
      if (!ok) mbar_wait(done, 0, 552);
    }
  } else {
    const int qd = warp & 3;
    const int row = r0 + qd * 32 + lane;
    const uint32_t lane_base = (uint32_t)(qd * 32) << 16;
    if (__all_sync(0xffffffffu, mbar_wait(done, 0, 751))) {
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < BN / 32; ++c) {
        float v[32];
        tmem_ld32(tmem + lane_base + (uint32_t)(c * 32), v);
        tc_wait_ld();
        if (row < P.rows) {
          float4* dst = reinterpret_cast<float4*>(P.part + ((int64_t)split * P.rows + row) * BN + c * 32);
#pragma unroll
          for (int q = 0; q < 8; ++q) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 64);
  }
}

// Adds the splits (ascending) and writes the gradients.
//   dA (problem 0): blocks of 32 k-rows; dA_q[j][k] = sum part[k][q*rp + j],
//                   transposed through shared memory so both sides coalesce
//   dB_q (problem q + 1): dB_q[n][j] = sum part[n][j]
struct Red {
  const float* part[MAXP];
  int rows[MAXP];
  int blocks[MAXP];  // reduce blocks of each problem
  float* dA[3];
  float* dB[3];
  int nseg, r, rp, splits, accumulate;
};

__global__ void __launch_bounds__(256) lora_grad_reduce(const __grid_constant__ Red R) {
  __shared__ float tile[32][65];
  int pi = 0, b = blockIdx.x;
  while (b >= R.blocks[pi]) {
    b -= R.blocks[pi];
    ++pi;
  }
  const int rows = R.rows[pi];
  const float* part = R.part[pi];
  if (pi == 0) {
    const int k0 = b * 32;
    for (int e = threadIdx.x; e < 32 * BN; e += 256) {
      const int rl = e / BN, c = e % BN, k = k0 + rl;
      float sum = 0.0f;
      if (k < rows)
        for (int sp = 0; sp < R.splits; ++sp) sum += part[((int64_t)sp * rows + k) * BN + c];
      tile[rl][c] = sum;
    }
    __syncthreads();
    const int live = R.nseg * R.r;
    for (int e = threadIdx.x; e < 32 * live; e += 256) {
      const int kl = e % 32, qj = e / 32, q = qj / R.r, j = qj % R.r, k = k0 + kl;
      if (k >= rows) continue;
      float* dst = R.dA[q] + (int64_t)j * rows + k;
      const float v = tile[kl][q * R.rp + j];
      *dst = R.accumulate ? *dst + v : v;
    }
  } else {
    const int q = pi - 1;
    const int64_t n_el = (int64_t)rows * R.r;
    for (int64_t e = (int64_t)b * 256 + threadIdx.x; e < n_el && e < ((int64_t)b + 1) * 256; e += 256) {
      const int64_t n = e / R.r;
      const int j = (int)(e % R.r);
      float sum = 0.0f;
      for (int sp = 0; sp < R.splits; ++sp) sum += part[((int64_t)sp * rows + n) * BN + j];
      float* dst = R.dB[q] + e;
      *dst = R.accumulate ? *dst + sum : sum;
    }
  }
}

struct Plan {
  int kbps, splits, tiles;
  size_t part[MAXP], total;
};
static Plan plan(int nseg, int64_t M, int64_t K, const int64_t* n_out) {
  Plan pl;
  memset(&pl, 0, sizeof(pl));
  const int64_t rows[MAXP] = {K, nseg > 0 ? n_out[0] : 0, nseg > 1 ? n_out[1] : 0, nseg > 2 ? n_out[2] : 0};
  for (int i = 0; i <= nseg; ++i) pl.tiles += (int)((rows[i] + BM - 1) / BM);
  const int nblk = (int)((M + BKT - 1) / BKT);
  int want = (TARGET_CTAS + pl.tiles - 1) / pl.tiles;
  want = std::max(1, std::min(want, std::min(4, nblk)));
  pl.kbps = (nblk + want - 1) / want;
  pl.splits = (nblk + pl.kbps - 1) / pl.kbps;
  for (int i = 0; i <= nseg; ++i) {
    pl.part[i] = ((size_t)pl.splits * (size_t)rows[i] * BN * sizeof(float) + 255) / 256 * 256;
    pl.total += pl.part[i];
  }
  return pl;
}

static lsq_status tmap_rows(CUtensorMap* m, const void* base, int64_t inner, int64_t M) {
  return encode_tmap_2d(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, (uint64_t)inner, (uint64_t)M,
                        (uint64_t)inner * 2, 64, BKT, CU_TENSOR_MAP_SWIZZLE_128B);
}

// dA of every segment and dB of each: partial GEMMs, then the ordered reduction
static lsq_status launch(int nseg, int64_t M, int64_t K, const int64_t* n_out, const void* x, const void* const* dy,
                         const __nv_bfloat16* sg, __nv_bfloat16* const* su, float* const* dA, float* const* dB,
                         int r, int rp, int accumulate, char* ws, cudaStream_t stream) {
  const Plan pl = plan(nseg, M, K, n_out);
  Maps maps;
  memset(&maps, 0, sizeof(maps));
  Params p;
  memset(&p, 0, sizeof(p));
  Red R;
  memset(&R, 0, sizeof(R));
  p.nprob = nseg + 1;
  p.M = (int)M;
  p.kbps = pl.kbps;
  p.splits = pl.splits;
  lsq_status st;
  int first = 0;
  char* cur = ws;
  for (int i = 0; i <= nseg; ++i) {
    const int64_t rows = i == 0 ? K : n_out[i - 1];
    if ((st = tmap_rows(&maps.a[i], i == 0 ? x : dy[i - 1], rows, M)) != LSQ_OK) return st;
    if ((st = tmap_rows(&maps.b[i], i == 0 ? (const void*)sg : (const void*)su[i - 1], 64, M)) != LSQ_OK)
      return st;
    Prob& pr = p.pr[i];
    pr.part = reinterpret_cast<float*>(cur);
    pr.rows = (int)rows;
    pr.first = first;
    first += (int)((rows + BM - 1) / BM);
    cur += pl.part[i];
    R.part[i] = pr.part;
    R.rows[i] = (int)rows;
    R.blocks[i] = i == 0 ? (int)((rows + 31) / 32) : (int)((rows * r + 255) / 256);
  }
  static int configured[64] = {0};
  int dev = 0;
  LSQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev >= 0 && dev < 64 && !configured[dev]) {
    LSQ_CUDA_TRY(cudaFuncSetAttribute(lora_grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES));
    configured[dev] = 1;
  }
  lora_grad_kernel<<<dim3(first, pl.splits), NTHREADS, SMEM_BYTES, stream>>>(maps, p);
  LSQ_LAUNCH_CHECK("lora_grad_kernel");
  for (int i = 0; i < nseg; ++i) {
    R.dA[i] = dA[i];
    R.dB[i] = dB[i];
  }
  R.nseg = nseg;
  R.r = r;
  R.rp = rp;
  R.splits = pl.splits;
  R.accumulate = accumulate ? 1 : 0;
  int nb = 0;
  for (int i = 0; i <= nseg; ++i) nb += R.blocks[i];
  lora_grad_reduce<<<nb, 256, 0, stream>>>(R);
  LSQ_LAUNCH_CHECK("lora_grad_reduce");
  return LSQ_OK;
}

}  // namespace lg
}  // namespace lsq

using namespace lsq;

namespace lsq {
// bytes the backward must have (the rank-r part and the dA / dB partials; 0 without an adapter)
size_t bwd_base_bytes(int nseg, int64_t M, int64_t k_in, const int64_t* n_out, int r) {
  if (r <= 0) return 0;
  return tc::bwd_rank_bytes(nseg, M, k_in, n_out, r) + lg::plan(nseg, M, k_in, n_out).total;
}
}  // namespace lsq

extern "C" size_t lsq_nf4_lora_bwd_workspace_size(int32_t nseg, int64_t M, int64_t k_in, const int64_t* n_out,
                                                  int32_t r) {
  if (nseg < 1 || nseg > 3 || r < 0 || r > 64 || M < 1 || k_in < 64 || !n_out) return 256;
  return bwd_base_bytes(nseg, M, k_in, n_out, r) + nf4g::sk_region_bytes();
}

namespace lsq {
namespace tc {
// A second stream of this host thread on the current device, with a fork and a
// join event: the backward runs the dA / dB kernels there, concurrently with
// the dX GEMM (they read the same s*G and neither writes what the other reads),
// so that the SMs the dX GEMM leaves idle do that work.  Created on first use,
// kept for the thread's life.
struct SideStream {
  cudaStream_t s = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};
static lsq_status side_stream(SideStream** out) {
  thread_local SideStream ss[64];
  int dev = 0;
  LSQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= 64) return fail(LSQ_EUNSUPPORTED, "side stream: device %d out of range", dev);
  SideStream& d = ss[dev];
  if (!d.s) {
    LSQ_CUDA_TRY(cudaStreamCreateWithFlags(&d.s, cudaStreamNonBlocking));
    LSQ_CUDA_TRY(cudaEventCreateWithFlags(&d.fork, cudaEventDisableTiming));
    LSQ_CUDA_TRY(cudaEventCreateWithFlags(&d.join, cudaEventDisableTiming));
  }
  *out = &d;
  return LSQ_OK;
}

// state: the rank state a forward with lsq_nf4_lora_fwd_multi_ex left, or null
static lsq_status bwd_impl(int32_t nseg, const lsq_nf4_weight* W, const void* x, const void* const* dy, int64_t M,
                           const void* const* A, const void* const* B, int32_t r, float s, const float* const* u,
                           void* dx, float* const* dA, float* const* dB, int32_t accumulate, void* workspace,
                           size_t workspace_bytes, cudaStream_t cs, void* state, const char* who) {
  if (nseg < 1 || nseg > 3) return fail(LSQ_EINVAL, "%s: 1..3 segments (got %d)", who, nseg);
  if (!W || !dy) return fail(LSQ_EINVAL, "%s: NULL argument", who);
  lsq_status st = check_device();
  if (st != LSQ_OK) return st;
  const int64_t K = W[0].k_in;
  if (M < 1 || M > (1 << 30)) return fail(LSQ_EINVAL, "%s: M out of range", who);
  if (K < 64 || K % 64 != 0) return fail(LSQ_EINVAL, "%s: k_in must be a multiple of 64", who);
  if (r < 0 || r > 64) return fail(LSQ_EINVAL, "%s: LoRA rank must be in [0, 64]", who);
  const int rp = r > 0 ? (r + 15) / 16 * 16 : 0;
  if (nseg * rp > 64) return fail(LSQ_EUNSUPPORTED, "%s: nseg * round16(r) must be <= 64", who);
  if (dx && !aligned(dx, 16)) return fail(LSQ_EINVAL, "%s: dx must be 16-byte aligned", who);
  if (r > 0 && (!x || !aligned(x, 16))) return fail(LSQ_EINVAL, "%s: x NULL or not 16-byte aligned", who);
  int64_t n_out[3];
  for (int i = 0; i < nseg; ++i) {
    const lsq_nf4_weight& w = W[i];
    if (!w.codes || !w.absmax || w.k_in != K || w.n_out < 8 || w.n_out % 8 != 0)
      return fail(LSQ_EINVAL, "%s: segment %d weight is NULL or has a bad shape", who, i);
    if (!aligned(w.codes, 16) || !aligned(w.absmax, 4)) return fail(LSQ_EINVAL, "%s: weight alignment", who);
    if (!dy[i] || !aligned(dy[i], 16)) return fail(LSQ_EINVAL, "%s: dy[%d] NULL or not 16-byte aligned", who, i);
    n_out[i] = w.n_out;
    if (r > 0) {
      if (!A || !B || !dA || !dB || !A[i] || !B[i] || !dA[i] || !dB[i] || (!state && (!u || !u[i])))
        return fail(LSQ_EINVAL, "%s: LoRA operands/gradients NULL with r > 0", who);
      if (!aligned(A[i], 16) || (!state && !aligned(u[i], 16)))
        return fail(LSQ_EINVAL, "%s: LoRA A and U must be 16-byte aligned", who);
    }
  }
  if (r == 0 && !dx) return LSQ_OK;
  __nv_bfloat16* sg = nullptr;
  __nv_bfloat16* at = nullptr;
  __nv_bfloat16* su[3] = {nullptr, nullptr, nullptr};
  char* part = nullptr;
  const size_t need = bwd_base_bytes(nseg, M, K, n_out, r);
  char* sk_ws = nullptr;
  size_t sk_bytes = 0;
  if (workspace && aligned(workspace, 256) && workspace_bytes > need) {  // room for the dX GEMM's stream-K
    sk_ws = static_cast<char*>(workspace) + need;
    sk_bytes = workspace_bytes - need;
  }
  if (r > 0) {
    if (!workspace || workspace_bytes < need || !aligned(workspace, 256))
      return fail(LSQ_EINVAL, "%s: workspace needs %zu bytes, 256-byte aligned (got %zu)", who, need,
                  workspace_bytes);
    char* ws = static_cast<char*>(workspace);
    // s*G = s dY B (bf16, the dX kernel's LoRA block and dA's operand), s*U, A^T
    StatePtrs sp;
    if (state) {
      if (!aligned(state, 256)) return fail(LSQ_EINVAL, "%s: rank state must be 256-byte aligned", who);
      sp = state_ptrs(state, nseg, state_plan(nseg, M, K, n_out, r));
    }
    if ((st = tc::bwd_rank_part(nseg, W, dy, M, A, B, u, r, s, ws, &sg, su, &at, cs, state ? &sp : nullptr)) !=
        LSQ_OK)
      return st;
    part = ws + tc::bwd_rank_bytes(nseg, M, K, n_out, r);
  }
  SideStream* side = nullptr;
  if (dx && r > 0 && (st = side_stream(&side)) != LSQ_OK) return st;
  if (side) LSQ_CUDA_TRY(cudaEventRecord(side->fork, cs));  // s*G and the operands are in place
  // dX first, so that its clusters are placed before the dA / dB kernels take the remaining SMs
  if (dx && (st = tc::launch_dx(nseg, W, dy, M, sg, at, dx, sk_ws, sk_bytes, cs)) != LSQ_OK) return st;
  if (r == 0) return LSQ_OK;
  if (!side) return lg::launch(nseg, M, K, n_out, x, dy, sg, su, dA, dB, r, rp, accumulate, part, cs);
  LSQ_CUDA_TRY(cudaStreamWaitEvent(side->s, side->fork, 0));
  if ((st = lg::launch(nseg, M, K, n_out, x, dy, sg, su, dA, dB, r, rp, accumulate, part, side->s)) != LSQ_OK)
    return st;
  LSQ_CUDA_TRY(cudaEventRecord(side->join, side->s));
  LSQ_CUDA_TRY(cudaStreamWaitEvent(cs, side->join, 0));  // the caller's stream sees dA / dB before anything later
  return LSQ_OK;
}
}  // namespace tc
}  // namespace lsq

extern "C" lsq_status lsq_nf4_lora_bwd_multi(int32_t nseg, const lsq_nf4_weight* W, const void* x,
                                             const void* const* dy, int64_t M, const void* const* A,
                                             const void* const* B, int32_t r, float s, const float* const* u,
                                             void* dx, float* const* dA, float* const* dB, int32_t accumulate,
                                             void* workspace, size_t workspace_bytes, lsq_cuda_stream stream) {
  return tc::bwd_impl(nseg, W, x, dy, M, A, B, r, s, u, dx, dA, dB, accumulate, workspace, workspace_bytes,
                      (cudaStream_t)stream, nullptr, "lsq_nf4_lora_bwd");
}

extern "C" lsq_status lsq_nf4_lora_bwd_multi_ex(int32_t nseg, const lsq_nf4_weight* W, const void* x,
                                                const void* const* dy, int64_t M, const void* const* A,
                                                const void* const* B, int32_t r, float s, const float* const* u,
                                                const void* state, void* dx, float* const* dA, float* const* dB,
                                                int32_t accumulate, void* workspace, size_t workspace_bytes,
                                                lsq_cuda_stream stream) {
  if (r > 0 && !state) return fail(LSQ_EINVAL, "lsq_nf4_lora_bwd_ex: a rank state is needed with r > 0");
  return tc::bwd_impl(nseg, W, x, dy, M, A, B, r, s, u, dx, dA, dB, accumulate, workspace, workspace_bytes,
                      (cudaStream_t)stream, const_cast<void*>(state), "lsq_nf4_lora_bwd_ex");
}

extern "C" lsq_status lsq_nf4_lora_bwd(const lsq_nf4_weight* W, const void* x, const void* dy, int64_t M,
                                       const void* A, const void* B, int32_t r, float s, const float* u, void* dx,
                                       float* dA, float* dB, int32_t accumulate, void* workspace,
                                       size_t workspace_bytes, lsq_cuda_stream stream) {
  const void* d[1] = {dy};
  const void* a[1] = {A};
  const void* b[1] = {B};
  const float* uu[1] = {u};
  float* da[1] = {dA};
  float* db[1] = {dB};
  return lsq_nf4_lora_bwd_multi(1, W, x, d, M, a, b, r, s, uu, dx, da, db, accumulate, workspace, workspace_bytes,
                                stream);
}
