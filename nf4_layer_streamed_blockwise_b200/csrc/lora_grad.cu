// Backward of the fused NF4-LoRA linear:
//   dX = sum_seg dY_seg deq(W_seg) + s G_seg A_seg     (tensor cores, gemm_tc.cu)
//   dB_seg = s dY_seg^T U_seg,  dA_seg = s G_seg^T X    (here)
// dA and dB are skinny products (r <= 64 columns) reduced over the M token
// rows.  They are HBM-bound reads of dY and X, done as a deterministic
// two-stage reduction: stage 1 gives each CTA a 64-column panel and a chunk of
// rows and writes fp32 partial sums; stage 2 adds the partials in a fixed
// order.  No atomics, so the result is bit-identical run to run.
#include "common.cuh"
#include "host_common.h"

namespace lsq {
namespace tc {
lsq_status launch_dx(int nseg, const lsq_nf4_weight* W, const void* const* dy, int64_t M, const void* const* A,
                     const void* const* B, int r, float s, void* dx, float* const* g_out, cudaStream_t stream);
}

namespace lg {

constexpr int PANEL = 64;
constexpr int ROWS = 32;        // rows of Q staged per step
constexpr int TARGET_CTAS = 296;

// part[chunk][c][j] = sum_{m in chunk} P[m, c] * Q[m, j]
__global__ void __launch_bounds__(256) skinny_partial(const __nv_bfloat16* __restrict__ P, int64_t M, int64_t C,
                                                      const float* __restrict__ Q, int r, int64_t mchunk,
                                                      float* __restrict__ part) {
  __shared__ float sQ[ROWS * 64];
  const int64_t c = (int64_t)blockIdx.x * PANEL + (threadIdx.x & 63);
  const int jg = threadIdx.x >> 6;  // j = jg + 4 q
  const int64_t mb0 = (int64_t)blockIdx.y * mchunk;
  const int64_t mb1 = mb0 + mchunk < M ? mb0 + mchunk : M;
  float acc[16];
#pragma unroll
  for (int q = 0; q < 16; ++q) acc[q] = 0.0f;
  for (int64_t mb = mb0; mb < mb1; mb += ROWS) {
    const int rows = (int)((mb1 - mb) < ROWS ? (mb1 - mb) : ROWS);
    __syncthreads();
    for (int idx = threadIdx.x; idx < rows * r; idx += 256) sQ[idx] = Q[mb * r + idx];
    __syncthreads();
    if (c < C) {
      const __nv_bfloat16* pp = P + mb * C + c;
      int mm = 0;
      for (; mm + 4 <= rows; mm += 4) {
        float pv[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) pv[u] = __bfloat162float(pp[(int64_t)(mm + u) * C]);
#pragma unroll
        for (int u = 0; u < 4; ++u) {
#pragma unroll
          for (int q = 0; q < 16; ++q) {
            const int j = jg + 4 * q;
            if (j < r) acc[q] = fmaf(pv[u], sQ[(mm + u) * r + j], acc[q]);
          }
        }
      }
      for (; mm < rows; ++mm) {
        const float pv = __bfloat162float(pp[(int64_t)mm * C]);
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const int j = jg + 4 * q;
          if (j < r) acc[q] = fmaf(pv, sQ[mm * r + j], acc[q]);
        }
      }
    }
  }
  if (c < C) {
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      const int j = jg + 4 * q;
      if (j < r) part[((int64_t)blockIdx.y * C + c) * r + j] = acc[q];
    }
  }
}

// out[c, j] (transpose: out[j, c]) (+)= s * sum_k part[k][c][j], k ascending
__global__ void __launch_bounds__(256) skinny_reduce(const float* __restrict__ part, int nchunks, int64_t C, int r,
                                                     float s, float* __restrict__ out, int transpose, int accumulate) {
  const int64_t n = C * r;
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < n; idx += (int64_t)gridDim.x * blockDim.x) {
    float sum = 0.0f;
    for (int k = 0; k < nchunks; ++k) sum += part[(int64_t)k * n + idx];
    const int64_t c = idx / r, j = idx % r;
    float* dst = transpose ? out + j * C + c : out + idx;
    const float v = s * sum;
    *dst = accumulate ? *dst + v : v;
  }
}

static int64_t nchunks_for(int64_t M, int64_t C) {
  const int64_t panels = (C + PANEL - 1) / PANEL;
  int64_t k = (TARGET_CTAS + panels - 1) / panels;
  const int64_t maxk = (M + ROWS - 1) / ROWS;
  if (k > maxk) k = maxk;
  if (k < 1) k = 1;
  return k;
}

static size_t partial_bytes(int64_t M, int64_t C, int r) {
  return (size_t)nchunks_for(M, C) * (size_t)C * (size_t)r * sizeof(float);
}

static size_t round256(size_t b) { return (b + 255) / 256 * 256; }

static lsq_status skinny(const void* P, int64_t M, int64_t C, const float* Q, int r, float s, float* out,
                         int transpose, int accumulate, float* part, cudaStream_t stream) {
  const int64_t k = nchunks_for(M, C);
  const int64_t mchunk = ((M + k - 1) / k + ROWS - 1) / ROWS * ROWS;
  const int64_t kk = (M + mchunk - 1) / mchunk;
  dim3 g1((unsigned)((C + PANEL - 1) / PANEL), (unsigned)kk);
  skinny_partial<<<g1, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(P), M, C, Q, r, mchunk, part);
  LSQ_LAUNCH_CHECK("skinny_partial");
  int64_t g2 = (C * r + 255) / 256;
  if (g2 > 4096) g2 = 4096;
  skinny_reduce<<<(unsigned)g2, 256, 0, stream>>>(part, (int)kk, C, r, s, out, transpose, accumulate);
  LSQ_LAUNCH_CHECK("skinny_reduce");
  return LSQ_OK;
}

}  // namespace lg
}  // namespace lsq

using namespace lsq;

extern "C" size_t lsq_nf4_lora_bwd_workspace_size(int32_t nseg, int64_t M, int64_t k_in, const int64_t* n_out,
                                                  int32_t r) {
  if (nseg < 1 || nseg > 3 || r <= 0 || M < 1 || !n_out) return 256;
  size_t g = lg::round256((size_t)nseg * (size_t)M * (size_t)r * sizeof(float));
  size_t part = lg::partial_bytes(M, k_in, r);
  for (int i = 0; i < nseg; ++i) {
    const size_t b = lg::partial_bytes(M, n_out[i], r);
    if (b > part) part = b;
  }
  return g + lg::round256(part);
}

extern "C" lsq_status lsq_nf4_lora_bwd_multi(int32_t nseg, const lsq_nf4_weight* W, const void* x,
                                             const void* const* dy, int64_t M, const void* const* A,
                                             const void* const* B, int32_t r, float s, const float* const* u,
                                             void* dx, float* const* dA, float* const* dB, int32_t accumulate,
                                             void* workspace, size_t workspace_bytes, lsq_cuda_stream stream) {
  const char* who = "lsq_nf4_lora_bwd";
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
  int64_t n_out[3];
  for (int i = 0; i < nseg; ++i) {
    const lsq_nf4_weight& w = W[i];
    if (!w.codes || !w.absmax || w.k_in != K || w.n_out < 8 || w.n_out % 8 != 0)
      return fail(LSQ_EINVAL, "%s: segment %d weight is NULL or has a bad shape", who, i);
    if (!aligned(w.codes, 16) || !aligned(w.absmax, 4)) return fail(LSQ_EINVAL, "%s: weight alignment", who);
    if (!dy[i] || !aligned(dy[i], 16)) return fail(LSQ_EINVAL, "%s: dy[%d] NULL or not 16-byte aligned", who, i);
    n_out[i] = w.n_out;
    if (r > 0) {
      if (!x || !A || !B || !u || !dA || !dB || !A[i] || !B[i] || !u[i] || !dA[i] || !dB[i])
        return fail(LSQ_EINVAL, "%s: LoRA operands/gradients NULL with r > 0", who);
      if (!aligned(A[i], 16)) return fail(LSQ_EINVAL, "%s: LoRA A must be 16-byte aligned", who);
    }
  }
  if (r == 0 && !dx) return LSQ_OK;
  float* g[3] = {nullptr, nullptr, nullptr};
  float* part = nullptr;
  if (r > 0) {
    const size_t need = lsq_nf4_lora_bwd_workspace_size(nseg, M, K, n_out, r);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 256))
      return fail(LSQ_EINVAL, "%s: workspace needs %zu bytes, 256-byte aligned (got %zu)", who, need,
                  workspace_bytes);
    float* ws = static_cast<float*>(workspace);
    for (int i = 0; i < nseg; ++i) g[i] = ws + (size_t)i * M * r;
    part = reinterpret_cast<float*>(static_cast<char*>(workspace) +
                                    lg::round256((size_t)nseg * (size_t)M * (size_t)r * sizeof(float)));
  }
  cudaStream_t cs = (cudaStream_t)stream;
  if ((st = tc::launch_dx(nseg, W, dy, M, A, B, r, s, dx, g, cs)) != LSQ_OK) return st;
  if (r == 0) return LSQ_OK;
  for (int i = 0; i < nseg; ++i) {
    if ((st = lg::skinny(dy[i], M, n_out[i], u[i], r, s, dB[i], 0, accumulate, part, cs)) != LSQ_OK) return st;
    if ((st = lg::skinny(x, M, K, g[i], r, s, dA[i], 1, accumulate, part, cs)) != LSQ_OK) return st;
  }
  return LSQ_OK;
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
