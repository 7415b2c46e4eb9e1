// Backward of the fused NF4-LoRA linear:
//   G_seg = dY_seg B_seg                                 (split-K tensor-core kernel, gemm_nf4.cu)
//   dX = sum_seg dY_seg deq(W_seg) + s G_seg A_seg       (CTA-pair tensor-core kernel, gemm_nf4.cu)
//   dB_seg = s dY_seg^T U_seg,  dA_seg = s G_seg^T X      (here)
// dA and dB are skinny products (r <= 64 columns) reduced over the M token
// rows, i.e. HBM-bound reads of dY and X.  Deterministic two-stage reduction:
// stage 1 gives each CTA a 256-column panel and a chunk of rows (row tiles of
// P and Q double-buffered through shared memory with cp.async) and writes fp32
// partial sums; stage 2 adds the partials of each output in a fixed order.
// No atomics, so results are bit-identical run to run.  Every reduction of one
// backward call (dA and dB of up to three linears) shares one launch per stage.
#include <algorithm>

#include "common.cuh"
#include "host_common.h"

namespace lsq {
namespace lg {

constexpr int PANEL = 256;      // columns per CTA (4 per thread)
constexpr int TR = 16;          // rows per shared-memory tile
constexpr int THREADS = 256;
constexpr int TARGET_CTAS = 296;
constexpr int MAXRED = 6;

struct Red {
  const __nv_bfloat16* P;  // [M, C]
  const float* Q;          // [M, r]
  float* out;              // [C, r] or, transposed, [r, C]
  float* part;             // [chunks, C, r]
  int64_t C;
  int64_t mchunk;          // rows per chunk (multiple of TR)
  int chunks, panels, transpose;
};

struct RedSet {
  Red red[MAXRED];
  int n;
  int64_t M;
  int r, accumulate;
  float s;
};

__device__ __forceinline__ void cp_async16(void* dst, const void* src, bool valid) {
  const uint32_t d = smem_u32(dst);
  const int sz = valid ? 16 : 0;  // 0: fill with zeros
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(src), "r"(sz) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// stage 1: blockIdx.x = panel (+ offsets of earlier reductions), blockIdx.y = row chunk.
// Thread (cg, jg): columns c0 + 4 cg .. + 3, ranks j in [jg*jq, jg*jq + jq), jq = ceil(r/4);
// per row it reads 4 bf16 of P (one 8-byte load) and its jq values of Q
// (16-byte loads, the same address for the whole warp) for 4*jq FMAs.
template <int JQ>
__device__ __forceinline__ void skinny_body(const Red& R, int64_t M, int r, int blocky, int px,
                                            __nv_bfloat16 (*sP)[TR][PANEL], float (*sQ)[TR][64]) {
  const int64_t C = R.C;
  const int64_t c0 = (int64_t)px * PANEL;
  const int64_t mb0 = (int64_t)blocky * R.mchunk;
  const int64_t mb1 = mb0 + R.mchunk < M ? mb0 + R.mchunk : M;
  const int tid = threadIdx.x;
  const int cg = tid & 63, jg = tid >> 6;
  float acc[4][JQ];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int q = 0; q < JQ; ++q) acc[a][q] = 0.0f;

  auto load = [&](int buf, int64_t mb) {
    // P: TR rows x 256 columns = 512 chunks of 16 bytes (2 per thread)
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const int idx = tid + u * THREADS;
      const int row = idx >> 5, ch = idx & 31;
      const int64_t m = mb + row, c = c0 + ch * 8;
      const bool v = m < mb1 && c < C;
      cp_async16(&sP[buf][row][ch * 8], v ? (const void*)(R.P + m * C + c) : (const void*)R.P, v);
    }
    if ((r & 3) == 0) {
      const int per = r / 4;
      for (int idx = tid; idx < TR * per; idx += THREADS) {
        const int row = idx / per, ch = idx % per;
        const int64_t m = mb + row;
        const bool v = m < mb1;
        cp_async16(&sQ[buf][row][ch * 4], v ? (const void*)(R.Q + m * r + ch * 4) : (const void*)R.Q, v);
      }
    } else {
      for (int idx = tid; idx < TR * r; idx += THREADS) {
        const int row = idx / r, j = idx % r;
        const int64_t m = mb + row;
        sQ[buf][row][j] = m < mb1 ? R.Q[m * r + j] : 0.0f;
      }
    }
    cp_async_commit();
  };

  int buf = 0;
  if (mb0 < mb1) load(0, mb0);
  for (int64_t mb = mb0; mb < mb1; mb += TR) {
    const bool more = mb + TR < mb1;
    if (more) load(buf ^ 1, mb + TR);
    if (more) cp_async_wait<1>();
    else cp_async_wait<0>();
    __syncthreads();
#pragma unroll 4
    for (int row = 0; row < TR; ++row) {
      const uint2 pp = *reinterpret_cast<const uint2*>(&sP[buf][row][cg * 4]);
      const float p[4] = {bf16lo(pp.x), bf16hi(pp.x), bf16lo(pp.y), bf16hi(pp.y)};
      float qv[JQ];
      const float* qr = &sQ[buf][row][jg * JQ];
      if (JQ % 4 == 0) {
#pragma unroll
        for (int q = 0; q < JQ; q += 4) {
          const float4 f = *reinterpret_cast<const float4*>(qr + q);
          qv[q] = f.x;
          qv[q + 1] = f.y;
          qv[q + 2] = f.z;
          qv[q + 3] = f.w;
        }
      } else {
#pragma unroll
        for (int q = 0; q < JQ; ++q) qv[q] = qr[q];
      }
#pragma unroll
      for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int q = 0; q < JQ; ++q) acc[a][q] = fmaf(p[a], qv[q], acc[a][q]);
    }
    __syncthreads();
    buf ^= 1;
  }
#pragma unroll
  for (int a = 0; a < 4; ++a) {
    const int64_t c = c0 + cg * 4 + a;
    if (c >= C) continue;
#pragma unroll
    for (int q = 0; q < JQ; ++q) {
      const int j = jg * JQ + q;
      if (j < r) R.part[((int64_t)blocky * C + c) * r + j] = acc[a][q];
    }
  }
}

__global__ void __launch_bounds__(THREADS) skinny_partial(const __grid_constant__ RedSet rs) {
  __shared__ __align__(16) __nv_bfloat16 sP[2][TR][PANEL];
  __shared__ __align__(16) float sQ[2][TR][64];
  int rid = 0, px = blockIdx.x;
  while (rid + 1 < rs.n && px >= rs.red[rid].panels) {
    px -= rs.red[rid].panels;
    ++rid;
  }
  const Red& R = rs.red[rid];
  if ((int)blockIdx.y >= R.chunks) return;
  const int jq = (rs.r + 3) / 4;
  if (jq <= 1) skinny_body<1>(R, rs.M, rs.r, blockIdx.y, px, sP, sQ);
  else if (jq <= 2) skinny_body<2>(R, rs.M, rs.r, blockIdx.y, px, sP, sQ);
  else if (jq <= 4) skinny_body<4>(R, rs.M, rs.r, blockIdx.y, px, sP, sQ);
  else if (jq <= 8) skinny_body<8>(R, rs.M, rs.r, blockIdx.y, px, sP, sQ);
  else skinny_body<16>(R, rs.M, rs.r, blockIdx.y, px, sP, sQ);
}

// stage 2: out (+)= s * sum over chunks (ascending) of the partials
__global__ void __launch_bounds__(256) skinny_reduce(const __grid_constant__ RedSet rs) {
  const int rid = blockIdx.y;
  const Red& R = rs.red[rid];
  const int r = rs.r;
  const int64_t n = R.C * r;
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < n; idx += (int64_t)gridDim.x * blockDim.x) {
    float sum = 0.0f;
    for (int k = 0; k < R.chunks; ++k) sum += R.part[(int64_t)k * n + idx];
    const int64_t c = idx / r, j = idx % r;
    float* dst = R.transpose ? R.out + j * R.C + c : R.out + idx;
    const float v = rs.s * sum;
    *dst = rs.accumulate ? *dst + v : v;
  }
}

static int64_t panels_for(int64_t C) { return (C + PANEL - 1) / PANEL; }

static int64_t chunks_for(int64_t M, int64_t C) {
  int64_t k = (TARGET_CTAS + panels_for(C) - 1) / panels_for(C);
  const int64_t maxk = (M + TR - 1) / TR;
  if (k > maxk) k = maxk;
  if (k < 1) k = 1;
  return k;
}

static int64_t mchunk_for(int64_t M, int64_t k) { return ((M + k - 1) / k + TR - 1) / TR * TR; }

static size_t partial_bytes(int64_t M, int64_t C, int r) {
  const int64_t k = chunks_for(M, C);
  const int64_t kk = (M + mchunk_for(M, k) - 1) / mchunk_for(M, k);
  return ((size_t)kk * (size_t)C * (size_t)r * sizeof(float) + 255) / 256 * 256;
}

static size_t round256(size_t b) { return (b + 255) / 256 * 256; }

}  // namespace lg
}  // namespace lsq

using namespace lsq;

extern "C" size_t lsq_nf4_lora_bwd_workspace_size(int32_t nseg, int64_t M, int64_t k_in, const int64_t* n_out,
                                                  int32_t r) {
  if (nseg < 1 || nseg > 3 || r <= 0 || r > 64 || M < 1 || k_in < 64 || !n_out) return 256;
  size_t b = tc::bwd_rank_bytes(nseg, M, k_in, n_out, r);
  for (int i = 0; i < nseg; ++i) b += lg::partial_bytes(M, n_out[i], r) + lg::partial_bytes(M, k_in, r);
  return b;
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
      if (!A || !B || !u || !dA || !dB || !A[i] || !B[i] || !u[i] || !dA[i] || !dB[i])
        return fail(LSQ_EINVAL, "%s: LoRA operands/gradients NULL with r > 0", who);
      if (!aligned(A[i], 16) || !aligned(u[i], 16))
        return fail(LSQ_EINVAL, "%s: LoRA A and U must be 16-byte aligned", who);
    }
  }
  if (r == 0 && !dx) return LSQ_OK;
  float* g[3] = {nullptr, nullptr, nullptr};
  __nv_bfloat16* sg = nullptr;
  __nv_bfloat16* at = nullptr;
  char* part = nullptr;
  cudaStream_t cs = (cudaStream_t)stream;
  if (r > 0) {
    const size_t need = lsq_nf4_lora_bwd_workspace_size(nseg, M, K, n_out, r);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 256))
      return fail(LSQ_EINVAL, "%s: workspace needs %zu bytes, 256-byte aligned (got %zu)", who, need,
                  workspace_bytes);
    char* ws = static_cast<char*>(workspace);
    // G = dY B (fp32 for dA, s*G in bf16 for the dX kernel) and the padded operands
    if ((st = tc::bwd_rank_part(nseg, W, dy, M, A, B, r, s, ws, g, &sg, &at, cs)) != LSQ_OK) return st;
    part = ws + tc::bwd_rank_bytes(nseg, M, K, n_out, r);
  }
  if (dx && (st = tc::launch_dx(nseg, W, dy, M, sg, at, dx, cs)) != LSQ_OK) return st;
  if (r == 0) return LSQ_OK;
  lg::RedSet rs;
  memset(&rs, 0, sizeof(rs));
  rs.M = M;
  rs.r = r;
  rs.s = s;
  rs.accumulate = accumulate ? 1 : 0;
  int panels = 0, maxchunks = 1;
  int64_t maxn = 0;
  for (int i = 0; i < nseg; ++i) {
    for (int which = 0; which < 2; ++which) {  // dB_i = s dy_i^T U_i ; dA_i = s G_i^T x
      lg::Red& R = rs.red[rs.n++];
      R.P = static_cast<const __nv_bfloat16*>(which == 0 ? dy[i] : x);
      R.Q = which == 0 ? u[i] : g[i];
      R.out = which == 0 ? dB[i] : dA[i];
      R.C = which == 0 ? n_out[i] : K;
      R.transpose = which;
      const int64_t k = lg::chunks_for(M, R.C);
      R.mchunk = lg::mchunk_for(M, k);
      R.chunks = (int)((M + R.mchunk - 1) / R.mchunk);
      R.panels = (int)lg::panels_for(R.C);
      R.part = reinterpret_cast<float*>(part);
      part += lg::partial_bytes(M, R.C, r);
      panels += R.panels;
      if (R.chunks > maxchunks) maxchunks = R.chunks;
      if (R.C * r > maxn) maxn = R.C * r;
    }
  }
  lg::skinny_partial<<<dim3(panels, maxchunks), lg::THREADS, 0, cs>>>(rs);
  LSQ_LAUNCH_CHECK("skinny_partial");
  int64_t g2 = (maxn + 255) / 256;
  if (g2 > 1024) g2 = 1024;
  lg::skinny_reduce<<<dim3((unsigned)g2, rs.n), 256, 0, cs>>>(rs);
  LSQ_LAUNCH_CHECK("skinny_reduce");
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
