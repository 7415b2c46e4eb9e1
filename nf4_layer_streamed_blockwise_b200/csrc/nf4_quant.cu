// NF4 blockwise quantiser and dequantiser (format: see "NF4 blockwise format"
// in include/lsq.h).  Both are HBM-bound streaming kernels: the quantiser
// reads 2 bytes and writes 0.5 + 4/64 bytes per weight, one warp per 64-element
// block (each lane owns two neighbouring elements, i.e. one output byte).
#include <cuda_fp8.h>

#include "common.cuh"
#include "host_common.h"

namespace lsq {

struct QuantTables {
  float thr[15];
  float cb[16];
};

__global__ void __launch_bounds__(256) nf4_quantize_kernel(const uint32_t* __restrict__ w_pairs, int64_t nblocks,
                                                           uint8_t* __restrict__ codes, float* __restrict__ absmax,
                                                           const QuantTables t) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (blockIdx.x * (int64_t)blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
  for (int64_t b = warp; b < nblocks; b += nwarps) {
    const uint32_t pair = __ldg(w_pairs + b * 32 + lane);
    const float w0 = bf16lo(pair), w1 = bf16hi(pair);
    float a = fmaxf(fabsf(w0), fabsf(w1));
#pragma unroll
    for (int o = 16; o; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    uint32_t c0 = 7, c1 = 7;  // all-zero block: every code is the zero level
    if (a > 0.0f) {
      const float x0 = __fdiv_rn(w0, a), x1 = __fdiv_rn(w1, a);
      c0 = 0;
      c1 = 0;
#pragma unroll
      for (int i = 0; i < 15; ++i) {
        c0 += (x0 >= t.thr[i]);
        c1 += (x1 >= t.thr[i]);
      }
    }
    codes[b * 32 + lane] = (uint8_t)((c0 << 4) | c1);
    if (lane == 0) absmax[b] = a;
  }
}

__global__ void __launch_bounds__(256) nf4_dequantize_kernel(const uint8_t* __restrict__ codes,
                                                             const float* __restrict__ absmax, int64_t nbytes,
                                                             uint32_t* __restrict__ out_pairs, const QuantTables t) {
  __shared__ float cb[16];
  if (threadIdx.x < 16) cb[threadIdx.x] = t.cb[threadIdx.x];
  __syncthreads();
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < nbytes; i += (int64_t)gridDim.x * blockDim.x) {
    const uint32_t byte = codes[i];
    const float a = absmax[i >> 5];
    out_pairs[i] = pack_bf16x2(__fmul_rn(cb[byte >> 4], a), __fmul_rn(cb[byte & 15], a));
  }
}

static QuantTables tables() {
  QuantTables t;
  const float* thr = thresholds();
  const float* cbk = codebook();
  for (int i = 0; i < 15; ++i) t.thr[i] = thr[i];
  for (int i = 0; i < 16; ++i) t.cb[i] = cbk[i];
  return t;
}

}  // namespace lsq

extern "C" lsq_status lsq_nf4_quantize(const void* w_bf16, int64_t n_out, int64_t k_in, uint8_t* codes,
                                       float* absmax, lsq_cuda_stream stream) {
  using namespace lsq;
  if (!w_bf16 || !codes || !absmax) return fail(LSQ_EINVAL, "lsq_nf4_quantize: NULL pointer");
  if (n_out < 1 || k_in < 64 || k_in % 64 != 0)
    return fail(LSQ_EINVAL, "lsq_nf4_quantize: need n_out >= 1 and k_in a positive multiple of 64 (got %lld x %lld)",
                (long long)n_out, (long long)k_in);
  if (!aligned(w_bf16, 4) || !aligned(absmax, 4))
    return fail(LSQ_EINVAL, "lsq_nf4_quantize: weight and absmax must be 4-byte aligned");
  lsq_status st = check_device();
  if (st != LSQ_OK) return st;
  const int64_t nblocks = n_out * (k_in / 64);
  const int threads = 256;
  int64_t grid = (nblocks * 32 + threads - 1) / threads;
  const int64_t cap = (int64_t)num_sms() * 16;
  if (grid > cap) grid = cap;
  nf4_quantize_kernel<<<(unsigned)grid, threads, 0, (cudaStream_t)stream>>>(
      static_cast<const uint32_t*>(w_bf16), nblocks, codes, absmax, tables());
  LSQ_LAUNCH_CHECK("nf4_quantize_kernel");
  return LSQ_OK;
}

extern "C" lsq_status lsq_nf4_dequantize(const lsq_nf4_weight* w, void* w_bf16, lsq_cuda_stream stream) {
  using namespace lsq;
  if (!w || !w->codes || !w->absmax || !w_bf16) return fail(LSQ_EINVAL, "lsq_nf4_dequantize: NULL pointer");
  if (w->n_out < 1 || w->k_in < 64 || w->k_in % 64 != 0)
    return fail(LSQ_EINVAL, "lsq_nf4_dequantize: bad shape");
  if (!aligned(w_bf16, 4)) return fail(LSQ_EINVAL, "lsq_nf4_dequantize: output must be 4-byte aligned");
  lsq_status st = check_device();
  if (st != LSQ_OK) return st;
  const int64_t nbytes = w->n_out * w->k_in / 2;
  int64_t grid = (nbytes + 255) / 256;
  const int64_t cap = (int64_t)num_sms() * 16;
  if (grid > cap) grid = cap;
  nf4_dequantize_kernel<<<(unsigned)grid, 256, 0, (cudaStream_t)stream>>>(w->codes, w->absmax, nbytes,
                                                                          static_cast<uint32_t*>(w_bf16), tables());
  LSQ_LAUNCH_CHECK("nf4_dequantize_kernel");
  return LSQ_OK;
}

// ---------------------------------------------------------------------------
// Double-quantised absmax (format: "Double-quantised absmax" in include/lsq.h).
// The second level is applied offline, once per tensor; on the hot path only
// the expansion runs, on the copy stream right after each layer upload, so
// the host link carries one byte per 64-weight block instead of four and the
// fused GEMMs keep reading fp32 absmax from HBM.
namespace lsq {
namespace dq {

constexpr int BLOCK = 256;
constexpr float E4M3_MAX = 448.0f;
constexpr int MAX_ITEMS = 8;

// one CTA of 256 threads per block of 256 absmax values
__global__ void __launch_bounds__(BLOCK) absmax_dq_kernel(const float* __restrict__ absmax, int64_t nb,
                                                          uint8_t* __restrict__ codes, float2* __restrict__ params) {
  __shared__ float s_lo[BLOCK / 32], s_hi[BLOCK / 32];
  const int64_t i = (int64_t)blockIdx.x * BLOCK + threadIdx.x;
  const bool in = i < nb;
  const float a = in ? absmax[i] : 0.0f;
  float lo = in ? a : INFINITY, hi = in ? a : -INFINITY;
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    lo = fminf(lo, __shfl_xor_sync(0xffffffffu, lo, o));
    hi = fmaxf(hi, __shfl_xor_sync(0xffffffffu, hi, o));
  }
  if ((threadIdx.x & 31) == 0) {
    s_lo[threadIdx.x >> 5] = lo;
    s_hi[threadIdx.x >> 5] = hi;
  }
  __syncthreads();
  lo = s_lo[0];
  hi = s_hi[0];
#pragma unroll
  for (int w = 1; w < BLOCK / 32; ++w) {
    lo = fminf(lo, s_lo[w]);
    hi = fmaxf(hi, s_hi[w]);
  }
  // separate roundings, no contraction: the definition's fp32 steps
  const float centre = __fmul_rn(__fadd_rn(hi, lo), 0.5f);
  const float half = __fmul_rn(__fsub_rn(hi, lo), 0.5f);
  const float scale = __fdiv_rn(half, E4M3_MAX);
  if (threadIdx.x == 0) params[blockIdx.x] = make_float2(centre, scale);
  if (in) {
    uint8_t c = 0;
    if (scale != 0.0f) {
      const float x = __fdiv_rn(__fsub_rn(a, centre), scale);
      c = (uint8_t)__nv_cvt_float_to_fp8(x, __NV_SATFINITE, __NV_E4M3);  // nearest, ties to even, saturating
      if (c == 0x80) c = 0;                                             // zero is stored as +0
    }
    codes[i] = c;
  }
}

__device__ __forceinline__ float e4m3_to_f32(uint8_t c) {
  return __half2float(__half(__nv_cvt_fp8_to_halfraw((__nv_fp8_storage_t)c, __NV_E4M3)));  // exact
}

struct ExpandItem {
  const uint8_t* codes;
  const float2* params;
  float* out;
  int64_t nb;
};
struct ExpandJob {
  ExpandItem it[MAX_ITEMS];
  int64_t start[MAX_ITEMS + 1];  // prefix sums of nb
  int n;
};

// a' = fp32(fp32(e4m3(code) * scale) + centre) for every value of every item
__global__ void __launch_bounds__(256) absmax_expand_kernel(const __grid_constant__ ExpandJob job) {
  const int64_t total = job.start[job.n];
  for (int64_t g = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; g < total; g += (int64_t)gridDim.x * blockDim.x) {
    int k = 0;
    while (k + 1 < job.n && g >= job.start[k + 1]) ++k;
    const ExpandItem& e = job.it[k];
    const int64_t i = g - job.start[k];
    const float2 p = e.params[i / BLOCK];
    e.out[i] = __fadd_rn(__fmul_rn(e4m3_to_f32(e.codes[i]), p.y), p.x);
  }
}

// items: (codes, params, out, nb) triples relative to `base` (nullptr: absolute)
static lsq_status launch_expand(const char* base, const uint64_t* codes_off, const uint64_t* params_off,
                                const uint64_t* out_off, const int64_t* nb, int n, cudaStream_t stream) {
  ExpandJob job{};
  job.n = n;
  job.start[0] = 0;
  for (int k = 0; k < n; ++k) {
    const uintptr_t b = reinterpret_cast<uintptr_t>(base);
    job.it[k].codes = reinterpret_cast<const uint8_t*>(b + codes_off[k]);
    job.it[k].params = reinterpret_cast<const float2*>(b + params_off[k]);
    job.it[k].out = reinterpret_cast<float*>(b + out_off[k]);
    job.it[k].nb = nb[k];
    job.start[k + 1] = job.start[k] + nb[k];
  }
  if (job.start[n] == 0) return LSQ_OK;
  int64_t grid = (job.start[n] + 255) / 256;
  const int64_t cap = (int64_t)num_sms() * 8;
  if (grid > cap) grid = cap;
  absmax_expand_kernel<<<(unsigned)grid, 256, 0, stream>>>(job);
  LSQ_LAUNCH_CHECK("absmax_expand_kernel");
  return LSQ_OK;
}

}  // namespace dq
}  // namespace lsq

extern "C" lsq_status lsq_absmax_double_quantize(const float* absmax, int64_t nb, uint8_t* codes, float* params,
                                                 lsq_cuda_stream stream) {
  using namespace lsq;
  if (!absmax || !codes || !params) return fail(LSQ_EINVAL, "lsq_absmax_double_quantize: NULL pointer");
  if (nb < 1) return fail(LSQ_EINVAL, "lsq_absmax_double_quantize: nb must be >= 1");
  if (!aligned(absmax, 4) || !aligned(params, 8))
    return fail(LSQ_EINVAL, "lsq_absmax_double_quantize: absmax must be 4-byte and params 8-byte aligned");
  lsq_status st = check_device();
  if (st != LSQ_OK) return st;
  const int64_t nblk = (nb + dq::BLOCK - 1) / dq::BLOCK;
  if (nblk > 0x7fffffffLL) return fail(LSQ_EINVAL, "lsq_absmax_double_quantize: too many blocks");
  dq::absmax_dq_kernel<<<(unsigned)nblk, dq::BLOCK, 0, (cudaStream_t)stream>>>(absmax, nb, codes,
                                                                                reinterpret_cast<float2*>(params));
  LSQ_LAUNCH_CHECK("absmax_dq_kernel");
  return LSQ_OK;
}

extern "C" lsq_status lsq_absmax_expand(const uint8_t* codes, const float* params, int64_t nb, float* absmax,
                                        lsq_cuda_stream stream) {
  using namespace lsq;
  if (!codes || !params || !absmax) return fail(LSQ_EINVAL, "lsq_absmax_expand: NULL pointer");
  if (nb < 1) return fail(LSQ_EINVAL, "lsq_absmax_expand: nb must be >= 1");
  if (!aligned(absmax, 4) || !aligned(params, 8))
    return fail(LSQ_EINVAL, "lsq_absmax_expand: absmax must be 4-byte and params 8-byte aligned");
  lsq_status st = check_device();
  if (st != LSQ_OK) return st;
  const uint64_t c = (uint64_t)(uintptr_t)codes, p = (uint64_t)(uintptr_t)params, o = (uint64_t)(uintptr_t)absmax;
  return dq::launch_expand(nullptr, &c, &p, &o, &nb, 1, (cudaStream_t)stream);
}
