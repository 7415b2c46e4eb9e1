// NF4 blockwise quantiser and dequantiser (format: see "NF4 blockwise format"
// in include/lsq.h).  Both are HBM-bound streaming kernels: the quantiser
// reads 2 bytes and writes 0.5 + 4/64 bytes per weight, one warp per 64-element
// block (each lane owns two neighbouring elements, i.e. one output byte).
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
