// Decoder-layer kernels around the NF4-LoRA linears (Llama / Qwen): RMSNorm,
// RoPE, SwiGLU, embedding gather, causal-LM cross entropy, AdamW.  All are
// HBM-bound streaming kernels: 16-byte vector accesses, one CTA per row for
// the row reductions, fixed reduction trees (deterministic).
#include "common.cuh"
#include "host_common.h"

namespace lsq {
namespace ops {

__device__ __forceinline__ void unpack8(uint4 v, float* f) {
  f[0] = bf16lo(v.x); f[1] = bf16hi(v.x); f[2] = bf16lo(v.y); f[3] = bf16hi(v.y);
  f[4] = bf16lo(v.z); f[5] = bf16hi(v.z); f[6] = bf16lo(v.w); f[7] = bf16hi(v.w);
}
__device__ __forceinline__ uint4 pack8(const float* f) {
  return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                    pack_bf16x2(f[6], f[7]));
}

// block-wide sum with a fixed tree; every thread gets the result
template <int NT>
__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  __syncthreads();
  if (l == 0) red[w] = v;
  __syncthreads();
  float t = 0.0f;
#pragma unroll
  for (int i = 0; i < NT / 32; ++i) t += red[i];
  return t;
}

constexpr int RN_T = 256;

// ---------------------------------------------------------------- RMSNorm
__global__ void __launch_bounds__(RN_T) rmsnorm_fwd_kernel(const uint4* __restrict__ x, const uint4* __restrict__ g,
                                                           uint4* __restrict__ y, float* __restrict__ rstd, int d8,
                                                           float inv_d, float eps) {
  __shared__ float red[RN_T / 32];
  const int64_t row = blockIdx.x;
  const uint4* xr = x + row * d8;
  float ss = 0.0f;
  for (int c = threadIdx.x; c < d8; c += RN_T) {
    float f[8];
    unpack8(xr[c], f);
#pragma unroll
    for (int i = 0; i < 8; ++i) ss = fmaf(f[i], f[i], ss);
  }
  const float tot = block_sum<RN_T>(ss, red);
  const float rs = 1.0f / sqrtf(tot * inv_d + eps);
  if (threadIdx.x == 0 && rstd) rstd[row] = rs;
  for (int c = threadIdx.x; c < d8; c += RN_T) {
    float f[8], gv[8];
    unpack8(xr[c], f);
    unpack8(g[c], gv);
#pragma unroll
    for (int i = 0; i < 8; ++i) f[i] = f[i] * rs * gv[i];
    y[row * d8 + c] = pack8(f);
  }
}

// dx = rs*(dy*g) - x * rs^3 * mean(dy*g*x);  out = dres_in + dx
__global__ void __launch_bounds__(RN_T) rmsnorm_bwd_kernel(const uint4* __restrict__ dy, const uint4* __restrict__ x,
                                                           const uint4* __restrict__ g, const float* __restrict__ rstd,
                                                           const uint4* dres_in, uint4* dres_out, int d8, float inv_d) {
  __shared__ float red[RN_T / 32];
  const int64_t row = blockIdx.x;
  const uint4* xr = x + row * d8;
  const uint4* dr = dy + row * d8;
  float dot = 0.0f;
  for (int c = threadIdx.x; c < d8; c += RN_T) {
    float f[8], dv[8], gv[8];
    unpack8(xr[c], f);
    unpack8(dr[c], dv);
    unpack8(g[c], gv);
#pragma unroll
    for (int i = 0; i < 8; ++i) dot = fmaf(dv[i] * gv[i], f[i], dot);
  }
  const float tot = block_sum<RN_T>(dot, red);
  const float rs = rstd[row];
  const float k = rs * rs * rs * tot * inv_d;
  for (int c = threadIdx.x; c < d8; c += RN_T) {
    float f[8], dv[8], gv[8], o[8];
    unpack8(xr[c], f);
    unpack8(dr[c], dv);
    unpack8(g[c], gv);
    if (dres_in) unpack8(dres_in[row * d8 + c], o);
    else {
#pragma unroll
      for (int i = 0; i < 8; ++i) o[i] = 0.0f;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) o[i] += rs * dv[i] * gv[i] - f[i] * k;
    dres_out[row * d8 + c] = pack8(o);
  }
}

// The same two RMSNorm passes with the row held in registers between the reduction and the
// output (one read of x, dy and the residual gradient per row) and all of a thread's loads issued
// before its first use: RN2_T threads per row, V 16-byte words per thread (d <= 8 V RN2_T).
constexpr int RN2_T = 128;

template <int V>
__global__ void __launch_bounds__(RN2_T) rmsnorm_fwd_reg_kernel(const uint4* __restrict__ x,
                                                                const uint4* __restrict__ g, uint4* __restrict__ y,
                                                                float* __restrict__ rstd, int d8, float inv_d,
                                                                float eps) {
  __shared__ float red[RN2_T / 32];
  const int64_t row = blockIdx.x;
  const uint4* xr = x + row * d8;
  uint4 xv[V];
#pragma unroll
  for (int i = 0; i < V; ++i) {
    const int c = threadIdx.x + i * RN2_T;
    xv[i] = c < d8 ? xr[c] : make_uint4(0u, 0u, 0u, 0u);
  }
  float ss = 0.0f;
#pragma unroll
  for (int i = 0; i < V; ++i) {
    float f[8];
    unpack8(xv[i], f);
#pragma unroll
    for (int j = 0; j < 8; ++j) ss = fmaf(f[j], f[j], ss);
  }
  const float tot = block_sum<RN2_T>(ss, red);
  const float rs = 1.0f / sqrtf(tot * inv_d + eps);
  if (threadIdx.x == 0 && rstd) rstd[row] = rs;
#pragma unroll
  for (int i = 0; i < V; ++i) {
    const int c = threadIdx.x + i * RN2_T;
    if (c >= d8) break;
    float f[8], gv[8];
    unpack8(xv[i], f);
    unpack8(g[c], gv);
#pragma unroll
    for (int j = 0; j < 8; ++j) f[j] = f[j] * rs * gv[j];
    y[row * d8 + c] = pack8(f);
  }
}

template <int V>
__global__ void __launch_bounds__(RN2_T) rmsnorm_bwd_reg_kernel(const uint4* __restrict__ dy,
                                                                const uint4* __restrict__ x,
                                                                const uint4* __restrict__ g,
                                                                const float* __restrict__ rstd,
                                                                const uint4* dres_in, uint4* dres_out, int d8,
                                                                float inv_d) {
  __shared__ float red[RN2_T / 32];
  const int64_t row = blockIdx.x;
  const uint4* xr = x + row * d8;
  const uint4* dr = dy + row * d8;
  const uint4 z = make_uint4(0u, 0u, 0u, 0u);
  uint4 xv[V], dv4[V], gv4[V], rv[V];
#pragma unroll
  for (int i = 0; i < V; ++i) {
    const int c = threadIdx.x + i * RN2_T;
    const bool in = c < d8;
    xv[i] = in ? xr[c] : z;
    dv4[i] = in ? dr[c] : z;
    gv4[i] = in ? g[c] : z;
    rv[i] = (in && dres_in) ? dres_in[row * d8 + c] : z;  // in flight across the reduction
  }
  float dot = 0.0f;
#pragma unroll
  for (int i = 0; i < V; ++i) {
    float f[8], dv[8], gv[8];
    unpack8(xv[i], f);
    unpack8(dv4[i], dv);
    unpack8(gv4[i], gv);
#pragma unroll
    for (int j = 0; j < 8; ++j) dot = fmaf(dv[j] * gv[j], f[j], dot);
  }
  const float tot = block_sum<RN2_T>(dot, red);
  const float rs = rstd[row];
  const float k = rs * rs * rs * tot * inv_d;
#pragma unroll
  for (int i = 0; i < V; ++i) {
    const int c = threadIdx.x + i * RN2_T;
    if (c >= d8) break;
    float f[8], dv[8], gv[8], o[8];
    unpack8(xv[i], f);
    unpack8(dv4[i], dv);
    unpack8(gv4[i], gv);
    unpack8(rv[i], o);  // zero without a residual gradient
#pragma unroll
    for (int j = 0; j < 8; ++j) o[j] += rs * dv[j] * gv[j] - f[j] * k;
    dres_out[row * d8 + c] = pack8(o);
  }
}

// ---------------------------------------------------------------- RoPE
// one CTA per (batch, position): the hd/2 angles pos * theta^(-2i/hd) are
// computed once in double, then every head at that position is rotated; with
// vec (hd a multiple of 16, x 16-byte aligned) each thread moves 8 pairs per
// 16-byte load and store.
__global__ void __launch_bounds__(128) rope_kernel(__nv_bfloat16* __restrict__ x, int seq, int heads, int hd,
                                                   double log_theta, int inverse, int vec) {
  extern __shared__ float cs[];  // [hd/2] cos, [hd/2] sin
  const int half = hd / 2;
  const int64_t bs = blockIdx.x;
  const int pos = (int)(bs % seq);
  for (int i = threadIdx.x; i < half; i += blockDim.x) {
    const double inv = exp(-2.0 * i / hd * log_theta);
    double s, c;
    sincos((double)pos * inv, &s, &c);
    cs[i] = (float)c;
    cs[half + i] = inverse ? -(float)s : (float)s;
  }
  __syncthreads();
  __nv_bfloat16* base = x + bs * (int64_t)heads * hd;
  if (vec) {
    const int nv = half / 8;  // 8-pair chunks per head
    for (int idx = threadIdx.x; idx < heads * nv; idx += blockDim.x) {
      const int h = idx / nv, i0 = (idx % nv) * 8;
      uint4* p1 = reinterpret_cast<uint4*>(base + (int64_t)h * hd + i0);
      uint4* p2 = reinterpret_cast<uint4*>(base + (int64_t)h * hd + half + i0);
      float a[8], b[8], o1[8], o2[8];
      unpack8(*p1, a);
      unpack8(*p2, b);
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        const float c = cs[i0 + k], sn = cs[half + i0 + k];
        o1[k] = a[k] * c - b[k] * sn;
        o2[k] = b[k] * c + a[k] * sn;
      }
      *p1 = pack8(o1);
      *p2 = pack8(o2);
    }
    return;
  }
  for (int idx = threadIdx.x; idx < heads * half; idx += blockDim.x) {
    const int h = idx / half, i = idx % half;
    __nv_bfloat16* p = base + (int64_t)h * hd + i;
    const float x1 = __bfloat162float(p[0]), x2 = __bfloat162float(p[half]);
    const float c = cs[i], s = cs[half + i];
    p[0] = __float2bfloat16_rn(x1 * c - x2 * s);
    p[half] = __float2bfloat16_rn(x2 * c + x1 * s);
  }
}

// (cos, sin) of pos * theta^(-2i/hd) for every position and frequency, with
// rope_kernel's double-precision angle and rounding to fp32, then the hd/2
// frequencies theta^(-2i/hd) themselves (fp32) after the n pairs
__global__ void __launch_bounds__(256) rope_table_kernel(float2* __restrict__ table, int64_t n, int half, int hd,
                                                         double log_theta) {
  for (int64_t idx = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; idx < n + half;
       idx += (int64_t)gridDim.x * blockDim.x) {
    if (idx >= n) {
      reinterpret_cast<float*>(table + n)[idx - n] = (float)exp(-2.0 * (int)(idx - n) / hd * log_theta);
      continue;
    }
    const int pos = (int)(idx / half), i = (int)(idx % half);
    const double inv = exp(-2.0 * i / hd * log_theta);
    double sn, c;
    sincos((double)pos * inv, &sn, &c);
    table[idx] = make_float2((float)c, (float)sn);
  }
}

// rope_kernel's rotation with the angles from a table (inverse: the transpose),
// for heads of hd % 16 == 0 on 16-byte aligned rows; one CTA per (batch, position)
__global__ void __launch_bounds__(128) rope_from_table_kernel(__nv_bfloat16* __restrict__ x,
                                                              const float2* __restrict__ table, int seq, int heads,
                                                              int hd, int inverse) {
  const int half = hd / 2;
  const int64_t bs = blockIdx.x;
  const float2* cs = table + (int64_t)(bs % seq) * half;
  __nv_bfloat16* base = x + bs * (int64_t)heads * hd;
  const int nv = half / 8;
  for (int idx = threadIdx.x; idx < heads * nv; idx += blockDim.x) {
    const int h = idx / nv, i0 = (idx % nv) * 8;
    uint4* p1 = reinterpret_cast<uint4*>(base + (int64_t)h * hd + i0);
    uint4* p2 = reinterpret_cast<uint4*>(base + (int64_t)h * hd + half + i0);
    float a[8], b[8], o1[8], o2[8];
    unpack8(*p1, a);
    unpack8(*p2, b);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float2 t = cs[i0 + k];
      const float c = t.x, sn = inverse ? -t.y : t.y;
      o1[k] = a[k] * c - b[k] * sn;
      o2[k] = b[k] * c + a[k] * sn;
    }
    *p1 = pack8(o1);
    *p2 = pack8(o2);
  }
}

// ---------------------------------------------------------------- SwiGLU
__device__ __forceinline__ float sigmoidf_(float g) { return 1.0f / (1.0f + expf(-g)); }

__global__ void __launch_bounds__(256) swiglu_fwd_kernel(const uint4* __restrict__ g, const uint4* __restrict__ u,
                                                         uint4* __restrict__ m, int64_t n8) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
    float gv[8], uv[8], o[8];
    unpack8(g[i], gv);
    unpack8(u[i], uv);
#pragma unroll
    for (int k = 0; k < 8; ++k) o[k] = gv[k] * sigmoidf_(gv[k]) * uv[k];
    m[i] = pack8(o);
  }
}

__global__ void __launch_bounds__(256) swiglu_bwd_kernel(const uint4* __restrict__ dm, const uint4* g, const uint4* u,
                                                         uint4* dg, uint4* du, int64_t n8) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n8; i += (int64_t)gridDim.x * blockDim.x) {
    float dv[8], gv[8], uv[8], og[8], ou[8];
    unpack8(dm[i], dv);
    unpack8(g[i], gv);
    unpack8(u[i], uv);
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const float sg = sigmoidf_(gv[k]);
      const float silu = gv[k] * sg;
      ou[k] = dv[k] * silu;
      og[k] = dv[k] * uv[k] * sg * (1.0f + gv[k] * (1.0f - sg));
    }
    dg[i] = pack8(og);
    du[i] = pack8(ou);
  }
}

// ---------------------------------------------------------------- embedding
__global__ void __launch_bounds__(128) embed_kernel(const int32_t* __restrict__ ids, const uint4* __restrict__ table,
                                                    uint4* __restrict__ h, int d8, int64_t vocab) {
  const int64_t row = blockIdx.x;
  const int32_t id = ids[row];
  const bool ok = id >= 0 && id < vocab;
  if (!ok && threadIdx.x == 0) report(LSQ_EINVAL, 801);
  for (int c = threadIdx.x; c < d8; c += blockDim.x)
    h[row * d8 + c] = ok ? table[(int64_t)id * d8 + c] : make_uint4(0, 0, 0, 0);
}

// ---------------------------------------------------------------- cross entropy
constexpr int XE_T = 512;

// per row: lse, row loss, dlogits = (softmax - onehot) * inv_count
__global__ void __launch_bounds__(XE_T) xent_row_kernel(const float* __restrict__ logits, const int32_t* __restrict__ ids,
                                                        int seq, int64_t V, float inv_count,
                                                        __nv_bfloat16* __restrict__ dlogits,
                                                        float* __restrict__ row_loss) {
  __shared__ float rm[XE_T / 32], rsum[XE_T / 32];
  const int64_t row = blockIdx.x;
  const int t = (int)(row % seq);
  const float* lr = logits + row * V;
  __nv_bfloat16* dr = dlogits + row * V;
  if (t == seq - 1) {  // no next token: ignored row
    for (int64_t c = threadIdx.x; c < V; c += XE_T) dr[c] = __float2bfloat16_rn(0.0f);
    if (threadIdx.x == 0) row_loss[row] = 0.0f;
    return;
  }
  const int32_t tgt = ids[row + 1];
  float m = -INFINITY, s = 0.0f;
  for (int64_t c = threadIdx.x; c < V; c += XE_T) {
    const float v = lr[c];
    if (v > m) {
      s = s * expf(m - v) + 1.0f;
      m = v;
    } else {
      s += expf(v - m);
    }
  }
  // combine (m, s) pairs: warp tree, then a fixed pass over the warps
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o), s2 = __shfl_xor_sync(0xffffffffu, s, o);
    const float mm = fmaxf(m, m2);
    s = (m == -INFINITY ? 0.0f : s * expf(m - mm)) + (m2 == -INFINITY ? 0.0f : s2 * expf(m2 - mm));
    m = mm;
  }
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) {
    rm[w] = m;
    rsum[w] = s;
  }
  __syncthreads();
  float M = -INFINITY, SS = 0.0f;
  for (int i = 0; i < XE_T / 32; ++i) {
    const float mm = fmaxf(M, rm[i]);
    SS = (M == -INFINITY ? 0.0f : SS * expf(M - mm)) + (rm[i] == -INFINITY ? 0.0f : rsum[i] * expf(rm[i] - mm));
    M = mm;
  }
  const float lse = M + logf(SS);
  const bool tgt_ok = tgt >= 0 && tgt < V;
  if (threadIdx.x == 0) {
    if (!tgt_ok) report(LSQ_EINVAL, 802);
    row_loss[row] = tgt_ok ? lse - lr[tgt] : 0.0f;
  }
  for (int64_t c = threadIdx.x; c < V; c += XE_T) {
    float p = expf(lr[c] - lse);
    if (c == tgt) p -= 1.0f;
    dr[c] = __float2bfloat16_rn(p * inv_count);
  }
}

__global__ void __launch_bounds__(1024) xent_mean_kernel(const float* __restrict__ row_loss, int64_t rows, float inv_count,
                                                         float* __restrict__ loss) {
  __shared__ float red[32];
  float s = 0.0f;
  for (int64_t i = threadIdx.x; i < rows; i += 1024) s += row_loss[i];
  const float tot = block_sum<1024>(s, red);
  if (threadIdx.x == 0) *loss = tot * inv_count;
}

// ---------------------------------------------------------------- sequence log-probabilities and DPO
// (preference losses on the same streamed base with the adapter off as the
// reference: aiany.app listing, "How It Works (concise)"; the objective is
// DPO, Rafailov et al. 2023, eq. 7)

// per row: lse and log p(target) (0 on the last row of a sequence)
__global__ void __launch_bounds__(XE_T) seqlp_row_kernel(const float* __restrict__ logits,
                                                         const int32_t* __restrict__ ids, int seq, int64_t V,
                                                         float* __restrict__ row_lse, float* __restrict__ row_lp) {
  __shared__ float rm[XE_T / 32], rsum[XE_T / 32];
  const int64_t row = blockIdx.x;
  const int t = (int)(row % seq);
  const float* lr = logits + row * V;
  float m = -INFINITY, s = 0.0f;
  for (int64_t c = threadIdx.x; c < V; c += XE_T) {
    const float v = lr[c];
    if (v > m) {
      s = s * expf(m - v) + 1.0f;
      m = v;
    } else {
      s += expf(v - m);
    }
  }
#pragma unroll
  for (int o = 16; o; o >>= 1) {
    const float m2 = __shfl_xor_sync(0xffffffffu, m, o), s2 = __shfl_xor_sync(0xffffffffu, s, o);
    const float mm = fmaxf(m, m2);
    s = (m == -INFINITY ? 0.0f : s * expf(m - mm)) + (m2 == -INFINITY ? 0.0f : s2 * expf(m2 - mm));
    m = mm;
  }
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) {
    rm[w] = m;
    rsum[w] = s;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float M = -INFINITY, SS = 0.0f;
    for (int i = 0; i < XE_T / 32; ++i) {
      const float mm = fmaxf(M, rm[i]);
      SS = (M == -INFINITY ? 0.0f : SS * expf(M - mm)) + (rm[i] == -INFINITY ? 0.0f : rsum[i] * expf(rm[i] - mm));
      M = mm;
    }
    const float lse = M + logf(SS);
    row_lse[row] = lse;
    float lp = 0.0f;
    if (t < seq - 1) {
      const int32_t tgt = ids[row + 1];
      if (tgt >= 0 && tgt < V) lp = lr[tgt] - lse;
      else report(LSQ_EINVAL, 803);
    }
    row_lp[row] = lp;
  }
}

// per sequence: sum of its rows' log p in a fixed order
__global__ void __launch_bounds__(1024) seqlp_sum_kernel(const float* __restrict__ row_lp, int seq,
                                                         float* __restrict__ seq_logp) {
  __shared__ float red[32];
  const int64_t b = blockIdx.x;
  float s = 0.0f;
  for (int t = threadIdx.x; t < seq; t += 1024) s += row_lp[b * seq + t];
  const float tot = block_sum<1024>(s, red);
  if (threadIdx.x == 0) seq_logp[b] = tot;
}

// loss = mean_i softplus(-z_i), z_i = beta ((pi_c - ref_c) - (pi_r - ref_r)); dseq = d loss / d pi
__global__ void __launch_bounds__(32) dpo_loss_kernel(const float* __restrict__ pi, const float* __restrict__ ref,
                                                      int npairs, float beta, float* __restrict__ loss,
                                                      float* __restrict__ dseq) {
  if (threadIdx.x != 0) return;
  float tot = 0.0f;
  for (int i = 0; i < npairs; ++i) {
    const float z = beta * ((pi[2 * i] - ref[2 * i]) - (pi[2 * i + 1] - ref[2 * i + 1]));
    tot += fmaxf(-z, 0.0f) + log1pf(expf(-fabsf(z)));           // softplus(-z), no overflow
    const float sig_neg = z >= 0.0f ? expf(-z) / (1.0f + expf(-z)) : 1.0f / (1.0f + expf(z));  // sigmoid(-z)
    const float g = beta * sig_neg / (float)npairs;
    dseq[2 * i] = -g;
    dseq[2 * i + 1] = g;
  }
  *loss = tot / (float)npairs;
}

// dlogits = dseq[b] * (onehot(target) - softmax), zero on the last row of a sequence
__global__ void __launch_bounds__(XE_T) seqlp_bwd_kernel(const float* __restrict__ logits,
                                                         const int32_t* __restrict__ ids, int seq, int64_t V,
                                                         const float* __restrict__ row_lse,
                                                         const float* __restrict__ dseq,
                                                         __nv_bfloat16* __restrict__ dlogits) {
  const int64_t row = blockIdx.x;
  const int t = (int)(row % seq);
  const float* lr = logits + row * V;
  __nv_bfloat16* dr = dlogits + row * V;
  if (t == seq - 1) {
    for (int64_t c = threadIdx.x; c < V; c += XE_T) dr[c] = __float2bfloat16_rn(0.0f);
    return;
  }
  const float g = dseq[row / seq], lse = row_lse[row];
  const int32_t tgt = ids[row + 1];
  for (int64_t c = threadIdx.x; c < V; c += XE_T) {
    float p = -expf(lr[c] - lse);
    if (c == tgt) p += 1.0f;
    dr[c] = __float2bfloat16_rn(g * p);
  }
}

// ---------------------------------------------------------------- AdamW
__global__ void __launch_bounds__(256) adamw_kernel(float* __restrict__ p, const float* __restrict__ g,
                                                    float* __restrict__ m, float* __restrict__ v,
                                                    __nv_bfloat16* __restrict__ pb, int64_t n, float lr, float b1,
                                                    float b2, float eps, float wd, float bc1, float bc2) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x) {
    const float gi = g[i];
    const float mi = b1 * m[i] + (1.0f - b1) * gi;
    const float vi = b2 * v[i] + (1.0f - b2) * gi * gi;
    m[i] = mi;
    v[i] = vi;
    const float mh = mi / bc1, vh = vi / bc2;
    const float pi = p[i] - lr * (mh / (sqrtf(vh) + eps) + wd * p[i]);
    p[i] = pi;
    if (pb) pb[i] = __float2bfloat16_rn(pi);
  }
}

// the bf16 operand copies of fp32 masters, refreshed without an optimizer step
// (the rounding adamw_kernel applies after each update)
__global__ void __launch_bounds__(256) refresh_bf16_kernel(const float* __restrict__ p, __nv_bfloat16* __restrict__ pb,
                                                           int64_t n) {
  for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
    pb[i] = __float2bfloat16_rn(p[i]);
}

static unsigned grid_for(int64_t n, int threads) {
  int64_t g = (n + threads - 1) / threads;
  const int64_t cap = (int64_t)num_sms() * 32;
  if (g > cap) g = cap;
  if (g < 1) g = 1;
  return (unsigned)g;
}

}  // namespace ops
}  // namespace lsq

using namespace lsq;
using namespace lsq::ops;

extern "C" lsq_status lsq_rmsnorm_fwd(const void* x, const void* g, void* y, float* rstd, int64_t rows, int64_t d,
                                      float eps, lsq_cuda_stream stream) {
  if (!x || !g || !y) return fail(LSQ_EINVAL, "lsq_rmsnorm_fwd: NULL argument");
  if (rows < 1 || d < 8 || d % 8 != 0) return fail(LSQ_EINVAL, "lsq_rmsnorm_fwd: need rows >= 1, d % 8 == 0");
  if (!aligned(x, 16) || !aligned(g, 16) || !aligned(y, 16)) return fail(LSQ_EINVAL, "lsq_rmsnorm_fwd: alignment");
  lsq_status st = check_device();
  if (st != LSQ_OK) return st;
  const int d8 = (int)(d / 8), v = (d8 + RN2_T - 1) / RN2_T;
  const unsigned nb = (unsigned)rows;
  const float inv_d = 1.0f / (float)d;
  cudaStream_t cs = (cudaStream_t)stream;
  const uint4 *xx = (const uint4*)x, *gg = (const uint4*)g;
  uint4* yy = (uint4*)y;
  if (v <= 1) rmsnorm_fwd_reg_kernel<1><<<nb, RN2_T, 0, cs>>>(xx, gg, yy, rstd, d8, inv_d, eps);
  else if (v <= 2) rmsnorm_fwd_reg_kernel<2><<<nb, RN2_T, 0, cs>>>(xx, gg, yy, rstd, d8, inv_d, eps);
  else if (v <= 4) rmsnorm_fwd_reg_kernel<4><<<nb, RN2_T, 0, cs>>>(xx, gg, yy, rstd, d8, inv_d, eps);
  else if (v <= 8) rmsnorm_fwd_reg_kernel<8><<<nb, RN2_T, 0, cs>>>(xx, gg, yy, rstd, d8, inv_d, eps);
  else rmsnorm_fwd_kernel<<<nb, RN_T, 0, cs>>>(xx, gg, yy, rstd, d8, inv_d, eps);
  LSQ_LAUNCH_CHECK("rmsnorm_fwd_kernel");
  return LSQ_OK;
}

extern "C" lsq_status lsq_rmsnorm_bwd(const void* dy, const void* x, const void* g, const float* rstd,
                                      const void* dres_in, void* dres_out, int64_t rows, int64_t d,
                                      lsq_cuda_stream stream) {
  if (!dy || !x || !g || !rstd || !dres_out) return fail(LSQ_EINVAL, "lsq_rmsnorm_bwd: NULL argument");
  if (rows < 1 || d < 8 || d % 8 != 0) return fail(LSQ_EINVAL, "lsq_rmsnorm_bwd: need rows >= 1, d % 8 == 0");
  if (!aligned(dy, 16) || !aligned(x, 16) || !aligned(g, 16) || !aligned(dres_out, 16) ||
      (dres_in && !aligned(dres_in, 16)))
    return fail(LSQ_EINVAL, "lsq_rmsnorm_bwd: alignment");
  lsq_status st = check_device();
  if (st != LSQ_OK) return st;
  const int d8 = (int)(d / 8), v = (d8 + RN2_T - 1) / RN2_T;
  const unsigned nb = (unsigned)rows;
  const float inv_d = 1.0f / (float)d;
  cudaStream_t cs = (cudaStream_t)stream;
  const uint4 *dd = (const uint4*)dy, *xx = (const uint4*)x, *gg = (const uint4*)g, *ri = (const uint4*)dres_in;
  uint4* ro = (uint4*)dres_out;
  if (v <= 1) rmsnorm_bwd_reg_kernel<1><<<nb, RN2_T, 0, cs>>>(dd, xx, gg, rstd, ri, ro, d8, inv_d);
  else if (v <= 2) rmsnorm_bwd_reg_kernel<2><<<nb, RN2_T, 0, cs>>>(dd, xx, gg, rstd, ri, ro, d8, inv_d);
  else if (v <= 4) rmsnorm_bwd_reg_kernel<4><<<nb, RN2_T, 0, cs>>>(dd, xx, gg, rstd, ri, ro, d8, inv_d);
  else if (v <= 8) rmsnorm_bwd_reg_kernel<8><<<nb, RN2_T, 0, cs>>>(dd, xx, gg, rstd, ri, ro, d8, inv_d);
  else rmsnorm_bwd_kernel<<<nb, RN_T, 0, cs>>>(dd, xx, gg, rstd, ri, ro, d8, inv_d);
  LSQ_LAUNCH_CHECK("rmsnorm_bwd_kernel");
  return LSQ_OK;
}

extern "C" lsq_status lsq_rope(void* x, int64_t batch, int64_t seq, int64_t heads, int64_t hd, float theta,
                               int32_t inverse, lsq_cuda_stream stream) {
  if (!x) return fail(LSQ_EINVAL, "lsq_rope: NULL argument");
  if (batch < 1 || seq < 1 || heads < 1 || hd < 2 || hd % 2 != 0 || hd > 1024 || !(theta > 1.0f))
    return fail(LSQ_EINVAL, "lsq_rope: bad shape or theta");
  lsq_status st = check_device();
  if (st != LSQ_OK) return st;
  rope_kernel<<<(unsigned)(batch * seq), 128, (size_t)hd * sizeof(float), (cudaStream_t)stream>>>(
      static_cast<__nv_bfloat16*>(x), (int)seq, (int)heads, (int)hd, log((double)theta), inverse ? 1 : 0,
      (hd % 16 == 0 && aligned(x, 16)) ? 1 : 0);
  LSQ_LAUNCH_CHECK("rope_kernel");
  return LSQ_OK;
}

extern "C" size_t lsq_rope_table_size(int64_t seq, int64_t hd) {
  if (seq < 1 || hd < 2) return 16;
  return ((size_t)(seq * hd + hd / 2) * sizeof(float) + 15) / 16 * 16;
}

extern "C" lsq_status lsq_rope_table(float theta, int64_t seq, int64_t hd, float* table, lsq_cuda_stream stream) {
  if (!table) return fail(LSQ_EINVAL, "lsq_rope_table: NULL argument");
  if (seq < 1 || seq > (1 << 24) || hd < 2 || hd % 2 != 0 || hd > 1024 || !(theta > 1.0f))
    return fail(LSQ_EINVAL, "lsq_rope_table: bad shape or theta");
  lsq_status st = check_device();
  if (st != LSQ_OK) return st;
  const int64_t n = seq * (hd / 2);
  rope_table_kernel<<<grid_for(n + hd / 2, 256), 256, 0, (cudaStream_t)stream>>>(reinterpret_cast<float2*>(table), n,
                                                                         (int)(hd / 2), (int)hd, log((double)theta));
  LSQ_LAUNCH_CHECK("rope_table_kernel");
  return LSQ_OK;
}

namespace lsq {
namespace ops {
// the rotation (or its transpose) of x [batch, seq, heads, hd] with a table from lsq_rope_table
lsq_status rope_from_table(void* x, const float* table, int64_t batch, int64_t seq, int64_t heads, int64_t hd,
                           int inverse, cudaStream_t stream) {
  if (hd % 16 != 0 || !aligned(x, 16) || !aligned(table, 8))
    return fail(LSQ_EINVAL, "rope from a table: hd a multiple of 16 and 16-byte aligned rows");
  rope_from_table_kernel<<<(unsigned)(batch * seq), 128, 0, stream>>>(
      static_cast<__nv_bfloat16*>(x), reinterpret_cast<const float2*>(table), (int)seq, (int)heads, (int)hd, inverse);
  LSQ_LAUNCH_CHECK("rope_from_table_kernel");
  return LSQ_OK;
}
}  // namespace ops
}  // namespace lsq

extern "C" lsq_status lsq_swiglu_fwd(const void* g, const void* u, void* m, int64_t n, lsq_cuda_stream stream) {
  if (!g || !u || !m) return fail(LSQ_EINVAL, "lsq_swiglu_fwd: NULL argument");
  if (n < 8 || n % 8 != 0) return fail(LSQ_EINVAL, "lsq_swiglu_fwd: n must be a multiple of 8");
  if (!aligned(g, 16) || !aligned(u, 16) || !aligned(m, 16)) return fail(LSQ_EINVAL, "lsq_swiglu_fwd: alignment");
  lsq_status st = check_device();
  if (st != LSQ_OK) return st;
  swiglu_fwd_kernel<<<grid_for(n / 8, 256), 256, 0, (cudaStream_t)stream>>>((const uint4*)g, (const uint4*)u,
                                                                            (uint4*)m, n / 8);
  LSQ_LAUNCH_CHECK("swiglu_fwd_kernel");
  return LSQ_OK;
}

extern "C" lsq_status lsq_swiglu_bwd(const void* dm, const void* g, const void* u, void* dg, void* du, int64_t n,
                                     lsq_cuda_stream stream) {
  if (!dm || !g || !u || !dg || !du) return fail(LSQ_EINVAL, "lsq_swiglu_bwd: NULL argument");
  if (n < 8 || n % 8 != 0) return fail(LSQ_EINVAL, "lsq_swiglu_bwd: n must be a multiple of 8");
  if (!aligned(dm, 16) || !aligned(g, 16) || !aligned(u, 16) || !aligned(dg, 16) || !aligned(du, 16))
    return fail(LSQ_EINVAL, "lsq_swiglu_bwd: alignment");
  lsq_status st = check_device();
  if (st != LSQ_OK) return st;
  swiglu_bwd_kernel<<<grid_for(n / 8, 256), 256, 0, (cudaStream_t)stream>>>(
      (const uint4*)dm, (const uint4*)g, (const uint4*)u, (uint4*)dg, (uint4*)du, n / 8);
  LSQ_LAUNCH_CHECK("swiglu_bwd_kernel");
  return LSQ_OK;
}

extern "C" lsq_status lsq_embed_gather(const int32_t* ids, const void* table, void* h, int64_t rows, int64_t d,
                                       int64_t vocab, lsq_cuda_stream stream) {
  if (!ids || !table || !h) return fail(LSQ_EINVAL, "lsq_embed_gather: NULL argument");
  if (rows < 1 || d < 8 || d % 8 != 0 || vocab < 1) return fail(LSQ_EINVAL, "lsq_embed_gather: bad shape");
  if (!aligned(table, 16) || !aligned(h, 16)) return fail(LSQ_EINVAL, "lsq_embed_gather: alignment");
  lsq_status st = check_device();
  if (st != LSQ_OK) return st;
  embed_kernel<<<(unsigned)rows, 128, 0, (cudaStream_t)stream>>>(ids, (const uint4*)table, (uint4*)h, (int)(d / 8),
                                                                 vocab);
  LSQ_LAUNCH_CHECK("embed_kernel");
  return LSQ_OK;
}

extern "C" size_t lsq_xent_workspace_size(int64_t rows) {
  return (size_t)((rows > 0 ? rows : 1) * sizeof(float) + 255) / 256 * 256;
}

extern "C" lsq_status lsq_xent_fwd_bwd(const float* logits, const int32_t* ids, int64_t batch, int64_t seq, int64_t V,
                                       float* loss, void* dlogits, void* workspace, size_t workspace_bytes,
                                       lsq_cuda_stream stream) {
  if (!logits || !ids || !loss || !dlogits || !workspace) return fail(LSQ_EINVAL, "lsq_xent_fwd_bwd: NULL argument");
  if (batch < 1 || seq < 2 || V < 2) return fail(LSQ_EINVAL, "lsq_xent_fwd_bwd: need batch >= 1, seq >= 2, V >= 2");
  const int64_t rows = batch * seq;
  if (workspace_bytes < lsq_xent_workspace_size(rows)) return fail(LSQ_EINVAL, "lsq_xent_fwd_bwd: workspace too small");
  lsq_status st = check_device();
  if (st != LSQ_OK) return st;
  const float inv = 1.0f / (float)(batch * (seq - 1));
  float* rl = static_cast<float*>(workspace);
  xent_row_kernel<<<(unsigned)rows, XE_T, 0, (cudaStream_t)stream>>>(logits, ids, (int)seq, V, inv,
                                                                     static_cast<__nv_bfloat16*>(dlogits), rl);
  LSQ_LAUNCH_CHECK("xent_row_kernel");
  xent_mean_kernel<<<1, 1024, 0, (cudaStream_t)stream>>>(rl, rows, inv, loss);
  LSQ_LAUNCH_CHECK("xent_mean_kernel");
  return LSQ_OK;
}

extern "C" size_t lsq_seq_logprob_workspace_size(int64_t rows) {
  return (size_t)((rows > 0 ? rows : 1) * sizeof(float) + 255) / 256 * 256;
}

extern "C" lsq_status lsq_seq_logprob(const float* logits, const int32_t* ids, int64_t batch, int64_t seq, int64_t V,
                                      float* row_lse, float* seq_logp, void* workspace, size_t workspace_bytes,
                                      lsq_cuda_stream stream) {
  if (!logits || !ids || !row_lse || !seq_logp || !workspace) return fail(LSQ_EINVAL, "lsq_seq_logprob: NULL argument");
  if (batch < 1 || seq < 2 || V < 2) return fail(LSQ_EINVAL, "lsq_seq_logprob: need batch >= 1, seq >= 2, V >= 2");
  const int64_t rows = batch * seq;
  if (workspace_bytes < lsq_seq_logprob_workspace_size(rows))
    return fail(LSQ_EINVAL, "lsq_seq_logprob: workspace too small");
  lsq_status st = check_device();
  if (st != LSQ_OK) return st;
  float* rl = static_cast<float*>(workspace);
  seqlp_row_kernel<<<(unsigned)rows, XE_T, 0, (cudaStream_t)stream>>>(logits, ids, (int)seq, V, row_lse, rl);
  LSQ_LAUNCH_CHECK("seqlp_row_kernel");
  seqlp_sum_kernel<<<(unsigned)batch, 1024, 0, (cudaStream_t)stream>>>(rl, (int)seq, seq_logp);
  LSQ_LAUNCH_CHECK("seqlp_sum_kernel");
  return LSQ_OK;
}

extern "C" lsq_status lsq_dpo_loss(const float* policy_logp, const float* ref_logp, int32_t npairs, float beta,
                                   float* loss, float* dseq, lsq_cuda_stream stream) {
  if (!policy_logp || !ref_logp || !loss || !dseq) return fail(LSQ_EINVAL, "lsq_dpo_loss: NULL argument");
  if (npairs < 1) return fail(LSQ_EINVAL, "lsq_dpo_loss: npairs must be >= 1");
  lsq_status st = check_device();
  if (st != LSQ_OK) return st;
  dpo_loss_kernel<<<1, 32, 0, (cudaStream_t)stream>>>(policy_logp, ref_logp, npairs, beta, loss, dseq);
  LSQ_LAUNCH_CHECK("dpo_loss_kernel");
  return LSQ_OK;
}

extern "C" lsq_status lsq_seq_logprob_bwd(const float* logits, const int32_t* ids, int64_t batch, int64_t seq,
                                          int64_t V, const float* row_lse, const float* dseq, void* dlogits,
                                          lsq_cuda_stream stream) {
  if (!logits || !ids || !row_lse || !dseq || !dlogits) return fail(LSQ_EINVAL, "lsq_seq_logprob_bwd: NULL argument");
  if (batch < 1 || seq < 2 || V < 2) return fail(LSQ_EINVAL, "lsq_seq_logprob_bwd: need batch >= 1, seq >= 2, V >= 2");
  lsq_status st = check_device();
  if (st != LSQ_OK) return st;
  seqlp_bwd_kernel<<<(unsigned)(batch * seq), XE_T, 0, (cudaStream_t)stream>>>(
      logits, ids, (int)seq, V, row_lse, dseq, static_cast<__nv_bfloat16*>(dlogits));
  LSQ_LAUNCH_CHECK("seqlp_bwd_kernel");
  return LSQ_OK;
}

extern "C" lsq_status lsq_lora_refresh_bf16(const float* p, void* p_bf16, int64_t n, lsq_cuda_stream stream) {
  if (!p || !p_bf16) return fail(LSQ_EINVAL, "lsq_lora_refresh_bf16: NULL argument");
  if (n < 1) return fail(LSQ_EINVAL, "lsq_lora_refresh_bf16: need n >= 1");
  lsq_status st = check_device();
  if (st != LSQ_OK) return st;
  refresh_bf16_kernel<<<grid_for(n, 256), 256, 0, (cudaStream_t)stream>>>(p, static_cast<__nv_bfloat16*>(p_bf16), n);
  LSQ_LAUNCH_CHECK("refresh_bf16_kernel");
  return LSQ_OK;
}

extern "C" lsq_status lsq_adamw_step(float* p, const float* g, float* m, float* v, void* p_bf16, int64_t n,
                                     int32_t step, float lr, float beta1, float beta2, float eps, float weight_decay,
                                     lsq_cuda_stream stream) {
  if (!p || !g || !m || !v) return fail(LSQ_EINVAL, "lsq_adamw_step: NULL argument");
  if (n < 1 || step < 1) return fail(LSQ_EINVAL, "lsq_adamw_step: need n >= 1 and step >= 1");
  lsq_status st = check_device();
  if (st != LSQ_OK) return st;
  const float bc1 = (float)(1.0 - pow((double)beta1, (double)step));
  const float bc2 = (float)(1.0 - pow((double)beta2, (double)step));
  adamw_kernel<<<grid_for(n, 256), 256, 0, (cudaStream_t)stream>>>(p, g, m, v, static_cast<__nv_bfloat16*>(p_bf16), n,
                                                                   lr, beta1, beta2, eps, weight_decay, bc1, bc2);
  LSQ_LAUNCH_CHECK("adamw_kernel");
  return LSQ_OK;
}
