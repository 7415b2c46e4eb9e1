// Status reporting, device checks, the NF4 codebook and TMA descriptor
// encoding for the lsq library.
#include <cmath>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "host_common.h"

namespace lsq {

static thread_local char t_msg[512] = "";

lsq_status fail(lsq_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_msg, sizeof(t_msg), fmt, ap);
  va_end(ap);
  return s;
}

lsq_status cuda_fail(cudaError_t e, const char* what) {
  return fail(LSQ_ECUDA, "%s: %s", what, cudaGetErrorString(e));
}

static int g_dev_ok[64];  // 0 unknown, 1 ok, 2 unsupported
static int g_dev_sms[64];
static std::mutex g_dev_mu;

lsq_status check_device() {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(LSQ_EUNSUPPORTED, "device index %d out of range", dev);
  if (g_dev_ok[dev] == 1) return LSQ_OK;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  int major = 0, minor = 0, sms = 0;
  LSQ_CUDA_TRY(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
  LSQ_CUDA_TRY(cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev));
  LSQ_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  if (major != 10 || minor != 0) {
    g_dev_ok[dev] = 2;
    return fail(LSQ_EUNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a only", dev, major,
                minor);
  }
  g_dev_sms[dev] = sms;
  g_dev_ok[dev] = 1;
  return LSQ_OK;
}

int num_sms() {
  int dev = 0;
  cudaGetDevice(&dev);
  return (dev >= 0 && dev < 64 && g_dev_sms[dev] > 0) ? g_dev_sms[dev] : 148;
}

// ------------------------------------------------------------------ codebook
// NormalFloat-4 levels (QLoRA construction): 8 positive quantiles of the
// standard normal at probabilities evenly spaced from delta down to 1/2 (the
// 1/2 point excluded), 7 negative ones from 8 points, and an exact zero;
// scaled so the largest is 1; delta = 1 - (1/30 + 1/32)/2.  The inverse CDF
// is found by Newton's method on Phi(x) = erfc(-x/sqrt 2)/2, in double, then
// polished to the double nearest the root.
static double phi_cdf(double x) { return 0.5 * std::erfc(-x / std::sqrt(2.0)); }
static double phi_pdf(double x) { return std::exp(-0.5 * x * x) / std::sqrt(2.0 * M_PI); }

static double probit(double p) {
  double x = 0.0;
  for (int it = 0; it < 100; ++it) {
    double step = (phi_cdf(x) - p) / phi_pdf(x);
    double nx = x - step;
    if (nx == x) break;
    x = nx;
  }
  // polish: walk one ulp at a time while the neighbour is closer
  for (int it = 0; it < 8; ++it) {
    double up = std::nextafter(x, 1e300), dn = std::nextafter(x, -1e300);
    double e0 = std::fabs(phi_cdf(x) - p);
    if (std::fabs(phi_cdf(up) - p) < e0) x = up;
    else if (std::fabs(phi_cdf(dn) - p) < e0) x = dn;
    else break;
  }
  return x;
}

static float g_cb[16];
static float g_thr[15];
static std::once_flag g_cb_once;

static void build_codebook() {
  const double delta = 1.0 - 0.5 * (1.0 / 30.0 + 1.0 / 32.0);
  double v[16];
  int n = 0;
  {
    volatile double step = (0.5 - delta) / 8.0;  // 9 points, last (= 1/2) dropped
    for (int i = 0; i < 8; ++i) {
      volatile double t = (double)i * step;
      v[n++] = probit(t + delta);
    }
  }
  {
    volatile double step = (0.5 - delta) / 7.0;  // 8 points, last dropped
    for (int i = 0; i < 7; ++i) {
      volatile double t = (double)i * step;
      v[n++] = -probit(t + delta);
    }
  }
  v[n++] = 0.0;
  // sort ascending (insertion sort on 16 values)
  for (int i = 1; i < 16; ++i) {
    double key = v[i];
    int j = i - 1;
    while (j >= 0 && v[j] > key) {
      v[j + 1] = v[j];
      --j;
    }
    v[j + 1] = key;
  }
  const double mx = v[15];
  for (int i = 0; i < 16; ++i) g_cb[i] = (float)(v[i] / mx);
  // decision threshold between levels i and i+1: the smallest fp32 strictly
  // above their midpoint (exact in double); a value on the midpoint keeps the
  // lower level.
  for (int i = 0; i < 15; ++i) {
    double mid = ((double)g_cb[i] + (double)g_cb[i + 1]) * 0.5;
    float t = (float)mid;
    if ((double)t <= mid) t = std::nextafterf(t, 2.0f);
    g_thr[i] = t;
  }
}

const float* codebook() {
  std::call_once(g_cb_once, build_codebook);
  return g_cb;
}
const float* thresholds() {
  std::call_once(g_cb_once, build_codebook);
  return g_thr;
}

// ------------------------------------------------------------------ TMA
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

lsq_status encode_tmap_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner,
                          uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                          CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return fail(LSQ_ECUDA, "cuTensorMapEncodeTiled entry point unavailable");
  if (!aligned(base, 16) || row_bytes % 16 != 0)
    return fail(LSQ_EINVAL, "TMA operand needs a 16-byte aligned base and row pitch (pitch %llu)",
                (unsigned long long)row_bytes);
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t es[2] = {1, 1};
  CUresult r = fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, swz,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(LSQ_ECUDA, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return LSQ_OK;
}

// One thread waits, in stream order, until *flag == value (acquire load at GPU
// scope), giving up after limit_ns of the global timer with LSQ_ETIMEOUT at
// site 901: the same bounded wait the stream-K finishers run on their flags.
__global__ void wait_flag_kernel(const unsigned long long* flag, unsigned long long value, unsigned long long limit_ns) {
  const uint64_t t0 = globaltimer();
  while (true) {
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(flag) : "memory");
    if (v == value) return;
    if (globaltimer() - t0 > limit_ns) {
      report(LSQ_ETIMEOUT, 901);
      return;
    }
  }
}

}  // namespace lsq

extern "C" {

const char* lsq_status_str(lsq_status s) {
  switch (s) {
    case LSQ_OK: return "ok";
    case LSQ_EINVAL: return "invalid argument";
    case LSQ_ENOTPINNED: return "host memory is not page-locked";
    case LSQ_ECUDA: return "CUDA error";
    case LSQ_ETIMEOUT: return "device wait timed out";
    case LSQ_ESTATE: return "call out of order";
    case LSQ_EUNSUPPORTED: return "unsupported device or size";
    case LSQ_ECALLBACK: return "a caller-supplied callback failed";
  }
  return "unknown status";
}

const char* lsq_last_error(void) { return lsq::t_msg; }

int lsq_version(void) { return 100; }

lsq_status lsq_wait_flag(const uint64_t* flag, uint64_t value, int64_t limit_ns, lsq_cuda_stream stream) {
  if (!flag || !lsq::aligned(flag, 8)) return lsq::fail(LSQ_EINVAL, "lsq_wait_flag: flag NULL or not 8-byte aligned");
  if (limit_ns < 1 || limit_ns > 10000000000ll)
    return lsq::fail(LSQ_EINVAL, "lsq_wait_flag: limit_ns must be in [1, 1e10] (got %lld)", (long long)limit_ns);
  lsq_status st = lsq::check_device();
  if (st != LSQ_OK) return st;
  lsq::wait_flag_kernel<<<1, 1, 0, (cudaStream_t)stream>>>(reinterpret_cast<const unsigned long long*>(flag),
                                                          (unsigned long long)value, (unsigned long long)limit_ns);
  LSQ_LAUNCH_CHECK("wait_flag_kernel");
  return LSQ_OK;
}

lsq_status lsq_device_status(int32_t* status, int32_t* where) {
  if (!status || !where) return lsq::fail(LSQ_EINVAL, "NULL output");
  int s = 0, w = 0, zero = 0;
  LSQ_CUDA_TRY(cudaMemcpyFromSymbol(&s, lsq::g_status, sizeof(int)));
  LSQ_CUDA_TRY(cudaMemcpyFromSymbol(&w, lsq::g_status_where, sizeof(int)));
  LSQ_CUDA_TRY(cudaMemcpyToSymbol(lsq::g_status, &zero, sizeof(int)));
  LSQ_CUDA_TRY(cudaMemcpyToSymbol(lsq::g_status_where, &zero, sizeof(int)));
  *status = s;
  *where = w;
  return LSQ_OK;
}

lsq_status lsq_nf4_codebook(float out[16]) {
  if (!out) return lsq::fail(LSQ_EINVAL, "NULL output");
  std::memcpy(out, lsq::codebook(), 16 * sizeof(float));
  return LSQ_OK;
}

}  // extern "C"
