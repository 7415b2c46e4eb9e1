// Backward of the fused NF4-LoRA linear for callers that cannot allocate
// device memory.  Same computation and kernels as lsq_nf4_lora_bwd; the
// scratch (G = dY B, its partial sums, the padded LoRA operands and the dA/dB
// partial sums) lives in a fixed array that the library itself holds in
// device memory.
//
// Who needs it: code that runs where a cudaMalloc is not allowed or not
// possible - a host framework that owns the whole device memory pool and hands
// out no allocator, a process held to a hard memory cap where an extra
// allocation in the middle of a step could fail, or work enqueued while a
// stream is being captured.  Such a caller still passes every input and output
// buffer; only the scratch is provided here.
#include <mutex>

#include "host_common.h"

namespace lsq {
namespace noalloc {

// Largest scratch the entry point serves: 32 MiB, which covers any one linear
// of the 8B shape at 2048 tokens and r = 16 (9.1 MiB for a 4096 x 4096
// projection, 14.9 MiB for gate or up, 15.9 MiB for the 14336-wide down
// projection).  Every GPU that loads the library keeps this array for as
// long as the process lives.
constexpr size_t SCRATCH_BYTES = size_t(32) << 20;

static __device__ __align__(256) unsigned char g_bwd_scratch[SCRATCH_BYTES];

// Device address of g_bwd_scratch, looked up once per device (the symbol's
// name in host code is only a host-side handle, not a device address).
static void* g_addr[64];
static std::once_flag g_once[64];
static cudaError_t g_err[64];

static lsq_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "lsq_nf4_lora_bwd_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(LSQ_EUNSUPPORTED, "lsq_nf4_lora_bwd_noalloc: device %d out of range", dev);
  std::call_once(g_once[dev], [dev] {
    void* p = nullptr;
    g_err[dev] = cudaGetSymbolAddress(&p, g_bwd_scratch);
    g_addr[dev] = (g_err[dev] == cudaSuccess) ? p : nullptr;
  });
  if (g_err[dev] != cudaSuccess || !g_addr[dev])
    return cuda_fail(g_err[dev], "lsq_nf4_lora_bwd_noalloc: cudaGetSymbolAddress of the scratch array");
  *out = g_addr[dev];
  return LSQ_OK;
}

}  // namespace noalloc
}  // namespace lsq

extern "C" size_t lsq_nf4_lora_bwd_noalloc_max_scratch(void) { return lsq::noalloc::SCRATCH_BYTES; }

extern "C" lsq_status lsq_nf4_lora_bwd_noalloc(const lsq_nf4_weight* W, const void* x, const void* dy, int64_t M,
                                               const void* A, const void* B, int32_t r, float s, const float* u,
                                               void* dx, float* dA, float* dB, int32_t accumulate,
                                               lsq_cuda_stream stream) {
  using namespace lsq;
  if (!W) return fail(LSQ_EINVAL, "lsq_nf4_lora_bwd_noalloc: NULL weight");
  const int64_t n_out = W->n_out;
  if (M < 1 || r < 0 || r > 64 || W->k_in < 64) return fail(LSQ_EINVAL, "lsq_nf4_lora_bwd_noalloc: bad sizes");
  const size_t need = bwd_base_bytes(1, M, W->k_in, &n_out, r);
  if (need > noalloc::SCRATCH_BYTES)
    return fail(LSQ_EINVAL,
                "lsq_nf4_lora_bwd_noalloc: this size needs %zu bytes of scratch, more than the %zu-byte array the "
                "library holds; use lsq_nf4_lora_bwd with a caller workspace",
                need, noalloc::SCRATCH_BYTES);
  void* ws = nullptr;
  lsq_status st = noalloc::scratch_address(&ws);
  if (st != LSQ_OK) return st;
  return lsq_nf4_lora_bwd(W, x, dy, M, A, B, r, s, u, dx, dA, dB, accumulate, ws, noalloc::SCRATCH_BYTES, stream);
}
