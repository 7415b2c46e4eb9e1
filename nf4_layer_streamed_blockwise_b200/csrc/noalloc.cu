// Backward of the fused NF4-LoRA linear for callers that cannot allocate
// device memory.  Same computation and kernels as lsq_nf4_lora_bwd; the
// scratch (G = dY B, its partial sums, the padded LoRA operands, the dA/dB
// partial sums and the stream-K partials of the dX GEMM) lives in a fixed
// array that the library itself holds in device memory.
//
// Who needs it: code that runs where a cudaMalloc is not allowed or not
// possible - a host framework that owns the whole device memory pool and hands
// out no allocator, or a process held to a hard memory cap where an extra
// allocation in the middle of a step could fail.  Such a caller still passes
// every input and output buffer; only the scratch is provided here.
#include <atomic>

#include "host_common.h"

namespace lsq {
namespace noalloc {

// Largest scratch the entry point serves: 64 MiB.  That holds the stream-K
// region of the dX GEMM on a 148-SM part (4 KB of flags and one 512 x 256 fp32
// partial per SM-pair cluster, 37.9 MB) next to the rest of the scratch of any
// single linear of the 8B shape at 2048 tokens and r = 16 (9.1 MiB for a
// 4096 x 4096 projection, 14.9 MiB for gate or up, 15.9 MiB for the
// 14336-wide down projection), so at those sizes the call takes the same plan
// as lsq_nf4_lora_bwd with a workspace of lsq_nf4_lora_bwd_workspace_size()
// bytes and gives bit-identical results.  Where the rest of the scratch
// leaves no room for the stream-K region the dX GEMM runs whole tiles (its
// fp32 sums then run in another order).  Every GPU that loads the library
// keeps this array for as long as the process lives.
constexpr size_t SCRATCH_BYTES = size_t(64) << 20;

static __device__ __align__(256) unsigned char g_bwd_scratch[SCRATCH_BYTES];

// Device address of g_bwd_scratch per device (the symbol's name in host code
// is only a host-side handle, not a device address).  Only a successful
// lookup is kept: after a failure the next call looks it up again.
static std::atomic<void*> g_addr[64];

static lsq_status scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "lsq_nf4_lora_bwd_noalloc: cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(LSQ_EUNSUPPORTED, "lsq_nf4_lora_bwd_noalloc: device %d out of range", dev);
  void* p = g_addr[dev].load(std::memory_order_acquire);
  if (!p) {
    e = cudaGetSymbolAddress(&p, g_bwd_scratch);
    if (e != cudaSuccess || !p) {
      (void)cudaGetLastError();
      return cuda_fail(e, "lsq_nf4_lora_bwd_noalloc: cudaGetSymbolAddress of the scratch array");
    }
    g_addr[dev].store(p, std::memory_order_release);
  }
  *out = p;
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
