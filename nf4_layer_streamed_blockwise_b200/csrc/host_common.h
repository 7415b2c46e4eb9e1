// Host-side helpers of the lsq library: error reporting, device checks, the
// NF4 codebook and its decision thresholds, TMA tensor-map encoding.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdarg.h>
#include <stdint.h>

#include "../../include/lsq.h"

namespace lsq {

// Sets the thread's last-error message and returns s.
lsq_status fail(lsq_status s, const char* fmt, ...);
lsq_status cuda_fail(cudaError_t e, const char* what);

// Checks the current device is sm_100 (B200) once per device.
lsq_status check_device();

// Library codebook (16 ascending fp32 levels) and the 15 fp32 decision
// thresholds: code(x) = number of i with x >= thr[i].
const float* codebook();
const float* thresholds();

// 2-D tiled tensor map: dims {inner, outer} in elements, row pitch in bytes,
// box {box_inner, box_outer}; out-of-bounds elements read as zero.
lsq_status encode_tmap_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner,
                          uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                          CUtensorMapSwizzle swz);

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int num_sms();

}  // namespace lsq

#define LSQ_CUDA_TRY(call)                                        \
  do {                                                            \
    cudaError_t e_ = (call);                                      \
    if (e_ != cudaSuccess) return ::lsq::cuda_fail(e_, #call);    \
  } while (0)

#define LSQ_LAUNCH_CHECK(what)                                          \
  do {                                                                  \
    cudaError_t e_ = cudaGetLastError();                                \
    if (e_ != cudaSuccess) return ::lsq::cuda_fail(e_, what);           \
  } while (0)
