// Shared host/device helpers of libhq: status codes, launch checks, workspace carving.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hq.h"

namespace hq {

// Spin limit of every device-side wait (mbarrier, flag): about 2 s at the B200's clock.
// On expiry the waiting kernel records HQ_ERR_TIMEOUT and returns instead of hanging.
constexpr long long kWaitLimitCycles = 4000000000LL;

#define HQ_CUDA_TRY(expr)                                  \
  do {                                                     \
    cudaError_t _e = (expr);                               \
    if (_e != cudaSuccess) return HQ_ERR_CUDA;             \
  } while (0)

// Process-wide count of kernels this library has launched (a statistic for profiling; read
// through hq_debug_launch_count()).
uint64_t& launch_counter();

#define HQ_LAUNCH_CHECK()                                  \
  do {                                                     \
    cudaError_t _e = cudaPeekAtLastError();                \
    if (_e != cudaSuccess) {                               \
      (void)cudaGetLastError();                            \
      return HQ_ERR_CUDA;                                  \
    }                                                      \
    __atomic_fetch_add(&::hq::launch_counter(), 1, __ATOMIC_RELAXED); \
  } while (0)

inline bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

inline int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }
inline size_t round_up(size_t a, size_t b) { return (a + b - 1) / b * b; }

// Records a device-side failure code in a caller-visible status word (first writer wins).
__device__ __forceinline__ void record_status(int* status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

}  // namespace hq
