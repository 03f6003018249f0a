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

// Programmatic dependent launch along the factorisation's chain of short kernels (the small fp64
// products, their split-K reduce, the leaves): a kernel launched by launch_chained may be
// scheduled while its predecessor on the stream still runs.  It calls pdl_wait before touching
// memory (it returns once the predecessor has completed and its writes are visible), and
// pdl_launch_dependents near its end, so that its own successor is scheduled in turn without
// holding SM slots for long (slots the second stream's work would otherwise use).  In a kernel
// launched the ordinary way both are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
inline cudaError_t launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                  Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

// A launch_chained call with the error handling and the launch count of HQ_LAUNCH_CHECK.
#define HQ_LAUNCH_CHAINED(expr)                            \
  do {                                                     \
    cudaError_t _e = (expr);                               \
    if (_e != cudaSuccess) {                               \
      (void)cudaGetLastError();                            \
      return HQ_ERR_CUDA;                                  \
    }                                                      \
    __atomic_fetch_add(&::hq::launch_counter(), 1, __ATOMIC_RELAXED); \
  } while (0)

// Records a device-side failure code in a caller-visible status word (first writer wins).
__device__ __forceinline__ void record_status(int* status, int code) {
  if (status != nullptr) atomicCAS(status, 0, code);
}

// Index checks of the bounds-checking build (HQ_DEBUG_BOUNDS, built as libhq_bounds.so; the
// stand-in for a memory checker).  HQ_IN_BOUNDS(cond) guards one computed global access: in
// that build a false condition records where it failed (first failure wins: a tag of the source
// file's name in the high 16 bits, the line in the low 16) in a device word that
// hq_debug_bounds_status reads, and the guarded access is skipped.  In the regular build the
// condition is not evaluated and the macro is true.
constexpr int bounds_file_tag(const char* path) {
  const char* base = path;
  for (const char* c = path; *c != 0; ++c)
    if (*c == '/') base = c + 1;
  int h = 0;
  for (const char* c = base; *c != 0; ++c) h = (h * 31 + static_cast<unsigned char>(*c)) & 0x7FFF;
  return h | 1;
}
template <int V>
struct BoundsTag {
  static constexpr int value = V;
};
#ifdef HQ_DEBUG_BOUNDS
extern __device__ int g_hq_bounds_violation;
__device__ __forceinline__ bool bounds_check(bool ok, int where) {
  if (!ok) atomicCAS(&g_hq_bounds_violation, 0, where);
  return ok;
}
#define HQ_IN_BOUNDS(cond) \
  (::hq::bounds_check((cond), (::hq::BoundsTag<::hq::bounds_file_tag(__FILE__)>::value << 16) | __LINE__))
#else
#define HQ_IN_BOUNDS(cond) true
#endif

}  // namespace hq
