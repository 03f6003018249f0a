// hq_rtn_quantize_noalloc: round-to-nearest int4 quantisation for callers that cannot give the
// library a workspace.
//
// Some callers have no way to obtain device memory for scratch space at the moment they
// quantise: a host application that has already reserved all device memory for its own pool
// (so a cudaMalloc would fail or fragment it), a latency-critical service that forbids any
// allocation after start-up, or a plugin that runs under another framework's allocator and has
// no handle to it.  For them this entry point keeps its scratch -- the qerr partial sums and
// the small status header -- in one fixed array that lives in the library's own device memory
// for as long as the library is loaded, on every GPU that loads it.  The array is committed on a
// device when the library's module that holds it is loaded there; under CUDA's lazy module
// loading (the default) that is the first call on that device.  The caller still provides
// W, codes and scales.  The kernels are the same ones hq_rtn_quantize launches, so the results
// are identical.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/hq.h"
#include "common.cuh"
#include "kernels.cuh"

namespace hq {
namespace {

// Room for the header (256 bytes) and HQ_RTN_NOALLOC_MAX_GROUPS partial sums of two doubles.
constexpr size_t kNoallocHeader = 256;
constexpr size_t kNoallocBytes = kNoallocHeader + static_cast<size_t>(HQ_RTN_NOALLOC_MAX_GROUPS) * 2 * sizeof(double);

static __device__ __align__(256) unsigned char g_rtn_scratch[kNoallocBytes];

// The array's device address, per device and context.  In host code `g_rtn_scratch` names a
// host-side stand-in, not device memory, so the address is looked up with the device current
// (cudaGetSymbolAddress) and passed to the kernels.  The lookup is cached per device and keyed
// by the current context's id: after a device reset the module is loaded again, possibly at
// another address, and the new context's id forces a fresh lookup.
constexpr int kMaxDevices = 64;
struct ScratchSlot {
  unsigned long long ctx_id = 0;
  void* ptr = nullptr;
};
static ScratchSlot g_slot[kMaxDevices];
static std::mutex g_slot_mu;

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename Fn>
Fn driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<Fn>(p);
}

// Id of the context current on this thread (0 if none or unknown).
unsigned long long current_context_id() {
  static const CtxGetCurrentFn get_current = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
  static const CtxGetIdFn get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr || get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

hq_status scratch_for_current_device(uint8_t** out) {
  int dev = -1;
  HQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return HQ_ERR_UNSUPPORTED;
  unsigned long long id = current_context_id();
  if (id == 0) {  // the runtime has not made this device's context current on this thread yet
    HQ_CUDA_TRY(cudaSetDevice(dev));
    id = current_context_id();
  }
  std::lock_guard<std::mutex> lock(g_slot_mu);
  ScratchSlot& slot = g_slot[dev];
  if (slot.ptr == nullptr || id == 0 || slot.ctx_id != id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_rtn_scratch) != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();
      return HQ_ERR_CUDA;
    }
    slot.ptr = p;
    slot.ctx_id = id;
  }
  *out = static_cast<uint8_t*>(slot.ptr);
  return HQ_OK;
}

}  // namespace
}  // namespace hq

using namespace hq;

extern "C" hq_status hq_rtn_quantize_noalloc(const void* W, int w_dtype, int64_t N, int64_t K, int64_t group,
                                             const float* imp, uint8_t* codes, float* scales, double* qerr_out,
                                             double* qerr_dev, hq_stream_t stream) {
  if (W == nullptr || codes == nullptr || scales == nullptr || (w_dtype != HQ_F32 && w_dtype != HQ_BF16))
    return HQ_ERR_INVALID;
  if (N < 1 || K < 2 || group < 2 || K % group != 0) return HQ_ERR_INVALID;
  if (group % 2 != 0) return HQ_ERR_UNSUPPORTED;
  if (N > HQ_RTN_NOALLOC_MAX_GROUPS / (K / group)) return HQ_ERR_UNSUPPORTED;  // scratch too small
  static_assert(sizeof(WsHeader) <= kNoallocHeader, "header does not fit");
  uint8_t* ws = nullptr;
  hq_status st = scratch_for_current_device(&ws);
  if (st != HQ_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  st = launch_rtn(W, w_dtype, N, K, group, imp, codes, scales, qerr_dev, ws, s);
  if (st != HQ_OK || qerr_out == nullptr) return st;
  WsHeader h{};
  HQ_CUDA_TRY(cudaMemcpyAsync(&h, ws, sizeof(WsHeader), cudaMemcpyDeviceToHost, s));
  HQ_CUDA_TRY(cudaStreamSynchronize(s));
  *qerr_out = h.qerr;
  return HQ_OK;
}
