// hq_rtn_quantize_noalloc: round-to-nearest int4 quantisation for callers that cannot give the
// library a workspace.
//
// Some callers have no way to obtain device memory for scratch space at the moment they
// quantise: a host application that has already reserved all device memory for its own pool
// (so a cudaMalloc would fail or fragment it), a latency-critical service that forbids any
// allocation after start-up, or a plugin that runs under another framework's allocator and has
// no handle to it.  For them this entry point keeps its scratch -- the qerr partial sums and
// the small status header -- in one fixed array that lives in the library's own device memory
// for as long as the library is loaded, on every GPU that loads it.  The caller still provides
// W, codes and scales.  The kernels are the same ones hq_rtn_quantize launches, so the results
// are identical.
#include <cuda_runtime.h>

#include "../../include/hq.h"
#include "common.cuh"
#include "kernels.cuh"

namespace hq {
namespace {

// Room for the header (256 bytes) and HQ_RTN_NOALLOC_MAX_GROUPS partial sums of two doubles.
constexpr size_t kNoallocHeader = 256;
constexpr size_t kNoallocBytes = kNoallocHeader + static_cast<size_t>(HQ_RTN_NOALLOC_MAX_GROUPS) * 2 * sizeof(double);

static __device__ __align__(256) unsigned char g_rtn_scratch[kNoallocBytes];

// The array's device address on each device.  In host code `g_rtn_scratch` names a host-side
// stand-in, not device memory, so the address is looked up once per device (with that device
// current) and passed to the kernels.
constexpr int kMaxDevices = 64;
static void* g_scratch_ptr[kMaxDevices] = {};

hq_status scratch_for_current_device(uint8_t** out) {
  int dev = -1;
  HQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return HQ_ERR_UNSUPPORTED;
  void* p = __atomic_load_n(&g_scratch_ptr[dev], __ATOMIC_ACQUIRE);
  if (p == nullptr) {
    if (cudaGetSymbolAddress(&p, g_rtn_scratch) != cudaSuccess || p == nullptr) {
      (void)cudaGetLastError();
      return HQ_ERR_CUDA;
    }
    __atomic_store_n(&g_scratch_ptr[dev], p, __ATOMIC_RELEASE);
  }
  *out = static_cast<uint8_t*>(p);
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
