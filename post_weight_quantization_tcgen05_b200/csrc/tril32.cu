// The lower triangle of an fp32 K x K Hessian packed row by row without gaps (element (i, j),
// j <= i, at i (i + 1) / 2 + j): the exchange format of a Hessian whose token chunks were
// accumulated on several GPUs ("hipfire-calib-data" dataset card, "Hessian storage": the
// statistic is a sum over chunks, and only the lower triangle of the symmetric sum is needed).
// Summing the packed partial Hessians moves K (K + 1) / 2 values instead of K^2.
//
// One warp per row, rows spread over the grid; each row is one contiguous run in both layouts,
// so every warp access is a coalesced 128-byte segment (the packed start is only 4-byte
// aligned, so the accesses stay scalar).  HBM-bound: 4 K (K + 1) / 2 bytes read and written.
#include "common.cuh"
#include "kernels.cuh"

namespace hq {
namespace {

template <bool kPack>
__global__ void __launch_bounds__(256) tril32_kernel(const float* __restrict__ src, float* __restrict__ dst,
                                                     int64_t K) {
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x / 32);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * (blockDim.x / 32) + (threadIdx.x >> 5); i < K; i += warps) {
    const int64_t p = i * (i + 1) / 2;
    const int64_t r = i * K;
    for (int64_t j = lane; j <= i && HQ_IN_BOUNDS(p + j < K * (K + 1) / 2); j += 32) {
      if (kPack)
        dst[p + j] = src[r + j];
      else
        dst[r + j] = src[p + j];
    }
  }
}

}  // namespace

hq_status launch_tril32(const float* src, float* dst, int64_t K, bool pack, cudaStream_t s) {
  const int64_t grid = ceil_div(K, 8) < 148 * 8 ? ceil_div(K, 8) : 148 * 8;
  if (pack)
    tril32_kernel<true><<<static_cast<unsigned>(grid), 256, 0, s>>>(src, dst, K);
  else
    tril32_kernel<false><<<static_cast<unsigned>(grid), 256, 0, s>>>(src, dst, K);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

}  // namespace hq

using namespace hq;

extern "C" size_t hq_tril32_count(int64_t K) {
  if (K < 1) return 0;
  return static_cast<size_t>(K) * (K + 1) / 2;
}

extern "C" hq_status hq_hessian_pack_lower(const float* H, int64_t K, float* packed, hq_stream_t stream) {
  if (H == nullptr || packed == nullptr || K < 1) return HQ_ERR_INVALID;
  if (K > (int64_t(1) << 20)) return HQ_ERR_UNSUPPORTED;
  return launch_tril32(H, packed, K, true, static_cast<cudaStream_t>(stream));
}

extern "C" hq_status hq_hessian_unpack_lower(const float* packed, int64_t K, float* H, hq_stream_t stream) {
  if (H == nullptr || packed == nullptr || K < 1) return HQ_ERR_INVALID;
  if (K > (int64_t(1) << 20)) return HQ_ERR_UNSUPPORTED;
  return launch_tril32(packed, H, K, false, static_cast<cudaStream_t>(stream));
}
