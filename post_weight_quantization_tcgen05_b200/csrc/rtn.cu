// Round-to-nearest int4, the RTN baseline: symmetric absmax/7 rounding (ork-driver wiki
// "Exp 2026-08-18 GPTQ Int4", experiment summary), i.e. the GPTQ quantiser without error feedback.
// One warp per (row, group): absmax by shuffles, scale s = fp32(absmax / 7), codes
// c = clamp(rint(w / s), -8, 7) packed two per byte, fp64 qerr partials per warp.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.cuh"

namespace hq {

__device__ __forceinline__ float rtn_load(const void* W, int dt, int64_t idx) {
  return dt == HQ_BF16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(W)[idx]) : static_cast<const float*>(W)[idx];
}

__global__ void __launch_bounds__(128) rtn_kernel(const void* __restrict__ W, int dt, int64_t N, int64_t K, int G,
                                                  const float* __restrict__ imp, uint8_t* __restrict__ codes,
                                                  float* __restrict__ scales, double* __restrict__ partials) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t ng = K / G;
  const int64_t gid = static_cast<int64_t>(blockIdx.x) * 4 + warp;
  if (gid >= N * ng) return;
  const int64_t row = gid / ng, g = gid % ng;
  const int64_t base = row * K + g * G;
  float am = 0.f;
  for (int i = lane; i < G; i += 32) am = fmaxf(am, fabsf(rtn_load(W, dt, base + i)));
  for (int off = 16; off > 0; off >>= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, off));
  const float s = __fdiv_rn(am, 7.f);
  double num = 0.0, den = 0.0;
  for (int p = lane; p < G / 2; p += 32) {
    const float w0 = rtn_load(W, dt, base + 2 * p), w1 = rtn_load(W, dt, base + 2 * p + 1);
    float c0 = 0.f, c1 = 0.f;
    if (s > 0.f) {
      c0 = fminf(fmaxf(rintf(__fdiv_rn(w0, s)), -8.f), 7.f);
      c1 = fminf(fmaxf(rintf(__fdiv_rn(w1, s)), -8.f), 7.f);
    }
    if (HQ_IN_BOUNDS((g * G) / 2 + p < K / 2))
      codes[row * (K / 2) + (g * G) / 2 + p] =
        static_cast<uint8_t>((static_cast<int>(c0) & 0xF) | ((static_cast<int>(c1) & 0xF) << 4));
    const double i0 = imp != nullptr ? static_cast<double>(imp[g * G + 2 * p]) : 1.0;
    const double i1 = imp != nullptr ? static_cast<double>(imp[g * G + 2 * p + 1]) : 1.0;
    const double d0 = static_cast<double>(w0) - static_cast<double>(c0) * s;
    const double d1 = static_cast<double>(w1) - static_cast<double>(c1) * s;
    num += i0 * d0 * d0 + i1 * d1 * d1;
    den += i0 * static_cast<double>(w0) * w0 + i1 * static_cast<double>(w1) * w1;
  }
  for (int off = 16; off > 0; off >>= 1) {
    num += __shfl_down_sync(0xffffffffu, num, off);
    den += __shfl_down_sync(0xffffffffu, den, off);
  }
  if (lane == 0) {
    scales[row * ng + g] = s;
    partials[2 * gid] = num;
    partials[2 * gid + 1] = den;
  }
}

size_t rtn_workspace(int64_t N, int64_t K, int64_t group) {
  return round_up(sizeof(WsHeader), 256) + static_cast<size_t>(N) * (K / group) * 2 * sizeof(double);
}

hq_status launch_rtn(const void* W, int w_dtype, int64_t N, int64_t K, int64_t group, const float* imp,
                     uint8_t* codes, float* scales, double* qerr_dev, uint8_t* ws, cudaStream_t s) {
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws);
  double* partials = reinterpret_cast<double*>(ws + round_up(sizeof(WsHeader), 256));
  HQ_CUDA_TRY(cudaMemsetAsync(hdr, 0, sizeof(WsHeader), s));
  const int64_t warps = N * (K / group);
  const int64_t ctas = ceil_div(warps, 4);
  if (ctas > 0x7FFFFFFF) return HQ_ERR_UNSUPPORTED;
  rtn_kernel<<<static_cast<unsigned>(ctas), 128, 0, s>>>(W, w_dtype, N, K, static_cast<int>(group), imp, codes,
                                                         scales, partials);
  HQ_LAUNCH_CHECK();
  return launch_qerr_finalize(partials, warps, hdr, qerr_dev, s);
}

}  // namespace hq
