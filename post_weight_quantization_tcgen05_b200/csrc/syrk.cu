// Calibration Hessian accumulation H += X^T X over the lower triangle of H.
//
// bf16 X with K a multiple of 8 and a 16-byte aligned base goes through the tcgen05 GEMM
// (gemm_tc.cuh, kSyrkBF16): TMA brings 64-token x 64-channel bf16 boxes, the tensor core
// multiplies them as MN-major operands and accumulates 1024-token segments in TMEM in fp32,
// and the segments are summed in fp32 registers.  Every other input
// (fp32 X, odd K, unaligned X) takes the fp32 CUDA-core kernel below, which computes the same
// sum with exact products and fp32 accumulation.
#include <cuda_bf16.h>

#include "common.cuh"
#include "gemm_tc.cuh"
#include "kernels.cuh"
#include "tmap.cuh"

namespace hq {

// ---------------------------------------------------------------- CUDA-core path

constexpr int kSimtTile = 64;
constexpr int kSimtBK = 16;

template <typename TX>
__device__ __forceinline__ float load_x(const TX* p);
template <>
__device__ __forceinline__ float load_x<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float load_x<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// One 64 x 64 tile (bi >= bj) per CTA, 256 threads with 4 x 4 outputs each.
template <typename TX>
__global__ void __launch_bounds__(256) syrk_simt_kernel(float* __restrict__ H, const TX* __restrict__ X, int64_t T,
                                                        int64_t K) {
  int t = blockIdx.x;
  int bi = 0;
  while (t > bi) {
    t -= bi + 1;
    ++bi;
  }
  const int bj = t;
  const int64_t i0 = static_cast<int64_t>(bi) * kSimtTile;
  const int64_t j0 = static_cast<int64_t>(bj) * kSimtTile;
  __shared__ float xs_i[kSimtBK][kSimtTile];
  __shared__ float xs_j[kSimtBK][kSimtTile];
  const int tx = threadIdx.x % 16;
  const int ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int64_t t0 = 0; t0 < T; t0 += kSimtBK) {
    for (int e = threadIdx.x; e < kSimtBK * kSimtTile; e += 256) {
      const int r = e / kSimtTile, c = e % kSimtTile;
      const int64_t tt = t0 + r;
      xs_i[r][c] = (tt < T && i0 + c < K) ? load_x(X + tt * K + i0 + c) : 0.f;
      xs_j[r][c] = (tt < T && j0 + c < K) ? load_x(X + tt * K + j0 + c) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kSimtBK; ++r) {
      float a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        a[u] = xs_i[r][ty + 16 * u];
        b[u] = xs_j[r][tx + 16 * u];
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(a[u], b[v], acc[u][v]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int64_t i = i0 + ty + 16 * u;
    if (i >= K) continue;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int64_t j = j0 + tx + 16 * v;
      if (j <= i) H[i * K + j] += acc[u][v];
    }
  }
}

hq_status launch_syrk_simt(float* H, const void* X, int x_dtype, int64_t T, int64_t K, cudaStream_t s) {
  const int64_t nb = ceil_div(K, kSimtTile);
  const int64_t tiles = nb * (nb + 1) / 2;
  if (tiles > 0x7FFFFFFF) return HQ_ERR_UNSUPPORTED;
  if (x_dtype == HQ_F32)
    syrk_simt_kernel<float><<<static_cast<unsigned>(tiles), 256, 0, s>>>(H, static_cast<const float*>(X), T, K);
  else
    syrk_simt_kernel<__nv_bfloat16>
        <<<static_cast<unsigned>(tiles), 256, 0, s>>>(H, static_cast<const __nv_bfloat16*>(X), T, K);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

// ---------------------------------------------------------------- tensor-core path

bool syrk_tc_eligible(const void* X, int x_dtype, int64_t T, int64_t K) {
  return x_dtype == HQ_BF16 && (K % 8) == 0 && aligned(X, 16) && K <= (1 << 24) && T <= 0x7FFFFFFF;
}

hq_status launch_syrk_tc(float* H, const void* X, int64_t T, int64_t K, int* dev_status, cudaStream_t s) {
  CUtensorMap map;
  if (!make_tmap_2d(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, static_cast<uint64_t>(K), static_cast<uint64_t>(T),
                    static_cast<uint64_t>(K) * 2, 64, 64))
    return HQ_ERR_CUDA;
  HQ_CUDA_TRY(cudaFuncSetAttribute(umma_gemm_kernel<GemmMode::kSyrkBF16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   kGemmSmemBytes));
  const int tiles_m = static_cast<int>(ceil_div(K, kGemmBM));
  const int tiles_n = static_cast<int>(ceil_div(K, kGemmBN));
  int64_t tiles = 0;
  for (int bi = 0; bi < tiles_m; ++bi) tiles += syrk_tiles_in_row(bi, tiles_n);
  GemmArgs a{};
  a.C = H;
  a.ldc = K;
  a.M = static_cast<int>(K);
  a.Ncols = static_cast<int>(K);
  a.Kred = static_cast<int>(T);
  a.status = dev_status;
  const int tm = timer_start(kTimeSyrk, s);
  umma_gemm_kernel<GemmMode::kSyrkBF16><<<static_cast<unsigned>(tiles), gemm_threads(GemmMode::kSyrkBF16), kGemmSmemBytes, s>>>(map, map, a);
  HQ_LAUNCH_CHECK();
  timer_stop(tm, static_cast<double>(T) * K * (K + 1), s);  // 2 flops x T x K (K + 1) / 2 lower entries
  return HQ_OK;
}

}  // namespace hq
