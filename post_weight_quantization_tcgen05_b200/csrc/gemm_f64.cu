// fp64 GEMM on the CUDA cores for the factorisation:
//
//   C[m, n] = beta * C[m, n] + alpha * sum_k A[m * lda + k] * B[n * ldb + k]    m < M, n < N
//
// (both operands K-major, optionally only the lower part row0 + m >= col0 + n written).
// The damped Hessians of strongly correlated layers have condition numbers around 1e6, and the
// Schur-complement updates of the Cholesky recursion cancel a large common component, so the
// factorisation runs in fp64 end to end (fp32 loses about kappa * 6e-8 there, which measurably
// changes GPTQ codes).  128 x 128 tiles per CTA, 256 threads with 8 x 8 outputs each, k-chunks
// of 16 staged through shared memory (transposed to k-major), with the next chunk's global loads
// in flight while the current one is multiplied.
#include "common.cuh"
#include "kernels.cuh"

namespace hq {

constexpr int kDT = 128;  // tile
constexpr int kDK = 16;   // k-chunk
constexpr int kDP = kDT + 2;  // padded smem row (doubles)

__global__ void __launch_bounds__(256) f64_gemm_kernel(F64Gemm g) {
  if (g.skip != nullptr && *g.skip != 0) return;
  const int tiles_n = (g.N + kDT - 1) / kDT;
  const int m0 = (blockIdx.x / tiles_n) * kDT, n0 = (blockIdx.x % tiles_n) * kDT;
  if (g.lower && g.row0 + m0 + kDT - 1 < g.col0 + n0) return;
  __shared__ __align__(16) double As[kDK][kDP];
  __shared__ __align__(16) double Bs[kDK][kDP];
  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;  // output rows ty*8.., columns tx*8..
  // loader: each thread brings 8 doubles of A and 8 of B per chunk: rows lr, lr+64, k quad lk
  const int lr = tid >> 2, lk = (tid & 3) * 4;
  double ra[2][4], rb[2][4];
  auto load = [&](int k0) {
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int r = lr + 64 * h;
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int k = k0 + lk + u;
        ra[h][u] = (m0 + r < g.M && k < g.Kred) ? g.A[static_cast<int64_t>(m0 + r) * g.lda + k] : 0.0;
        rb[h][u] = (n0 + r < g.N && k < g.Kred) ? g.B[static_cast<int64_t>(n0 + r) * g.ldb + k] : 0.0;
      }
    }
  };
  double acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.0;
  load(0);
  for (int k0 = 0; k0 < g.Kred; k0 += kDK) {
    __syncthreads();
#pragma unroll
    for (int h = 0; h < 2; ++h)
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        As[lk + u][lr + 64 * h] = ra[h][u];
        Bs[lk + u][lr + 64 * h] = rb[h][u];
      }
    __syncthreads();
    if (k0 + kDK < g.Kred) load(k0 + kDK);
#pragma unroll
    for (int k = 0; k < kDK; ++k) {
      double a[8], b[8];
#pragma unroll
      for (int i = 0; i < 8; i += 2) {
        const double2 av = *reinterpret_cast<const double2*>(&As[k][ty * 8 + i]);
        const double2 bv = *reinterpret_cast<const double2*>(&Bs[k][tx * 8 + i]);
        a[i] = av.x;
        a[i + 1] = av.y;
        b[i] = bv.x;
        b[i + 1] = bv.y;
      }
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int j = 0; j < 8; ++j) acc[i][j] = fma(a[i], b[j], acc[i][j]);
    }
  }
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int m = m0 + ty * 8 + i;
    if (m >= g.M) continue;
    double* crow = g.C + static_cast<int64_t>(m) * g.ldc;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int n = n0 + tx * 8 + j;
      if (n >= g.N || (g.lower && g.row0 + m < g.col0 + n)) continue;
      crow[n] = (g.beta != 0.0 ? g.beta * crow[n] : 0.0) + g.alpha * acc[i][j];
    }
  }
}

hq_status f64_gemm(const F64Gemm& g, cudaStream_t s) {
  if (g.M <= 0 || g.N <= 0) return HQ_OK;
  const int64_t tiles = ceil_div(g.M, kDT) * ceil_div(g.N, kDT);
  if (tiles > 0x7FFFFFFF) return HQ_ERR_UNSUPPORTED;
  f64_gemm_kernel<<<static_cast<unsigned>(tiles), 256, 0, s>>>(g);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

}  // namespace hq
