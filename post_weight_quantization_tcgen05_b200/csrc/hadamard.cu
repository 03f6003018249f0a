// Hadamard rotation ahead of GPTQ (ork-driver wiki "Exp 2026-08-18 GPTQ Int4", experiment
// summary: GPTQ "composes with Hadamard = QuaRot: rotate then GPTQ").
//
// R = D blockdiag(M_B, ..., M_B) with D = diag(s) (s in {-1, +1}^K, drawn by the caller) and
// M_B = Hadamard_B / sqrt(B) the orthonormal Walsh-Hadamard matrix of order B (a power of two),
// Hadamard_B[i][j] = (-1)^popcount(i & j) (Sylvester).  R is orthogonal, so with W' = W R and
// X' = X R the layer's output is unchanged (W x = W' (R^T x)) and the calibration Hessian of the
// rotated activations is H' = R^T H R.  Both are computed by fast Walsh-Hadamard transforms
// (log2 B butterfly stages) on tiles in shared memory:
//   rows:    out[r][b B + j] = sum_i (s[b B + i] A[r][b B + i]) M_B[i][j]     (A R)
//   columns: A[b B + i][c] <- sum_k M_B[k][i] s[b B + k] A[b B + k][c]         (R^T A)
// each one read and one write of the matrix (HBM-bound).
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.cuh"

namespace hq {

constexpr int kHadMaxB = 1024;

// In-place fast Walsh-Hadamard transform of v[0 .. B) in shared memory (unnormalised), by the
// block's threads, each butterfly (v[i], v[i + h]) -> (v[i] + v[i + h], v[i] - v[i + h]).
__device__ __forceinline__ void fwht_smem(float* v, int B, int tid, int nthreads) {
  for (int h = 1; h < B; h <<= 1) {
    __syncthreads();
    for (int p = tid; p < B / 2; p += nthreads) {
      const int i = (p / h) * 2 * h + (p % h);
      const float a = v[i], b = v[i + h];
      v[i] = a + b;
      v[i + h] = a - b;
    }
  }
  __syncthreads();
}

// One CTA per (row, block): out[r][b B + j] = (1/sqrt B) sum_i s[b B + i] A[r][b B + i] H_B[i][j]
template <typename TA>
__global__ void __launch_bounds__(256) hadamard_rows_kernel(const TA* A, int64_t K, int B,
                                                            const float* __restrict__ s, float* out) {  // out may be A
  extern __shared__ float v[];
  const int64_t r = blockIdx.y;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * B;
  for (int i = threadIdx.x; i < B; i += blockDim.x) {
    float a;
    if constexpr (sizeof(TA) == 2) a = __bfloat162float(A[r * K + c0 + i]);
    else a = A[r * K + c0 + i];
    v[i] = a * s[c0 + i];
  }
  fwht_smem(v, B, threadIdx.x, blockDim.x);
  const float scale = rsqrtf(static_cast<float>(B));
  for (int i = threadIdx.x; i < B; i += blockDim.x) out[r * K + c0 + i] = v[i] * scale;
}

// One CTA per (block of B rows, 32 columns), in place: A[bB + i][c] <- (1/sqrt B) sum_k H_B[k][i]
// s[bB + k] A[bB + k][c]; the tile is kept column-major in shared memory (32 transforms of B).
__global__ void __launch_bounds__(256) hadamard_cols_kernel(float* __restrict__ A, int64_t K, int64_t ncols, int B,
                                                            const float* __restrict__ s) {
  extern __shared__ float t[];  // [32][B + 1]
  const int LD = B + 1;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * B;
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * 32;
  const int cw = static_cast<int>(ncols - c0 < 32 ? ncols - c0 : 32);
  for (int e = threadIdx.x; e < B * 32; e += blockDim.x) {
    const int i = e / 32, c = e % 32;  // coalesced along the row
    t[c * LD + i] = c < cw ? A[(r0 + i) * K + c0 + c] * s[r0 + i] : 0.f;
  }
  // 32 independent transforms of length B: butterflies over the flattened (column, pair) space
  for (int h = 1; h < B; h <<= 1) {
    __syncthreads();
    for (int p = threadIdx.x; p < 32 * (B / 2); p += blockDim.x) {
      const int c = p / (B / 2), q = p % (B / 2);
      const int i = (q / h) * 2 * h + (q % h);
      float* col = t + c * LD;
      const float a = col[i], b = col[i + h];
      col[i] = a + b;
      col[i + h] = a - b;
    }
  }
  __syncthreads();
  const float scale = rsqrtf(static_cast<float>(B));
  for (int e = threadIdx.x; e < B * 32; e += blockDim.x) {
    const int i = e / 32, c = e % 32;
    if (c < cw) A[(r0 + i) * K + c0 + c] = t[c * LD + i] * scale;
  }
}

// out = the symmetric matrix whose lower triangle (diagonal included) is H's, by 32 x 32 tiles:
// tile (bi, bj), bi >= bj, is read once and written at (bi, bj) and transposed at (bj, bi).
__global__ void __launch_bounds__(256) mirror_lower_kernel(const float* __restrict__ H, int64_t K,
                                                           float* __restrict__ out) {
  __shared__ float t[32][33];
  int64_t tt = blockIdx.x;
  int64_t bi = static_cast<int64_t>((sqrt(8.0 * static_cast<double>(tt) + 1.0) - 1.0) * 0.5);
  while (bi * (bi + 1) / 2 > tt) --bi;
  while ((bi + 1) * (bi + 2) / 2 <= tt) ++bi;
  const int64_t bj = tt - bi * (bi + 1) / 2;
  const int tx = threadIdx.x % 32, ty = threadIdx.x / 32;
  for (int r = ty; r < 32; r += 8) {
    const int64_t i = bi * 32 + r, j = bj * 32 + tx;
    float v = 0.f;
    if (i < K && j < K) {
      // in a diagonal tile the upper part comes from the transposed lower part
      v = (j <= i) ? H[i * K + j] : H[j * K + i];
      out[i * K + j] = v;
    }
    t[r][tx] = v;
  }
  __syncthreads();
  if (bi == bj) return;
  for (int r = ty; r < 32; r += 8) {
    const int64_t i = bj * 32 + r, j = bi * 32 + tx;  // out[bj tile][bi tile] = t^T
    if (i < K && j < K) out[i * K + j] = t[tx][r];
  }
}

hq_status launch_mirror_lower(const float* H, int64_t K, float* out, cudaStream_t st) {
  const int64_t nb = ceil_div(K, int64_t(32));
  const int64_t tiles = nb * (nb + 1) / 2;
  if (tiles > 0x7FFFFFFF) return HQ_ERR_UNSUPPORTED;
  mirror_lower_kernel<<<static_cast<unsigned>(tiles), 256, 0, st>>>(H, K, out);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

bool hadamard_shape_ok(int64_t K, int64_t B) {
  return B >= 2 && B <= kHadMaxB && (B & (B - 1)) == 0 && K >= B && K % B == 0 && K <= (int64_t(1) << 30);
}

hq_status launch_hadamard_rows(const void* A, int a_dtype, int64_t rows, int64_t K, int B, const float* s,
                               float* out, cudaStream_t st) {
  if (rows == 0) return HQ_OK;
  if (rows > 65535) {  // grid.y limit: in slices
    for (int64_t r0 = 0; r0 < rows; r0 += 65535) {
      const int64_t n = rows - r0 < 65535 ? rows - r0 : 65535;
      const size_t esz = a_dtype == HQ_BF16 ? 2 : 4;
      const hq_status e = launch_hadamard_rows(static_cast<const uint8_t*>(A) + r0 * K * esz, a_dtype, n, K, B, s,
                                               out + r0 * K, st);
      if (e != HQ_OK) return e;
    }
    return HQ_OK;
  }
  const dim3 grid(static_cast<unsigned>(K / B), static_cast<unsigned>(rows));
  const size_t smem = static_cast<size_t>(B) * sizeof(float);
  if (a_dtype == HQ_BF16)
    hadamard_rows_kernel<__nv_bfloat16><<<grid, 256, smem, st>>>(static_cast<const __nv_bfloat16*>(A), K, B, s, out);
  else
    hadamard_rows_kernel<float><<<grid, 256, smem, st>>>(static_cast<const float*>(A), K, B, s, out);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

hq_status launch_hadamard_cols(float* A, int64_t K, int B, const float* s, cudaStream_t st) {
  const dim3 grid(static_cast<unsigned>(ceil_div(K, int64_t(32))), static_cast<unsigned>(K / B));
  const size_t smem = static_cast<size_t>(32) * (B + 1) * sizeof(float);
  if (smem > 48 * 1024)
    HQ_CUDA_TRY(cudaFuncSetAttribute(hadamard_cols_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem)));
  hadamard_cols_kernel<<<grid, 256, smem, st>>>(A, K, K, B, s);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

}  // namespace hq
