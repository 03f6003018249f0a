// Projection of a symmetric Hessian onto the positive semidefinite cone ("hipfire-calib-data"
// dataset card, "REQUIRED: project to PSD before Cholesky" and "The fix": eigendecompose, clip
// the negative eigenvalues to zero, rebuild, symmetrise).
//
// The same matrix without an eigendecomposition: with H = V diag(l) V^T,
//   P = V diag(max(l, 0)) V^T = (H + H sign(H)) / 2,   sign(H) = V diag(sign(l)) V^T,
// and sign(H) is the limit of the Newton-Schulz iteration X <- X (3I - X^2) / 2 started at
// X0 = H / ||H||_F (every eigenvalue of X0 in [-1, 1]; each converges to its sign, a small one
// growing by 3/2 per step, then quadratically).  Each step forms X^2 = X X^T and X^3 = X (X^2)^T
// with the C -= A B^T product and then replaces X by its symmetric part: for an X that rounding
// has made slightly asymmetric, X X X^T is not the polar iteration's X X^T X, and without the
// symmetrisation that asymmetry grows until the iteration diverges (measured, fp64 included).
// An eigenvalue too small to be resolved in the steps given (below about 1.5^-steps ||H||_F)
// moves P by at most its size.  Finally P is symmetrised, (P + P^T) / 2, as in the pages' recipe.
//
// Arithmetic: fp32 iterates; the products X X and X (b X^2) on the tcgen05 tensor cores with
// operands split into a tf32 part and the fp32 remainder (3xTF32, upd_gemm), the contraction in
// chunks of kPsdChunk so that no accumulator chains more than 192 MMAs; the norm in fp64.
#include "common.cuh"
#include "kernels.cuh"

namespace hq {

constexpr int kPsdChunk = 1024;   // contraction columns per product launch
constexpr int kPsdRedBlocks = 592;

// workspace: [0, 8) 1 / ||H||_F, [128, 132) the status word, then the norm partials and six
// K x K fp32 matrices
size_t psd_workspace(int64_t K) {
  return 256 + round_up(static_cast<size_t>(kPsdRedBlocks) * sizeof(double), 256) +
         6 * round_up(static_cast<size_t>(K) * K * sizeof(float), 256);
}

__global__ void __launch_bounds__(256) sumsq_kernel(const float* __restrict__ H, int64_t n, double* __restrict__ part) {
  double s = 0.0;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const double v = H[i];
    s = fma(v, v, s);
  }
  __shared__ double red[256];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (static_cast<int>(threadIdx.x) < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) part[blockIdx.x] = red[0];
}

// inv[0] = 1 / ||H||_F (0 for a zero matrix), summed in a fixed order
__global__ void __launch_bounds__(256) inv_norm_kernel(const double* __restrict__ part, int nb, double* __restrict__ inv) {
  __shared__ double red[256];
  double s = 0.0;
  for (int i = threadIdx.x; i < nb; i += blockDim.x) s += part[i];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (static_cast<int>(threadIdx.x) < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) inv[0] = red[0] > 0.0 ? 1.0 / sqrt(red[0]) : 0.0;
}

__device__ __forceinline__ float tf32_part(float x) { return __uint_as_float(__float_as_uint(x) & 0xFFFFE000u); }

// X = H / ||H||_F
__global__ void psd_init_kernel(const float* __restrict__ H, int64_t n, const double* __restrict__ inv,
                                float* __restrict__ X) {
  const float s = static_cast<float>(*inv);
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    X[i] = H[i] * s;
}

// hi + lo = sc * src (hi a tf32 value, lo the exact fp32 remainder; sc a power of two or 1, so the
// scaling is exact); optionally C = cc * src and Z = 0.  hi may be src itself.
__global__ void psd_split_kernel(const float* src, int64_t n, float sc, float* hi, float* __restrict__ lo,
                                 float* __restrict__ C, float cc, float* __restrict__ Z) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const float x = src[i];
    if (C != nullptr) C[i] = cc * x;
    if (Z != nullptr) Z[i] = 0.f;
    const float v = sc * x;
    const float h = tf32_part(v);
    hi[i] = h;
    lo[i] = v - h;
  }
}

// H = (P + P^T) / 2, 32 x 32 tiles through shared memory (P and H distinct)
__global__ void __launch_bounds__(256) psd_symmetrize_kernel(const float* __restrict__ P, int64_t K,
                                                             float* __restrict__ H) {
  __shared__ float t[32][33];
  const int64_t nb = (K + 31) / 32;
  const int64_t bi = blockIdx.x / nb, bj = blockIdx.x % nb;
  const int tx = threadIdx.x % 32, ty = threadIdx.x / 32;  // 8 rows at a time
  for (int r = ty; r < 32; r += 8) {
    const int64_t i = bj * 32 + r, j = bi * 32 + tx;  // tile (bj, bi) of P, transposed below
    t[r][tx] = (i < K && j < K) ? P[i * K + j] : 0.f;
  }
  __syncthreads();
  for (int r = ty; r < 32; r += 8) {
    const int64_t i = bi * 32 + r, j = bj * 32 + tx;
    if (i < K && j < K) H[i * K + j] = 0.5f * (P[i * K + j] + t[tx][r]);
  }
}

// C -= A B^T over the whole contraction K, in chunks (A, B split into hi / lo, row stride K)
static hq_status psd_product(float* C, const float* Ah, const float* Al, const float* Bh, const float* Bl, int64_t K,
                             int* status, cudaStream_t s) {
  for (int64_t k0 = 0; k0 < K; k0 += kPsdChunk) {
    UpdGemm g{};
    g.C = C;
    g.ldc = K;
    g.M = static_cast<int>(K);
    g.N = static_cast<int>(K);
    g.Kred = static_cast<int>(K - k0 < kPsdChunk ? K - k0 : kPsdChunk);
    g.A_hi = Ah + k0;
    g.A_lo = Al + k0;
    g.lda = K;
    g.B_hi = Bh + k0;
    g.B_lo = Bl + k0;
    g.ldb = K;
    g.status = status;
    const hq_status st = upd_gemm(g, s);
    if (st != HQ_OK) return st;
  }
  return HQ_OK;
}

hq_status launch_psd(float* H, int64_t K, int steps, uint8_t* ws, int* status, cudaStream_t s) {
  const int64_t n = K * K;
  const size_t mat = round_up(static_cast<size_t>(n) * sizeof(float), 256);
  double* inv = reinterpret_cast<double*>(ws);
  double* part = reinterpret_cast<double*>(ws + 256);
  uint8_t* base = ws + 256 + round_up(static_cast<size_t>(kPsdRedBlocks) * sizeof(double), 256);
  float* Xa = reinterpret_cast<float*>(base);
  float* Xb = reinterpret_cast<float*>(base + mat);
  float* Xh = reinterpret_cast<float*>(base + 2 * mat);
  float* Xl = reinterpret_cast<float*>(base + 3 * mat);
  float* Yh = reinterpret_cast<float*>(base + 4 * mat);  // -X^2, then the tf32 part of -b (-X^2)
  float* Yl = reinterpret_cast<float*>(base + 5 * mat);
  const int grid = static_cast<int>(ceil_div(n, 256) < 148 * 8 ? ceil_div(n, 256) : 148 * 8);

  sumsq_kernel<<<kPsdRedBlocks, 256, 0, s>>>(H, n, part);
  HQ_LAUNCH_CHECK();
  inv_norm_kernel<<<1, 256, 0, s>>>(part, kPsdRedBlocks, inv);
  HQ_LAUNCH_CHECK();
  psd_init_kernel<<<grid, 256, 0, s>>>(H, n, inv, Xa);
  HQ_LAUNCH_CHECK();
  float* X = Xa;
  float* Xn = Xb;
  const int64_t nbt = ceil_div(K, 32);
  for (int it = 0; it < steps; ++it) {
    const float a = 1.5f, b = 0.5f;  // X <- a X - b X^3
    // Xh + Xl = X; Xn = a X; Yh = 0
    psd_split_kernel<<<grid, 256, 0, s>>>(X, n, 1.f, Xh, Xl, Xn, a, Yh);
    HQ_LAUNCH_CHECK();
    hq_status st = psd_product(Yh, Xh, Xl, Xh, Xl, K, status, s);  // Yh = -X X^T = -X^2
    if (st != HQ_OK) return st;
    psd_split_kernel<<<grid, 256, 0, s>>>(Yh, n, -b, Yh, Yl, nullptr, 0.f, nullptr);  // Yh + Yl = b X^2
    HQ_LAUNCH_CHECK();
    st = psd_product(Xn, Xh, Xl, Yh, Yl, K, status, s);  // Xn = a X - X (b X^2)
    if (st != HQ_OK) return st;
    psd_symmetrize_kernel<<<static_cast<unsigned>(nbt * nbt), 256, 0, s>>>(Xn, K, X);  // X = (Xn + Xn^T) / 2
    HQ_LAUNCH_CHECK();
  }
  // P = H / 2 + (H / 2) sign(H): Xn = H / 2, Yh + Yl = -H / 2, Xh + Xl = sign(H)
  psd_split_kernel<<<grid, 256, 0, s>>>(H, n, -0.5f, Yh, Yl, Xn, 0.5f, nullptr);
  HQ_LAUNCH_CHECK();
  psd_split_kernel<<<grid, 256, 0, s>>>(X, n, 1.f, Xh, Xl, nullptr, 0.f, nullptr);
  HQ_LAUNCH_CHECK();
  hq_status st = psd_product(Xn, Yh, Yl, Xh, Xl, K, status, s);
  if (st != HQ_OK) return st;
  psd_symmetrize_kernel<<<static_cast<unsigned>(nbt * nbt), 256, 0, s>>>(Xn, K, H);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

}  // namespace hq
