// Damping and the Cholesky chain of the GPTQ path ("Cholesky-based Hessian inverse", ork-
// driver wiki "Exp 2026-08-18 GPTQ Int4", experiment summary; damping relative to
// mean(diag H), "hipfire-calib-data" card, "REQUIRED: project to PSD before Cholesky").
//
// U, the upper Cholesky factor of (H + lambda I)^-1, is reached through the index reversal J:
// with M = J (H + lambda I) J = L L^T (L lower), U = J L^-1 J.  By uniqueness of the Cholesky
// factor this is the same U as Cholesky -> inverse -> Cholesky of the inverse, at half the
// flops.  Steps (all fp32 on the device):
//   1. lambda = damp * mean(diag H)            (fp64 reduction, one CTA)
//   2. A = J (H + lambda I) J, lower triangle  (tiled transpose; H's lower triangle is read)
//   3. A = L, blocked right-looking Cholesky   (64-wide panels: diagonal block in one CTA,
//      which also inverts it; panel solve by the inverted block; trailing update)
//   4. X = L^-1, recursive halving             (diagonal blocks from step 3, off-diagonal
//      blocks X21 = -X22 (L21 X11))
//   5. U^T = J X^T J written row-major         (U^T[c, j] = X[K-1-j, K-1-c], c >= j)
// A device flag `info` receives the first failing pivot (1-based) and stops later kernels.
#include "common.cuh"
#include "kernels.cuh"

namespace hq {

constexpr int NB = 64;

// ------------------------------------------------------------------------- 1. lambda

__global__ void __launch_bounds__(1024) damp_stats_kernel(const float* __restrict__ H, int64_t K, float damp,
                                                          double* __restrict__ lam, int* __restrict__ info) {
  __shared__ double red[1024];
  double s = 0.0;
  for (int64_t i = threadIdx.x; i < K; i += blockDim.x) s += static_cast<double>(H[i * K + i]);
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = 512; w > 0; w >>= 1) {
    if (static_cast<int>(threadIdx.x) < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double mean = red[0] / static_cast<double>(K);
    *lam = static_cast<double>(damp) * mean;
    if (!(mean > 0.0) || !isfinite(mean)) *info = -1;
  }
}

// ------------------------------------------------------------------------- 2. reverse + damp

__global__ void __launch_bounds__(256) reverse_damp_kernel(const float* __restrict__ H, int64_t K,
                                                           const double* __restrict__ lam, float* __restrict__ A,
                                                           const int* __restrict__ info) {
  if (*info != 0) return;
  __shared__ float t[32][33];
  int64_t tt = blockIdx.x;
  int64_t ta = static_cast<int64_t>((sqrt(8.0 * static_cast<double>(tt) + 1.0) - 1.0) * 0.5);
  while (ta * (ta + 1) / 2 > tt) --ta;
  while ((ta + 1) * (ta + 2) / 2 <= tt) ++ta;
  const int64_t tb = tt - ta * (ta + 1) / 2;
  const int64_t a0 = ta * 32, b0 = tb * 32;
  const int tx = threadIdx.x % 32, ty = threadIdx.x / 32;  // 32 x 8
  // t[j][i] = A[a0+i][b0+j] = H[K-1-(b0+j)][K-1-(a0+i)]  (lower triangle of H when a >= b)
  for (int j = ty; j < 32; j += 8) {
    const int64_t a = a0 + tx, b = b0 + j;
    float v = 0.f;
    if (a < K && b < K && a >= b) v = H[(K - 1 - b) * K + (K - 1 - a)];
    t[j][tx] = v;
  }
  __syncthreads();
  const double l = *lam;
  for (int i = ty; i < 32; i += 8) {
    const int64_t a = a0 + i, b = b0 + tx;
    if (a >= K || b >= K) continue;
    float v;
    if (a > b)
      v = t[tx][i];
    else if (a == b)
      v = static_cast<float>(static_cast<double>(t[tx][i]) + l);
    else
      v = 0.f;
    A[a * K + b] = v;
  }
}

// ------------------------------------------------------------------------- 3. Cholesky

// Factor the NB x NB diagonal block at (p, p) in shared memory, write L11 (upper part zeroed)
// back into A and its inverse into Dinv[p].
__global__ void __launch_bounds__(256) potrf_diag_kernel(float* __restrict__ A, int64_t K, int p,
                                                         float* __restrict__ Dinv, int* __restrict__ info) {
  if (*info != 0) return;
  __shared__ float S[NB][NB + 1];
  __shared__ float X[NB][NB + 1];
  __shared__ int bad;
  const int64_t o = static_cast<int64_t>(p) * NB;
  for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) {
    const int r = e / NB, c = e % NB;
    S[r][c] = (c <= r) ? A[(o + r) * K + o + c] : 0.f;
  }
  if (threadIdx.x == 0) bad = 0;
  __syncthreads();
  for (int k = 0; k < NB; ++k) {
    if (threadIdx.x == 0) {
      const float d = S[k][k];
      if (!(d > 0.f) || !isfinite(d)) {
        bad = 1;
        atomicCAS(info, 0, static_cast<int>(o + k + 1));
      } else {
        S[k][k] = sqrtf(d);
      }
    }
    __syncthreads();
    if (bad) return;
    const float lkk = S[k][k];
    for (int i = k + 1 + threadIdx.x; i < NB; i += blockDim.x) S[i][k] = S[i][k] / lkk;
    __syncthreads();
    const int m = NB - k - 1;
    for (int e = threadIdx.x; e < m * m; e += blockDim.x) {
      const int i = k + 1 + e / m, j = k + 1 + e % m;
      if (j <= i) S[i][j] = fmaf(-S[i][k], S[j][k], S[i][j]);
    }
    __syncthreads();
  }
  // inverse of the lower-triangular block, one column per thread (forward substitution)
  if (threadIdx.x < NB) {
    const int j = threadIdx.x;
    for (int i = 0; i < j; ++i) X[i][j] = 0.f;
    X[j][j] = 1.f / S[j][j];
    for (int i = j + 1; i < NB; ++i) {
      float acc = 0.f;
      for (int k = j; k < i; ++k) acc = fmaf(S[i][k], X[k][j], acc);
      X[i][j] = -acc / S[i][i];
    }
  }
  __syncthreads();
  float* D = Dinv + static_cast<int64_t>(p) * NB * NB;
  for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) {
    const int r = e / NB, c = e % NB;
    A[(o + r) * K + o + c] = (c <= r) ? S[r][c] : 0.f;
    D[e] = X[r][c];
  }
}

// L21 = A21 * L11^-T = A21 * Dinv^T for the NB-row slab per CTA below the diagonal block.
__global__ void __launch_bounds__(256) trsm_panel_kernel(float* __restrict__ A, int64_t K, int p,
                                                         const float* __restrict__ Dinv,
                                                         const int* __restrict__ info) {
  if (*info != 0) return;
  __shared__ float As[NB][NB + 1];
  __shared__ float Ds[NB][NB + 1];
  const int64_t o = static_cast<int64_t>(p) * NB;
  const int64_t r0 = o + NB + static_cast<int64_t>(blockIdx.x) * NB;
  const float* D = Dinv + static_cast<int64_t>(p) * NB * NB;
  for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) {
    const int r = e / NB, c = e % NB;
    As[r][c] = (r0 + r < K) ? A[(r0 + r) * K + o + c] : 0.f;
    Ds[r][c] = D[e];
  }
  __syncthreads();
  for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) {
    const int r = e / NB, j = e % NB;
    if (r0 + r >= K) continue;
    float acc = 0.f;
    for (int k = 0; k <= j; ++k) acc = fmaf(As[r][k], Ds[j][k], acc);  // Dinv lower: k <= j
    A[(r0 + r) * K + o + j] = acc;
  }
}

// ------------------------------------------------------------------------- CUDA-core GEMM

// C[m, n] = beta * C[m, n] + alpha * sum_k A(m, k) B(k, n), with A(m, k) = A[m*sam + k*sak]
// and B(k, n) = B[k*sbk + n*sbn].  lower_only: only tiles/elements with m >= n (row and
// column indices offset by diag_off: element kept when m + diag_off >= n).
struct SimtGemm {
  const float* A;
  int64_t sam, sak;
  const float* B;
  int64_t sbk, sbn;
  float* C;
  int64_t ldc;
  int M, N, Kc;
  float alpha, beta;
  int lower_only;
};

__global__ void __launch_bounds__(256) gemm_simt_kernel(SimtGemm g, const int* __restrict__ info) {
  if (info != nullptr && *info != 0) return;
  const int tiles_n = (g.N + 63) / 64;
  const int tm = blockIdx.x / tiles_n, tn = blockIdx.x % tiles_n;
  if (g.lower_only && tn > tm) return;
  const int m0 = tm * 64, n0 = tn * 64;
  __shared__ float As[16][64];
  __shared__ float Bs[16][64];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < g.Kc; k0 += 16) {
    for (int e = threadIdx.x; e < 16 * 64; e += 256) {
      const int kk = e / 64, c = e % 64;
      const int k = k0 + kk;
      As[kk][c] = (k < g.Kc && m0 + c < g.M) ? g.A[(m0 + c) * g.sam + k * g.sak] : 0.f;
      Bs[kk][c] = (k < g.Kc && n0 + c < g.N) ? g.B[k * g.sbk + (n0 + c) * g.sbn] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        a[u] = As[kk][ty + 16 * u];
        b[u] = Bs[kk][tx + 16 * u];
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
    const int m = m0 + ty + 16 * u;
    if (m >= g.M) continue;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int n = n0 + tx + 16 * v;
      if (n >= g.N || (g.lower_only && n > m)) continue;
      float* c = g.C + static_cast<int64_t>(m) * g.ldc + n;
      *c = (g.beta == 0.f ? 0.f : g.beta * *c) + g.alpha * acc[u][v];
    }
  }
}

static hq_status gemm_simt(const SimtGemm& g, const int* info, cudaStream_t s) {
  if (g.M <= 0 || g.N <= 0) return HQ_OK;
  const int64_t tiles = ceil_div(g.M, 64) * ceil_div(g.N, 64);
  gemm_simt_kernel<<<static_cast<unsigned>(tiles), 256, 0, s>>>(g, info);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

// ------------------------------------------------------------------------- 4. L^-1

static hq_status invert_lower_rec(const float* L, float* X, float* T, int64_t K, int64_t off, int64_t n,
                                  const float* Dinv, const int* info, cudaStream_t s) {
  if (n == NB) {
    // X block = Dinv[off / NB]
    HQ_CUDA_TRY(cudaMemcpy2DAsync(X + off * K + off, K * sizeof(float), Dinv + (off / NB) * NB * NB,
                                  NB * sizeof(float), NB * sizeof(float), NB, cudaMemcpyDeviceToDevice, s));
    return HQ_OK;
  }
  const int64_t nblk = n / NB;
  const int64_t n1 = (nblk / 2) * NB, n2 = n - n1;
  hq_status st = invert_lower_rec(L, X, T, K, off, n1, Dinv, info, s);
  if (st != HQ_OK) return st;
  st = invert_lower_rec(L, X, T, K, off + n1, n2, Dinv, info, s);
  if (st != HQ_OK) return st;
  // T = L21 X11   (n2 x n1)
  SimtGemm g1{};
  g1.A = L + (off + n1) * K + off;
  g1.sam = K;
  g1.sak = 1;
  g1.B = X + off * K + off;
  g1.sbk = K;
  g1.sbn = 1;
  g1.C = T;
  g1.ldc = n1;
  g1.M = static_cast<int>(n2);
  g1.N = static_cast<int>(n1);
  g1.Kc = static_cast<int>(n1);
  g1.alpha = 1.f;
  g1.beta = 0.f;
  st = gemm_simt(g1, info, s);
  if (st != HQ_OK) return st;
  // X21 = -X22 T  (n2 x n1)
  SimtGemm g2{};
  g2.A = X + (off + n1) * K + off + n1;
  g2.sam = K;
  g2.sak = 1;
  g2.B = T;
  g2.sbk = n1;
  g2.sbn = 1;
  g2.C = X + (off + n1) * K + off;
  g2.ldc = K;
  g2.M = static_cast<int>(n2);
  g2.N = static_cast<int>(n1);
  g2.Kc = static_cast<int>(n2);
  g2.alpha = -1.f;
  g2.beta = 0.f;
  return gemm_simt(g2, info, s);
}

// ------------------------------------------------------------------------- 5. U^T

// Ut[c][j] = X[K-1-j][K-1-c] for c >= j, 0 above the diagonal.  32 x 32 tiles via smem.
__global__ void __launch_bounds__(256) anti_transpose_kernel(const float* __restrict__ X, int64_t K,
                                                             float* __restrict__ Ut, const int* __restrict__ info) {
  if (*info != 0) return;
  __shared__ float t[32][33];
  const int64_t tiles = (K + 31) / 32;
  const int64_t tc = blockIdx.x / tiles, tj = blockIdx.x % tiles;
  const int64_t c0 = tc * 32, j0 = tj * 32;
  const int tx = threadIdx.x % 32, ty = threadIdx.x / 32;
  // source rows K-1-j (j in tile), columns K-1-c (c in tile)
  for (int jj = ty; jj < 32; jj += 8) {
    const int64_t j = j0 + jj, c = c0 + tx;
    float v = 0.f;
    if (j < K && c < K && c >= j) v = X[(K - 1 - j) * K + (K - 1 - c)];
    t[jj][tx] = v;  // t[j][c]
  }
  __syncthreads();
  for (int cc = ty; cc < 32; cc += 8) {
    const int64_t c = c0 + cc, j = j0 + tx;
    if (c < K && j < K) Ut[c * K + j] = t[tx][cc];
  }
}

// ------------------------------------------------------------------------- driver

size_t factor_workspace_floats(int64_t K) {
  // A (K^2), X (K^2), T (K^2/4), Dinv (K * NB)
  return static_cast<size_t>(K) * K * 2 + static_cast<size_t>(K / 2) * (K - K / 2 + NB) + static_cast<size_t>(K) * NB;
}

hq_status launch_factor(const float* H, int64_t K, float damp, float* A, float* X, float* T, float* Dinv,
                        double* lam, int* info, float* Ut, cudaStream_t s) {
  damp_stats_kernel<<<1, 1024, 0, s>>>(H, K, damp, lam, info);
  HQ_LAUNCH_CHECK();
  {
    const int64_t nb = ceil_div(K, 32);
    reverse_damp_kernel<<<static_cast<unsigned>(nb * (nb + 1) / 2), 256, 0, s>>>(H, K, lam, A, info);
    HQ_LAUNCH_CHECK();
  }
  const int np = static_cast<int>(K / NB);
  for (int p = 0; p < np; ++p) {
    potrf_diag_kernel<<<1, 256, 0, s>>>(A, K, p, Dinv, info);
    HQ_LAUNCH_CHECK();
    const int rows_below = static_cast<int>(K - static_cast<int64_t>(p + 1) * NB);
    if (rows_below <= 0) break;
    trsm_panel_kernel<<<static_cast<unsigned>(ceil_div(rows_below, NB)), 256, 0, s>>>(A, K, p, Dinv, info);
    HQ_LAUNCH_CHECK();
    SimtGemm g{};
    const int64_t o = static_cast<int64_t>(p + 1) * NB;
    g.A = A + o * K + p * NB;  // L21 rows (o.., panel cols)
    g.sam = K;
    g.sak = 1;
    g.B = A + o * K + p * NB;  // B(k, n) = L21[n][k]
    g.sbk = 1;
    g.sbn = K;
    g.C = A + o * K + o;
    g.ldc = K;
    g.M = rows_below;
    g.N = rows_below;
    g.Kc = NB;
    g.alpha = -1.f;
    g.beta = 1.f;
    g.lower_only = 1;
    hq_status st = gemm_simt(g, info, s);
    if (st != HQ_OK) return st;
  }
  HQ_CUDA_TRY(cudaMemsetAsync(X, 0, static_cast<size_t>(K) * K * sizeof(float), s));
  hq_status st = invert_lower_rec(A, X, T, K, 0, K, Dinv, info, s);
  if (st != HQ_OK) return st;
  {
    const int64_t nt = ceil_div(K, 32);
    anti_transpose_kernel<<<static_cast<unsigned>(nt * nt), 256, 0, s>>>(X, K, Ut, info);
    HQ_LAUNCH_CHECK();
  }
  return HQ_OK;
}

}  // namespace hq
