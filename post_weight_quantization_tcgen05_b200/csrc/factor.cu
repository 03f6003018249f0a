// Damping and the Cholesky chain of the GPTQ path ("Cholesky-based Hessian inverse", ork-
// driver wiki "Exp 2026-08-18 GPTQ Int4", experiment summary; damping relative to
// mean(diag H), "hipfire-calib-data" card, "REQUIRED: project to PSD before Cholesky").
//
// U, the upper Cholesky factor of (H + lambda I)^-1, is reached through the index reversal J:
// with M = J (H + lambda I) J = L L^T (L lower), U = J L^-1 J.  By uniqueness of the Cholesky
// factor this is the same U as Cholesky -> inverse -> Cholesky of the inverse, at half the
// flops.  Only X = L^-1 is ever needed, so the factorisation and the inversion are one
// recursion on M:
//
//   chol_inv([A11 .; A21 A22]):  X11 = chol_inv(A11)
//                                T   = A21 X11^T          (= L21)
//                                A22 = A22 - T T^T        (Schur complement, lower part)
//                                X22 = chol_inv(A22)
//                                Y^T = X11^T T^T          (Y = T X11)
//                                X21 = -X22 Y
//
// Every product takes both operands K-major (row-major [rows, contraction]), so X^T is kept
// next to X (leaves write both, X21^T is copied by a tiled transpose).  Everything runs in fp64
// (gemm_f64.cu for the products; each declares its triangular operand so that tiles skip the
// zero part of the contraction).  Leaves are 64 x 64 blocks factored and inverted by one CTA
// (chol_inv_leaf_kernel).  Steps:
//   1. lambda = damp * mean(diag H)            (fp64 reduction, one CTA)
//   2. A = J (H + lambda I) J in fp64, lower triangle (tiled transpose of H's lower triangle)
//   3. X = L^-1 and X^T by the recursion above
//   4. U = J X J and U^T = J X^T J, both row-major (180-degree rotated copies)
// A device flag `info` receives the first failing pivot (1-based, in M's order) and stops
// every later kernel.
#include "common.cuh"
#include "kernels.cuh"

namespace hq {

constexpr int kLeaf = 64;

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
                                                           const double* __restrict__ lam, double* __restrict__ A,
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
    double v;
    if (a > b)
      v = static_cast<double>(t[tx][i]);
    else if (a == b)
      v = static_cast<double>(t[tx][i]) + l;
    else
      v = 0.0;
    A[a * K + b] = v;
  }
}

// ------------------------------------------------------------------------- 3a. leaf

// 1 / d for d > 0 (normal, finite): the hardware approximation (rcp.approx.ftz.f64) refined by
// two Newton-Raphson steps for the reciprocal, r <- r + r (1 - d r), each of which squares the
// relative error; within 2 ulp of the correctly rounded quotient.  About a third of the latency
// of the IEEE division, which sits on the leaf's critical path once per pivot.
__device__ __forceinline__ double rcp_nr(double d) {
  double r;
  asm("rcp.approx.ftz.f64 %0, %1;" : "=d"(r) : "d"(d));
  double e = fma(-d, r, 1.0);
  r = fma(r, e, r);
  e = fma(-d, r, 1.0);
  return fma(r, e, r);
}

__global__ void rcp_nr_kernel(const double* __restrict__ d, double* __restrict__ out, int64_t n) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    out[i] = rcp_nr(d[i]);
}

hq_status launch_rcp_nr(const double* d, double* out, int64_t n, cudaStream_t s) {
  if (n <= 0) return HQ_OK;
  const int64_t grid = ceil_div(n, 256) < 148 * 16 ? ceil_div(n, 256) : 148 * 16;
  rcp_nr_kernel<<<static_cast<unsigned>(grid), 256, 0, s>>>(d, out, n);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

// Factor the 64 x 64 lower block at A as L D L^T (unit L) by right-looking elimination, and
// at the same time eliminate Y = L^-1 (unit lower); writes X = D^-1/2 Y = (L D^1/2)^-1, the
// inverse of the Cholesky factor (zeros above the diagonal), and X^T.  fp64.  The lower
// triangle of the leaf is cut into 136 tiles of 4 x 4; thread t < 136 owns tile t of both S and
// Y, in registers.  Before step k, the owners publish column k of the Schur complement (with
// zeros at rows <= k), row k of Y (zeros right of k) and 1 / d_k through double-buffered shared
// memory; one barrier per step.  Because of those zeros every thread applies the same rank-1
// update to all 32 of its elements without masks (the part of a tile the step does not touch
// gets a zero factor).  Only the elements step k + 1 publishes (one column of the S tile, one
// row of the Y tile) are updated before the barrier; the rest of step k's update is applied
// after it, while step k + 1's shared-memory loads are in flight.  The step loop is unrolled by
// four so that positions inside a tile are compile-time register indices.  Pivots are checked
// once at the end (a bad pivot only produces values that are then discarded).
constexpr int kLB = kLeaf;                                 // 64
constexpr int kLeafTiles = (kLB / 4) * (kLB / 4 + 1) / 2;  // 136
constexpr int kLeafThreads = 160;                          // 5 warps, one tile per thread

__device__ __forceinline__ void leaf_tile(int idx, int& ti, int& tj) {
  int r = static_cast<int>((sqrtf(8.f * idx + 1.f) - 1.f) * 0.5f);
  while (r * (r + 1) / 2 > idx) --r;
  while ((r + 1) * (r + 2) / 2 <= idx) ++r;
  ti = r;
  tj = idx - r * (r + 1) / 2;
}

__global__ void __launch_bounds__(kLeafThreads, 1) chol_inv_leaf_kernel(const double* __restrict__ A, int64_t lda,
                                                                         double* __restrict__ X,
                                                                         double* __restrict__ XT, int64_t ldx,
                                                                         int* __restrict__ info, int diag_off) {
  if (*info != 0) return;
  __shared__ __align__(16) double colbuf[2][kLB];
  __shared__ __align__(16) double yrow[2][kLB];
  __shared__ double pinv[2];
  __shared__ double dbuf[kLB];
  __shared__ int bad;
  const int t = threadIdx.x;
  const bool own = t < kLeafTiles;
  int ti, tj;
  leaf_tile(own ? t : 0, ti, tj);
  const int i0 = 4 * ti, j0 = 4 * tj;
  double v[16], y[16];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      v[r * 4 + c] = (own && j0 + c <= i0 + r) ? A[(i0 + r) * lda + j0 + c] : 0.0;
      y[r * 4 + c] = (own && i0 + r == j0 + c) ? 1.0 : 0.0;
    }
  if (t < kLB) {
    colbuf[0][t] = colbuf[1][t] = 0.0;
    yrow[0][t] = yrow[1][t] = 0.0;
  }
  if (t == 0) bad = kLB;
  __syncthreads();
  // publish column 0 (rows > 0), row 0 of Y and 1 / d_0
  if (own && tj == 0) {
#pragma unroll
    for (int r = 0; r < 4; ++r) colbuf[0][i0 + r] = (ti > 0 || r > 0) ? v[r * 4] : 0.0;
  }
  if (own && ti == 0) {
#pragma unroll
    for (int c = 0; c < 4; ++c) yrow[0][j0 + c] = y[c];
    pinv[0] = rcp_nr(v[0]);
  }
  __syncthreads();

  // factors of the previous step, whose update is finished at the start of this one
  double pa[4] = {0.0, 0.0, 0.0, 0.0}, pb[4] = {0.0, 0.0, 0.0, 0.0}, pyb[4] = {0.0, 0.0, 0.0, 0.0};
  for (int kt = 0; kt < kLB / 4; ++kt) {
#pragma unroll
    for (int kc = 0; kc < 4; ++kc) {
      const int buf = kc & 1;  // == k & 1
      const bool last = (kt == kLB / 4 - 1) && kc == 3;
      // step k - 1's update, except column kc of S and row kc of Y (done before its barrier)
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (c != kc) v[r * 4 + c] = fma(-pa[r], pb[c], v[r * 4 + c]);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        if (r == kc) continue;
#pragma unroll
        for (int c = 0; c < 4; ++c) y[r * 4 + c] = fma(-pa[r], pyb[c], y[r * 4 + c]);
      }
      if (last) break;  // pivot 63 updates nothing: no row lies below it
      const double inv_d = pinv[buf];
      const double2 ca0 = *reinterpret_cast<const double2*>(&colbuf[buf][i0]);
      const double2 ca1 = *reinterpret_cast<const double2*>(&colbuf[buf][i0 + 2]);
      const double2 cb0 = *reinterpret_cast<const double2*>(&colbuf[buf][j0]);
      const double2 cb1 = *reinterpret_cast<const double2*>(&colbuf[buf][j0 + 2]);
      const double2 yb0 = *reinterpret_cast<const double2*>(&yrow[buf][j0]);
      const double2 yb1 = *reinterpret_cast<const double2*>(&yrow[buf][j0 + 2]);
      // L[i][k] (zero at and above the pivot), S[j][k] (zero at and left of it), Y[k][j]
      const double a[4] = {ca0.x * inv_d, ca0.y * inv_d, ca1.x * inv_d, ca1.y * inv_d};
      const double b[4] = {cb0.x, cb0.y, cb1.x, cb1.y};
      const double yb[4] = {yb0.x, yb0.y, yb1.x, yb1.y};

      // elements published for step k + 1: column k + 1 of S, row k + 1 of Y, d_{k+1}
      const int ktn = (kc == 3) ? kt + 1 : kt;
      const int cn = (kc + 1) & 3;
      const int nb = buf ^ 1;
#pragma unroll
      for (int r = 0; r < 4; ++r) v[r * 4 + cn] = fma(-a[r], b[cn], v[r * 4 + cn]);
#pragma unroll
      for (int c = 0; c < 4; ++c) y[cn * 4 + c] = fma(-a[cn], yb[c], y[cn * 4 + c]);
      if (own && tj == ktn) {
#pragma unroll
        for (int r = 0; r < 4; ++r) colbuf[nb][i0 + r] = (ti > ktn || r > cn) ? v[r * 4 + cn] : 0.0;
        // a new tile column: the last row of the previous diagonal tile still holds a value in
        // this buffer (published two steps ago)
        if (cn == 0 && ti == ktn) colbuf[nb][i0 - 1] = 0.0;
      }
      if (own && ti == ktn) {
#pragma unroll
        for (int c = 0; c < 4; ++c) yrow[nb][j0 + c] = y[cn * 4 + c];
        if (tj == ktn) pinv[nb] = rcp_nr(v[cn * 4 + cn]);
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        pa[r] = a[r];
        pb[r] = b[r];
        pyb[r] = yb[r];
      }
      __syncthreads();
    }
  }
  // pivots d_i (the diagonal of S when it was eliminated); the first bad one fails the leaf
  if (own && ti == tj) {
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      const double d = v[r * 4 + r];
      dbuf[i0 + r] = d;
      if (!(d >= 2.2250738585072014e-308) || !isfinite(d)) atomicMin(&bad, i0 + r);  // not normal, > 0
    }
  }
  __syncthreads();
  if (bad < kLB) {
    if (t == 0) atomicCAS(info, 0, diag_off + bad + 1);
    return;
  }
  if (!own) return;
  // X[i][j] = Y[i][j] / sqrt(d_i)
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const double sc = 1.0 / sqrt(dbuf[i0 + r]);
#pragma unroll
    for (int c = 0; c < 4; ++c) y[r * 4 + c] *= sc;
  }
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    double* xr = X + static_cast<int64_t>(i0 + r) * ldx + j0;
#pragma unroll
    for (int c = 0; c < 4; ++c) xr[c] = y[r * 4 + c];
  }
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    double* xr = XT + static_cast<int64_t>(j0 + c) * ldx + i0;
#pragma unroll
    for (int r = 0; r < 4; ++r) xr[r] = y[r * 4 + c];
  }
}

// ------------------------------------------------------------------------- 3b. recursion

struct FactorCtx {
  double* A;
  double* X;
  double* XT;
  double* tmp_end;  // end of the temporaries region
  int64_t K;
  int* info;
  int* status;
  cudaStream_t s;
};

// `scratch` (up to the end of the temporaries) receives split-K partial tiles.
static hq_status gemm(const FactorCtx& c, double* scratch, double* C, int64_t ldc, int M, int N, int Kred,
                      const double* A, int64_t lda, const double* B, int64_t ldb, double alpha, double beta,
                      bool lower, int tri) {
  F64Gemm g{};
  g.C = C;
  g.ldc = ldc;
  g.M = M;
  g.N = N;
  g.Kred = Kred;
  g.A = A;
  g.lda = lda;
  g.B = B;
  g.ldb = ldb;
  g.alpha = alpha;
  g.beta = beta;
  g.lower = lower ? 1 : 0;
  g.tri = tri;
  g.scratch = scratch;
  g.scratch_elems = c.tmp_end - scratch;
  g.skip = c.info;
  return f64_gemm(g, c.s);
}

// dst[j][i] = src[i][j] for an R x C block (32 x 32 tiles through shared memory).
__global__ void __launch_bounds__(256) transpose_kernel(const double* __restrict__ src, int64_t lds, int64_t R,
                                                        int64_t C, double* __restrict__ dst, int64_t ldd,
                                                        const int* __restrict__ info) {
  if (*info != 0) return;
  __shared__ double t[32][33];
  const int64_t tiles_c = (C + 31) / 32;
  const int64_t r0 = (blockIdx.x / tiles_c) * 32, c0 = (blockIdx.x % tiles_c) * 32;
  const int tx = threadIdx.x % 32, ty = threadIdx.x / 32;
  for (int i = ty; i < 32; i += 8)
    if (r0 + i < R && c0 + tx < C) t[i][tx] = src[(r0 + i) * lds + c0 + tx];
  __syncthreads();
  for (int j = ty; j < 32; j += 8)
    if (c0 + j < C && r0 + tx < R) dst[(c0 + j) * ldd + r0 + tx] = t[tx][j];
}

// X = L^-1 and X^T for the n x n block of A at (off, off); `tmp` has room for the temporaries
// of this level and all levels below (2 * n2 * n1 here, about a quarter of that per level below).
static hq_status chol_inv(const FactorCtx& c, int64_t off, int64_t n, double* tmp) {
  const int64_t K = c.K;
  if (n == kLeaf) {
    chol_inv_leaf_kernel<<<1, kLeafThreads, 0, c.s>>>(c.A + off * K + off, K, c.X + off * K + off,
                                                      c.XT + off * K + off, K, c.info, static_cast<int>(off));
    HQ_LAUNCH_CHECK();
    return HQ_OK;
  }
  const int64_t n1 = (n / kLeaf / 2) * kLeaf, n2 = n - n1;
  double* T = tmp;             // n2 x n1: L21
  double* YT = tmp + n2 * n1;  // n1 x n2: (L21 X11)^T
  double* rest = YT + n2 * n1;
  const double* A21 = c.A + (off + n1) * K + off;
  double* A22 = c.A + (off + n1) * K + off + n1;
  const double* X11 = c.X + off * K + off;
  const double* XT11 = c.XT + off * K + off;
  double* X21 = c.X + (off + n1) * K + off;
  const double* X22 = c.X + (off + n1) * K + off + n1;
  double* XT12 = c.XT + off * K + off + n1;
  const int in1 = static_cast<int>(n1), in2 = static_cast<int>(n2);
  hq_status st = chol_inv(c, off, n1, rest);
  if (st != HQ_OK) return st;
  st = gemm(c, rest, T, n1, in2, in1, in1, A21, K, X11, K, 1.0, 0.0, false, kTriBLower);  // T = A21 X11^T
  if (st != HQ_OK) return st;
  st = gemm(c, rest, A22, K, in2, in2, in1, T, n1, T, n1, -1.0, 1.0, true, kTriNone);     // A22 -= T T^T
  if (st != HQ_OK) return st;
  st = chol_inv(c, off + n1, n2, rest);
  if (st != HQ_OK) return st;
  st = gemm(c, rest, YT, n2, in1, in2, in1, XT11, K, T, n1, 1.0, 0.0, false, kTriAUpper); // Y^T = X11^T T^T
  if (st != HQ_OK) return st;
  st = gemm(c, rest, X21, K, in2, in1, in2, X22, K, YT, n2, -1.0, 0.0, false, kTriALower); // X21 = -X22 Y
  if (st != HQ_OK) return st;
  const int64_t tiles = ceil_div(n2, 32) * ceil_div(n1, 32);
  transpose_kernel<<<static_cast<unsigned>(tiles), 256, 0, c.s>>>(X21, K, n2, n1, XT12, K, c.info);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

// ------------------------------------------------------------------------- 4. U, U^T

// U[j][c] = X[K-1-j][K-1-c] and U^T[j][c] = X^T[K-1-j][K-1-c], rounded to fp32: 180-degree
// rotations (U upper, U^T lower, zeros elsewhere because X and X^T hold zeros there).
__global__ void rotate_kernel(const double* __restrict__ X, const double* __restrict__ XT, int64_t K,
                              float* __restrict__ U, float* __restrict__ Ut, const int* __restrict__ info) {
  if (*info != 0) return;
  const int64_t n = K * K;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t src = n - 1 - e;  // (K-1-j)*K + (K-1-c) for e = j*K + c
    U[e] = static_cast<float>(X[src]);
    Ut[e] = static_cast<float>(XT[src]);
  }
}

// ------------------------------------------------------------------------- driver

hq_status launch_factor(const float* H, int64_t K, float damp, double* A, double* X, double* XT, double* T,
                        double* lam, int* info, int* status, float** Ut, float** U, cudaStream_t s) {
  (void)status;
  if (K % kLeaf != 0) return HQ_ERR_UNSUPPORTED;
  damp_stats_kernel<<<1, 1024, 0, s>>>(H, K, damp, lam, info);
  HQ_LAUNCH_CHECK();
  {
    const int64_t nb = ceil_div(K, 32);
    reverse_damp_kernel<<<static_cast<unsigned>(nb * (nb + 1) / 2), 256, 0, s>>>(H, K, lam, A, info);
    HQ_LAUNCH_CHECK();
  }
  HQ_CUDA_TRY(cudaMemsetAsync(X, 0, static_cast<size_t>(K) * K * sizeof(double), s));
  HQ_CUDA_TRY(cudaMemsetAsync(XT, 0, static_cast<size_t>(K) * K * sizeof(double), s));
  FactorCtx c{A, X, XT, T + K * K, K, info, status, s};
  hq_status st = chol_inv(c, 0, K, T);
  if (st != HQ_OK) return st;
  // A is dead now: U^T and U (fp32) go into its storage
  *Ut = reinterpret_cast<float*>(A);
  *U = reinterpret_cast<float*>(A) + K * K;
  const int64_t grid = ceil_div(K * K, 4 * 256) < 148 * 32 ? ceil_div(K * K, 4 * 256) : 148 * 32;
  rotate_kernel<<<static_cast<unsigned>(grid), 256, 0, s>>>(X, XT, K, *U, *Ut, info);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

}  // namespace hq
