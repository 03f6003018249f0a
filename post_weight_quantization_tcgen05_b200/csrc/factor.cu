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
// next to X (leaves write both; the product that forms X21 also writes X21^T).  Everything is
// fp64-accurate: products with all dimensions >= kI8xMinDim run on the int8 tensor cores from
// exact int8 slices (gemm_i8x.cu), the others on the fp64 tensor cores (gemm_f64.cu); each
// declares its triangular operand so that tiles skip the zero part of the contraction.  Leaves are 128 x 128 blocks factored and inverted by one CTA
// (chol_inv_leaf_kernel).  Steps:
//   1. lambda = damp * mean(diag H)            (fp64 reduction, one CTA)
//   2. A = J (H + lambda I) J in fp64, lower triangle (tiled transpose of H's lower triangle)
//   3. X = L^-1 and X^T by the recursion above (zeros are read only inside the diagonal leaf
//      blocks, so for the sweep's split output only those blocks are cleared first)
//   4. U = J X J and U^T = J X^T J, both row-major (180-degree rotated copies)
// A device flag `info` receives the first failing pivot (1-based, in M's order) and stops
// every later kernel.
#include <algorithm>
#include <vector>

#include "common.cuh"
#include "kernels.cuh"

namespace hq {

constexpr int kLeaf = 128;

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

// L D L^T of a symmetric 4 x 4 block given by its lower part s (row-major 4 x 4; only
// s[r][c], c <= r, read): pivots d, the strict lower part m of L^-1 (m10 m20 m30 m21 m31 m32)
// and w = S^-1 (row-major 4 x 4, both triangles).
__device__ __forceinline__ void ldl4_inverse(const double (&s)[16], double (&d)[4], double (&m)[6],
                                             double (&w)[16]) {
  d[0] = s[0];
  const double r0 = rcp_nr(d[0]);
  const double l10 = s[4] * r0, l20 = s[8] * r0, l30 = s[12] * r0;
  d[1] = fma(-l10, s[4], s[5]);
  const double r1 = rcp_nr(d[1]);
  const double t21 = fma(-l20, s[4], s[9]), t31 = fma(-l30, s[4], s[13]);
  const double l21 = t21 * r1, l31 = t31 * r1;
  d[2] = fma(-l21, t21, fma(-l20, s[8], s[10]));
  const double r2 = rcp_nr(d[2]);
  const double t32 = fma(-l31, t21, fma(-l30, s[8], s[14]));
  const double l32 = t32 * r2;
  d[3] = fma(-l32, t32, fma(-l31, t31, fma(-l30, s[12], s[15])));
  const double r3 = rcp_nr(d[3]);
  // M = L^-1 (unit lower)
  const double m10 = -l10, m21 = -l21, m32 = -l32;
  const double m20 = -fma(l21, m10, l20);
  const double m31 = -fma(l32, m21, l31);
  const double m30 = -fma(l32, m20, fma(l31, m10, l30));
  m[0] = m10; m[1] = m20; m[2] = m30; m[3] = m21; m[4] = m31; m[5] = m32;
  // W = M^T D^-1 M: W[a][b] = sum_{k >= max(a, b)} M[k][a] M[k][b] / d_k
  const double w33 = r3, w32 = r3 * m32, w31 = r3 * m31, w30 = r3 * m30;
  const double q2 = r2 * m21, q3 = r3 * m32;  // reused products
  const double w22 = fma(q3, m32, r2);
  const double w21 = fma(q3, m31, q2);
  const double w20 = fma(q3, m30, r2 * m20);
  const double w11 = fma(r3 * m31, m31, fma(q2, m21, r1));
  const double w10 = fma(r3 * m31, m30, fma(q2, m20, r1 * m10));
  const double w00 = fma(r3 * m30, m30, fma(r2 * m20, m20, fma(r1 * m10, m10, r0)));
  w[0] = w00; w[1] = w10; w[2] = w20; w[3] = w30;
  w[4] = w10; w[5] = w11; w[6] = w21; w[7] = w31;
  w[8] = w20; w[9] = w21; w[10] = w22; w[11] = w32;
  w[12] = w30; w[13] = w31; w[14] = w32; w[15] = w33;
}

// X = L^-1 and X^T for the 128 x 128 lower block at A, where A = L L^T (Cholesky), in one CTA of
// 16 warps, fp64, in three phases.  With 4 x 4 pivot blocks B, A = M S M^T where M is block unit
// lower triangular (off-diagonal blocks the multipliers N = M - I) and S block diagonal (the
// pivot blocks S_BB = L_B D_B L_B^T); so L = M diag(L_B D_B^1/2) and
// X = diag(D_B^-1/2 L_B^-1) M^-1.  The Schur complement S and the multipliers N live in shared
// memory as the 136 lower 8 x 8 tiles of each.
//   1. Block right-looking elimination, warp I owning tile row I.  Block step kt (B = rows and
//      columns 4kt .. 4kt+3), with the panel P = S[:, B] read with zeros at rows <= 4kt+3 and
//      W = S_BB^-1 = L_B^-T D_B^-1 L_B^-1 (computed in the previous step): warp I computes
//      G_I = P_I W (one fp64 MMA), stores it as N's block, and updates its tiles right of B,
//      S[I][J] -= G_I P_J^T (one fp64 MMA m8n8k4 per 8 x 8 tile); the warp owning the next pivot
//      block's diagonal tile updates that tile first and computes the next W (and keeps D_B,
//      L_B^-1) while the others go on; one barrier per block step.
//   2. Z = M^-1: the diagonal tiles Z_JJ = I - N_JJ, then the off-diagonal blocks by recursive
//      doubling over blocks of 1, 2, 4 and 8 tile rows, Z21 = -Z22 (N21 Z11), the tiles of each
//      level spread over all 16 warps (leaf_inverse_level); Z takes S's tiles.
//   3. X = diag(D_B^-1/2 L_B^-1) Z, written to X and X^T.
// Pivots (the entries of D) are checked after phase 1 (a bad pivot only produces values that
// are then discarded).  Updating the inverse alongside the elimination instead (the identity
// eliminated with S) costs twice the barrier-synchronised tile work per step.
constexpr int kLB = kLeaf;                    // 128
constexpr int kLT = kLB / 8;                  // 16 tile rows, one per warp
constexpr int kLTiles = kLT * (kLT + 1) / 2;  // 136
constexpr int kLeafThreads = 32 * kLT;
constexpr size_t kLeafSmem = (2 * kLTiles * 64 + 2 * 16 + kLB + (kLB / 4) * 6 + 2 * kLB * 4) * sizeof(double);

// Element (r, c) of lower tile (I, J): tiles row by row, 64 doubles each, the two 4-column
// halves of rows 2, 3, 6, 7 swapped (fragment loads of 8 rows x 4 columns and of 4 rows x 8
// columns then hit distinct banks in each half-warp; 16-byte pairs stay contiguous).
__device__ __forceinline__ int lt_idx(int I, int J, int r, int c) {
  return (I * (I + 1) / 2 + J) * 64 + r * 8 + (c ^ (((r >> 1) & 1) << 2));
}

// D (8 x 8) += A (8 x 4) B (4 x 8): lane (g = lane / 4, t = lane % 4) holds A[g][t], B[t][g] and
// D[g][2t], D[g][2t + 1].
__device__ __forceinline__ void dmma_leaf(double& d0, double& d1, double a, double b) {
  asm("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};\n"
      : "+d"(d0), "+d"(d1)
      : "d"(a), "d"(b));
}

// W, D, L^-1 of pivot block `blk` from its 4 x 4 block `pb` (row-major, lower part read; every lane
// of the calling warp computes them; lane 0 stores).
__device__ __forceinline__ void leaf_block_inverse(const double* pb, int blk, double* wdst, double* dsm, double* msm,
                                                   int lane) {
  double sd[16], d[4], m[6], w[16];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) sd[r * 4 + c] = (c <= r) ? pb[r * 4 + c] : 0.0;
  ldl4_inverse(sd, d, m, w);
  if (lane == 0) {
#pragma unroll
    for (int q = 0; q < 16; ++q) wdst[q] = w[q];
#pragma unroll
    for (int q = 0; q < 4; ++q) dsm[4 * blk + q] = d[q];
#pragma unroll
    for (int q = 0; q < 6; ++q) msm[blk * 6 + q] = m[q];
  }
}

// One level of the leaf's triangular inverse by recursive doubling: with Z = M^-1 known on the
// diagonal blocks of S tiles, every pair of them (tile rows b0 .. b0 + 2S - 1) gets its
// off-diagonal block from the inverse of a 2 x 2 block lower triangular matrix,
//   Z21 = -Z22 (M21 Z11),  M21 = N21,
// as 8 x 8 tile products (two fp64 MMAs each, the two k halves in separate accumulators).  The
// 8 S tiles of the level go to the 16 warps, their columns rotated so that every warp gets long
// and short sums alike.  T = M21 Z11 is stored in Z21's tiles, and Z21 is held in registers until
// every warp has read T.  Ends with a CTA barrier.
template <int S>
__device__ __forceinline__ void leaf_inverse_level(double* Zs, const double* Ns, int warp, int fg, int ft) {
  constexpr int kTiles = 8 * S;
  constexpr int kPer = (kTiles + kLT - 1) / kLT;
  auto tile = [&](int u, int& I, int& J, int& b0) {
    const int q = warp + kLT * u;
    const int p = q / (S * S), i = (q % (S * S)) / S, j = (q + 3 * u) % S;
    b0 = 2 * S * p;
    I = b0 + S + i;
    J = b0 + j;
    return q < kTiles;
  };
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    int I, J, b0;
    if (!tile(u, I, J, b0)) continue;
    double c0 = 0.0, c1 = 0.0, e0 = 0.0, e1 = 0.0;
#pragma unroll
    for (int k = 0; k < S; ++k) {
      const int K = b0 + k;  // T_IJ = sum_{K >= J} N_IK Z_KJ over the first block
      if (K >= J) {
        dmma_leaf(c0, c1, Ns[lt_idx(I, K, fg, ft)], Zs[lt_idx(K, J, ft, fg)]);
        dmma_leaf(e0, e1, Ns[lt_idx(I, K, fg, 4 + ft)], Zs[lt_idx(K, J, 4 + ft, fg)]);
      }
    }
    *reinterpret_cast<double2*>(&Zs[lt_idx(I, J, fg, 2 * ft)]) = make_double2(c0 + e0, c1 + e1);
  }
  __syncthreads();
  double2 z[kPer];
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    int I, J, b0;
    z[u] = make_double2(0.0, 0.0);
    if (!tile(u, I, J, b0)) continue;
    double c0 = 0.0, c1 = 0.0, e0 = 0.0, e1 = 0.0;
#pragma unroll
    for (int k = 0; k < S; ++k) {
      const int K = b0 + S + k;  // Z21_IJ = -sum_{K <= I} Z_IK T_KJ over the second block
      if (K <= I) {
        dmma_leaf(c0, c1, Zs[lt_idx(I, K, fg, ft)], Zs[lt_idx(K, J, ft, fg)]);
        dmma_leaf(e0, e1, Zs[lt_idx(I, K, fg, 4 + ft)], Zs[lt_idx(K, J, 4 + ft, fg)]);
      }
    }
    z[u] = make_double2(-(c0 + e0), -(c1 + e1));
  }
  __syncthreads();
#pragma unroll
  for (int u = 0; u < kPer; ++u) {
    int I, J, b0;
    if (tile(u, I, J, b0)) *reinterpret_cast<double2*>(&Zs[lt_idx(I, J, fg, 2 * ft)]) = z[u];
  }
  __syncthreads();
}

__global__ void __launch_bounds__(kLeafThreads, 1) chol_inv_leaf_kernel(const double* __restrict__ A, int64_t lda,
                                                                         double* __restrict__ X,
                                                                         double* __restrict__ XT, int64_t ldx,
                                                                         int* __restrict__ info, int diag_off) {
  pdl_wait();
  if (*info != 0) return;
  // the block lies inside the matrix (uniform over the CTA: no thread is left at a barrier)
  if (!HQ_IN_BOUNDS(diag_off >= 0 && diag_off + kLB <= ldx && kLB <= lda)) return;
  extern __shared__ __align__(16) double lsm[];
  double* Ssm = lsm;                 // S tiles (later Z = M^-1)
  double* Ysm = Ssm + kLTiles * 64;  // multiplier tiles N (later the output coefficients)
  double* wsm = Ysm + kLTiles * 64;  // W of the current and of the next block, 4 x 4 each
  double* dsm = wsm + 2 * 16;        // pivots
  double* msm = dsm + kLB;           // strict lower part of L_B^-1 per block (6 each)
  __shared__ int bad;
  const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
  const int fg = lane / 4, ft = lane % 4;

  double* pan = msm + (kLB / 4) * 6;  // [2][kLB][4]: the panel of the current and the next block
  const int I = warp;
  // N = 0 (the multipliers' tiles), S: tile row I in registers, lane (g = fg, t = ft) holding
  // elements (g, 2t) and (g, 2t + 1) of each tile (I, J), J <= I (zero above the diagonal)
  for (int e = tid; e < kLTiles * 64 / 2; e += kLeafThreads)
    reinterpret_cast<double2*>(Ysm)[e] = make_double2(0.0, 0.0);
  double2 sreg[kLT];
#pragma unroll
  for (int J = 0; J < kLT; ++J) {
    sreg[J] = make_double2(0.0, 0.0);
    if (J <= I) {
      const int r = 8 * I + fg, c = 8 * J + 2 * ft;
      const double2 v = *reinterpret_cast<const double2*>(A + static_cast<int64_t>(r) * lda + c);
      sreg[J] = make_double2(c <= r ? v.x : 0.0, c + 1 <= r ? v.y : 0.0);
    }
  }
  // the panel of pivot block 0 (tile column 0, columns 0..3): lanes t < 2 hold it
  if (ft < 2) *reinterpret_cast<double2*>(&pan[(8 * I + fg) * 4 + 2 * ft]) = sreg[0];
  if (tid == 0) bad = kLB;
  __syncthreads();
  if (warp == 0) leaf_block_inverse(pan, 0, wsm, dsm, msm, lane);
  __syncthreads();

  // block steps, fully unrolled (tile indices are then compile-time register indices)
#pragma unroll
  for (int kt = 0; kt < kLB / 4; ++kt) {
    const int JB = kt >> 1, h = kt & 1;
    const int J0 = JB + h;        // first tile row / column with an element beyond the pivot block
    const int lim = 4 * kt + 3;   // rows <= lim have no part in the update
    const double* pc = pan + (kt & 1) * kLB * 4;  // this block's panel P (rows x its 4 columns)
    if (I >= J0) {
      // -G_I = -P_I W: A = P_I (8 x 4, zero at rows <= lim), B = W padded to 4 x 8
      double a;
      {
        const double p = (8 * I + fg > lim) ? pc[(8 * I + fg) * 4 + ft] : 0.0;
        const double wv = (fg < 4) ? wsm[(kt & 1) * 16 + ft * 4 + fg] : 0.0;  // W[t][g]
        double g0 = 0.0, g1 = 0.0;
        dmma_leaf(g0, g1, p, wv);
        const int src = 4 * fg + (ft >> 1);  // lane holding G[g][t]
        const double x0 = __shfl_sync(0xffffffffu, g0, src), x1 = __shfl_sync(0xffffffffu, g1, src);
        a = -((ft & 1) ? x1 : x0);
      }
      // the multiplier block G_I (rows of tile I, the pivot block's 4 columns) -> N
      Ysm[lt_idx(I, JB, fg, 4 * h + ft)] = -a;
      // S[I][J] -= G_I P_J^T for J0 <= J <= I, in registers; the pivot block's own columns stay
#pragma unroll
      for (int J = J0; J < kLT; ++J) {
        if (J <= I) {
          const double b = (8 * J + fg > lim) ? pc[(8 * J + fg) * 4 + ft] : 0.0;  // P_J[g][t]
          double2 cv = sreg[J];
          dmma_leaf(cv.x, cv.y, a, b);
          if (!(J == JB && h == 0 && ft < 2)) sreg[J] = cv;
        }
      }
    }
    if (kt + 1 < kLB / 4) {
      // publish the next block's panel (tile column JBn, columns 4 hn .. 4 hn + 3), then the warp
      // owning its diagonal tile computes its W while the others go on
      const int JBn = (kt + 1) >> 1, hn = (kt + 1) & 1;
      double* pn = pan + ((kt + 1) & 1) * kLB * 4;
      if (I >= JBn && (ft >> 1) == hn)
        *reinterpret_cast<double2*>(&pn[(8 * I + fg) * 4 + 2 * (ft - 2 * hn)]) = sreg[JBn];
      if (I == JBn) {
        __syncwarp();
        leaf_block_inverse(pn + (8 * JBn + 4 * hn) * 4, kt + 1, wsm + ((kt + 1) & 1) * 16, dsm, msm, lane);
      }
    }
    __syncthreads();
  }
  // pivots; the first bad one fails the leaf
  if (tid < kLB) {
    const double dd = dsm[tid];
    if (!(dd >= 2.2250738585072014e-308) || !isfinite(dd)) atomicMin(&bad, tid);  // not normal, > 0
  }
  __syncthreads();
  if (bad < kLB) {
    if (tid == 0) atomicCAS(info, 0, diag_off + bad + 1);
    return;
  }
  // Z = (I + N)^-1, the inverse of the block unit lower triangular factor (S is no longer needed
  // and takes Z): the diagonal tiles Z_JJ = I - N_JJ (N_JJ is the diagonal tile's lower-left
  // 4 x 4 block, N_JJ^2 = 0), then the off-diagonal blocks by recursive doubling over blocks of
  // 1, 2, 4 and 8 tile rows.
  {
    const int J = warp;
    {
      double2 z;
      const int c0 = 2 * ft;
      const double n0 = (fg >= 4 && c0 < 4) ? Ysm[lt_idx(J, J, fg, c0)] : 0.0;
      const double n1 = (fg >= 4 && c0 + 1 < 4) ? Ysm[lt_idx(J, J, fg, c0 + 1)] : 0.0;
      z.x = (fg == c0 ? 1.0 : 0.0) - n0;
      z.y = (fg == c0 + 1 ? 1.0 : 0.0) - n1;
      *reinterpret_cast<double2*>(&Ssm[lt_idx(J, J, fg, c0)]) = z;
    }
  }
  __syncthreads();
  leaf_inverse_level<1>(Ssm, Ysm, warp, fg, ft);
  leaf_inverse_level<2>(Ssm, Ysm, warp, fg, ft);
  leaf_inverse_level<4>(Ssm, Ysm, warp, fg, ft);
  leaf_inverse_level<8>(Ssm, Ysm, warp, fg, ft);
  // X tile (I, J) = C_I Z tile (I, J), with C_I = diag(D_b^-1/2 L_b^-1, D_b'^-1/2 L_b'^-1) the
  // block-diagonal 8 x 8 matrix of tile row I's two pivot blocks (two fp64 MMAs per tile);
  // written to X (row-major) and X^T straight from the fragments.  Elements above the diagonal
  // come out zero, as X and X^T already hold there.
  pdl_launch_dependents();  // the successor may be scheduled during the output phase
  double* csm = Ysm;  // (N is no longer needed) row i: the 4 coefficients of its block's row
  {
    const int i = tid;  // row i of the leaf, block i / 4, row r = i % 4 of that block
    if (i < kLB) {
      const double dl = dsm[i];
      double mv[6];
#pragma unroll
      for (int q = 0; q < 6; ++q) mv[q] = msm[(i / 4) * 6 + q];
      const int r = i % 4;
      const double sc = 1.0 / sqrt(dl);
      // row r of L_b^-1: (m10 m20 m30 m21 m31 m32) = M[1][0] M[2][0] M[3][0] M[2][1] M[3][1] M[3][2]
      const double c0 = r == 0 ? 1.0 : (r == 1 ? mv[0] : (r == 2 ? mv[1] : mv[2]));
      const double c1 = r == 1 ? 1.0 : (r == 2 ? mv[3] : (r == 3 ? mv[4] : 0.0));
      const double c2 = r == 2 ? 1.0 : (r == 3 ? mv[5] : 0.0);
      const double c3 = r == 3 ? 1.0 : 0.0;
      csm[i * 4 + 0] = c0 * sc;
      csm[i * 4 + 1] = c1 * sc;
      csm[i * 4 + 2] = c2 * sc;
      csm[i * 4 + 3] = c3 * sc;
    }
    __syncthreads();
  }
  for (int T = warp; T < kLTiles; T += kLT) {
    int TI = static_cast<int>((sqrtf(8.f * T + 1.f) - 1.f) * 0.5f);
    if (TI * (TI + 1) / 2 > T) --TI;
    if ((TI + 1) * (TI + 2) / 2 <= T) ++TI;
    const int TJ = T - TI * (TI + 1) / 2;
    // k = 0..3 (rows 0..3 of the Y tile) feed output rows 0..3; k = 4..7 feed rows 4..7
    const double a0 = (fg < 4) ? csm[(8 * TI + fg) * 4 + ft] : 0.0;
    const double a1 = (fg >= 4) ? csm[(8 * TI + fg) * 4 + ft] : 0.0;
    const double b0 = Ssm[lt_idx(TI, TJ, ft, fg)];      // Z[8TI + t][8TJ + g]
    const double b1 = Ssm[lt_idx(TI, TJ, 4 + ft, fg)];  // Z[8TI + 4 + t][8TJ + g]
    double x0 = 0.0, x1 = 0.0;
    dmma_leaf(x0, x1, a0, b0);
    dmma_leaf(x0, x1, a1, b1);
    const int i = 8 * TI + fg, j = 8 * TJ + 2 * ft;
    *reinterpret_cast<double2*>(&X[static_cast<int64_t>(i) * ldx + j]) = make_double2(x0, x1);
    XT[static_cast<int64_t>(j) * ldx + i] = x0;
    XT[static_cast<int64_t>(j + 1) * ldx + i] = x1;
  }
}

// X and X^T := 0 on the diagonal kLeaf x kLeaf blocks (one CTA per block).
__global__ void __launch_bounds__(256) zero_diag_blocks_kernel(double* __restrict__ X, double* __restrict__ XT,
                                                               int64_t K) {
  const int64_t d0 = static_cast<int64_t>(blockIdx.x) * kLeaf;
  for (int e = threadIdx.x; e < kLeaf * kLeaf / 2; e += blockDim.x) {
    const int r = e / (kLeaf / 2), c = 2 * (e % (kLeaf / 2));
    const int64_t off = (d0 + r) * K + d0 + c;
    *reinterpret_cast<double2*>(X + off) = make_double2(0.0, 0.0);
    *reinterpret_cast<double2*>(XT + off) = make_double2(0.0, 0.0);
  }
}

// ------------------------------------------------------------------------- 3b. recursion

// A second stream per (host thread, device) for the work off the recursion's critical path,
// and a pool of events for the dependencies between the two streams (created on first use,
// kept for the thread's lifetime).
struct SideStream {
  cudaStream_t s2 = nullptr;
  std::vector<cudaEvent_t> ev;
  size_t used = 0;
  ~SideStream() {
    for (cudaEvent_t e : ev) cudaEventDestroy(e);
    if (s2 != nullptr) cudaStreamDestroy(s2);
  }
};

static hq_status side_stream(SideStream** out) {
  constexpr int kMaxDevices = 64;
  thread_local SideStream pool[kMaxDevices];
  int dev = -1;
  HQ_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return HQ_ERR_UNSUPPORTED;
  SideStream& ss = pool[dev];
  if (ss.s2 == nullptr) HQ_CUDA_TRY(cudaStreamCreateWithFlags(&ss.s2, cudaStreamNonBlocking));
  ss.used = 0;
  *out = &ss;
  return HQ_OK;
}

struct FactorCtx {
  double* A;
  double* X;
  double* XT;
  double* tmp_end;  // end of the temporaries region
  int64_t K;
  int* info;
  int* status;
  cudaStream_t s;   // the caller's stream: the critical path
  SideStream* side;  // s2: Y^T products and transposes
  uint8_t* slices[2];  // int8 slices of the large products' operands: [0] for s, [1] for s2
  size_t slices_bytes;  // each
};

// Products with all three dimensions at least this large run on the int8 tensor cores
// (gemm_i8x.cu), the rest on the fp64 tensor cores (gemm_f64.cu).
constexpr int64_t kI8xMinDim = 1024;

static bool use_i8x(int64_t M, int64_t N, int64_t Kred) {
  return M >= kI8xMinDim && N >= kI8xMinDim && Kred >= kI8xMinDim && Kred <= kI8xMaxKred;
}

size_t factor_slice_bytes(int64_t K) {
  const int64_t n1 = (K / kLeaf / 2) * kLeaf, n2 = K - n1;
  const int64_t dims[4][3] = {{n2, n1, n1}, {n1, n2, n1}, {n2, n2, n1}, {n2, n1, n2}};
  size_t b = 0;
  for (const auto& d : dims)
    if (use_i8x(d[0], d[1], d[2])) b = std::max(b, i8x_scratch_bytes(d[0], d[1], d[2]));
  return round_up(b, 256);  // the second stream's half starts right after the first
}

// `from` -> `to`: work enqueued on `to` from now on waits for everything enqueued on `from` so far.
static hq_status stream_dep(SideStream* ss, cudaStream_t from, cudaStream_t to) {
  if (ss->used == ss->ev.size()) {
    cudaEvent_t e;
    HQ_CUDA_TRY(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
    ss->ev.push_back(e);
  }
  cudaEvent_t e = ss->ev[ss->used++];
  HQ_CUDA_TRY(cudaEventRecord(e, from));
  HQ_CUDA_TRY(cudaStreamWaitEvent(to, e, 0));
  return HQ_OK;
}

// `scratch` (up to the end of the temporaries; NULL: no split) receives split-K partial tiles.
static hq_status gemm(const FactorCtx& c, cudaStream_t s, double* scratch, double* C, int64_t ldc, int M, int N,
                      int Kred, const double* A, int64_t lda, const double* B, int64_t ldb, double alpha,
                      double beta, bool lower, int tri, double* Ct = nullptr, int64_t ldct = 0) {
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
  g.scratch_elems = scratch == nullptr ? 0 : c.tmp_end - scratch;
  g.skip = c.info;
  g.status = c.status;
  g.Ct = Ct;
  g.ldct = ldct;
  if (use_i8x(M, N, Kred)) {
    uint8_t* sl = c.slices[s == c.s ? 0 : 1];
    if (sl != nullptr && i8x_scratch_bytes(M, N, Kred) <= c.slices_bytes) return i8x_gemm(g, sl, c.slices_bytes, s);
  }
  return f64_gemm(g, s);
}

// X = L^-1 and X^T for the n x n block of A at (off, off); `tmp` has room for the temporaries
// of this level and all levels below (2 * n2 * n1 here, about a quarter of that per level below).
// Critical path on c.s: left half, T, the Schur update, right half, X21 (with X21^T).  Y^T (needs
// only T and the left half) runs on the side stream, overlapping the right half's leaves and
// small products; it takes no split-K scratch (the region beyond this level's temporaries
// belongs to the right half meanwhile).
static hq_status chol_inv(const FactorCtx& c, int64_t off, int64_t n, double* tmp) {
  const int64_t K = c.K;
  if (n == kLeaf) {
    const int tm = timer_start(kTimeLeaf, c.s);
    HQ_LAUNCH_CHAINED(launch_chained(chol_inv_leaf_kernel, dim3(1), dim3(kLeafThreads), kLeafSmem, c.s,
                                     c.A + off * K + off, K, c.X + off * K + off, c.XT + off * K + off, K, c.info,
                                     static_cast<int>(off)));
    timer_stop(tm, 2.0 * kLeaf * kLeaf * kLeaf / 3.0, c.s);  // Cholesky n^3/3 + triangular inverse n^3/3
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
  cudaStream_t s2 = timing_serialized() ? c.s : c.side->s2;
  hq_status st = chol_inv(c, off, n1, rest);
  if (st != HQ_OK) return st;
  st = gemm(c, c.s, rest, T, n1, in2, in1, in1, A21, K, X11, K, 1.0, 0.0, false, kTriBLower);  // T = A21 X11^T
  if (st != HQ_OK) return st;
  st = stream_dep(c.side, c.s, s2);
  if (st != HQ_OK) return st;
  st = gemm(c, s2, nullptr, YT, n2, in1, in2, in1, XT11, K, T, n1, 1.0, 0.0, false, kTriAUpper);  // Y^T = X11^T T^T
  if (st != HQ_OK) return st;
  st = gemm(c, c.s, rest, A22, K, in2, in2, in1, T, n1, T, n1, -1.0, 1.0, true, kTriNone);       // A22 -= T T^T
  if (st != HQ_OK) return st;
  st = chol_inv(c, off + n1, n2, rest);
  if (st != HQ_OK) return st;
  st = stream_dep(c.side, s2, c.s);  // Y^T
  if (st != HQ_OK) return st;
  // X21 = -X22 Y, and its transpose into X^T
  return gemm(c, c.s, rest, X21, K, in2, in1, in2, X22, K, YT, n2, -1.0, 0.0, false, kTriALower, XT12, K);
}

// ------------------------------------------------------------------------- 4. U, U^T

// U[j][c] = X[K-1-j][K-1-c] and U^T[j][c] = X^T[K-1-j][K-1-c], rounded to fp32: 180-degree
// rotations (U upper, U^T lower, zeros elsewhere because X and X^T hold zeros there).
// With `scaled`, U^T[j][c] is divided by U[c][c] in fp64 first (U'^T, U' = diag(U)^-1 U, the
// form the GPTQ sweep and its lazy updates use).  With Ut_hi != NULL, also the strict lower part
// of the result as a tf32 part (low 13 mantissa bits cleared) plus the exact fp32 remainder, the
// operands of the 3xTF32 lazy updates; with Ut == NULL as well, only that split part is produced.
__global__ void rotate_kernel(const double* __restrict__ X, const double* __restrict__ XT, int64_t K,
                              float* __restrict__ U, float* __restrict__ Ut, float* __restrict__ Ut_hi,
                              float* __restrict__ Ut_lo, bool scaled, const int* __restrict__ info) {
  if (*info != 0) return;
  const int64_t n = K * K;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < n;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t src = n - 1 - e;  // (K-1-j)*K + (K-1-c) for e = j*K + c
    // with Ut == NULL only the strict lower split is wanted: the rest is neither read nor written
    if (Ut == nullptr && e % K >= e / K) continue;
    if (U != nullptr) U[e] = static_cast<float>(X[src]);
    double ut64 = XT[src];  // U^T[e / K][e % K] = U[e % K][e / K]
    if (scaled) ut64 /= X[(K - 1 - e % K) * (K + 1)];  // divided by U[e % K][e % K]
    const float ut = static_cast<float>(ut64);
    if (Ut != nullptr) Ut[e] = ut;
    if (Ut_hi != nullptr && e % K < e / K) {
      const float hi = __uint_as_float(__float_as_uint(ut) & 0xFFFFE000u);
      Ut_hi[e] = hi;
      Ut_lo[e] = ut - hi;
    }
  }
}

// The diagonal blocks of U' = diag(U)^-1 U in the GPTQ sweep's packed order
// (sweep_upack_offset), U[j][c] = X[K-1-j][K-1-c].
__global__ void sweep_pack_kernel(const double* __restrict__ X, int64_t K, float* __restrict__ Up,
                                  const int* __restrict__ info) {
  if (*info != 0) return;
  constexpr int B = kSweepBlk;
  const int64_t total = K * B;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = e / (B * B);
    const int r = static_cast<int>(e % (B * B));
    const int j = r / B, l = (r % B) / 8, m = r % 8;
    const int c = 16 * (j / 16 + m) + l;
    float v = 0.f;
    if (c > j && c < B) {
      const int64_t gj = b * B + j, gc = b * B + c;
      v = static_cast<float>(X[(K - 1 - gj) * K + (K - 1 - gc)] / X[(K - 1 - gj) * (K + 1)]);
    }
    if (HQ_IN_BOUNDS(b < K / B)) Up[b * B * B + sweep_upack_offset(j, l, m)] = v;
  }
}

// The bands of U' (kSweepBand): Ub[b][k][c] = U'[b B + k][(b + 1) B + c], the same fp64 quotient
// rounded once as in the packed blocks and in U'^T; 0 past column K - 1.
__global__ void sweep_band_kernel(const double* __restrict__ X, int64_t K, float* __restrict__ Ub,
                                  const int* __restrict__ info) {
  if (*info != 0) return;
  constexpr int B = kSweepBlk;
  const int64_t total = K * kSweepBand;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < total;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t b = e / (static_cast<int64_t>(B) * kSweepBand);
    const int r = static_cast<int>(e % (static_cast<int64_t>(B) * kSweepBand));
    const int64_t gj = b * B + r / kSweepBand, gc = (b + 1) * B + r % kSweepBand;
    float v = 0.f;
    if (gc < K) v = static_cast<float>(X[(K - 1 - gj) * K + (K - 1 - gc)] / X[(K - 1 - gj) * (K + 1)]);
    Ub[e] = v;
  }
}

// ------------------------------------------------------------------------- driver

hq_status launch_factor(const float* H, int64_t K, float damp, double* A, double* X, double* XT, double* T,
                        uint8_t* slices, double* lam, int* info, int* status, bool sweep_form, float* Ut, float* U,
                        float* Ut_hi, float* Ut_lo, cudaStream_t s) {
  if (K % kLeaf != 0 || K % kSweepBlk != 0) return HQ_ERR_UNSUPPORTED;
  HQ_CUDA_TRY(cudaFuncSetAttribute(chol_inv_leaf_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   static_cast<int>(kLeafSmem)));
  damp_stats_kernel<<<1, 1024, 0, s>>>(H, K, damp, lam, info);
  HQ_LAUNCH_CHECK();
  {
    const int64_t nb = ceil_div(K, 32);
    reverse_damp_kernel<<<static_cast<unsigned>(nb * (nb + 1) / 2), 256, 0, s>>>(H, K, lam, A, info);
    HQ_LAUNCH_CHECK();
  }
  const bool split_only = sweep_form && Ut == nullptr;
  if (split_only) {
    // the products' triangular tiles and the leaves read zeros only inside the diagonal leaf
    // blocks, and nothing downstream reads X or X^T outside their triangles
    zero_diag_blocks_kernel<<<static_cast<unsigned>(K / kLeaf), 256, 0, s>>>(X, XT, K);
    HQ_LAUNCH_CHECK();
  } else {
    HQ_CUDA_TRY(cudaMemsetAsync(X, 0, static_cast<size_t>(K) * K * sizeof(double), s));
    HQ_CUDA_TRY(cudaMemsetAsync(XT, 0, static_cast<size_t>(K) * K * sizeof(double), s));
  }
  SideStream* side = nullptr;
  hq_status st = side_stream(&side);
  if (st != HQ_OK) return st;
  const size_t sb = factor_slice_bytes(K);
  FactorCtx c{A, X, XT, T + K * K, K, info, status, s, side, {nullptr, nullptr}, sb};
  if (slices != nullptr && sb > 0) {
    c.slices[0] = slices;
    c.slices[1] = slices + sb;
  }
  st = stream_dep(side, s, side->s2);  // the side stream starts after everything before this call
  if (st != HQ_OK) return st;
  st = chol_inv(c, 0, K, T);
  // the caller's stream waits for the side stream's last work, also when enqueueing failed midway
  const hq_status st_join = stream_dep(side, side->s2, s);
  if (st != HQ_OK) return st;
  if (st_join != HQ_OK) return st_join;
  // A and the temporaries are dead now: the outputs may overlay them
  const int64_t grid = ceil_div(K * K, 4 * 256) < 148 * 32 ? ceil_div(K * K, 4 * 256) : 148 * 32;
  rotate_kernel<<<static_cast<unsigned>(grid), 256, 0, s>>>(X, XT, K, sweep_form ? nullptr : U, Ut, Ut_hi, Ut_lo,
                                                            sweep_form, info);
  HQ_LAUNCH_CHECK();
  if (sweep_form && U != nullptr) {
    const int64_t pg = ceil_div(K * kSweepBlk, 256) < 148 * 16 ? ceil_div(K * kSweepBlk, 256) : 148 * 16;
    sweep_pack_kernel<<<static_cast<unsigned>(pg), 256, 0, s>>>(X, K, U, info);
    HQ_LAUNCH_CHECK();
    const int64_t bg = ceil_div(K * kSweepBand, 256) < 148 * 16 ? ceil_div(K * kSweepBand, 256) : 148 * 16;
    sweep_band_kernel<<<static_cast<unsigned>(bg), 256, 0, s>>>(X, K, U + K * kSweepBlk, info);
    HQ_LAUNCH_CHECK();
  }
  return HQ_OK;
}

}  // namespace hq
