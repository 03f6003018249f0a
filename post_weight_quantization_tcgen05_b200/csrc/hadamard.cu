// Hadamard rotation ahead of GPTQ (ork-driver wiki "Exp 2026-08-18 GPTQ Int4", experiment
// summary: GPTQ "composes with Hadamard = QuaRot: rotate then GPTQ").
//
// R = D blockdiag(M_B, ..., M_B) with D = diag(s) (s in {-1, +1}^K, drawn by the caller) and
// M_B = Hadamard_B / sqrt(B) the orthonormal Walsh-Hadamard matrix of order B (a power of two),
// Hadamard_B[i][j] = (-1)^popcount(i & j) (Sylvester).  R is orthogonal, so with W' = W R and
// X' = X R the layer's output is unchanged (W x = W' (R^T x)) and the calibration Hessian of the
// rotated activations is H' = R^T H R.  Both are computed by fast Walsh-Hadamard transforms
// (log2 B butterfly stages):
//   rows:    out[r][b B + j] = sum_i (s[b B + i] A[r][b B + i]) M_B[i][j]     (A R)
//   columns: A[b B + i][c] <- sum_k M_B[k][i] s[b B + k] A[b B + k][c]         (R^T A)
// W R is one read and one write of W.  Since R is block diagonal, block (bi, bj) of H' is
// M D_bi H_bi,bj D_bj M and depends on that block of H alone; H' is symmetric, so only the lower
// blocks are transformed: pass 1 writes G = R^T H on them (columns, H's lower triangle read), pass 2
// turns them into H' = G R in place (rows) and writes each off-diagonal block's transpose into the
// upper blocks.  All of it is HBM-bound.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.cuh"

namespace hq {

constexpr int kHadMaxB = 1024;

// ---------------------------------------------------------------------------------------------
// Blocks of 32 and more (the fast path).  The unnormalised Walsh-Hadamard transform of length B
// is log2 B butterfly stages (v[i], v[i + h]) -> (v[i] + v[i + h], v[i] - v[i + h]) over the bits h
// of the index, in any order; here the index bits are split between registers and lanes (or
// warps), so no stage needs a barrier.
// ---------------------------------------------------------------------------------------------

// Butterflies over every bit of the register index of v[0 .. N).
template <int N>
__device__ __forceinline__ void reg_fwht(float (&v)[N]) {
#pragma unroll
  for (int h = 1; h < N; h <<= 1)
#pragma unroll
    for (int i = 0; i < N; ++i)
      if ((i & h) == 0) {
        const float a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
}

// Length-32E transform held by one warp, element lane * E + i in v[i] of that lane: the low
// log2 E bits in registers, the five lane bits by shuffles.
template <int E>
__device__ __forceinline__ void warp_fwht(float (&v)[E], int lane) {
  reg_fwht<E>(v);
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
    const bool upper = (lane & m) != 0;
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const float o = __shfl_xor_sync(0xffffffffu, v[i], m);
      v[i] = upper ? o - v[i] : v[i] + o;
    }
  }
}

template <int E>
__device__ __forceinline__ void load_vec(const float* p, float (&v)[E]) {
  if constexpr (E % 4 == 0) {
#pragma unroll
    for (int q = 0; q < E / 4; ++q) {
      const float4 x = reinterpret_cast<const float4*>(p)[q];
      v[4 * q] = x.x; v[4 * q + 1] = x.y; v[4 * q + 2] = x.z; v[4 * q + 3] = x.w;
    }
  } else if constexpr (E == 2) {
    const float2 x = *reinterpret_cast<const float2*>(p);
    v[0] = x.x; v[1] = x.y;
  } else {
    v[0] = *p;
  }
}

template <int E>
__device__ __forceinline__ void load_vec(const __nv_bfloat16* p, float (&v)[E]) {
  if constexpr (E % 8 == 0) {
#pragma unroll
    for (int q = 0; q < E / 8; ++q) {
      const uint4 x = reinterpret_cast<const uint4*>(p)[q];
      const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        v[8 * q + 2 * k] = __uint_as_float(w[k] << 16);
        v[8 * q + 2 * k + 1] = __uint_as_float(w[k] & 0xFFFF0000u);
      }
    }
  } else if constexpr (E == 4) {
    const uint2 x = *reinterpret_cast<const uint2*>(p);
    v[0] = __uint_as_float(x.x << 16); v[1] = __uint_as_float(x.x & 0xFFFF0000u);
    v[2] = __uint_as_float(x.y << 16); v[3] = __uint_as_float(x.y & 0xFFFF0000u);
  } else if constexpr (E == 2) {
    const uint32_t x = *reinterpret_cast<const uint32_t*>(p);
    v[0] = __uint_as_float(x << 16); v[1] = __uint_as_float(x & 0xFFFF0000u);
  } else {
    v[0] = __bfloat162float(*p);
  }
}

template <int E>
__device__ __forceinline__ void store_vec(float* p, const float (&v)[E]) {
  if constexpr (E % 4 == 0) {
#pragma unroll
    for (int q = 0; q < E / 4; ++q)
      reinterpret_cast<float4*>(p)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  } else if constexpr (E == 2) {
    *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
  } else {
    *p = v[0];
  }
}

// out = A R for a row-major [rows, K] matrix seen as rows * K / B contiguous blocks of B = 32E
// elements; block q starts at element q B and its signs at (q B) mod K.  One warp per block, U
// blocks in flight per warp, grid-stride.  out may be A (each warp reads its blocks whole before
// writing them).
template <typename TA, int E, int U>
__global__ void __launch_bounds__(256) hadamard_rows_warp_kernel(const TA* A, int64_t nblk, int64_t K,
                                                                 const float* __restrict__ s, float* out) {
  constexpr int B = 32 * E;
  const int lane = threadIdx.x & 31;
  const int64_t warps = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  const float scale = rsqrtf(static_cast<float>(B));
  for (int64_t q0 = (static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5)) * U; q0 < nblk;
       q0 += warps * U) {
    float v[U][E];
#pragma unroll
    for (int u = 0; u < U; ++u)
      if (q0 + u < nblk) load_vec<E>(A + (q0 + u) * B + lane * E, v[u]);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (q0 + u >= nblk) break;  // uniform over the warp
      float sg[E];
      load_vec<E>(s + ((q0 + u) * B) % K + lane * E, sg);
#pragma unroll
      for (int i = 0; i < E; ++i) v[u][i] *= sg[i];
      warp_fwht<E>(v[u], lane);
#pragma unroll
      for (int i = 0; i < E; ++i) v[u][i] *= scale;
      store_vec<E>(out + (q0 + u) * B + lane * E, v[u]);
    }
  }
}

// Block pair (bi, bj), bi >= bj, of the lower block triangle from its index u = bi (bi + 1) / 2 + bj.
__device__ __forceinline__ void lower_block_pair(int64_t u, int64_t& bi, int64_t& bj) {
  bi = static_cast<int64_t>((sqrt(8.0 * static_cast<double>(u) + 1.0) - 1.0) * 0.5);
  while (bi * (bi + 1) / 2 > u) --bi;
  while ((bi + 1) * (bi + 2) / 2 <= u) ++bi;
  bj = u - bi * (bi + 1) / 2;
}

// Hessian pass 1, G = R^T H on the lower blocks: for bi >= bj and the 32 columns c0 .. c0 + 31 of
// block column bj,  G[bi B + i][c] = (1/sqrt B) sum_k Hadamard_B[k][i] s[bi B + k] H[bi B + k][c],
// H read as the symmetric matrix of its lower triangle (inside a diagonal block the upper part is
// read transposed, coalesced).  One CTA of B = 32W threads per (block pair, 32-column strip): the
// strip goes through shared memory [B][33]; thread (w, lane) transforms rows 32w .. 32w + 31 of
// column `lane` in registers (the five low index bits), then, after one barrier, rows m + 32w' of
// one column for the W values w' (the high bits).
template <int W>
__global__ void __launch_bounds__(32 * W) hadamard_cols_lower_kernel(const float* __restrict__ H, int64_t K,
                                                                     const float* __restrict__ s,
                                                                     float* __restrict__ G) {
  constexpr int B = 32 * W;
  constexpr int LD = 33;
  extern __shared__ float t[];  // [B][LD]
  int64_t bi, bj;
  lower_block_pair(blockIdx.x / W, bi, bj);
  const int64_t r0 = bi * B, c0 = bj * B + 32 * (blockIdx.x % W);
  const bool diag = bi == bj;
  const int tid = threadIdx.x, lane = tid & 31, w = tid >> 5;
  constexpr int LB = W >= 16 ? 8 : 32;  // loads in flight per thread (registers at 512+ threads)
#pragma unroll
  for (int m0 = 0; m0 < 32; m0 += LB) {
    float x[LB];
#pragma unroll
    for (int m = 0; m < LB; ++m) {
      const int64_t i = w + W * (m0 + m);
      x[m] = (!diag || c0 + lane <= r0 + i) ? H[(r0 + i) * K + c0 + lane] : 0.f;
    }
#pragma unroll
    for (int m = 0; m < LB; ++m) {
      const int i = w + W * (m0 + m);
      if (!diag || c0 + lane <= r0 + i) t[i * LD + lane] = x[m];
    }
  }
  if (diag) {  // (r0 + tid, c0 + k) above the diagonal = H[c0 + k][r0 + tid]
#pragma unroll
    for (int k0 = 0; k0 < 32; k0 += LB) {
      float x[LB];
#pragma unroll
      for (int k = 0; k < LB; ++k) x[k] = (c0 + k0 + k > r0 + tid) ? H[(c0 + k0 + k) * K + r0 + tid] : 0.f;
#pragma unroll
      for (int k = 0; k < LB; ++k)
        if (c0 + k0 + k > r0 + tid) t[tid * LD + k0 + k] = x[k];
    }
  }
  __syncthreads();
  const float scale = rsqrtf(static_cast<float>(B));
  float v[32];
#pragma unroll
  for (int m = 0; m < 32; ++m) v[m] = t[(32 * w + m) * LD + lane] * s[r0 + 32 * w + m];
  reg_fwht<32>(v);
  if constexpr (W == 1) {
#pragma unroll
    for (int m = 0; m < 32; ++m)
      if (HQ_IN_BOUNDS(r0 + m < K && c0 + lane < K)) G[(r0 + m) * K + c0 + lane] = v[m] * scale;
  } else {
#pragma unroll
    for (int m = 0; m < 32; ++m) t[(32 * w + m) * LD + lane] = v[m];  // the elements this thread read
    __syncthreads();
#pragma unroll
    for (int g = 0; g < 32 / W; ++g) {
      const int m = w * (32 / W) + g;
      float u[W];
#pragma unroll
      for (int w2 = 0; w2 < W; ++w2) u[w2] = t[(32 * w2 + m) * LD + lane];
      reg_fwht<W>(u);
#pragma unroll
      for (int w2 = 0; w2 < W; ++w2)
        if (HQ_IN_BOUNDS(r0 + 32 * w2 + m < K && c0 + lane < K)) G[(r0 + 32 * w2 + m) * K + c0 + lane] = u[w2] * scale;
    }
  }
}

// Hessian pass 2, in place on G: H'[r][bj B + j] = (1/sqrt B) sum_k G[r][bj B + k] s[bj B + k]
// Hadamard_B[k][j] for the 32 rows r0 .. r0 + 31 of block row bi and block column bj <= bi, written
// at (r, bj B + j) and, off the diagonal, at (bj B + j, r) as well (H' is symmetric; the upper
// blocks are read by no CTA of this pass).  One CTA of 8 warps per (block pair, 32-row strip), a
// warp per row (warp_fwht); the transposed copy goes through shared memory [32][LD], column j at
// j + j / 32 so that both the row writes and the column reads are free of bank conflicts.
template <int E, int R>
__global__ void __launch_bounds__(256) hadamard_rows_mirror_kernel(float* G, int64_t K, const float* __restrict__ s) {
  constexpr int B = 32 * E;
  constexpr int LD = (B + B / 32) | 1;
  extern __shared__ float t[];  // [32][LD]
  int64_t bi, bj;
  lower_block_pair(blockIdx.x / E, bi, bj);  // B / 32 = E strips of 32 rows per block row
  const int64_t r0 = bi * B + 32 * (blockIdx.x % E), cb = bj * B;
  const bool diag = bi == bj;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const float scale = rsqrtf(static_cast<float>(B));
  float sg[E];
  load_vec<E>(s + cb + lane * E, sg);
#pragma unroll
  for (int k0 = 0; k0 < 4; k0 += R) {  // rows w + 8k, R of them in flight
    float v[R][E];
#pragma unroll
    for (int k = 0; k < R; ++k) load_vec<E>(G + (r0 + w + 8 * (k0 + k)) * K + cb + lane * E, v[k]);
#pragma unroll
    for (int k = 0; k < R; ++k) {
      const int rl = w + 8 * (k0 + k);
#pragma unroll
      for (int i = 0; i < E; ++i) v[k][i] *= sg[i];
      warp_fwht<E>(v[k], lane);
#pragma unroll
      for (int i = 0; i < E; ++i) v[k][i] *= scale;
      store_vec<E>(G + (r0 + rl) * K + cb + lane * E, v[k]);
      if (!diag) {
#pragma unroll
        for (int i = 0; i < E; ++i) {
          const int j = lane * E + i;
          t[rl * LD + j + (j >> 5)] = v[k][i];
        }
      }
    }
  }
  if (diag) return;  // uniform over the CTA
  __syncthreads();
  for (int e = threadIdx.x; e < 32 * B; e += blockDim.x) {
    const int j = e >> 5, rl = e & 31;
    if (HQ_IN_BOUNDS(cb + j < K && r0 + rl < K)) G[(cb + j) * K + r0 + rl] = t[rl * LD + j + (j >> 5)];
  }
}

// ---------------------------------------------------------------------------------------------
// Blocks of 2 .. 16: one CTA per transform through shared memory (simple, for small blocks).
// ---------------------------------------------------------------------------------------------

// In-place fast Walsh-Hadamard transform of v[0 .. B) in shared memory (unnormalised), by the
// block's threads.
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
  int64_t bi, bj;
  lower_block_pair(blockIdx.x, bi, bj);
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

// ---------------------------------------------------------------------------------------------
// Launchers
// ---------------------------------------------------------------------------------------------

bool hadamard_shape_ok(int64_t K, int64_t B) {
  return B >= 2 && B <= kHadMaxB && (B & (B - 1)) == 0 && K >= B && K % B == 0 && K <= (int64_t(1) << 30);
}

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int hadamard_sms() {
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  return sms;
}

template <typename TA, int E>
hq_status rows_warp(const TA* A, int64_t rows, int64_t K, const float* s, float* out, cudaStream_t st) {
  constexpr int U = E <= 8 ? 4 : (E == 16 ? 2 : 1);
  const int64_t nblk = rows * (K / (32 * E));
  const int64_t ctas = ceil_div(ceil_div(nblk, int64_t(U)), int64_t(8));
  const int64_t cap = static_cast<int64_t>(hadamard_sms()) * 8;
  hadamard_rows_warp_kernel<TA, E, U><<<static_cast<unsigned>(ctas < cap ? ctas : cap), 256, 0, st>>>(A, nblk, K, s,
                                                                                                       out);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

template <typename TA>
hq_status rows_warp_dispatch(const TA* A, int64_t rows, int64_t K, int B, const float* s, float* out,
                             cudaStream_t st) {
  switch (B) {
    case 32: return rows_warp<TA, 1>(A, rows, K, s, out, st);
    case 64: return rows_warp<TA, 2>(A, rows, K, s, out, st);
    case 128: return rows_warp<TA, 4>(A, rows, K, s, out, st);
    case 256: return rows_warp<TA, 8>(A, rows, K, s, out, st);
    case 512: return rows_warp<TA, 16>(A, rows, K, s, out, st);
    case 1024: return rows_warp<TA, 32>(A, rows, K, s, out, st);
    default: return HQ_ERR_UNSUPPORTED;
  }
}

template <int W>
hq_status cols_lower(const float* H, int64_t K, const float* s, float* G, cudaStream_t st) {
  constexpr int B = 32 * W;
  const int64_t nb = K / B;
  const int64_t ctas = nb * (nb + 1) / 2 * W;
  if (ctas > 0x7FFFFFFF) return HQ_ERR_UNSUPPORTED;
  const size_t smem = static_cast<size_t>(B) * 33 * sizeof(float);
  if (smem > 48 * 1024)
    HQ_CUDA_TRY(cudaFuncSetAttribute(hadamard_cols_lower_kernel<W>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem)));
  hadamard_cols_lower_kernel<W><<<static_cast<unsigned>(ctas), 32 * W, smem, st>>>(H, K, s, G);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

template <int E>
hq_status rows_mirror(float* G, int64_t K, const float* s, cudaStream_t st) {
  constexpr int B = 32 * E;
  constexpr int R = E <= 8 ? 4 : (E == 16 ? 2 : 1);
  const int64_t nb = K / B;
  const int64_t ctas = nb * (nb + 1) / 2 * E;
  if (ctas > 0x7FFFFFFF) return HQ_ERR_UNSUPPORTED;
  const size_t smem = static_cast<size_t>(32) * ((B + B / 32) | 1) * sizeof(float);
  if (smem > 48 * 1024)
    HQ_CUDA_TRY(cudaFuncSetAttribute(hadamard_rows_mirror_kernel<E, R>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     static_cast<int>(smem)));
  hadamard_rows_mirror_kernel<E, R><<<static_cast<unsigned>(ctas), 256, smem, st>>>(G, K, s);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

hq_status hessian_fast(const float* H, int64_t K, int B, const float* s, float* out, cudaStream_t st) {
  hq_status e = HQ_ERR_UNSUPPORTED;
  switch (B) {
    case 32: e = cols_lower<1>(H, K, s, out, st); break;
    case 64: e = cols_lower<2>(H, K, s, out, st); break;
    case 128: e = cols_lower<4>(H, K, s, out, st); break;
    case 256: e = cols_lower<8>(H, K, s, out, st); break;
    case 512: e = cols_lower<16>(H, K, s, out, st); break;
    case 1024: e = cols_lower<32>(H, K, s, out, st); break;
    default: break;
  }
  if (e != HQ_OK) return e;
  switch (B) {
    case 32: return rows_mirror<1>(out, K, s, st);
    case 64: return rows_mirror<2>(out, K, s, st);
    case 128: return rows_mirror<4>(out, K, s, st);
    case 256: return rows_mirror<8>(out, K, s, st);
    case 512: return rows_mirror<16>(out, K, s, st);
    case 1024: return rows_mirror<32>(out, K, s, st);
    default: return HQ_ERR_UNSUPPORTED;
  }
}

}  // namespace

hq_status launch_mirror_lower(const float* H, int64_t K, float* out, cudaStream_t st) {
  const int64_t nb = ceil_div(K, int64_t(32));
  const int64_t tiles = nb * (nb + 1) / 2;
  if (tiles > 0x7FFFFFFF) return HQ_ERR_UNSUPPORTED;
  mirror_lower_kernel<<<static_cast<unsigned>(tiles), 256, 0, st>>>(H, K, out);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

hq_status launch_hadamard_rows(const void* A, int a_dtype, int64_t rows, int64_t K, int B, const float* s,
                               float* out, cudaStream_t st) {
  if (rows == 0) return HQ_OK;
  if (B >= 32 && aligned16(A) && aligned16(s) && aligned16(out)) {
    if (a_dtype == HQ_BF16) return rows_warp_dispatch(static_cast<const __nv_bfloat16*>(A), rows, K, B, s, out, st);
    return rows_warp_dispatch(static_cast<const float*>(A), rows, K, B, s, out, st);
  }
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

hq_status launch_hadamard_hessian(const float* H, int64_t K, int B, const float* s, float* out, cudaStream_t st) {
  if (B >= 32 && aligned16(s) && aligned16(out)) return hessian_fast(H, K, B, s, out, st);
  hq_status e = launch_mirror_lower(H, K, out, st);
  if (e != HQ_OK) return e;
  e = launch_hadamard_rows(out, HQ_F32, K, K, B, s, out, st);
  if (e != HQ_OK) return e;
  return launch_hadamard_cols(out, K, B, s, st);
}

}  // namespace hq
