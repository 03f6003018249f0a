// GPTQ error-compensated column sweep (ork-driver wiki "Exp 2026-08-18 GPTQ Int4",
// experiment summary: error-feedback sweep, uniform symmetric int4 [-8, 7], per-(row, group)
// scale absmax/7, dequant w = code * scale; qerr definition in the same page).
//
// The sweep walks K in 128-column blocks.  For each block:
//   * sweep_block_kernel: the sequential part.  Four lanes share one row (lane l owns the
//     columns 4m + l of the block, 32 fp32 values in registers); the 128 x 128 diagonal block
//     of U sits in shared memory.  Per column j: group scale at a group start (4-lane absmax),
//     broadcast of w_j from its owner lane, code c = clamp(rint(w_j / s), -8, 7), error
//     e = (w_j - c s) / U[j, j], and the in-block feedback w_k -= e U[j, k] for k > j.  It
//     writes the block's errors (fp32, row-major [N, 128]), the packed int4 codes, the scales
//     and fp64 partial sums of the qerr numerator and denominator over the ORIGINAL weights.
//   * the lazy trailing update W[:, J+128:] -= Err * U[J:J+128, J+128:], a dense contraction
//     run on the tensor cores (tcgen05 kind::tf32, gemm_tc.cuh) with B = U^T row-major.
// U^T comes from factor.cu.  The working copy of W is fp32 in the workspace.
#include <cuda_bf16.h>

#include "common.cuh"
#include "gemm_tc.cuh"
#include "kernels.cuh"
#include "tmap.cuh"

namespace hq {

constexpr int kBlk = 128;       // sweep block width
constexpr int kRowsPerCta = 32;  // 4 warps x 8 rows (4 lanes per row)

struct SweepArgs {
  float* Wf;
  int64_t N, K;
  const float* Ut;
  int group;
  float* Err;
  uint8_t* codes;
  float* scales;
  const void* W;
  int w_dtype;
  const float* imp;
  double* partials;  // [K/128][gridDim.x][2]
  const int* info;
};

__device__ __forceinline__ float load_w(const void* W, int dt, int64_t idx) {
  return dt == HQ_BF16 ? __bfloat162float(static_cast<const __nv_bfloat16*>(W)[idx]) : static_cast<const float*>(W)[idx];
}

__device__ __forceinline__ float quant_code(float w, float s) {
  if (!(s > 0.f)) return 0.f;
  float c = rintf(__fdiv_rn(w, s));
  return fminf(fmaxf(c, -8.f), 7.f);
}

// GS: group size when it is 32, 64 or 128 (scales computed inside the block), or 0 when the
// group spans several blocks (scale computed at the group's first block from Wf).
template <int GS>
__global__ void __launch_bounds__(128) sweep_block_kernel(SweepArgs a, int j0) {
  if (*a.info != 0) return;
  extern __shared__ float sm[];
  float* Us = sm;                                    // [128][129]: Us[j][k] = U[j0+j][j0+k]
  float* err_s = Us + kBlk * (kBlk + 1);             // [32][128]
  float* scl_s = err_s + kRowsPerCta * kBlk;         // [32][4]
  int8_t* code_s = reinterpret_cast<int8_t*>(scl_s + kRowsPerCta * 4);  // [32][128]

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31, l = lane & 3, rg = lane >> 2;
  const int rl = warp * 8 + rg;  // row within the CTA
  const int64_t row = static_cast<int64_t>(blockIdx.x) * kRowsPerCta + rl;
  const bool valid = row < a.N;
  const int64_t K = a.K;

  for (int e = tid; e < kBlk * kBlk; e += blockDim.x) {
    const int k = e / kBlk, j = e % kBlk;
    Us[j * (kBlk + 1) + k] = (k >= j) ? a.Ut[(j0 + k) * K + j0 + j] : 0.f;
  }
  float w[32];
  const float* wrow = a.Wf + row * K + j0;
#pragma unroll
  for (int m = 0; m < 32; ++m) w[m] = valid ? wrow[4 * m + l] : 0.f;

  float s = 0.f;
  if (GS == 0) {
    const int G = a.group;
    const int64_t g = j0 / G;
    if (j0 % G == 0) {
      float am = 0.f;
      if (valid)
        for (int i = l; i < G; i += 4) am = fmaxf(am, fabsf(a.Wf[row * K + j0 + i]));
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
      s = __fdiv_rn(am, 7.f);
      if (valid && l == 0) a.scales[row * (K / G) + g] = s;
    } else {
      s = valid ? a.scales[row * (K / G) + g] : 0.f;
    }
    if (l == 0) scl_s[rl * 4] = s;
  }
  __syncthreads();

#pragma unroll
  for (int j = 0; j < kBlk; ++j) {
    if (GS != 0 && (j % (GS == 0 ? 1 : GS)) == 0) {
      float am = 0.f;
#pragma unroll
      for (int m = j / 4; m < (j + GS) / 4; ++m) am = fmaxf(am, fabsf(w[m]));
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
      am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));
      s = __fdiv_rn(am, 7.f);
      if (l == 0) scl_s[rl * 4 + j / (GS == 0 ? 1 : GS)] = s;
    }
    const float wj = __shfl_sync(0xffffffffu, w[j / 4], (lane & ~3) | (j & 3));
    const float c = quant_code(wj, s);
    const float d = fmaf(-c, s, wj);
    const float e = __fdiv_rn(d, Us[j * (kBlk + 1) + j]);
    if (l == (j & 3)) {
      err_s[rl * kBlk + j] = e;
      code_s[rl * kBlk + j] = static_cast<int8_t>(c);
    }
    const float* urow = Us + j * (kBlk + 1);
#pragma unroll
    for (int m = j / 4; m < 32; ++m) w[m] = fmaf(-e, urow[4 * m + l], w[m]);
  }
  __syncthreads();

  // errors -> Err [N, 128], codes -> packed bytes, scales, qerr partials
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kRowsPerCta;
  for (int e = tid; e < kRowsPerCta * kBlk; e += blockDim.x) {
    const int r = e / kBlk, k = e % kBlk;
    if (r0 + r < a.N) a.Err[(r0 + r) * kBlk + k] = err_s[r * kBlk + k];
  }
  for (int e = tid; e < kRowsPerCta * (kBlk / 2); e += blockDim.x) {
    const int r = e / (kBlk / 2), p = e % (kBlk / 2);
    if (r0 + r < a.N) {
      const int lo = code_s[r * kBlk + 2 * p] & 0xF, hi = code_s[r * kBlk + 2 * p + 1] & 0xF;
      a.codes[(r0 + r) * (K / 2) + j0 / 2 + p] = static_cast<uint8_t>(lo | (hi << 4));
    }
  }
  if (GS != 0) {
    constexpr int ng = (GS == 0) ? 1 : kBlk / GS;
    for (int e = tid; e < kRowsPerCta * ng; e += blockDim.x) {
      const int r = e / ng, g = e % ng;
      if (r0 + r < a.N) a.scales[(r0 + r) * (K / (GS == 0 ? 1 : GS)) + j0 / (GS == 0 ? 1 : GS) + g] = scl_s[r * 4 + g];
    }
  }
  double num = 0.0, den = 0.0;
  for (int e = tid; e < kRowsPerCta * kBlk; e += blockDim.x) {
    const int r = e / kBlk, k = e % kBlk;
    if (r0 + r >= a.N) continue;
    const double wo = static_cast<double>(load_w(a.W, a.w_dtype, (r0 + r) * K + j0 + k));
    const double sc = static_cast<double>(GS != 0 ? scl_s[r * 4 + k / (GS == 0 ? 1 : GS)] : scl_s[r * 4]);
    const double q = static_cast<double>(code_s[r * kBlk + k]) * sc;
    const double im = a.imp != nullptr ? static_cast<double>(a.imp[j0 + k]) : 1.0;
    num += im * (wo - q) * (wo - q);
    den += im * wo * wo;
  }
  // deterministic CTA reduction: warp shuffles, then the four warp sums in order
  for (int off = 16; off > 0; off >>= 1) {
    num += __shfl_down_sync(0xffffffffu, num, off);
    den += __shfl_down_sync(0xffffffffu, den, off);
  }
  __shared__ double red[4][2];
  if (lane == 0) {
    red[warp][0] = num;
    red[warp][1] = den;
  }
  __syncthreads();
  if (tid == 0) {
    double* p = a.partials + (static_cast<int64_t>(j0 / kBlk) * gridDim.x + blockIdx.x) * 2;
    p[0] = red[0][0] + red[1][0] + red[2][0] + red[3][0];
    p[1] = red[0][1] + red[1][1] + red[2][1] + red[3][1];
  }
}

constexpr size_t kSweepSmem = (kBlk * (kBlk + 1) + kRowsPerCta * kBlk + kRowsPerCta * 4) * sizeof(float) +
                              kRowsPerCta * kBlk;

__global__ void w_prep_kernel(const void* __restrict__ W, int dt, int64_t n, float* __restrict__ Wf) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    Wf[i] = load_w(W, dt, i);
}

__global__ void __launch_bounds__(256) qerr_finalize_kernel(const double* __restrict__ partials, int64_t count,
                                                            WsHeader* hdr, double* qerr_dev) {
  __shared__ double rn[256], rd[256];
  double n = 0.0, d = 0.0;
  for (int64_t i = threadIdx.x; i < count; i += blockDim.x) {
    n += partials[2 * i];
    d += partials[2 * i + 1];
  }
  rn[threadIdx.x] = n;
  rd[threadIdx.x] = d;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (static_cast<int>(threadIdx.x) < w) {
      rn[threadIdx.x] += rn[threadIdx.x + w];
      rd[threadIdx.x] += rd[threadIdx.x + w];
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double q = rd[0] > 0.0 ? sqrt(rn[0] / rd[0]) : 0.0;
    hdr->num = rn[0];
    hdr->den = rd[0];
    hdr->qerr = q;
    if (qerr_dev != nullptr) *qerr_dev = q;
  }
}

hq_status launch_qerr_finalize(const double* partials, int64_t count, WsHeader* hdr, double* qerr_dev,
                               cudaStream_t s) {
  qerr_finalize_kernel<<<1, 256, 0, s>>>(partials, count, hdr, qerr_dev);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

// ------------------------------------------------------------------------- layout / driver

bool gptq_shape_ok(int64_t N, int64_t K, int64_t group) {
  if (N < 1 || K < kBlk || K % kBlk != 0 || group < 32 || group % 32 != 0 || K % group != 0) return false;
  if (!(group == 32 || group == 64 || group == 128 || group % kBlk == 0)) return false;
  if (K > 65536 || N > (int64_t(1) << 31) - kRowsPerCta) return false;
  return true;
}

GptqLayout gptq_layout(int64_t N, int64_t K, int64_t /*group*/) {
  GptqLayout L{};
  const size_t al = 256;
  L.sweep_grid = static_cast<int>(ceil_div(N, kRowsPerCta));
  size_t off = 0;
  L.header = off;
  off = round_up(off + sizeof(WsHeader), al);
  L.partials = off;
  off = round_up(off + static_cast<size_t>(K / kBlk) * L.sweep_grid * 2 * sizeof(double), al);
  L.wf = off;
  off = round_up(off + static_cast<size_t>(N) * K * sizeof(float), al);
  L.err = off;
  off = round_up(off + static_cast<size_t>(N) * kBlk * sizeof(float), al);
  L.a = off;
  off = round_up(off + static_cast<size_t>(K) * K * sizeof(float), al);
  L.x = off;
  off = round_up(off + static_cast<size_t>(K) * K * sizeof(float), al);
  L.t = off;
  off = round_up(off + static_cast<size_t>(K / 2) * (K - K / 2 + 64) * sizeof(float), al);
  L.dinv = off;
  off = round_up(off + static_cast<size_t>(K) * 64 * sizeof(float), al);
  L.total = off;
  return L;
}

static hq_status launch_update_simt(float* Wf, int64_t N, int64_t K, int j0, const float* Err, const float* Ut,
                                    const int* info, cudaStream_t s);

hq_status launch_gptq(const void* W, int w_dtype, int64_t N, int64_t K, const float* H, int64_t group, float damp,
                      const float* imp, uint8_t* codes, float* scales, double* qerr_dev, uint8_t* ws,
                      int update_impl, cudaStream_t s) {
  const GptqLayout L = gptq_layout(N, K, group);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws + L.header);
  double* partials = reinterpret_cast<double*>(ws + L.partials);
  float* Wf = reinterpret_cast<float*>(ws + L.wf);
  float* Err = reinterpret_cast<float*>(ws + L.err);
  float* A = reinterpret_cast<float*>(ws + L.a);
  float* X = reinterpret_cast<float*>(ws + L.x);
  float* T = reinterpret_cast<float*>(ws + L.t);
  float* Dinv = reinterpret_cast<float*>(ws + L.dinv);
  HQ_CUDA_TRY(cudaMemsetAsync(hdr, 0, sizeof(WsHeader), s));

  hq_status st = launch_factor(H, K, damp, A, X, T, Dinv, &hdr->lam, &hdr->info, /*Ut=*/A, s);
  if (st != HQ_OK) return st;
  const float* Ut = A;

  {
    const int64_t n = N * K;
    const int grid = static_cast<int>(ceil_div(n, 256) < 148 * 16 ? ceil_div(n, 256) : 148 * 16);
    w_prep_kernel<<<grid, 256, 0, s>>>(W, w_dtype, n, Wf);
    HQ_LAUNCH_CHECK();
  }

  SweepArgs a{};
  a.Wf = Wf;
  a.N = N;
  a.K = K;
  a.Ut = Ut;
  a.group = static_cast<int>(group);
  a.Err = Err;
  a.codes = codes;
  a.scales = scales;
  a.W = W;
  a.w_dtype = w_dtype;
  a.imp = imp;
  a.partials = partials;
  a.info = &hdr->info;

  void (*kern)(SweepArgs, int) = nullptr;
  switch (group) {
    case 32: kern = sweep_block_kernel<32>; break;
    case 64: kern = sweep_block_kernel<64>; break;
    case 128: kern = sweep_block_kernel<128>; break;
    default: kern = sweep_block_kernel<0>; break;
  }
  HQ_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kSweepSmem)));

  CUtensorMap mapE, mapU;
  if (update_impl == 0) {
    if (!make_tmap_2d(&mapE, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Err, kBlk, static_cast<uint64_t>(N), kBlk * 4, 32, 128))
      return HQ_ERR_CUDA;
    if (!make_tmap_2d(&mapU, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, Ut, static_cast<uint64_t>(K), static_cast<uint64_t>(K),
                      static_cast<uint64_t>(K) * 4, 32, 256))
      return HQ_ERR_CUDA;
    HQ_CUDA_TRY(cudaFuncSetAttribute(umma_gemm_kernel<GemmMode::kUpdateTF32>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize, kGemmSmemBytes));
  }

  const int nblk = static_cast<int>(K / kBlk);
  for (int b = 0; b < nblk; ++b) {
    const int j0 = b * kBlk;
    kern<<<L.sweep_grid, 128, kSweepSmem, s>>>(a, j0);
    HQ_LAUNCH_CHECK();
    const int64_t ncols = K - j0 - kBlk;
    if (ncols <= 0) continue;
    if (update_impl == 0) {
      GemmArgs g{};
      g.C = Wf;
      g.ldc = K;
      g.M = static_cast<int>(N);
      g.Ncols = static_cast<int>(ncols);
      g.Kred = kBlk;
      g.col0 = j0 + kBlk;
      g.b_x0 = j0;
      g.b_y0 = j0 + kBlk;
      g.tiles_n = static_cast<int>(ceil_div(ncols, kGemmBN));
      g.skip = &hdr->info;
      g.status = &hdr->status;
      const int64_t ctas = ceil_div(N, kGemmBM) * g.tiles_n;
      umma_gemm_kernel<GemmMode::kUpdateTF32><<<static_cast<unsigned>(ctas), gemm_threads(GemmMode::kUpdateTF32), kGemmSmemBytes, s>>>(
          mapE, mapU, g);
      HQ_LAUNCH_CHECK();
    } else {
      st = launch_update_simt(Wf, N, K, j0, Err, Ut, &hdr->info, s);
      if (st != HQ_OK) return st;
    }
  }
  return launch_qerr_finalize(partials, static_cast<int64_t>(nblk) * L.sweep_grid, hdr, qerr_dev, s);
}

// CUDA-core fp32 version of the trailing update (cross-check of the tensor-core kernel).
__global__ void __launch_bounds__(256) update_simt_kernel(float* __restrict__ Wf, int64_t N, int64_t K, int j0,
                                                          const float* __restrict__ Err,
                                                          const float* __restrict__ Ut, const int* __restrict__ info) {
  if (*info != 0) return;
  const int64_t ncols = K - j0 - kBlk;
  const int64_t tiles_n = (ncols + 63) / 64;
  const int64_t tm = blockIdx.x / tiles_n, tn = blockIdx.x % tiles_n;
  const int64_t m0 = tm * 64, n0 = tn * 64;
  __shared__ float As[16][64];
  __shared__ float Bs[16][64];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < kBlk; k0 += 16) {
    for (int e = threadIdx.x; e < 16 * 64; e += 256) {
      const int kk = e % 16, c = e / 16;
      As[kk][c] = (m0 + c < N) ? Err[(m0 + c) * kBlk + k0 + kk] : 0.f;
      Bs[kk][c] = (n0 + c < ncols) ? Ut[(j0 + kBlk + n0 + c) * K + j0 + k0 + kk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk)
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(As[kk][ty + 16 * u], Bs[kk][tx + 16 * v], acc[u][v]);
    __syncthreads();
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int64_t m = m0 + ty + 16 * u;
    if (m >= N) continue;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int64_t n = n0 + tx + 16 * v;
      if (n < ncols) Wf[m * K + j0 + kBlk + n] -= acc[u][v];
    }
  }
}

static hq_status launch_update_simt(float* Wf, int64_t N, int64_t K, int j0, const float* Err, const float* Ut,
                                    const int* info, cudaStream_t s) {
  const int64_t ncols = K - j0 - kBlk;
  const int64_t ctas = ceil_div(N, 64) * ceil_div(ncols, 64);
  update_simt_kernel<<<static_cast<unsigned>(ctas), 256, 0, s>>>(Wf, N, K, j0, Err, Ut, info);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

}  // namespace hq
