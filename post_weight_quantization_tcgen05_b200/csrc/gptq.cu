// GPTQ error-compensated column sweep (ork-driver wiki "Exp 2026-08-18 GPTQ Int4",
// experiment summary: error-feedback sweep, uniform symmetric int4 [-8, 7], per-(row, group)
// scale absmax/7, dequant w = code * scale; qerr definition in the same page).
//
// The sweep walks K in 128-column blocks grouped into panels of P columns (P = 512, or a
// multiple of the group size when groups are wider than a block).  Per block:
//   * sweep_block_kernel: the sequential part.  A group of eight lanes carries two rows;
//     lane l holds columns l, l+8, l+16, ... of both rows as 16 "slots" each, in registers.
//     The columns are visited in rounds of eight: at the end of a round every lane shifts its
//     slots down by one, so the column being quantised is always slot 0 of lane (j mod 8), a
//     compile-time lane inside the 8-way unrolled round, and the loop body stays small enough
//     for the instruction cache.  Per column j and row: group scale at a group start (8-lane
//     absmax), broadcast of w_j, code c = clamp(rint(w_j / s), -8, 7), error
//     e = (w_j - c s) / U[j, j], and the feedback w_k -= e U[j, k] for k > j.  U's row j is
//     pre-permuted (and XOR-swizzled against bank conflicts) in shared memory so that each
//     lane reads its 16 values with four 16-byte loads, used for both of its rows.  It writes the block's
//     errors into the panel's error buffer, the packed int4 codes, the scales and fp64 partial
//     sums of the qerr numerator and denominator over the ORIGINAL weights.
//   * inner lazy update of the rest of the panel, W[:, b+128 : panel end] -= Err_b U[b, ...]
//     (contraction 128; the panel's N x P working weights stay in L2);
// and after the panel the outer lazy update W[:, panel end:] -= Err_panel U[panel, ...] with
// contraction P.  Both updates are dense contractions on the tensor cores (gemm_tf32.cuh, by
// default 3xTF32) with B = U^T row-major.  Blocking only reorders exact sums: every column
// still receives the feedback of every earlier column before it is quantised.
// U^T comes from factor.cu.  The working copy of W is fp32 in the workspace.
#include <cuda_bf16.h>

#include "common.cuh"
#include "kernels.cuh"

namespace hq {

constexpr int kBlk = 128;        // sweep block width
constexpr int kLanesPerRow = 8;
constexpr int kSlots = kBlk / kLanesPerRow;  // 16 columns per lane
constexpr int kRowsPerCta = 32;              // 4 warps x 4 lane groups x 2 rows
constexpr int kSweepThreads = 128;

struct SweepArgs {
  float* Wf;
  int64_t N, K;
  const float* U;    // U row-major (upper triangular)
  int group;
  float* Err;        // panel error buffer [N, P] (the tf32 part when Err_lo is set)
  float* Err_lo;     // NULL, or the fp32 remainder of each error (Err + Err_lo = error)
  int64_t err_ld;    // P
  int err_col;       // column of this block inside the panel buffer
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

// c = clamp(rint(w / s), -8, 7) with w / s the IEEE fp32 quotient.  w * (1/s) is within a
// couple of ulps of the quotient, so it rounds the same way unless it lies within 1e-5 of a
// half-integer; only then is the exact division taken.  Rounding to nearest-even uses the
// 1.5 * 2^23 shift (exact for |q| < 2^22; larger values are clamped anyway).
__device__ __forceinline__ float quant_code(float w, float s, float rs) {
  if (!(s > 0.f)) return 0.f;
  constexpr float kShift = 12582912.f;
  float q = w * rs;
  float r = (q + kShift) - kShift;
  if (fabsf(q - r) > 0.5f - 1e-5f) r = rintf(__fdiv_rn(w, s));
  return fminf(fmaxf(r, -8.f), 7.f);
}

// GS: group size when it is 32, 64 or 128 (scales computed inside the block), or 0 when the
// group spans several blocks (scale computed at the group's first block from Wf).
// Offset (in floats) of chunk q (4 floats) of lane l's 16 U values for column j.  The XOR
// keeps the eight lanes of a quarter-warp on eight different 16-byte bank groups.
__device__ __forceinline__ int ur_off(int j, int l, int q) { return (j * kLanesPerRow + l) * kSlots + 4 * (q ^ (l >> 1)); }

template <int GS>
__global__ void __launch_bounds__(kSweepThreads) sweep_block_kernel(SweepArgs a, int j0) {
  if (*a.info != 0) return;
  constexpr int LD = kBlk + 1;  // padded row of the staging buffer
  constexpr int kGS = (GS == 0 ? kLanesPerRow : GS) / kLanesPerRow;  // slots per group
  extern __shared__ float sm[];
  float* Ur = sm;                                  // [128 j][8 lanes][16 slots], swizzled
  float* stage = Ur + kBlk * kBlk;                 // [32][129]: weights in, errors out
  float* scl_s = stage + kRowsPerCta * LD;         // [32][4]
  float* inv_diag = scl_s + kRowsPerCta * 4;       // [128]: 1 / U[j][j]
  int8_t* code_s = reinterpret_cast<int8_t*>(inv_diag + kBlk);  // [32][128]

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31, l = lane & (kLanesPerRow - 1);
  const int rl0 = warp * (32 / kLanesPerRow) + lane / kLanesPerRow;  // rows rl0 and rl0 + 16
  const int rl1 = rl0 + kRowsPerCta / 2;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * kRowsPerCta;
  const int64_t K = a.K;

  // Ur: U[j0 + j][j0 + 8 * (j / 8 + m) + l] for slot m of lane l, zero past the block.
  for (int e = tid; e < kBlk * kBlk; e += kSweepThreads) Ur[e] = 0.f;
  __syncthreads();
#pragma unroll 4
  for (int e = tid; e < kBlk * (kBlk / 4); e += kSweepThreads) {
    const int j = e >> 5, q4 = e & 31;  // row j, columns 4 q4 .. 4 q4 + 3
    const float4 u = reinterpret_cast<const float4*>(a.U + (j0 + j) * K + j0)[q4];
    const float uv[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int col = 4 * q4 + i;
      const int m = col / kLanesPerRow - j / kLanesPerRow;
      if (m >= 0) Ur[ur_off(j, col % kLanesPerRow, m >> 2) + (m & 3)] = uv[i];
    }
  }
  // weights: coalesced 512-byte rows into the staging buffer
  for (int r = warp; r < kRowsPerCta; r += kSweepThreads / 32) {
    const float4 v = (r0 + r < a.N) ? reinterpret_cast<const float4*>(a.Wf + (r0 + r) * K + j0)[lane]
                                    : make_float4(0.f, 0.f, 0.f, 0.f);
    float* d = stage + r * LD + 4 * lane;
    d[0] = v.x;
    d[1] = v.y;
    d[2] = v.z;
    d[3] = v.w;
  }
  __syncthreads();
  for (int j = tid; j < kBlk; j += kSweepThreads) inv_diag[j] = __frcp_rn(a.U[(j0 + j) * K + j0 + j]);
  float w0[kSlots], w1[kSlots];
#pragma unroll
  for (int m = 0; m < kSlots; ++m) {
    w0[m] = stage[rl0 * LD + kLanesPerRow * m + l];
    w1[m] = stage[rl1 * LD + kLanesPerRow * m + l];
  }

  float s0 = 0.f, rs0 = 0.f, s1 = 0.f, rs1 = 0.f;
  if (GS == 0) {
    // the group spans several blocks: its scale is taken at its first block from the current
    // weights of all its columns, and read back in the later blocks
    const int G = a.group;
    const int64_t g = j0 / G;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int rl = h ? rl1 : rl0;
      const int64_t row = r0 + rl;
      const bool valid = row < a.N;
      float sc;
      if (j0 % G == 0) {
        float am = 0.f;
        if (valid)
          for (int i = l; i < G; i += kLanesPerRow) am = fmaxf(am, fabsf(a.Wf[row * K + j0 + i]));
#pragma unroll
        for (int x = 1; x < kLanesPerRow; x <<= 1) am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, x));
        sc = __fdiv_rn(am, 7.f);
        if (valid && l == 0) a.scales[row * (K / G) + g] = sc;
      } else {
        sc = valid ? a.scales[row * (K / G) + g] : 0.f;
      }
      if (l == 0) scl_s[rl * 4] = sc;
      if (h) {
        s1 = sc;
        rs1 = __frcp_rn(sc);
      } else {
        s0 = sc;
        rs0 = __frcp_rn(sc);
      }
    }
  }
  __syncthreads();

  float* err0 = stage + rl0 * LD;
  float* err1 = stage + rl1 * LD;
  int8_t* code0 = code_s + rl0 * kBlk;
  int8_t* code1 = code_s + rl1 * kBlk;
  const int src_base = lane & ~(kLanesPerRow - 1);
#pragma unroll 1
  for (int R = 0; R < kSlots; ++R) {
#pragma unroll
    for (int jr = 0; jr < kLanesPerRow; ++jr) {
      const int j = kLanesPerRow * R + jr;
      if (GS != 0 && jr == 0 && (R % kGS) == 0) {
        float am0 = 0.f, am1 = 0.f;
#pragma unroll
        for (int m = 0; m < kGS; ++m) {
          am0 = fmaxf(am0, fabsf(w0[m]));
          am1 = fmaxf(am1, fabsf(w1[m]));
        }
#pragma unroll
        for (int x = 1; x < kLanesPerRow; x <<= 1) {
          am0 = fmaxf(am0, __shfl_xor_sync(0xffffffffu, am0, x));
          am1 = fmaxf(am1, __shfl_xor_sync(0xffffffffu, am1, x));
        }
        s0 = __fdiv_rn(am0, 7.f);
        s1 = __fdiv_rn(am1, 7.f);
        rs0 = __frcp_rn(s0);
        rs1 = __frcp_rn(s1);
        if (l == 0) {
          scl_s[rl0 * 4 + j / (GS == 0 ? 1 : GS)] = s0;
          scl_s[rl1 * 4 + j / (GS == 0 ? 1 : GS)] = s1;
        }
      }
      float u[kSlots];
#pragma unroll
      for (int q = 0; q < kSlots / 4; ++q) {
        const float4 t = *reinterpret_cast<const float4*>(Ur + ur_off(j, l, q));
        u[4 * q] = t.x;
        u[4 * q + 1] = t.y;
        u[4 * q + 2] = t.z;
        u[4 * q + 3] = t.w;
      }
      const float idg = inv_diag[j];
      const float wj0 = __shfl_sync(0xffffffffu, w0[0], src_base | jr);
      const float wj1 = __shfl_sync(0xffffffffu, w1[0], src_base | jr);
      const float c0 = quant_code(wj0, s0, rs0);
      const float c1 = quant_code(wj1, s1, rs1);
      const float e0 = fmaf(-c0, s0, wj0) * idg;
      const float e1 = fmaf(-c1, s1, wj1) * idg;
      if (l == jr) {
        err0[j] = e0;
        err1[j] = e1;
        code0[j] = static_cast<int8_t>(c0);
        code1[j] = static_cast<int8_t>(c1);
      }
      if (l > jr) {
        w0[0] = fmaf(-e0, u[0], w0[0]);
        w1[0] = fmaf(-e1, u[0], w1[0]);
      }
#pragma unroll
      for (int m = 1; m < kSlots; ++m) {
        w0[m] = fmaf(-e0, u[m], w0[m]);
        w1[m] = fmaf(-e1, u[m], w1[m]);
      }
    }
#pragma unroll
    for (int m = 0; m < kSlots - 1; ++m) {
      w0[m] = w0[m + 1];
      w1[m] = w1[m + 1];
    }
    w0[kSlots - 1] = 0.f;
    w1[kSlots - 1] = 0.f;
  }
  __syncthreads();

  // errors -> panel buffer (coalesced rows), codes -> packed bytes, scales, qerr partials
  for (int r = warp; r < kRowsPerCta; r += kSweepThreads / 32) {
    if (r0 + r >= a.N) break;
    const float* src = stage + r * LD + 4 * lane;
    const float4 e4 = make_float4(src[0], src[1], src[2], src[3]);
    if (a.Err_lo == nullptr) {
      reinterpret_cast<float4*>(a.Err + (r0 + r) * a.err_ld + a.err_col)[lane] = e4;
    } else {  // split for the 3xTF32 updates: tf32 part (low 13 mantissa bits cleared) + remainder
      const float4 h4 = make_float4(__uint_as_float(__float_as_uint(e4.x) & 0xFFFFE000u),
                                    __uint_as_float(__float_as_uint(e4.y) & 0xFFFFE000u),
                                    __uint_as_float(__float_as_uint(e4.z) & 0xFFFFE000u),
                                    __uint_as_float(__float_as_uint(e4.w) & 0xFFFFE000u));
      reinterpret_cast<float4*>(a.Err + (r0 + r) * a.err_ld + a.err_col)[lane] = h4;
      reinterpret_cast<float4*>(a.Err_lo + (r0 + r) * a.err_ld + a.err_col)[lane] =
          make_float4(e4.x - h4.x, e4.y - h4.y, e4.z - h4.z, e4.w - h4.w);
    }
    // lane writes bytes 2*lane, 2*lane+1 of the row's 64 code bytes
    const int8_t* cs = code_s + r * kBlk + 4 * lane;
    const uint32_t b0 = (cs[0] & 0xF) | ((cs[1] & 0xF) << 4);
    const uint32_t b1 = (cs[2] & 0xF) | ((cs[3] & 0xF) << 4);
    reinterpret_cast<uint16_t*>(a.codes + (r0 + r) * (K / 2) + j0 / 2)[lane] = static_cast<uint16_t>(b0 | (b1 << 8));
  }
  if (GS != 0) {
    constexpr int ng = (GS == 0) ? 1 : kBlk / GS;
    for (int e = tid; e < kRowsPerCta * ng; e += kSweepThreads) {
      const int r = e / ng, g = e % ng;
      if (r0 + r < a.N) a.scales[(r0 + r) * (K / (GS == 0 ? 1 : GS)) + j0 / (GS == 0 ? 1 : GS) + g] = scl_s[r * 4 + g];
    }
  }
  double num = 0.0, den = 0.0;
  for (int r = warp; r < kRowsPerCta; r += kSweepThreads / 32) {
    if (r0 + r >= a.N) break;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int k = 4 * lane + i;
      const double wo = static_cast<double>(load_w(a.W, a.w_dtype, (r0 + r) * K + j0 + k));
      const double sc = static_cast<double>(GS != 0 ? scl_s[r * 4 + k / (GS == 0 ? 1 : GS)] : scl_s[r * 4]);
      const double q = static_cast<double>(code_s[r * kBlk + k]) * sc;
      const double im = a.imp != nullptr ? static_cast<double>(a.imp[j0 + k]) : 1.0;
      num += im * (wo - q) * (wo - q);
      den += im * wo * wo;
    }
  }
  for (int off = 16; off > 0; off >>= 1) {
    num += __shfl_down_sync(0xffffffffu, num, off);
    den += __shfl_down_sync(0xffffffffu, den, off);
  }
  __shared__ double red[kSweepThreads / 32][2];
  if (lane == 0) {
    red[warp][0] = num;
    red[warp][1] = den;
  }
  __syncthreads();
  if (tid == 0) {
    double sn = 0.0, sd = 0.0;
    for (int wq = 0; wq < kSweepThreads / 32; ++wq) {
      sn += red[wq][0];
      sd += red[wq][1];
    }
    double* p = a.partials + (static_cast<int64_t>(j0 / kBlk) * gridDim.x + blockIdx.x) * 2;
    p[0] = sn;
    p[1] = sd;
  }
}

constexpr size_t kSweepSmem =
    (kBlk * kBlk + kRowsPerCta * (kBlk + 1) + kRowsPerCta * 4 + kBlk) * sizeof(float) + kRowsPerCta * kBlk;

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

// Panel width of the two-level update: 512 columns, or a multiple of a group wider than a
// block so that every group lies inside one panel.
static int64_t panel_width(int64_t K, int64_t group) {
  const int64_t base = group > kBlk ? group : kBlk;
  int64_t P = base * ((512 / base) > 1 ? (512 / base) : 1);
  return P < K ? P : K;
}

GptqLayout gptq_layout(int64_t N, int64_t K, int64_t group) {
  GptqLayout L{};
  const size_t al = 256;
  L.sweep_grid = static_cast<int>(ceil_div(N, kRowsPerCta));
  const int64_t P = panel_width(K, group);
  size_t off = 0;
  L.header = off;
  off = round_up(off + sizeof(WsHeader), al);
  L.partials = off;
  off = round_up(off + static_cast<size_t>(K / kBlk) * L.sweep_grid * 2 * sizeof(double), al);
  L.wf = off;
  off = round_up(off + static_cast<size_t>(N) * K * sizeof(float), al);
  L.err = off;
  off = round_up(off + static_cast<size_t>(N) * P * sizeof(float), al);
  L.err_lo = off;  // remainder part of the errors for the 3xTF32 updates
  off = round_up(off + static_cast<size_t>(N) * P * sizeof(float), al);
  L.a = off;  // fp64 A, later U^T and U in fp32
  off = round_up(off + static_cast<size_t>(K) * K * sizeof(double), al);
  L.x = off;
  off = round_up(off + static_cast<size_t>(K) * K * sizeof(double), al);
  L.xt = off;
  off = round_up(off + static_cast<size_t>(K) * K * sizeof(double), al);
  L.t = off;
  off = round_up(off + static_cast<size_t>(K) * K * sizeof(double), al);
  L.total = off;
  return L;
}

// W[:, c0 : c0+ncols] -= E[:, 0:kred] * U[k0 : k0+kred, c0 : c0+ncols]   (E row stride lde)
static hq_status sweep_update(int impl, float* Wf, int64_t N, int64_t K, int64_t c0, int64_t ncols, const float* E,
                              const float* E_lo, int64_t lde, int64_t k0, int64_t kred, const float* Ut,
                              const float* Ut_hi, const float* Ut_lo, const int* info, int* status, cudaStream_t s);

hq_status launch_gptq(const void* W, int w_dtype, int64_t N, int64_t K, const float* H, int64_t group, float damp,
                      const float* imp, uint8_t* codes, float* scales, double* qerr_dev, uint8_t* ws,
                      int update_impl, cudaStream_t s) {
  const GptqLayout L = gptq_layout(N, K, group);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws + L.header);
  double* partials = reinterpret_cast<double*>(ws + L.partials);
  float* Wf = reinterpret_cast<float*>(ws + L.wf);
  float* Err = reinterpret_cast<float*>(ws + L.err);
  float* Err_lo = reinterpret_cast<float*>(ws + L.err_lo);
  double* A = reinterpret_cast<double*>(ws + L.a);
  double* X = reinterpret_cast<double*>(ws + L.x);
  double* XT = reinterpret_cast<double*>(ws + L.xt);
  double* T = reinterpret_cast<double*>(ws + L.t);
  HQ_CUDA_TRY(cudaMemsetAsync(hdr, 0, sizeof(WsHeader), s));

  float* Ut = nullptr;
  float* U = nullptr;
  float* Ut_hi = nullptr;
  float* Ut_lo = nullptr;
  const bool split = (update_impl == 0);  // 3xTF32 updates take pre-split operands
  hq_status st = launch_factor(H, K, damp, A, X, XT, T, &hdr->lam, &hdr->info, &hdr->status, &Ut, &U, split, &Ut_hi,
                               &Ut_lo, s);
  if (st != HQ_OK) return st;

  {
    const int64_t n = N * K;
    const int grid = static_cast<int>(ceil_div(n, 256) < 148 * 16 ? ceil_div(n, 256) : 148 * 16);
    w_prep_kernel<<<grid, 256, 0, s>>>(W, w_dtype, n, Wf);
    HQ_LAUNCH_CHECK();
  }

  const int64_t P = panel_width(K, group);
  SweepArgs a{};
  a.Wf = Wf;
  a.N = N;
  a.K = K;
  a.U = U;
  a.group = static_cast<int>(group);
  a.Err = Err;
  a.Err_lo = split ? Err_lo : nullptr;
  a.err_ld = P;
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

  for (int64_t p0 = 0; p0 < K; p0 += P) {
    const int64_t p1 = (p0 + P < K) ? p0 + P : K;
    for (int64_t j0 = p0; j0 < p1; j0 += kBlk) {
      a.err_col = static_cast<int>(j0 - p0);
      const int tm = timer_start(kTimeSweep, s);
      kern<<<L.sweep_grid, kSweepThreads, kSweepSmem, s>>>(a, static_cast<int>(j0));
      HQ_LAUNCH_CHECK();
      // bytes: the block of working weights in, its errors out (fp32), the block of U^T, packed
      // codes and the block's scales out
      timer_stop(tm, static_cast<double>(N) * kBlk * 8.0 + kBlk * kBlk * 4.0 + N * (kBlk / 2.0) +
                         N * (static_cast<double>(kBlk) / group) * 4.0, s);
      const int64_t j1 = j0 + kBlk;
      if (j1 < p1) {  // inner update of the rest of the panel
        st = sweep_update(update_impl, Wf, N, K, j1, p1 - j1, Err + (j0 - p0), Err_lo + (j0 - p0), P, j0, kBlk, Ut,
                          Ut_hi, Ut_lo, &hdr->info, &hdr->status, s);
        if (st != HQ_OK) return st;
      }
    }
    if (p1 < K) {  // outer update of everything right of the panel
      st = sweep_update(update_impl, Wf, N, K, p1, K - p1, Err, Err_lo, P, p0, p1 - p0, Ut, Ut_hi, Ut_lo, &hdr->info,
                        &hdr->status, s);
      if (st != HQ_OK) return st;
    }
  }
  return launch_qerr_finalize(partials, static_cast<int64_t>(K / kBlk) * L.sweep_grid, hdr, qerr_dev, s);
}

// CUDA-core fp32 version of the lazy update (cross-check of the tensor-core kernel).
__global__ void __launch_bounds__(256) update_simt_kernel(float* __restrict__ C, int64_t ldc, int64_t M,
                                                          int64_t ncols, const float* __restrict__ E, int64_t lde,
                                                          const float* __restrict__ B, int64_t ldb, int64_t kred,
                                                          const int* __restrict__ info) {
  if (*info != 0) return;
  const int64_t tiles_n = (ncols + 63) / 64;
  const int64_t tm = blockIdx.x / tiles_n, tn = blockIdx.x % tiles_n;
  const int64_t m0 = tm * 64, n0 = tn * 64;
  __shared__ float As[16][64];
  __shared__ float Bs[16][64];
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int64_t k0 = 0; k0 < kred; k0 += 16) {
    for (int e = threadIdx.x; e < 16 * 64; e += 256) {
      const int kk = e % 16, c = e / 16;
      const bool kin = k0 + kk < kred;
      As[kk][c] = (kin && m0 + c < M) ? E[(m0 + c) * lde + k0 + kk] : 0.f;
      Bs[kk][c] = (kin && n0 + c < ncols) ? B[(n0 + c) * ldb + k0 + kk] : 0.f;
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
    if (m >= M) continue;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int64_t n = n0 + tx + 16 * v;
      if (n < ncols) C[m * ldc + n] -= acc[u][v];
    }
  }
}

static hq_status sweep_update(int impl, float* Wf, int64_t N, int64_t K, int64_t c0, int64_t ncols, const float* E,
                              const float* E_lo, int64_t lde, int64_t k0, int64_t kred, const float* Ut,
                              const float* Ut_hi, const float* Ut_lo, const int* info, int* status, cudaStream_t s) {
  const float* B = Ut + c0 * K + k0;  // B(n, k) = U^T[c0 + n][k0 + k] = U[k0 + k][c0 + n]
  if (impl == 0) {  // 3xTF32 from the pre-split operands (E, E_lo from the sweep; U^T split once)
    UpdGemm g{};
    g.C = Wf + c0;
    g.ldc = K;
    g.M = static_cast<int>(N);
    g.N = static_cast<int>(ncols);
    g.Kred = static_cast<int>(kred);
    g.A_hi = E;
    g.A_lo = E_lo;
    g.lda = lde;
    g.B_hi = Ut_hi + c0 * K + k0;
    g.B_lo = Ut_lo + c0 * K + k0;
    g.ldb = K;
    g.skip = info;
    g.status = status;
    return upd_gemm(g, s);
  }
  if (impl == 1) {
    const int64_t ctas = ceil_div(N, 64) * ceil_div(ncols, 64);
    update_simt_kernel<<<static_cast<unsigned>(ctas), 256, 0, s>>>(Wf + c0, K, N, ncols, E, lde, B, K, kred, info);
    HQ_LAUNCH_CHECK();
    return HQ_OK;
  }
  Tf32Gemm g{};
  g.C = Wf + c0;
  g.ldc = K;
  g.M = static_cast<int>(N);
  g.N = static_cast<int>(ncols);
  g.Kred = static_cast<int>(kred);
  g.A = E;
  g.lda = lde;
  g.B = B;
  g.ldb = K;
  g.alpha = -1.f;
  g.beta = 1.f;
  g.split3 = (impl == 0);
  g.skip = info;
  g.status = status;
  return tf32_gemm(g, s);
}

}  // namespace hq
