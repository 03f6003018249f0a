// GPTQ error-compensated column sweep (ork-driver wiki "Exp 2026-08-18 GPTQ Int4",
// experiment summary: error-feedback sweep, uniform symmetric int4 [-8, 7], per-(row, group)
// scale absmax/7, dequant w = code * scale; qerr definition in the same page).
//
// The sweep walks K in 128-column blocks grouped into panels of P columns (P = 512, or a
// multiple of the group size when groups are wider than a block).  Per block:
//   * sweep_block_kernel: the sequential part.  Sixteen lanes share two rows: lane l holds
//     columns l, l+16, ..., l+112 of both rows as 8 "slots" each, in registers.  The columns
//     are visited in rounds of sixteen; at the end of a round every lane shifts its slots down
//     by one, so the column being quantised is always slot 0 of lane (j mod 16), a
//     compile-time lane inside the 16-way unrolled round.  Per column j and row: group scale
//     at a group start (16-lane absmax), broadcast of w_j, code c = clamp(rint(w_j / s), -8, 7),
//     residual d = w_j - c s, and the feedback w_k -= d U'[j, k] for k > j, where
//     U' = diag(U)^-1 U is U with each row divided by its diagonal entry, so that
//     d U'[j, k] = e U[j, k] with the error e = d / U[j, j] of the method.  The factorisation
//     hands over each 128 x 128 diagonal block of U' already permuted into the lanes' slot
//     order (zero on and below the diagonal) so that a lane reads its 8 values for column j
//     with two conflict-free 16-byte loads shared by its two rows.  At the end of a round each
//     lane re-derives the code and residual of the column it holds in slot 0 (the same
//     arithmetic on the same final weight) and stages them; the block then writes the
//     residuals into the panel's buffer, the packed int4 codes, the scales and fp64 partial
//     sums of the qerr numerator and denominator over the ORIGINAL weights.  A CTA holds
//     ceil(N / 148) rows rounded up to a multiple of four, so one wave covers the layer.
//   * inner lazy update of the rest of the panel, W[:, b+128 : panel end] -= D_b U'[b, ...]
//     (contraction 128; the panel's N x P working weights stay in L2);
// and after the panel the outer lazy update W[:, panel end:] -= D_panel U'[panel, ...] with
// contraction P.  Both updates are dense contractions on the tensor cores (gemm_upd.cu,
// 3xTF32) with B = U'^T row-major.  Blocking only reorders exact sums: every column still
// receives the feedback of every earlier column before it is quantised.
// U'^T and the packed diagonal blocks of U' come from factor.cu.  The working copy of W is
// fp32 in the workspace.
#include <cuda_bf16.h>

#include <type_traits>

#include "common.cuh"
#include "kernels.cuh"

namespace hq {

constexpr int kBlk = 128;                    // sweep block width (== kSweepBlk)
constexpr int kLanesPerRow = 16;             // lanes sharing one row's 128 columns
constexpr int kSlots = kBlk / kLanesPerRow;  // 8 columns per lane and row
constexpr int kRowsPerWarp = 4;              // two 16-lane groups x two rows
constexpr int kMaxSweepThreads = 1024;
constexpr int kMaxRowsPerCta = kMaxSweepThreads / 32 * kRowsPerWarp;  // 128
static_assert(kBlk == kSweepBlk, "packed U' blocks are made for this block width");

// Rows per CTA: the layer's rows spread over one wave of 148 CTAs, a multiple of 4, 4..128.
static int sweep_rows_per_cta(int64_t N) {
  int64_t r = ceil_div(N, int64_t(148));
  r = ceil_div(r, int64_t(kRowsPerWarp)) * kRowsPerWarp;
  if (r < kRowsPerWarp) r = kRowsPerWarp;
  if (r > kMaxRowsPerCta) r = kMaxRowsPerCta;
  return static_cast<int>(r);
}

// Rows per CTA up to which the updates inside a panel run in the sweep kernel itself (one launch
// per panel; fp32 FMAs on the CUDA cores from the band of U'); with more rows they run as
// tensor-core GEMM launches between the blocks.
constexpr int kFusedMaxRows = 64;
constexpr int kUsK = 32;       // band rows per staged chunk
constexpr int kLD = kBlk + 4;  // row of the residual stage, 16-byte aligned

static size_t sweep_smem_bytes(int rows, bool fused) {
  size_t floats = static_cast<size_t>(kBlk) * kBlk + static_cast<size_t>(rows) * kLD + rows * 4 + kBlk;
  if (fused) floats += 2 * static_cast<size_t>(kUsK) * kBlk;
  return floats * sizeof(float) + static_cast<size_t>(rows) * kBlk;
}

struct SweepArgs {
  float* Wf;
  int64_t N, K;
  const float* Upack;  // packed diagonal blocks of U' (sweep_upack_offset order), kBlk^2 floats each
  const float* band;   // the bands of U' (kSweepBand), read by the in-kernel panel updates
  int group;
  float* Err;        // panel residual buffer [N, P] (the tf32 part when Err_lo is set)
  float* Err_lo;     // NULL, or the fp32 remainder of each residual (Err + Err_lo = residual)
  int64_t err_ld;    // P
  int err_col;       // column of the launch's first block inside the panel buffer
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

// c = clamp(rint(w / s), -8, 7) with w / s the IEEE fp32 quotient; rs = 1 / s, or 0 when
// s == 0 (then c = 0 for every finite w).  w * rs is within a couple of ulps of the quotient,
// so it rounds the same way unless it lies within 1e-5 of a half-integer; only then is the
// exact division taken.  Rounding to nearest-even uses the 1.5 * 2^23 shift (exact for
// |q| < 2^22; larger values are clamped anyway).  Two rows at a time, one branch for both.
// The rare exact path, out of line so that the unrolled sweep loop stays compact.
__device__ __noinline__ float exact_round_quotient(float w, float s) { return rintf(__fdiv_rn(w, s)); }

__device__ __forceinline__ void quant_pair(float wa, float sa, float rsa, float wb, float sb, float rsb, float& ca,
                                           float& cb) {
  constexpr float kShift = 12582912.f;
  constexpr float kNear = 0.5f - 1e-5f;
  const float qa = wa * rsa, qb = wb * rsb;
  float ra = (qa + kShift) - kShift;
  float rb = (qb + kShift) - kShift;
  if (fmaxf(fabsf(qa - ra), fabsf(qb - rb)) > kNear) {
    if (fabsf(qa - ra) > kNear) ra = exact_round_quotient(wa, sa);
    if (fabsf(qb - rb) > kNear) rb = exact_round_quotient(wb, sb);
  }
  ca = fminf(fmaxf(ra, -8.f), 7.f);
  cb = fminf(fmaxf(rb, -8.f), 7.f);
}

__device__ __forceinline__ float recip_or_zero(float s) { return s > 0.f ? __frcp_rn(s) : 0.f; }

// The updates a block owes the later blocks of its panel, for this CTA's rows:
//   W[r, j0 + kBlk : p1) -= D[r, :] U'[j0 : j0 + kBlk, j0 + kBlk : p1)
// D the block's residuals (the stage `dst`), U' read from the block's band, fp32 FMAs in k order.
// Warp w takes rows 4w .. 4w + 3 (the CTA has exactly rows / 4 warps) and lane l the columns
// 4l .. 4l + 3 of each 128-column chunk; the band passes through shared memory in 32 x 128
// chunks by cp.async, the next chunk in flight while one is used.  Called by all threads with
// the caller's cp.async groups possibly pending; returns with none pending, after a barrier.
__device__ __forceinline__ void panel_update(const SweepArgs& a, int j0, int p1, int64_t r0, const float* dst,
                                             float* Us) {
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t K = a.K;
  const int j1 = j0 + kBlk;
  constexpr int kKC = kBlk / kUsK;  // band chunks per 128 columns
  const int nunits = (p1 - j1) / kBlk * kKC;
  const float* band = a.band + static_cast<int64_t>(j0 / kBlk) * kBlk * kSweepBand;
  if (!HQ_IN_BOUNDS(p1 <= K && p1 - j1 > 0 && p1 - j1 <= kSweepBand && (p1 - j1) % kBlk == 0)) {
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
    return;  // uniform over the CTA
  }
  const uint32_t us0 = static_cast<uint32_t>(__cvta_generic_to_shared(Us));
  auto stage = [&](int u) {  // chunk u: band rows 32 (u % 4) .., columns 128 (u / 4) ..
    const float* src = band + static_cast<int64_t>((u % kKC) * kUsK) * kSweepBand + (u / kKC) * kBlk;
    const uint32_t d0 = us0 + static_cast<uint32_t>((u & 1) * kUsK * kBlk * 4);
    for (int e = tid; e < kUsK * kBlk / 4; e += blockDim.x) {
      const int k = e / (kBlk / 4), q = e % (kBlk / 4);
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d0 + 16u * e), "l"(src + k * kSweepBand + 4 * q)
                   : "memory");
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  stage(0);
  float acc[4][4];
#pragma unroll
  for (int r = 0; r < 4; ++r)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;
#pragma unroll 1
  for (int u = 0; u < nunits; ++u) {
    if (u + 1 < nunits) {
      stage(u + 1);
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    } else {
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    }
    __syncthreads();
    const int kc = u % kKC;
    const float* ub = Us + (u & 1) * kUsK * kBlk + 4 * lane;
    const float* db = dst + (4 * warp) * kLD + kc * kUsK;
#pragma unroll
    for (int k = 0; k < kUsK; k += 4) {
      float dv[4][4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float4 d4 = *reinterpret_cast<const float4*>(db + r * kLD + k);
        dv[r][0] = d4.x;
        dv[r][1] = d4.y;
        dv[r][2] = d4.z;
        dv[r][3] = d4.w;
      }
#pragma unroll
      for (int kk = 0; kk < 4; ++kk) {
        const float4 u4 = *reinterpret_cast<const float4*>(ub + (k + kk) * kBlk);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          acc[r][0] = fmaf(dv[r][kk], u4.x, acc[r][0]);
          acc[r][1] = fmaf(dv[r][kk], u4.y, acc[r][1]);
          acc[r][2] = fmaf(dv[r][kk], u4.z, acc[r][2]);
          acc[r][3] = fmaf(dv[r][kk], u4.w, acc[r][3]);
        }
      }
    }
    if (kc == kKC - 1) {  // this 128-column chunk is complete: W -= acc
      const int64_t col = j1 + (u / kKC) * kBlk + 4 * lane;
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const int64_t row = r0 + 4 * warp + r;
        if (row < a.N && HQ_IN_BOUNDS(col + 3 < K)) {
          float4* wp = reinterpret_cast<float4*>(a.Wf + row * K + col);
          float4 w = *wp;
          w.x -= acc[r][0];
          w.y -= acc[r][1];
          w.z -= acc[r][2];
          w.w -= acc[r][3];
          *wp = w;
        }
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] = 0.f;
      }
    }
    __syncthreads();  // this chunk's buffer is refilled two chunks later
  }
}


// GS: group size when it is 32, 64 or 128 (scales computed inside the block), or 0 when the
// group spans several blocks (scale computed at the group's first block from Wf).
// The CTA sweeps the blocks j0 = p0, p0 + kBlk, .. < p1 of its rows.  With kFused the updates that
// each block owes the later blocks of the panel [p0, p1) run here as well (panel_update), between
// the blocks; otherwise a launch covers one block and the host runs those updates as GEMMs.
template <int GS, bool kFused>
__global__ void __launch_bounds__(kFused ? kFusedMaxRows / kRowsPerWarp * 32 : kMaxSweepThreads)
    sweep_block_kernel(SweepArgs a, int p0, int p1) {
  if (*a.info != 0) return;
  extern __shared__ float4 sm4[];
  float* Ur = reinterpret_cast<float*>(sm4);      // packed U' block
  const int rows = static_cast<int>(blockDim.x / 32) * kRowsPerWarp;
  float* dst = Ur + kBlk * kBlk;                   // [rows][kLD]: residuals
  float* scl_s = dst + rows * kLD;                 // [rows][4]
  float* sup_s = scl_s + rows * 4;                 // [kBlk]: U'[j][j + 1], 0 for the last j
  float* Us = sup_s + kBlk;                        // kFused: [2][kUsK][kBlk], chunks of the band
  int8_t* code_s = reinterpret_cast<int8_t*>(Us + (kFused ? 2 * kUsK * kBlk : 0));  // [rows][kBlk]

  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31, l = lane & (kLanesPerRow - 1);
  const int rlA = warp * kRowsPerWarp + (lane >> 4), rlB = rlA + 2;
  const int64_t r0 = static_cast<int64_t>(blockIdx.x) * rows;
  const int64_t rowA = r0 + rlA, rowB = r0 + rlB;
  const bool vA = rowA < a.N, vB = rowB < a.N;
  const int64_t K = a.K;

  // packed U' block of the columns from jb on -> shared memory, all copies in flight at once
  auto load_upack = [&](int jb) {
    const float4* src = reinterpret_cast<const float4*>(a.Upack + static_cast<int64_t>(jb / kBlk) * (kBlk * kBlk));
    const uint32_t dst0 = static_cast<uint32_t>(__cvta_generic_to_shared(sm4));
    if (HQ_IN_BOUNDS(jb >= 0 && jb + kBlk <= a.K))
      for (int e = tid; e < kBlk * kBlk / 4; e += blockDim.x)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst0 + 16u * e), "l"(src + e) : "memory");
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  load_upack(p0);
#pragma unroll 1
  for (int j0 = p0;; j0 += kBlk) {  // up to the last block (`more` false; always after one without kFused)
  if (!HQ_IN_BOUNDS(j0 >= 0 && j0 + kBlk <= a.K && a.err_col + (j0 - p0) + kBlk <= a.err_ld)) {
    asm volatile("cp.async.wait_all;" ::: "memory");
    return;  // uniform over the CTA
  }
  {
    for (int t = tid; t < kBlk; t += blockDim.x) {
      const int c = t + 1;
      sup_s[t] = c < kBlk ? a.Upack[static_cast<int64_t>(j0 / kBlk) * (kBlk * kBlk) +
                                    sweep_upack_offset(t, c & (kLanesPerRow - 1), c / kLanesPerRow - t / kLanesPerRow)]
                          : 0.f;
    }
  }
  float w0[kSlots], w1[kSlots];
#pragma unroll
  for (int m = 0; m < kSlots; ++m) {
    w0[m] = vA ? a.Wf[rowA * K + j0 + kLanesPerRow * m + l] : 0.f;
    w1[m] = vB ? a.Wf[rowB * K + j0 + kLanesPerRow * m + l] : 0.f;
  }

  float sA = 0.f, rsA = 0.f, sB = 0.f, rsB = 0.f;
  if (GS == 0) {
    // the group spans several blocks: its scale is taken at its first block from the current
    // weights of all its columns, and read back in the later blocks
    const int G = a.group;
    const int64_t g = j0 / G;
    if (j0 % G == 0) {
      float amA = 0.f, amB = 0.f;
      for (int i = l; i < G; i += kLanesPerRow) {
        if (vA) amA = fmaxf(amA, fabsf(a.Wf[rowA * K + j0 + i]));
        if (vB) amB = fmaxf(amB, fabsf(a.Wf[rowB * K + j0 + i]));
      }
#pragma unroll
      for (int x = 1; x < kLanesPerRow; x <<= 1) {
        amA = fmaxf(amA, __shfl_xor_sync(0xffffffffu, amA, x));
        amB = fmaxf(amB, __shfl_xor_sync(0xffffffffu, amB, x));
      }
      sA = __fdiv_rn(amA, 7.f);
      sB = __fdiv_rn(amB, 7.f);
      if (l == 0 && vA) a.scales[rowA * (K / G) + g] = sA;
      if (l == 0 && vB) a.scales[rowB * (K / G) + g] = sB;
    } else {
      sA = vA ? a.scales[rowA * (K / G) + g] : 0.f;
      sB = vB ? a.scales[rowB * (K / G) + g] : 0.f;
    }
    rsA = recip_or_zero(sA);
    rsB = recip_or_zero(sB);
  }
  asm volatile("cp.async.wait_all;" ::: "memory");
  __syncthreads();


  const int src_base = lane & kLanesPerRow;  // first lane of this 16-lane group
  // Every lane carries the current value of the column being quantised (curA, curB): the
  // value of column j + 1 is fetched from its owner lane BEFORE column j's feedback and then
  // updated locally with the same fma the owner applies, so the broadcast is off the
  // column-to-column dependency chain and the result is bit-identical to the owner's slot.
  float curA = __shfl_sync(0xffffffffu, w0[0], src_base);
  float curB = __shfl_sync(0xffffffffu, w1[0], src_base);
  // One round of 16 columns with S live slots: in round R slot m holds column 16 (R + m) + l, so
  // slots m >= 8 - R lie past the block (zero, and zero in U'); rounds 2r and 2r + 1 update the
  // first 8 - 2r slots only (the skipped updates would add zero to zero).
  auto sweep_round = [&](int R, auto slots) {
    constexpr int S = decltype(slots)::value;
#pragma unroll
    for (int jr = 0; jr < kLanesPerRow; ++jr) {
      const int j = kLanesPerRow * R + jr;
      if (GS != 0 && jr == 0 && (R % (GS == 0 ? 1 : GS / kLanesPerRow)) == 0) {
        constexpr int kGS = (GS == 0 ? kLanesPerRow : GS) / kLanesPerRow;  // slots per group
        float amA = 0.f, amB = 0.f;
#pragma unroll
        for (int m = 0; m < kGS; ++m) {
          amA = fmaxf(amA, fabsf(w0[m]));
          amB = fmaxf(amB, fabsf(w1[m]));
        }
#pragma unroll
        for (int x = 1; x < kLanesPerRow; x <<= 1) {
          amA = fmaxf(amA, __shfl_xor_sync(0xffffffffu, amA, x));
          amB = fmaxf(amB, __shfl_xor_sync(0xffffffffu, amB, x));
        }
        sA = __fdiv_rn(amA, 7.f);
        sB = __fdiv_rn(amB, 7.f);
        rsA = recip_or_zero(sA);
        rsB = recip_or_zero(sB);
        if (l == 0) {
          scl_s[rlA * 4 + j / (GS == 0 ? kBlk : GS)] = sA;
          scl_s[rlB * 4 + j / (GS == 0 ? kBlk : GS)] = sB;
        }
      }
      const float4 u0 = *reinterpret_cast<const float4*>(Ur + sweep_upack_offset(j, l, 0));
      const float4 u1 = S > 4 ? *reinterpret_cast<const float4*>(Ur + sweep_upack_offset(j, l, 4))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
      const float uu[8] = {u0.x, u0.y, u0.z, u0.w, u1.x, u1.y, u1.z, u1.w};
      const float usup = sup_s[j];
      // column j + 1 before column j's feedback: slot 0 of lane jr + 1, or after the round's
      // last column slot 1 of lane 0
      const float preA = __shfl_sync(0xffffffffu, jr + 1 < kLanesPerRow ? w0[0] : w0[1], src_base | ((jr + 1) & 15));
      const float preB = __shfl_sync(0xffffffffu, jr + 1 < kLanesPerRow ? w1[0] : w1[1], src_base | ((jr + 1) & 15));
      float ca, cb;
      quant_pair(curA, sA, rsA, curB, sB, rsB, ca, cb);
      const float da = fmaf(-ca, sA, curA);
      const float db = fmaf(-cb, sB, curB);
      // U' is zero in the packed block on and left of column j: lanes l <= jr keep slot 0
#pragma unroll
      for (int m = 0; m < S; ++m) {
        w0[m] = fmaf(-da, uu[m], w0[m]);
        w1[m] = fmaf(-db, uu[m], w1[m]);
      }
      curA = fmaf(-da, usup, preA);
      curB = fmaf(-db, usup, preB);
    }
  };
#pragma unroll 1
  for (int R = 0; R < kSlots; ++R) {
    switch (R >> 1) {
      case 0: sweep_round(R, std::integral_constant<int, 8>{}); break;
      case 1: sweep_round(R, std::integral_constant<int, 6>{}); break;
      case 2: sweep_round(R, std::integral_constant<int, 4>{}); break;
      default: sweep_round(R, std::integral_constant<int, 2>{}); break;
    }
    {  // slot 0 of lane l now holds the final weight of column 16 R + l
      const int col = kLanesPerRow * R + l;
      float cA, cB;
      quant_pair(w0[0], sA, rsA, w1[0], sB, rsB, cA, cB);
      dst[rlA * kLD + col] = fmaf(-cA, sA, w0[0]);
      dst[rlB * kLD + col] = fmaf(-cB, sB, w1[0]);
      code_s[rlA * kBlk + col] = static_cast<int8_t>(cA);
      code_s[rlB * kBlk + col] = static_cast<int8_t>(cB);
    }
#pragma unroll
    for (int m = 0; m < kSlots - 1; ++m) {
      w0[m] = w0[m + 1];
      w1[m] = w1[m + 1];
    }
    w0[kSlots - 1] = 0.f;
    w1[kSlots - 1] = 0.f;
  }
  if (GS == 0 && l == 0) {
    scl_s[rlA * 4] = sA;
    scl_s[rlB * 4] = sB;
  }
  __syncthreads();
  const bool more = kFused && j0 + kBlk < p1;
  if (more) load_upack(j0 + kBlk);  // Ur is free: the next block's U' arrives during the epilogue

  // residuals -> panel buffer (coalesced rows), codes -> packed bytes, scales, qerr partials
  const int err_col = a.err_col + (j0 - p0);
  const int nwarps = static_cast<int>(blockDim.x / 32);
  for (int r = warp; r < rows; r += nwarps) {
    if (r0 + r >= a.N) break;
    const float* srcr = dst + r * kLD + 4 * lane;
    const float4 e4 = make_float4(srcr[0], srcr[1], srcr[2], srcr[3]);
    if (a.Err_lo == nullptr) {
      reinterpret_cast<float4*>(a.Err + (r0 + r) * a.err_ld + err_col)[lane] = e4;
    } else {  // split for the 3xTF32 updates: tf32 part (low 13 mantissa bits cleared) + remainder
      const float4 h4 = make_float4(__uint_as_float(__float_as_uint(e4.x) & 0xFFFFE000u),
                                    __uint_as_float(__float_as_uint(e4.y) & 0xFFFFE000u),
                                    __uint_as_float(__float_as_uint(e4.z) & 0xFFFFE000u),
                                    __uint_as_float(__float_as_uint(e4.w) & 0xFFFFE000u));
      reinterpret_cast<float4*>(a.Err + (r0 + r) * a.err_ld + err_col)[lane] = h4;
      reinterpret_cast<float4*>(a.Err_lo + (r0 + r) * a.err_ld + err_col)[lane] =
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
    for (int e = tid; e < rows * ng; e += blockDim.x) {
      const int r = e / ng, g = e % ng;
      if (r0 + r < a.N) a.scales[(r0 + r) * (K / (GS == 0 ? 1 : GS)) + j0 / (GS == 0 ? 1 : GS) + g] = scl_s[r * 4 + g];
    }
  }
  // qerr partial sums over the ORIGINAL weights in fp64: warp w takes rows w + i * nwarps
  // (i < 4, exactly the CTA's rows), lane columns 4 lane .. 4 lane + 3; all loads issued first
  double num = 0.0, den = 0.0;
  {
    float wo[kRowsPerWarp][4];
#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
      const int64_t row = r0 + warp + i * nwarps;
#pragma unroll
      for (int c = 0; c < 4; ++c) wo[i][c] = row < a.N ? load_w(a.W, a.w_dtype, row * K + j0 + 4 * lane + c) : 0.f;
    }
    float im[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) im[c] = a.imp != nullptr ? a.imp[j0 + 4 * lane + c] : 1.f;
#pragma unroll
    for (int i = 0; i < kRowsPerWarp; ++i) {
      const int r = warp + i * nwarps;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int k = 4 * lane + c;
        const double w64 = static_cast<double>(wo[i][c]);
        const double sc = static_cast<double>(GS != 0 ? scl_s[r * 4 + k / (GS == 0 ? 1 : GS)] : scl_s[r * 4]);
        const double q = static_cast<double>(code_s[r * kBlk + k]) * sc;
        num += static_cast<double>(im[c]) * (w64 - q) * (w64 - q);
        den += static_cast<double>(im[c]) * w64 * w64;
      }
    }
  }
  for (int off = 16; off > 0; off >>= 1) {
    num += __shfl_down_sync(0xffffffffu, num, off);
    den += __shfl_down_sync(0xffffffffu, den, off);
  }
  __shared__ double red[kMaxSweepThreads / 32][2];
  if (lane == 0) {
    red[warp][0] = num;
    red[warp][1] = den;
  }
  __syncthreads();
  if (tid == 0) {
    double sn = 0.0, sd = 0.0;
    for (int wq = 0; wq < nwarps; ++wq) {
      sn += red[wq][0];
      sd += red[wq][1];
    }
    double* p = a.partials + (static_cast<int64_t>(j0 / kBlk) * gridDim.x + blockIdx.x) * 2;
    p[0] = sn;
    p[1] = sd;
  }
  if (!more) break;
  panel_update(a, j0, p1, r0, dst, Us);
  }
}

__global__ void w_prep_kernel(const void* __restrict__ W, int dt, int64_t n, float* __restrict__ Wf) {
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < n;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x)
    Wf[i] = load_w(W, dt, i);
}

__global__ void __launch_bounds__(256) qerr_finalize_kernel(const double* __restrict__ partials, int64_t count,
                                                            WsHeader* hdr, double* qerr_dev,
                                                            const int* __restrict__ finfo) {
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
    // an all-zero layer has qerr 0; non-finite sums (a NaN or infinite weight) stay non-finite
    const double q = rd[0] == 0.0 ? 0.0 : sqrt(rn[0] / rd[0]);
    hdr->num = rn[0];
    hdr->den = rd[0];
    hdr->qerr = q;
    if (finfo != nullptr) hdr->info = *finfo;  // the factorisation's status, for the host
    if (qerr_dev != nullptr) *qerr_dev = q;
  }
}

hq_status launch_qerr_finalize(const double* partials, int64_t count, WsHeader* hdr, double* qerr_dev,
                               cudaStream_t s, const int* finfo) {
  qerr_finalize_kernel<<<1, 256, 0, s>>>(partials, count, hdr, qerr_dev, finfo);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

// ------------------------------------------------------------------------- layout / driver

bool gptq_shape_ok(int64_t N, int64_t K, int64_t group) {
  if (N < 1 || K < kBlk || K % kBlk != 0 || group < 32 || group % 32 != 0 || K % group != 0) return false;
  if (!(group == 32 || group == 64 || group == 128 || group % kBlk == 0)) return false;
  if (K > 65536 || N > (int64_t(1) << 31) - kMaxRowsPerCta) return false;
  return true;
}

// Panel width of the two-level update: 512 columns, or a multiple of a group wider than a
// block so that every group lies inside one panel.
static int64_t panel_width(int64_t K, int64_t group) {
  const int64_t base = group > kBlk ? group : kBlk;
  int64_t P = base * ((512 / base) > 1 ? (512 / base) : 1);
  return P < K ? P : K;
}

FactorLayout factor_layout(int64_t K) {
  FactorLayout F{};
  const size_t al = 256;
  size_t off = 0;
  F.hdr = off;
  off = round_up(off + sizeof(FactorHeader), al);
  F.upack = off;  // packed diagonal blocks of U', then its bands (contiguous: one output of the factorisation)
  F.band = off + static_cast<size_t>(K) * kBlk * sizeof(float);
  off = round_up(off + static_cast<size_t>(K) * (kBlk + kSweepBand) * sizeof(float), al);
  F.hi = off;     // U'^T strict lower triangle: tf32 part (or, for the CUDA-core updates, U'^T itself)
  off = round_up(off + static_cast<size_t>(K) * K * sizeof(float), al);
  F.lo = off;     // its fp32 remainder
  off = round_up(off + static_cast<size_t>(K) * K * sizeof(float), al);
  F.total = off;
  return F;
}

// The factorisation's scratch from offset `off` on: the recursion's temporaries T and the matrix A
// side by side (a factor buffer produced in place overlays both once they are dead), X = L^-1,
// X^T, and the int8 slices of the large products.
static void factor_scratch_layout(int64_t K, size_t off, GptqLayout& L) {
  const size_t al = 256;
  const size_t kk = static_cast<size_t>(K) * K * sizeof(double);
  L.t = off;
  off = round_up(off + kk, al);
  L.a = off;
  off = round_up(off + kk, al);
  // a factor buffer made in place (launch_gptq) must end before X, which its producers read
  const size_t fend = round_up(L.t + factor_layout(K).total, al);
  if (off < fend) off = fend;
  L.x = off;
  off = round_up(off + kk, al);
  L.xt = off;
  off = round_up(off + kk, al);
  L.slices = off;
  off = round_up(off + 2 * factor_slice_bytes(K), al);
  L.total = off;
}

GptqLayout gptq_layout(int64_t N, int64_t K, int64_t group) {
  GptqLayout L{};
  const size_t al = 256;
  L.sweep_rows = sweep_rows_per_cta(N);
  L.sweep_grid = static_cast<int>(ceil_div(N, int64_t(L.sweep_rows)));
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
  L.sweep_total = off;
  factor_scratch_layout(K, off, L);
  return L;
}

GptqLayout factor_ws_layout(int64_t K) {
  GptqLayout L{};
  L.header = 0;
  factor_scratch_layout(K, round_up(sizeof(WsHeader), 256), L);
  return L;
}

__global__ void factor_header_kernel(const WsHeader* __restrict__ hdr, FactorHeader* __restrict__ fh) {
  fh->info = hdr->info;
  fh->lam = hdr->lam;
}

hq_status launch_factorize(const float* H, int64_t K, float damp, uint8_t* ws, const GptqLayout& L, uint8_t* factor,
                           bool plain_ut, cudaStream_t s) {
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws + L.header);
  const FactorLayout F = factor_layout(K);
  float* hi = reinterpret_cast<float*>(factor + F.hi);
  float* lo = reinterpret_cast<float*>(factor + F.lo);
  hq_status st = launch_factor(H, K, damp, reinterpret_cast<double*>(ws + L.a), reinterpret_cast<double*>(ws + L.x),
                               reinterpret_cast<double*>(ws + L.xt), reinterpret_cast<double*>(ws + L.t),
                               ws + L.slices, &hdr->lam, &hdr->info, &hdr->status, true, plain_ut ? hi : nullptr,
                               reinterpret_cast<float*>(factor + F.upack), plain_ut ? nullptr : hi,
                               plain_ut ? nullptr : lo, s);
  if (st != HQ_OK) return st;
  factor_header_kernel<<<1, 1, 0, s>>>(hdr, reinterpret_cast<FactorHeader*>(factor + F.hdr));
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

// W[:, c0 : c0+ncols] -= D[:, 0:kred] * U'[k0 : k0+kred, c0 : c0+ncols]   (residuals D, row stride lde)
static hq_status sweep_update(int impl, float* Wf, int64_t N, int64_t K, int64_t c0, int64_t ncols, const float* E,
                              const float* E_lo, int64_t lde, int64_t k0, int64_t kred, const float* Ut_hi,
                              const float* Ut_lo, const int* info, int* status, cudaStream_t s);

hq_status launch_sweep(const void* W, int w_dtype, int64_t N, int64_t K, int64_t group, const float* imp,
                       uint8_t* codes, float* scales, double* qerr_dev, uint8_t* ws, const uint8_t* factor,
                       int update_impl, bool reset_header, cudaStream_t s) {
  const GptqLayout L = gptq_layout(N, K, group);
  const FactorLayout F = factor_layout(K);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws + L.header);
  double* partials = reinterpret_cast<double*>(ws + L.partials);
  float* Wf = reinterpret_cast<float*>(ws + L.wf);
  float* Err = reinterpret_cast<float*>(ws + L.err);
  float* Err_lo = reinterpret_cast<float*>(ws + L.err_lo);
  const FactorHeader* fh = reinterpret_cast<const FactorHeader*>(factor + F.hdr);
  const float* Upack = reinterpret_cast<const float*>(factor + F.upack);
  const float* band = reinterpret_cast<const float*>(factor + F.band);
  const float* Ut_hi = reinterpret_cast<const float*>(factor + F.hi);
  const float* Ut_lo = reinterpret_cast<const float*>(factor + F.lo);
  const int* info = &fh->info;
  if (reset_header) HQ_CUDA_TRY(cudaMemsetAsync(hdr, 0, sizeof(WsHeader), s));
  const bool split = (update_impl == 0);  // 3xTF32 updates take pre-split operands

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
  a.Upack = Upack;
  a.band = band;
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
  a.info = info;

  // the updates inside a panel run in the sweep kernel when a CTA's rows are few and the panel
  // lies inside the bands of U'
  const bool fused = L.sweep_rows <= kFusedMaxRows && P <= kBlk + kSweepBand;
  void (*kern)(SweepArgs, int, int) = nullptr;
  switch (group) {
    case 32: kern = fused ? sweep_block_kernel<32, true> : sweep_block_kernel<32, false>; break;
    case 64: kern = fused ? sweep_block_kernel<64, true> : sweep_block_kernel<64, false>; break;
    case 128: kern = fused ? sweep_block_kernel<128, true> : sweep_block_kernel<128, false>; break;
    default: kern = fused ? sweep_block_kernel<0, true> : sweep_block_kernel<0, false>; break;
  }
  const size_t smem = sweep_smem_bytes(L.sweep_rows, fused);
  const int threads = L.sweep_rows / kRowsPerWarp * 32;
  HQ_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem)));
  // bytes of one block: its working weights in, its residuals out (fp32), its block of U', packed
  // codes and scales out
  const double block_bytes = static_cast<double>(N) * kBlk * 8.0 + kBlk * kBlk * 4.0 + N * (kBlk / 2.0) +
                             N * (static_cast<double>(kBlk) / group) * 4.0;

  hq_status st = HQ_OK;
  for (int64_t p0 = 0; p0 < K; p0 += P) {
    const int64_t p1 = (p0 + P < K) ? p0 + P : K;
    if (fused) {
      a.err_col = 0;
      const int tm = timer_start(kTimeSweep, s);
      kern<<<L.sweep_grid, threads, smem, s>>>(a, static_cast<int>(p0), static_cast<int>(p1));
      HQ_LAUNCH_CHECK();
      // plus, for the updates inside the panel, the later columns' weights in and out and the band
      double bytes = 0.0;
      for (int64_t j1 = p0 + kBlk; j1 <= p1; j1 += kBlk)
        bytes += block_bytes + (static_cast<double>(N) * 8.0 + kBlk * 4.0) * static_cast<double>(p1 - j1);
      timer_stop(tm, bytes, s);
    } else {
      for (int64_t j0 = p0; j0 < p1; j0 += kBlk) {
        a.err_col = static_cast<int>(j0 - p0);
        const int tm = timer_start(kTimeSweep, s);
        kern<<<L.sweep_grid, threads, smem, s>>>(a, static_cast<int>(j0), static_cast<int>(j0 + kBlk));
        HQ_LAUNCH_CHECK();
        timer_stop(tm, block_bytes, s);
        const int64_t j1 = j0 + kBlk;
        if (j1 < p1) {  // inner update of the rest of the panel
          st = sweep_update(update_impl, Wf, N, K, j1, p1 - j1, Err + (j0 - p0), Err_lo + (j0 - p0), P, j0, kBlk,
                            Ut_hi, Ut_lo, info, &hdr->status, s);
          if (st != HQ_OK) return st;
        }
      }
    }
    if (p1 < K) {  // outer update of everything right of the panel
      st = sweep_update(update_impl, Wf, N, K, p1, K - p1, Err, Err_lo, P, p0, p1 - p0, Ut_hi, Ut_lo, info,
                        &hdr->status, s);
      if (st != HQ_OK) return st;
    }
  }
  return launch_qerr_finalize(partials, static_cast<int64_t>(K / kBlk) * L.sweep_grid, hdr, qerr_dev, s, info);
}

hq_status launch_gptq(const void* W, int w_dtype, int64_t N, int64_t K, const float* H, int64_t group, float damp,
                      const float* imp, uint8_t* codes, float* scales, double* qerr_dev, uint8_t* ws,
                      int update_impl, cudaStream_t s) {
  const GptqLayout L = gptq_layout(N, K, group);
  HQ_CUDA_TRY(cudaMemsetAsync(ws + L.header, 0, sizeof(WsHeader), s));
  // the factor buffer overlays the recursion's temporaries and A, both dead once it is written
  uint8_t* factor = ws + L.t;
  static_assert(sizeof(FactorHeader) <= 256, "factor header");
  hq_status st = launch_factorize(H, K, damp, ws, L, factor, update_impl != 0, s);
  if (st != HQ_OK) return st;
  return launch_sweep(W, w_dtype, N, K, group, imp, codes, scales, qerr_dev, ws, factor, update_impl, false, s);
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
                              const float* E_lo, int64_t lde, int64_t k0, int64_t kred, const float* Ut_hi,
                              const float* Ut_lo, const int* info, int* status, cudaStream_t s) {
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
  // fp32 CUDA cores, with U'^T itself in the place of its tf32 part:
  // B(n, k) = U'^T[c0 + n][k0 + k] = U'[k0 + k][c0 + n]
  const int64_t ctas = ceil_div(N, 64) * ceil_div(ncols, 64);
  update_simt_kernel<<<static_cast<unsigned>(ctas), 256, 0, s>>>(Wf + c0, K, N, ncols, E, lde, Ut_hi + c0 * K + k0,
                                                                  K, kred, info);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

}  // namespace hq
