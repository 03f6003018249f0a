// Warp-specialised tcgen05 GEMM used by two stages of the path:
//
//   kSyrkBF16   H[i, j] += sum_t X[t, i] X[t, j] over the lower-triangle tiles of H
//               (bf16 X, both operands MN-major straight from X's row-major layout);
//   kUpdateTF32 C[r, col0 + c] -= sum_k A[r, k] B[b_y0 + c, b_x0 + k]
//               (tf32, both operands K-major): the GPTQ trailing update
//               W[:, J+B:] -= Err * U[J:J+B, J+B:] with B = U^T stored row-major.
//
// One 128 x 256 output tile per CTA, accumulated in TMEM.  Warp 0 is the TMA producer, warp 1
// allocates TMEM and issues the MMAs (one thread), the remaining warps drain the accumulator
// (tcgen05.ld) and apply the epilogue.  A 4-stage shared-memory ring of 128-byte-swizzled
// tiles connects TMA and the tensor core through mbarriers.
//
// The tensor core's fp32 accumulation loses precision in proportion to the number of MMAs
// chained into one accumulator (measured: 1.2e-5 relative Frobenius error after 256 chained
// K=16 steps).  The SYRK therefore chains at most kSyrkSegK contraction rows (1024 tokens,
// 64 MMAs) per TMEM accumulator: two accumulators (512 TMEM columns) alternate, and eight
// epilogue warps add each finished segment into fp32 registers with round-to-nearest while
// the tensor core fills the other accumulator.  The update GEMM contracts only 128 columns.
//
// Every wait is bounded: on expiry the CTA records HQ_ERR_TIMEOUT, waits (bounded) for its
// in-flight TMA and MMA work, frees TMEM and returns.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace hq {

enum class GemmMode { kSyrkBF16 = 0, kUpdateTF32 = 1 };

struct GemmArgs {
  float* C;       // fp32 output, row-major
  int64_t ldc;    // its leading dimension (elements)
  int M;          // output rows
  int Ncols;      // output columns (kUpdateTF32) / K (kSyrkBF16)
  int Kred;       // contraction length
  int col0;       // first output column (kUpdateTF32)
  int b_x0;       // contraction offset into B's tensor map (kUpdateTF32)
  int b_y0;       // row offset into B's tensor map (kUpdateTF32)
  int tiles_n;    // column tiles (kUpdateTF32)
  const int* skip;  // optional device flag: non-zero -> CTA does nothing (failed factorisation)
  int* status;    // optional device status word
};

constexpr int kGemmBM = 128;
constexpr int kGemmBN = 256;
constexpr int kGemmStages = 4;
constexpr int kGemmStageBytes = 49152;  // A 16 KB + B 32 KB in both modes
constexpr int kGemmSmemBytes = kGemmStages * kGemmStageBytes + 1024 /*align*/ + 256 /*barriers*/;
constexpr int kSyrkSegK = 1024;         // contraction rows chained in one TMEM accumulator

// Producer warp + MMA warp + epilogue warps (8 for the SYRK: two per TMEM lane quadrant,
// 128 columns each; 4 for the update: one per quadrant, 256 columns each).
__host__ __device__ constexpr int gemm_threads(GemmMode m) { return m == GemmMode::kSyrkBF16 ? 320 : 192; }

// Lower-triangle tile enumeration of a K x K output with BM x BN tiles: tile row bi holds
// column tiles bj with bj * BN <= bi * BM + BM - 1.
__host__ __device__ inline int syrk_tiles_in_row(int bi, int tiles_n) {
  int c = (bi * kGemmBM + kGemmBM - 1) / kGemmBN + 1;
  return c < tiles_n ? c : tiles_n;
}

template <GemmMode MODE>
__global__ void __launch_bounds__(gemm_threads(MODE), 1)
    umma_gemm_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                     GemmArgs args) {
  constexpr bool kSyrk = (MODE == GemmMode::kSyrkBF16);
  constexpr int kAccCols = kSyrk ? 512 : 256;        // TMEM columns allocated
  constexpr int kEpiWarps = kSyrk ? 8 : 4;
  constexpr int BK = kSyrk ? 64 : 32;                // contraction rows per stage (128 bytes)
  constexpr int kSegIters = kSyrk ? kSyrkSegK / BK : (1 << 30);

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kGemmStages * kGemmStageBytes);
  uint64_t* empty = full + kGemmStages;
  uint64_t* accf = empty + kGemmStages;  // [2] accumulator filled
  uint64_t* acce = accf + 2;             // [2] accumulator drained
  uint64_t* drain = acce + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (args.skip != nullptr && *args.skip != 0) return;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- tile coordinates
  int tm, tn;
  if (kSyrk) {
    const int tiles_n = (args.Ncols + kGemmBN - 1) / kGemmBN;
    int t = blockIdx.x;
    int bi = 0;
    while (true) {
      int c = syrk_tiles_in_row(bi, tiles_n);
      if (t < c) break;
      t -= c;
      ++bi;
    }
    tm = bi;
    tn = t;
  } else {
    tm = blockIdx.x / args.tiles_n;
    tn = blockIdx.x % args.tiles_n;
  }
  const int m0 = tm * kGemmBM;
  const int n0 = tn * kGemmBN;
  const int kiters = (args.Kred + BK - 1) / BK;
  const int nseg = (kiters + kSegIters - 1) / kSegIters;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kGemmStages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(&accf[a], 1);
      ptx::mbar_init(&acce[a], kEpiWarps);
    }
    ptx::mbar_init(drain, 1);
    *abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, kAccCols);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  auto fail = [&]() {
    *abort_flag = 1;
    record_status(args.status, HQ_ERR_TIMEOUT);
  };

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    ptx::prefetch_tensormap(&mapA);
    ptx::prefetch_tensormap(&mapB);
    int issued = 0;
    bool ok = true;
    for (int k = 0; k < kiters; ++k) {
      const int s = k % kGemmStages;
      const int round = k / kGemmStages;
      if (k >= kGemmStages && !ptx::mbar_wait(&empty[s], (round - 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      uint8_t* sa = smem + s * kGemmStageBytes;
      uint8_t* sb = sa + 16384;
      ptx::mbar_arrive_expect_tx(&full[s], kGemmStageBytes);
      if (kSyrk) {
        const int t0 = k * BK;
        ptx::tma_load_2d(sa, &mapA, m0, t0, &full[s]);
        ptx::tma_load_2d(sa + 8192, &mapA, m0 + 64, t0, &full[s]);
#pragma unroll
        for (int c = 0; c < 4; ++c) ptx::tma_load_2d(sb + c * 8192, &mapB, n0 + 64 * c, t0, &full[s]);
      } else {
        const int kx = k * BK;
        ptx::tma_load_2d(sa, &mapA, kx, m0, &full[s]);
        ptx::tma_load_2d(sb, &mapB, args.b_x0 + kx, args.b_y0 + n0, &full[s]);
      }
      ++issued;
    }
    if (!ok) {
      fail();
      // let the copies already issued land before the CTA's shared memory goes away
      const int first = issued > kGemmStages ? issued - kGemmStages : 0;
      for (int k = first; k < issued; ++k) ptx::mbar_wait(&full[k % kGemmStages], (k / kGemmStages) & 1, nullptr);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t kIdesc = kSyrk ? ptx::idesc(ptx::kFmtBF16, kGemmBM, kGemmBN, true, true)
                                      : ptx::idesc(ptx::kFmtTF32, kGemmBM, kGemmBN, false, false);
    bool ok = true;
    int k = 0;
    for (int seg = 0; seg < nseg && ok; ++seg) {
      const int acc = seg & 1;
      if (seg >= 2 && !ptx::mbar_wait(&acce[acc], ((seg >> 1) - 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const uint32_t dacc = tmem + static_cast<uint32_t>(acc * kGemmBN);
      const int kbeg = seg * kSegIters;
      const int kend = (kiters < kbeg + kSegIters) ? kiters : kbeg + kSegIters;
      for (; k < kend; ++k) {
        const int s = k % kGemmStages;
        if (!ptx::mbar_wait(&full[s], (k / kGemmStages) & 1, abort_flag)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t sa = ptx::smem_u32(smem + s * kGemmStageBytes);
        const uint32_t sb = sa + 16384;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          uint64_t ad, bd;
          if (kSyrk) {
            // MN-major: 64-element chunks 8 KB apart (LBO), 8-row groups 1 KB apart (SBO);
            // each MMA consumes 16 rows of t = 2 KB.
            ad = ptx::sdesc_sw128(sa + kk * 2048, 8192, 1024);
            bd = ptx::sdesc_sw128(sb + kk * 2048, 8192, 1024);
            ptx::mma_bf16(dacc, ad, bd, kIdesc, (k > kbeg || kk > 0) ? 1u : 0u);
          } else {
            // K-major: 8-row groups 1 KB apart (SBO); each MMA consumes 8 tf32 = 32 bytes.
            ad = ptx::sdesc_sw128(sa + kk * 32, 16, 1024);
            bd = ptx::sdesc_sw128(sb + kk * 32, 16, 1024);
            ptx::mma_tf32(dacc, ad, bd, kIdesc, (k > kbeg || kk > 0) ? 1u : 0u);
          }
        }
        ptx::mma_commit(&empty[s]);
      }
      if (ok) ptx::mma_commit(&accf[acc]);
    }
    if (!ok) {
      fail();
      ptx::mma_commit(drain);
      ptx::mbar_wait(drain, 0, nullptr);
    }
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const int r = m0 + q * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    if (kSyrk) {
      const int h = (warp - 2) >> 2;  // which 128-column half of the tile
      float sum[128];
#pragma unroll
      for (int i = 0; i < 128; ++i) sum[i] = 0.f;
      bool ok = true;
      for (int seg = 0; seg < nseg; ++seg) {
        const int acc = seg & 1;
        if (!ptx::mbar_wait(&accf[acc], (seg >> 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        ptx::tmem_add128(tmem + lane_off + static_cast<uint32_t>(acc * kGemmBN + h * 128), sum);
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&acce[acc]);
      }
      if (!ok) fail();
      // H tile += sums, coalesced: once every MMA has completed the stage ring is free; the
      // sums go there as a 128 x 256 tile (row r: 16-byte piece p at p ^ (r & 7)), then each
      // warp adds rows of it to H with 16-byte accesses along the row.  Every epilogue warp
      // meets the named barrier, also after a failed wait.
      float4* tile = reinterpret_cast<float4*>(smem);
      const int rl = q * 32 + lane;  // tile row
      if (ok) {
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const int p = h * 32 + k;
          tile[rl * 64 + (p ^ (rl & 7))] = make_float4(sum[4 * k], sum[4 * k + 1], sum[4 * k + 2], sum[4 * k + 3]);
        }
      }
      asm volatile("bar.sync 1, 256;" ::: "memory");
      if (ok) {
        const bool vec = (reinterpret_cast<uintptr_t>(args.C) & 15) == 0 && (args.ldc % 4) == 0;
        for (int rr = warp - 2; rr < kGemmBM; rr += kEpiWarps) {
          const int row = m0 + rr;
          if (row >= args.M) break;
          float* hrow = args.C + static_cast<int64_t>(row) * args.ldc;
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            const int p = lane + 32 * half;  // 16-byte piece of the tile row
            const int col = n0 + 4 * p;
            const float4 v = tile[rr * 64 + (p ^ (rr & 7))];
            if (vec && col + 3 <= row && col + 3 < args.Ncols) {  // entirely in the lower part
              float4 o = *reinterpret_cast<float4*>(hrow + col);
              o.x += v.x;
              o.y += v.y;
              o.z += v.z;
              o.w += v.w;
              *reinterpret_cast<float4*>(hrow + col) = o;
            } else {
              const float vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int e = 0; e < 4; ++e)
                if (col + e <= row && col + e < args.Ncols) hrow[col + e] += vv[e];
            }
          }
        }
      }
    } else {
      if (kiters == 0 || ptx::mbar_wait(&accf[0], 0, abort_flag)) {
        ptx::tc_fence_after();
        for (int c = 0; c < kGemmBN; c += 16) {
          float v[16];
          ptx::tmem_ld16(tmem + lane_off + c, v);
          if (r < args.M) {
            float* row = args.C + static_cast<int64_t>(r) * args.ldc + args.col0;
            const int cb = n0 + c;
            if (cb + 16 <= args.Ncols && ((reinterpret_cast<uintptr_t>(row + cb) & 15) == 0)) {
#pragma unroll
              for (int i = 0; i < 16; i += 4) {
                float4 w = *reinterpret_cast<float4*>(row + cb + i);
                w.x -= v[i];
                w.y -= v[i + 1];
                w.z -= v[i + 2];
                w.w -= v[i + 3];
                *reinterpret_cast<float4*>(row + cb + i) = w;
              }
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i)
                if (cb + i < args.Ncols) row[cb + i] -= v[i];
            }
          }
        }
      } else {
        fail();
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kAccCols);
  }
}

}  // namespace hq
