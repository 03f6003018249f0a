// General fp32 GEMM on the tcgen05 tensor cores (kind::tf32), used by the factorisation and by
// the GPTQ trailing updates:
//
//   C[m, n] = beta * C[m, n] + alpha * sum_k A[m, k] * B(n, k)     m < M, n < N
//
// A and B are row-major fp32 views [M, Kred] and [N, Kred] (both K-major operands: B(n, k) =
// B[n, k]).  Optionally only the lower part (row0 + m >= col0 + n) of C is written.
//
// Precision.  With SPLIT3 every operand x is split in shared memory into hi = x with its low
// 13 mantissa bits cleared (exactly tf32) and lo = x - hi (exact in fp32), and the product is
// hi*hi + hi*lo + lo*hi: about 2^-21 relative error per product instead of tf32's 2^-11.
// Accumulation chains in TMEM are kept short (kSegStages stages per accumulator) and the
// segments are summed in fp32 registers with round-to-nearest, because long tensor-core
// accumulation chains were measured to drift (about 5e-8 relative per chained MMA).
//
// Roles: warp 0 TMA producer; warp 1 TMEM allocation + MMA issue (one thread); warps 2-5
// epilogue (one TMEM lane quadrant each, 128 columns, running sums in registers); with SPLIT3
// warps 6-9 split the freshly loaded tiles.  One 128 x 128 output tile per CTA.  All waits are
// bounded (see ptx.cuh); a timed-out CTA records HQ_ERR_TIMEOUT, drains and returns.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace hq {

struct Tf32GemmArgs {
  float* C;
  int64_t ldc;
  int M, N, Kred;
  float alpha, beta;
  int lower;          // write only elements with row0 + m >= col0 + n
  int row0, col0;
  int tiles_n;
  const int* skip;    // optional device flag: non-zero -> no work
  int* status;        // optional device status word
};

template <bool SPLIT3>
struct Tf32Cfg {
  static constexpr int BM = 128, BN = 128, BK = 32;
  static constexpr int kTileBytes = 16384;                       // 128 rows x 128 bytes
  static constexpr int kStageBytes = SPLIT3 ? 4 * kTileBytes : 2 * kTileBytes;  // A, B (+ A_lo, B_lo)
  static constexpr int kStages = SPLIT3 ? 3 : 6;
  static constexpr int kSegStages = SPLIT3 ? 4 : 8;              // 48 / 32 chained MMAs per segment
  static constexpr int kThreads = SPLIT3 ? 320 : 192;
  static constexpr int kSmemBytes = kStages * kStageBytes + 1024 + 256;
};

__device__ __forceinline__ float tf32_hi(float x) { return __uint_as_float(__float_as_uint(x) & 0xFFFFE000u); }

template <bool SPLIT3>
__global__ void __launch_bounds__(Tf32Cfg<SPLIT3>::kThreads, 1)
    tf32_gemm_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                     Tf32GemmArgs args) {
  using Cfg = Tf32Cfg<SPLIT3>;
  constexpr int S = Cfg::kStages;
  constexpr int TB = Cfg::kTileBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * Cfg::kStageBytes);
  uint64_t* conv = full + S;
  uint64_t* empty = conv + S;
  uint64_t* accf = empty + S;
  uint64_t* acce = accf + 2;
  uint64_t* drain = acce + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (args.skip != nullptr && *args.skip != 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tm = blockIdx.x / args.tiles_n, tn = blockIdx.x % args.tiles_n;
  const int m0 = tm * Cfg::BM, n0 = tn * Cfg::BN;
  // a tile entirely above the diagonal writes nothing
  if (args.lower && args.row0 + m0 + Cfg::BM - 1 < args.col0 + n0) return;
  const int kiters = (args.Kred + Cfg::BK - 1) / Cfg::BK;
  const int nseg = (kiters + Cfg::kSegStages - 1) / Cfg::kSegStages;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&conv[s], 128);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(&accf[a], 1);
      ptx::mbar_init(&acce[a], 4);
    }
    ptx::mbar_init(drain, 1);
    *abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, 256);
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
      const int s = k % S;
      if (k >= S && !ptx::mbar_wait(&empty[s], ((k / S) - 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      uint8_t* sa = smem + s * Cfg::kStageBytes;
      uint8_t* sb = sa + TB;
      ptx::mbar_arrive_expect_tx(&full[s], 2 * TB);
      ptx::tma_load_2d(sa, &mapA, k * Cfg::BK, m0, &full[s]);
      ptx::tma_load_2d(sb, &mapB, k * Cfg::BK, n0, &full[s]);
      ++issued;
    }
    if (!ok) {
      fail();
      const int first = issued > S ? issued - S : 0;
      for (int k = first; k < issued; ++k) ptx::mbar_wait(&full[k % S], (k / S) & 1, nullptr);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t kIdesc = ptx::idesc(ptx::kFmtTF32, Cfg::BM, Cfg::BN, false, false);
    bool ok = true;
    int k = 0;
    for (int seg = 0; seg < nseg && ok; ++seg) {
      const int acc = seg & 1;
      if (seg >= 2 && !ptx::mbar_wait(&acce[acc], ((seg >> 1) - 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const uint32_t dacc = tmem + static_cast<uint32_t>(acc * Cfg::BN);
      const int kbeg = seg * Cfg::kSegStages;
      const int kend = (kiters < kbeg + Cfg::kSegStages) ? kiters : kbeg + Cfg::kSegStages;
      for (; k < kend; ++k) {
        const int s = k % S;
        if (!ptx::mbar_wait(SPLIT3 ? &conv[s] : &full[s], (k / S) & 1, abort_flag)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t sa = ptx::smem_u32(smem + s * Cfg::kStageBytes);
        const uint32_t sb = sa + TB;
        const uint32_t sal = sa + 2 * TB, sbl = sa + 3 * TB;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
          const uint64_t ad = ptx::sdesc_sw128(sa + kk * 32, 16, 1024);
          const uint64_t bd = ptx::sdesc_sw128(sb + kk * 32, 16, 1024);
          const uint32_t first = (k > kbeg || kk > 0) ? 1u : 0u;
          ptx::mma_tf32(dacc, ad, bd, kIdesc, first);
          if (SPLIT3) {
            const uint64_t adl = ptx::sdesc_sw128(sal + kk * 32, 16, 1024);
            const uint64_t bdl = ptx::sdesc_sw128(sbl + kk * 32, 16, 1024);
            ptx::mma_tf32(dacc, ad, bdl, kIdesc, 1u);
            ptx::mma_tf32(dacc, adl, bd, kIdesc, 1u);
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
  } else if (SPLIT3 && warp >= 6) {
    // ------------------------------------------------------------ hi / lo split
    const int t = threadIdx.x - 192;  // 0..127
    for (int k = 0; k < kiters; ++k) {
      const int s = k % S;
      if (!ptx::mbar_wait(&full[s], (k / S) & 1, abort_flag)) {
        fail();
        break;
      }
      float4* hi = reinterpret_cast<float4*>(smem + s * Cfg::kStageBytes);          // A then B
      float4* lo = reinterpret_cast<float4*>(smem + s * Cfg::kStageBytes + 2 * TB);  // A_lo then B_lo
#pragma unroll 4
      for (int i = t; i < 2 * TB / 16; i += 128) {
        float4 x = hi[i];
        float4 h = make_float4(tf32_hi(x.x), tf32_hi(x.y), tf32_hi(x.z), tf32_hi(x.w));
        hi[i] = h;
        lo[i] = make_float4(x.x - h.x, x.y - h.y, x.z - h.z, x.w - h.w);
      }
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      ptx::mbar_arrive(&conv[s]);
    }
  } else if (warp >= 2 && warp < 6) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
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
      ptx::tmem_add128(tmem + lane_off + static_cast<uint32_t>(acc * Cfg::BN), sum);
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&acce[acc]);
    }
    if (!ok) fail();
    // stage the tile through shared memory (stage 0 is idle once the last MMA completed):
    // row r of the tile at r * 512 bytes, 16-byte chunk c stored at c ^ (r & 7)
    float4* tile = reinterpret_cast<float4*>(smem);
    const int rloc = q * 32 + lane;
    if (ok) {
#pragma unroll
      for (int c = 0; c < 32; ++c)
        tile[rloc * 32 + (c ^ (rloc & 7))] = make_float4(sum[4 * c], sum[4 * c + 1], sum[4 * c + 2], sum[4 * c + 3]);
    }
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (ok) {
      // warp q writes rows q, q+4, ...: lane = 16-byte chunk of a coalesced 512-byte row.
      // Eight rows per batch so that the loads of C are all in flight before any store.
      const bool full_tile = (m0 + Cfg::BM <= args.M) && (n0 + Cfg::BN <= args.N) && !args.lower &&
                             ((reinterpret_cast<uintptr_t>(args.C) & 15) == 0) && (args.ldc % 4 == 0);
      const int n = n0 + 4 * lane;
      for (int rb = 0; rb < Cfg::BM / 4; rb += 8) {
        float4 old[8];
        if (args.beta != 0.f) {
#pragma unroll
          for (int u = 0; u < 8; ++u) {
            const int m = m0 + q + 4 * (rb + u);
            old[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            if (full_tile) {
              old[u] = *reinterpret_cast<const float4*>(args.C + static_cast<int64_t>(m) * args.ldc + n);
            } else if (m < args.M) {
              const float* cr = args.C + static_cast<int64_t>(m) * args.ldc;
              if (n + 0 < args.N) old[u].x = cr[n + 0];
              if (n + 1 < args.N) old[u].y = cr[n + 1];
              if (n + 2 < args.N) old[u].z = cr[n + 2];
              if (n + 3 < args.N) old[u].w = cr[n + 3];
            }
          }
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int rr = q + 4 * (rb + u);
          const int m = m0 + rr;
          const float4 v = tile[rr * 32 + (lane ^ (rr & 7))];
          float4 o;
          if (args.beta != 0.f) {
            o.x = fmaf(args.alpha, v.x, args.beta * old[u].x);
            o.y = fmaf(args.alpha, v.y, args.beta * old[u].y);
            o.z = fmaf(args.alpha, v.z, args.beta * old[u].z);
            o.w = fmaf(args.alpha, v.w, args.beta * old[u].w);
          } else {
            o = make_float4(args.alpha * v.x, args.alpha * v.y, args.alpha * v.z, args.alpha * v.w);
          }
          if (full_tile) {
            *reinterpret_cast<float4*>(args.C + static_cast<int64_t>(m) * args.ldc + n) = o;
          } else if (m < args.M) {
            float* cr = args.C + static_cast<int64_t>(m) * args.ldc;
            const float ov[4] = {o.x, o.y, o.z, o.w};
#pragma unroll
            for (int i = 0; i < 4; ++i)
              if (n + i < args.N && !(args.lower && args.row0 + m < args.col0 + n + i)) cr[n + i] = ov[i];
          }
        }
      }
    }
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 256);
  }
}

}  // namespace hq
