// Calibration Hessian accumulation H += X^T X over the lower triangle of H.
//
// bf16 X with K a multiple of 8 and a 16-byte aligned base goes through the persistent tcgen05
// kernel below; every other input (fp32 X, odd K, unaligned X) takes the fp32 CUDA-core kernel,
// which computes the same sum with exact products and fp32 accumulation.
//
// Tensor-core path: one CTA per SM walks 128 x 256 lower-triangle tiles of H (static round
// robin; all tiles cost the same).  When the last round would hold at most half the SMs' worth
// of tiles (600 tiles on 148 SMs at K = 6144: 4 rounds and 8 tiles), those tiles are cut by
// 1024-token segments into pieces spread over the idle SMs (the tensor core takes about the same
// time per instruction at any N up to 256, so narrower tiles would not fill the gap).  Warp 0 issues TMA loads of 64-token x 64-channel bf16 boxes
// into a 4-stage ring of 48 KB stages (A: channels m0..m0+127, B: n0..n0+255, both MN-major);
// warp 1 allocates all 512 TMEM columns and issues kind::f16 MMAs from one thread; warps 2-9
// drain the accumulators.  The tensor core's fp32 accumulation loses precision in proportion to
// the number of MMAs chained into one accumulator (measured: 1.2e-5 relative Frobenius error
// after 256 chained K=16 steps; 4096-token segments failed the 1e-5 budget), so at most
// kSyrkSegK tokens (64 MMAs) are chained per accumulator: two 256-column accumulators alternate
// segment by segment, across tile boundaries too, and the epilogue warps (two per TMEM lane
// quadrant, 128 columns each) add every finished segment into fp32 registers while the tensor
// core fills the other accumulator.  After a tile's last segment each thread adds its row's 128
// sums to H (lower part only) with 16-byte reductions performed in L2 (red.global.add.v4.f32):
// nothing is read back, so the epilogue warps return at once to the next tile's segments (a
// read-modify-write from the SM measured 2-12 % slower).  An element of a whole tile receives
// one addition per call, so its result does not depend on timing; the pieces of a cut tile add
// their partial sums in whatever order they finish, so those elements may differ in the last
// bit from run to run.
//
// Every wait is bounded: on expiry the CTA records HQ_ERR_TIMEOUT, waits (bounded) for its
// in-flight TMA and MMA work, frees TMEM and returns.
#include <cuda_bf16.h>

#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"
#include "tmap.cuh"

namespace hq {

// ---------------------------------------------------------------- CUDA-core path

constexpr int kSimtTile = 64;
constexpr int kSimtBK = 16;

template <typename TX>
__device__ __forceinline__ float load_x(const TX* p);
template <>
__device__ __forceinline__ float load_x<float>(const float* p) { return *p; }
template <>
__device__ __forceinline__ float load_x<__nv_bfloat16>(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// One 64 x 64 tile (bi >= bj) per CTA, 256 threads with 4 x 4 outputs each.
template <typename TX>
__global__ void __launch_bounds__(256) syrk_simt_kernel(float* __restrict__ H, const TX* __restrict__ X, int64_t T,
                                                        int64_t K) {
  int t = blockIdx.x;
  int bi = 0;
  while (t > bi) {
    t -= bi + 1;
    ++bi;
  }
  const int bj = t;
  const int64_t i0 = static_cast<int64_t>(bi) * kSimtTile;
  const int64_t j0 = static_cast<int64_t>(bj) * kSimtTile;
  __shared__ float xs_i[kSimtBK][kSimtTile];
  __shared__ float xs_j[kSimtBK][kSimtTile];
  const int tx = threadIdx.x % 16;
  const int ty = threadIdx.x / 16;
  float acc[4][4] = {};
  for (int64_t t0 = 0; t0 < T; t0 += kSimtBK) {
    for (int e = threadIdx.x; e < kSimtBK * kSimtTile; e += 256) {
      const int r = e / kSimtTile, c = e % kSimtTile;
      const int64_t tt = t0 + r;
      xs_i[r][c] = (tt < T && i0 + c < K) ? load_x(X + tt * K + i0 + c) : 0.f;
      xs_j[r][c] = (tt < T && j0 + c < K) ? load_x(X + tt * K + j0 + c) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kSimtBK; ++r) {
      float a[4], b[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        a[u] = xs_i[r][ty + 16 * u];
        b[u] = xs_j[r][tx + 16 * u];
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
    const int64_t i = i0 + ty + 16 * u;
    if (i >= K) continue;
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int64_t j = j0 + tx + 16 * v;
      if (j <= i && HQ_IN_BOUNDS(j < K)) H[i * K + j] += acc[u][v];
    }
  }
}

hq_status launch_syrk_simt(float* H, const void* X, int x_dtype, int64_t T, int64_t K, cudaStream_t s) {
  const int64_t nb = ceil_div(K, kSimtTile);
  const int64_t tiles = nb * (nb + 1) / 2;
  if (tiles > 0x7FFFFFFF) return HQ_ERR_UNSUPPORTED;
  if (x_dtype == HQ_F32)
    syrk_simt_kernel<float><<<static_cast<unsigned>(tiles), 256, 0, s>>>(H, static_cast<const float*>(X), T, K);
  else
    syrk_simt_kernel<__nv_bfloat16>
        <<<static_cast<unsigned>(tiles), 256, 0, s>>>(H, static_cast<const __nv_bfloat16*>(X), T, K);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

// ---------------------------------------------------------------- tensor-core path

constexpr int kSyBM = 128;
constexpr int kSyBN = 256;
constexpr int kSyBK = 64;               // tokens per stage
constexpr int kSyStages = 4;
constexpr int kSyStageBytes = 49152;    // A 16 KB + B 32 KB
constexpr int kSySmem = kSyStages * kSyStageBytes + 1024 /*align*/ + 256 /*barriers*/;
constexpr int kSyrkSegK = 1024;         // tokens chained in one TMEM accumulator
constexpr int kSySegIters = kSyrkSegK / kSyBK;
constexpr int kSyEpiWarps = 8;
constexpr int kSyThreads = 64 + 32 * kSyEpiWarps;
constexpr int kSySMs = 148;

// Lower-triangle tile enumeration of a K x K output with 128 x 256 tiles: tile row bi holds
// column tiles bj with bj * 256 <= bi * 128 + 127.
__host__ __device__ inline int syrk_tiles_in_row(int bi, int tiles_n) {
  int c = (bi * kSyBM + kSyBM - 1) / kSyBN + 1;
  return c < tiles_n ? c : tiles_n;
}

// Tile order: bands of kSyBand tile rows; inside a band column-tile by column-tile, and inside a
// column down the band's rows that hold it.  The 148 tiles in flight at a time then cover a
// compact block of H, so the X columns they read are few and shared through L2.
constexpr int kSyBand = 16;

__device__ inline void syrk_tile_coords(int t, int tiles_m, int tiles_n, int& m0, int& n0) {
  for (int r0 = 0; r0 < tiles_m; r0 += kSyBand) {
    const int r1 = r0 + kSyBand < tiles_m ? r0 + kSyBand : tiles_m;
    int band = 0;
    for (int bi = r0; bi < r1; ++bi) band += syrk_tiles_in_row(bi, tiles_n);
    if (t >= band) {
      t -= band;
      continue;
    }
    for (int bj = 0;; ++bj) {
      // rows of the band holding column tile bj: bi with syrk_tiles_in_row(bi) > bj
      int first = r1;
      for (int bi = r0; bi < r1; ++bi)
        if (syrk_tiles_in_row(bi, tiles_n) > bj) {
          first = bi;
          break;
        }
      const int n = r1 - first;
      if (t < n) {
        m0 = (first + t) * kSyBM;
        n0 = bj * kSyBN;
        return;
      }
      t -= n;
    }
  }
  m0 = n0 = 0;  // not reached for t < tiles
}

struct SyrkArgs {
  float* H;
  int K;         // H is K x K, row-major
  int T;         // tokens
  int tiles;     // lower-triangle tiles
  int full_rounds;  // tiles every CTA takes whole (round robin)
  int left;         // tiles left after the full rounds
  int pieces;       // pieces each left tile is cut into (by 1024-token segments)
  int* status;
  long long wait_limit;  // cycles a pipeline wait may take before the CTA gives up
  int withhold_stage;    // -1, or a ring stage whose first release the MMA issuer skips (the
                         // test of the timeout path: the producer's wait for it then expires)
};

// The work of CTA b: tiles b + i grid for i < full_rounds (all segments), then, if b < left
// pieces, piece b % pieces of left tile full_rounds grid + b / pieces (a contiguous range of its
// segments).  A launch whose last round would leave most SMs idle so spreads that round's few
// tiles over them; the pieces of a tile add their partial sums into H on their own.
__device__ inline int syrk_items(const SyrkArgs& a) {
  return a.full_rounds + (static_cast<int>(blockIdx.x) < a.left * a.pieces ? 1 : 0);
}
__device__ inline void syrk_item(const SyrkArgs& a, int i, int nseg, int& t, int& s0, int& s1) {
  const int b = blockIdx.x;
  if (i < a.full_rounds) {
    t = b + i * static_cast<int>(gridDim.x);
    s0 = 0;
    s1 = nseg;
    return;
  }
  const int p = b % a.pieces;
  t = a.full_rounds * static_cast<int>(gridDim.x) + b / a.pieces;
  s0 = p * nseg / a.pieces;
  s1 = (p + 1) * nseg / a.pieces;
}

__global__ void __launch_bounds__(kSyThreads, 1)
    syrk_tc_kernel(const __grid_constant__ CUtensorMap mapX, SyrkArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kSyStages * kSyStageBytes);
  uint64_t* empty = full + kSyStages;
  uint64_t* accf = empty + kSyStages;  // [2] accumulator filled
  uint64_t* acce = accf + 2;           // [2] accumulator drained
  uint64_t* drain = acce + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tiles_m = (args.K + kSyBM - 1) / kSyBM;
  const int tiles_n = (args.K + kSyBN - 1) / kSyBN;
  const int kiters = (args.T + kSyBK - 1) / kSyBK;
  const int nseg = (kiters + kSySegIters - 1) / kSySegIters;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kSyStages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(&accf[a], 1);
      ptx::mbar_init(&acce[a], kSyEpiWarps);
    }
    ptx::mbar_init(drain, 1);
    *abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, 512);
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
    ptx::prefetch_tensormap(&mapX);
    int g = 0;  // stages issued by this CTA
    bool ok = true;
    const int nitems = syrk_items(args);
    for (int it = 0; it < nitems && ok; ++it) {
      int t, s0, s1, m0, n0;
      syrk_item(args, it, nseg, t, s0, s1);
      syrk_tile_coords(t, tiles_m, tiles_n, m0, n0);
      const int k1 = (kiters < s1 * kSySegIters) ? kiters : s1 * kSySegIters;
      for (int k = s0 * kSySegIters; k < k1; ++k, ++g) {
        const int s = g % kSyStages;
        if (g >= kSyStages && !ptx::mbar_wait(&empty[s], ((g / kSyStages) - 1) & 1, abort_flag, args.wait_limit)) {
          ok = false;
          break;
        }
        uint8_t* sa = smem + s * kSyStageBytes;
        uint8_t* sb = sa + 16384;
        const int t0 = k * kSyBK;
        // record only: a tile's loads are never skipped (the stage's byte count is already
        // announced), and the copy engine fills coordinates past the tensor with zeros
        (void)HQ_IN_BOUNDS(m0 < args.K && n0 < args.K && t0 < args.T);
        ptx::mbar_arrive_expect_tx(&full[s], kSyStageBytes);
        ptx::tma_load_2d(sa, &mapX, m0, t0, &full[s]);
        ptx::tma_load_2d(sa + 8192, &mapX, m0 + 64, t0, &full[s]);
#pragma unroll
        for (int c = 0; c < 4; ++c) ptx::tma_load_2d(sb + c * 8192, &mapX, n0 + 64 * c, t0, &full[s]);
      }
    }
    if (!ok) {
      fail();
      // let the copies already issued land before the CTA's shared memory goes away
      const int first = g > kSyStages ? g - kSyStages : 0;
      for (int k = first; k < g; ++k) ptx::mbar_wait(&full[k % kSyStages], (k / kSyStages) & 1, nullptr);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t kIdesc = ptx::idesc(ptx::kFmtBF16, kSyBM, kSyBN, true, true);
    bool ok = true;
    int g = 0;   // stages consumed
    int sg = 0;  // segments issued (accumulator = sg & 1)
    const int nitems = syrk_items(args);
    for (int it = 0; it < nitems && ok; ++it) {
      int t, s0, s1;
      syrk_item(args, it, nseg, t, s0, s1);
      int k = s0 * kSySegIters;
      for (int seg = s0; seg < s1 && ok; ++seg, ++sg) {
        const int acc = sg & 1;
        if (sg >= 2 && !ptx::mbar_wait(&acce[acc], ((sg >> 1) - 1) & 1, abort_flag, args.wait_limit)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t dacc = tmem + static_cast<uint32_t>(acc * kSyBN);
        const int kbeg = seg * kSySegIters;
        const int kend = (kiters < kbeg + kSySegIters) ? kiters : kbeg + kSySegIters;
        for (; k < kend; ++k, ++g) {
          const int s = g % kSyStages;
          if (!ptx::mbar_wait(&full[s], (g / kSyStages) & 1, abort_flag, args.wait_limit)) {
            ok = false;
            break;
          }
          ptx::tc_fence_after();
          const uint32_t sa = ptx::smem_u32(smem + s * kSyStageBytes);
          const uint32_t sb = sa + 16384;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            // MN-major: 64-element chunks 8 KB apart (LBO), 8-row groups 1 KB apart (SBO);
            // each MMA consumes 16 tokens = 2 KB.
            const uint64_t ad = ptx::sdesc_sw128(sa + kk * 2048, 8192, 1024);
            const uint64_t bd = ptx::sdesc_sw128(sb + kk * 2048, 8192, 1024);
            ptx::mma_bf16(dacc, ad, bd, kIdesc, (k > kbeg || kk > 0) ? 1u : 0u);
          }
          if (!(g == args.withhold_stage && g < kSyStages)) ptx::mma_commit(&empty[s]);
        }
        if (ok) ptx::mma_commit(&accf[acc]);
      }
    }
    if (!ok) {
      fail();
      ptx::mma_commit(drain);
      ptx::mbar_wait(drain, 0, nullptr);
    }
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;             // TMEM lane quadrant this warp may access
    const int h = (warp - 2) >> 2;      // which 128-column half of the tile
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const bool vec = (reinterpret_cast<uintptr_t>(args.H) & 15) == 0 && (args.K % 4) == 0;
    bool ok = true;
    int sg = 0;
    const int nitems = syrk_items(args);
    for (int it = 0; it < nitems && ok; ++it) {
      int t, s0, s1, m0, n0;
      syrk_item(args, it, nseg, t, s0, s1);
      syrk_tile_coords(t, tiles_m, tiles_n, m0, n0);
      float sum[128];
#pragma unroll
      for (int i = 0; i < 128; ++i) sum[i] = 0.f;
      for (int seg = s0; seg < s1; ++seg, ++sg) {
        const int acc = sg & 1;
        if (!ptx::mbar_wait(&accf[acc], (sg >> 1) & 1, abort_flag, args.wait_limit)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        ptx::tmem_add128(tmem + lane_off + static_cast<uint32_t>(acc * kSyBN + h * 128), sum);
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&acce[acc]);
      }
      if (!ok) break;
      // row `row`, columns c0 .. c0 + 127 of H += sum (lower part only)
      const int row = m0 + q * 32 + lane;
      // a tile may overhang H (its upper half can start past column K - 1); each write below
      // checks its own column
      if (row < args.K && HQ_IN_BOUNDS(n0 < args.K)) {
        float* hrow = args.H + static_cast<int64_t>(row) * args.K;
        const int c0 = n0 + h * 128;
#pragma unroll
        for (int k = 0; k < 32; ++k) {
          const int col = c0 + 4 * k;
          if (vec && col + 3 <= row && col + 3 < args.K) {
            asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(hrow + col), "f"(sum[4 * k]),
                         "f"(sum[4 * k + 1]), "f"(sum[4 * k + 2]), "f"(sum[4 * k + 3])
                         : "memory");
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e)
              if (col + e <= row && col + e < args.K) atomicAdd(hrow + col + e, sum[4 * k + e]);
          }
        }
      }
    }
    if (!ok) fail();
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

bool syrk_tc_eligible(const void* X, int x_dtype, int64_t T, int64_t K) {
  return x_dtype == HQ_BF16 && (K % 8) == 0 && aligned(X, 16) && K <= (1 << 24) && T <= 0x7FFFFFFF;
}

hq_status launch_syrk_tc(float* H, const void* X, int64_t T, int64_t K, int* dev_status, cudaStream_t s,
                         long long wait_limit, int withhold_stage) {
  CUtensorMap map;
  if (!make_tmap_2d(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, X, static_cast<uint64_t>(K), static_cast<uint64_t>(T),
                    static_cast<uint64_t>(K) * 2, 64, 64))
    return HQ_ERR_CUDA;
  HQ_CUDA_TRY(cudaFuncSetAttribute(syrk_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSySmem));
  const int tiles_m = static_cast<int>(ceil_div(K, kSyBM));
  const int tiles_n = static_cast<int>(ceil_div(K, kSyBN));
  int64_t tiles = 0;
  for (int bi = 0; bi < tiles_m; ++bi) tiles += syrk_tiles_in_row(bi, tiles_n);
  if (tiles > 0x7FFFFFFF) return HQ_ERR_UNSUPPORTED;
  SyrkArgs a{};
  a.H = H;
  a.K = static_cast<int>(K);
  a.T = static_cast<int>(T);
  a.tiles = static_cast<int>(tiles);
  // whole tiles round robin; a last round of at most half the SMs' worth of tiles is cut into
  // pieces of whole 1024-token segments and spread over the SMs it would leave idle
  const int nseg = static_cast<int>(ceil_div(ceil_div(T, kSyBK), kSySegIters));
  int grid = static_cast<int>(tiles < kSySMs ? tiles : kSySMs);
  a.full_rounds = static_cast<int>(tiles / grid);
  a.left = static_cast<int>(tiles - static_cast<int64_t>(a.full_rounds) * grid);
  a.pieces = 1;
  if (tiles < kSySMs) {  // one partial round only: cut every tile
    a.full_rounds = 0;
    a.left = static_cast<int>(tiles);
    a.pieces = std::max(1, std::min(kSySMs / a.left, nseg));
    grid = a.left * a.pieces;
  } else if (a.left > 0) {
    a.pieces = std::max(1, std::min(grid / a.left, nseg));
  }
  a.status = dev_status;
  a.wait_limit = wait_limit;
  a.withhold_stage = withhold_stage;
  const int tm = timer_start(kTimeSyrk, s);
  syrk_tc_kernel<<<grid, kSyThreads, kSySmem, s>>>(map, a);
  HQ_LAUNCH_CHECK();
  timer_stop(tm, static_cast<double>(T) * K * (K + 1), s);  // 2 flops x T x K (K + 1) / 2 lower entries
  return HQ_OK;
}

}  // namespace hq
