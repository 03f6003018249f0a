// The GPTQ lazy trailing update on the tcgen05 tensor cores, fp32-accurate (3xTF32):
//
//   C[m, n] -= sum_k A(m, k) B(n, k)      m < M, n < N
//   A(m, k) = A_hi[m * lda + k] + A_lo[m * lda + k]      (the sweep's residuals D, split)
//   B(n, k) = B_hi[n * ldb + k] + B_lo[n * ldb + k]      (U'^T, split)
//
// Both operands arrive split into a tf32 part (low 13 mantissa bits zero) and the fp32
// remainder, so the kernel only streams them: the product is hi*hi + hi*lo + lo*hi, three
// kind::tf32 MMAs per k-step into the same TMEM accumulator (about 2^-21 relative per product).
// Persistent: one CTA per SM walks 128 x BN output tiles (BN = 256, or 128 / 64 when the
// wide tiles would leave SMs without two tiles each, as in the small inner updates of a panel);
// warp 0 issues TMA loads (a 4-stage ring of stages A_hi, A_lo [128 x 16], B_hi, B_lo
// [BN x 16], 64-byte swizzle), warp 1 issues the MMAs into one of two 128 x BN fp32
// accumulators (2 BN TMEM columns), and warps 2-5 drain the other accumulator into C while the
// next tile is being multiplied: C moves in 128 x 32 chunks by TMA (load into a double-buffered
// shared-memory chunk, subtract there, TMA store back), the next chunk's load in flight while
// one chunk is being worked on.
// Every wait is bounded; a CTA that times out records HQ_ERR_TIMEOUT and stops.
#include "common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"
#include "tmap.cuh"

namespace hq {
namespace {

constexpr int kBM = 128, kBK = 16;                // 16 fp32 = one 64-byte swizzled row per k-slice
constexpr int kStages = 4;
constexpr int kATile = kBM * kBK * 4;              // 8 KB
constexpr int kChunk = 32;                         // epilogue: C columns per TMA round trip
constexpr int kCBuf = kBM * kChunk * 4;            // 16 KB, 128-byte swizzled rows
constexpr int kEpiBytes = 2 * kCBuf;               // double-buffered C chunks
constexpr int kThreads = 192;
constexpr int kSMs = 148;

// Tile width BN (256, 128 or 64 output columns): the narrow tiles spread the small inner
// updates of a panel over more SMs.
template <int BN>
struct UpdTile {
  static constexpr int kBTile = BN * kBK * 4;             // 16 / 8 / 4 KB
  static constexpr int kStage = 2 * kATile + 2 * kBTile;  // 48 / 32 / 24 KB
  static constexpr int kSmem = kStages * kStage + kEpiBytes + 1024 + 256;
  static constexpr int kTmemCols = 2 * BN;                // two accumulators
};

struct UpdArgs {
  float* C;
  int64_t ldc;
  int M, N, Kred;
  int tiles_m, tiles_n;
  const int* skip;
  int* status;
};

template <int BN>
__global__ void __launch_bounds__(kThreads, 1)
    upd_gemm_kernel(const __grid_constant__ CUtensorMap mAh, const __grid_constant__ CUtensorMap mAl,
                    const __grid_constant__ CUtensorMap mBh, const __grid_constant__ CUtensorMap mBl,
                    const __grid_constant__ CUtensorMap mC, UpdArgs args) {
  constexpr int kBN = BN;
  constexpr int kBTile = UpdTile<BN>::kBTile;
  constexpr int kStage = UpdTile<BN>::kStage;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* cbuf = smem + kStages * kStage;  // two C chunks
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStage + kEpiBytes);
  uint64_t* empty = full + kStages;
  uint64_t* accf = empty + kStages;
  uint64_t* acce = accf + 2;
  uint64_t* cfull = acce + 2;
  uint64_t* drain = cfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (args.skip != nullptr && *args.skip != 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntiles = args.tiles_m * args.tiles_n;
  const int kiters = (args.Kred + kBK - 1) / kBK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      ptx::mbar_init(&accf[a], 1);
      ptx::mbar_init(&acce[a], 4);
      ptx::mbar_init(&cfull[a], 1);
    }
    ptx::mbar_init(drain, 1);
    *abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, UpdTile<BN>::kTmemCols);
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
    ptx::prefetch_tensormap(&mAh);
    ptx::prefetch_tensormap(&mAl);
    ptx::prefetch_tensormap(&mBh);
    ptx::prefetch_tensormap(&mBl);
    int g = 0;  // stages issued
    bool ok = true;
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
      const int m0 = (t / args.tiles_n) * kBM, n0 = (t % args.tiles_n) * kBN;
      for (int k = 0; k < kiters; ++k, ++g) {
        const int s = g % kStages;
        if (g >= kStages && !ptx::mbar_wait(&empty[s], ((g / kStages) - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        uint8_t* st = smem + s * kStage;
        ptx::mbar_arrive_expect_tx(&full[s], kStage);
        ptx::tma_load_2d(st, &mAh, k * kBK, m0, &full[s]);
        ptx::tma_load_2d(st + kATile, &mAl, k * kBK, m0, &full[s]);
        ptx::tma_load_2d(st + 2 * kATile, &mBh, k * kBK, n0, &full[s]);
        ptx::tma_load_2d(st + 2 * kATile + kBTile, &mBl, k * kBK, n0, &full[s]);
      }
    }
    if (!ok) {
      fail();
      // wait (bounded only by the copies themselves) for the loads already in flight
      const int first = g > kStages ? g - kStages : 0;
      for (int k = first; k < g; ++k) ptx::mbar_wait(&full[k % kStages], (k / kStages) & 1, nullptr);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t kIdesc = ptx::idesc(ptx::kFmtTF32, kBM, kBN, false, false);
    int g = 0, i = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++i) {
      const int acc = i & 1;
      if (i >= 2 && !ptx::mbar_wait(&acce[acc], ((i >> 1) - 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      const uint32_t dacc = tmem + static_cast<uint32_t>(acc * kBN);
      for (int k = 0; k < kiters; ++k, ++g) {
        const int s = g % kStages;
        if (!ptx::mbar_wait(&full[s], (g / kStages) & 1, abort_flag)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t ah = ptx::smem_u32(smem + s * kStage);
        const uint32_t al = ah + kATile, bh = ah + 2 * kATile, bl = bh + kBTile;
#pragma unroll
        for (int kk = 0; kk < kBK / 8; ++kk) {
          const uint64_t dah = ptx::sdesc_sw64(ah + kk * 32, 16, 512);
          const uint64_t dal = ptx::sdesc_sw64(al + kk * 32, 16, 512);
          const uint64_t dbh = ptx::sdesc_sw64(bh + kk * 32, 16, 512);
          const uint64_t dbl = ptx::sdesc_sw64(bl + kk * 32, 16, 512);
          ptx::mma_tf32(dacc, dah, dbh, kIdesc, (k > 0 || kk > 0) ? 1u : 0u);
          ptx::mma_tf32(dacc, dah, dbl, kIdesc, 1u);
          ptx::mma_tf32(dacc, dal, dbh, kIdesc, 1u);
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
    // ------------------------------------------------------------ epilogue: C -= accumulator
    // thread = tile row (TMEM lane); chunk e of this CTA = tile e / 8, columns 32 (e % 8) ..
    const int q = warp & 3;  // TMEM lane quadrant = tile rows 32 q .. 32 q + 31
    const int row = q * 32 + lane;
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    const bool leader = (warp == 2 && lane == 0);
    constexpr int kCPT = kBN / kChunk;  // chunks per tile
    int my_tiles = 0;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x) ++my_tiles;
    const int nchunks = my_tiles * kCPT;
    auto chunk_xy = [&](int e, int& x, int& y) {
      const int t = blockIdx.x + (e / kCPT) * gridDim.x;
      y = (t / args.tiles_n) * kBM;
      x = (t % args.tiles_n) * kBN + (e % kCPT) * kChunk;
    };
    auto load_chunk = [&](int e) {  // leader only
      int x, y;
      chunk_xy(e, x, y);
      ptx::mbar_arrive_expect_tx(&cfull[e & 1], kCBuf);
      ptx::tma_load_2d(cbuf + (e & 1) * kCBuf, &mC, x, y, &cfull[e & 1]);
    };
    if (leader) {
      if (nchunks > 0) load_chunk(0);
      if (nchunks > 1) load_chunk(1);
    }
    // every warp runs all iterations and meets the named barrier each time, also after a
    // failed wait (it then skips the work), so the barrier cannot be left waiting
    bool ok = true;
    for (int e = 0; e < nchunks; ++e) {
      const int i = e / kCPT, c = e % kCPT, acc = i & 1;
      if (ok && c == 0) {
        ok = ptx::mbar_wait(&accf[acc], (i >> 1) & 1, abort_flag);
        ptx::tc_fence_after();
      }
      uint32_t v[32];
      if (ok) {
        ptx::tmem_ld32_nowait(tmem + lane_off + static_cast<uint32_t>(acc * kBN + c * kChunk), v);
        ptx::tmem_wait_ld();
        if (c == kCPT - 1) {  // the accumulator is free for the tile after next
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&acce[acc]);
        }
        ok = ptx::mbar_wait(&cfull[e & 1], (e >> 1) & 1, abort_flag);
      }
      if (ok) {
        // row `row` of the chunk: 16-byte piece j at j ^ (row & 7) (128-byte swizzle)
        float4* crow = reinterpret_cast<float4*>(cbuf + (e & 1) * kCBuf + row * 128);
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          float4 o = crow[j ^ (row & 7)];
          o.x -= __uint_as_float(v[4 * j]);
          o.y -= __uint_as_float(v[4 * j + 1]);
          o.z -= __uint_as_float(v[4 * j + 2]);
          o.w -= __uint_as_float(v[4 * j + 3]);
          crow[j ^ (row & 7)] = o;
        }
      }
      ptx::fence_async_smem();
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (leader && ok && *abort_flag == 0) {
        int x, y;
        chunk_xy(e, x, y);
        ptx::tma_store_2d(&mC, cbuf + (e & 1) * kCBuf, x, y);
        ptx::bulk_commit();
        if (e + 2 < nchunks) {
          ptx::bulk_wait_read<0>();  // this buffer's store has read it: reuse it for chunk e + 2
          load_chunk(e + 2);
        }
      }
    }
    if (!ok) fail();
    if (leader) ptx::bulk_wait<0>();  // all stores complete before the CTA exits
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, UpdTile<BN>::kTmemCols);
  }
}

}  // namespace

template <int BN>
static hq_status upd_gemm_bn(const UpdGemm& g, cudaStream_t s) {
  const uint64_t kred = static_cast<uint64_t>(g.Kred);
  CUtensorMap mAh, mAl, mBh, mBl, mC;
  if (!make_tmap_2d(&mAh, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, g.A_hi, kred, static_cast<uint64_t>(g.M),
                    static_cast<uint64_t>(g.lda) * 4, kBK, kBM, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_tmap_2d(&mAl, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, g.A_lo, kred, static_cast<uint64_t>(g.M),
                    static_cast<uint64_t>(g.lda) * 4, kBK, kBM, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_tmap_2d(&mBh, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, g.B_hi, kred, static_cast<uint64_t>(g.N),
                    static_cast<uint64_t>(g.ldb) * 4, kBK, BN, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_tmap_2d(&mBl, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, g.B_lo, kred, static_cast<uint64_t>(g.N),
                    static_cast<uint64_t>(g.ldb) * 4, kBK, BN, CU_TENSOR_MAP_SWIZZLE_64B) ||
      !make_tmap_2d(&mC, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, g.C, static_cast<uint64_t>(g.N), static_cast<uint64_t>(g.M),
                    static_cast<uint64_t>(g.ldc) * 4, kChunk, kBM))
    return HQ_ERR_CUDA;
  UpdArgs a{};
  a.C = g.C;
  a.ldc = g.ldc;
  a.M = g.M;
  a.N = g.N;
  a.Kred = g.Kred;
  a.tiles_m = static_cast<int>(ceil_div(g.M, kBM));
  a.tiles_n = static_cast<int>(ceil_div(g.N, BN));
  a.skip = g.skip;
  a.status = g.status;
  const int64_t ntiles = static_cast<int64_t>(a.tiles_m) * a.tiles_n;
  if (ntiles > 0x7FFFFFFF) return HQ_ERR_UNSUPPORTED;
  const int grid = static_cast<int>(ntiles < kSMs ? ntiles : kSMs);
  constexpr int smem = UpdTile<BN>::kSmem;
  HQ_CUDA_TRY(cudaFuncSetAttribute(upd_gemm_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  const int tm = timer_start(kTimeTf32Gemm, s);
  upd_gemm_kernel<BN><<<grid, kThreads, smem, s>>>(mAh, mAl, mBh, mBl, mC, a);
  HQ_LAUNCH_CHECK();
  timer_stop(tm, 2.0 * g.M * g.N * static_cast<double>(g.Kred), s);  // the product's flops
  return HQ_OK;
}

// The widest tile that still gives every SM two tiles, else the narrowest.
hq_status upd_gemm(const UpdGemm& g, cudaStream_t s) {
  if (g.M <= 0 || g.N <= 0 || g.Kred <= 0) return HQ_OK;
  const void* ptrs[5] = {g.A_hi, g.A_lo, g.B_hi, g.B_lo, g.C};
  for (const void* p : ptrs)
    if (!aligned(p, 16)) return HQ_ERR_UNSUPPORTED;
  if (g.lda % 4 != 0 || g.ldb % 4 != 0 || g.ldc % 4 != 0) return HQ_ERR_UNSUPPORTED;
  const int64_t tm = ceil_div(static_cast<int64_t>(g.M), int64_t(kBM));
  if (tm * ceil_div(static_cast<int64_t>(g.N), int64_t(256)) >= 2 * kSMs) return upd_gemm_bn<256>(g, s);
  if (tm * ceil_div(static_cast<int64_t>(g.N), int64_t(128)) >= 2 * kSMs) return upd_gemm_bn<128>(g, s);
  return upd_gemm_bn<64>(g, s);
}

}  // namespace hq
