// fp64 GEMM for the factorisation, on the fp64 tensor cores (mma.sync m8n8k4 .f64):
//
//   C[m, n] = beta * C[m, n] + alpha * sum_k A[m * lda + k] * B[n * ldb + k]    m < M, n < N
//
// (both operands K-major; optionally only the lower part m >= n written; a triangular operand
// can be declared so that each tile skips the part of the contraction where it is zero).
// The damped Hessians of strongly correlated layers have condition numbers around 1e6, and the
// Schur-complement updates of the Cholesky recursion cancel a large common component, so the
// factorisation runs in fp64 end to end (fp32 loses about kappa * 6e-8 there, which measurably
// changes GPTQ codes).  The fp64 MMA rounds like an fp64 FMA chain; on B200 it sustains about
// 37 TFLOP/s against about 33 for CUDA-core DFMA, with a fraction of the issue slots.
//
// Design: BT x BT output tiles (BT = 128: 8 warps of 32 x 64; BT = 64: 4 warps of 32 x 32;
// BT = 32: 4 warps of 16 x 16).
// Operands stream through a 4-stage cp.async ring of [BT rows][16 k] slices; element (r, k) of a
// slice sits at r * 16 + (k ^ ((r & 3) << 2)), so that a fragment load (8 rows x 4 consecutive
// k) touches distinct banks in each half-warp, and 16-byte pairs stay contiguous for cp.async.
// Tiles are launched most expensive first (their contraction length depends on the triangular
// operand).  When a problem has too few tiles to fill the GPU, the contraction is split over
// CTAs that write partial tiles to scratch, and a second kernel adds the partials in a fixed
// order (so results do not depend on scheduling).  (Letting the last CTA of each tile add them
// instead was measured slower: one CTA then reads every partial of its tile.)  The written C
// can also be stored transposed (Ct).
#include <algorithm>

#include "common.cuh"
#include "kernels.cuh"

namespace hq {
namespace {

constexpr int kDK = 16;  // k per stage
constexpr int kStages = 4;
constexpr int kSMs = 148;

template <int BT>
struct F64Cfg {
  static constexpr int kWarpsM = BT == 128 ? 4 : 2;
  static constexpr int kWarpsN = 2;
  static constexpr int kThreads = 32 * kWarpsM * kWarpsN;
  static constexpr int kWM = BT / kWarpsM;  // warp tile rows (32)
  static constexpr int kWN = BT / kWarpsN;  // warp tile cols (64 or 32)
  static constexpr int kFM = kWM / 8;       // 8 x 8 MMA tiles per warp tile, rows
  static constexpr int kFN = kWN / 8;       // ... cols
  static constexpr int kStageElems = 2 * BT * kDK;
  static constexpr int kSmemBytes = kStages * kStageElems * static_cast<int>(sizeof(double));
  static constexpr int kPairs = BT * kDK / 2 / kThreads;  // 16-byte copies per operand per stage per thread
};

__device__ __forceinline__ void cp_async16(double* smem, const double* gmem, bool valid) {
  const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
  const int n = valid ? 16 : 0;  // 0: nothing read, the destination is zero-filled
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(s), "l"(gmem), "r"(n) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

// D (8 x 8) += A (8 x 4) B (4 x 8): lane (g = lane / 4, t = lane % 4) holds A[g][t], B[t][g] and
// D[g][2t], D[g][2t + 1].
__device__ __forceinline__ void dmma(double& d0, double& d1, double a, double b) {
  asm("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0,%1}, {%2}, {%3}, {%0,%1};\n"
               : "+d"(d0), "+d"(d1)
               : "d"(a), "d"(b));
}

__device__ __forceinline__ int swz(int r, int k) { return r * kDK + (k ^ ((r & 3) << 2)); }

// Tile t of the launch order -> (tile row, tile column).
__device__ __forceinline__ void tile_of(const F64Gemm& g, int BT, int t, int& mt, int& nt) {
  const int tm = (g.M + BT - 1) / BT, tn = (g.N + BT - 1) / BT;
  if (g.lower) {  // lower tiles only, row by row (all of equal cost)
    int r = static_cast<int>((sqrtf(8.f * t + 1.f) - 1.f) * 0.5f);
    while (r * (r + 1) / 2 > t) --r;
    while ((r + 1) * (r + 2) / 2 <= t) ++r;
    mt = r;
    nt = t - r * (r + 1) / 2;
    return;
  }
  switch (g.tri) {
    case kTriBLower:  // contraction length grows with the column tile
      nt = tn - 1 - t / tm;
      mt = t % tm;
      break;
    case kTriALower:  // grows with the row tile
      mt = tm - 1 - t / tn;
      nt = t % tn;
      break;
    default:  // kTriAUpper shrinks with the row tile; kTriNone is uniform
      mt = t / tn;
      nt = t % tn;
      break;
  }
}

template <int BT>
__global__ void __launch_bounds__(F64Cfg<BT>::kThreads) f64_gemm_kernel(F64Gemm g, int splits) {
  using Cfg = F64Cfg<BT>;
  extern __shared__ __align__(16) double smem[];
  pdl_wait();
  if (g.skip != nullptr && *g.skip != 0) {
    pdl_launch_dependents();
    return;
  }
  const int t = blockIdx.x / splits, sp = blockIdx.x % splits;
  int mt, nt;
  tile_of(g, BT, t, mt, nt);
  const int m0 = mt * BT, n0 = nt * BT;
  // contraction range of this tile (a triangular operand is zero outside it), slice aligned
  int kbeg = 0, kend = g.Kred;
  if (g.tri == kTriAUpper) kbeg = m0;                 // A[m][k] = 0 for k < m
  if (g.tri == kTriALower) kend = min(kend, m0 + BT);  // A[m][k] = 0 for k > m
  if (g.tri == kTriBLower) kend = min(kend, n0 + BT);  // B[n][k] = 0 for k > n
  const int nch_all = kend > kbeg ? (kend - kbeg) / kDK : 0;
  const int base = nch_all / splits, rem = nch_all % splits;
  const int nch = base + (sp < rem ? 1 : 0);
  const int kfirst = kbeg + (sp * base + min(sp, rem)) * kDK;

  const int tid = threadIdx.x, lane = tid % 32, warp = tid / 32;
  const int wm0 = (warp / Cfg::kWarpsN) * Cfg::kWM, wn0 = (warp % Cfg::kWarpsN) * Cfg::kWN;
  const int fg = lane / 4, ft = lane % 4;

  // loader: 16-byte pair p = tid + threads * u of a slice is row p / 8, k 2 * (p % 8)
  auto load_stage = [&](int stage, int k0) {
    double* As = smem + stage * Cfg::kStageElems;
    double* Bs = As + BT * kDK;
#pragma unroll
    for (int u = 0; u < Cfg::kPairs; ++u) {
      const int p = tid + Cfg::kThreads * u;
      const int r = p / 8, k = 2 * (p % 8);
      const int dst = swz(r, k);
      const bool kin = HQ_IN_BOUNDS(k0 + k + 1 < g.Kred);
      const bool va = m0 + r < g.M && kin, vb = n0 + r < g.N && kin;
      cp_async16(As + dst, g.A + static_cast<int64_t>(va ? m0 + r : m0) * g.lda + k0 + k, va);
      cp_async16(Bs + dst, g.B + static_cast<int64_t>(vb ? n0 + r : n0) * g.ldb + k0 + k, vb);
    }
  };

#pragma unroll
  for (int s = 0; s < kStages - 1; ++s) {
    if (s < nch) load_stage(s, kfirst + s * kDK);
    cp_async_commit();
  }
  double acc[Cfg::kFM][Cfg::kFN][2];
#pragma unroll
  for (int i = 0; i < Cfg::kFM; ++i)
#pragma unroll
    for (int j = 0; j < Cfg::kFN; ++j) acc[i][j][0] = acc[i][j][1] = 0.0;

  for (int c = 0; c < nch; ++c) {
    cp_async_wait<kStages - 2>();  // slice c has landed (this thread's part)
    __syncthreads();               // ... everyone's; and slice c - 1 is no longer read
    {
      const int cn = c + kStages - 1;
      if (cn < nch) load_stage(cn % kStages, kfirst + cn * kDK);
      cp_async_commit();
    }
    const double* As = smem + (c % kStages) * Cfg::kStageElems;
    const double* Bs = As + BT * kDK;
#pragma unroll
    for (int k4 = 0; k4 < kDK; k4 += 4) {
      double a[Cfg::kFM], b[Cfg::kFN];
#pragma unroll
      for (int i = 0; i < Cfg::kFM; ++i) a[i] = As[swz(wm0 + 8 * i + fg, k4 + ft)];
#pragma unroll
      for (int j = 0; j < Cfg::kFN; ++j) b[j] = Bs[swz(wn0 + 8 * j + fg, k4 + ft)];
#pragma unroll
      for (int i = 0; i < Cfg::kFM; ++i)
#pragma unroll
        for (int j = 0; j < Cfg::kFN; ++j) dmma(acc[i][j][0], acc[i][j][1], a[i], b[j]);
    }
  }
  cp_async_wait<0>();
  pdl_launch_dependents();  // the successor may be scheduled while this CTA writes its tile

  // lane holds C rows wm0 + 8 i + fg, columns wn0 + 8 j + 2 ft + {0, 1}
  const int64_t MN = static_cast<int64_t>(g.M) * g.N;
  double* P = splits > 1 ? g.scratch + sp * MN : nullptr;
#pragma unroll
  for (int i = 0; i < Cfg::kFM; ++i) {
    const int m = m0 + wm0 + 8 * i + fg;
    if (m >= g.M) continue;
#pragma unroll
    for (int j = 0; j < Cfg::kFN; ++j) {
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int n = n0 + wn0 + 8 * j + 2 * ft + h;
        if (n >= g.N) continue;
        if (P != nullptr) {
          P[static_cast<int64_t>(m) * g.N + n] = acc[i][j][h];
        } else if (!(g.lower && m < n) && HQ_IN_BOUNDS(n < g.ldc && (g.Ct == nullptr || m < g.ldct))) {
          double* cp = g.C + static_cast<int64_t>(m) * g.ldc + n;
          const double v = (g.beta != 0.0 ? g.beta * *cp : 0.0) + g.alpha * acc[i][j][h];
          *cp = v;
          if (g.Ct != nullptr) g.Ct[static_cast<int64_t>(n) * g.ldct + m] = v;
        }
      }
    }
  }
}

// C = beta C + alpha * (sum of the partial tiles, split 0 first).
__global__ void __launch_bounds__(256) f64_splitk_reduce_kernel(F64Gemm g, int splits) {
  pdl_wait();
  pdl_launch_dependents();
  if (g.skip != nullptr && *g.skip != 0) return;
  const int64_t MN = static_cast<int64_t>(g.M) * g.N;
  for (int64_t e = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; e < MN;
       e += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int m = static_cast<int>(e / g.N), n = static_cast<int>(e % g.N);
    if ((g.lower && m < n) || !HQ_IN_BOUNDS(n < g.ldc && (g.Ct == nullptr || m < g.ldct))) continue;
    double sum = 0.0;
    for (int s = 0; s < splits; ++s) sum += g.scratch[s * MN + e];
    double* c = g.C + static_cast<int64_t>(m) * g.ldc + n;
    const double v = (g.beta != 0.0 ? g.beta * *c : 0.0) + g.alpha * sum;
    *c = v;
    if (g.Ct != nullptr) g.Ct[static_cast<int64_t>(n) * g.ldct + m] = v;
  }
}

template <int BT>
int64_t tile_count(const F64Gemm& g) {
  const int64_t tm = ceil_div(g.M, BT), tn = ceil_div(g.N, BT);
  return g.lower ? tm * (tm + 1) / 2 : tm * tn;
}

// Algorithmic flops of a product: 2 per multiply-add that a triangular operand does not zero
// (for `lower`, only the written elements count).
double f64_gemm_flops(const F64Gemm& g) {
  const double M = g.M, N = g.N, K = g.Kred;
  auto tri_sum = [K](double n) {  // sum_{i < n} min(i + 1, K)
    return n <= K ? n * (n + 1) / 2 : K * (K + 1) / 2 + (n - K) * K;
  };
  if (g.lower) return 2.0 * M * (M + 1) / 2 * K;
  switch (g.tri) {
    case kTriBLower: return 2.0 * M * tri_sum(N);
    case kTriALower: return 2.0 * N * tri_sum(M);
    case kTriAUpper: return 2.0 * N * (M <= K ? M * K - M * (M - 1) / 2 : K * (K + 1) / 2);  // sum max(K - m, 0)
    default: return 2.0 * M * N * K;
  }
}

template <int BT>
hq_status launch_f64(const F64Gemm& g, int64_t tiles, int splits, cudaStream_t s) {
  using Cfg = F64Cfg<BT>;
  const int64_t ctas = tiles * splits;
  if (ctas > 0x7FFFFFFF) return HQ_ERR_UNSUPPORTED;
  HQ_CUDA_TRY(cudaFuncSetAttribute(f64_gemm_kernel<BT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   Cfg::kSmemBytes));
  const int tm = timer_start(BT == 128 ? kTimeF64Gemm128 : kTimeF64Gemm64, s);
  HQ_LAUNCH_CHAINED(launch_chained(f64_gemm_kernel<BT>, dim3(static_cast<unsigned>(ctas)), dim3(Cfg::kThreads),
                                   Cfg::kSmemBytes, s, g, splits));
  if (splits > 1) {
    const int64_t MN = static_cast<int64_t>(g.M) * g.N;
    const int64_t grid = std::min<int64_t>(ceil_div(MN, 256), kSMs * 8);
    HQ_LAUNCH_CHAINED(launch_chained(f64_splitk_reduce_kernel, dim3(static_cast<unsigned>(grid)), dim3(256), 0, s, g,
                                     splits));
  }
  timer_stop(tm, f64_gemm_flops(g), s);
  return HQ_OK;
}

// Number of contraction splits: at least `target_ctas` CTAs where possible, every split at
// least four slices long, all partial tiles within the scratch.
int choose_splits(const F64Gemm& g, int64_t tiles, int64_t target_ctas) {
  if (g.scratch == nullptr || tiles >= target_ctas) return 1;
  const int64_t avg_chunks = (g.Kred / kDK) / (g.tri != kTriNone ? 2 : 1);
  int64_t sp = ceil_div(target_ctas, tiles);
  sp = std::min<int64_t>(sp, std::max<int64_t>(1, avg_chunks / 4));
  sp = std::min<int64_t>(sp, 16);
  const int64_t MN = static_cast<int64_t>(g.M) * g.N;
  sp = std::min<int64_t>(sp, g.scratch_elems / MN);
  return static_cast<int>(std::max<int64_t>(sp, 1));
}

}  // namespace

hq_status f64_gemm(const F64Gemm& g, cudaStream_t s) {
  if (g.M <= 0 || g.N <= 0) return HQ_OK;
  if (g.Kred % kDK != 0 || (g.lower && g.M != g.N)) return HQ_ERR_UNSUPPORTED;
  if ((reinterpret_cast<uintptr_t>(g.A) | reinterpret_cast<uintptr_t>(g.B)) % 16 != 0 || g.lda % 2 != 0 ||
      g.ldb % 2 != 0)
    return HQ_ERR_UNSUPPORTED;
  // 128-wide tiles (one CTA per SM) when they fill the SMs at least once, else 64-wide (up to
  // three per SM, split along the contraction when fewer than two per SM), and for the small
  // products of the recursion's lower levels 32-wide tiles without a split: they finish in about
  // one kernel's latency, where a split costs a second launch (measured: the K = 5120
  // factorisation 5.24 ms against 5.92 with 64-wide split tiles)
  const int64_t t128 = tile_count<128>(g);
  if (t128 >= kSMs) return launch_f64<128>(g, t128, 1, s);
  const int64_t t64 = tile_count<64>(g);
  if (t64 >= kSMs) return launch_f64<64>(g, t64, choose_splits(g, t64, 2 * kSMs), s);
  return launch_f64<32>(g, tile_count<32>(g), 1, s);
}

// fp64 MMA issue rate with nothing else in the way: each warp runs 8 independent accumulator
// chains (the operands are registers; one store per thread at the end).
__global__ void __launch_bounds__(256) fp64_mma_rate_kernel(double* out, int iters) {
  double c0[8], c1[8];
  const double a = 1.0 + threadIdx.x * 1e-9, b = 0.999999;
#pragma unroll
  for (int i = 0; i < 8; ++i) c0[i] = c1[i] = i * 1e-3;
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int i = 0; i < 8; ++i) dmma(c0[i], c1[i], a, b);
  }
  double acc = 0.0;
#pragma unroll
  for (int i = 0; i < 8; ++i) acc += c0[i] + c1[i];
  out[blockIdx.x * blockDim.x + threadIdx.x] = acc;
}

}  // namespace hq

using namespace hq;

extern "C" double hq_debug_fp64_mma_rate(void* scratch, int64_t scratch_bytes, hq_stream_t stream) {
  constexpr int kBlocks = 2 * kSMs, kThreads = 256, kIters = 20000;
  if (scratch == nullptr || scratch_bytes < static_cast<int64_t>(kBlocks) * kThreads * 8) return -1.0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  double* out = static_cast<double*>(scratch);
  fp64_mma_rate_kernel<<<kBlocks, kThreads, 0, s>>>(out, 100);  // warm-up
  cudaEvent_t e0, e1;
  if (cudaEventCreate(&e0) != cudaSuccess) return -1.0;
  if (cudaEventCreate(&e1) != cudaSuccess) {
    cudaEventDestroy(e0);
    return -1.0;
  }
  cudaEventRecord(e0, s);
  fp64_mma_rate_kernel<<<kBlocks, kThreads, 0, s>>>(out, kIters);
  cudaEventRecord(e1, s);
  float ms = 0.f;
  const bool ok = cudaEventSynchronize(e1) == cudaSuccess && cudaEventElapsedTime(&ms, e0, e1) == cudaSuccess;
  cudaEventDestroy(e0);
  cudaEventDestroy(e1);
  if (!ok || ms <= 0.f) {
    (void)cudaGetLastError();
    return -1.0;
  }
  const double flops = 2.0 * 256 * 8 * static_cast<double>(kIters) * kBlocks * (kThreads / 32);
  return flops / (ms * 1e-3) / 1e12;
}
