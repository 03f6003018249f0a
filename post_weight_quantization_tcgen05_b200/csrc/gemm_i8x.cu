// fp64-accurate GEMM on the int8 tensor cores (tcgen05.mma kind::i8), by error-free slicing of
// the fp64 operands (the Ozaki scheme: Ozaki, Ogita, Oishi & Rump 2012; run on integer matrix
// units by Ootomo, Ozaki & Yokota 2024):
//
//   C[m, n] = beta * C[m, n] + alpha * sum_k A(m, k) B(n, k)      m < M, n < N
//   A(m, k) = A[m * lda + k],  B(n, k) = B[n * ldb + k]           (both operands K-major)
//
// Slicing (i8x_slice_kernel, four warps per row).  Row r of an operand is scaled by 2^-e_r, e_r the
// smallest exponent with max_k |x[r, k]| < 2^e_r, and cut into kSlices signed 7-bit integers:
//   y_0 = x 2^-e_r;  d_s = trunc(128 y_s) in [-127, 127];  y_{s+1} = 128 y_s - d_s,
// so x = 2^e_r sum_s d_s 2^(-7 (s + 1)) + 2^(e_r - 7 S) y_S with |y_S| < 1: the base-128 digits of
// |x| 2^-e_r, signed like x.  The kernel reads them off the fp64 bit pattern with integer shifts
// (slice_digits), which gives the same digits as the fp64 steps above.
// The slices are int8, zero outside the part of the row the product reads (a declared triangular
// operand) and past Kred, stored in the shared-memory image of the product's pipeline stages
// (layouts A and B at slice_atom_a / slice_atom_b below).
//
// Product.  x_a x_b = 2^(e_a + e_b) sum_{s,t} d_s d_t 2^(-7 (s + t + 2)): every slice product is
// an exact integer, and the pairs of one anti-diagonal s + t = g share the scale 2^(-7 (g + 2)).
// The pairs with g <= kSlices - 1 are kept (28 of the 49 for 7 slices); the dropped ones and the
// slicing remainders are below about (kSlices + 2) 2^(-7 kSlices) = 1.6e-14 of |x_a| |x_b|
// relative to each operand's row maximum.  Per 128 x 64 output tile the kernel accumulates each
// anti-diagonal in its own int32 TMEM accumulator (7 x 64 columns); the sums are exact while
// 7 * 127^2 * Kred < 2^31 (Kred <= 16384).  The epilogue converts each accumulator to fp64,
// scales it by its power of two, adds the diagonals smallest first, scales by 2^(e_a + e_b) and
// alpha and adds beta C (C is not read when beta == 0); optionally it also stores the result
// transposed (Ct), from the staged chunk, one coalesced row of Ct per column.
//
// Kernel (i8x_gemm_kernel, persistent, one CTA per SM, 192 threads): warp 0 copies each stage
// of the A and the B tile (all 7 slices, 32 bytes of k) with one bulk copy each, 28 KB and 14 KB
// contiguous, into a 4-stage ring; warp 1 issues the kind::i8 MMAs of each stage from one thread
// (M = 128, K = 32; A slice s against the band of B slices 0 .. 6 - s as one operand, N = 64 (7 - s)
// split at 256: 10 MMAs doing the 28 slice-pair products); warps 2-5 drain the accumulators of a
// finished tile (TMEM lane
// quadrant = 32 tile rows each), stage 16-column chunks of the fp64 result in shared memory and
// update C with coalesced 16-byte accesses.  A declared triangular operand shortens each tile's
// contraction to the part where it can be non-zero; tiles are enumerated longest first and dealt
// to the CTAs in waves walked alternately forward and backward.  Every wait is
// bounded; on expiry the CTA records HQ_ERR_TIMEOUT, waits for what it issued and returns.
#include "common.cuh"
#include "kernels.cuh"
#include "ptx.cuh"

namespace hq {
namespace {

constexpr int kSlices = kI8xSlices;
constexpr int kBM = 128, kBN = 64, kBK = 32;       // tile rows, tile columns, contraction bytes per stage
constexpr int kStages = 4;
constexpr int kASlice = kBM * kBK;                  // 4 KB: one slice of an A tile's stage
constexpr int kBSlice = kBN * kBK;                  // 2 KB: one slice of a B tile's stage
constexpr int kStageBytes = kSlices * (kASlice + kBSlice);
constexpr int kABlockBytes = kSlices * kASlice;     // one stage of an A tile: 28 KB, one bulk copy
constexpr int kBBlockBytes = kSlices * kBSlice;     // one stage of a B tile: 14 KB, one bulk copy
constexpr int kEpiWarps = 4;
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr int kChunk = 16;                          // epilogue columns per round
constexpr int kStLd = kChunk + 1;                   // staging row stride (doubles)
constexpr int kEpiBytes = kEpiWarps * 32 * kStLd * 8;
constexpr int kSmem = kStages * kStageBytes + kEpiBytes + 1024 + 256;
constexpr int kTmemCols = 512;                      // kSlices * kBN = 448 used
constexpr int kSMs = 148;
static_assert(kSlices * kBN <= kTmemCols, "accumulators do not fit in TMEM");
static_assert(kStageBytes % 1024 == 0, "stage tiles must stay 1024-byte aligned");

constexpr int kNonFiniteRow = -0x7FFFFFFF;  // exponent marking a row with a NaN or an infinity

// Part of row r (in units of 128 columns) where a declared triangular operand can be non-zero:
// [klo, khi).  `which` 0 = operand A, 1 = operand B.
__host__ __device__ inline void tri_row_range(int tri, int which, int64_t r, int64_t Kred, int64_t& klo,
                                              int64_t& khi) {
  klo = 0;
  khi = Kred;
  const int64_t blk = (r / 128) * 128;
  if (which == 0 && tri == kTriAUpper) klo = blk < Kred ? blk : Kred;
  if (which == 0 && tri == kTriALower) khi = blk + 128 < Kred ? blk + 128 : Kred;
  if (which == 1 && tri == kTriBLower) khi = blk + 128 < Kred ? blk + 128 : Kred;
}

// ------------------------------------------------------------------------- slicing

// Slices of one fp64 value x with |x| < 2^e (e the row exponent), from its bit pattern: with
// x = m 2^(q - 52) (m the 53-bit significand, q the unbiased exponent), the integer
// X = trunc(|x| 2^(7 kSlices - e)) = m >> (52 - 7 kSlices + e - q) has at most 7 kSlices bits, and
// its base-128 digits, most significant first and signed like x, are the slices.  Exactly the
// digits of the sequential construction: truncating toward zero keeps every remainder's sign.
// Packs digit s of x into byte b of w[s].
__device__ __forceinline__ void slice_digits(double x, int e, int b, uint32_t (&w)[kSlices]) {
  const unsigned long long bits = static_cast<unsigned long long>(__double_as_longlong(x));
  const int be = static_cast<int>((bits >> 52) & 0x7FF);
  const unsigned long long m = (bits & 0xFFFFFFFFFFFFFull) | (be != 0 ? (1ull << 52) : 0ull);
  const int q = (be != 0 ? be : 1) - 1023;
  // q < e for normal x, so sh > 0; a subnormal x has fewer significant bits than q says and
  // can need a left shift (X stays below 2^(7 kSlices) since |x| < 2^e)
  const int sh = 52 - 7 * kSlices + e - q;
  const unsigned long long X = sh >= 64 ? 0ull : (sh >= 0 ? (m >> sh) : (m << (-sh)));
  const bool neg = (bits >> 63) != 0;
#pragma unroll
  for (int s = 0; s < kSlices; ++s) {
    int d = static_cast<int>((X >> (7 * (kSlices - 1 - s))) & 127ull);
    d = neg ? -d : d;
    w[s] |= (static_cast<uint32_t>(d) & 0xFFu) << (8 * b);
  }
}

// Slice layouts in global memory: the exact shared-memory image of one pipeline stage, so that a
// stage of a tile is one contiguous bulk copy.  An operand's rows are cut into blocks of the tile
// height (kBM rows for A, kBN for B; the last block padded, its padding rows never written and
// read only into outputs that are not stored), its contraction into 32-byte chunks; the unit is
// the 256-byte atom of 8 rows x 32 bytes in the 32-byte swizzle (the two 16-byte halves of rows
// 4-7 swapped), and the atoms of (chunk, block) lie together:
//   A: [chunk][block][8-row group][slice][atom]   slice s of the tile = 16 atoms 7 x 256 bytes apart
//   B: [chunk][block][slice][8-row group][atom]   the slices stacked along N, as one K-major band
__device__ __forceinline__ int64_t slice_atom_a(int64_t kc, int64_t r, int s, int64_t nblk) {
  return ((kc * nblk + r / kBM) * (kBM / 8) + (r % kBM) / 8) * kSlices + s;
}
__device__ __forceinline__ int64_t slice_atom_b(int64_t kc, int64_t r, int s, int64_t nblk) {
  return ((kc * nblk + r / kBN) * kSlices + s) * (kBN / 8) + (r % kBN) / 8;
}
// byte of (row r, contraction byte c of its 32-byte chunk) inside the atom
__device__ __forceinline__ int slice_in_atom(int64_t r, int c) {
  const int rr = static_cast<int>(r & 7);
  return (rr << 5) | (c ^ (((rr >> 2) & 1) << 4));
}

// kSliceWarps warps per row (two rows per 256-thread CTA): the row maximum over the part the
// product reads (a strided pass, then a warp and a CTA reduction), e_r, then the kSlices int8
// slices of the row, 512 columns per round (each thread 4 consecutive values: two 16-byte loads,
// one 4-byte store per slice and layout written: A, B or both).  The maximum does not depend on
// the order of the reduction.
constexpr int kSliceWarps = 4;
constexpr int kSliceRowThreads = 32 * kSliceWarps;

__global__ void __launch_bounds__(256) i8x_slice_kernel(const double* __restrict__ X, int64_t ldx, int64_t rows,
                                                        int64_t Kred, int64_t Kpad, int tri, int which,
                                                        int8_t* __restrict__ out_a, int64_t nblk_a,
                                                        int8_t* __restrict__ out_b, int64_t nblk_b,
                                                        int* __restrict__ exps, const int* __restrict__ skip) {
  if (skip != nullptr && *skip != 0) return;
  __shared__ double red_mx[256 / 32];
  __shared__ int red_bad[256 / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int t = threadIdx.x % kSliceRowThreads;  // thread within the row's group
  const int64_t r = static_cast<int64_t>(blockIdx.x) * (256 / kSliceRowThreads) + threadIdx.x / kSliceRowThreads;
  const bool valid = r < rows;
  int64_t klo = 0, khi = 0;
  if (valid) tri_row_range(tri, which, r, Kred, klo, khi);
  const double* xr = X + (valid ? r : 0) * ldx;
  // 16-byte loads need an even row start and ldx; otherwise scalar loads
  const bool vec = ((reinterpret_cast<uintptr_t>(xr) & 15) == 0);
  double mx = 0.0;
  bool bad = false;
  for (int64_t k = klo + t; k < khi; k += kSliceRowThreads) {
    const double v = xr[k];
    bad |= !isfinite(v);
    mx = fmax(mx, fabs(v));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmax(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  bad = __any_sync(0xffffffffu, bad);
  if (lane == 0) {
    red_mx[warp] = mx;
    red_bad[warp] = bad ? 1 : 0;
  }
  __syncthreads();  // every thread of the CTA reaches it: the invalid rows only skip their work
  const int w0 = (threadIdx.x / kSliceRowThreads) * kSliceWarps;
  mx = red_mx[w0];
  bad = red_bad[w0] != 0;
#pragma unroll
  for (int w = 1; w < kSliceWarps; ++w) {
    mx = fmax(mx, red_mx[w0 + w]);
    bad |= red_bad[w0 + w] != 0;
  }
  if (!valid) return;
  // a row holding a NaN or an infinity is marked, and its products come out NaN
  const int e = bad ? kNonFiniteRow : (mx > 0.0 ? ilogb(mx) + 1 : 0);
  if (t == 0) exps[r] = e;
  for (int64_t k0 = 4 * t; k0 < Kpad; k0 += 4 * kSliceRowThreads) {
    double v[4];
    if (vec && k0 >= klo && k0 + 4 <= khi) {
      const double2 a = *reinterpret_cast<const double2*>(xr + k0);
      const double2 b = *reinterpret_cast<const double2*>(xr + k0 + 2);
      v[0] = a.x;
      v[1] = a.y;
      v[2] = b.x;
      v[3] = b.y;
    } else {
#pragma unroll
      for (int b = 0; b < 4; ++b) v[b] = (k0 + b >= klo && k0 + b < khi) ? xr[k0 + b] : 0.0;
    }
    uint32_t w[kSlices];
#pragma unroll
    for (int s2 = 0; s2 < kSlices; ++s2) w[s2] = 0u;
    if (!bad) {
#pragma unroll
      for (int b = 0; b < 4; ++b) slice_digits(v[b], e, b, w);
    }
    if (!HQ_IN_BOUNDS(k0 + 4 <= Kpad && khi <= Kred)) continue;
    const int64_t kc = k0 / kBK;
    const int in_atom = slice_in_atom(r, static_cast<int>(k0 % kBK));
    if (out_a != nullptr && HQ_IN_BOUNDS(r / kBM < nblk_a))
      for (int s2 = 0; s2 < kSlices; ++s2)
        *reinterpret_cast<uint32_t*>(out_a + (slice_atom_a(kc, r, s2, nblk_a) << 8) + in_atom) = w[s2];
    if (out_b != nullptr && HQ_IN_BOUNDS(r / kBN < nblk_b))
      for (int s2 = 0; s2 < kSlices; ++s2)
        *reinterpret_cast<uint32_t*>(out_b + (slice_atom_b(kc, r, s2, nblk_b) << 8) + in_atom) = w[s2];
  }
}

// ------------------------------------------------------------------------- product

struct I8xArgs {
  const int8_t* pa;  // A slices, layout A (one stage of a tile = kABlockBytes contiguous bytes)
  const int8_t* pb;  // B slices, layout B (kBBlockBytes per stage of a tile)
  int nblk_a, nblk_b;
  double* C;
  int64_t ldc;
  double* Ct;  // optional transposed copy of what is written
  int64_t ldct;
  int M, N, Kpad;
  int tiles_m, tiles_n, tiles;
  double alpha, beta;
  int lower, tri;
  const int* eA;
  const int* eB;
  const int* skip;
  int* status;
};

// Tile t in execution order -> (m0, n0, first and last contraction stage).  Longest contraction
// first: with A upper the low tile rows, with A lower the high ones, with B lower the high tile
// columns.  With `lower`, only tiles holding an element m >= n are enumerated.
__device__ inline void i8x_tile(const I8xArgs& a, int t, int& m0, int& n0, int& kb0, int& kb1) {
  int tm, tn;
  if (a.lower) {
    // tile row tm holds column tiles 0 .. min(2 tm + 1, tiles_n - 1); rows walked from the last
    int rem = t;
    tm = a.tiles_m - 1;
    for (;; --tm) {
      const int cnt = (2 * tm + 2 < a.tiles_n) ? 2 * tm + 2 : a.tiles_n;
      if (rem < cnt || tm == 0) {
        tn = rem;
        break;
      }
      rem -= cnt;
    }
  } else if (a.tri == kTriBLower) {
    tn = a.tiles_n - 1 - t / a.tiles_m;
    tm = t % a.tiles_m;
  } else if (a.tri == kTriALower) {
    tm = a.tiles_m - 1 - t / a.tiles_n;
    tn = t % a.tiles_n;
  } else {
    tm = t / a.tiles_n;
    tn = t % a.tiles_n;
  }
  m0 = tm * kBM;
  n0 = tn * kBN;
  int64_t lo = 0, hi = a.Kpad;
  if (a.tri == kTriAUpper) lo = m0;
  if (a.tri == kTriALower) hi = m0 + kBM;
  if (a.tri == kTriBLower) hi = (n0 / 128) * 128 + 128;
  if (hi > a.Kpad) hi = a.Kpad;
  if (lo > hi) lo = hi;
  kb0 = static_cast<int>(lo / kBK);
  kb1 = static_cast<int>((hi + kBK - 1) / kBK);
}

// The i-th tile of persistent CTA b of G: waves of G tiles walked alternately forward and backward.
// Tiles are enumerated longest contraction first, so a CTA that takes a wave's longest tile takes
// the next wave's shortest; on the factorisation's triangular products (tile lengths falling
// linearly) this brings the busiest CTA from about 1.18 to 1.02 times the mean work.
__device__ __forceinline__ int i8x_cta_tile(int i, int b, int G) { return i * G + ((i & 1) ? G - 1 - b : b); }

// K-major operand tile with 32-byte rows and the 32-byte swizzle (layout type 6): 8-row atoms
// of 256 bytes, consecutive atoms (8 rows further along M or N) `sbo` bytes apart.
__device__ __forceinline__ uint64_t sdesc_sw32(uint32_t saddr, uint32_t sbo = 256) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>(16 >> 4) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1) << 46;
  d |= static_cast<uint64_t>(6) << 61;
  return d;
}

// kind::i8 MMA, D[tmem] (+)= A[smem] B[smem]^T.  Use selects what happens to the A operand in
// the tensor core's collector buffer: 0 read from shared memory and dropped (the default), 1 read
// and kept (fill), 2 taken from the buffer and kept (use), 3 taken from the buffer and dropped
// (lastuse).
template <int Use>
__device__ __forceinline__ void mma_i8(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
#define HQ_I8_MMA(Q)                                                                              \
  asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"                               \
               "tcgen05.mma.cta_group::1.kind::i8" Q " [%0], %1, %2, %3, p;\n\t}\n" ::"r"(tmem_d), \
               "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)                                \
               : "memory")
  if constexpr (Use == 1)
    HQ_I8_MMA(".collector::a::fill");
  else if constexpr (Use == 2)
    HQ_I8_MMA(".collector::a::use");
  else if constexpr (Use == 3)
    HQ_I8_MMA(".collector::a::lastuse");
  else
    HQ_I8_MMA("");
#undef HQ_I8_MMA
}

// The MMAs of one stage.  The B slices of a stage lie one after another in shared memory, so B
// slices 0 .. kSlices - 1 - P form a single K-major matrix of kBN (kSlices - P) rows, and
// A slice P times that band lands slice pair (P, t) in columns kBN (P + t) .. of the accumulator:
// exactly the columns of anti-diagonal P + t.  One wide MMA per A slice (split at 256 columns)
// instead of one narrow MMA per slice pair: the tensor core's time per instruction hardly
// depends on N, so wide instructions keep it busy.  10 MMAs per stage for 7 slices.
template <int P, int C>
__device__ __forceinline__ void mma_band(uint32_t tmem, uint64_t ad, uint32_t sb, uint32_t first) {
  constexpr int total = kBN * (kSlices - P);
  constexpr int n0 = 256 * C;
  if constexpr (n0 < total) {
    constexpr int n = (total - n0) < 256 ? (total - n0) : 256;
    static_assert(n % 16 == 0 && n >= 16, "MMA width");
    constexpr uint32_t idesc = (2u << 4) | (1u << 7) | (1u << 10) | ((static_cast<uint32_t>(n) >> 3) << 17) |
                               ((static_cast<uint32_t>(kBM) >> 4) << 24);
    mma_i8<0>(tmem + static_cast<uint32_t>(P * kBN + n0), ad, sdesc_sw32(sb + n0 * kBK), idesc,
              (first && P == 0) ? 0u : 1u);
    mma_band<P, C + 1>(tmem, ad, sb, first);
  }
}
template <int P>
__device__ __forceinline__ void mma_stage(uint32_t tmem, uint32_t sa, uint32_t sb, uint32_t first) {
  if constexpr (P < kSlices) {
    mma_band<P, 0>(tmem, sdesc_sw32(sa + P * 256, 256 * kSlices), sb, first);
    mma_stage<P + 1>(tmem, sa, sb, first);
  }
}

// 32 lanes x 16 consecutive 32-bit TMEM columns, no wait.
__device__ __forceinline__ void tmem_ld16_nowait(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__global__ void __launch_bounds__(kThreads, 1)
    i8x_gemm_kernel(const __grid_constant__ I8xArgs args) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  double* stage_c = reinterpret_cast<double*>(smem + kStages * kStageBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kStages * kStageBytes + kEpiBytes);
  uint64_t* empty = full + kStages;
  uint64_t* accf = empty + kStages;  // accumulators filled (one tile's MMAs done)
  uint64_t* acce = accf + 1;         // accumulators drained
  uint64_t* drain = acce + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  if (args.skip != nullptr && *args.skip != 0) return;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      ptx::mbar_init(&full[s], 1);
      ptx::mbar_init(&empty[s], 1);
    }
    ptx::mbar_init(accf, 1);
    ptx::mbar_init(acce, kEpiWarps);
    ptx::mbar_init(drain, 1);
    *abort_flag = 0;
    ptx::fence_barrier_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(tmem_slot, kTmemCols);
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
    // ------------------------------------------------------------ bulk-copy producer
    int g = 0;
    bool ok = true;
    for (int j = 0, t = i8x_cta_tile(0, blockIdx.x, gridDim.x); t < args.tiles && ok;
         t = i8x_cta_tile(++j, blockIdx.x, gridDim.x)) {
      int m0, n0, kb0, kb1;
      i8x_tile(args, t, m0, n0, kb0, kb1);
      for (int kb = kb0; kb < kb1; ++kb, ++g) {
        const int s = g % kStages;
        if (g >= kStages && !ptx::mbar_wait(&empty[s], ((g / kStages) - 1) & 1, abort_flag)) {
          ok = false;
          break;
        }
        uint8_t* st = smem + s * kStageBytes;
        ptx::mbar_arrive_expect_tx(&full[s], kStageBytes);
        // the stage of the A tile and of the B tile: one contiguous copy each
        const bool in = HQ_IN_BOUNDS(kb < args.Kpad / kBK && m0 / kBM < args.nblk_a && n0 / kBN < args.nblk_b);
        const int8_t* srca = args.pa + (in ? (static_cast<int64_t>(kb) * args.nblk_a + m0 / kBM) * kABlockBytes : 0);
        const int8_t* srcb = args.pb + (in ? (static_cast<int64_t>(kb) * args.nblk_b + n0 / kBN) * kBBlockBytes : 0);
        asm volatile(
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                ptx::smem_u32(st)),
            "l"(srca), "r"(kABlockBytes), "r"(ptx::smem_u32(&full[s]))
            : "memory");
        asm volatile(
            "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                ptx::smem_u32(st + kABlockBytes)),
            "l"(srcb), "r"(kBBlockBytes), "r"(ptx::smem_u32(&full[s]))
            : "memory");
      }
    }
    if (!ok) {
      fail();
      const int first = g > kStages ? g - kStages : 0;
      for (int k = first; k < g; ++k) ptx::mbar_wait(&full[k % kStages], (k / kStages) & 1, nullptr);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    int g = 0, i = 0;
    bool ok = true;
    for (int t = i8x_cta_tile(0, blockIdx.x, gridDim.x); t < args.tiles && ok; t = i8x_cta_tile(++i, blockIdx.x, gridDim.x)) {
      int m0, n0, kb0, kb1;
      i8x_tile(args, t, m0, n0, kb0, kb1);
      if (i >= 1 && !ptx::mbar_wait(acce, (i - 1) & 1, abort_flag)) {
        ok = false;
        break;
      }
      ptx::tc_fence_after();
      for (int kb = kb0; kb < kb1; ++kb, ++g) {
        const int s = g % kStages;
        if (!ptx::mbar_wait(&full[s], (g / kStages) & 1, abort_flag)) {
          ok = false;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t sa = ptx::smem_u32(smem + s * kStageBytes);
        const uint32_t sb = sa + kSlices * kASlice;
        // the first stage of a tile overwrites each accumulator with its first product (P == 0)
        mma_stage<0>(tmem, sa, sb, kb == kb0 ? 1u : 0u);
        ptx::mma_commit(&empty[s]);
      }
      if (!ok) break;
      ptx::mma_commit(accf);  // (a tile with an empty contraction issues no MMA: its result is 0)
    }
    if (!ok) {
      fail();
      ptx::mma_commit(drain);
      ptx::mbar_wait(drain, 0, nullptr);
    }
  } else if (warp >= 2) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quadrant: tile rows 32 q .. 32 q + 31
    const uint32_t lane_off = static_cast<uint32_t>(q * 32) << 16;
    double* st = stage_c + (warp - 2) * 32 * kStLd;
    bool ok = true;
    int i = 0;
    for (int t = i8x_cta_tile(0, blockIdx.x, gridDim.x); t < args.tiles; t = i8x_cta_tile(++i, blockIdx.x, gridDim.x)) {
      int m0, n0, kb0, kb1;
      i8x_tile(args, t, m0, n0, kb0, kb1);
      if (ok) {
        ok = ptx::mbar_wait(accf, i & 1, abort_flag);
        ptx::tc_fence_after();
      }
      if (!ok) break;
      const int row = m0 + q * 32 + lane;
      const int er = (row < args.M) ? args.eA[row] : 0;
      const bool empty_k = kb1 <= kb0;
      for (int c = 0; c < kBN / kChunk; ++c) {
        double v[kChunk];
#pragma unroll
        for (int j = 0; j < kChunk; ++j) v[j] = 0.0;
        if (!empty_k) {
          uint32_t r[kSlices][16];
#pragma unroll
          for (int d = 0; d < kSlices; ++d)
            tmem_ld16_nowait(tmem + lane_off + static_cast<uint32_t>(d * kBN + c * kChunk), r[d]);
          ptx::tmem_wait_ld();
          // smallest diagonal first: sum_d acc_d 2^(-7 (d + 2)), then 2^e_row
#pragma unroll
          for (int d = kSlices - 1; d >= 0; --d) {
            const double sc = ldexp(1.0, -7 * (d + 2));
#pragma unroll
            for (int j = 0; j < kChunk; ++j) v[j] = fma(static_cast<double>(static_cast<int>(r[d][j])), sc, v[j]);
          }
#pragma unroll
          for (int j = 0; j < kChunk; ++j) v[j] = er == kNonFiniteRow ? __longlong_as_double(0x7FF8000000000000LL)
                                                                       : ldexp(v[j], er);
        }
        if (c == kBN / kChunk - 1) {  // every accumulator column of this tile has been read
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(acce);
        }
#pragma unroll
        for (int j = 0; j < kChunk; ++j) st[lane * kStLd + j] = v[j];
        __syncwarp();
        // the warp's 32 rows x 16 columns: 4 rows per instruction, 8 lanes x 2 columns per row
        const int cl = 2 * (lane & 7);
        const int col = n0 + c * kChunk + cl;
        const int ec0 = (col < args.N) ? args.eB[col] : 0;
        const int ec1 = (col + 1 < args.N) ? args.eB[col + 1] : 0;
#pragma unroll
        for (int it = 0; it < 8; ++it) {
          const int rl = 4 * it + (lane >> 3);
          const int m = m0 + q * 32 + rl;
          if (m >= args.M || !HQ_IN_BOUNDS(col < args.ldc)) continue;
          double* crow = args.C + static_cast<int64_t>(m) * args.ldc;
          const double nan = __longlong_as_double(0x7FF8000000000000LL);
          const double p0 = ec0 == kNonFiniteRow ? nan : args.alpha * ldexp(st[rl * kStLd + cl], ec0);
          const double p1 = ec1 == kNonFiniteRow ? nan : args.alpha * ldexp(st[rl * kStLd + cl + 1], ec1);
          const bool w0 = col < args.N && (!args.lower || m >= col);
          const bool w1 = col + 1 < args.N && (!args.lower || m >= col + 1);
          if (w0) {
            const double v = args.beta == 0.0 ? p0 : fma(args.beta, crow[col], p0);
            crow[col] = v;
            st[rl * kStLd + cl] = v;
          }
          if (w1) {
            const double v = args.beta == 0.0 ? p1 : fma(args.beta, crow[col + 1], p1);
            crow[col + 1] = v;
            st[rl * kStLd + cl + 1] = v;
          }
        }
        __syncwarp();
        if (args.Ct != nullptr) {  // the transpose: row n of Ct takes the warp's 32 rows, one per lane
          const int m = m0 + q * 32 + lane;
#pragma unroll 4
          for (int j = 0; j < kChunk; ++j) {
            const int n = n0 + c * kChunk + j;
            if (m < args.M && n < args.N && (!args.lower || m >= n) && HQ_IN_BOUNDS(m < args.ldct))
              args.Ct[static_cast<int64_t>(n) * args.ldct + m] = st[lane * kStLd + j];
          }
        }
        __syncwarp();
      }
    }
    if (!ok) fail();
  }

  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, kTmemCols);
  }
}

// Slices of X's rows into layout A (out_a) and/or layout B (out_b); either may be null.
hq_status slice(const double* X, int64_t ldx, int64_t rows, int64_t Kred, int64_t Kpad, int tri, int which,
                int8_t* out_a, int8_t* out_b, int* exps, const int* skip, cudaStream_t s) {
  const int64_t grid = ceil_div(rows, 256 / kSliceRowThreads);
  i8x_slice_kernel<<<static_cast<unsigned>(grid), 256, 0, s>>>(X, ldx, rows, Kred, Kpad, tri, which, out_a,
                                                              ceil_div(rows, kBM), out_b, ceil_div(rows, kBN),
                                                              exps, skip);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

}  // namespace

int64_t i8x_kpad(int64_t Kred) { return (Kred + kBK - 1) / kBK * kBK; }

// Slices of A (rows padded to whole kBM blocks) and of B (whole kBN blocks), then the row exponents.
size_t i8x_slices_a_bytes(int64_t M, int64_t kp) {
  return round_up(static_cast<size_t>(kSlices) * round_up(static_cast<size_t>(M), kBM) * kp, 256);
}
size_t i8x_slices_b_bytes(int64_t N, int64_t kp) {
  return round_up(static_cast<size_t>(kSlices) * round_up(static_cast<size_t>(N), kBN) * kp, 256);
}

size_t i8x_scratch_bytes(int64_t M, int64_t N, int64_t Kred) {
  const size_t kp = static_cast<size_t>(i8x_kpad(Kred));
  const size_t a = i8x_slices_a_bytes(M, kp);
  const size_t b = i8x_slices_b_bytes(N, kp);
  return a + b + round_up(static_cast<size_t>(M) * 4, 256) + round_up(static_cast<size_t>(N) * 4, 256);
}

bool i8x_eligible(const F64Gemm& g) {
  return g.Kred >= 1 && g.Kred <= kI8xMaxKred && g.M >= 1 && g.N >= 1 && (!g.lower || g.M == g.N);
}

hq_status i8x_gemm(const F64Gemm& g, uint8_t* scratch, size_t scratch_bytes, cudaStream_t s) {
  if (g.M <= 0 || g.N <= 0) return HQ_OK;
  if (!i8x_eligible(g)) return HQ_ERR_UNSUPPORTED;
  if (scratch == nullptr || !aligned(scratch, 256) || scratch_bytes < i8x_scratch_bytes(g.M, g.N, g.Kred))
    return HQ_ERR_WORKSPACE;
  const int64_t kp = i8x_kpad(g.Kred);
  int8_t* pa = reinterpret_cast<int8_t*>(scratch);
  // the same matrix as both operands (A22 -= T T^T): read and sliced once, written in both layouts
  const bool same = g.A == g.B && g.lda == g.ldb && g.M == g.N && g.tri == kTriNone;
  int8_t* pb = pa + i8x_slices_a_bytes(g.M, kp);
  int* ea = reinterpret_cast<int*>(pb + i8x_slices_b_bytes(g.N, kp));
  int* eb = same ? ea : ea + round_up(static_cast<size_t>(g.M) * 4, 256) / 4;
  const int ts = timer_start(kTimeI8xSlice, s);
  hq_status st = slice(g.A, g.lda, g.M, g.Kred, kp, g.tri, 0, pa, same ? pb : nullptr, ea, g.skip, s);
  if (st != HQ_OK) return st;
  if (!same) {
    st = slice(g.B, g.ldb, g.N, g.Kred, kp, g.tri, 1, nullptr, pb, eb, g.skip, s);
    if (st != HQ_OK) return st;
  }
  // bytes: each operand's rows read once in fp64, kSlices slices written
  timer_stop(ts, (same ? 1.0 : 2.0) * 0.5 * (g.M + g.N) * (8.0 * g.Kred + kSlices * static_cast<double>(kp)), s);
  I8xArgs a{};
  a.pa = pa;
  a.pb = pb;
  a.nblk_a = static_cast<int>(ceil_div(g.M, kBM));
  a.nblk_b = static_cast<int>(ceil_div(g.N, kBN));
  a.C = g.C;
  a.ldc = g.ldc;
  a.Ct = g.Ct;
  a.ldct = g.ldct;
  a.M = g.M;
  a.N = g.N;
  a.Kpad = static_cast<int>(kp);
  a.tiles_m = static_cast<int>(ceil_div(g.M, kBM));
  a.tiles_n = static_cast<int>(ceil_div(g.N, kBN));
  int64_t tiles = 0;
  if (g.lower) {
    for (int tmi = 0; tmi < a.tiles_m; ++tmi) tiles += (2 * tmi + 2 < a.tiles_n) ? 2 * tmi + 2 : a.tiles_n;
  } else {
    tiles = static_cast<int64_t>(a.tiles_m) * a.tiles_n;
  }
  if (tiles > 0x7FFFFFFF) return HQ_ERR_UNSUPPORTED;
  a.tiles = static_cast<int>(tiles);
  a.alpha = g.alpha;
  a.beta = g.beta;
  a.lower = g.lower;
  a.tri = g.tri;
  a.eA = ea;
  a.eB = eb;
  a.skip = g.skip;
  a.status = g.status;
  HQ_CUDA_TRY(cudaFuncSetAttribute(i8x_gemm_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem));
  const int grid = static_cast<int>(tiles < kSMs ? tiles : kSMs);
  const int tm = timer_start(kTimeI8xGemm, s);
  i8x_gemm_kernel<<<grid, kThreads, kSmem, s>>>(a);
  HQ_LAUNCH_CHECK();
  // work: 2 flops per multiply-add a declared triangular operand leaves non-zero (the fp64
  // product's own count, as for the fp64 kernel)
  double flops = 2.0 * g.M * g.N * static_cast<double>(g.Kred);
  if (g.tri != kTriNone || g.lower) flops *= 0.5;
  timer_stop(tm, flops, s);
  return HQ_OK;
}

}  // namespace hq
