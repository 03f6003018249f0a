// Internal launchers shared between the translation units of libhq (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hq.h"
#include "common.cuh"

namespace hq {

// syrk.cu
bool syrk_tc_eligible(const void* X, int x_dtype, int64_t T, int64_t K);
// wait_limit: cycles a pipeline wait may take before the kernel records HQ_ERR_TIMEOUT and stops;
// withhold_stage >= 0 (tests of that path only): the MMA issuer never releases that ring stage.
hq_status launch_syrk_tc(float* H, const void* X, int64_t T, int64_t K, int* dev_status, cudaStream_t s,
                         long long wait_limit = kWaitLimitCycles, int withhold_stage = -1);
hq_status launch_syrk_simt(float* H, const void* X, int x_dtype, int64_t T, int64_t K, cudaStream_t s);

// tril32.cu: the lower triangle of H packed row by row (pack: H -> packed; else packed -> H's
// lower triangle)
hq_status launch_tril32(const float* src, float* dst, int64_t K, bool pack, cudaStream_t s);

// codec.cu
hq_status launch_tril_encode(const float* H, int64_t K, uint8_t* out, cudaStream_t s);
hq_status launch_tril_decode(const uint8_t* in, int64_t K, float* H, cudaStream_t s);

// gemm_upd.cu: C -= (A_hi + A_lo) (B_hi + B_lo)^T in 3xTF32 on tcgen05 (the GPTQ lazy updates),
// operands pre-split into tf32 and remainder parts, K-major, 16-byte aligned rows.
struct UpdGemm {
  float* C;
  int64_t ldc;
  int M, N, Kred;
  const float* A_hi;
  const float* A_lo;
  int64_t lda;
  const float* B_hi;
  const float* B_lo;
  int64_t ldb;
  const int* skip;
  int* status;
};
hq_status upd_gemm(const UpdGemm& g, cudaStream_t s);

// psd.cu: H <- its projection onto the PSD cone (steps Newton-Schulz steps for sign(H));
// workspace of psd_workspace(K) bytes, 256-byte aligned; `status` a device int (timeouts).
size_t psd_workspace(int64_t K);
hq_status launch_psd(float* H, int64_t K, int steps, uint8_t* ws, int* status, cudaStream_t s);

// hadamard.cu: rotation by R = diag(s) blockdiag(Hadamard_B / sqrt B)
bool hadamard_shape_ok(int64_t K, int64_t B);
hq_status launch_hadamard_rows(const void* A, int a_dtype, int64_t rows, int64_t K, int B, const float* s,
                               float* out, cudaStream_t st);  // out = A R (out may be A when fp32)
hq_status launch_hadamard_cols(float* A, int64_t K, int B, const float* s, cudaStream_t st);  // A <- R^T A
hq_status launch_mirror_lower(const float* H, int64_t K, float* out, cudaStream_t st);
// out = R^T H R (both triangles), H read as the symmetric matrix of its lower triangle; out != H.
hq_status launch_hadamard_hessian(const float* H, int64_t K, int B, const float* s, float* out, cudaStream_t st);

// timing.cu: optional event timing of kernel classes (hq_debug_timing_*).  timer_start returns
// -1 (and records nothing) unless the class is being timed; `work` is the launch's algorithmic
// flops or bytes.
enum TimerClass {
  kTimeF64Gemm128 = 0,  // f64_gemm_kernel, 128-wide tiles (flops)
  kTimeF64Gemm64 = 1,   // f64_gemm_kernel, 64-wide tiles, with its split-K reduction (flops)
  kTimeLeaf = 2,        // chol_inv_leaf_kernel (flops of Cholesky + triangular inverse)
  kTimeSweep = 3,       // sweep_block_kernel (bytes)
  kTimeTf32Gemm = 4,    // upd_gemm_kernel (flops of the product, not of its 3 tf32 passes)
  kTimeSyrk = 5,        // tcgen05 SYRK (flops)
  kTimeI8xGemm = 6,     // i8x_gemm_kernel (flops of the fp64 product it emulates)
  kTimeI8xSlice = 7,    // i8x_slice_kernel (bytes: fp64 operand read, int8 slices written)
};
int timer_start(int cls, cudaStream_t s);
void timer_stop(int idx, double work, cudaStream_t s);
// True after hq_debug_timing_serialize(1): work that would overlap on a second stream then runs
// on the caller's stream, so that each launch's events bracket that launch alone (as in a
// serialised profiler launch list).
bool timing_serialized();

// gemm_f64.cu: C = beta C + alpha A B^T in fp64 on the fp64 tensor cores
enum F64Tri { kTriNone = 0, kTriAUpper = 1, kTriALower = 2, kTriBLower = 3 };
struct F64Gemm {
  double* C;
  int64_t ldc;
  int M, N, Kred;   // Kred a multiple of 16
  const double* A;  // A(m, k) = A[m * lda + k]
  int64_t lda;
  const double* B;  // B(n, k) = B[n * ldb + k]
  int64_t ldb;
  double alpha, beta;
  int lower;        // write only m >= n (M == N)
  int tri;          // F64Tri: which operand is triangular (zero outside its triangle)
  double* scratch;  // room for split-K partial tiles (may be NULL: no split)
  int64_t scratch_elems;
  const int* skip;
  int* status;      // device status word for bounded-wait timeouts (may be NULL)
  double* Ct;       // optional: every written C[m][n] also stored at Ct[n * ldct + m]
  int64_t ldct;
};
hq_status f64_gemm(const F64Gemm& g, cudaStream_t s);

// gemm_i8x.cu: the same product, fp64-accurate, on the int8 tensor cores (tcgen05 kind::i8) from
// kI8xSlices int8 slices per operand row.  `scratch` (256-byte aligned) holds the slices and the
// row exponents: i8x_scratch_bytes(M, N, Kred) bytes.  Kred <= kI8xMaxKred keeps the int32 sums
// exact.
constexpr int kI8xSlices = 7;
constexpr int64_t kI8xMaxKred = 16384;
int64_t i8x_kpad(int64_t Kred);
size_t i8x_scratch_bytes(int64_t M, int64_t N, int64_t Kred);
bool i8x_eligible(const F64Gemm& g);
hq_status i8x_gemm(const F64Gemm& g, uint8_t* scratch, size_t scratch_bytes, cudaStream_t s);

// factor.cu: out[i] = 1 / d[i] by the leaf's Newton-Raphson reciprocal (for tests)
hq_status launch_rcp_nr(const double* d, double* out, int64_t n, cudaStream_t s);

// Packed diagonal blocks of U' = diag(U)^-1 U for the GPTQ sweep: block b (kSweepBlk^2 floats)
// holds, for row j of the block, lane l (0..15) and slot m (0..7), the entry
// U'[b kSweepBlk + j][b kSweepBlk + c] with c = 16 (j / 16 + m) + l when j < c < kSweepBlk,
// and 0 otherwise (on and below the diagonal, and past the block).  A lane's 8 slots are two
// 16-byte chunks, swapped for lanes 4-7 and 12-15 so that eight lanes reading chunk q of one
// row j hit 32 different banks.
constexpr int kSweepBlk = 128;
__host__ __device__ __forceinline__ int sweep_upack_offset(int j, int l, int m) {
  return ((j * 16 + l) * 2 + ((m >> 2) ^ ((l >> 2) & 1))) * 4 + (m & 3);
}
// The band of U' right of each diagonal block, for the updates inside a 512-column panel:
// band b (kSweepBlk x kSweepBand floats, row-major) holds U'[b kSweepBlk + k][(b + 1) kSweepBlk + c]
// for k < kSweepBlk, c < kSweepBand (0 past column K - 1).
constexpr int kSweepBand = 384;

// factor.cu: the upper Cholesky factor U of the inverse of the damped Hessian, in fp32, from an
// fp64 factorisation.  A, X, XT, T are K x K fp64 scratch; `slices` (NULL: every product on the
// fp64 tensor cores) holds 2 * factor_slice_bytes(K) bytes, 256-byte aligned: the int8 slices of
// the large products' operands, one half per stream.  Outputs (each may be NULL; they must not
// overlap X or XT; they may overlap A and T, which are dead by then):
//   sweep_form == false: U (row-major, upper) and Ut = U^T (row-major, lower).
//   sweep_form == true:  U receives the packed diagonal blocks of U' = diag(U)^-1 U (K / kSweepBlk
//                        blocks, see sweep_upack_offset; K a multiple of kSweepBlk) followed by
//                        its bands (K kSweepBand floats, see kSweepBand), and Ut = U'^T
//                        (row-major, lower, unit diagonal).
//   Ut_hi, Ut_lo: the strict lower triangle of the same Ut split into a tf32 part and the fp32
//                 remainder (their upper parts are not written).
// With Ut == NULL and sweep_form, only the strict lower triangle of Ut is ever formed.
size_t factor_slice_bytes(int64_t K);
hq_status launch_factor(const float* H, int64_t K, float damp, double* A, double* X, double* XT, double* T,
                        uint8_t* slices, double* lam, int* info, int* status, bool sweep_form, float* Ut, float* U,
                        float* Ut_hi, float* Ut_lo, cudaStream_t s);

// The factor buffer: everything the GPTQ sweep needs from the factorisation, in one block that
// ranks sharing a layer's rows can broadcast.  Header, packed diagonal blocks of U', its bands, and the
// strict lower triangle of U'^T split into its tf32 part (hi) and fp32 remainder (lo); for the
// CUDA-core updates hi holds U'^T itself.
struct FactorHeader {
  int info;  // factorisation status: 0 ok, k > 0 first failing pivot, -1 mean(diag) <= 0
  int pad;
  double lam;
};
struct FactorLayout {
  size_t hdr, upack, band, hi, lo, total;
};
FactorLayout factor_layout(int64_t K);

// gptq.cu
struct GptqLayout {
  size_t header, partials, wf, err, err_lo, sweep_total, t, a, x, xt, slices, total;
  int sweep_rows, sweep_grid;  // rows per sweep CTA, sweep CTAs
};
// Device-side header at the start of the GPTQ / RTN workspace.
struct WsHeader {
  int info;      // factorisation: 0 ok, k > 0 first failing pivot (1-based), -1 mean(diag) <= 0
  int status;    // HQ_ERR_TIMEOUT when a bounded wait expired
  double lam;    // damping added to the diagonal
  double qerr;   // final qerr
  double num, den;
};
bool gptq_shape_ok(int64_t N, int64_t K, int64_t group);
GptqLayout gptq_layout(int64_t N, int64_t K, int64_t group);
// The workspace of the factorisation alone: the header at 0, then its scratch (t .. slices).
GptqLayout factor_ws_layout(int64_t K);
// Damping and factorisation into `factor` (factor_layout(K).total bytes); `ws` laid out as L.
// plain_ut: U'^T unsplit in the hi slot (the CUDA-core updates) instead of the split.
hq_status launch_factorize(const float* H, int64_t K, float damp, uint8_t* ws, const GptqLayout& L, uint8_t* factor,
                           bool plain_ut, cudaStream_t s);
// The sweep of W's N rows against a factor buffer, in a workspace whose first L.sweep_total bytes
// follow gptq_layout(N, K, group).  update_impl 0: 3xTF32 tensor cores, 1: fp32 CUDA cores (the
// factor then holds U'^T unsplit).
hq_status launch_sweep(const void* W, int w_dtype, int64_t N, int64_t K, int64_t group, const float* imp,
                       uint8_t* codes, float* scales, double* qerr_dev, uint8_t* ws, const uint8_t* factor,
                       int update_impl, bool reset_header, cudaStream_t s);
hq_status launch_gptq(const void* W, int w_dtype, int64_t N, int64_t K, const float* H, int64_t group, float damp,
                      const float* imp, uint8_t* codes, float* scales, double* qerr_dev, uint8_t* ws,
                      int update_impl, cudaStream_t s);

// rtn.cu
size_t rtn_workspace(int64_t N, int64_t K, int64_t group);
hq_status launch_rtn(const void* W, int w_dtype, int64_t N, int64_t K, int64_t group, const float* imp,
                     uint8_t* codes, float* scales, double* qerr_dev, uint8_t* ws, cudaStream_t s);

// gptq.cu: qerr reduction shared by GPTQ and RTN
// (finfo: optional device int copied into hdr->info, the factorisation's status)
hq_status launch_qerr_finalize(const double* partials, int64_t count, WsHeader* hdr, double* qerr_dev,
                               cudaStream_t s, const int* finfo = nullptr);

}  // namespace hq
