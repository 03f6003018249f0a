/*
 * hq_debug.h -- stage-level entry points of libhq.so for parity tests and profiling.
 * They run single stages of the path that hq.h composes, so each stage can be compared
 * with the oracle on its own.  Same conventions as hq.h (device pointers, caller-owned
 * memory, refusal before launch, asynchronous unless stated).
 */
#ifndef HQ_DEBUG_H
#define HQ_DEBUG_H

#include "hq.h"

#ifdef __cplusplus
extern "C" {
#endif

/*
 * The damping + factorisation stage of hq_gptq_quantize alone: writes U^T (fp32 [K, K],
 * row-major; U^T[c, j] = U[j, c] for c >= j, zero above the diagonal) where U is the upper
 * Cholesky factor of (H + damp * mean(diag H) I)^-1 ([gptq] experiment summary, "Cholesky-
 * based Hessian inverse").  Uses hq_gptq_factor_workspace_bytes(K) bytes of workspace (which
 * hq_gptq_workspace_bytes(N, K, group) always exceeds).
 * Synchronises `stream` and returns HQ_ERR_NOT_PD / HQ_ERR_INVALID like hq_gptq_quantize.
 */
hq_status hq_debug_factor(const float* H, int64_t K, float damp, float* Ut_out, void* workspace,
                          size_t workspace_bytes, hq_stream_t stream);

/*
 * hq_gptq_quantize with an explicit choice of the lazy-update kernel:
 * update_impl 0 = tcgen05 tensor cores in 3xTF32 (the default path), 1 = fp32 CUDA cores
 * (reference for the tensor-core one).
 */
hq_status hq_debug_gptq_quantize_impl(const void* W, int w_dtype, int64_t N, int64_t K, const float* H,
                                      int64_t group, float damp, const float* imp, uint8_t* codes,
                                      float* scales, double* qerr_out, double* qerr_dev, void* workspace,
                                      size_t workspace_bytes, int update_impl, hq_stream_t stream);

/*
 * hq_hessian_accumulate with an explicit kernel choice: impl 0 = automatic (tcgen05 for
 * eligible bf16 inputs), 1 = fp32 CUDA-core kernel for every input.
 */
hq_status hq_debug_hessian_accumulate_impl(float* H, const void* X, int x_dtype, int64_t T, int64_t K,
                                           int* dev_status, int impl, hq_stream_t stream);

/*
 * The failure path of the tensor-core SYRK's bounded waits, made to run on purpose (no
 * counterpart on the pages; the library's rule that a device-side wait never hangs).  The
 * tcgen05 SYRK of hq_hessian_accumulate on bf16 X with
 *   wait_limit_cycles : 1000 .. 4e9, the SM cycles any pipeline wait may take before the CTA
 *                       records HQ_ERR_TIMEOUT in *dev_status, stops issuing, waits for the copies
 *                       and tensor-core work it already issued, frees its tensor memory and returns;
 *   withhold_stage    : -1 (an ordinary call), or 0 .. 3: the MMA issuer never releases that
 *                       stage of the 4-stage operand ring after its first use, so the producer's
 *                       wait to refill it expires (when X has more than 4 x 64 tokens) before it
 *                       issues another load.  The stream and context stay usable; H is then
 *                       partly or not updated.
 *   dev_status : device int, required (zeroed by the caller).  X bf16 [T, K], K % 8 == 0, 16-byte
 *                aligned (the tensor-core path), else HQ_ERR_UNSUPPORTED.  Asynchronous.
 */
hq_status hq_debug_hessian_accumulate_timeout(float* H, const void* X, int64_t T, int64_t K, int* dev_status,
                                              int64_t wait_limit_cycles, int withhold_stage, hq_stream_t stream);

/*
 * The GPTQ lazy-update product (persistent tcgen05 kernel, 3xTF32 from pre-split operands):
 *   C[m, n] -= sum_k (A_hi + A_lo)[m * lda + k] (B_hi + B_lo)[n * ldb + k]   (hi*lo + lo*hi +
 *   hi*hi; lo*lo dropped), m < M, n < N.  All pointers 16-byte aligned, lda, ldb, ldc multiples
 * of 4.  No counterpart on the pages: a building block of the path.
 */
hq_status hq_debug_upd_gemm(float* C, int64_t ldc, int M, int N, int Kred, const float* A_hi, const float* A_lo,
                            int64_t lda, const float* B_hi, const float* B_lo, int64_t ldb, hq_stream_t stream);

/*
 * The fp64 GEMM of the factorisation (fp64 tensor cores, mma.sync m8n8k4):
 *   C[m, n] = beta * C[m, n] + alpha * sum_k A[m * lda + k] * B[n * ldb + k]
 * for m < M, n < N (if `lower`, M == N and only elements with m >= n are written).
 * tri declares a triangular operand whose zeros the kernel skips (the result is the same
 * when the operand really is zero there): 0 none, 1 A upper (A[m][k] = 0 for k < m),
 * 2 A lower (A[m][k] = 0 for k > m), 3 B lower (B[n][k] = 0 for k > n).
 * Kred a multiple of 16; A, B 16-byte aligned, lda and ldb even.  `scratch` (scratch_elems doubles, may be
 * NULL) lets the kernel split the contraction when the problem has few output tiles; the
 * partial sums are added in a fixed order, so results are identical run to run.
 * No counterpart on the pages: a building block of the path.
 */
hq_status hq_debug_f64_gemm(double* C, int64_t ldc, int M, int N, int Kred, const double* A, int64_t lda,
                            const double* B, int64_t ldb, double alpha, double beta, int lower, int tri,
                            double* scratch, int64_t scratch_elems, hq_stream_t stream);

/*
 * The same product as hq_debug_f64_gemm, fp64-accurate on the int8 tensor cores: every operand
 * row scaled by a power of two and cut into 7 signed 7-bit int8 slices (exact in fp64), the 28
 * slice-pair products of anti-diagonals 0..6 accumulated exactly in int32 by tcgen05 kind::i8
 * MMAs, recombined in fp64 (error-free slicing after Ozaki, Ogita, Oishi & Rump; no counterpart
 * on the pages: a building block of the factorisation).  Relative error about 1e-14 of the
 * product of the operands' row maxima per term.  `tri` as for hq_debug_f64_gemm, at 128-row
 * granularity: the slices read only the 128-aligned band of each row where the declared
 * triangular operand can be non-zero (entries outside it are never read, whatever they hold).
 * Rows holding a NaN or an infinity give NaN products.  Kred <= 16384 (the int32 sums stay
 * exact).  `scratch`: device, 256-byte aligned, hq_debug_i8x_scratch_bytes(M, N, Kred) bytes
 * (the slices and the row exponents).  A, B 8-byte aligned.  C is not read when beta == 0.
 */
size_t hq_debug_i8x_scratch_bytes(int M, int N, int Kred);
hq_status hq_debug_i8x_gemm(double* C, int64_t ldc, int M, int N, int Kred, const double* A, int64_t lda,
                            const double* B, int64_t ldb, double alpha, double beta, int lower, int tri, void* scratch,
                            size_t scratch_bytes, hq_stream_t stream);

/*
 * out[i] = 1 / d[i] (fp64) by the reciprocal the factorisation's leaf kernel uses for its pivots
 * (hardware approximation refined by two Newton-Raphson steps), for d[i] positive, normal and
 * finite (other inputs give unspecified values).  n >= 0.  No counterpart on the pages.
 */
hq_status hq_debug_rcp_f64(const double* d, double* out, int64_t n, hq_stream_t stream);

/*
 * Event timing of kernel classes, for profiling from the caller's side.  While a class's bit
 * is set in class_mask, every launch of that class records a CUDA event pair on its own
 * stream, with the launch's algorithmic work: 0 = fp64 GEMM, 128-wide tiles (flops);
 * 1 = fp64 GEMM, 64-wide tiles, including its split-K reduction (flops); 2 = factorisation
 * leaf (flops of a 128 x 128 Cholesky and triangular inverse); 3 = GPTQ block sweep (bytes);
 * 4 = tf32 lazy-update GEMM (flops of the product); 5 = tcgen05 SYRK (flops); 6 = int8-sliced
 * fp64 GEMM product kernel (flops of the fp64 product it computes, triangular operands counted
 * once); 7 = its slicing kernels (bytes: fp64 operands read, int8 slices written).
 * hq_debug_timing_start clears the records and sets the mask; hq_debug_timing_read
 * synchronises the recorded events and returns the sum of durations (ms), of work and the
 * number of launches of one class; hq_debug_timing_stop clears the mask.  Events are created
 * on first use and kept.  One process-wide record: not for concurrent use.
 * hq_debug_timing_serialize(1): from then on (until hq_debug_timing_serialize(0)) the
 * factorisation runs its off-critical-path products on the caller's stream instead of a second
 * stream, so that every recorded duration covers its own launch alone (shares then compare with
 * a serialised profiler launch list); results are unchanged.  Off by default.  No counterpart
 * on the pages.
 */
hq_status hq_debug_timing_start(int class_mask);
hq_status hq_debug_timing_serialize(int on);
hq_status hq_debug_timing_stop(void);
hq_status hq_debug_timing_read(int kernel_class, double* ms_total, double* work_total, int64_t* launches);

/*
 * fp64 MMA (mma.sync m8n8k4 .f64) rate in TFLOP/s of a kernel that does nothing else (8
 * independent accumulators per warp, two CTAs of 256 threads per SM), timed with CUDA events
 * on `stream`; synchronises it.  `scratch`: device buffer of at least 296 * 256 * 8 bytes.
 * Returns a negative value on failure.  Context for the fp64 GEMM's roofline; no counterpart
 * on the pages.
 */
double hq_debug_fp64_mma_rate(void* scratch, int64_t scratch_bytes, hq_stream_t stream);

/* Number of kernels libhq.so has launched in this process so far (all devices, all
 * threads).  A statistic for profiling; never reset. */
uint64_t hq_debug_launch_count(void);

/*
 * The bounds-checking build.  libhq_bounds.so is the same library compiled with HQ_DEBUG_BOUNDS:
 * the kernels check their computed global indices against the extents they were given, and the
 * first failing check (a tag of the source file's name in bits 16-30, the source line in bits
 * 0-15) is recorded in a device word while the access it guards is skipped.  It stands in for a
 * memory checker on machines where none can run.  No counterpart on the pages.
 *
 * hq_debug_bounds_status: *enabled = 1 in the bounds-checking build (0 in libhq.so, where
 *   *violation is always 0); *violation = the recorded failure, 0 if none; the word is then
 *   cleared.  Synchronises the current device (a blocking copy from a device symbol).
 * hq_debug_bounds_selftest: launches one check that fails by construction (an index equal to
 *   the range's length; nothing is accessed), so that the next hq_debug_bounds_status reports
 *   it.  HQ_ERR_UNSUPPORTED in libhq.so, which launches nothing.
 */
hq_status hq_debug_bounds_status(int* enabled, int* violation);
hq_status hq_debug_bounds_selftest(hq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* HQ_DEBUG_H */
