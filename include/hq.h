/*
 * hq.h -- C ABI of libhq.so: Hessian-aware int4 weight quantisation (GPTQ) of one linear
 * layer on an NVIDIA B200 (sm_100a), and the Bf16TrilDiagF32 Hessian codec.
 *
 * Sources of the operations (page title, section):
 *   [calib] "hipfire-calib-data" dataset card -- "Hessian storage: Bf16TrilDiagF32
 *           (quant_type 130)"; "REQUIRED: project to PSD before Cholesky"; "The fix".
 *   [gptq]  ork-driver wiki "Exp 2026-08-18 GPTQ Int4" -- experiment summary (GPTQ sweep,
 *           Cholesky-based Hessian inverse, uniform symmetric int4 [-8,7] with a
 *           per-(row,group) scale, dequant w = code*scale), the qerr definition, the
 *           test_offline_load notes (optional qerr output, byte-identical codes).
 *   [imat]  AtomicChat Qwen3.8-27B GGUF card -- "The importance matrix" (statistics are
 *           sums over chunks; importance = mean squared activation per channel).
 *
 * Conventions for every entry point:
 *   - Array pointers are DEVICE pointers owned by the caller unless a parameter says
 *     "host".  The library allocates no memory; a caller that runs calls concurrently gives
 *     each its own workspace.  (hq_rtn_quantize_noalloc instead uses one fixed scratch array
 *     that is part of the library's device image.)
 *   - Matrices are row-major and densely packed (leading dimension = column count).
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is enqueued on it.
 *   - Invalid arguments are refused with HQ_ERR_INVALID (or HQ_ERR_UNSUPPORTED for a
 *     well-formed shape this build does not handle) BEFORE anything is launched; nothing
 *     is ever silently substituted.  On any error the contents of outputs are undefined.
 *   - All kernels run on the device that is current when the call is made.
 */
#ifndef HQ_H
#define HQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void* hq_stream_t; /* a cudaStream_t */

typedef enum {
  HQ_OK = 0,
  HQ_ERR_INVALID = 1,     /* bad pointer, size, dtype or parameter value */
  HQ_ERR_UNSUPPORTED = 2, /* a shape this build refuses (e.g. K not a multiple of 128) */
  HQ_ERR_NOT_PD = 3,      /* damped Hessian not positive definite (Cholesky pivot <= 0) */
  HQ_ERR_TIMEOUT = 4,     /* a bounded device-side wait expired; outputs undefined */
  HQ_ERR_CUDA = 5,        /* a CUDA runtime call or kernel launch failed */
  HQ_ERR_WORKSPACE = 6    /* workspace NULL, misaligned (256 B) or smaller than required */
} hq_status;

typedef enum { HQ_F32 = 0, HQ_BF16 = 1 } hq_dtype;

/* Human-readable name of a status code (static storage). */
const char* hq_status_string(int status);

/* ABI version of this header (incremented on any incompatible change). */
int hq_abi_version(void);

/*
 * H += X^T X  -- calibration Hessian accumulation ([calib] "Hessian storage": full
 * Hessians XX^T with X laid out [channels, tokens]; [imat]: the statistic is a sum over
 * chunks, so a corpus is fed chunk by chunk into the same H).
 *   H      : fp32 [K, K], read-modify-write of the LOWER triangle including the diagonal
 *            (element (i, j), i >= j).  The strict upper triangle is never read or written.
 *   X      : [T, K] tokens x channels, dtype x_dtype (HQ_BF16 or HQ_F32).  Products are
 *            exact (bf16*bf16 or fp32*fp32) and accumulated in fp32.
 *   T >= 0 (T == 0 is a no-op), K >= 1.
 *   dev_status : optional device int; if non-NULL a kernel that hits a bounded-wait timeout
 *            stores HQ_ERR_TIMEOUT there (the caller zeroes it beforehand).
 * Asynchronous: returns after enqueueing.  H must not alias X.  Repeated calls give the same
 * bits, except that on the tensor-core path a call whose tiles leave a short last round (at most
 * half of the GPU's 148 SMs) splits those tiles by tokens, and their entries then receive
 * partial sums in a run-dependent order (differences of the last bit of fp32).
 */
hq_status hq_hessian_accumulate(float* H, const void* X, int x_dtype, int64_t T, int64_t K,
                                int* dev_status, hq_stream_t stream);

/*
 * imp[k] = H[k, k] / tokens  -- importance vector = mean squared activation per channel
 * ([gptq] qerr paragraph: diag(H)[k] = sum_t a_k^2, the imatrix is its mean).
 *   H fp32 [K, K] (diagonal read), imp fp32 [K] out.  tokens >= 1.  Asynchronous.
 */
hq_status hq_imatrix(const float* H, int64_t K, int64_t tokens, float* imp, hq_stream_t stream);

/* Bytes of workspace hq_gptq_quantize needs for this shape (0 if the shape is invalid). */
size_t hq_gptq_workspace_bytes(int64_t N, int64_t K, int64_t group);

/*
 * GPTQ int4 quantisation of one layer ([gptq] experiment summary):
 *   lambda = damp * mean(diag H); U = upper Cholesky factor of (H + lambda I)^-1;
 *   columns j = 0..K-1 in order, for every row n:
 *     at a group start: s = fp32(max |Wc[n, j:j+group]| / 7) from the current weights;
 *     c = clamp(rint(Wc[n,j] / s), -8, 7) (s == 0 -> c = 0); q = c * s;
 *     e = (Wc[n,j] - q) / U[j,j];  Wc[n,k] -= e * U[j,k] for k > j.
 *   qerr = sqrt(sum imp[k] (W[n,k] - q[n,k])^2 / sum imp[k] W[n,k]^2) over the ORIGINAL W,
 *   imp = 1 when NULL ([gptq] qerr definition).
 * Arguments:
 *   W      : [N, K] row-major, dtype w_dtype (HQ_BF16 or HQ_F32); not modified.
 *   H      : fp32 [K, K] undamped Hessian; only the lower triangle incl. diagonal is read;
 *            not modified.
 *   group  : group size along K; must divide K and be a multiple of 32.
 *   K      : a multiple of 128.  N >= 1.
 *   damp   : > 0 and finite; mean(diag H) must be > 0.
 *   imp    : optional fp32 [K] importance (NULL -> all ones); only affects qerr.
 *   codes  : uint8 [N, K/2] out; byte (n, p) = (c[n,2p] & 0xF) | (c[n,2p+1] & 0xF) << 4,
 *            4-bit two's complement (the even column in the low nibble).
 *   scales : fp32 [N, K/group] out, row-major.
 *   qerr_out : optional HOST double* (NULL -> not returned).
 *   qerr_dev : optional DEVICE double* (NULL -> not written); written asynchronously.
 *   workspace : device buffer of at least hq_gptq_workspace_bytes(N, K, group) bytes,
 *            256-byte aligned, owned by the caller, not shared with a concurrent call.
 * The call synchronises `stream` once at its end to read the factorisation status, and
 * returns HQ_ERR_NOT_PD if a Cholesky pivot was not positive.  Part of the factorisation runs
 * on a second stream that the library creates once per host thread and device (with a few
 * events, kept for the thread's lifetime); it is joined back into `stream` before the call's
 * later work, so ordering on `stream` is as if everything ran there.  codes and scales do not
 * depend on whether qerr is requested, and are identical run to run.
 * Non-finite inputs: a NaN or infinite weight affects only its own row's codes and scales
 * (rows are independent) and makes qerr non-finite; a non-finite mean(diag H) is refused as
 * HQ_ERR_INVALID after the damping stage; any other NaN or infinity in H's lower triangle
 * reaches a Cholesky pivot and is reported as HQ_ERR_NOT_PD.
 */
hq_status hq_gptq_quantize(const void* W, int w_dtype, int64_t N, int64_t K, const float* H,
                           int64_t group, float damp, const float* imp, uint8_t* codes,
                           float* scales, double* qerr_out, double* qerr_dev, void* workspace,
                           size_t workspace_bytes, hq_stream_t stream);

/*
 * hq_gptq_quantize in two stages, for a layer whose rows are quantised on several devices
 * against one factorisation: given U, the sweep's feedback stays inside each row ([gptq]
 * experiment summary: the error-feedback sweep runs row by row over the columns), so one device
 * factorises, the factor buffer is broadcast (it is plain bytes), and every device sweeps its own
 * rows.  hq_gptq_factorize + hq_gptq_sweep give the same codes, scales and qerr as
 * hq_gptq_quantize on the same rows.
 *
 * hq_gptq_factor_bytes(K): size of the factor buffer: a small header (factorisation status and
 *   lambda), the 128 x 128 diagonal blocks of U' = diag(U)^-1 U in the sweep's packed order, the
 *   384 columns of U' right of each diagonal block (the in-panel updates), and the strict lower
 *   triangle of U'^T split into a tf32 part and its fp32 remainder (about 8 K^2 bytes).  0 for an unsupported K (K a multiple of 128, at most 65536).
 * hq_gptq_factor_workspace_bytes(K): scratch of hq_gptq_factorize (the fp64 factorisation).
 * hq_gptq_sweep_workspace_bytes(N, K, group): scratch of hq_gptq_sweep (no fp64 matrices).
 *
 * hq_gptq_factorize: lambda = damp * mean(diag H), U'^T of (H + lambda I)^-1 into `factor`
 *   (device, 256-byte aligned, at least hq_gptq_factor_bytes(K) bytes; HQ_ERR_INVALID otherwise).
 *   H, damp, K as for hq_gptq_quantize.  Synchronises `stream` and returns HQ_ERR_NOT_PD or
 *   HQ_ERR_INVALID like hq_gptq_quantize; the factor's header then records the failure, so a
 *   buffer broadcast after a failed factorisation makes every hq_gptq_sweep on it return the
 *   same status.
 * hq_gptq_sweep: the sweep of W [N, K] against a factor buffer (device, 256-byte aligned, read
 *   only, made by hq_gptq_factorize for the same K); W, group, imp, codes, scales, qerr_out,
 *   qerr_dev as for hq_gptq_quantize; workspace at least hq_gptq_sweep_workspace_bytes(N, K,
 *   group).  Synchronises `stream` once at the end; HQ_ERR_NOT_PD / HQ_ERR_INVALID when the
 *   factor records a failed factorisation.  hq_qerr_terms reads this workspace too.
 */
size_t hq_gptq_factor_bytes(int64_t K);
size_t hq_gptq_factor_workspace_bytes(int64_t K);
size_t hq_gptq_sweep_workspace_bytes(int64_t N, int64_t K, int64_t group);
hq_status hq_gptq_factorize(const float* H, int64_t K, float damp, void* factor, size_t factor_bytes,
                            void* workspace, size_t workspace_bytes, hq_stream_t stream);
hq_status hq_gptq_sweep(const void* W, int w_dtype, int64_t N, int64_t K, const void* factor,
                        int64_t group, const float* imp, uint8_t* codes, float* scales,
                        double* qerr_out, double* qerr_dev, void* workspace, size_t workspace_bytes,
                        hq_stream_t stream);

/*
 * The two fp64 sums behind the qerr of the last hq_gptq_quantize or hq_rtn_quantize that ran
 * with this workspace ([gptq] qerr definition): terms_dev[0] = sum imp[k] (W[n,k] - q[n,k])^2,
 * terms_dev[1] = sum imp[k] W[n,k]^2, so that qerr = sqrt(terms[0] / terms[1]).  For callers that
 * split a layer's rows over several calls or devices: the sums of the parts add up (in any
 * order, up to fp64 rounding) to the whole layer's.
 *   workspace : the workspace of that call (device, 256-byte aligned), read only.
 *   terms_dev : DEVICE double[2] out, written asynchronously on `stream` after the call's work
 *               when enqueued on the same stream.
 * Returns HQ_ERR_INVALID for NULL pointers; nothing else is checked (the workspace must hold a
 * finished call's results).
 */
hq_status hq_qerr_terms(const void* workspace, double* terms_dev, hq_stream_t stream);

/*
 * qerr from its two sums ([gptq] qerr definition): *qerr_dev = sqrt(terms_dev[0] / terms_dev[1]),
 * 0 when terms_dev[1] == 0 (an all-zero layer); non-finite sums give a non-finite qerr.  For
 * callers that added the sums of a layer's row shards (e.g. by an all-reduce).  Device pointers;
 * asynchronous.
 */
hq_status hq_qerr_from_terms(const double* terms_dev, double* qerr_dev, hq_stream_t stream);

/* Bytes of workspace hq_rtn_quantize needs (0 if the shape is invalid). */
size_t hq_rtn_workspace_bytes(int64_t N, int64_t K, int64_t group);

/*
 * Round-to-nearest int4 with the same quantiser and no error feedback, the RTN baseline of
 * symmetric absmax/7 rounding ([gptq] experiment summary): s = fp32(max|W[n,group]|/7),
 * c = clamp(rint(W/s), -8, 7).  Same argument meanings and output layouts as
 * hq_gptq_quantize.  Synchronises `stream` only when qerr_out != NULL.
 */
hq_status hq_rtn_quantize(const void* W, int w_dtype, int64_t N, int64_t K, int64_t group,
                          const float* imp, uint8_t* codes, float* scales, double* qerr_out,
                          double* qerr_dev, void* workspace, size_t workspace_bytes,
                          hq_stream_t stream);

/*
 * hq_rtn_quantize without a workspace, for callers that cannot hand the library scratch memory
 * when they quantise: an application that has already reserved all device memory for its own
 * pool, a service that forbids allocation after start-up, a plugin living under another
 * framework's allocator.  The pages have no counterpart to this entry point; it is a deployment
 * convenience.  Same arguments, results and output layouts as hq_rtn_quantize, minus
 * `workspace` / `workspace_bytes`.
 *   - Scratch (qerr partial sums, status) lives in one fixed array in the library's device
 *     memory: HQ_RTN_NOALLOC_MAX_GROUPS * 16 + 256 bytes (16 MiB + 256 B), held on every GPU
 *     where the library's module holding it has been loaded, until the process exits.
 *     N * (K / group) above HQ_RTN_NOALLOC_MAX_GROUPS is refused with HQ_ERR_UNSUPPORTED
 *     before any launch; exactly HQ_RTN_NOALLOC_MAX_GROUPS groups are accepted.
 *   - The call allocates nothing itself (no cudaMalloc, no allocating library routine).  The
 *     array is committed when that module is loaded on a device; under CUDA's lazy module
 *     loading (the default, CUDA_MODULE_LOADING=LAZY) that is the first call on the device,
 *     which can therefore fail with HQ_ERR_CUDA if the device has no free memory left.  A caller
 *     that must not allocate later makes one warm-up call on each device before it reserves its
 *     memory pool or starts a stream capture; later calls commit nothing new.
 *   - The first call on a device (and the first after the current context changes, e.g. after
 *     a device reset) looks up the array's device address (cudaGetSymbolAddress) with that
 *     device current, and caches it per device and context.
 *   - Every call on a device shares the one array and it keeps the last call's contents; each
 *     call re-initialises what it needs.  Calls whose GPU work overlaps (different streams,
 *     different host threads) race on it: serialise them.
 */
#define HQ_RTN_NOALLOC_MAX_GROUPS 1048576
hq_status hq_rtn_quantize_noalloc(const void* W, int w_dtype, int64_t N, int64_t K, int64_t group,
                                  const float* imp, uint8_t* codes, float* scales, double* qerr_out,
                                  double* qerr_dev, hq_stream_t stream);

/* Bytes of workspace hq_hessian_project_psd needs (0 if K is unsupported). */
size_t hq_psd_workspace_bytes(int64_t K);

/*
 * H <- its projection onto the positive semidefinite cone ([calib] "REQUIRED: project to PSD
 * before Cholesky", "The fix"): the matrix that eigendecomposing H = V diag(l) V^T, clipping the
 * negative eigenvalues to zero, rebuilding and symmetrising gives.  Computed without an
 * eigendecomposition as (H + H sign(H)) / 2, sign(H) from `steps` Newton-Schulz steps
 * X <- X (3I - X^2) / 2 on the tensor cores started at H / ||H||_F, then (P + P^T) / 2.  fp32
 * iterates, 3xTF32 products.  An eigenvalue below about 1.5^-steps ||H||_F in magnitude is not
 * resolved and moves the result by at most its size; 40 steps resolve 1e-7 ||H||_F.  Cost:
 * 4 (steps + 1/2) K^3 flops.
 *   H         : fp32 [K, K] device, both triangles (e.g. from hq_hessian_unpack_bf16tril),
 *               symmetric; overwritten.  16-byte aligned, K a multiple of 4, K <= 65536.
 *   steps     : 0 .. 1000 (0 gives (H + H H / ||H||_F) / 2 symmetrised: no projection).
 *   workspace : device, 256-byte aligned, at least hq_psd_workspace_bytes(K) bytes.
 * Synchronises `stream` at the end (HQ_ERR_TIMEOUT if a bounded wait in a product expired).
 */
hq_status hq_hessian_project_psd(float* H, int64_t K, int steps, void* workspace, size_t workspace_bytes,
                                 hq_stream_t stream);

/*
 * Hadamard rotation ahead of GPTQ ([gptq] experiment summary: GPTQ composes with Hadamard,
 * "rotate then GPTQ").  R = diag(signs) blockdiag(M, ..., M), M = Hadamard_block / sqrt(block)
 * the orthonormal Walsh-Hadamard matrix (Sylvester: M[i][j] = (-1)^popcount(i & j) / sqrt(block)).
 * R is orthogonal: quantising W' = W R against H' = R^T H R (the Hessian of the rotated
 * activations X R) and feeding the layer R^T x leaves its output unchanged.
 *   block : a power of two, 2 .. 1024, dividing K.
 *   signs : device fp32 [K] of +1 / -1, drawn by the caller (the method's random signs).
 * hq_hadamard_rotate_weights: W_out (fp32 [N, K], may equal W when W is fp32) = W R; W bf16 or
 *   fp32 [N, K].
 * hq_hadamard_rotate_hessian: H_out (fp32 [K, K], both triangles, distinct from H) = R^T H R,
 *   H read as the symmetric matrix of its lower triangle (diagonal included); H unchanged.
 * Asynchronous.  HQ_ERR_UNSUPPORTED for a block that is not a power of two dividing K.
 * Any alignment is accepted; blocks of 32 and more with 16-byte aligned W, W_out / H_out and
 * signs take the warp-level kernels (one read and one write of W; two passes over H's lower
 * blocks), other cases simpler shared-memory kernels with the same results up to rounding order.
 */
hq_status hq_hadamard_rotate_weights(const void* W, int w_dtype, int64_t N, int64_t K, int64_t block,
                                     const float* signs, float* W_out, hq_stream_t stream);
hq_status hq_hadamard_rotate_hessian(const float* H, int64_t K, int64_t block, const float* signs, float* H_out,
                                     hq_stream_t stream);

/*
 * The lower triangle of an fp32 Hessian packed row by row without gaps, element (i, j), j <= i,
 * at i (i + 1) / 2 + j: hq_tril32_count(K) = K (K + 1) / 2 values.  The exchange format of a
 * Hessian accumulated over token chunks on several devices ([calib] "Hessian storage": H is a
 * sum over chunks; [imat]: partial statistics merge by addition): the packed partial sums are
 * added (an all-reduce) and unpacked, moving about half the bytes of the full matrix.  Exact
 * copies.
 * hq_hessian_pack_lower: H fp32 [K, K] (lower triangle incl. diagonal read) -> packed.
 * hq_hessian_unpack_lower: packed -> H's lower triangle incl. diagonal (the strict upper
 *   triangle is not written).  Device pointers, K >= 1, asynchronous.
 */
size_t hq_tril32_count(int64_t K);
hq_status hq_hessian_pack_lower(const float* H, int64_t K, float* packed, hq_stream_t stream);
hq_status hq_hessian_unpack_lower(const float* packed, int64_t K, float* H, hq_stream_t stream);

/* Bf16TrilDiagF32 payload size: K*4 + K*(K-1)/2*2 bytes ([calib] "Hessian storage"). */
size_t hq_bf16tril_bytes(int64_t K);

/*
 * Bf16TrilDiagF32 encode ([calib] "Hessian storage: Bf16TrilDiagF32 (quant_type 130)"):
 *   out[0 : 4K)            = H[i,i] as little-endian fp32, i = 0..K-1;
 *   out[4K + 2*(i(i-1)/2 + j)] = (fp32 bits of H[i,j]) >> 16 as little-endian u16, i > j
 *                            (bf16 by truncation, not rounding).
 *   H fp32 [K, K] (diagonal and strict lower triangle read), out hq_bf16tril_bytes(K) bytes.
 *   K >= 1.  Asynchronous.  Bit-exact by definition.  K % 4 == 0, K <= 46340 and 16-byte
 *   aligned H and out take the one-pass vector kernel; other cases a per-row kernel (same bytes).
 */
hq_status hq_hessian_pack_bf16tril(const float* H, int64_t K, uint8_t* out, hq_stream_t stream);

/*
 * Bf16TrilDiagF32 decode, "mirrored on read": H[i,i] = diagonal; H[i,j] = H[j,i] =
 * fp32(bits << 16) for i > j.  in: hq_bf16tril_bytes(K) bytes; H_full fp32 [K, K] out (both
 * triangles written).  K >= 1.  Asynchronous.  K % 4 == 0, K <= 46340, 16-byte aligned H_full
 * and 8-byte aligned in take the word-gather kernel; other cases a scalar-gather kernel (same
 * values).
 */
hq_status hq_hessian_unpack_bf16tril(const uint8_t* in, int64_t K, float* H_full,
                                     hq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* HQ_H */
