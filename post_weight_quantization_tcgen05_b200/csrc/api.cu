// The C ABI of libhq.so (include/hq.h, include/hq_debug.h): argument validation, workspace
// carving and stage orchestration.  Every computation happens in the kernels of the other
// translation units; this file only checks arguments and enqueues work.
#include <math.h>
#include <string.h>

#include "../../include/hq.h"
#include "../../include/hq_debug.h"
#include "common.cuh"
#include "kernels.cuh"

namespace hq {
uint64_t& launch_counter() {
  static uint64_t n = 0;
  return n;
}
}  // namespace hq

using namespace hq;

namespace {

constexpr int kAbiVersion = 1;

bool valid_dtype(int d) { return d == HQ_F32 || d == HQ_BF16; }

hq_status finish_sync(cudaStream_t s, const WsHeader* dev_hdr, double* qerr_out) {
  WsHeader h{};
  HQ_CUDA_TRY(cudaMemcpyAsync(&h, dev_hdr, sizeof(WsHeader), cudaMemcpyDeviceToHost, s));
  HQ_CUDA_TRY(cudaStreamSynchronize(s));
  if (h.status == HQ_ERR_TIMEOUT) return HQ_ERR_TIMEOUT;
  if (h.info == -1) return HQ_ERR_INVALID;
  if (h.info > 0) return HQ_ERR_NOT_PD;
  if (qerr_out != nullptr) *qerr_out = h.qerr;
  return HQ_OK;
}

hq_status check_gptq_args(const void* W, int w_dtype, int64_t N, int64_t K, const float* H, int64_t group, float damp,
                          uint8_t* codes, float* scales) {
  if (W == nullptr || H == nullptr || codes == nullptr || scales == nullptr) return HQ_ERR_INVALID;
  if (!valid_dtype(w_dtype)) return HQ_ERR_INVALID;
  if (N < 1 || K < 1 || group < 1) return HQ_ERR_INVALID;
  if (!(damp > 0.f) || !isfinite(damp)) return HQ_ERR_INVALID;
  if (K % group != 0) return HQ_ERR_INVALID;
  if (!gptq_shape_ok(N, K, group)) return HQ_ERR_UNSUPPORTED;
  return HQ_OK;
}

hq_status gptq_common(const void* W, int w_dtype, int64_t N, int64_t K, const float* H, int64_t group, float damp,
                      const float* imp, uint8_t* codes, float* scales, double* qerr_out, double* qerr_dev,
                      void* workspace, size_t workspace_bytes, int update_impl, cudaStream_t s) {
  hq_status st = check_gptq_args(W, w_dtype, N, K, H, group, damp, codes, scales);
  if (st != HQ_OK) return st;
  const GptqLayout L = gptq_layout(N, K, group);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < L.total) return HQ_ERR_WORKSPACE;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  st = launch_gptq(W, w_dtype, N, K, H, group, damp, imp, codes, scales, qerr_dev, ws, update_impl, s);
  if (st != HQ_OK) return st;
  return finish_sync(s, reinterpret_cast<const WsHeader*>(ws + L.header), qerr_out);
}

// qerr = sqrt(num / den) from the two sums, 0 for an all-zero layer (the qerr finaliser's rule).
__global__ void qerr_from_terms_kernel(const double* __restrict__ terms, double* __restrict__ q) {
  const double num = terms[0], den = terms[1];
  *q = den == 0.0 ? 0.0 : sqrt(num / den);
}

// Both the GPTQ and the RTN workspace start with the status header (layout offset 0).
__global__ void qerr_terms_kernel(const WsHeader* __restrict__ hdr, double* __restrict__ out) {
  out[0] = hdr->num;
  out[1] = hdr->den;
}

}  // namespace

#ifdef HQ_DEBUG_BOUNDS
namespace hq {
__device__ int g_hq_bounds_violation = 0;

// One check that fails by construction (index n of an n-element range); nothing is accessed.
__global__ void bounds_selftest_kernel(int n) {
  const int idx = n;
  if (HQ_IN_BOUNDS(idx < n)) return;
}
}  // namespace hq
#endif

extern "C" {

const char* hq_status_string(int status) {
  switch (status) {
    case HQ_OK: return "HQ_OK";
    case HQ_ERR_INVALID: return "HQ_ERR_INVALID";
    case HQ_ERR_UNSUPPORTED: return "HQ_ERR_UNSUPPORTED";
    case HQ_ERR_NOT_PD: return "HQ_ERR_NOT_PD";
    case HQ_ERR_TIMEOUT: return "HQ_ERR_TIMEOUT";
    case HQ_ERR_CUDA: return "HQ_ERR_CUDA";
    case HQ_ERR_WORKSPACE: return "HQ_ERR_WORKSPACE";
    default: return "HQ_ERR_UNKNOWN";
  }
}

int hq_abi_version(void) { return kAbiVersion; }

uint64_t hq_debug_launch_count(void) { return __atomic_load_n(&launch_counter(), __ATOMIC_RELAXED); }

hq_status hq_debug_bounds_status(int* enabled, int* violation) {
  if (enabled == nullptr || violation == nullptr) return HQ_ERR_INVALID;
#ifdef HQ_DEBUG_BOUNDS
  int v = 0;
  HQ_CUDA_TRY(cudaMemcpyFromSymbol(&v, g_hq_bounds_violation, sizeof(int)));
  const int zero = 0;
  HQ_CUDA_TRY(cudaMemcpyToSymbol(g_hq_bounds_violation, &zero, sizeof(int)));
  *enabled = 1;
  *violation = v;
#else
  *enabled = 0;
  *violation = 0;
#endif
  return HQ_OK;
}

hq_status hq_debug_bounds_selftest(hq_stream_t stream) {
#ifdef HQ_DEBUG_BOUNDS
  bounds_selftest_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(4);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
#else
  (void)stream;
  return HQ_ERR_UNSUPPORTED;
#endif
}

hq_status hq_debug_hessian_accumulate_impl(float* H, const void* X, int x_dtype, int64_t T, int64_t K,
                                           int* dev_status, int impl, hq_stream_t stream) {
  if (H == nullptr || K < 1 || T < 0 || !valid_dtype(x_dtype) || (impl != 0 && impl != 1)) return HQ_ERR_INVALID;
  if (T > 0 && X == nullptr) return HQ_ERR_INVALID;
  if (T == 0) return HQ_OK;
  if (K > (int64_t(1) << 20) || T > 0x7FFFFFFF) return HQ_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (impl == 0 && syrk_tc_eligible(X, x_dtype, T, K)) return launch_syrk_tc(H, X, T, K, dev_status, s);
  return launch_syrk_simt(H, X, x_dtype, T, K, s);
}

hq_status hq_debug_hessian_accumulate_timeout(float* H, const void* X, int64_t T, int64_t K, int* dev_status,
                                              int64_t wait_limit_cycles, int withhold_stage, hq_stream_t stream) {
  if (H == nullptr || X == nullptr || dev_status == nullptr || K < 1 || T < 1) return HQ_ERR_INVALID;
  if (wait_limit_cycles < 1000 || wait_limit_cycles > kWaitLimitCycles || withhold_stage < -1 || withhold_stage > 3)
    return HQ_ERR_INVALID;
  if (!syrk_tc_eligible(X, HQ_BF16, T, K) || K > (int64_t(1) << 20) || T > 0x7FFFFFFF) return HQ_ERR_UNSUPPORTED;
  return launch_syrk_tc(H, X, T, K, dev_status, static_cast<cudaStream_t>(stream), wait_limit_cycles,
                        withhold_stage);
}

hq_status hq_hessian_accumulate(float* H, const void* X, int x_dtype, int64_t T, int64_t K, int* dev_status,
                                hq_stream_t stream) {
  return hq_debug_hessian_accumulate_impl(H, X, x_dtype, T, K, dev_status, 0, stream);
}

__global__ void imatrix_kernel(const float* __restrict__ H, int64_t K, double inv_tokens, float* __restrict__ imp) {
  for (int64_t k = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; k < K;
       k += static_cast<int64_t>(gridDim.x) * blockDim.x)
    imp[k] = static_cast<float>(static_cast<double>(H[k * K + k]) * inv_tokens);
}

hq_status hq_imatrix(const float* H, int64_t K, int64_t tokens, float* imp, hq_stream_t stream) {
  if (H == nullptr || imp == nullptr || K < 1 || tokens < 1) return HQ_ERR_INVALID;
  const int grid = static_cast<int>(ceil_div(K, 256) < 1024 ? ceil_div(K, 256) : 1024);
  imatrix_kernel<<<grid, 256, 0, static_cast<cudaStream_t>(stream)>>>(H, K, 1.0 / static_cast<double>(tokens), imp);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

size_t hq_gptq_workspace_bytes(int64_t N, int64_t K, int64_t group) {
  if (!gptq_shape_ok(N, K, group)) return 0;
  return gptq_layout(N, K, group).total;
}

hq_status hq_gptq_quantize(const void* W, int w_dtype, int64_t N, int64_t K, const float* H, int64_t group,
                           float damp, const float* imp, uint8_t* codes, float* scales, double* qerr_out,
                           double* qerr_dev, void* workspace, size_t workspace_bytes, hq_stream_t stream) {
  return gptq_common(W, w_dtype, N, K, H, group, damp, imp, codes, scales, qerr_out, qerr_dev, workspace,
                     workspace_bytes, 0, static_cast<cudaStream_t>(stream));
}

size_t hq_gptq_factor_bytes(int64_t K) {
  if (!gptq_shape_ok(1, K, 128)) return 0;
  return factor_layout(K).total;
}

size_t hq_gptq_factor_workspace_bytes(int64_t K) {
  if (!gptq_shape_ok(1, K, 128)) return 0;
  return factor_ws_layout(K).total;
}

size_t hq_gptq_sweep_workspace_bytes(int64_t N, int64_t K, int64_t group) {
  if (!gptq_shape_ok(N, K, group)) return 0;
  return gptq_layout(N, K, group).sweep_total;
}

hq_status hq_gptq_factorize(const float* H, int64_t K, float damp, void* factor, size_t factor_bytes, void* workspace,
                            size_t workspace_bytes, hq_stream_t stream) {
  if (H == nullptr || factor == nullptr) return HQ_ERR_INVALID;
  if (!(damp > 0.f) || !isfinite(damp)) return HQ_ERR_INVALID;
  if (!gptq_shape_ok(1, K, 128)) return HQ_ERR_UNSUPPORTED;
  if (!aligned(factor, 256) || factor_bytes < factor_layout(K).total) return HQ_ERR_INVALID;
  const GptqLayout L = factor_ws_layout(K);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < L.total) return HQ_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws + L.header);
  HQ_CUDA_TRY(cudaMemsetAsync(hdr, 0, sizeof(WsHeader), s));
  hq_status st = launch_factorize(H, K, damp, ws, L, static_cast<uint8_t*>(factor), false, s);
  if (st != HQ_OK) return st;
  return finish_sync(s, hdr, nullptr);
}

hq_status hq_gptq_sweep(const void* W, int w_dtype, int64_t N, int64_t K, const void* factor, int64_t group,
                        const float* imp, uint8_t* codes, float* scales, double* qerr_out, double* qerr_dev,
                        void* workspace, size_t workspace_bytes, hq_stream_t stream) {
  if (W == nullptr || factor == nullptr || codes == nullptr || scales == nullptr || !valid_dtype(w_dtype))
    return HQ_ERR_INVALID;
  if (N < 1 || K < 1 || group < 1 || K % group != 0) return HQ_ERR_INVALID;
  if (!gptq_shape_ok(N, K, group)) return HQ_ERR_UNSUPPORTED;
  if (!aligned(factor, 256)) return HQ_ERR_INVALID;
  const GptqLayout L = gptq_layout(N, K, group);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < L.sweep_total) return HQ_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  hq_status st = launch_sweep(W, w_dtype, N, K, group, imp, codes, scales, qerr_dev, ws,
                              static_cast<const uint8_t*>(factor), 0, true, s);
  if (st != HQ_OK) return st;
  return finish_sync(s, reinterpret_cast<const WsHeader*>(ws + L.header), qerr_out);
}

hq_status hq_qerr_from_terms(const double* terms_dev, double* qerr_dev, hq_stream_t stream) {
  if (terms_dev == nullptr || qerr_dev == nullptr) return HQ_ERR_INVALID;
  qerr_from_terms_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(terms_dev, qerr_dev);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

hq_status hq_debug_gptq_quantize_impl(const void* W, int w_dtype, int64_t N, int64_t K, const float* H,
                                      int64_t group, float damp, const float* imp, uint8_t* codes, float* scales,
                                      double* qerr_out, double* qerr_dev, void* workspace, size_t workspace_bytes,
                                      int update_impl, hq_stream_t stream) {
  if (update_impl < 0 || update_impl > 1) return HQ_ERR_INVALID;
  return gptq_common(W, w_dtype, N, K, H, group, damp, imp, codes, scales, qerr_out, qerr_dev, workspace,
                     workspace_bytes, update_impl, static_cast<cudaStream_t>(stream));
}

hq_status hq_debug_factor(const float* H, int64_t K, float damp, float* Ut_out, void* workspace,
                          size_t workspace_bytes, hq_stream_t stream) {
  if (H == nullptr || Ut_out == nullptr) return HQ_ERR_INVALID;
  if (!(damp > 0.f) || !isfinite(damp)) return HQ_ERR_INVALID;
  if (!gptq_shape_ok(1, K, 128)) return HQ_ERR_UNSUPPORTED;
  const GptqLayout L = factor_ws_layout(K);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < L.total) return HQ_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  WsHeader* hdr = reinterpret_cast<WsHeader*>(ws + L.header);
  HQ_CUDA_TRY(cudaMemsetAsync(hdr, 0, sizeof(WsHeader), s));
  hq_status st = launch_factor(H, K, damp, reinterpret_cast<double*>(ws + L.a), reinterpret_cast<double*>(ws + L.x),
                               reinterpret_cast<double*>(ws + L.xt), reinterpret_cast<double*>(ws + L.t), ws + L.slices,
                               &hdr->lam, &hdr->info, &hdr->status, false, Ut_out, nullptr, nullptr, nullptr, s);
  if (st != HQ_OK) return st;
  return finish_sync(s, hdr, nullptr);
}

hq_status hq_debug_rcp_f64(const double* d, double* out, int64_t n, hq_stream_t stream) {
  if (n < 0 || (n > 0 && (d == nullptr || out == nullptr))) return HQ_ERR_INVALID;
  return launch_rcp_nr(d, out, n, static_cast<cudaStream_t>(stream));
}

hq_status hq_debug_f64_gemm(double* C, int64_t ldc, int M, int N, int Kred, const double* A, int64_t lda,
                            const double* B, int64_t ldb, double alpha, double beta, int lower, int tri,
                            double* scratch, int64_t scratch_elems, hq_stream_t stream) {
  if (C == nullptr || A == nullptr || B == nullptr || M < 0 || N < 0 || Kred < 1) return HQ_ERR_INVALID;
  if (ldc < N || lda < Kred || ldb < Kred || tri < kTriNone || tri > kTriBLower || scratch_elems < 0)
    return HQ_ERR_INVALID;
  if (!aligned(A, 16) || !aligned(B, 16) || !aligned(C, 8) || lda % 2 != 0 || ldb % 2 != 0) return HQ_ERR_INVALID;
  if (Kred % 16 != 0 || (lower && M != N)) return HQ_ERR_UNSUPPORTED;
  F64Gemm g{};
  g.C = C;
  g.ldc = ldc;
  g.M = M;
  g.N = N;
  g.Kred = Kred;
  g.A = A;
  g.lda = lda;
  g.B = B;
  g.ldb = ldb;
  g.alpha = alpha;
  g.beta = beta;
  g.lower = lower ? 1 : 0;
  g.tri = tri;
  g.scratch = scratch;
  g.scratch_elems = scratch == nullptr ? 0 : scratch_elems;
  g.skip = nullptr;
  return f64_gemm(g, static_cast<cudaStream_t>(stream));
}

size_t hq_debug_i8x_scratch_bytes(int M, int N, int Kred) {
  if (M < 1 || N < 1 || Kred < 1) return 0;
  return i8x_scratch_bytes(M, N, Kred);
}

hq_status hq_debug_i8x_gemm(double* C, int64_t ldc, int M, int N, int Kred, const double* A, int64_t lda,
                            const double* B, int64_t ldb, double alpha, double beta, int lower, int tri, void* scratch,
                            size_t scratch_bytes, hq_stream_t stream) {
  if (C == nullptr || A == nullptr || B == nullptr || M < 0 || N < 0 || Kred < 1) return HQ_ERR_INVALID;
  if (ldc < N || lda < Kred || ldb < Kred || tri < kTriNone || tri > kTriBLower) return HQ_ERR_INVALID;
  if (lower && M != N) return HQ_ERR_UNSUPPORTED;
  if (Kred > kI8xMaxKred) return HQ_ERR_UNSUPPORTED;
  F64Gemm g{};
  g.C = C;
  g.ldc = ldc;
  g.M = M;
  g.N = N;
  g.Kred = Kred;
  g.A = A;
  g.lda = lda;
  g.B = B;
  g.ldb = ldb;
  g.alpha = alpha;
  g.beta = beta;
  g.lower = lower ? 1 : 0;
  g.tri = tri;
  return i8x_gemm(g, static_cast<uint8_t*>(scratch), scratch_bytes, static_cast<cudaStream_t>(stream));
}

hq_status hq_debug_upd_gemm(float* C, int64_t ldc, int M, int N, int Kred, const float* A_hi, const float* A_lo,
                            int64_t lda, const float* B_hi, const float* B_lo, int64_t ldb, hq_stream_t stream) {
  if (C == nullptr || A_hi == nullptr || A_lo == nullptr || B_hi == nullptr || B_lo == nullptr || M < 0 || N < 0 ||
      Kred < 1)
    return HQ_ERR_INVALID;
  if (ldc < N || lda < Kred || ldb < Kred) return HQ_ERR_INVALID;
  UpdGemm g{};
  g.C = C;
  g.ldc = ldc;
  g.M = M;
  g.N = N;
  g.Kred = Kred;
  g.A_hi = A_hi;
  g.A_lo = A_lo;
  g.lda = lda;
  g.B_hi = B_hi;
  g.B_lo = B_lo;
  g.ldb = ldb;
  return upd_gemm(g, static_cast<cudaStream_t>(stream));
}

size_t hq_rtn_workspace_bytes(int64_t N, int64_t K, int64_t group) {
  if (N < 1 || K < 2 || group < 2 || group % 2 != 0 || K % group != 0) return 0;
  return rtn_workspace(N, K, group);
}

hq_status hq_rtn_quantize(const void* W, int w_dtype, int64_t N, int64_t K, int64_t group, const float* imp,
                          uint8_t* codes, float* scales, double* qerr_out, double* qerr_dev, void* workspace,
                          size_t workspace_bytes, hq_stream_t stream) {
  if (W == nullptr || codes == nullptr || scales == nullptr || !valid_dtype(w_dtype)) return HQ_ERR_INVALID;
  if (N < 1 || K < 2 || group < 2 || K % group != 0) return HQ_ERR_INVALID;
  if (group % 2 != 0) return HQ_ERR_UNSUPPORTED;
  const size_t need = rtn_workspace(N, K, group);
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < need) return HQ_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  hq_status st = launch_rtn(W, w_dtype, N, K, group, imp, codes, scales, qerr_dev, ws, s);
  if (st != HQ_OK) return st;
  if (qerr_out == nullptr) return HQ_OK;
  return finish_sync(s, reinterpret_cast<const WsHeader*>(ws), qerr_out);
}

hq_status hq_qerr_terms(const void* workspace, double* terms_dev, hq_stream_t stream) {
  if (workspace == nullptr || terms_dev == nullptr) return HQ_ERR_INVALID;
  qerr_terms_kernel<<<1, 1, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<const WsHeader*>(workspace),
                                                                     terms_dev);
  HQ_LAUNCH_CHECK();
  return HQ_OK;
}

size_t hq_psd_workspace_bytes(int64_t K) {
  return (K >= 4 && K % 4 == 0 && K <= 65536) ? psd_workspace(K) : 0;
}

hq_status hq_hessian_project_psd(float* H, int64_t K, int steps, void* workspace, size_t workspace_bytes,
                                 hq_stream_t stream) {
  if (H == nullptr || K < 1 || steps < 0 || steps > 1000) return HQ_ERR_INVALID;
  if (K % 4 != 0 || K > 65536 || !aligned(H, 16)) return HQ_ERR_UNSUPPORTED;
  if (workspace == nullptr || !aligned(workspace, 256) || workspace_bytes < psd_workspace(K)) return HQ_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  int* status = reinterpret_cast<int*>(ws + 128);
  HQ_CUDA_TRY(cudaMemsetAsync(status, 0, sizeof(int), s));
  hq_status st = launch_psd(H, K, steps, ws, status, s);
  if (st != HQ_OK) return st;
  int h_status = 0;
  HQ_CUDA_TRY(cudaMemcpyAsync(&h_status, status, sizeof(int), cudaMemcpyDeviceToHost, s));
  HQ_CUDA_TRY(cudaStreamSynchronize(s));
  return h_status == HQ_ERR_TIMEOUT ? HQ_ERR_TIMEOUT : HQ_OK;
}

hq_status hq_hadamard_rotate_weights(const void* W, int w_dtype, int64_t N, int64_t K, int64_t block,
                                     const float* signs, float* W_out, hq_stream_t stream) {
  if (W == nullptr || signs == nullptr || W_out == nullptr || N < 0 || !valid_dtype(w_dtype)) return HQ_ERR_INVALID;
  if (!hadamard_shape_ok(K, block)) return HQ_ERR_UNSUPPORTED;
  if (w_dtype == HQ_BF16 && static_cast<const void*>(W_out) == W) return HQ_ERR_INVALID;
  return launch_hadamard_rows(W, w_dtype, N, K, static_cast<int>(block), signs, W_out,
                              static_cast<cudaStream_t>(stream));
}

hq_status hq_hadamard_rotate_hessian(const float* H, int64_t K, int64_t block, const float* signs, float* H_out,
                                     hq_stream_t stream) {
  if (H == nullptr || signs == nullptr || H_out == nullptr) return HQ_ERR_INVALID;
  if (H == H_out) return HQ_ERR_INVALID;
  if (!hadamard_shape_ok(K, block)) return HQ_ERR_UNSUPPORTED;
  return launch_hadamard_hessian(H, K, static_cast<int>(block), signs, H_out, static_cast<cudaStream_t>(stream));
}

size_t hq_bf16tril_bytes(int64_t K) {
  if (K < 1) return 0;
  return static_cast<size_t>(K) * 4 + static_cast<size_t>(K) * (K - 1) / 2 * 2;
}

hq_status hq_hessian_pack_bf16tril(const float* H, int64_t K, uint8_t* out, hq_stream_t stream) {
  if (H == nullptr || out == nullptr || K < 1) return HQ_ERR_INVALID;
  if (!aligned(out, 16) || !aligned(H, 4)) return HQ_ERR_INVALID;
  if (K > (int64_t(1) << 20)) return HQ_ERR_UNSUPPORTED;
  return launch_tril_encode(H, K, out, static_cast<cudaStream_t>(stream));
}

hq_status hq_hessian_unpack_bf16tril(const uint8_t* in, int64_t K, float* H_full, hq_stream_t stream) {
  if (in == nullptr || H_full == nullptr || K < 1) return HQ_ERR_INVALID;
  if (!aligned(in, 16) || !aligned(H_full, 4)) return HQ_ERR_INVALID;
  if (K > (int64_t(1) << 20)) return HQ_ERR_UNSUPPORTED;
  return launch_tril_decode(in, K, H_full, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
