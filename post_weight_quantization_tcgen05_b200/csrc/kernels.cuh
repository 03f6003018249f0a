// Internal launchers shared between the translation units of libhq (not part of the ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/hq.h"

namespace hq {

// syrk.cu
bool syrk_tc_eligible(const void* X, int x_dtype, int64_t T, int64_t K);
hq_status launch_syrk_tc(float* H, const void* X, int64_t T, int64_t K, int* dev_status, cudaStream_t s);
hq_status launch_syrk_simt(float* H, const void* X, int x_dtype, int64_t T, int64_t K, cudaStream_t s);

// codec.cu
hq_status launch_tril_encode(const float* H, int64_t K, uint8_t* out, cudaStream_t s);
hq_status launch_tril_decode(const uint8_t* in, int64_t K, float* H, cudaStream_t s);

// factor.cu
size_t factor_workspace_floats(int64_t K);
hq_status launch_factor(const float* H, int64_t K, float damp, float* A, float* X, float* T, float* Dinv,
                        double* lam, int* info, float* Ut, cudaStream_t s);

// sweep.cu
struct GptqLayout {
  size_t header, partials, wf, err, a, x, t, dinv, total;
  int sweep_grid;
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
hq_status launch_gptq(const void* W, int w_dtype, int64_t N, int64_t K, const float* H, int64_t group, float damp,
                      const float* imp, uint8_t* codes, float* scales, double* qerr_dev, uint8_t* ws,
                      int update_impl, cudaStream_t s);

// rtn.cu
size_t rtn_workspace(int64_t N, int64_t K, int64_t group);
hq_status launch_rtn(const void* W, int w_dtype, int64_t N, int64_t K, int64_t group, const float* imp,
                     uint8_t* codes, float* scales, double* qerr_dev, uint8_t* ws, cudaStream_t s);

// gptq.cu: qerr reduction shared by GPTQ and RTN
hq_status launch_qerr_finalize(const double* partials, int64_t count, WsHeader* hdr, double* qerr_dev,
                               cudaStream_t s);

}  // namespace hq
