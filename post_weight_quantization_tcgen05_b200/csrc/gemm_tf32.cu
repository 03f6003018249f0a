// Host launcher of the tcgen05 tf32 GEMM (gemm_tf32.cuh).
#include "common.cuh"
#include "gemm_tf32.cuh"
#include "kernels.cuh"
#include "tmap.cuh"

namespace hq {

template <bool SPLIT3>
static hq_status launch_tf32(const CUtensorMap& ma, const CUtensorMap& mb, const Tf32GemmArgs& a, int tiles,
                             cudaStream_t s) {
  using Cfg = Tf32Cfg<SPLIT3>;
  auto kern = tf32_gemm_kernel<SPLIT3>;
  HQ_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::kSmemBytes));
  const int tm = timer_start(kTimeTf32Gemm, s);
  kern<<<tiles, Cfg::kThreads, Cfg::kSmemBytes, s>>>(ma, mb, a);
  HQ_LAUNCH_CHECK();
  timer_stop(tm, 2.0 * a.M * a.N * static_cast<double>(a.Kred), s);  // the product's flops
  return HQ_OK;
}

hq_status tf32_gemm(const Tf32Gemm& g, cudaStream_t s) {
  if (g.M <= 0 || g.N <= 0) return HQ_OK;
  if (!aligned(g.A, 16) || !aligned(g.B, 16) || (g.lda % 4) || (g.ldb % 4)) return HQ_ERR_UNSUPPORTED;
  const uint64_t kred = static_cast<uint64_t>(g.Kred > 0 ? g.Kred : 1);
  CUtensorMap ma, mb;
  if (!make_tmap_2d(&ma, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, g.A, kred, static_cast<uint64_t>(g.M),
                    static_cast<uint64_t>(g.lda) * 4, 32, 128))
    return HQ_ERR_CUDA;
  if (!make_tmap_2d(&mb, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, g.B, kred, static_cast<uint64_t>(g.N),
                    static_cast<uint64_t>(g.ldb) * 4, 32, 128))
    return HQ_ERR_CUDA;
  Tf32GemmArgs a{};
  a.C = g.C;
  a.ldc = g.ldc;
  a.M = g.M;
  a.N = g.N;
  a.Kred = g.Kred;
  a.alpha = g.alpha;
  a.beta = g.beta;
  a.lower = g.lower;
  a.row0 = g.row0;
  a.col0 = g.col0;
  a.tiles_n = static_cast<int>(ceil_div(g.N, 128));
  a.skip = g.skip;
  a.status = g.status;
  const int64_t tiles = ceil_div(g.M, 128) * a.tiles_n;
  if (tiles > 0x7FFFFFFF) return HQ_ERR_UNSUPPORTED;
  const int t = static_cast<int>(tiles);
  return g.split3 ? launch_tf32<true>(ma, mb, a, t, s) : launch_tf32<false>(ma, mb, a, t, s);
}

}  // namespace hq
