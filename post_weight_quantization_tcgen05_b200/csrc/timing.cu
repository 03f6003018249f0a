// Optional per-kernel timing with CUDA events recorded on the launching stream, for profiling
// from the caller's side (the benchmark asks for the duration of one kernel class inside its
// timed region).  Off by default; when off, a launch site pays one relaxed load.
#include <mutex>
#include <vector>

#include "common.cuh"
#include "kernels.cuh"

namespace hq {
namespace {

struct TimedLaunch {
  cudaEvent_t start = nullptr, stop = nullptr;
  int cls = 0;
  double work = 0.0;
};

std::mutex g_mu;
int g_mask = 0;                     // classes being timed (bit per TimerClass)
int g_serialize = 0;                // hq_debug_timing_serialize
std::vector<TimedLaunch> g_pool;    // events are created once and reused
size_t g_used = 0;

}  // namespace

int timer_start(int cls, cudaStream_t s) {
  if ((__atomic_load_n(&g_mask, __ATOMIC_RELAXED) & (1 << cls)) == 0) return -1;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_used == g_pool.size()) {
    TimedLaunch t;
    if (cudaEventCreate(&t.start) != cudaSuccess || cudaEventCreate(&t.stop) != cudaSuccess) {
      (void)cudaGetLastError();
      return -1;
    }
    g_pool.push_back(t);
  }
  TimedLaunch& t = g_pool[g_used];
  if (cudaEventRecord(t.start, s) != cudaSuccess) {
    (void)cudaGetLastError();
    return -1;
  }
  t.cls = cls;
  t.work = 0.0;
  return static_cast<int>(g_used++);
}

bool timing_serialized() { return __atomic_load_n(&g_serialize, __ATOMIC_RELAXED) != 0; }

void timer_stop(int idx, double work, cudaStream_t s) {
  if (idx < 0) return;
  std::lock_guard<std::mutex> lk(g_mu);
  if (static_cast<size_t>(idx) >= g_used) return;
  g_pool[idx].work = work;
  if (cudaEventRecord(g_pool[idx].stop, s) != cudaSuccess) (void)cudaGetLastError();
}

}  // namespace hq

using namespace hq;

extern "C" hq_status hq_debug_timing_start(int class_mask) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_used = 0;
  __atomic_store_n(&g_mask, class_mask, __ATOMIC_RELAXED);
  return HQ_OK;
}

extern "C" hq_status hq_debug_timing_serialize(int on) {
  __atomic_store_n(&g_serialize, on != 0 ? 1 : 0, __ATOMIC_RELAXED);
  return HQ_OK;
}

extern "C" hq_status hq_debug_timing_stop(void) {
  __atomic_store_n(&g_mask, 0, __ATOMIC_RELAXED);
  return HQ_OK;
}

extern "C" hq_status hq_debug_timing_read(int cls, double* ms_total, double* work_total, int64_t* launches) {
  if (ms_total == nullptr || work_total == nullptr || launches == nullptr) return HQ_ERR_INVALID;
  std::lock_guard<std::mutex> lk(g_mu);
  double ms = 0.0, work = 0.0;
  int64_t n = 0;
  for (size_t i = 0; i < g_used; ++i) {
    if (g_pool[i].cls != cls) continue;
    HQ_CUDA_TRY(cudaEventSynchronize(g_pool[i].stop));
    float e = 0.f;
    HQ_CUDA_TRY(cudaEventElapsedTime(&e, g_pool[i].start, g_pool[i].stop));
    ms += e;
    work += g_pool[i].work;
    ++n;
  }
  *ms_total = ms;
  *work_total = work;
  *launches = n;
  return HQ_OK;
}
