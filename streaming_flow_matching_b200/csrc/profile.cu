// Event-based device timing of this library's kernels and a launch counter.
#include <atomic>
#include <vector>

#include "common.cuh"

namespace sfm {

namespace {
struct ProfState {
  bool on = false;
  int used = 0;
  std::vector<cudaEvent_t> ev;   // 2 per recorded launch
  std::vector<int> kind;
};
thread_local ProfState g_prof;
std::atomic<unsigned long long> g_launches{0};
}  // namespace

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

bool profiling_active() { return g_prof.on; }



ProfScope::ProfScope(int kind, cudaStream_t s) : s_(s) {
  if (!g_prof.on || g_prof.used * 2 + 1 >= (int)g_prof.ev.size()) return;
  idx_ = g_prof.used++;
  g_prof.kind[idx_] = kind;
  cudaEventRecord(g_prof.ev[2 * idx_], s_);
}

ProfScope::~ProfScope() {
  if (idx_ >= 0) cudaEventRecord(g_prof.ev[2 * idx_ + 1], s_);
}

}  // namespace sfm

using namespace sfm;

extern "C" {

int sfm_profile_begin(int max_launches) {
  if (max_launches < 1) return SFM_EINVAL;
  for (cudaEvent_t e : g_prof.ev) cudaEventDestroy(e);
  g_prof = ProfState();
  g_prof.ev.resize(2 * (size_t)max_launches, nullptr);
  g_prof.kind.assign(max_launches, 0);
  for (auto& e : g_prof.ev)
    if (cudaEventCreate(&e) != cudaSuccess) {
      for (cudaEvent_t x : g_prof.ev)
        if (x) cudaEventDestroy(x);
      g_prof = ProfState();
      return record_cuda(cudaGetLastError());
    }
  g_prof.on = true;
  return SFM_OK;
}

int sfm_profile_end(double* ms, long long* launches) {
  if (!ms || !launches) return SFM_EINVAL;
  for (int k = 0; k < SFM_PROF_KINDS; ++k) {
    ms[k] = 0.0;
    launches[k] = 0;
  }
  int rc = SFM_OK;
  for (int i = 0; i < g_prof.used && rc == SFM_OK; ++i) {
    cudaError_t e = cudaEventSynchronize(g_prof.ev[2 * i + 1]);
    float t = 0.f;
    if (e == cudaSuccess) e = cudaEventElapsedTime(&t, g_prof.ev[2 * i], g_prof.ev[2 * i + 1]);
    if (e != cudaSuccess) {
      rc = record_cuda(e);
      break;
    }
    ms[g_prof.kind[i]] += t;
    launches[g_prof.kind[i]] += 1;
  }
  for (cudaEvent_t e : g_prof.ev) cudaEventDestroy(e);
  g_prof = ProfState();
  return rc;
}

unsigned long long sfm_kernel_launch_count(void) { return g_launches.load(); }

}  // extern "C"
