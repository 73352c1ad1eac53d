// profile.cu -- launch timing of the coupling kernels with CUDA events.
//
// While recording is on, every launch of a tracked kernel is bracketed by two
// CUDA events recorded on the launch's own stream, so the elapsed time between
// them is that kernel's device duration (and includes nothing launched on
// other streams).  Reading the record waits for the events of the launches
// made since recording was switched on, sums their durations per kernel and
// releases the events.  Events are host-side driver objects; no device memory
// is allocated.  The record is process-wide and guarded by a mutex.
#include <mutex>
#include <vector>

#include "internal.h"
#include "ssc.h"

namespace ssc {
namespace {

struct Mark {
  int kernel;
  cudaEvent_t start, stop;
};

std::mutex g_prof_mu;
bool g_prof_on = false;
std::vector<Mark> g_marks;
Mark g_open = {-1, nullptr, nullptr};

}  // namespace

void prof_launch_begin(cudaStream_t st) {
  std::lock_guard<std::mutex> lock(g_prof_mu);
  if (!g_prof_on) return;
  Mark m = {-1, nullptr, nullptr};
  if (cudaEventCreate(&m.start) != cudaSuccess) return;
  if (cudaEventCreate(&m.stop) != cudaSuccess) {
    cudaEventDestroy(m.start);
    return;
  }
  cudaEventRecord(m.start, st);
  g_open = m;
}

void prof_launch_end(cudaStream_t st, int kernel) {
  std::lock_guard<std::mutex> lock(g_prof_mu);
  if (!g_prof_on || !g_open.start) return;
  cudaEventRecord(g_open.stop, st);
  g_open.kernel = kernel;
  g_marks.push_back(g_open);
  g_open = {-1, nullptr, nullptr};
}

}  // namespace ssc

namespace {
void release_all() {
  for (auto& m : ssc::g_marks) {
    cudaEventDestroy(m.start);
    cudaEventDestroy(m.stop);
  }
  ssc::g_marks.clear();
}
}  // namespace

extern "C" int ssc_profile_enable(int on) {
  if (on < 0 || on > 2) return SSC_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(ssc::g_prof_mu);
  if (on == 1) release_all();
  ssc::g_prof_on = on != 0;
  return SSC_OK;
}

extern "C" int ssc_profile_read(int kernel, double* total_ms, int* launches) {
  if (!total_ms || !launches || kernel < 0 || kernel >= SSC_PROF_KERNELS) return SSC_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(ssc::g_prof_mu);
  double sum = 0.0;
  int count = 0;
  for (auto& m : ssc::g_marks) {
    if (m.kernel != kernel) continue;
    float ms = 0.f;
    if (cudaEventSynchronize(m.stop) != cudaSuccess || cudaEventElapsedTime(&ms, m.start, m.stop) != cudaSuccess)
      return SSC_ERR_CUDA;
    sum += ms;
    ++count;
  }
  *total_ms = sum;
  *launches = count;
  return SSC_OK;
}
