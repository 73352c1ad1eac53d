// fps_noalloc.cu -- ssc_fps_patches without a caller workspace.
//
// Some callers cannot allocate device memory at all: code that runs inside a
// host application which owns every device allocation and only hands over its
// input and output buffers, or a loop that must not allocate (or ask anyone to
// allocate) between steps.  For them this entry point keeps the scratch space
// that ssc_fps_patches takes from its workspace (the per-patch counters, the
// fill cursors and, for point counts beyond the on-chip path, the running
// distances) in one fixed array that lives in the library's own device memory.
//
// The array is a file-scope __device__ variable, so every GPU that loads the
// library holds it until the process exits.  Host code cannot use the array's
// name as a device address; the address is looked up once per device with
// cudaGetSymbolAddress, with that device current, on the first call made on
// that device, and kept for the rest of the process (a host program that
// resets the device's primary context must not call this entry point on it
// again).  All calls share the one array and it keeps the last call's
// contents: the counters that must start at zero are cleared by every call
// (on the stream, like the rest of the work), and calls that overlap on the
// GPU -- on different streams or from different host threads -- race on it.
#include <mutex>

#include "internal.h"
#include "ssc.h"

namespace {

constexpr size_t kScratchBytes = 3u << 20;  // 3 MiB: covers n <= 262144, P <= 65535

static __device__ __align__(256) unsigned char g_fps_scratch[kScratchBytes];

std::mutex g_mu;
void* g_addr[64] = {nullptr};

// Device address of the scratch array on the current device (set up once).
int scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return SSC_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_fps_scratch) != cudaSuccess || !p) return SSC_ERR_CUDA;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return SSC_OK;
}

}  // namespace

extern "C" int ssc_fps_patches_noalloc(const float* pts, int n, int P, int seed_vertex,
                                       int* centers, int* owner, int* offsets, int* members,
                                       ssc_stream_t stream) {
  if (!pts || !centers || !owner || !offsets || !members) return SSC_ERR_INVALID_ARG;
  if (n < 1 || P < 1 || P > n || seed_vertex < 0 || seed_vertex >= n) return SSC_ERR_INVALID_ARG;
  if (n > SSC_FPS_NOALLOC_MAX_N || P > SSC_FPS_NOALLOC_MAX_P) return SSC_ERR_UNSUPPORTED;
  if (ssc::fps_workspace_bytes(n, P) > kScratchBytes) return SSC_ERR_UNSUPPORTED;
  void* ws = nullptr;
  const int rc = scratch_address(&ws);
  if (rc != SSC_OK) return rc;
  (void)cudaGetLastError();
  const ssc::WaitCtl ctl = ssc::library_wait_ctl();
  if (!ctl.status) return SSC_ERR_CUDA;
  return ssc::launch_fps_patches(pts, n, P, seed_vertex, centers, owner, offsets, members, ws,
                                 static_cast<cudaStream_t>(stream), ctl) == cudaSuccess
             ? SSC_OK
             : SSC_ERR_CUDA;
}
