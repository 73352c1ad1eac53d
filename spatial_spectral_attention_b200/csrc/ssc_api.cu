// ssc_api.cu -- the C ABI of libssc (declared in include/ssc.h): argument
// checks, workspace carving and the launch sequence of every call.  No call
// allocates device memory and none synchronises the host (except
// ssc_device_status, whose job is to read the status word back).  Launches
// that are independent of the ones before them go to a per-thread side stream
// and are joined back into the caller's stream before their results are used.
#include <algorithm>
#include <cmath>
#include <cstdint>

#include "ssc.h"
#include "internal.h"

using namespace ssc;

namespace {

__device__ unsigned g_status_word;  // bit 0: a wait ran out; bit 1: bad index

unsigned long long g_wait_limit_ns = 2000000000ull;

unsigned* status_ptr() {
  static unsigned* ptrs[64] = {nullptr};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  if (!ptrs[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status_word) != cudaSuccess) return nullptr;
    ptrs[dev] = static_cast<unsigned*>(p);
  }
  return ptrs[dev];
}

WaitCtl make_ctl() {
  WaitCtl c;
  c.status = status_ptr();
  c.limit_ns = g_wait_limit_ns;
  return c;
}

int cuda_status(cudaError_t e) { return e == cudaSuccess ? SSC_OK : SSC_ERR_CUDA; }

// A side stream for launches that do not depend on the work just before them
// on the caller's stream (the Geo patch-major gather runs beside the tile
// schedule, the backward's accumulator zeroing beside its row prep).  One per
// host thread and device, with its two events, made on the thread's first call
// outside stream capture; when there is none (or the caller's stream is the
// side stream) the work stays on the caller's stream, in the same order.
struct Side {
  cudaStream_t st = nullptr;
  cudaEvent_t fork = nullptr, join = nullptr;
};

Side* side_for(cudaStream_t st) {
  thread_local Side sides[64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  Side& s = sides[dev];
  if (!s.st) {
    cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing(st, &cs) != cudaSuccess || cs != cudaStreamCaptureStatusNone)
      return nullptr;
    Side n;
    if (cudaStreamCreateWithFlags(&n.st, cudaStreamNonBlocking) != cudaSuccess) return nullptr;
    if (cudaEventCreateWithFlags(&n.fork, cudaEventDisableTiming) != cudaSuccess ||
        cudaEventCreateWithFlags(&n.join, cudaEventDisableTiming) != cudaSuccess) {
      if (n.fork) cudaEventDestroy(n.fork);
      cudaStreamDestroy(n.st);
      return nullptr;
    }
    s = n;
  }
  return s.st == st ? nullptr : &s;
}

// Starts a fork: the side stream waits for everything enqueued on st so far.
// Returns the stream that the independent launches go to (st itself when
// there is no side stream) and sets *side (nullptr when there is none).
cudaError_t fork_begin(cudaStream_t st, Side** side, cudaStream_t* to) {
  *side = side_for(st);
  *to = st;
  if (!*side) return cudaSuccess;
  cudaError_t e = cudaEventRecord((*side)->fork, st);
  if (e == cudaSuccess) e = cudaStreamWaitEvent((*side)->st, (*side)->fork, 0);
  if (e == cudaSuccess) *to = (*side)->st;
  return e;
}

// Ends a fork: st waits for the side stream's launches since fork_begin.
cudaError_t fork_end(cudaStream_t st, Side* side) {
  if (!side) return cudaSuccess;
  cudaError_t e = cudaEventRecord(side->join, side->st);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(st, side->join, 0);
  return e;
}

}  // namespace

WaitCtl ssc::library_wait_ctl() { return make_ctl(); }

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int check_common(const void* Q, int ldq, const void* K, int ldk, const void* V, int ldv, int nN,
                 int nM, int d, int k, float scale, int dtype) {
  if (!Q || !K || !V) return SSC_ERR_INVALID_ARG;
  if (nN < 1 || nM < 1 || k < 1) return SSC_ERR_INVALID_ARG;
  if (!(std::isfinite(scale) && scale > 0.f)) return SSC_ERR_INVALID_ARG;
  if (dtype != SSC_BF16 && dtype != SSC_F32) return SSC_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SSC_ERR_UNSUPPORTED;
  if (k > 256) return SSC_ERR_UNSUPPORTED;
  if (ldq < d || ldk < d || ldv < k) return SSC_ERR_INVALID_ARG;
  if (dtype == SSC_BF16) {
    // Q and K are read by TMA in place; V of any stride is re-packed when needed
    if (!aligned16(Q) || !aligned16(K)) return SSC_ERR_ALIGNMENT;
    if (ldq % 8 || ldk % 8) return SSC_ERR_ALIGNMENT;
    if (reinterpret_cast<uintptr_t>(V) & 1u) return SSC_ERR_ALIGNMENT;
  } else {
    const uintptr_t m = reinterpret_cast<uintptr_t>(Q) | reinterpret_cast<uintptr_t>(K) |
                        reinterpret_cast<uintptr_t>(V);
    if (m & 3u) return SSC_ERR_ALIGNMENT;
  }
  return SSC_OK;
}

int check_out(const float* p, int ld, int cols) {
  if (!p) return SSC_ERR_INVALID_ARG;
  if (ld < cols) return SSC_ERR_INVALID_ARG;
  if (!aligned16(p)) return SSC_ERR_ALIGNMENT;
  return SSC_OK;
}

int check_patches(const int* offN, const int* memN, int PN, int nN, const int* offM,
                  const int* memM, int PM, int nM, const int* topk, int R) {
  if (!offN || !memN || !offM || !memM || !topk) return SSC_ERR_INVALID_ARG;
  if (PN < 1 || PM < 1 || PN > nN || PM > nM || PN > 65535 || PM > 65535) return SSC_ERR_INVALID_ARG;
  if (R < 1 || R > PM) return SSC_ERR_INVALID_ARG;
  return SSC_OK;
}

size_t kp_of(int k) {
  size_t kp = (k + 15) / 16 * 16;
  if (kp % 64 == 48) kp += 16;
  return kp;
}

cudaError_t zero_matrix(float* p, int ld, int rows, int cols, cudaStream_t st) {
  if (ld == cols) return cudaMemsetAsync(p, 0, sizeof(float) * (size_t)rows * cols, st);
  return cudaMemset2DAsync(p, sizeof(float) * (size_t)ld, 0, sizeof(float) * (size_t)cols, rows, st);
}

// ---- workspace layouts (sizes only when base == nullptr)
struct DenseWs {
  RowTile* tiles;
  KeySeg* segs;
  int* prefix;
  __nv_bfloat16* dOb;
  __nv_bfloat16* Vpad;  // V re-packed with a 16-byte aligned row pitch
  float* D;
  float* part;  // split query tiles of the pair forward (partial O, max, sum)
};
size_t dense_ws(void* base, int nN, int nM, int d, int k, int dtype, DenseWs* w) {
  Carve c(base);
  DenseWs x;
  x.tiles = c.take<RowTile>(dense_num_tiles(nN));
  x.segs = c.take<KeySeg>(dense_num_segs(nM));
  x.prefix = c.take<int>(dense_num_tiles(nN) + 1);
  x.dOb = dtype == SSC_BF16 ? c.take<__nv_bfloat16>((size_t)nN * kp_of(k)) : nullptr;
  x.Vpad = dtype == SSC_BF16 ? c.take<__nv_bfloat16>((size_t)nM * kp_of(k)) : nullptr;
  x.D = c.take<float>(nN);
  x.part = dtype == SSC_BF16 && tc_pair_supported(d, k) ? c.take<float>(tc_pair_part_floats(k)) : nullptr;
  if (w) *w = x;
  return c.used + 256;
}

struct GeoWs {
  void* Qp;
  void* Kp;
  void* Vp;
  void* dOp;
  float* D;
  float* lsep;
  float* dKg;  // dK in the patch-major key order (bf16 path), scattered to vertex order after
  RowTile* tiles;
  KeySeg* segs;
  int* counts;
  int* prefix;
  int* sched_scratch;
  int* inv_off;
  int* inv_p;
  int* inv_scratch;
  unsigned long long* tag;  // fingerprint of the forward that filled the workspace
  int ldq, ldk, ldv, ldg;
};
size_t geo_ws(void* base, int nN, int nM, int d, int k, int PN, int PM, int R, int dtype, GeoWs* w) {
  Carve c(base);
  GeoWs x;
  const bool bf = dtype == SSC_BF16;
  const size_t es = bf ? 2 : 4;
  x.ldq = d;
  x.ldk = d;
  x.ldv = bf ? (int)kp_of(k) : k;
  x.ldg = bf ? (int)kp_of(k) : k;
  x.Qp = c.take<uint8_t>((size_t)nN * x.ldq * es);
  x.Kp = c.take<uint8_t>((size_t)nM * x.ldk * es);
  x.Vp = c.take<uint8_t>((size_t)nM * x.ldv * es);
  x.dOp = c.take<uint8_t>((size_t)nN * x.ldg * es);
  x.D = c.take<float>(nN);
  x.lsep = c.take<float>(nN);
  x.dKg = dtype == SSC_BF16 ? c.take<float>((size_t)nM * d) : nullptr;
  x.tiles = c.take<RowTile>(geo_max_tiles(nN, PN));
  x.segs = c.take<KeySeg>(geo_max_segs(nM, PM, PN, R));
  x.counts = c.take<int>(2);
  x.prefix = c.take<int>(geo_max_tiles(nN, PN) + 1);
  x.sched_scratch = c.take<int>(geo_schedule_scratch_ints(PN));
  x.inv_off = c.take<int>(PM + 1);
  x.inv_p = c.take<int>((size_t)PN * R);
  x.inv_scratch = c.take<int>(invert_topk_scratch_ints(PM));
  x.tag = c.take<unsigned long long>(1);
  if (w) *w = x;
  return c.used + 256;
}

// Fingerprint of a Geo call: sizes, dtype and the addresses of its operands
// and tables (64-bit FNV-1a over the values).
unsigned long long geo_fingerprint(const void* Q, const void* K, const void* V, int nN, int nM,
                                   int d, int k, int dtype, const int* offN, const int* memN,
                                   int PN, const int* offM, const int* memM, int PM,
                                   const int* topk, int R) {
  const unsigned long long v[] = {
      (unsigned long long)reinterpret_cast<uintptr_t>(Q), (unsigned long long)reinterpret_cast<uintptr_t>(K),
      (unsigned long long)reinterpret_cast<uintptr_t>(V), (unsigned long long)reinterpret_cast<uintptr_t>(offN),
      (unsigned long long)reinterpret_cast<uintptr_t>(memN), (unsigned long long)reinterpret_cast<uintptr_t>(offM),
      (unsigned long long)reinterpret_cast<uintptr_t>(memM), (unsigned long long)reinterpret_cast<uintptr_t>(topk),
      (unsigned long long)nN, (unsigned long long)nM, (unsigned long long)d, (unsigned long long)k,
      (unsigned long long)dtype, (unsigned long long)PN, (unsigned long long)PM, (unsigned long long)R};
  unsigned long long h = 1469598103934665603ull;
  for (unsigned long long x : v)
    for (int b = 0; b < 8; ++b) {
      h ^= (x >> (8 * b)) & 0xffull;
      h *= 1099511628211ull;
    }
  return h;
}

bool ws_ok(void* ws, size_t have, size_t need) {
  return ws && have >= need && (reinterpret_cast<uintptr_t>(ws) & 255u) == 0;
}

// The bf16 V operand as the tensor-core kernels read it: in place when its
// rows are 16-byte aligned, else re-packed into the workspace.
// V for the tensor-core kernels: used in place when its rows are 16-byte
// aligned, else re-packed into the workspace with a pitch of kp.  With
// ones_col = k (possible when k is not a multiple of 16, so the pitch has a
// padding column) V is always re-packed and that column is set to one.
cudaError_t dense_v(const void* V, int ldv, int nM, int k, const DenseWs& w,
                    const __nv_bfloat16** Vout, int* ldout, cudaStream_t st, unsigned* status,
                    int ones_col = -1) {
  if (ones_col < 0 && ldv % 8 == 0 && aligned16(V)) {
    *Vout = static_cast<const __nv_bfloat16*>(V);
    *ldout = ldv;
    return cudaSuccess;
  }
  *Vout = w.Vpad;
  *ldout = (int)kp_of(k);
  return launch_gather_rows_bf16(V, ldv, 0, nullptr, nM, nM, k, w.Vpad, (int)kp_of(k), status, st,
                                 ones_col);
}

}  // namespace

extern "C" {

const char* ssc_status_string(int status) {
  switch (status) {
    case SSC_OK: return "ok";
    case SSC_ERR_INVALID_ARG: return "invalid argument (size, null pointer or index table)";
    case SSC_ERR_UNSUPPORTED: return "unsupported size (d must be 64 or 128, 1 <= k <= 256)";
    case SSC_ERR_ALIGNMENT: return "misaligned pointer or leading dimension";
    case SSC_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case SSC_ERR_CUDA: return "CUDA call failed";
    case SSC_ERR_TIMEOUT: return "a device-side wait ran out of time";
    default: return "unknown status";
  }
}

int ssc_version(void) { return (0 << 16) | 1; }

unsigned long long ssc_kernel_launches(void) { return g_launches.load(); }

int ssc_device_status(ssc_stream_t stream, int clear, int* status) {
  if (!status) return SSC_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(st) != cudaSuccess) return SSC_ERR_CUDA;
  unsigned* p = status_ptr();
  if (!p) return SSC_ERR_CUDA;
  unsigned word = 0;
  if (cudaMemcpy(&word, p, sizeof(word), cudaMemcpyDeviceToHost) != cudaSuccess) return SSC_ERR_CUDA;
  if (clear) {
    unsigned zero = 0;
    if (cudaMemcpy(p, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess) return SSC_ERR_CUDA;
  }
  *status = (word & kStatusTimeout) ? SSC_ERR_TIMEOUT
            : (word & kStatusBadIndex) ? SSC_ERR_INVALID_ARG
                                        : SSC_OK;
  return SSC_OK;
}

int ssc_set_wait_limit_ns(unsigned long long ns) {
  g_wait_limit_ns = ns ? ns : 2000000000ull;
  return SSC_OK;
}

int ssc_debug_wait_timeout(unsigned long long limit_ns, ssc_stream_t stream) {
  WaitCtl c = make_ctl();
  if (!c.status) return SSC_ERR_CUDA;
  c.limit_ns = limit_ns ? limit_ns : 1000000ull;
  return cuda_status(launch_wait_timeout_probe(static_cast<cudaStream_t>(stream), c));
}

int ssc_debug_stall_next_launch(int which) {
  if (which < 0 || which > 2) return SSC_ERR_INVALID_ARG;
  tc_debug_stall_next(which);
  return SSC_OK;
}

// ------------------------------------------------------------ patches
int ssc_debug_fps_cluster_size(int cl) {
  if (cl != 0 && cl != 8 && cl != 16) return SSC_ERR_INVALID_ARG;
  fps_force_cluster_size(cl);
  return SSC_OK;
}

size_t ssc_fps_patches_workspace_size(int n, int P) {
  if (n < 1 || P < 1) return 0;
  return fps_workspace_bytes(n, P);
}

int ssc_fps_patches(const float* pts, int n, int P, int seed_vertex, int* centers, int* owner,
                    int* offsets, int* members, void* ws, size_t ws_bytes, ssc_stream_t stream) {
  if (!pts || !centers || !owner || !offsets || !members) return SSC_ERR_INVALID_ARG;
  if (n < 1 || P < 1 || P > n || P > 65535 || n > (1 << 24)) return SSC_ERR_INVALID_ARG;
  if (seed_vertex < 0 || seed_vertex >= n) return SSC_ERR_INVALID_ARG;
  if (!ws_ok(ws, ws_bytes, fps_workspace_bytes(n, P))) return SSC_ERR_WORKSPACE;
  (void)cudaGetLastError();  // clear a stale error left by an earlier, unrelated call
  WaitCtl c = make_ctl();
  if (!c.status) return SSC_ERR_CUDA;
  return cuda_status(launch_fps_patches(pts, n, P, seed_vertex, centers, owner, offsets, members, ws,
                                        static_cast<cudaStream_t>(stream), c));
}

size_t ssc_fps_patches_mesh_workspace_size(int n, int P) {
  if (n < 1 || P < 1) return 0;
  return fps_mesh_workspace_bytes(n, P);
}

int ssc_fps_patches_mesh(const int* adj_off, const int* adj, const double* edge_len, int n, int nnz,
                         int P, int seed_vertex, int* centers, int* owner, int* offsets,
                         int* members, void* ws, size_t ws_bytes, ssc_stream_t stream) {
  if (!adj_off || !centers || !owner || !offsets || !members) return SSC_ERR_INVALID_ARG;
  if (nnz > 0 && (!adj || !edge_len)) return SSC_ERR_INVALID_ARG;
  if (n < 1 || nnz < 0 || P < 1 || P > n || P > 65535) return SSC_ERR_INVALID_ARG;
  if (seed_vertex < 0 || seed_vertex >= n) return SSC_ERR_INVALID_ARG;
  if (!ws_ok(ws, ws_bytes, fps_mesh_workspace_bytes(n, P))) return SSC_ERR_WORKSPACE;
  (void)cudaGetLastError();  // clear a stale error left by an earlier, unrelated call
  WaitCtl c = make_ctl();
  return cuda_status(launch_fps_mesh(adj_off, adj, edge_len, n, nnz, P, seed_vertex, centers, owner,
                                     offsets, members, ws, static_cast<cudaStream_t>(stream), c));
}

size_t ssc_patch_scores_topk_workspace_size(int PN, int PM, int d) {
  if (PN < 1 || PM < 1 || d < 1) return 0;
  return scores_topk_workspace_bytes(PN, PM, d);
}

int ssc_patch_scores_topk(const void* FN, int ldn, int nN, const void* FM, int ldm, int nM, int d,
                          int dtype, const int* offN, const int* memN, int PN, const int* offM,
                          const int* memM, int PM, int R, int* topk, double* scores, void* ws,
                          size_t ws_bytes, ssc_stream_t stream) {
  if (!FN || !FM || !offN || !memN || !offM || !memM || !topk) return SSC_ERR_INVALID_ARG;
  if (d < 1 || d > 1024 || ldn < d || ldm < d || nN < 1 || nM < 1) return SSC_ERR_INVALID_ARG;
  if (dtype != SSC_BF16 && dtype != SSC_F32) return SSC_ERR_INVALID_ARG;
  if (PN < 1 || PM < 1 || PN > nN || PM > nM || PN > 65535 || PM > 65535) return SSC_ERR_INVALID_ARG;
  if (R < 1 || R > PM) return SSC_ERR_INVALID_ARG;
  if (!ws_ok(ws, ws_bytes, scores_topk_workspace_bytes(PN, PM, d))) return SSC_ERR_WORKSPACE;
  (void)cudaGetLastError();  // clear a stale error left by an earlier, unrelated call
  WaitCtl c = make_ctl();
  return cuda_status(launch_scores_topk(FN, ldn, nN, FM, ldm, nM, d, dtype, offN, memN, PN, offM,
                                        memM, PM, R, topk, scores, ws, c.status,
                                        static_cast<cudaStream_t>(stream)));
}

// ------------------------------------------------------------ dense
size_t ssc_dense_coupling_workspace_size(int nN, int nM, int d, int k, int dtype) {
  if (nN < 1 || nM < 1 || k < 1) return 0;
  return dense_ws(nullptr, nN, nM, d, k, dtype, nullptr);
}

int ssc_dense_coupling_fwd(const void* Q, int ldq, const void* K, int ldk, const void* V, int ldv,
                           int nN, int nM, int d, int k, float scale, int dtype, float* O, int ldo,
                           float* lse, void* ws, size_t ws_bytes, ssc_stream_t stream) {
  int rc = check_common(Q, ldq, K, ldk, V, ldv, nN, nM, d, k, scale, dtype);
  if (rc) return rc;
  if ((rc = check_out(O, ldo, k))) return rc;
  if (!lse) return SSC_ERR_INVALID_ARG;
  if (!ws_ok(ws, ws_bytes, dense_ws(nullptr, nN, nM, d, k, dtype, nullptr))) return SSC_ERR_WORKSPACE;
  (void)cudaGetLastError();  // clear a stale error left by an earlier, unrelated call
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DenseWs w;
  dense_ws(ws, nN, nM, d, k, dtype, &w);
  cudaError_t e = launch_dense_schedule(nN, nM, w.tiles, w.segs, w.prefix, st);
  if (e != cudaSuccess) return SSC_ERR_CUDA;
  if (dtype == SSC_F32) {
    SimtArgs a{static_cast<const float*>(Q), static_cast<const float*>(K),
               static_cast<const float*>(V), ldq, ldk, ldv, nN, nM, d, k, scale, w.tiles, w.segs,
               nullptr, dense_num_tiles(nN), nullptr, nullptr};
    return cuda_status(launch_simt_fwd(a, O, ldo, lse, st));
  }
  WaitCtl ctl = make_ctl();
  const __nv_bfloat16* Vt;
  int ldvt;
  // the pair forward takes the softmax row sum from a column of ones in V when
  // the V pitch has a padding column
  const bool pair = tc_pair_supported(d, k);
  const int sum_col = pair && k % 16 != 0 ? k : -1;
  if ((e = dense_v(V, ldv, nM, k, w, &Vt, &ldvt, st, ctl.status, sum_col)) != cudaSuccess)
    return SSC_ERR_CUDA;
  if (pair)
    return cuda_status(launch_tc_fwd_pair(static_cast<const __nv_bfloat16*>(Q), ldq,
                                          static_cast<const __nv_bfloat16*>(K), ldk, Vt, ldvt, nN,
                                          nM, d, k, scale, O, ldo, lse, w.part, sum_col, st, ctl));
  TcArgs a{static_cast<const __nv_bfloat16*>(Q), static_cast<const __nv_bfloat16*>(K), Vt, ldq, ldk,
           ldvt, nN, nM, d, k, scale, w.tiles, w.segs, nullptr, dense_num_tiles(nN), w.prefix, nullptr,
           nullptr};
  return cuda_status(launch_tc_fwd(a, O, ldo, lse, st, ctl));
}

int ssc_dense_coupling_bwd(const void* Q, int ldq, const void* K, int ldk, const void* V, int ldv,
                           int nN, int nM, int d, int k, float scale, int dtype, const float* O,
                           int ldo, const float* lse, const float* dO, int lddo, float* dQ, int lddq,
                           float* dK, int lddk, float* dV, int lddv, void* ws, size_t ws_bytes,
                           ssc_stream_t stream) {
  int rc = check_common(Q, ldq, K, ldk, V, ldv, nN, nM, d, k, scale, dtype);
  if (rc) return rc;
  if (!O || !lse || !dO || ldo < k || lddo < k) return SSC_ERR_INVALID_ARG;
  if ((rc = check_out(dQ, lddq, d)) || (rc = check_out(dK, lddk, d))) return rc;
  if (dV && (rc = check_out(dV, lddv, k))) return rc;
  if (!ws_ok(ws, ws_bytes, dense_ws(nullptr, nN, nM, d, k, dtype, nullptr))) return SSC_ERR_WORKSPACE;
  (void)cudaGetLastError();  // clear a stale error left by an earlier, unrelated call
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  WaitCtl ctl = make_ctl();
  DenseWs w;
  dense_ws(ws, nN, nM, d, k, dtype, &w);
  cudaError_t e = launch_dense_schedule(nN, nM, w.tiles, w.segs, w.prefix, st);
  if (e != cudaSuccess) return SSC_ERR_CUDA;
  if (dtype == SSC_F32) {
    e = launch_bwd_prep(dO, lddo, O, ldo, lse, nullptr, nN, nN, k, nullptr, 0, nullptr, 0, w.D,
                        nullptr, ctl.status, st);
    if (e != cudaSuccess) return SSC_ERR_CUDA;
    SimtArgs a{static_cast<const float*>(Q), static_cast<const float*>(K),
               static_cast<const float*>(V), ldq, ldk, ldv, nN, nM, d, k, scale, w.tiles, w.segs,
               nullptr, dense_num_tiles(nN), nullptr, nullptr};
    if ((e = launch_simt_bwd_dq(a, dO, lddo, lse, w.D, dQ, lddq, st)) != cudaSuccess)
      return SSC_ERR_CUDA;
    SimtKeyArgs g{nullptr, 0, nullptr, nullptr, nullptr, ctl.status};
    return cuda_status(launch_simt_bwd_dkdv(a, g, dO, lddo, lse, w.D, dK, lddk, dV, lddv, st));
  }
  const int kp = (int)kp_of(k);
  // the zeroing of the accumulators and the V re-pack run on the side stream
  // beside the row prep (neither touches what the other reads or writes)
  Side* side;
  cudaStream_t zs;
  if ((e = fork_begin(st, &side, &zs)) != cudaSuccess) return SSC_ERR_CUDA;
  const __nv_bfloat16* Vt = nullptr;
  int ldvt = 0;
  e = zero_matrix(dK, lddk, nM, d, zs);
  if (e == cudaSuccess) e = zero_matrix(dQ, lddq, nN, d, zs);
  if (e == cudaSuccess && dV) e = zero_matrix(dV, lddv, nM, k, zs);
  if (e == cudaSuccess) e = dense_v(V, ldv, nM, k, w, &Vt, &ldvt, zs, ctl.status);
  if (e == cudaSuccess)
    e = launch_bwd_prep(dO, lddo, O, ldo, lse, nullptr, nN, nN, k, w.dOb, kp, nullptr, 0, w.D,
                        nullptr, ctl.status, st);
  const cudaError_t j = fork_end(st, side);
  if (e != cudaSuccess || j != cudaSuccess) return SSC_ERR_CUDA;
  TcArgs a{static_cast<const __nv_bfloat16*>(Q), static_cast<const __nv_bfloat16*>(K), Vt, ldq, ldk,
           ldvt, nN, nM, d, k, scale, w.tiles, w.segs, nullptr, dense_num_tiles(nN), w.prefix, nullptr,
           nullptr};
  // dQ and dK query-stationary; dV key-stationary in a kernel of its own
  if ((e = launch_tc_bwd(a, w.dOb, kp, lse, w.D, dQ, lddq, dK, lddk, nullptr, 0, st, ctl)) !=
      cudaSuccess)
    return SSC_ERR_CUDA;
  if (!dV) return SSC_OK;
  return cuda_status(launch_tc_dv_dense(static_cast<const __nv_bfloat16*>(Q), ldq,
                                        static_cast<const __nv_bfloat16*>(K), ldk, w.dOb, kp, lse, nN,
                                        nM, d, k, scale, dV, lddv, st, ctl));
}

size_t ssc_dense_coupling_fwd_e4m3_workspace_size(int nN, int nM, int d, int k) {
  if (nN < 1 || nM < 1 || k < 1 || d != 128) return 0;
  Carve c(nullptr);
  c.take<uint8_t>((size_t)nN * d);
  c.take<uint8_t>((size_t)nM * d);
  c.take<unsigned>(2);
  c.take<float>(1);
  c.used = round_up(c.used, 256);
  return c.used + dense_ws(nullptr, nN, nM, d, k, SSC_BF16, nullptr);
}

int ssc_dense_coupling_fwd_e4m3(const void* Q, int ldq, const void* K, int ldk, const void* V,
                                int ldv, int nN, int nM, int d, int k, float scale, float* O,
                                int ldo, float* lse, void* ws, size_t ws_bytes,
                                ssc_stream_t stream) {
  int rc = check_common(Q, ldq, K, ldk, V, ldv, nN, nM, d, k, scale, SSC_BF16);
  if (rc) return rc;
  if (d != 128) return SSC_ERR_UNSUPPORTED;
  if ((rc = check_out(O, ldo, k))) return rc;
  if (!lse) return SSC_ERR_INVALID_ARG;
  if (!ws_ok(ws, ws_bytes, ssc_dense_coupling_fwd_e4m3_workspace_size(nN, nM, d, k)))
    return SSC_ERR_WORKSPACE;
  (void)cudaGetLastError();  // clear a stale error left by an earlier, unrelated call
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  WaitCtl ctl = make_ctl();
  Carve c(ws);
  auto* Q8 = c.take<uint8_t>((size_t)nN * d);
  auto* K8 = c.take<uint8_t>((size_t)nM * d);
  auto* amax2 = c.take<unsigned>(2);
  auto* deq = c.take<float>(1);
  c.used = round_up(c.used, 256);
  DenseWs w;
  dense_ws(c.base + c.used, nN, nM, d, k, SSC_BF16, &w);
  cudaError_t e = launch_dense_schedule(nN, nM, w.tiles, w.segs, w.prefix, st);
  if (e != cudaSuccess) return SSC_ERR_CUDA;
  if ((e = launch_quantize_e4m3(static_cast<const __nv_bfloat16*>(Q), ldq, nN,
                                static_cast<const __nv_bfloat16*>(K), ldk, nM, d, Q8, K8, amax2, deq,
                                st)) != cudaSuccess)
    return SSC_ERR_CUDA;
  const __nv_bfloat16* Vt;
  int ldvt;
  if ((e = dense_v(V, ldv, nM, k, w, &Vt, &ldvt, st, ctl.status)) != cudaSuccess) return SSC_ERR_CUDA;
  TcArgs a{reinterpret_cast<const __nv_bfloat16*>(Q8), reinterpret_cast<const __nv_bfloat16*>(K8), Vt,
           d, d, ldvt, nN, nM, d, k, scale, w.tiles, w.segs, nullptr, dense_num_tiles(nN), w.prefix,
           nullptr, nullptr};
  return cuda_status(launch_tc_fwd_e4m3(a, deq, O, ldo, lse, st, ctl));
}

int ssc_dense_coupling_bwd_deterministic(const void* Q, int ldq, const void* K, int ldk,
                                         const void* V, int ldv, int nN, int nM, int d, int k,
                                         float scale, int dtype, const float* O, int ldo,
                                         const float* lse, const float* dO, int lddo, float* dQ,
                                         int lddq, float* dK, int lddk, float* dV, int lddv,
                                         void* ws, size_t ws_bytes, ssc_stream_t stream) {
  // the fp32 check mode is deterministic already (query- and key-stationary, no atomics)
  if (dtype == SSC_F32)
    return ssc_dense_coupling_bwd(Q, ldq, K, ldk, V, ldv, nN, nM, d, k, scale, dtype, O, ldo, lse, dO,
                                  lddo, dQ, lddq, dK, lddk, dV, lddv, ws, ws_bytes, stream);
  int rc = check_common(Q, ldq, K, ldk, V, ldv, nN, nM, d, k, scale, dtype);
  if (rc) return rc;
  if (!O || !lse || !dO || ldo < k || lddo < k) return SSC_ERR_INVALID_ARG;
  if ((rc = check_out(dQ, lddq, d)) || (rc = check_out(dK, lddk, d))) return rc;
  if (dV && (rc = check_out(dV, lddv, k))) return rc;
  if (!ws_ok(ws, ws_bytes, dense_ws(nullptr, nN, nM, d, k, dtype, nullptr))) return SSC_ERR_WORKSPACE;
  (void)cudaGetLastError();  // clear a stale error left by an earlier, unrelated call
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  WaitCtl ctl = make_ctl();
  DenseWs w;
  dense_ws(ws, nN, nM, d, k, dtype, &w);
  cudaError_t e = launch_dense_schedule(nN, nM, w.tiles, w.segs, w.prefix, st);
  if (e != cudaSuccess) return SSC_ERR_CUDA;
  const int kp = (int)kp_of(k);
  // the zeroing of the accumulators and the V re-pack run on the side stream
  // beside the row prep (neither touches what the other reads or writes)
  Side* side;
  cudaStream_t zs;
  if ((e = fork_begin(st, &side, &zs)) != cudaSuccess) return SSC_ERR_CUDA;
  const __nv_bfloat16* Vt = nullptr;
  int ldvt = 0;
  e = zero_matrix(dK, lddk, nM, d, zs);
  if (e == cudaSuccess) e = zero_matrix(dQ, lddq, nN, d, zs);
  if (e == cudaSuccess && dV) e = zero_matrix(dV, lddv, nM, k, zs);
  if (e == cudaSuccess) e = dense_v(V, ldv, nM, k, w, &Vt, &ldvt, zs, ctl.status);
  if (e == cudaSuccess)
    e = launch_bwd_prep(dO, lddo, O, ldo, lse, nullptr, nN, nN, k, w.dOb, kp, nullptr, 0, w.D,
                        nullptr, ctl.status, st);
  const cudaError_t j = fork_end(st, side);
  if (e != cudaSuccess || j != cudaSuccess) return SSC_ERR_CUDA;
  return cuda_status(launch_tc_bwd_deterministic(
      static_cast<const __nv_bfloat16*>(Q), ldq, static_cast<const __nv_bfloat16*>(K), ldk, Vt, ldvt,
      w.dOb, kp, lse, w.D, w.tiles, w.segs, w.prefix, nN, nM, d, k, scale, dQ, lddq, dK, lddk, dV,
      lddv, st, ctl));
}

// ------------------------------------------------------------ geo
size_t ssc_geo_coupling_workspace_size(int nN, int nM, int d, int k, int PN, int PM, int R,
                                       int dtype) {
  if (nN < 1 || nM < 1 || k < 1 || PN < 1 || PM < 1 || R < 1) return 0;
  return geo_ws(nullptr, nN, nM, d, k, PN, PM, R, dtype, nullptr);
}

namespace {

// Gathers Q, K, V into patch-major order and builds the tile schedule.
int geo_setup(const void* Q, int ldq, const void* K, int ldk, const void* V, int ldv, int nN, int nM,
              int d, int k, int dtype, const int* offN, const int* memN, int PN, const int* offM,
              const int* memM, int PM, const int* topk, int R, const GeoWs& w, cudaStream_t st,
              const WaitCtl& ctl) {
  // the gather reads no top-R output: it runs on the side stream beside the schedule
  Side* side;
  cudaStream_t gs;
  cudaError_t e = fork_begin(st, &side, &gs);
  if (e != cudaSuccess) return SSC_ERR_CUDA;
  if (dtype == SSC_BF16) {
    // Q, K and V into patch-major order in one launch
    const __nv_bfloat16* in[3] = {static_cast<const __nv_bfloat16*>(Q),
                                  static_cast<const __nv_bfloat16*>(K),
                                  static_cast<const __nv_bfloat16*>(V)};
    const int in_ld[3] = {ldq, ldk, ldv};
    const int* map[3] = {memN, memM, memM};
    const int rows[3] = {nN, nM, nM};
    const int cols[3] = {d, d, k};
    __nv_bfloat16* out[3] = {static_cast<__nv_bfloat16*>(w.Qp), static_cast<__nv_bfloat16*>(w.Kp),
                             static_cast<__nv_bfloat16*>(w.Vp)};
    const int out_ld[3] = {w.ldq, w.ldk, w.ldv};
    e = launch_gather3_bf16(in, in_ld, map, rows, rows, cols, out, out_ld, ctl.status, gs);
  } else {
    if ((e = launch_gather_rows_f32(static_cast<const float*>(Q), ldq, memN, nN, nN, d,
                                    static_cast<float*>(w.Qp), w.ldq, ctl.status, gs)) == cudaSuccess &&
        (e = launch_gather_rows_f32(static_cast<const float*>(K), ldk, memM, nM, nM, d,
                                    static_cast<float*>(w.Kp), w.ldk, ctl.status, gs)) == cudaSuccess)
      e = launch_gather_rows_f32(static_cast<const float*>(V), ldv, memM, nM, nM, k,
                                 static_cast<float*>(w.Vp), w.ldv, ctl.status, gs);
  }
  if (e == cudaSuccess)
    e = launch_geo_schedule(offN, PN, nN, offM, PM, nM, topk, R, w.tiles, w.segs, w.counts,
                            w.prefix, w.sched_scratch, ctl.status, st, w.tag,
                            geo_fingerprint(Q, K, V, nN, nM, d, k, dtype, offN, memN, PN, offM,
                                            memM, PM, topk, R));
  // joined on every path, so that a captured stream is never left forked
  const cudaError_t j = fork_end(st, side);
  return cuda_status(e != cudaSuccess ? e : j);
}

}  // namespace

namespace {

// The Geo forward once the arguments are checked and the workspace carved.
int geo_fwd_run(const void* Q, int ldq, const void* K, int ldk, const void* V, int ldv, int nN,
                int nM, int d, int k, float scale, int dtype, const int* offN, const int* memN,
                int PN, const int* offM, const int* memM, int PM, const int* topk, int R, float* O,
                int ldo, float* lse, const GeoWs& w, cudaStream_t st, const WaitCtl& ctl) {
  int rc;
  if ((rc = geo_setup(Q, ldq, K, ldk, V, ldv, nN, nM, d, k, dtype, offN, memN, PN, offM, memM, PM,
                      topk, R, w, st, ctl)))
    return rc;
  if (dtype == SSC_F32) {
    SimtArgs a{static_cast<const float*>(w.Qp), static_cast<const float*>(w.Kp),
               static_cast<const float*>(w.Vp), w.ldq, w.ldk, w.ldv, nN, nM, d, k, scale, w.tiles,
               w.segs, w.counts, 0, memN, memM};
    return cuda_status(launch_simt_fwd(a, O, ldo, lse, st));
  }
  TcArgs a{static_cast<const __nv_bfloat16*>(w.Qp), static_cast<const __nv_bfloat16*>(w.Kp),
           static_cast<const __nv_bfloat16*>(w.Vp), w.ldq, w.ldk, w.ldv, nN, nM, d, k, scale,
           w.tiles, w.segs, w.counts, 0, w.prefix, memN, memM};
  return cuda_status(launch_tc_fwd(a, O, ldo, lse, st, ctl));
}

// The Geo backward once the arguments are checked and the workspace carved;
// with reuse the patch-major operands and the schedule are the forward's.
int geo_bwd_run(const void* Q, int ldq, const void* K, int ldk, const void* V, int ldv, int nN,
                int nM, int d, int k, float scale, int dtype, const int* offN, const int* memN,
                int PN, const int* offM, const int* memM, int PM, const int* topk, int R,
                const float* O, int ldo, const float* lse, const float* dO, int lddo, float* dQ,
                int lddq, float* dK, int lddk, float* dV, int lddv, const GeoWs& w,
                cudaStream_t st, const WaitCtl& ctl, bool reuse) {
  int rc;
  if (!reuse && (rc = geo_setup(Q, ldq, K, ldk, V, ldv, nN, nM, d, k, dtype, offN, memN, PN, offM,
                                memM, PM, topk, R, w, st, ctl)))
    return rc;
  // the forward that filled the workspace must be this call's
  const unsigned long long fp =
      reuse ? geo_fingerprint(Q, K, V, nN, nM, d, k, dtype, offN, memN, PN, offM, memM, PM, topk, R)
            : 0;
  cudaError_t e;
  if (dtype == SSC_F32) {
    if (reuse && launch_check_tag(w.tag, fp, ctl.status, st) != cudaSuccess) return SSC_ERR_CUDA;
    e = launch_bwd_prep(dO, lddo, O, ldo, lse, memN, nN, nN, k, nullptr, 0,
                        static_cast<float*>(w.dOp), w.ldg, w.D, w.lsep, ctl.status, st);
    if (e != cudaSuccess) return SSC_ERR_CUDA;
    if ((e = launch_invert_topk(topk, PN, R, PM, w.inv_off, w.inv_p, w.inv_scratch, st)) !=
        cudaSuccess)
      return SSC_ERR_CUDA;
    SimtArgs a{static_cast<const float*>(w.Qp), static_cast<const float*>(w.Kp),
               static_cast<const float*>(w.Vp), w.ldq, w.ldk, w.ldv, nN, nM, d, k, scale, w.tiles,
               w.segs, w.counts, 0, memN, memM};
    if ((e = launch_simt_bwd_dq(a, static_cast<const float*>(w.dOp), w.ldg, w.lsep, w.D, dQ, lddq,
                                st)) != cudaSuccess)
      return SSC_ERR_CUDA;
    SimtKeyArgs g{offM, PM, offN, w.inv_off, w.inv_p, ctl.status};
    return cuda_status(launch_simt_bwd_dkdv(a, g, static_cast<const float*>(w.dOp), w.ldg, w.lsep,
                                            w.D, dK, lddk, dV, lddv, st));
  }
  // dK is reduced in the patch-major key order (contiguous key rows, so TMA
  // reductions apply) and scattered to vertex order afterwards: memM lists
  // every source vertex once, so the scatter writes each row of dK once (with
  // inconsistent tables the results are unspecified, as the header states).
  // The fingerprint check and the zeroing of the accumulators touch nothing
  // that the row prep reads or writes: they run on the side stream beside it.
  Side* side;
  cudaStream_t zs;
  if ((e = fork_begin(st, &side, &zs)) != cudaSuccess) return SSC_ERR_CUDA;
  if (reuse) e = launch_check_tag(w.tag, fp, ctl.status, zs);
  if (e == cudaSuccess) e = zero_matrix(w.dKg, d, nM, d, zs);
  if (e == cudaSuccess) e = zero_matrix(dQ, lddq, nN, d, zs);
  if (e == cudaSuccess && dV) e = zero_matrix(dV, lddv, nM, k, zs);
  if (e == cudaSuccess)
    e = launch_bwd_prep(dO, lddo, O, ldo, lse, memN, nN, nN, k, static_cast<__nv_bfloat16*>(w.dOp),
                        w.ldg, nullptr, 0, w.D, w.lsep, ctl.status, st);
  const cudaError_t j = fork_end(st, side);
  if (e != cudaSuccess || j != cudaSuccess) return SSC_ERR_CUDA;
  TcArgs a{static_cast<const __nv_bfloat16*>(w.Qp), static_cast<const __nv_bfloat16*>(w.Kp),
           static_cast<const __nv_bfloat16*>(w.Vp), w.ldq, w.ldk, w.ldv, nN, nM, d, k, scale,
           w.tiles, w.segs, w.counts, 0, w.prefix, memN, memM};
  if ((e = launch_tc_bwd(a, static_cast<const __nv_bfloat16*>(w.dOp), w.ldg, w.lsep, w.D, dQ, lddq,
                         dK, lddk, dV, lddv, st, ctl, w.dKg)) != cudaSuccess)
    return SSC_ERR_CUDA;
  return cuda_status(launch_scatter_rows_f32(w.dKg, d, memM, nM, nM, d, dK, lddk, ctl.status, st));
}

int geo_bwd(const void* Q, int ldq, const void* K, int ldk, const void* V, int ldv, int nN, int nM,
            int d, int k, float scale, int dtype, const int* offN, const int* memN, int PN,
            const int* offM, const int* memM, int PM, const int* topk, int R, const float* O,
            int ldo, const float* lse, const float* dO, int lddo, float* dQ, int lddq, float* dK,
            int lddk, float* dV, int lddv, void* ws, size_t ws_bytes, ssc_stream_t stream,
            bool reuse) {
  int rc = check_common(Q, ldq, K, ldk, V, ldv, nN, nM, d, k, scale, dtype);
  if (rc) return rc;
  if ((rc = check_patches(offN, memN, PN, nN, offM, memM, PM, nM, topk, R))) return rc;
  if (!O || !lse || !dO || ldo < k || lddo < k) return SSC_ERR_INVALID_ARG;
  if ((rc = check_out(dQ, lddq, d)) || (rc = check_out(dK, lddk, d))) return rc;
  if (dV && (rc = check_out(dV, lddv, k))) return rc;
  if (!ws_ok(ws, ws_bytes, geo_ws(nullptr, nN, nM, d, k, PN, PM, R, dtype, nullptr)))
    return SSC_ERR_WORKSPACE;
  (void)cudaGetLastError();  // clear a stale error left by an earlier, unrelated call
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  WaitCtl ctl = make_ctl();
  GeoWs w;
  geo_ws(ws, nN, nM, d, k, PN, PM, R, dtype, &w);
  return geo_bwd_run(Q, ldq, K, ldk, V, ldv, nN, nM, d, k, scale, dtype, offN, memN, PN, offM,
                     memM, PM, topk, R, O, ldo, lse, dO, lddo, dQ, lddq, dK, lddk, dV, lddv, w, st,
                     ctl, reuse);
}

}  // namespace

int ssc_geo_coupling_fwd(const void* Q, int ldq, const void* K, int ldk, const void* V, int ldv,
                         int nN, int nM, int d, int k, float scale, int dtype, const int* offN,
                         const int* memN, int PN, const int* offM, const int* memM, int PM,
                         const int* topk, int R, float* O, int ldo, float* lse, void* ws,
                         size_t ws_bytes, ssc_stream_t stream) {
  int rc = check_common(Q, ldq, K, ldk, V, ldv, nN, nM, d, k, scale, dtype);
  if (rc) return rc;
  if ((rc = check_patches(offN, memN, PN, nN, offM, memM, PM, nM, topk, R))) return rc;
  if ((rc = check_out(O, ldo, k))) return rc;
  if (!lse) return SSC_ERR_INVALID_ARG;
  if (!ws_ok(ws, ws_bytes, geo_ws(nullptr, nN, nM, d, k, PN, PM, R, dtype, nullptr)))
    return SSC_ERR_WORKSPACE;
  (void)cudaGetLastError();  // clear a stale error left by an earlier, unrelated call
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  WaitCtl ctl = make_ctl();
  GeoWs w;
  geo_ws(ws, nN, nM, d, k, PN, PM, R, dtype, &w);
  return geo_fwd_run(Q, ldq, K, ldk, V, ldv, nN, nM, d, k, scale, dtype, offN, memN, PN, offM, memM,
                     PM, topk, R, O, ldo, lse, w, st, ctl);
}

int ssc_geo_coupling_bwd(const void* Q, int ldq, const void* K, int ldk, const void* V, int ldv,
                         int nN, int nM, int d, int k, float scale, int dtype, const int* offN,
                         const int* memN, int PN, const int* offM, const int* memM, int PM,
                         const int* topk, int R, const float* O, int ldo, const float* lse,
                         const float* dO, int lddo, float* dQ, int lddq, float* dK, int lddk,
                         float* dV, int lddv, void* ws, size_t ws_bytes, ssc_stream_t stream) {
  return geo_bwd(Q, ldq, K, ldk, V, ldv, nN, nM, d, k, scale, dtype, offN, memN, PN, offM, memM, PM,
                 topk, R, O, ldo, lse, dO, lddo, dQ, lddq, dK, lddk, dV, lddv, ws, ws_bytes, stream,
                 false);
}

int ssc_geo_coupling_bwd_reuse(const void* Q, int ldq, const void* K, int ldk, const void* V,
                               int ldv, int nN, int nM, int d, int k, float scale, int dtype,
                               const int* offN, const int* memN, int PN, const int* offM,
                               const int* memM, int PM, const int* topk, int R, const float* O,
                               int ldo, const float* lse, const float* dO, int lddo, float* dQ,
                               int lddq, float* dK, int lddk, float* dV, int lddv, void* ws,
                               size_t ws_bytes, ssc_stream_t stream) {
  return geo_bwd(Q, ldq, K, ldk, V, ldv, nN, nM, d, k, scale, dtype, offN, memN, PN, offM, memM, PM,
                 topk, R, O, ldo, lse, dO, lddo, dQ, lddq, dK, lddk, dV, lddv, ws, ws_bytes, stream,
                 true);
}

// ------------------------------------------------------------ batched pairs
namespace {

// A batch of pairs stored back to back is one problem of batch times the rows:
// Q [batch nN, ldq], K and V [batch nM, ld] as matrices.
bool batch_ok(int batch, int nN, int nM) {
  return batch >= 1 && (long long)batch * nN <= (1 << 30) && (long long)batch * nM <= (1 << 30);
}

struct DenseBatchWs {
  DenseWs w;       // tiles/segs/prefix of the block-diagonal schedule, dOb, Vpad, D
  void* pair_ws;   // fp32 check mode: the single-pair workspace, reused pair after pair
};

size_t dense_batch_ws(void* base, int batch, int nN, int nM, int d, int k, int dtype,
                      DenseBatchWs* out) {
  Carve c(base);
  DenseBatchWs x;
  const int nt = dense_num_tiles(nN), ns = dense_num_segs(nM);
  x.w.tiles = c.take<RowTile>((size_t)batch * nt);
  x.w.segs = c.take<KeySeg>((size_t)batch * ns);
  x.w.prefix = c.take<int>((size_t)batch * nt + 1);
  x.w.dOb = dtype == SSC_BF16 ? c.take<__nv_bfloat16>((size_t)batch * nN * kp_of(k)) : nullptr;
  x.w.Vpad = dtype == SSC_BF16 ? c.take<__nv_bfloat16>((size_t)batch * nM * kp_of(k)) : nullptr;
  x.w.D = c.take<float>((size_t)batch * nN);
  x.w.part = nullptr;
  const size_t pw = dtype == SSC_F32 ? dense_ws(nullptr, nN, nM, d, k, dtype, nullptr) : 0;
  x.pair_ws = c.take<uint8_t>(pw);
  if (out) *out = x;
  return c.used + 256;
}

struct GeoBatchWs {
  int *offN, *memN, *offM, *memM, *topk;  // the concatenated tables
  GeoWs w;
};

size_t geo_batch_ws(void* base, int batch, int nN, int nM, int d, int k, int PN, int PM, int R,
                    int dtype, GeoBatchWs* out) {
  Carve c(base);
  GeoBatchWs x;
  x.offN = c.take<int>((size_t)batch * PN + 1);
  x.memN = c.take<int>((size_t)batch * nN);
  x.offM = c.take<int>((size_t)batch * PM + 1);
  x.memM = c.take<int>((size_t)batch * nM);
  x.topk = c.take<int>((size_t)batch * PN * R);
  c.used = round_up(c.used, 256);
  const size_t g = geo_ws(c.base ? c.base + c.used : nullptr, batch * nN, batch * nM, d, k,
                          batch * PN, batch * PM, R, dtype, &x.w);
  c.used += g;
  if (out) *out = x;
  return c.used + 256;
}

// The batched tables: per-shape offsets and members shifted into one problem.
int geo_batch_tables(int batch, int nN, int nM, const int* offN, const int* memN, int PN,
                     const int* offM, const int* memM, int PM, const int* topk, int R,
                     const GeoBatchWs& b, cudaStream_t st, const WaitCtl& ctl) {
  if (launch_concat_tables(offN, memN, PN, nN, batch, b.offN, b.memN, ctl.status, st) !=
          cudaSuccess ||
      launch_concat_tables(offM, memM, PM, nM, batch, b.offM, b.memM, ctl.status, st) !=
          cudaSuccess ||
      (topk && launch_concat_topk(topk, PN, R, PM, batch, b.topk, ctl.status, st) != cudaSuccess))
    return SSC_ERR_CUDA;
  return SSC_OK;
}

int check_batched_patches(int batch, const int* offN, const int* memN, int PN, int nN,
                          const int* offM, const int* memM, int PM, int nM, const int* topk, int R) {
  if (!batch_ok(batch, nN, nM)) return SSC_ERR_INVALID_ARG;
  int rc = check_patches(offN, memN, PN, nN, offM, memM, PM, nM, topk, R);
  if (rc) return rc;
  if ((long long)batch * PN > 65535 || (long long)batch * PM > 65535) return SSC_ERR_INVALID_ARG;
  return SSC_OK;
}

}  // namespace

size_t ssc_dense_coupling_batched_workspace_size(int batch, int nN, int nM, int d, int k,
                                                 int dtype) {
  if (!batch_ok(batch, nN, nM) || nN < 1 || nM < 1 || k < 1) return 0;
  return dense_batch_ws(nullptr, batch, nN, nM, d, k, dtype, nullptr);
}

int ssc_dense_coupling_fwd_batched(int batch, const void* Q, int ldq, const void* K, int ldk,
                                   const void* V, int ldv, int nN, int nM, int d, int k,
                                   float scale, int dtype, float* O, int ldo, float* lse, void* ws,
                                   size_t ws_bytes, ssc_stream_t stream) {
  if (!batch_ok(batch, nN, nM)) return SSC_ERR_INVALID_ARG;
  int rc = check_common(Q, ldq, K, ldk, V, ldv, nN, nM, d, k, scale, dtype);
  if (rc) return rc;
  if ((rc = check_out(O, ldo, k))) return rc;
  if (!lse) return SSC_ERR_INVALID_ARG;
  if (!ws_ok(ws, ws_bytes, dense_batch_ws(nullptr, batch, nN, nM, d, k, dtype, nullptr)))
    return SSC_ERR_WORKSPACE;
  (void)cudaGetLastError();  // clear a stale error left by an earlier, unrelated call
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DenseBatchWs b;
  dense_batch_ws(ws, batch, nN, nM, d, k, dtype, &b);
  if (dtype == SSC_F32) {
    // check mode: pair after pair through the single-pair call
    const size_t pw = dense_ws(nullptr, nN, nM, d, k, dtype, nullptr);
    const auto* q = static_cast<const float*>(Q);
    const auto* kk = static_cast<const float*>(K);
    const auto* v = static_cast<const float*>(V);
    for (int i = 0; i < batch; ++i)
      if ((rc = ssc_dense_coupling_fwd(q + (size_t)i * nN * ldq, ldq, kk + (size_t)i * nM * ldk, ldk,
                                       v + (size_t)i * nM * ldv, ldv, nN, nM, d, k, scale, dtype,
                                       O + (size_t)i * nN * ldo, ldo, lse + (size_t)i * nN,
                                       b.pair_ws, pw, stream)))
        return rc;
    return SSC_OK;
  }
  WaitCtl ctl = make_ctl();
  cudaError_t e = launch_batched_schedule(batch, nN, nM, b.w.tiles, b.w.segs, b.w.prefix, st);
  if (e != cudaSuccess) return SSC_ERR_CUDA;
  const __nv_bfloat16* Vt;
  int ldvt;
  if ((e = dense_v(V, ldv, batch * nM, k, b.w, &Vt, &ldvt, st, ctl.status)) != cudaSuccess)
    return SSC_ERR_CUDA;
  TcArgs a{static_cast<const __nv_bfloat16*>(Q), static_cast<const __nv_bfloat16*>(K), Vt, ldq, ldk,
           ldvt, batch * nN, batch * nM, d, k, scale, b.w.tiles, b.w.segs, nullptr,
           batch * dense_num_tiles(nN), b.w.prefix, nullptr, nullptr};
  return cuda_status(launch_tc_fwd(a, O, ldo, lse, st, ctl));
}

int ssc_dense_coupling_bwd_batched(int batch, const void* Q, int ldq, const void* K, int ldk,
                                   const void* V, int ldv, int nN, int nM, int d, int k,
                                   float scale, int dtype, const float* O, int ldo,
                                   const float* lse, const float* dO, int lddo, float* dQ,
                                   int lddq, float* dK, int lddk, float* dV, int lddv, void* ws,
                                   size_t ws_bytes, ssc_stream_t stream) {
  if (!batch_ok(batch, nN, nM)) return SSC_ERR_INVALID_ARG;
  int rc = check_common(Q, ldq, K, ldk, V, ldv, nN, nM, d, k, scale, dtype);
  if (rc) return rc;
  if (!O || !lse || !dO || ldo < k || lddo < k) return SSC_ERR_INVALID_ARG;
  if ((rc = check_out(dQ, lddq, d)) || (rc = check_out(dK, lddk, d))) return rc;
  if (dV && (rc = check_out(dV, lddv, k))) return rc;
  if (!ws_ok(ws, ws_bytes, dense_batch_ws(nullptr, batch, nN, nM, d, k, dtype, nullptr)))
    return SSC_ERR_WORKSPACE;
  (void)cudaGetLastError();  // clear a stale error left by an earlier, unrelated call
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  DenseBatchWs b;
  dense_batch_ws(ws, batch, nN, nM, d, k, dtype, &b);
  if (dtype == SSC_F32) {
    const size_t pw = dense_ws(nullptr, nN, nM, d, k, dtype, nullptr);
    const auto* q = static_cast<const float*>(Q);
    const auto* kk = static_cast<const float*>(K);
    const auto* v = static_cast<const float*>(V);
    for (int i = 0; i < batch; ++i)
      if ((rc = ssc_dense_coupling_bwd(
               q + (size_t)i * nN * ldq, ldq, kk + (size_t)i * nM * ldk, ldk, v + (size_t)i * nM * ldv,
               ldv, nN, nM, d, k, scale, dtype, O + (size_t)i * nN * ldo, ldo, lse + (size_t)i * nN,
               dO + (size_t)i * nN * lddo, lddo, dQ + (size_t)i * nN * lddq, lddq,
               dK + (size_t)i * nM * lddk, lddk, dV ? dV + (size_t)i * nM * lddv : nullptr, lddv,
               b.pair_ws, pw, stream)))
        return rc;
    return SSC_OK;
  }
  WaitCtl ctl = make_ctl();
  const int kp = (int)kp_of(k);
  const int rowsN = batch * nN, rowsM = batch * nM;
  cudaError_t e = launch_batched_schedule(batch, nN, nM, b.w.tiles, b.w.segs, b.w.prefix, st);
  if (e != cudaSuccess) return SSC_ERR_CUDA;
  if ((e = launch_bwd_prep(dO, lddo, O, ldo, lse, nullptr, rowsN, rowsN, k, b.w.dOb, kp, nullptr, 0,
                           b.w.D, nullptr, ctl.status, st)) != cudaSuccess)
    return SSC_ERR_CUDA;
  if ((e = zero_matrix(dK, lddk, rowsM, d, st)) != cudaSuccess) return SSC_ERR_CUDA;
  if ((e = zero_matrix(dQ, lddq, rowsN, d, st)) != cudaSuccess) return SSC_ERR_CUDA;
  if (dV && (e = zero_matrix(dV, lddv, rowsM, k, st)) != cudaSuccess) return SSC_ERR_CUDA;
  const __nv_bfloat16* Vt;
  int ldvt;
  if ((e = dense_v(V, ldv, rowsM, k, b.w, &Vt, &ldvt, st, ctl.status)) != cudaSuccess)
    return SSC_ERR_CUDA;
  TcArgs a{static_cast<const __nv_bfloat16*>(Q), static_cast<const __nv_bfloat16*>(K), Vt, ldq, ldk,
           ldvt, rowsN, rowsM, d, k, scale, b.w.tiles, b.w.segs, nullptr,
           batch * dense_num_tiles(nN), b.w.prefix, nullptr, nullptr};
  // dQ and dK (TMA-reduced into the contiguous key rows), dV query-stationary
  return cuda_status(launch_tc_bwd(a, b.w.dOb, kp, lse, b.w.D, dQ, lddq, dK, lddk, dV, lddv, st, ctl));
}

size_t ssc_geo_coupling_batched_workspace_size(int batch, int nN, int nM, int d, int k, int PN,
                                               int PM, int R, int dtype) {
  if (!batch_ok(batch, nN, nM) || nN < 1 || nM < 1 || k < 1 || PN < 1 || PM < 1 || R < 1) return 0;
  return geo_batch_ws(nullptr, batch, nN, nM, d, k, PN, PM, R, dtype, nullptr);
}

int ssc_geo_coupling_fwd_batched(int batch, const void* Q, int ldq, const void* K, int ldk,
                                 const void* V, int ldv, int nN, int nM, int d, int k, float scale,
                                 int dtype, const int* offN, const int* memN, int PN,
                                 const int* offM, const int* memM, int PM, const int* topk, int R,
                                 float* O, int ldo, float* lse, void* ws, size_t ws_bytes,
                                 ssc_stream_t stream) {
  int rc = check_common(Q, ldq, K, ldk, V, ldv, nN, nM, d, k, scale, dtype);
  if (rc) return rc;
  if ((rc = check_batched_patches(batch, offN, memN, PN, nN, offM, memM, PM, nM, topk, R))) return rc;
  if ((rc = check_out(O, ldo, k))) return rc;
  if (!lse) return SSC_ERR_INVALID_ARG;
  if (!ws_ok(ws, ws_bytes, geo_batch_ws(nullptr, batch, nN, nM, d, k, PN, PM, R, dtype, nullptr)))
    return SSC_ERR_WORKSPACE;
  (void)cudaGetLastError();  // clear a stale error left by an earlier, unrelated call
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  WaitCtl ctl = make_ctl();
  GeoBatchWs b;
  geo_batch_ws(ws, batch, nN, nM, d, k, PN, PM, R, dtype, &b);
  if ((rc = geo_batch_tables(batch, nN, nM, offN, memN, PN, offM, memM, PM, topk, R, b, st, ctl)))
    return rc;
  return geo_fwd_run(Q, ldq, K, ldk, V, ldv, batch * nN, batch * nM, d, k, scale, dtype, b.offN,
                     b.memN, batch * PN, b.offM, b.memM, batch * PM, b.topk, R, O, ldo, lse, b.w, st,
                     ctl);
}

int ssc_geo_coupling_bwd_batched(int batch, const void* Q, int ldq, const void* K, int ldk,
                                 const void* V, int ldv, int nN, int nM, int d, int k, float scale,
                                 int dtype, const int* offN, const int* memN, int PN,
                                 const int* offM, const int* memM, int PM, const int* topk, int R,
                                 const float* O, int ldo, const float* lse, const float* dO,
                                 int lddo, float* dQ, int lddq, float* dK, int lddk, float* dV,
                                 int lddv, void* ws, size_t ws_bytes, ssc_stream_t stream) {
  int rc = check_common(Q, ldq, K, ldk, V, ldv, nN, nM, d, k, scale, dtype);
  if (rc) return rc;
  if ((rc = check_batched_patches(batch, offN, memN, PN, nN, offM, memM, PM, nM, topk, R))) return rc;
  if (!O || !lse || !dO || ldo < k || lddo < k) return SSC_ERR_INVALID_ARG;
  if ((rc = check_out(dQ, lddq, d)) || (rc = check_out(dK, lddk, d))) return rc;
  if (dV && (rc = check_out(dV, lddv, k))) return rc;
  if (!ws_ok(ws, ws_bytes, geo_batch_ws(nullptr, batch, nN, nM, d, k, PN, PM, R, dtype, nullptr)))
    return SSC_ERR_WORKSPACE;
  (void)cudaGetLastError();  // clear a stale error left by an earlier, unrelated call
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  WaitCtl ctl = make_ctl();
  GeoBatchWs b;
  geo_batch_ws(ws, batch, nN, nM, d, k, PN, PM, R, dtype, &b);
  if ((rc = geo_batch_tables(batch, nN, nM, offN, memN, PN, offM, memM, PM, topk, R, b, st, ctl)))
    return rc;
  return geo_bwd_run(Q, ldq, K, ldk, V, ldv, batch * nN, batch * nM, d, k, scale, dtype, b.offN,
                     b.memN, batch * PN, b.offM, b.memM, batch * PM, b.topk, R, O, ldo, lse, dO,
                     lddo, dQ, lddq, dK, lddk, dV, lddv, b.w, st, ctl, false);
}

size_t ssc_patch_scores_topk_batched_workspace_size(int batch, int nN, int nM, int PN, int PM,
                                                    int d) {
  if (batch < 1 || nN < 1 || nM < 1 || PN < 1 || PM < 1 || d < 1) return 0;
  Carve c(nullptr);
  c.take<int>((size_t)batch * PN + 1);
  c.take<int>((size_t)batch * nN);
  c.take<int>((size_t)batch * PM + 1);
  c.take<int>((size_t)batch * nM);
  c.used = round_up(c.used, 256);
  return c.used + scores_topk_workspace_bytes(PN, PM, d, batch) + 256;
}

int ssc_patch_scores_topk_batched(int batch, const void* FN, int ldn, int nN, const void* FM,
                                  int ldm, int nM, int d, int dtype, const int* offN,
                                  const int* memN, int PN, const int* offM, const int* memM, int PM,
                                  int R, int* topk, double* scores, void* ws, size_t ws_bytes,
                                  ssc_stream_t stream) {
  if (!FN || !FM || !offN || !memN || !offM || !memM || !topk) return SSC_ERR_INVALID_ARG;
  if (!batch_ok(batch, nN, nM)) return SSC_ERR_INVALID_ARG;
  if (d < 1 || d > 1024 || ldn < d || ldm < d || nN < 1 || nM < 1) return SSC_ERR_INVALID_ARG;
  if (dtype != SSC_BF16 && dtype != SSC_F32) return SSC_ERR_INVALID_ARG;
  if (PN < 1 || PM < 1 || PN > nN || PM > nM || PN > 65535 || PM > 65535) return SSC_ERR_INVALID_ARG;
  if ((long long)batch * PN > (1 << 30) || (long long)batch * PM > (1 << 30)) return SSC_ERR_INVALID_ARG;
  if (R < 1 || R > PM) return SSC_ERR_INVALID_ARG;
  if (!ws_ok(ws, ws_bytes, ssc_patch_scores_topk_batched_workspace_size(batch, nN, nM, PN, PM, d)))
    return SSC_ERR_WORKSPACE;
  (void)cudaGetLastError();  // clear a stale error left by an earlier, unrelated call
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  WaitCtl ctl = make_ctl();
  Carve c(ws);
  GeoBatchWs b;
  b.offN = c.take<int>((size_t)batch * PN + 1);
  b.memN = c.take<int>((size_t)batch * nN);
  b.offM = c.take<int>((size_t)batch * PM + 1);
  b.memM = c.take<int>((size_t)batch * nM);
  c.used = round_up(c.used, 256);
  int rc = geo_batch_tables(batch, nN, nM, offN, memN, PN, offM, memM, PM, nullptr, R, b, st, ctl);
  if (rc) return rc;
  return cuda_status(launch_scores_topk(FN, ldn, nN, FM, ldm, nM, d, dtype, b.offN, b.memN, PN,
                                        b.offM, b.memM, PM, R, topk, scores, c.base + c.used,
                                        ctl.status, st, batch));
}

// ------------------------------------------------------------ linear (ELU)
namespace {

struct LinWs {
  __nv_bfloat16* Vp;  // V re-packed with a pitch of lin_kv(k) when its rows are not 16-byte aligned
  __nv_bfloat16* Y;   // backward rows [dO / den, -D / den]
  float* part;        // per-CTA partial sums of the reductions
  LinWeights w1, w2;  // [KV | z] and [dKV | dz]
};

size_t lin_ws(void* base, int nN, int nM, int k, LinWs* w) {
  Carve c(base);
  LinWs x;
  const int kv = lin_kv(k);
  x.Vp = c.take<__nv_bfloat16>((size_t)nM * kv);
  x.Y = c.take<__nv_bfloat16>((size_t)nN * kv);
  x.part = c.take<float>((size_t)std::max(lin_reduce_grid(nN), lin_reduce_grid(nM)) * 128 * 256);
  for (LinWeights* lw : {&x.w1, &x.w2}) {
    lw->W = c.take<__nv_bfloat16>(128 * 256);
    lw->WT = c.take<__nv_bfloat16>(256 * 128);
    lw->W32 = nullptr;
  }
  if (w) *w = x;
  return c.used + 256;
}

int lin_check(const void* Q, int ldq, const void* K, int ldk, const void* V, int ldv, int nN,
              int nM, int d, int k) {
  if (!Q || !K || !V) return SSC_ERR_INVALID_ARG;
  if (nN < 1 || nM < 1 || k < 1) return SSC_ERR_INVALID_ARG;
  if (d != 64 && d != 128) return SSC_ERR_UNSUPPORTED;
  if (k > 255) return SSC_ERR_UNSUPPORTED;
  if (ldq < d || ldk < d || ldv < k) return SSC_ERR_INVALID_ARG;
  if (!aligned16(Q) || !aligned16(K) || ldq % 8 || ldk % 8) return SSC_ERR_ALIGNMENT;
  if (reinterpret_cast<uintptr_t>(V) & 1u) return SSC_ERR_ALIGNMENT;
  return SSC_OK;
}

// V as the tensor cores read it: in place when its rows are 16-byte aligned,
// else re-packed into the workspace (pitch lin_kv(k), zero padded).
cudaError_t lin_v(const void* V, int ldv, int nM, int k, const LinWs& w, const __nv_bfloat16** Vout,
                  int* ldout, cudaStream_t st, unsigned* status) {
  if (ldv % 8 == 0 && aligned16(V)) {
    *Vout = static_cast<const __nv_bfloat16*>(V);
    *ldout = ldv;
    return cudaSuccess;
  }
  *Vout = w.Vp;
  *ldout = lin_kv(k);
  return launch_gather_rows_bf16(V, ldv, 0, nullptr, nM, nM, k, w.Vp, lin_kv(k), status, st);
}

}  // namespace

size_t ssc_linear_coupling_workspace_size(int nN, int nM, int d, int k) {
  if (nN < 1 || nM < 1 || k < 1 || k > 255 || (d != 64 && d != 128)) return 0;
  return lin_ws(nullptr, nN, nM, k, nullptr);
}

int ssc_linear_coupling_fwd(const void* Q, int ldq, const void* K, int ldk, const void* V, int ldv,
                            int nN, int nM, int d, int k, float* O, int ldo, float* den, void* ws,
                            size_t ws_bytes, ssc_stream_t stream) {
  int rc = lin_check(Q, ldq, K, ldk, V, ldv, nN, nM, d, k);
  if (rc) return rc;
  if ((rc = check_out(O, ldo, k))) return rc;
  if (!den) return SSC_ERR_INVALID_ARG;
  if (!ws_ok(ws, ws_bytes, lin_ws(nullptr, nN, nM, k, nullptr))) return SSC_ERR_WORKSPACE;
  (void)cudaGetLastError();  // clear a stale error left by an earlier, unrelated call
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  WaitCtl ctl = make_ctl();
  LinWs w;
  lin_ws(ws, nN, nM, k, &w);
  const int kv = lin_kv(k);
  const __nv_bfloat16* Vt;
  int ldvt;
  if ((lin_v(V, ldv, nM, k, w, &Vt, &ldvt, st, ctl.status)) != cudaSuccess) return SSC_ERR_CUDA;
  // [KV | z] = phi(K)^T [V | 1]
  if ((launch_lin_reduce(static_cast<const __nv_bfloat16*>(K), ldk, Vt, ldvt, nM, d, k, kv, k,
                             w.part, w.w1, st, ctl)) != cudaSuccess)
    return SSC_ERR_CUDA;
  // O = phi(Q) KV / phi(Q) z
  return cuda_status(launch_lin_rows(0, static_cast<const __nv_bfloat16*>(Q), ldq, d, nN, w.w1.WT,
                                     d, k, kv, 0, -1, nullptr, 0, O, ldo, den, st, ctl));
}

int ssc_linear_coupling_bwd(const void* Q, int ldq, const void* K, int ldk, const void* V, int ldv,
                            int nN, int nM, int d, int k, const float* O, int ldo,
                            const float* den, const float* dO, int lddo, float* dQ, int lddq,
                            float* dK, int lddk, float* dV, int lddv, void* ws, size_t ws_bytes,
                            ssc_stream_t stream) {
  int rc = lin_check(Q, ldq, K, ldk, V, ldv, nN, nM, d, k);
  if (rc) return rc;
  if (!O || !den || !dO || ldo < k || lddo < k) return SSC_ERR_INVALID_ARG;
  if ((rc = check_out(dQ, lddq, d)) || (rc = check_out(dK, lddk, d))) return rc;
  if (dV && (rc = check_out(dV, lddv, k))) return rc;
  if (!ws_ok(ws, ws_bytes, lin_ws(nullptr, nN, nM, k, nullptr))) return SSC_ERR_WORKSPACE;
  (void)cudaGetLastError();  // clear a stale error left by an earlier, unrelated call
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  WaitCtl ctl = make_ctl();
  LinWs w;
  lin_ws(ws, nN, nM, k, &w);
  const int kv = lin_kv(k);
  const auto* Qb = static_cast<const __nv_bfloat16*>(Q);
  const auto* Kb = static_cast<const __nv_bfloat16*>(K);
  const __nv_bfloat16* Vt;
  int ldvt;
  if ((lin_v(V, ldv, nM, k, w, &Vt, &ldvt, st, ctl.status)) != cudaSuccess) return SSC_ERR_CUDA;
  // [KV | z] again (the forward's sums are not kept), then Y and [dKV | dz]
  if ((launch_lin_reduce(Kb, ldk, Vt, ldvt, nM, d, k, kv, k, w.part, w.w1, st, ctl)) !=
          cudaSuccess ||
      (launch_lin_prep(dO, lddo, O, ldo, den, nN, k, w.Y, kv, st)) != cudaSuccess ||
      (launch_lin_reduce(Qb, ldq, w.Y, kv, nN, d, kv, kv, -1, w.part, w.w2, st, ctl)) !=
          cudaSuccess)
    return SSC_ERR_CUDA;
  // dQ = (Y [KV | z]^T) * phi'(Q);  dK = ([V | 1] [dKV | dz]^T) * phi'(K)
  if ((launch_lin_rows(2, w.Y, kv, kv, nN, w.w1.W, d, k, 128, kv / 16, -1, Qb, ldq, dQ, lddq,
                           nullptr, st, ctl)) != cudaSuccess ||
      (launch_lin_rows(2, Vt, ldvt, k, nM, w.w2.W, d, k, 128, kv / 16, k, Kb, ldk, dK, lddk,
                           nullptr, st, ctl)) != cudaSuccess)
    return SSC_ERR_CUDA;
  if (!dV) return SSC_OK;
  // dV = phi(K) dKV
  return cuda_status(launch_lin_rows(1, Kb, ldk, d, nM, w.w2.WT, d, k, (k + 15) / 16 * 16, 0, -1,
                                     nullptr, 0, dV, lddv, nullptr, st, ctl));
}

}  // extern "C"
