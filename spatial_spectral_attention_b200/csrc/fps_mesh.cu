// fps_mesh.cu -- geodesic farthest-point sampling and nearest-centre patches
// on a triangle-mesh graph, bit-exact in fp64.
//
// Source: ai4snews digest of "Spatial-Spectral Coupling as Attention",
// "Interpretation" (the surface is partitioned with geodesic farthest-point
// sampling) and the project page, "Geo-FlashAttention" (geodesic patches).
// The geodesic distance is the shortest path along mesh edges: the edge
// lengths of a path added in fp64 from the source outward, minimised over
// paths.  Next centre = the vertex farthest from its nearest centre (ties to
// the lowest index); a vertex joins its nearest centre (ties to the lowest
// patch index: a later centre takes a vertex only when strictly nearer).
//
// Design.  FPS is P dependent rounds; after round t only the vertices that
// the new centre reaches strictly sooner than every earlier centre change.
// One CTA of 1024 threads keeps the running distance of every vertex in
// memory (fp64 bit patterns: for non-negative values the unsigned order is
// the numeric order, so a 64-bit atomicMin lowers a distance) and relaxes
// outward from the new centre, hop by hop, through frontier queues (a stamp
// per vertex keeps each vertex once per queue).  Label-correcting relaxation
// reaches the same fixpoint as Dijkstra's label setting because adding a
// non-negative fp64 length is monotone and never decreases a value, so the
// distances, and every comparison made on them, are bit-identical to the
// definition.  The round ends with a block-wide argmax.  One barrier per hop
// (three queue counters rotate, so the counter a hop appends to was reset a
// barrier earlier).  Within a hop the edges of a frontier vertex are split
// over eight threads and each edge costs one atomicMin; queue membership is a
// bit in shared memory, so the hop's dependent chain is a handful of L2 trips.
#include <cfloat>
#include <climits>

#include "internal.h"
#include "ssc.h"

namespace ssc {
namespace {

constexpr int kMeshThreads = 1024;
constexpr int kEdgeLanes = 8;  // threads per frontier vertex (its edges are split over them)
constexpr unsigned long long kInfBits = 0x7ff0000000000000ull;  // +inf
// Vertex counts up to this keep the queue marks in shared memory (two bit
// masks); larger meshes mark with stamps in global memory.
constexpr int kSmemMarkMaxN = 1 << 19;  // 2 x 64 KB of marks

__device__ __forceinline__ double dist_of(const unsigned long long* dist, int v) {
  return __longlong_as_double((long long)__ldcg(dist + v));
}

// SMEM_MARK: queue membership in two shared-memory bit masks (alternating by
// hop, the one for the hop after next cleared during the current hop); else in
// a global stamp per vertex (unique per hop).
template <bool SMEM_MARK>
__global__ void __launch_bounds__(kMeshThreads, 1)
    fps_mesh_kernel(const int* __restrict__ off, const int* __restrict__ adj,
                    const double* __restrict__ w, int n, int nnz, int P, int seed,
                    int* __restrict__ centers, int* __restrict__ owner,
                    unsigned long long* __restrict__ dist, int* __restrict__ qa,
                    int* __restrict__ qb, int* __restrict__ stamp, int* __restrict__ bucket,
                    unsigned* status) {
  extern __shared__ unsigned s_mark[];  // [2][words] when SMEM_MARK
  __shared__ int s_cnt[3];
  __shared__ double s_wv[kMeshThreads / 32];
  __shared__ int s_wi[kMeshThreads / 32];
  __shared__ int s_c;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int words = (n + 31) >> 5;
  for (int v = tid; v < n; v += kMeshThreads) {
    dist[v] = kInfBits;
    owner[v] = -1;
    if (!SMEM_MARK) stamp[v] = 0;
  }
  if (tid < 3) s_cnt[tid] = 0;
  int c = seed;
  int sid = 0;  // global-stamp variant: stamp of the current queue (unique over the run)
  bool bad = false;
  for (int t = 0; t < P; ++t) {
    if (SMEM_MARK)
      for (int i = tid; i < 2 * words; i += kMeshThreads) s_mark[i] = 0u;
    __syncthreads();  // previous round (and the marks) done
    // ---- start the round at the new centre (only when it is not a centre yet)
    if (tid == 0) {
      centers[t] = c;
      s_cnt[0] = 0;
      if (__ldcg(dist + c) > 0ull) {
        dist[c] = 0ull;
        owner[c] = t;
        qa[0] = c;
        s_cnt[0] = 1;
      }
      s_cnt[1] = 0;
      s_cnt[2] = 0;
    }
    __syncthreads();
    int* cur = qa;
    int* nxt = qb;
    for (int hop = 0;; ++hop) {
      const int cnt = s_cnt[hop % 3];
      if (cnt == 0) break;
      if (hop > n) {  // cannot happen: every shortest path has fewer than n edges
        bad = true;
        break;
      }
      ++sid;
      if (tid == 0) s_cnt[(hop + 2) % 3] = 0;  // next appended to two hops on
      unsigned* mark = s_mark + (hop & 1) * words;
      if (SMEM_MARK) {
        unsigned* later = s_mark + ((hop + 1) & 1) * words;  // used by the next hop
        for (int i = tid; i < words; i += kMeshThreads) later[i] = 0u;
      }
      // frontier vertex i / kEdgeLanes, its edges split over kEdgeLanes threads
      for (int i = tid; i < cnt * kEdgeLanes; i += kMeshThreads) {
        const int v = __ldcg(cur + i / kEdgeLanes);
        const int slot = i % kEdgeLanes;
        const double dv = dist_of(dist, v);
        int e0 = off[v], e1 = off[v + 1];
        if (e0 < 0 || e1 > nnz || e1 < e0) {
          bad = true;
          e0 = max(0, min(e0, nnz));
          e1 = max(e0, min(e1, nnz));
        }
        for (int e = e0 + slot; e < e1; e += kEdgeLanes) {
          const int u = adj[e];
          const double we = w[e];
          if (u < 0 || u >= n || !(we >= 0.0)) {
            bad = true;
            continue;
          }
          const unsigned long long nb = (unsigned long long)__double_as_longlong(__dadd_rn(dv, we));
          const unsigned long long old = atomicMin(dist + u, nb);
          if (nb < old) {
            owner[u] = t;
            bool fresh;
            if (SMEM_MARK) {
              const unsigned bit = 1u << (u & 31);
              fresh = !(atomicOr(mark + (u >> 5), bit) & bit);
            } else {
              fresh = atomicExch(stamp + u, sid) != sid;
            }
            if (fresh) nxt[atomicAdd(&s_cnt[(hop + 1) % 3], 1)] = u;
          }
        }
      }
      __syncthreads();
      int* tmp = cur;
      cur = nxt;
      nxt = tmp;
    }
    if (t + 1 == P) break;
    // ---- next centre: the largest distance, ties to the lowest vertex index
    // (four independent loads in flight per thread; within a thread the
    // vertices are visited in ascending order and the first maximum is kept)
    double bv = -1.0;
    int bi = INT_MAX;
    for (int v0 = tid; v0 < n; v0 += 4 * kMeshThreads) {
      double dd[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int v = v0 + u * kMeshThreads;
        dd[u] = v < n ? dist_of(dist, v) : -1.0;
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (dd[u] > bv) {
          bv = dd[u];
          bi = v0 + u * kMeshThreads;
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
      if (ov > bv || (ov == bv && oi < bi)) {
        bv = ov;
        bi = oi;
      }
    }
    if (lane == 0) {
      s_wv[warp] = bv;
      s_wi[warp] = bi;
    }
    __syncthreads();
    if (warp == 0) {
      bv = s_wv[lane];
      bi = s_wi[lane];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const double ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) {
          bv = ov;
          bi = oi;
        }
      }
      if (lane == 0) s_c = bi;
    }
    __syncthreads();
    c = s_c;
  }
  __syncthreads();
  // patch of every vertex for the tables: vertices no centre reaches (owner
  // -1) go to a trailing bucket P, listed after the last patch
  for (int v = tid; v < n; v += kMeshThreads) {
    const int o = owner[v];
    bucket[v] = o < 0 ? P : o;
  }
  if (bad && status) atomicOr(status, kStatusBadIndex);
}

}  // namespace

size_t fps_mesh_workspace_bytes(int n, int P) {
  Carve c(nullptr);
  c.take<unsigned long long>(n);  // running distances
  c.take<int>(n);                 // frontier queues
  c.take<int>(n);
  c.take<int>(n);                 // queue stamps
  c.take<int>(n);                 // patch of each vertex, unreached vertices in bucket P
  c.take<int>(P + 1);             // patch counts (with the bucket of unreached vertices)
  c.take<int>(P + 1);             // fill cursors
  c.take<int>(P + 2);             // offsets with the bucket
  return c.used + 256;
}

cudaError_t launch_fps_mesh(const int* off, const int* adj, const double* w, int n, int nnz, int P,
                            int seed, int* centers, int* owner, int* offsets, int* members,
                            void* ws, cudaStream_t st, const WaitCtl& ctl) {
  Carve c(ws);
  auto* dist = c.take<unsigned long long>(n);
  int* qa = c.take<int>(n);
  int* qb = c.take<int>(n);
  int* stamp = c.take<int>(n);
  int* bucket = c.take<int>(n);
  int* counts = c.take<int>(P + 1);
  int* cursor = c.take<int>(P + 1);
  int* off_b = c.take<int>(P + 2);
  count_launch();
  cudaError_t e;
  prof_launch_begin(st);
  if (n <= kSmemMarkMaxN) {
    const int smem = 2 * ((n + 31) / 32) * (int)sizeof(unsigned);
    if ((e = cudaFuncSetAttribute(fps_mesh_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                  smem)) != cudaSuccess)
      return e;
    fps_mesh_kernel<true><<<1, kMeshThreads, smem, st>>>(off, adj, w, n, nnz, P, seed, centers, owner,
                                                         dist, qa, qb, stamp, bucket, ctl.status);
  } else {
    fps_mesh_kernel<false><<<1, kMeshThreads, 0, st>>>(off, adj, w, n, nnz, P, seed, centers, owner,
                                                       dist, qa, qb, stamp, bucket, ctl.status);
  }
  prof_launch_end(st, SSC_PROF_FPS);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // tables over P + 1 buckets; offsets [0, P] are the patches' (offsets[P] =
  // vertices reached), members the full permutation
  if ((e = launch_patch_tables(bucket, n, P + 1, off_b, members, counts, cursor, st)) != cudaSuccess)
    return e;
  return cudaMemcpyAsync(offsets, off_b, sizeof(int) * (size_t)(P + 1), cudaMemcpyDeviceToDevice, st);
}

}  // namespace ssc
