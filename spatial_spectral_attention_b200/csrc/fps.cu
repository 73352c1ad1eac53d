// fps.cu -- geodesic farthest-point sampling, nearest-centre assignment and
// the patch tables (offsets + members), bit-exact in fp64.
//
// Source: "Spatial-Spectral Coupling as Attention" digest, "Interpretation"
// (the surface is partitioned with geodesic farthest-point sampling) and the
// project page, "Geo-FlashAttention" (partition both shapes into patches).
// On the unit sphere geodesic distance is the great-circle distance, which
// falls as the dot product rises, so the kernel ranks on the fp64 dot
// ((x0*y0 + x1*y1) + x2*y2) of the fp32 coordinates.
//
// Design: FPS is P dependent rounds (argmax of a running minimum distance), so
// its cost is round latency, not bandwidth.  One thread-block cluster of CL
// CTAs (16 where the GPU allows it) holds every point on chip: coordinates in
// shared memory, the running largest dot and patch of each point in registers.
// Each round a CTA reduces its candidate, pushes it into every CTA's shared
// memory through DSMEM, and one cluster barrier later every CTA knows the next
// centre.  No grid-wide synchronisation.
#include <atomic>
#include <cfloat>
#include <climits>
#include <cooperative_groups.h>

#include "internal.h"
#include "ssc.h"

namespace cg = cooperative_groups;

namespace ssc {
namespace {

constexpr int kFpsThreads = 1024;

struct Cand {
  double val;
  int idx;
};

// a precedes b: smaller largest-dot (farther), ties to the lower vertex.
__device__ __forceinline__ bool cand_before(const Cand& a, const Cand& b) {
  return a.val < b.val || (a.val == b.val && a.idx < b.idx);
}

__device__ __forceinline__ double dot3_rn(float a0, float a1, float a2, float b0, float b1,
                                          float b2) {
  double p0 = __dmul_rn((double)a0, (double)b0);
  double p1 = __dmul_rn((double)a1, (double)b1);
  double p2 = __dmul_rn((double)a2, (double)b2);
  return __dadd_rn(__dadd_rn(p0, p1), p2);
}

__device__ __forceinline__ double dot3_rn(double a0, double a1, double a2, double b0, double b1,
                                          double b2) {
  return __dadd_rn(__dadd_rn(__dmul_rn(a0, b0), __dmul_rn(a1, b1)), __dmul_rn(a2, b2));
}

// Unsigned key that orders like the double (no NaN here): the sign bit is
// flipped for non-negative values, every bit for negative ones; -0 is first
// made +0, since the two compare equal.
__device__ __forceinline__ unsigned long long order_key(double v) {
  const long long b = __double_as_longlong(v + 0.0);
  return b >= 0 ? (unsigned long long)b ^ 0x8000000000000000ull : ~(unsigned long long)b;
}

// The warp's first candidate in cand_before order, agreed by every lane: three
// min reductions (key high word, key low word among the lanes holding the
// smallest high word, vertex index among the lanes holding the smallest key).
__device__ __forceinline__ Cand warp_min(Cand c) {
  const unsigned long long k = order_key(c.val);
  const unsigned hi = (unsigned)(k >> 32), lo = (unsigned)k;
  const unsigned mh = __reduce_min_sync(0xffffffffu, hi);
  const unsigned ml = __reduce_min_sync(0xffffffffu, hi == mh ? lo : 0xffffffffu);
  const bool top = hi == mh && lo == ml;
  const unsigned mi = __reduce_min_sync(0xffffffffu, top ? (unsigned)c.idx : 0xffffffffu);
  const unsigned who = __ballot_sync(0xffffffffu, top && (unsigned)c.idx == mi);
  return Cand{__shfl_sync(0xffffffffu, c.val, __ffs(who) - 1), (int)mi};
}

// A candidate by the order key of its largest dot (order_key, so that the
// integer order is the double order) and its vertex index.
struct KCand {
  unsigned long long key;
  int idx;
};
__device__ __forceinline__ bool kcand_before(const KCand& a, const KCand& b) {
  return a.key < b.key || (a.key == b.key && a.idx < b.idx);
}
// The warp's first candidate, agreed by every lane (three min reductions).
__device__ __forceinline__ KCand warp_min_key(const KCand& c) {
  const unsigned hi = (unsigned)(c.key >> 32), lo = (unsigned)c.key;
  const unsigned mh = __reduce_min_sync(0xffffffffu, hi);
  const unsigned ml = __reduce_min_sync(0xffffffffu, hi == mh ? lo : 0xffffffffu);
  const unsigned mi =
      __reduce_min_sync(0xffffffffu, (hi == mh && lo == ml) ? (unsigned)c.idx : 0xffffffffu);
  return KCand{((unsigned long long)mh << 32) | ml, (int)mi};
}

// A CTA's candidate as it travels through distributed shared memory: its key,
// index and coordinates (so the next round needs no global load).
struct CandXYZ {
  unsigned long long key;
  int idx;
  float x, y, z;
};

// Address of the same shared-memory variable in the CTA of cluster rank `rank`.
__device__ __forceinline__ uint32_t mapa_shared(uint32_t addr, int rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
// 16-byte store into another CTA's shared memory that completes its bytes on
// that CTA's mbarrier (both addresses in the cluster window).
__device__ __forceinline__ void st_async_v4(uint32_t raddr, const uint4& v, uint32_t rbar) {
  asm volatile(
      "st.async.shared::cluster.mbarrier::complete_tx::bytes.v4.b32 [%0], {%1, %2, %3, %4}, [%5];" ::"r"(
          raddr),
      "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w), "r"(rbar)
      : "memory");
}

// Cluster FPS: the CTA of rank r owns points [r*per, min(n,(r+1)*per));
// their coordinates sit in shared memory (structure of arrays), the running
// largest dot (as its order key) and patch of each point in registers (PPT
// points per thread).  A round: every thread updates its points; a thread's
// best candidate, and its warp's, are recomputed only when one of its points
// changed (largest dots only grow, so an unchanged minimum stays the minimum);
// warp 0 reduces the warps' candidates and its lane j stores the CTA's (with
// the point's coordinates) into slot `rank` of CTA j with st.async, which
// completes on CTA j's slot barrier of the round's parity.  Each CTA's warp 0
// then waits on its own barrier (armed once per round for the CL slots: no
// cluster-wide barrier), reduces the slots and publishes the next centre and
// its coordinates in shared memory.  The two slot buffers alternate by round:
// CTA r can store round t + 2 into CTA j's buffer only after receiving CTA j's
// round t + 1 candidate, which CTA j sends after reading its round t slots.
// Every wait is bounded; on expiry the status word records the timeout and
// every CTA leaves its rounds (the others' waits run out in turn).
template <int PPT>
__global__ void __launch_bounds__(kFpsThreads, 1)
    fps_cluster_kernel(const float* __restrict__ pts, int n, int P, int seed, int per,
                       int* __restrict__ centers, int* __restrict__ owner, WaitCtl ctl) {
  cg::cluster_group cluster = cg::this_cluster();
  const int CL = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  extern __shared__ float sx[];  // [3 or 4][PPT * kFpsThreads]: x, y, z (and |x|_1)
  __shared__ KCand warp_c[kFpsThreads / 32];
  __shared__ __align__(16) uint4 slots[2][16][2];  // 32 bytes per CTA: key, idx, x, y, z
  __shared__ uint64_t bar_slot[2];
  __shared__ CandXYZ s_next;
  __shared__ int s_abort;

  const int tid = threadIdx.x;
  const int cap = PPT * kFpsThreads;
  const int v0 = rank * per;
  const int cnt = max(0, min(n - v0, per));
  constexpr bool kFilter = PPT <= 10;
  for (int i = tid; i < cnt; i += kFpsThreads) {
    const float x = pts[3 * (size_t)(v0 + i)], y = pts[3 * (size_t)(v0 + i) + 1],
                z = pts[3 * (size_t)(v0 + i) + 2];
    sx[i] = x;
    sx[cap + i] = y;
    sx[2 * cap + i] = z;
    if (kFilter) sx[3 * cap + i] = fabsf(x) + fabsf(y) + fabsf(z);
  }
  // Per point: the order key of its largest dot so far (comparisons of keys
  // are comparisons of the fp64 values) and its patch.
  unsigned long long bkey[PPT];
  int own[PPT];
  uint32_t chosen = 0;
  // fp32 filter (PPT <= 10): bestf = the largest dot rounded toward -inf.  The
  // exact fp64 dot g of a point and the new centre differs from the fp32 dot
  // ga (fma chain in the same order) by at most 3 roundings of 2^-24 of
  // S = |x0 b0| + |x1 b1| + |x2 b2| <= |x|_1 max_k |b_k| (plus 2^-148 when the
  // products are subnormal); with the margin tol = 2^-20 |x|_1 max_k |b_k| +
  // 2^-126 (which also covers the rounding of ga + tol and of the fp64 sum),
  // ga + tol < bestf implies g < best: the point keeps its best and owner, and
  // the fp64 dot is skipped.  Every other case (including non-finite ga or tol)
  // takes the exact fp64 comparison, so the results are those of the plain
  // fp64 definition.
  float bestf[kFilter ? PPT : 1];
  const unsigned long long key_lowest = order_key(-DBL_MAX);
#pragma unroll
  for (int i = 0; i < PPT; ++i) {
    bkey[i] = key_lowest;
    own[i] = -1;
    if (kFilter) bestf[i] = -INFINITY;
    if (i * kFpsThreads + tid >= cnt) chosen |= 1u << i;  // padding never competes
  }
  if (tid == 0) {
    mbar_init(&bar_slot[0], 1);
    mbar_init(&bar_slot[1], 1);
    s_abort = 0;
    fence_barrier_init();
  }
  __syncthreads();
  cluster.sync();  // every CTA's slot barriers exist before the first remote store
  int c = seed;
  float c0 = __ldg(pts + 3 * (size_t)c), c1 = __ldg(pts + 3 * (size_t)c + 1),
        c2 = __ldg(pts + 3 * (size_t)c + 2);
  KCand mine{~0ull, INT_MAX};  // this thread's best candidate
  for (int t = 0; t < P; ++t) {
    if (rank == 0 && tid == 0) centers[t] = c;
    // arm this round's slot barrier for the CL candidates (they may land first:
    // the barrier's byte count goes below zero until this arrival)
    if (tid == 0 && t + 1 < P) mbar_arrive_expect_tx(&bar_slot[t & 1], 32u * CL);
    bool dirty = t == 0;  // a point of this thread changed: recompute its candidate
    const double d0 = (double)c0, d1 = (double)c1, d2 = (double)c2;
    const float btol = fmaxf(fabsf(c0), fmaxf(fabsf(c1), fabsf(c2))) * 0x1p-20f;
#pragma unroll
    for (int i = 0; i < PPT; ++i) {
      const int li = i * kFpsThreads + tid;
      if (v0 + li == c) {
        chosen |= 1u << i;
        own[i] = t;
        dirty = true;
      }
      if (!(chosen >> i & 1u)) {
        const float x0 = sx[li], x1 = sx[cap + li], x2 = sx[2 * cap + li];
        bool exact = true;
        if (kFilter) {
          const float ga = fmaf(x2, c2, fmaf(x1, c1, x0 * c0));
          const float tol = fmaf(sx[3 * cap + li], btol, FLT_MIN);
          exact = !(ga + tol < bestf[i] && fabsf(ga) + tol <= FLT_MAX);
        }
        if (exact) {
          const double g = dot3_rn((double)x0, (double)x1, (double)x2, d0, d1, d2);
          const unsigned long long gk = order_key(g);
          if (gk > bkey[i]) {
            bkey[i] = gk;
            own[i] = t;
            if (kFilter) bestf[i] = __double2float_rd(g);
            dirty = true;
          }
        }
      }
    }
    if (t + 1 == P) break;
    if (dirty) {
      mine = KCand{~0ull, INT_MAX};
#pragma unroll
      for (int i = 0; i < PPT; ++i) {
        const KCand me{bkey[i], v0 + i * kFpsThreads + tid};
        if (!(chosen >> i & 1u) && kcand_before(me, mine)) mine = me;
      }
    }
    // the warp's candidate (in warp_c across rounds) changes only with a lane's
    if (__any_sync(0xffffffffu, dirty)) {
      const KCand w = warp_min_key(mine);
      if ((tid & 31) == 0) warp_c[tid >> 5] = w;
    }
    __syncthreads();
    if (tid < 32) {
      const KCand w = warp_min_key(warp_c[tid]);
      if (tid < CL) {
        // this CTA's candidate, with its coordinates, into slot `rank` of CTA `tid`
        float x = 0.f, y = 0.f, z = 0.f;
        if (w.idx != INT_MAX) {
          const int li = w.idx - v0;
          x = sx[li];
          y = sx[cap + li];
          z = sx[2 * cap + li];
        }
        const uint32_t ra = mapa_shared(smem_u32(&slots[t & 1][rank][0]), tid);
        const uint32_t rb = mapa_shared(smem_u32(&bar_slot[t & 1]), tid);
        st_async_v4(ra, make_uint4((uint32_t)w.key, (uint32_t)(w.key >> 32), (uint32_t)w.idx,
                                   __float_as_uint(x)),
                    rb);
        st_async_v4(ra + 16, make_uint4(__float_as_uint(y), __float_as_uint(z), 0u, 0u), rb);
      }
      // the CL candidates of this round in this CTA's slots (ties to the lower vertex)
      const bool ok = mbar_wait_cluster(&bar_slot[t & 1], (t >> 1) & 1, ctl, &s_abort);
      KCand x{~0ull, INT_MAX};
      uint4 a = make_uint4(0u, 0u, 0u, 0u), b = a;
      if (ok && tid < CL) {
        a = slots[t & 1][tid][0];
        b = slots[t & 1][tid][1];
        x = KCand{((unsigned long long)a.y << 32) | a.x, (int)a.z};
      }
      const KCand win = warp_min_key(x);
      if (ok && tid < CL && x.idx == win.idx)
        s_next = CandXYZ{x.key, x.idx, __uint_as_float(a.w), __uint_as_float(b.x), __uint_as_float(b.y)};
    }
    __syncthreads();
    if (s_abort) break;  // a wait ran out: leave the rounds (the status word says so)
    c = s_next.idx;
    c0 = s_next.x;
    c1 = s_next.y;
    c2 = s_next.z;
  }
#pragma unroll
  for (int i = 0; i < PPT; ++i) {
    const int li = i * kFpsThreads + tid;
    if (li < cnt) owner[v0 + li] = own[i];
  }
  cluster.sync();  // no CTA leaves while others may still write its slots
}

// Unsigned key that orders like the float (no NaN); -0 is first made +0.
__device__ __forceinline__ unsigned order_key_f(float v) {
  const int b = __float_as_int(v + 0.0f);
  return b >= 0 ? (unsigned)b ^ 0x80000000u : ~(unsigned)b;
}
__device__ __forceinline__ float from_order_key_f(unsigned k) {
  return __int_as_float((int)((k & 0x80000000u) ? (k ^ 0x80000000u) : ~k));
}
// Spreads the 10 low bits of v three apart (bit i to bit 3 i).
__device__ __forceinline__ unsigned spread10(unsigned v) {
  v &= 1023u;
  v = (v | (v << 16)) & 0x030000ffu;
  v = (v | (v << 8)) & 0x0300f00fu;
  v = (v | (v << 4)) & 0x030c30c3u;
  v = (v | (v << 2)) & 0x09249249u;
  return v;
}
// Morton code of a point with 10 bits per axis over the box [lo, lo + 1023 / s].
__device__ __forceinline__ unsigned morton3(float x, float y, float z, const float (&lo)[3],
                                           const float (&s)[3]) {
  const float p[3] = {x, y, z};
  unsigned q[3];
#pragma unroll
  for (int k = 0; k < 3; ++k) q[k] = (unsigned)fminf(fmaxf((p[k] - lo[k]) * s[k], 0.f), 1023.f);
  return spread10(q[0]) | (spread10(q[1]) << 1) | (spread10(q[2]) << 2);
}

// Cluster FPS with spatial culling (8 to 10 points per thread).  At the
// start each CTA sorts its points by Morton code (bitonic sort in shared
// memory) and lays them out so that warp w holds the 32 PPT consecutive points
// [32 PPT w, 32 PPT (w + 1)) of that order: a compact group with a reference
// point g (its centroid) and radius R >= max |p - g| (rounded up).  For every
// point p of the group and the round's centre c, dot(p, c) <= dot(g, c) +
// R |c|.  When that bound plus a margin for its fp32 rounding (and for the
// fp64 dot's) lies below the smallest bestf (largest dot so far, rounded
// toward -inf) of the group's remaining points, no point of the warp can
// change in this round and the warp skips its points; otherwise they are
// updated as in fps_cluster_kernel (fp32 filter, exact fp64 comparison).  The
// results, and the candidate order (largest dot, then original vertex index),
// are those of the plain fp64 definition.  The centre's CTA and slot travel
// with the candidate, so only the thread holding the centre marks it.  The
// candidate exchange is that of fps_cluster_kernel (st.async into every CTA's
// slot, completing on the receiver's barrier, bounded waits).
template <int PPT>
__global__ void __launch_bounds__(kFpsThreads, 1)
    fps_cull_kernel(const float* __restrict__ pts, int n, int P, int seed, int per,
                    int* __restrict__ centers, int* __restrict__ owner, WaitCtl ctl) {
  cg::cluster_group cluster = cg::this_cluster();
  const int CL = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  constexpr int cap = PPT * kFpsThreads;
  constexpr int NS = PPT <= 1 ? 1024 : PPT <= 2 ? 2048 : PPT <= 4 ? 4096 : PPT <= 8 ? 8192 : 16384;
  // Dynamic shared memory: x, y, z, |x|_1 of every slot (floats), then its
  // original vertex (int, -1 for padding).  The sort buffer (NS 64-bit keys)
  // uses the same bytes before they are filled.
  extern __shared__ float sx[];
  int* so = reinterpret_cast<int*>(sx + 4 * cap);
  unsigned long long* sortbuf = reinterpret_cast<unsigned long long*>(sx);
  __shared__ KCand warp_c[kFpsThreads / 32];
  __shared__ int warp_slot[kFpsThreads / 32];
  __shared__ __align__(16) uint4 slots[2][16][2];  // key, idx, x | y, z, slot
  __shared__ uint64_t bar_slot[2];
  __shared__ CandXYZ s_next;
  __shared__ int s_next_rank, s_next_slot;
  __shared__ unsigned s_box[6];
  __shared__ int s_abort;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int v0 = rank * per;
  const int cnt = max(0, min(n - v0, per));
  if (tid == 0) {
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      s_box[k] = 0xffffffffu;
      s_box[3 + k] = 0u;
    }
    s_next_rank = -1;
    s_next_slot = 0;
    s_abort = 0;
    mbar_init(&bar_slot[0], 1);
    mbar_init(&bar_slot[1], 1);
    fence_barrier_init();
  }
  __syncthreads();
  // 1. bounding box of the CTA's points
  {
    unsigned mn[3] = {~0u, ~0u, ~0u}, mx[3] = {0u, 0u, 0u};
    for (int i = tid; i < cnt; i += kFpsThreads)
#pragma unroll
      for (int k = 0; k < 3; ++k) {
        const unsigned kk = order_key_f(pts[3 * (size_t)(v0 + i) + k]);
        mn[k] = min(mn[k], kk);
        mx[k] = max(mx[k], kk);
      }
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      mn[k] = __reduce_min_sync(0xffffffffu, mn[k]);
      mx[k] = __reduce_max_sync(0xffffffffu, mx[k]);
      if (lane == 0) {
        atomicMin(&s_box[k], mn[k]);
        atomicMax(&s_box[3 + k], mx[k]);
      }
    }
  }
  __syncthreads();
  // 2. Morton keys and an ascending bitonic sort of (key << 32 | local index)
  if (cnt > 0) {
    float lo[3], sc[3];
#pragma unroll
    for (int k = 0; k < 3; ++k) {
      lo[k] = from_order_key_f(s_box[k]);
      const float ext = from_order_key_f(s_box[3 + k]) - lo[k];
      sc[k] = ext > 0.f ? 1023.f / ext : 0.f;
    }
    for (int s = tid; s < NS; s += kFpsThreads) {
      unsigned long long e = ~0ull;
      if (s < cnt)
        e = ((unsigned long long)morton3(pts[3 * (size_t)(v0 + s)], pts[3 * (size_t)(v0 + s) + 1],
                                         pts[3 * (size_t)(v0 + s) + 2], lo, sc)
             << 32) |
            (unsigned)s;
      sortbuf[s] = e;
    }
    __syncthreads();
    for (int k = 2; k <= NS; k <<= 1)
      for (int j = k >> 1; j > 0; j >>= 1) {
        for (int i = tid; i < NS; i += kFpsThreads) {
          const int ixj = i ^ j;
          if (ixj > i) {
            const unsigned long long a = sortbuf[i], b = sortbuf[ixj];
            if ((a > b) == ((i & k) == 0)) {
              sortbuf[i] = b;
              sortbuf[ixj] = a;
            }
          }
        }
        __syncthreads();
      }
  }
  // 3. slot (i, tid) = sx index i kFpsThreads + tid holds sorted position
  //    32 PPT warp + 32 i + lane
  int perm[PPT];
#pragma unroll
  for (int i = 0; i < PPT; ++i) {
    const int s = 32 * PPT * warp + 32 * i + lane;
    perm[i] = s < cnt ? (int)(sortbuf[s] & 0xffffffffull) : -1;
  }
  __syncthreads();  // the sort buffer is read; its bytes become the slot arrays
#pragma unroll
  for (int i = 0; i < PPT; ++i) {
    const int li = i * kFpsThreads + tid;
    float x = 0.f, y = 0.f, z = 0.f;
    if (perm[i] >= 0) {
      x = pts[3 * (size_t)(v0 + perm[i])];
      y = pts[3 * (size_t)(v0 + perm[i]) + 1];
      z = pts[3 * (size_t)(v0 + perm[i]) + 2];
    }
    sx[li] = x;
    sx[cap + li] = y;
    sx[2 * cap + li] = z;
    sx[3 * cap + li] = fabsf(x) + fabsf(y) + fabsf(z);
    so[li] = perm[i] >= 0 ? v0 + perm[i] : -1;
    if (perm[i] >= 0 && v0 + perm[i] == seed) {
      s_next_rank = rank;
      s_next_slot = li;
    }
  }
  // 4. the warp's group: centroid g and radius R (rounded up: the fp32
  //    differences, squares, sum and square root stay within 2^-18 of R)
  float gx = 0.f, gy = 0.f, gz = 0.f, gR = 0.f;
  {
    float ax = 0.f, ay = 0.f, az = 0.f, m = 0.f;
#pragma unroll
    for (int i = 0; i < PPT; ++i)
      if (perm[i] >= 0) {
        const int li = i * kFpsThreads + tid;
        ax += sx[li];
        ay += sx[cap + li];
        az += sx[2 * cap + li];
        m += 1.f;
      }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      ax += __shfl_xor_sync(0xffffffffu, ax, o);
      ay += __shfl_xor_sync(0xffffffffu, ay, o);
      az += __shfl_xor_sync(0xffffffffu, az, o);
      m += __shfl_xor_sync(0xffffffffu, m, o);
    }
    if (m > 0.f) {
      gx = ax / m;
      gy = ay / m;
      gz = az / m;
    }
    float r2 = 0.f;
#pragma unroll
    for (int i = 0; i < PPT; ++i)
      if (perm[i] >= 0) {
        const int li = i * kFpsThreads + tid;
        const float dx = sx[li] - gx, dy = sx[cap + li] - gy, dz = sx[2 * cap + li] - gz;
        r2 = fmaxf(r2, fmaf(dz, dz, fmaf(dy, dy, dx * dx)));
      }
    r2 = from_order_key_f(__reduce_max_sync(0xffffffffu, order_key_f(r2)));
    gR = sqrtf(r2) * (1.0f + 0x1p-18f) + FLT_MIN;
  }
  const float g1 = fabsf(gx) + fabsf(gy) + fabsf(gz);
  unsigned long long bkey[PPT];
  int own[PPT];
  float bestf[PPT];
  uint32_t chosen = 0;
  const unsigned long long key_lowest = order_key(-DBL_MAX);
#pragma unroll
  for (int i = 0; i < PPT; ++i) {
    bkey[i] = key_lowest;
    own[i] = -1;
    bestf[i] = -INFINITY;
    if (perm[i] < 0) chosen |= 1u << i;  // padding never competes
  }
  __syncthreads();
  cluster.sync();  // every CTA's slot barriers exist before the first remote store
  int c = seed, c_rank = s_next_rank, c_slot = s_next_slot;
  float c0 = __ldg(pts + 3 * (size_t)c), c1 = __ldg(pts + 3 * (size_t)c + 1),
        c2 = __ldg(pts + 3 * (size_t)c + 2);
  KCand mine{~0ull, INT_MAX};  // this thread's best candidate and its slot
  int mslot = 0;
  float mw = -INFINITY;  // smallest bestf among the warp's remaining points
  for (int t = 0; t < P; ++t) {
    if (rank == 0 && tid == 0) centers[t] = c;
    if (tid == 0 && t + 1 < P) mbar_arrive_expect_tx(&bar_slot[t & 1], 32u * CL);
    bool dirty = t == 0;
    if (c_rank == rank && (c_slot & (kFpsThreads - 1)) == tid) {
#pragma unroll
      for (int i = 0; i < PPT; ++i)
        if (i == c_slot / kFpsThreads) {
          chosen |= 1u << i;
          own[i] = t;
        }
      dirty = true;
    }
    // the group bound: skip the warp when no remaining point can change
    const float cinf = fmaxf(fabsf(c0), fmaxf(fabsf(c1), fabsf(c2)));
    const float cn = sqrtf(fmaf(c2, c2, fmaf(c1, c1, c0 * c0))) * (1.0f + 0x1p-18f);
    const float ub = fmaf(gz, c2, fmaf(gy, c1, gx * c0)) + gR * cn;
    const float um = fmaf(fmaf(g1, cinf, gR * cn), 0x1p-20f, FLT_MIN);
    const bool skip = ub + um < mw && fabsf(ub) + um <= FLT_MAX;
    if (!skip) {
      const double d0 = (double)c0, d1 = (double)c1, d2 = (double)c2;
      const float btol = cinf * 0x1p-20f;
#pragma unroll
      for (int i = 0; i < PPT; ++i) {
        if (chosen >> i & 1u) continue;
        const int li = i * kFpsThreads + tid;
        const float x0 = sx[li], x1 = sx[cap + li], x2 = sx[2 * cap + li];
        const float ga = fmaf(x2, c2, fmaf(x1, c1, x0 * c0));
        const float tol = fmaf(sx[3 * cap + li], btol, FLT_MIN);
        if (ga + tol < bestf[i] && fabsf(ga) + tol <= FLT_MAX) continue;
        const double g = dot3_rn((double)x0, (double)x1, (double)x2, d0, d1, d2);
        const unsigned long long gk = order_key(g);
        if (gk > bkey[i]) {
          bkey[i] = gk;
          own[i] = t;
          bestf[i] = __double2float_rd(g);
          dirty = true;
        }
      }
    }
    if (t + 1 == P) break;
    if (dirty) {
      mine = KCand{~0ull, INT_MAX};
#pragma unroll
      for (int i = 0; i < PPT; ++i) {
        if (chosen >> i & 1u) continue;
        const int li = i * kFpsThreads + tid;
        const KCand me{bkey[i], so[li]};
        if (kcand_before(me, mine)) {
          mine = me;
          mslot = li;
        }
      }
    }
    if (__any_sync(0xffffffffu, dirty)) {
      const KCand w = warp_min_key(mine);
      const unsigned who = __ballot_sync(0xffffffffu, mine.key == w.key && mine.idx == w.idx);
      const int ws = __shfl_sync(0xffffffffu, mslot, __ffs(who) - 1);
      if (lane == 0) {
        warp_c[warp] = w;
        warp_slot[warp] = ws;
      }
      float tb = INFINITY;
#pragma unroll
      for (int i = 0; i < PPT; ++i)
        if (!(chosen >> i & 1u)) tb = fminf(tb, bestf[i]);
      mw = from_order_key_f(__reduce_min_sync(0xffffffffu, order_key_f(tb)));
    }
    __syncthreads();
    if (tid < 32) {
      const KCand w = warp_min_key(warp_c[tid]);
      const unsigned who = __ballot_sync(0xffffffffu, warp_c[tid].key == w.key && warp_c[tid].idx == w.idx);
      const int wslot = warp_slot[__ffs(who) - 1];
      if (tid < CL) {
        // this CTA's candidate, coordinates and slot into slot `rank` of CTA `tid`
        float x = 0.f, y = 0.f, z = 0.f;
        if (w.idx != INT_MAX) {
          x = sx[wslot];
          y = sx[cap + wslot];
          z = sx[2 * cap + wslot];
        }
        const uint32_t ra = mapa_shared(smem_u32(&slots[t & 1][rank][0]), tid);
        const uint32_t rb = mapa_shared(smem_u32(&bar_slot[t & 1]), tid);
        st_async_v4(ra, make_uint4((uint32_t)w.key, (uint32_t)(w.key >> 32), (uint32_t)w.idx,
                                   __float_as_uint(x)),
                    rb);
        st_async_v4(ra + 16, make_uint4(__float_as_uint(y), __float_as_uint(z), (uint32_t)wslot, 0u),
                    rb);
      }
      const bool ok = mbar_wait_cluster(&bar_slot[t & 1], (t >> 1) & 1, ctl, &s_abort);
      KCand x{~0ull, INT_MAX};
      uint4 a = make_uint4(0u, 0u, 0u, 0u), b = a;
      if (ok && tid < CL) {
        a = slots[t & 1][tid][0];
        b = slots[t & 1][tid][1];
        x = KCand{((unsigned long long)a.y << 32) | a.x, (int)a.z};
      }
      const KCand win = warp_min_key(x);
      if (ok && tid < CL && x.idx == win.idx) {
        s_next = CandXYZ{x.key, x.idx, __uint_as_float(a.w), __uint_as_float(b.x), __uint_as_float(b.y)};
        s_next_rank = tid;
        s_next_slot = (int)b.z;
      }
    }
    __syncthreads();
    if (s_abort) break;  // a wait ran out: leave the rounds (the status word says so)
    c = s_next.idx;
    c0 = s_next.x;
    c1 = s_next.y;
    c2 = s_next.z;
    c_rank = s_next_rank;
    c_slot = s_next_slot;
  }
#pragma unroll
  for (int i = 0; i < PPT; ++i) {
    const int li = i * kFpsThreads + tid;
    if (so[li] >= 0) owner[so[li]] = own[i];
  }
  cluster.sync();  // no CTA leaves while others may still write its slots
}

// Fallback for n beyond what the cluster holds on chip: the same rounds with
// the per-point state in global memory.
__global__ void __launch_bounds__(kFpsThreads, 1)
    fps_cluster_mem_kernel(const float* __restrict__ pts, int n, int P, int seed,
                           int* __restrict__ centers, int* __restrict__ owner,
                           double* __restrict__ best, unsigned char* __restrict__ chosen) {
  cg::cluster_group cluster = cg::this_cluster();
  const int CL = (int)cluster.num_blocks();
  const int rank = (int)cluster.block_rank();
  __shared__ Cand warp_c[kFpsThreads / 32];
  __shared__ Cand slots[2][16];
  __shared__ int s_next;
  const int tid = threadIdx.x;
  const int stride = CL * kFpsThreads;
  for (int v = rank * kFpsThreads + tid; v < n; v += stride) {
    best[v] = -DBL_MAX;
    chosen[v] = 0;
    owner[v] = -1;
  }
  int c = seed;
  for (int t = 0; t < P; ++t) {
    if (rank == 0 && tid == 0) centers[t] = c;
    const float c0 = __ldg(pts + 3 * (size_t)c), c1 = __ldg(pts + 3 * (size_t)c + 1),
                c2 = __ldg(pts + 3 * (size_t)c + 2);
    Cand mine{DBL_MAX, INT_MAX};
    for (int v = rank * kFpsThreads + tid; v < n; v += stride) {
      if (v == c) {
        chosen[v] = 1;
        owner[v] = t;
      }
      if (!chosen[v]) {
        double g = dot3_rn(pts[3 * (size_t)v], pts[3 * (size_t)v + 1], pts[3 * (size_t)v + 2], c0,
                           c1, c2);
        double b = best[v];
        if (g > b) {
          b = g;
          best[v] = g;
          owner[v] = t;
        }
        Cand me{b, v};
        if (cand_before(me, mine)) mine = me;
      }
    }
    if (t + 1 == P) break;
    mine = warp_min(mine);
    if ((tid & 31) == 0) warp_c[tid >> 5] = mine;
    __syncthreads();
    if (tid < 32) {
      Cand w = warp_min(warp_c[tid]);
      if (tid < CL) {
        Cand* dst = cluster.map_shared_rank(&slots[t & 1][rank], tid);
        dst->val = w.val;
        dst->idx = w.idx;
      }
    }
    cluster.sync();
    if (tid < 32) {
      Cand w{DBL_MAX, INT_MAX};
      if (tid < CL) w = slots[t & 1][tid];
      w = warp_min(w);
      if (tid == 0) s_next = w.idx;
    }
    __syncthreads();
    c = s_next;
  }
  cluster.sync();
}

// ---- patch tables
__global__ void count_kernel(const int* __restrict__ owner, int n, int* __restrict__ counts) {
  for (int v = blockIdx.x * blockDim.x + threadIdx.x; v < n; v += gridDim.x * blockDim.x)
    atomicAdd(counts + owner[v], 1);
}

// Single-block exclusive scan: offsets[0] = 0, offsets[p+1] = sum counts[0..p].
__global__ void __launch_bounds__(1024) scan_offsets_kernel(const int* __restrict__ counts, int P,
                                                            int* __restrict__ offsets,
                                                            int* __restrict__ cursor) {
  __shared__ int part[1024];
  const int tid = threadIdx.x;
  const int per = (P + 1023) / 1024;
  const int b = tid * per, e = min(P, b + per);
  int s = 0;
  for (int p = b; p < e; ++p) s += counts[p];
  part[tid] = s;
  __syncthreads();
  for (int o = 1; o < 1024; o <<= 1) {
    int x = tid >= o ? part[tid - o] : 0;
    __syncthreads();
    part[tid] += x;
    __syncthreads();
  }
  int run = part[tid] - s;
  for (int p = b; p < e; ++p) {
    offsets[p] = run;
    cursor[p] = run;
    run += counts[p];
  }
  if (tid == 1023) offsets[P] = part[1023];
}

__global__ void fill_kernel(const int* __restrict__ owner, int n, int* __restrict__ cursor,
                            int* __restrict__ members) {
  for (int v = blockIdx.x * blockDim.x + threadIdx.x; v < n; v += gridDim.x * blockDim.x)
    members[atomicAdd(cursor + owner[v], 1)] = v;
}

constexpr int kSortCap = 4096;

// Puts the members of every patch in ascending vertex order: a bitonic sort in
// shared memory for patches up to kSortCap vertices, an ordered compaction of
// the owner array for larger ones (there are at most n / kSortCap of those).
__global__ void __launch_bounds__(512) sort_segments_kernel(const int* __restrict__ owner, int n,
                                                            const int* __restrict__ offsets,
                                                            int* __restrict__ members) {
  __shared__ int buf[kSortCap];
  __shared__ int warp_tot[16];
  const int p = blockIdx.x;
  const int b = offsets[p], len = offsets[p + 1] - b;
  const int tid = threadIdx.x;
  if (len <= 1) return;
  if (len <= kSortCap) {
    int m = 1;
    while (m < len) m <<= 1;
    for (int i = tid; i < m; i += blockDim.x) buf[i] = i < len ? members[b + i] : INT_MAX;
    __syncthreads();
    for (int size = 2; size <= m; size <<= 1) {
      for (int stride = size >> 1; stride > 0; stride >>= 1) {
        for (int i = tid; i < m; i += blockDim.x) {
          int j = i ^ stride;
          if (j > i) {
            bool up = (i & size) == 0;
            int a = buf[i], c = buf[j];
            if ((a > c) == up) {
              buf[i] = c;
              buf[j] = a;
            }
          }
        }
        __syncthreads();
      }
    }
    for (int i = tid; i < len; i += blockDim.x) members[b + i] = buf[i];
    return;
  }
  // ordered compaction over all vertices
  int base = b;
  for (int v0 = 0; v0 < n; v0 += blockDim.x) {
    int v = v0 + tid;
    int flag = (v < n && owner[v] == p) ? 1 : 0;
    unsigned bal = __ballot_sync(0xffffffffu, flag);
    int lane = tid & 31, w = tid >> 5;
    if (lane == 0) warp_tot[w] = __popc(bal);
    __syncthreads();
    int before = 0, total = 0;
    for (int i = 0; i < (int)(blockDim.x / 32); ++i) {
      if (i < w) before += warp_tot[i];
      total += warp_tot[i];
    }
    if (flag) members[base + before + __popc(bal & ((1u << lane) - 1u))] = v;
    base += total;
    __syncthreads();
  }
}

std::atomic<int> g_cl_forced{0};

// 16-CTA clusters where the device allows non-portable cluster sizes, else 8
// (the query runs once, thread-safely, on first use; a forced size wins).
int fps_cluster_size() {
  const int forced = g_cl_forced.load(std::memory_order_relaxed);
  if (forced) return forced;
  static const int cl = [] {
    const int r = cudaFuncSetAttribute(fps_cluster_kernel<1>,
                                       cudaFuncAttributeNonPortableClusterSizeAllowed, 1) ==
                          cudaSuccess
                      ? 16
                      : 8;
    cudaGetLastError();
    return r;
  }();
  return cl;
}

template <int PPT>
cudaError_t launch_reg(const float* pts, int n, int P, int seed, int* centers, int* owner, int CL,
                       cudaStream_t st, const WaitCtl& ctl) {
  // 8 to 10 points per thread: the culling kernel (x, y, z, |x|_1 and the
  // original vertex per slot).  With fewer points per thread a round is bound
  // by the candidate exchange, not by the point updates, and the sort and the
  // per-warp bound did not pay (60k on 16 CTAs: 1.59 vs 1.47 us per round);
  // beyond 10 the culling kernel's state does not fit in shared memory.
  constexpr bool kCull = PPT >= 8 && PPT <= 10;
  void (*kern)(const float*, int, int, int, int, int*, int*, WaitCtl);
  if constexpr (kCull) kern = fps_cull_kernel<PPT>;
  else kern = fps_cluster_kernel<PPT>;
  // floats per slot: culling kernel 5 (x, y, z, |x|_1, vertex); cluster kernel
  // 4 with its fp32 filter (PPT <= 10: x, y, z, |x|_1), else 3
  const int smem = (kCull ? 5 : (PPT <= 10 ? 4 : 3)) * PPT * kFpsThreads * (int)sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  if (CL > 8) cudaFuncSetAttribute(kern, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
  const int per = (n + CL - 1) / CL;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(CL);
  cfg.blockDim = dim3(kFpsThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = CL;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  count_launch();
  prof_launch_begin(st);
  e = cudaLaunchKernelEx(&cfg, kern, pts, n, P, seed, per, centers, owner, ctl);
  prof_launch_end(st, SSC_PROF_FPS);
  return e;
}

}  // namespace

void fps_force_cluster_size(int cl) {
  g_cl_forced.store(cl == 8 || cl == 16 ? cl : 0, std::memory_order_relaxed);
}

size_t fps_workspace_bytes(int n, int P) {
  Carve c(nullptr);
  c.take<int>(P);       // counts
  c.take<int>(P);       // cursor
  c.take<double>(n);    // best (memory-resident fallback)
  c.take<uint8_t>(n);   // chosen
  return c.used + 256;
}

cudaError_t launch_fps_patches(const float* pts, int n, int P, int seed, int* centers, int* owner,
                               int* offsets, int* members, void* ws, cudaStream_t st,
                               const WaitCtl& ctl) {
  Carve c(ws);
  int* counts = c.take<int>(P);
  int* cursor = c.take<int>(P);
  double* best = c.take<double>(n);
  uint8_t* chosen = c.take<uint8_t>(n);
  int CL = fps_cluster_size();
  if (CL == 16) {
    // make sure a 16-CTA cluster of this shape can be resident, else use 8
    cudaLaunchConfig_t q = {};
    q.gridDim = dim3(16);
    q.blockDim = dim3(kFpsThreads);
    q.dynamicSmemBytes = 3 * 16 * kFpsThreads * sizeof(float);
    cudaLaunchAttribute qa[1];
    qa[0].id = cudaLaunchAttributeClusterDimension;
    qa[0].val.clusterDim.x = 16;
    qa[0].val.clusterDim.y = 1;
    qa[0].val.clusterDim.z = 1;
    q.attrs = qa;
    q.numAttrs = 1;
    int nclusters = 0;
    cudaFuncSetAttribute(fps_cluster_kernel<16>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                         (int)q.dynamicSmemBytes);
    cudaFuncSetAttribute(fps_cluster_kernel<16>, cudaFuncAttributeNonPortableClusterSizeAllowed, 1);
    if (cudaOccupancyMaxActiveClusters(&nclusters, fps_cluster_kernel<16>, &q) != cudaSuccess ||
        nclusters < 1)
      CL = 8;
    cudaGetLastError();
  }
  const long per = (n + CL - 1) / CL;
  const long ppt = (per + kFpsThreads - 1) / kFpsThreads;
  cudaError_t e;
  if (ppt <= 1) e = launch_reg<1>(pts, n, P, seed, centers, owner, CL, st, ctl);
  else if (ppt <= 2) e = launch_reg<2>(pts, n, P, seed, centers, owner, CL, st, ctl);
  else if (ppt <= 4) e = launch_reg<4>(pts, n, P, seed, centers, owner, CL, st, ctl);
  else if (ppt <= 8) e = launch_reg<8>(pts, n, P, seed, centers, owner, CL, st, ctl);
  else if (ppt <= 10) e = launch_reg<10>(pts, n, P, seed, centers, owner, CL, st, ctl);
  else if (ppt <= 16) e = launch_reg<16>(pts, n, P, seed, centers, owner, CL, st, ctl);
  else {
    if (CL > 8)
      cudaFuncSetAttribute(fps_cluster_mem_kernel, cudaFuncAttributeNonPortableClusterSizeAllowed,
                           1);
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(CL);
    cfg.blockDim = dim3(kFpsThreads);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = CL;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    count_launch();
    prof_launch_begin(st);
    e = cudaLaunchKernelEx(&cfg, fps_cluster_mem_kernel, pts, n, P, seed, centers, owner, best,
                           chosen);
    prof_launch_end(st, SSC_PROF_FPS);
  }
  if (e != cudaSuccess) return e;
  return launch_patch_tables(owner, n, P, offsets, members, counts, cursor, st);
}

cudaError_t launch_patch_tables(const int* owner, int n, int P, int* offsets, int* members,
                                int* counts, int* cursor, cudaStream_t st) {
  cudaError_t e;
  if ((e = cudaMemsetAsync(counts, 0, sizeof(int) * P, st)) != cudaSuccess) return e;
  const int nb = (int)std::min<long>(1184, (n + 255) / 256);
  count_kernel<<<nb, 256, 0, st>>>(owner, n, counts);
  count_launch();
  scan_offsets_kernel<<<1, 1024, 0, st>>>(counts, P, offsets, cursor);
  count_launch();
  fill_kernel<<<nb, 256, 0, st>>>(owner, n, cursor, members);
  count_launch();
  sort_segments_kernel<<<P, 512, 0, st>>>(owner, n, offsets, members);
  count_launch();
  return cudaGetLastError();
}

}  // namespace ssc
