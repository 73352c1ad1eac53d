// patch_topk.cu -- patch pooling, patch scores and top-R source patches.
//
// Source: "Spatial-Spectral Coupling as Attention", project page, section
// "Geo-FlashAttention": pool source keys, score source patches using the
// descriptors and keep the top R per target patch.  Pooling is the mean
// descriptor of a patch; the score of (target p, source q) is the dot product
// of the two means.  All arithmetic is fp64 in a fixed order with explicit
// round-to-nearest intrinsics (no FMA contraction), so the results are
// bit-identical to the plain definition evaluated in the same order:
//   mean: sum over the patch's members in ascending vertex order, one divide;
//   score: sum over c = 0..d-1 of mu_N(p)_c * mu_M(q)_c, in order.
// Top R: the R best q by (score descending, q ascending).
//
// Bound: pooling reads each descriptor once (HBM); scores are a small fp64
// product (PN*PM*d multiply-adds); selection re-reads one score row per round.
#include <cfloat>
#include <climits>

#include "internal.h"

namespace ssc {
namespace {

template <bool F32>
__device__ __forceinline__ double load_elem(const void* F, size_t i) {
  if constexpr (F32) return (double)static_cast<const float*>(F)[i];
  else return (double)__bfloat162float(static_cast<const __nv_bfloat16*>(F)[i]);
}

// One block per patch, one thread per descriptor channel; the member indices
// are staged in shared memory and each thread issues the loads of kPoolBatch
// members before adding them, in member order (the fixed summation order keeps
// the result bit-exact; only the loads run ahead).
// Offsets are clamped into [0, n] and member indices outside [0, n) skipped;
// either sets the bad-index bit of the status word.
constexpr int kPoolStage = 1024;  // member indices staged per round
constexpr int kPoolBatch = 32;    // loads in flight per thread
template <bool F32>
__global__ void pool_kernel(const void* __restrict__ F, int ld, int n, int d,
                            const int* __restrict__ off, const int* __restrict__ mem,
                            double* __restrict__ mu, unsigned* status) {
  __shared__ int s_mem[kPoolStage];
  const int p = blockIdx.x;
  int b = off[p], e = off[p + 1];
  if (b < 0 || e <= b || e > n) {
    if (threadIdx.x == 0) atomicOr(status, kStatusBadIndex);
    b = min(max(b, 0), n);
    e = min(max(e, b), n);
  }
  // one pass over the members per group of blockDim.x channels
  for (int c0 = 0; c0 < d; c0 += blockDim.x) {
    const int c = c0 + threadIdx.x;
    double s = 0.0;
    for (int r0 = b; r0 < e; r0 += kPoolStage) {
      const int nr = min(kPoolStage, e - r0);
      __syncthreads();
      for (int i = threadIdx.x; i < nr; i += blockDim.x) {
        const int v = mem[r0 + i];
        if (v < 0 || v >= n) atomicOr(status, kStatusBadIndex);
        s_mem[i] = v;
      }
      __syncthreads();
      if (c >= d) continue;
      for (int i0 = 0; i0 < nr; i0 += kPoolBatch) {
        double x[kPoolBatch];
#pragma unroll
        for (int u = 0; u < kPoolBatch; ++u) {
          const int v = i0 + u < nr ? s_mem[i0 + u] : -1;
          x[u] = (v >= 0 && v < n) ? load_elem<F32>(F, (size_t)v * ld + c) : 0.0;
        }
#pragma unroll
        for (int u = 0; u < kPoolBatch; ++u) {
          const int v = i0 + u < nr ? s_mem[i0 + u] : -1;
          if (v >= 0 && v < n) s = __dadd_rn(s, x[u]);
        }
      }
    }
    if (c < d) mu[(size_t)p * d + c] = __ddiv_rn(s, (double)max(e - b, 1));
  }
}

constexpr int kST = 32;  // score tile (target x source patches)
constexpr int kSC = 16;  // channels staged per step

// scores[p, q] for a 32 x 32 tile per block; each thread owns 4 outputs and
// sums its products strictly in channel order.
__global__ void __launch_bounds__(256) scores_kernel(const double* __restrict__ muN, int PN,
                                                     const double* __restrict__ muM, int PM, int d,
                                                     double* __restrict__ sc) {
  __shared__ double a[kST][kSC + 1];
  __shared__ double b[kST][kSC + 1];
  const int p0 = blockIdx.y * kST, q0 = blockIdx.x * kST;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 8 rows of threads
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int c0 = 0; c0 < d; c0 += kSC) {
    for (int i = threadIdx.x; i < kST * kSC; i += 256) {
      int r = i / kSC, cc = i % kSC;
      a[r][cc] = (p0 + r < PN && c0 + cc < d) ? muN[(size_t)(p0 + r) * d + c0 + cc] : 0.0;
      b[r][cc] = (q0 + r < PM && c0 + cc < d) ? muM[(size_t)(q0 + r) * d + c0 + cc] : 0.0;
    }
    __syncthreads();
    const int cmax = min(kSC, d - c0);
    for (int cc = 0; cc < cmax; ++cc) {
      const double bv = b[tx][cc];
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = __dadd_rn(acc[i], __dmul_rn(a[ty + 8 * i][cc], bv));
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int p = p0 + ty + 8 * i, q = q0 + tx;
    if (p < PN && q < PM) sc[(size_t)p * PM + q] = acc[i];
  }
}

struct Pick {
  double s;
  int q;
};
// a ranks before b: higher score, ties to the lower patch index.
__device__ __forceinline__ bool pick_before(const Pick& a, const Pick& b) {
  return a.s > b.s || (a.s == b.s && a.q < b.q);
}

// One block per target patch; round r finds the best candidate ranked after
// the round r-1 winner, so no candidate needs marking.
__global__ void __launch_bounds__(256) topk_kernel(const double* __restrict__ sc, int PM, int R,
                                                   int* __restrict__ topk) {
  __shared__ Pick warp_best[8];
  __shared__ Pick s_prev;
  const int p = blockIdx.x;
  const double* row = sc + (size_t)p * PM;
  Pick prev{DBL_MAX, -1};
  bool first = true;
  for (int r = 0; r < R; ++r) {
    Pick mine{-DBL_MAX, INT_MAX};
    bool have = false;
    for (int q = threadIdx.x; q < PM; q += blockDim.x) {
      Pick c{row[q], q};
      if (!first && !pick_before(prev, c)) continue;
      if (!have || pick_before(c, mine)) {
        mine = c;
        have = true;
      }
    }
    if (!have) mine = Pick{-DBL_MAX, INT_MAX};
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      Pick x;
      x.s = __shfl_xor_sync(0xffffffffu, mine.s, o);
      x.q = __shfl_xor_sync(0xffffffffu, mine.q, o);
      if (x.q != INT_MAX && (mine.q == INT_MAX || pick_before(x, mine))) mine = x;
    }
    if ((threadIdx.x & 31) == 0) warp_best[threadIdx.x >> 5] = mine;
    __syncthreads();
    if (threadIdx.x == 0) {
      Pick w = warp_best[0];
      for (int i = 1; i < (int)(blockDim.x / 32); ++i) {
        Pick x = warp_best[i];
        if (x.q != INT_MAX && (w.q == INT_MAX || pick_before(x, w))) w = x;
      }
      s_prev = w;
      topk[(size_t)p * R + r] = w.q;
    }
    __syncthreads();
    prev = s_prev;
    first = false;
    __syncthreads();
  }
}

}  // namespace

size_t scores_topk_workspace_bytes(int PN, int PM, int d) {
  Carve c(nullptr);
  c.take<double>((size_t)PN * d);
  c.take<double>((size_t)PM * d);
  c.take<double>((size_t)PN * PM);
  return c.used + 256;
}

cudaError_t launch_scores_topk(const void* FN, int ldn, int nN, const void* FM, int ldm, int nM,
                               int d, int dtype, const int* offN, const int* memN, int PN,
                               const int* offM, const int* memM, int PM, int R, int* topk,
                               double* scores, void* ws, unsigned* status, cudaStream_t st) {
  Carve c(ws);
  double* muN = c.take<double>((size_t)PN * d);
  double* muM = c.take<double>((size_t)PM * d);
  double* sc_ws = c.take<double>((size_t)PN * PM);
  double* sc = scores ? scores : sc_ws;
  const int pt = d >= 128 ? 128 : 64;
  if (dtype == 1) {
    pool_kernel<true><<<PN, pt, 0, st>>>(FN, ldn, nN, d, offN, memN, muN, status);
    count_launch();
    pool_kernel<true><<<PM, pt, 0, st>>>(FM, ldm, nM, d, offM, memM, muM, status);
    count_launch();
  } else {
    pool_kernel<false><<<PN, pt, 0, st>>>(FN, ldn, nN, d, offN, memN, muN, status);
    count_launch();
    pool_kernel<false><<<PM, pt, 0, st>>>(FM, ldm, nM, d, offM, memM, muM, status);
    count_launch();
  }
  dim3 grid((PM + kST - 1) / kST, (PN + kST - 1) / kST);
  scores_kernel<<<grid, 256, 0, st>>>(muN, PN, muM, PM, d, sc);
  count_launch();
  topk_kernel<<<PN, 256, 0, st>>>(sc, PM, R, topk);
  count_launch();
  return cudaGetLastError();
}

}  // namespace ssc
