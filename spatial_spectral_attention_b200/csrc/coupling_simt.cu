// coupling_simt.cu -- fp32 check mode of the coupling on CUDA cores.
//
// Same operation as the bf16 tensor-core path ("Spatial-Spectral Coupling as
// Attention", project page, "Spatial-spectral coupling is attention" and
// "Geo-FlashAttention"), evaluated in fp32 with an online softmax so that it
// can be held to a 1e-4 tolerance against the fp64 definition.  One warp owns
// one query row (forward, dQ) or one key row (dK, dV); 32 keys (or rows) are
// processed per step, one per lane, with warp-shuffle max/sum reductions.
// This path favours clarity over speed; the bf16 path is the fast one.
#include <algorithm>
#include <cmath>

#include "internal.h"

namespace ssc {
namespace {

constexpr int kWarps = 8;
constexpr int kMaxD = 128;
constexpr int kMaxK = 256;

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float dotf(const float* __restrict__ a, const float* __restrict__ b,
                                      int n) {
  float s = 0.f;
  for (int c = 0; c < n; ++c) s = fmaf(a[c], b[c], s);
  return s;
}

__global__ void __launch_bounds__(kWarps * 32) simt_fwd_kernel(SimtArgs a, float* __restrict__ O,
                                                               int ldo, float* __restrict__ lse) {
  __shared__ float qs[kWarps][kMaxD];
  const int ntiles = a.ntiles_dev ? *a.ntiles_dev : a.ntiles_host;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kt = (a.k + 31) / 32;
  for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
    const RowTile tile = a.tiles[t];
    for (int rr = warp; rr < tile.nrows; rr += kWarps) {
      const int row = tile.row0 + rr;
      for (int c = lane; c < a.d; c += 32) qs[warp][c] = a.Q[(size_t)row * a.ldq + c];
      __syncwarp();
      float m = -INFINITY, l = 0.f;
      float acc[kMaxK / 32];
#pragma unroll
      for (int i = 0; i < kMaxK / 32; ++i) acc[i] = 0.f;
      for (int sgi = 0; sgi < tile.nseg; ++sgi) {
        const KeySeg sg = a.segs[tile.seg0 + sgi];
        for (int j0 = 0; j0 < sg.nkeys; j0 += 32) {
          const int j = j0 + lane;
          float s = -INFINITY;
          if (j < sg.nkeys) s = a.scale * dotf(qs[warp], a.K + (size_t)(sg.key0 + j) * a.ldk, a.d);
          const float mn = fmaxf(m, warp_max(s));
          const float alpha = expf(m - mn);  // m = -inf at the start: alpha = 0
          const float p = j < sg.nkeys ? expf(s - mn) : 0.f;
          l = l * alpha + warp_sum(p);
#pragma unroll
          for (int i = 0; i < kMaxK / 32; ++i) acc[i] *= alpha;
          const int cnt = min(32, sg.nkeys - j0);
          for (int jj = 0; jj < cnt; ++jj) {
            const float pj = __shfl_sync(0xffffffffu, p, jj);
            const float* vrow = a.V + (size_t)(sg.key0 + j0 + jj) * a.ldv;
#pragma unroll
            for (int i = 0; i < kMaxK / 32; ++i) {
              const int c = lane + 32 * i;
              if (i < kt && c < a.k) acc[i] = fmaf(pj, vrow[c], acc[i]);
            }
          }
          m = mn;
        }
      }
      const int orow = a.row_map ? a.row_map[row] : row;
      if (orow < 0 || orow >= a.nN) continue;  // reported by the gather of Q
      const float inv = 1.f / l;
#pragma unroll
      for (int i = 0; i < kMaxK / 32; ++i) {
        const int c = lane + 32 * i;
        if (i < kt && c < a.k) O[(size_t)orow * ldo + c] = acc[i] * inv;
      }
      if (lane == 0) lse[orow] = m + logf(l);
      __syncwarp();
    }
  }
}

// lse and D are in the (permuted) row order of Q.
__global__ void __launch_bounds__(kWarps * 32)
    simt_dq_kernel(SimtArgs a, const float* __restrict__ dO, int lddo, const float* __restrict__ lse,
                   const float* __restrict__ D, float* __restrict__ dQ, int lddq) {
  __shared__ float qs[kWarps][kMaxD];
  __shared__ float gs[kWarps][kMaxK];
  const int ntiles = a.ntiles_dev ? *a.ntiles_dev : a.ntiles_host;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
    const RowTile tile = a.tiles[t];
    for (int rr = warp; rr < tile.nrows; rr += kWarps) {
      const int row = tile.row0 + rr;
      for (int c = lane; c < a.d; c += 32) qs[warp][c] = a.Q[(size_t)row * a.ldq + c];
      for (int c = lane; c < a.k; c += 32) gs[warp][c] = dO[(size_t)row * lddo + c];
      __syncwarp();
      const float L = lse[row], Di = D[row];
      float acc[kMaxD / 32] = {0.f, 0.f, 0.f, 0.f};
      for (int sgi = 0; sgi < tile.nseg; ++sgi) {
        const KeySeg sg = a.segs[tile.seg0 + sgi];
        for (int j0 = 0; j0 < sg.nkeys; j0 += 32) {
          const int j = j0 + lane;
          float ds = 0.f;
          if (j < sg.nkeys) {
            const size_t kr = (size_t)(sg.key0 + j);
            const float s = a.scale * dotf(qs[warp], a.K + kr * a.ldk, a.d);
            const float p = expf(s - L);
            const float dp = dotf(gs[warp], a.V + kr * a.ldv, a.k);
            ds = p * (dp - Di);
          }
          const int cnt = min(32, sg.nkeys - j0);
          for (int jj = 0; jj < cnt; ++jj) {
            const float dsj = __shfl_sync(0xffffffffu, ds, jj);
            const float* krow = a.K + (size_t)(sg.key0 + j0 + jj) * a.ldk;
#pragma unroll
            for (int i = 0; i < kMaxD / 32; ++i) {
              const int c = lane + 32 * i;
              if (c < a.d) acc[i] = fmaf(dsj, krow[c], acc[i]);
            }
          }
        }
      }
      const int orow = a.row_map ? a.row_map[row] : row;
      if (orow < 0 || orow >= a.nN) continue;  // reported by the gather of Q
#pragma unroll
      for (int i = 0; i < kMaxD / 32; ++i) {
        const int c = lane + 32 * i;
        if (c < a.d) dQ[(size_t)orow * lddq + c] = a.scale * acc[i];
      }
      __syncwarp();
    }
  }
}

// Key-stationary dK/dV.  Block b covers key rows [kb, ke) and the query-row
// ranges that see them: all rows (dense) or the rows of the target patches
// listed for source patch b.
__global__ void __launch_bounds__(kWarps * 32)
    simt_dkdv_kernel(SimtArgs a, SimtKeyArgs g, const float* __restrict__ dO, int lddo,
                     const float* __restrict__ lse, const float* __restrict__ D,
                     float* __restrict__ dK, int lddk, float* __restrict__ dV, int lddv) {
  __shared__ float ks[kWarps][kMaxD];
  __shared__ float vs[kWarps][kMaxK];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int b = blockIdx.x;
  int kb, ke, nranges;
  if (g.inv_off) {
    kb = min(max(g.offM[b], 0), a.nM);
    ke = min(max(g.offM[b + 1], kb), a.nM);
    nranges = g.inv_off[b + 1] - g.inv_off[b];
  } else {
    kb = b * 64;
    ke = min(a.nM, kb + 64);
    nranges = 1;
  }
  const int kt = (a.k + 31) / 32;
  for (int j = kb + warp; j < ke; j += kWarps) {
    for (int c = lane; c < a.d; c += 32) ks[warp][c] = a.K[(size_t)j * a.ldk + c];
    for (int c = lane; c < a.k; c += 32) vs[warp][c] = a.V[(size_t)j * a.ldv + c];
    __syncwarp();
    float dk[kMaxD / 32] = {0.f, 0.f, 0.f, 0.f};
    float dv[kMaxK / 32];
#pragma unroll
    for (int i = 0; i < kMaxK / 32; ++i) dv[i] = 0.f;
    for (int ri = 0; ri < nranges; ++ri) {
      int r0, r1;
      if (g.inv_off) {
        const int p = g.inv_p[g.inv_off[b] + ri];
        r0 = min(max(g.offN[p], 0), a.nN);
        r1 = min(max(g.offN[p + 1], r0), a.nN);
      } else {
        r0 = 0;
        r1 = a.nN;
      }
      for (int i0 = r0; i0 < r1; i0 += 32) {
        const int i = i0 + lane;
        float p = 0.f, ds = 0.f;
        if (i < r1) {
          const float s = a.scale * dotf(a.Q + (size_t)i * a.ldq, ks[warp], a.d);
          p = expf(s - lse[i]);
          const float dp = dotf(dO + (size_t)i * lddo, vs[warp], a.k);
          ds = p * (dp - D[i]);
        }
        const int cnt = min(32, r1 - i0);
        for (int ii = 0; ii < cnt; ++ii) {
          const float pi = __shfl_sync(0xffffffffu, p, ii);
          const float dsi = __shfl_sync(0xffffffffu, ds, ii);
          const float* qrow = a.Q + (size_t)(i0 + ii) * a.ldq;
          const float* grow = dO + (size_t)(i0 + ii) * lddo;
#pragma unroll
          for (int t = 0; t < kMaxD / 32; ++t) {
            const int c = lane + 32 * t;
            if (c < a.d) dk[t] = fmaf(dsi, qrow[c], dk[t]);
          }
          if (dV) {
#pragma unroll
            for (int t = 0; t < kMaxK / 32; ++t) {
              const int c = lane + 32 * t;
              if (t < kt && c < a.k) dv[t] = fmaf(pi, grow[c], dv[t]);
            }
          }
        }
      }
    }
    const int orow = a.col_map ? a.col_map[j] : j;
    if (orow < 0 || orow >= a.nM) {
      if (lane == 0) atomicOr(g.status, kStatusBadIndex);
      continue;
    }
#pragma unroll
    for (int t = 0; t < kMaxD / 32; ++t) {
      const int c = lane + 32 * t;
      if (c < a.d) dK[(size_t)orow * lddk + c] = a.scale * dk[t];
    }
    if (dV) {
#pragma unroll
      for (int t = 0; t < kMaxK / 32; ++t) {
        const int c = lane + 32 * t;
        if (t < kt && c < a.k) dV[(size_t)orow * lddv + c] = dv[t];
      }
    }
    __syncwarp();
  }
}

int simt_grid(const SimtArgs& a) {
  const int n = a.ntiles_dev ? 148 * 8 : a.ntiles_host;
  return std::max(1, std::min(n, 148 * 8));
}

}  // namespace

cudaError_t launch_simt_fwd(const SimtArgs& a, float* O, int ldo, float* lse, cudaStream_t st) {
  simt_fwd_kernel<<<simt_grid(a), kWarps * 32, 0, st>>>(a, O, ldo, lse);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_simt_bwd_dq(const SimtArgs& a, const float* dO, int lddo, const float* lse,
                               const float* D, float* dQ, int lddq, cudaStream_t st) {
  simt_dq_kernel<<<simt_grid(a), kWarps * 32, 0, st>>>(a, dO, lddo, lse, D, dQ, lddq);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_simt_bwd_dkdv(const SimtArgs& a, const SimtKeyArgs& g, const float* dO,
                                 int lddo, const float* lse, const float* D, float* dK, int lddk,
                                 float* dV, int lddv, cudaStream_t st) {
  const int blocks = g.inv_off ? g.PM : (a.nM + 63) / 64;
  simt_dkdv_kernel<<<blocks, kWarps * 32, 0, st>>>(a, g, dO, lddo, lse, D, dK, lddk, dV, lddv);
  count_launch();
  return cudaGetLastError();
}

}  // namespace ssc
