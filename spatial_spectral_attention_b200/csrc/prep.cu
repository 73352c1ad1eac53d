// prep.cu -- data movement around the coupling kernels: row gathers into the
// patch-major order Geo-FlashAttention works in, the backward preparation
// (bf16 upstream gradient and D_i = <dO_i, O_i>), and the tile schedules.
//
// Patch-major order (project page, "Geo-FlashAttention": each target patch
// attends to its selected source patches): after the gather, the rows of patch
// p are the contiguous range offsets[p] .. offsets[p+1] of the gathered
// buffer, so every selected source patch is a run of consecutive key rows that
// one TMA box can fetch.  All kernels here are HBM-bound copies: 16-byte
// vector accesses, one warp per row.
#include <algorithm>

#include <type_traits>

#include <cuda_fp8.h>

#include "internal.h"
#include "ssc.h"

namespace ssc {
namespace {

// Patch p of a table with n rows, clamped into [0, n] and non-decreasing;
// an inconsistent table sets the bad-index bit (and yields empty patches).
__device__ __forceinline__ int2 patch_range(const int* off, int p, int n, unsigned* status) {
  int b = off[p], e = off[p + 1];
  if (b < 0 || e < b || e > n) {
    atomicOr(status, kStatusBadIndex);
    b = min(max(b, 0), n);
    e = min(max(e, b), n);
  }
  return make_int2(b, e);
}

__device__ __forceinline__ int checked_src(const int* map, int r, int src_rows, unsigned* status) {
  const int src = map ? map[r] : r;
  if (src < 0 || src >= src_rows) {
    atomicOr(status, kStatusBadIndex);
    return -1;
  }
  return src;
}

// Padding columns [cols, out_ld) are zero, except column ones_col (when >= 0),
// which is set to one: a column of ones in V makes the P V product carry the
// softmax row sum.
__global__ void gather_bf16_from_bf16(const __nv_bfloat16* __restrict__ in, int in_ld,
                                      const int* __restrict__ map, int rows, int src_rows, int cols,
                                      __nv_bfloat16* __restrict__ out, int out_ld, int vec_ok,
                                      int ones_col, unsigned* status) {
  const int warps = gridDim.x * (blockDim.x >> 5);
  const int lane = threadIdx.x & 31;
  for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    const int src = checked_src(map, r, src_rows, status);
    __nv_bfloat16* o = out + (size_t)r * out_ld;
    if (src < 0) {
      for (int c = lane; c < out_ld; c += 32) o[c] = __float2bfloat16(0.f);
      continue;
    }
    const __nv_bfloat16* a = in + (size_t)src * in_ld;
    if (vec_ok == 2) {
      const int nvec = cols >> 3;  // full 8-element (16-byte) chunks
      for (int v = lane; v < nvec; v += 32)
        reinterpret_cast<uint4*>(o)[v] = __ldg(reinterpret_cast<const uint4*>(a) + v);
      for (int c = (nvec << 3) + lane; c < out_ld; c += 32)
        o[c] = c < cols ? a[c] : __float2bfloat16(c == ones_col ? 1.f : 0.f);
    } else if (vec_ok == 1) {
      const int nvec = cols >> 2;  // full 4-element (8-byte) chunks
      for (int v = lane; v < nvec; v += 32)
        reinterpret_cast<uint2*>(o)[v] = __ldg(reinterpret_cast<const uint2*>(a) + v);
      for (int c = (nvec << 2) + lane; c < out_ld; c += 32)
        o[c] = c < cols ? a[c] : __float2bfloat16(c == ones_col ? 1.f : 0.f);
    } else {
      for (int c = lane; c < out_ld; c += 32)
        o[c] = c < cols ? a[c] : __float2bfloat16(c == ones_col ? 1.f : 0.f);
    }
  }
}

// One thread per VEC-element piece of an output row (VEC = 8: 16-byte pieces,
// 4: 8-byte pieces); every piece is an independent, aligned copy, so the whole
// matrix moves with full coalescing and no per-row dependency chain.  Padding
// columns [cols, out_ld) are zero except ones_col (when >= 0), which is one.
template <int VEC>
__global__ void gather_bf16_pieces(const __nv_bfloat16* __restrict__ in, int in_ld,
                                   const int* __restrict__ map, int rows, int src_rows, int cols,
                                   __nv_bfloat16* __restrict__ out, int out_ld, int ones_col,
                                   unsigned* status) {
  using Vec = typename std::conditional<VEC == 8, uint4, uint2>::type;
  const int pieces = out_ld / VEC;
  const long long total = (long long)rows * pieces;
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (long long)gridDim.x * blockDim.x) {
    const int r = (int)(i / pieces);
    const int c0 = (int)(i - (long long)r * pieces) * VEC;
    const int src = checked_src(map, r, src_rows, status);
    Vec* o = reinterpret_cast<Vec*>(out + (size_t)r * out_ld + c0);
    if (src >= 0 && c0 + VEC <= cols) {
      *o = __ldg(reinterpret_cast<const Vec*>(in + (size_t)src * in_ld + c0));
    } else {
      uint32_t w[VEC / 2];  // bf16 pairs, element 2q in the low half of word q
#pragma unroll
      for (int q = 0; q < VEC / 2; ++q) {
        uint32_t h[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int c = c0 + 2 * q + e;
          const __nv_bfloat16 b = (src >= 0 && c < cols) ? in[(size_t)src * in_ld + c]
                                                         : __float2bfloat16(c == ones_col ? 1.f : 0.f);
          h[e] = __bfloat16_as_ushort(b);
        }
        w[q] = h[0] | (h[1] << 16);
      }
      if constexpr (VEC == 8) *o = make_uint4(w[0], w[1], w[2], w[3]);
      else *o = make_uint2(w[0], w[1]);
    }
  }
}

// Up to three bf16 row gathers in one launch (the patch-major Q, K and V of
// Geo-FlashAttention).  Job j covers the global pieces [begin_j, begin_j+1);
// its pieces are `vec` elements wide (8: 16 bytes, 4: 8 bytes, 1: one
// element).  Each thread loads four pieces before it stores them, so four
// loads per thread are in flight.  Semantics per job as gather_bf16_pieces.
struct GatherJob {
  const __nv_bfloat16* in;
  const int* map;
  __nv_bfloat16* out;
  int in_ld, rows, src_rows, cols, out_ld;
  int vec;     // elements per output piece (8, 4 or 1)
  int split;   // vec = 8 pieces read as two 8-byte halves (rows 8-byte aligned only)
  int pieces;  // output pieces per row, out_ld / vec (< 512)
  unsigned long long magic;  // floor(2^40 / pieces) + 1: r = (i * magic) >> 40 = i / pieces
};
struct GatherJobs {
  GatherJob j[3];
};

// Output piece li of a job (row li / pieces, columns from (li % pieces) vec):
// the row's source through the map, read in one or two loads when the piece
// lies within the source columns, element by element (zero past them) else.
// The division by the job's piece count is a multiply by its inverse (exact
// for li < 2^30 and pieces < 512: li (magic pieces - 2^40) < 2^39).
__device__ __forceinline__ uint4 gather_piece(const GatherJob& g, int li, unsigned* status,
                                              __nv_bfloat16** dst) {
  const int r = (int)(((unsigned long long)(unsigned)li * g.magic) >> 40);
  const int c0 = (li - r * g.pieces) * g.vec;
  const int src = checked_src(g.map, r, g.src_rows, status);
  *dst = g.out + (size_t)r * g.out_ld + c0;
  if (src >= 0 && c0 + g.vec <= g.cols) {
    const __nv_bfloat16* a = g.in + (size_t)src * g.in_ld + c0;
    if (g.vec == 8) {
      if (g.split) {
        const uint2 x = __ldg(reinterpret_cast<const uint2*>(a));
        const uint2 y = __ldg(reinterpret_cast<const uint2*>(a) + 1);
        return make_uint4(x.x, x.y, y.x, y.y);
      }
      return __ldg(reinterpret_cast<const uint4*>(a));
    }
    if (g.vec == 4) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(a));
      return make_uint4(v.x, v.y, 0u, 0u);
    }
    return make_uint4(__bfloat16_as_ushort(a[0]), 0u, 0u, 0u);
  }
  // wholly past the source columns (the padding of the row) or a dead row: zeros
  if (src < 0 || c0 >= g.cols) return make_uint4(0u, 0u, 0u, 0u);
  // an 8-element piece with 4 source columns left (k = 4 mod 8): one 8-byte
  // load (vec = 8 pieces come from rows that are 8-byte aligned at least)
  if (g.vec == 8 && c0 + 4 == g.cols) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(g.in + (size_t)src * g.in_ld + c0));
    return make_uint4(v.x, v.y, 0u, 0u);
  }
  uint32_t w[4] = {0u, 0u, 0u, 0u};
  for (int e = 0; e < g.vec; ++e) {
    const int c = c0 + e;
    const uint32_t h = (src >= 0 && c < g.cols) ? __bfloat16_as_ushort(g.in[(size_t)src * g.in_ld + c]) : 0u;
    w[e >> 1] |= h << (16 * (e & 1));
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ void put_piece(__nv_bfloat16* dst, int vec, uint4 v) {
  if (vec == 8) *reinterpret_cast<uint4*>(dst) = v;
  else if (vec == 4) *reinterpret_cast<uint2*>(dst) = make_uint2(v.x, v.y);
  else *dst = __ushort_as_bfloat16((unsigned short)(v.x & 0xffffu));
}

// The three jobs one after the other, each over the whole grid, four pieces
// per thread in flight (loads before stores); the job loop is unrolled so that
// every job's parameters are read at fixed offsets.  32-bit piece indices (the
// launcher falls back to one launch per job when the pieces do not fit).
__global__ void gather_jobs_kernel(const __grid_constant__ GatherJobs jobs, unsigned* status) {
  const int stride = gridDim.x * blockDim.x;
  const int tid = blockIdx.x * blockDim.x + threadIdx.x;
#pragma unroll
  for (int jj = 0; jj < 3; ++jj) {
    const GatherJob& g = jobs.j[jj];
    const int n = g.rows * g.pieces;
    for (int i0 = tid; i0 < n; i0 += 4 * stride) {
      uint4 v[4];
      __nv_bfloat16* dst[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = i0 + u * stride;
        if (i < n) v[u] = gather_piece(g, i, status, &dst[u]);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (i0 + u * stride < n) put_piece(dst[u], g.vec, v[u]);
    }
  }
}

__global__ void gather_bf16_from_f32(const float* __restrict__ in, int in_ld,
                                     const int* __restrict__ map, int rows, int src_rows, int cols,
                                     __nv_bfloat16* __restrict__ out, int out_ld, unsigned* status) {
  const int warps = gridDim.x * (blockDim.x >> 5);
  const int lane = threadIdx.x & 31;
  for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    const int src = checked_src(map, r, src_rows, status);
    const float* a = in + (size_t)(src < 0 ? 0 : src) * in_ld;
    __nv_bfloat16* o = out + (size_t)r * out_ld;
    for (int c = lane; c < out_ld; c += 32)
      o[c] = __float2bfloat16((c < cols && src >= 0) ? a[c] : 0.f);
  }
}

__global__ void gather_f32_kernel(const float* __restrict__ in, int in_ld,
                                  const int* __restrict__ map, int rows, int src_rows, int cols,
                                  float* __restrict__ out, int out_ld, unsigned* status) {
  const int warps = gridDim.x * (blockDim.x >> 5);
  const int lane = threadIdx.x & 31;
  for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    const int src = checked_src(map, r, src_rows, status);
    const float* a = in + (size_t)(src < 0 ? 0 : src) * in_ld;
    float* o = out + (size_t)r * out_ld;
    for (int c = lane; c < out_ld; c += 32) o[c] = (c < cols && src >= 0) ? a[c] : 0.f;
  }
}

__global__ void bwd_prep_kernel(const float* __restrict__ dO, int lddo, const float* __restrict__ O,
                                int ldo, const float* __restrict__ lse, const int* __restrict__ map,
                                int rows, int src_rows, int k, __nv_bfloat16* __restrict__ dOb,
                                int ldb, float* __restrict__ dOf, int ldf, float* __restrict__ D,
                                float* __restrict__ lse_out, int vec4, unsigned* status) {
  const int warps = gridDim.x * (blockDim.x >> 5);
  const int lane = threadIdx.x & 31;
  if (vec4 && k <= 256) {
    // 2 rows per warp and step; each lane's (at most 2) float4 of dO and O of
    // both rows are loaded before any is used.  Per row the arithmetic is
    // that of the loop below, in the same order.
    const int w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int c4n = k >> 2;
    for (int r0 = 2 * w; r0 < rows; r0 += 2 * warps) {
      int src0[2];
      float4 gv[2][2], ov[2][2];
#pragma unroll
      for (int u = 0; u < 2; ++u) src0[u] = r0 + u < rows ? checked_src(map, r0 + u, src_rows, status) : -1;
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int src = src0[u] < 0 ? 0 : src0[u];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int c4 = lane + 32 * i;
          gv[u][i] = make_float4(0.f, 0.f, 0.f, 0.f);
          ov[u][i] = make_float4(0.f, 0.f, 0.f, 0.f);
          if (r0 + u < rows && c4 < c4n) {
            if (src0[u] >= 0) gv[u][i] = __ldg(reinterpret_cast<const float4*>(dO + (size_t)src * lddo) + c4);
            ov[u][i] = __ldg(reinterpret_cast<const float4*>(O + (size_t)src * ldo) + c4);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int r = r0 + u;
        if (r >= rows) break;
        const int src = src0[u] < 0 ? 0 : src0[u];
        float acc = 0.f;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const int c4 = lane + 32 * i;
          if (c4 >= c4n) break;
          float4 v = gv[u][i];
          if (dOb) {
            const __nv_bfloat162 b01 = __floats2bfloat162_rn(v.x, v.y);
            const __nv_bfloat162 b23 = __floats2bfloat162_rn(v.z, v.w);
            reinterpret_cast<uint2*>(dOb + (size_t)r * ldb)[c4] = make_uint2(
                *reinterpret_cast<const uint32_t*>(&b01), *reinterpret_cast<const uint32_t*>(&b23));
            v = make_float4(__low2float(b01), __high2float(b01), __low2float(b23), __high2float(b23));
          }
          if (dOf) reinterpret_cast<float4*>(dOf + (size_t)r * ldf)[c4] = v;
          acc = fmaf(v.x, ov[u][i].x, acc);
          acc = fmaf(v.y, ov[u][i].y, acc);
          acc = fmaf(v.z, ov[u][i].z, acc);
          acc = fmaf(v.w, ov[u][i].w, acc);
        }
        const float* g = dO + (size_t)src * lddo;
        const float* o = O + (size_t)src * ldo;
        for (int c = (k & ~3) + lane; c < k; c += 32) {
          float v = src0[u] < 0 ? 0.f : g[c];
          if (dOb) {
            __nv_bfloat16 b = __float2bfloat16(v);
            dOb[(size_t)r * ldb + c] = b;
            v = __bfloat162float(b);
          }
          if (dOf) dOf[(size_t)r * ldf + c] = v;
          acc = fmaf(v, o[c], acc);
        }
        if (dOb)
          for (int c = k + lane; c < ldb; c += 32) dOb[(size_t)r * ldb + c] = __float2bfloat16(0.f);
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        if (lane == 0) {
          D[r] = acc;
          if (lse_out) lse_out[r] = src0[u] < 0 ? 0.f : lse[src];
        }
      }
    }
    return;
  }
  for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    const int src0 = checked_src(map, r, src_rows, status);
    const int src = src0 < 0 ? 0 : src0;
    const float* g = dO + (size_t)src * lddo;
    const float* o = O + (size_t)src * ldo;
    float acc = 0.f;
    if (vec4) {
      // 4 columns per lane and step: 16-byte loads of dO and O, 8-byte bf16 stores
      for (int c4 = lane; c4 < (k >> 2); c4 += 32) {
        float4 v = src0 < 0 ? make_float4(0.f, 0.f, 0.f, 0.f)
                            : __ldg(reinterpret_cast<const float4*>(g) + c4);
        const float4 ov = __ldg(reinterpret_cast<const float4*>(o) + c4);
        if (dOb) {
          const __nv_bfloat162 b01 = __floats2bfloat162_rn(v.x, v.y);
          const __nv_bfloat162 b23 = __floats2bfloat162_rn(v.z, v.w);
          reinterpret_cast<uint2*>(dOb + (size_t)r * ldb)[c4] =
              make_uint2(*reinterpret_cast<const uint32_t*>(&b01), *reinterpret_cast<const uint32_t*>(&b23));
          v = make_float4(__low2float(b01), __high2float(b01), __low2float(b23), __high2float(b23));
        }
        if (dOf) reinterpret_cast<float4*>(dOf + (size_t)r * ldf)[c4] = v;
        acc = fmaf(v.x, ov.x, acc);
        acc = fmaf(v.y, ov.y, acc);
        acc = fmaf(v.z, ov.z, acc);
        acc = fmaf(v.w, ov.w, acc);
      }
    }
    for (int c = (vec4 ? (k & ~3) : 0) + lane; c < k; c += 32) {
      float v = src0 < 0 ? 0.f : g[c];
      if (dOb) {
        __nv_bfloat16 b = __float2bfloat16(v);
        dOb[(size_t)r * ldb + c] = b;
        v = __bfloat162float(b);
      }
      if (dOf) dOf[(size_t)r * ldf + c] = v;
      acc = fmaf(v, o[c], acc);
    }
    if (dOb)
      for (int c = k + lane; c < ldb; c += 32) dOb[(size_t)r * ldb + c] = __float2bfloat16(0.f);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
    if (lane == 0) {
      D[r] = acc;
      if (lse_out) lse_out[r] = src0 < 0 ? 0.f : lse[src];
    }
  }
}

__global__ void dense_schedule_kernel(int nN, int nM, RowTile* __restrict__ tiles,
                                      KeySeg* __restrict__ segs, int* __restrict__ prefix) {
  const int nt = (nN + kTileRows - 1) / kTileRows, ns = (nM + kTileRows - 1) / kTileRows;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i <= max(nt, ns); i += gridDim.x * blockDim.x) {
    if (i < nt) tiles[i] = RowTile{i * kTileRows, min(kTileRows, nN - i * kTileRows), 0, ns};
    if (i < ns) segs[i] = KeySeg{i * kTileRows, min(kTileRows, nM - i * kTileRows)};
    if (i <= nt) prefix[i] = i * ns;
  }
}

// Block-diagonal schedule of `batch` dense pairs stored back to back: row
// tile t of pair b covers query rows b nN + [128 t, ...) and visits only the
// key tiles of pair b (rows b nM + [128 j, ...)).
__global__ void batched_schedule_kernel(int batch, int nN, int nM, RowTile* __restrict__ tiles,
                                        KeySeg* __restrict__ segs, int* __restrict__ prefix) {
  const int nt = (nN + kTileRows - 1) / kTileRows, ns = (nM + kTileRows - 1) / kTileRows;
  const long m = (long)batch * max(nt, ns);
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i <= m; i += (long)gridDim.x * blockDim.x) {
    if (i < (long)batch * nt) {
      const int b = (int)(i / nt), t = (int)(i % nt);
      tiles[i] = RowTile{b * nN + t * kTileRows, min(kTileRows, nN - t * kTileRows), b * ns, ns};
    }
    if (i < (long)batch * ns) {
      const int b = (int)(i / ns), j = (int)(i % ns);
      segs[i] = KeySeg{b * nM + j * kTileRows, min(kTileRows, nM - j * kTileRows)};
    }
    if (i <= (long)batch * nt) prefix[i] = (int)(i * ns);
  }
}

// Patch tables of `batch` shapes (offsets [batch][P+1] into members
// [batch][n], vertex ids local to the shape) as the tables of one problem of
// batch n vertices and batch P patches: offsets and members shifted by b n.
// Entries outside their shape's range, offsets whose first value is not 0 or
// last is not n, become out-of-range values that the consumers drop, and set
// the bad-index bit.
__global__ void concat_tables_kernel(const int* __restrict__ off, const int* __restrict__ mem,
                                     int P, int n, int batch, int* __restrict__ off_out,
                                     int* __restrict__ mem_out, unsigned* status) {
  const long noff = (long)batch * P, nmem = (long)batch * n;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i <= max(noff, nmem);
       i += (long)gridDim.x * blockDim.x) {
    if (i < noff) {
      const int b = (int)(i / P), q = (int)(i % P);
      int o = off[(size_t)b * (P + 1) + q];
      const bool bad = o < 0 || o > n || (q == 0 && o != 0) ||
                       (q == P - 1 && off[(size_t)b * (P + 1) + P] != n);
      if (bad) atomicOr(status, kStatusBadIndex);
      o = min(max(o, 0), n);
      off_out[i] = b * n + o;
    }
    if (i == noff) off_out[i] = batch * n;
    if (i < nmem) {
      const int b = (int)(i / n);
      const int v = mem[i];
      if (v < 0 || v >= n) {
        atomicOr(status, kStatusBadIndex);
        mem_out[i] = -1;
      } else {
        mem_out[i] = b * n + v;
      }
    }
  }
}

// top-R lists [batch][PN][R] with source patches local to the pair, shifted by
// b PM; entries outside [0, PM) become -1 (dropped downstream, bad-index bit).
__global__ void concat_topk_kernel(const int* __restrict__ topk, int PN, int R, int PM, int batch,
                                   int* __restrict__ out, unsigned* status) {
  const long m = (long)batch * PN * R;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < m; i += (long)gridDim.x * blockDim.x) {
    const int b = (int)(i / ((long)PN * R));
    const int q = topk[i];
    if (q < 0 || q >= PM) {
      atomicOr(status, kStatusBadIndex);
      out[i] = -1;
    } else {
      out[i] = b * PM + q;
    }
  }
}

// Largest magnitude of a bf16 matrix [rows, d] (leading dimension ld) into
// *amax, kept as fp32 bits (non-negative floats order like their bits).
__global__ void amax_kernel(const __nv_bfloat16* __restrict__ A, int ld, int rows, int d,
                            unsigned* amax) {
  float m = 0.f;
  const long total = (long)rows * d;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x)
    m = fmaxf(m, fabsf(__bfloat162float(A[(i / d) * ld + i % d])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
  if ((threadIdx.x & 31) == 0) atomicMax(amax, __float_as_uint(m));
}

// out[r, c] = e4m3(A[r, c] * 448 / amax) with saturation, rows of d bytes.
__global__ void quantize_e4m3_kernel(const __nv_bfloat16* __restrict__ A, int ld, int rows, int d,
                                     const unsigned* amax, uint8_t* __restrict__ out) {
  const float am = __uint_as_float(*amax);
  const float mul = am > 0.f ? 448.0f / am : 1.0f;
  const long total = (long)rows * d;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < total; i += (long)gridDim.x * blockDim.x)
    out[i] = (uint8_t)__nv_cvt_float_to_fp8(__bfloat162float(A[(i / d) * ld + i % d]) * mul,
                                            __NV_SATFINITE, __NV_E4M3);
}

// The factor that turns the e4m3 product back into Q K^T: (amaxQ / 448) (amaxK / 448).
__global__ void dequant_factor_kernel(const unsigned* amax2, float* f) {
  const float aq = __uint_as_float(amax2[0]), ak = __uint_as_float(amax2[1]);
  *f = (aq > 0.f ? aq / 448.0f : 1.0f) * (ak > 0.f ? ak / 448.0f : 1.0f);
}

// Single-block exclusive scan of two int arrays of length m; totals[0..1].
__global__ void __launch_bounds__(1024) scan2_kernel(const int* __restrict__ a, const int* __restrict__ b,
                                                     int m, int* __restrict__ abase,
                                                     int* __restrict__ bbase,
                                                     int* __restrict__ totals) {
  __shared__ int pa[1024], pb[1024];
  const int tid = threadIdx.x;
  const int per = (m + 1023) / 1024;
  const int lo = tid * per, hi = min(m, lo + per);
  int sa = 0, sb = 0;
  for (int i = lo; i < hi; ++i) {
    sa += a[i];
    sb += b ? b[i] : 0;
  }
  pa[tid] = sa;
  pb[tid] = sb;
  __syncthreads();
  for (int o = 1; o < 1024; o <<= 1) {
    int xa = tid >= o ? pa[tid - o] : 0, xb = tid >= o ? pb[tid - o] : 0;
    __syncthreads();
    pa[tid] += xa;
    pb[tid] += xb;
    __syncthreads();
  }
  int ra = pa[tid] - sa, rb = pb[tid] - sb;
  for (int i = lo; i < hi; ++i) {
    abase[i] = ra;
    ra += a[i];
    if (b) {
      bbase[i] = rb;
      rb += b[i];
    }
  }
  if (tid == 1023) {
    totals[0] = pa[1023];
    totals[1] = pb[1023];
  }
}

constexpr int kSchedThreads = 1024;
__device__ __forceinline__ void add_to(int& a, const int& b) { a += b; }
__device__ __forceinline__ void add_to(ulonglong2& a, const ulonglong2& b) {
  a.x += b.x;
  a.y += b.y;
}
__device__ __forceinline__ void sub_from(int& a, const int& b) { a -= b; }
__device__ __forceinline__ void sub_from(ulonglong2& a, const ulonglong2& b) {
  a.x -= b.x;
  a.y -= b.y;
}
__device__ __forceinline__ int shfl_up_t(int v, int o) { return __shfl_up_sync(0xffffffffu, v, o); }
__device__ __forceinline__ ulonglong2 shfl_up_t(ulonglong2 v, int o) {
  return make_ulonglong2(__shfl_up_sync(0xffffffffu, v.x, o), __shfl_up_sync(0xffffffffu, v.y, o));
}
// Exclusive prefix of every thread's x over the block of kSchedThreads threads
// (warp scans by shuffles, then a scan of the 32 warp totals): three block
// barriers.  *total receives the sum over the block.  part: 32 entries.
template <typename T>
__device__ T block_exclusive(T x, T* part, T* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  T inc = x;  // inclusive prefix within the warp
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const T y = shfl_up_t(inc, o);
    if (lane >= o) add_to(inc, y);
  }
  if (lane == 31) part[warp] = inc;
  __syncthreads();
  if (warp == 0) {
    T w = part[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const T y = shfl_up_t(w, o);
      if (lane >= o) add_to(w, y);
    }
    part[lane] = w;
  }
  __syncthreads();
  T r{};  // the warps before this one, then this warp's lanes before this one
  if (warp > 0) r = part[warp - 1];
  *total = part[31];
  __syncthreads();  // part is reused by the next scan
  add_to(r, inc);
  sub_from(r, x);
  return r;
}

// Block-wide exclusive scan of v[0..m) into base[0..m) by one block of
// kSchedThreads threads (each thread a contiguous run); returns the total.
__device__ int block_scan(const int* v, int m, int* base, int* part) {
  const int tid = threadIdx.x;
  const int per = (m + kSchedThreads - 1) / kSchedThreads;
  const int lo = min(m, tid * per), hi = min(m, lo + per);
  int sacc = 0;
  for (int i = lo; i < hi; ++i) sacc += v[i];
  int total;
  int r = block_exclusive(sacc, part, &total);
  for (int i = lo; i < hi; ++i) {
    base[i] = r;
    r += v[i];
  }
  return total;
}

// Exclusive prefix of the row tiles with the target patches ordered by
// decreasing segment count (ties by patch index): base[i] is the first tile of
// patch i.  Sort key: the patch's segment count below the largest, capped at
// 7, so the seven largest counts get a bucket each and the rest share the
// last one.  The eight per-bucket running counts are 16-bit fields of a
// ulonglong2 (the caller guarantees fewer than 65536 tiles), scanned like
// block_scan's ints.  Returns the total.
__device__ __forceinline__ int tile_bucket(int nseg, int maxseg) { return min(7, maxseg - nseg); }
__device__ __forceinline__ ulonglong2 bucket_field(int b, int count) {
  const unsigned long long v = (unsigned long long)count << (16 * (b & 3));
  return b < 4 ? make_ulonglong2(v, 0ull) : make_ulonglong2(0ull, v);
}
__device__ __forceinline__ int bucket_count(const ulonglong2& x, int b) {
  return (int)(((b < 4 ? x.x : x.y) >> (16 * (b & 3))) & 0xffffull);
}
__device__ int sorted_tile_scan(const int* pieces, const int* nsegs, int m, int maxseg, int* base,
                                ulonglong2* part) {
  const int tid = threadIdx.x;
  const int per = (m + kSchedThreads - 1) / kSchedThreads;
  const int lo = min(m, tid * per), hi = min(m, lo + per);
  ulonglong2 acc = make_ulonglong2(0ull, 0ull);
  for (int i = lo; i < hi; ++i) {
    const ulonglong2 f = bucket_field(tile_bucket(nsegs[i], maxseg), pieces[i]);
    acc.x += f.x;
    acc.y += f.y;
  }
  ulonglong2 tot;
  ulonglong2 r = block_exclusive(acc, part, &tot);
  int start[8], total = 0;
#pragma unroll
  for (int b = 0; b < 8; ++b) {
    start[b] = total;
    total += bucket_count(tot, b);
  }
  for (int i = lo; i < hi; ++i) {
    const int b = tile_bucket(nsegs[i], maxseg);
    int sb = 0;
#pragma unroll
    for (int u = 0; u < 8; ++u)
      if (u == b) sb = start[u];
    base[i] = sb + bucket_count(r, b);
    const ulonglong2 f = bucket_field(b, pieces[i]);
    r.x += f.x;
    r.y += f.y;
  }
  return total;
}

// Key ranges [k0, k0 + kn) of the source patches topk[p R + r0 + u], u < 8,
// with every load of the eight issued before any is used (kn = -1: past R or
// a bad patch index, which sets the bad-index bit).
__device__ __forceinline__ void source_ranges8(const int* __restrict__ topk, int p, int R, int r0,
                                               const int* __restrict__ offM, int PM, int nM,
                                               unsigned* status, int (&k0)[8], int (&kn)[8]) {
  int q[8], b[8], e[8];
#pragma unroll
  for (int u = 0; u < 8; ++u) q[u] = r0 + u < R ? topk[(size_t)p * R + r0 + u] : -1;
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const bool ok = r0 + u < R && q[u] >= 0 && q[u] < PM;
    b[u] = ok ? offM[q[u]] : 0;
    e[u] = ok ? offM[q[u] + 1] : 0;
  }
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    k0[u] = 0;
    kn[u] = -1;
    if (r0 + u >= R) continue;
    if (q[u] < 0 || q[u] >= PM) {
      atomicOr(status, kStatusBadIndex);
      continue;
    }
    int bb = b[u], ee = e[u];
    if (bb < 0 || ee < bb || ee > nM) {
      atomicOr(status, kStatusBadIndex);
      bb = min(max(bb, 0), nM);
      ee = min(max(ee, bb), nM);
    }
    k0[u] = bb;
    kn[u] = ee - bb;
  }
}

// The whole Geo schedule in one block: per target patch its row tiles and
// source segments (counts), their exclusive scans, the tile and segment
// lists (row tiles by decreasing segment count), the clamped totals and the
// tiles' segment prefix sums, in one launch.
__global__ void __launch_bounds__(kSchedThreads, 1) geo_schedule_kernel(
    const int* __restrict__ offN, int PN, int nN, const int* __restrict__ offM, int PM, int nM,
    const int* __restrict__ topk, int R, RowTile* __restrict__ tiles, KeySeg* __restrict__ segs,
    int* __restrict__ counts, int* __restrict__ prefix, int* __restrict__ pieces,
    int* __restrict__ nsegs, int* __restrict__ tbase, int* __restrict__ sbase, int tile_cap,
    int seg_cap, unsigned long long* tag, unsigned long long tag_value, unsigned* status) {
  __shared__ int part[32];          // warp totals of the block scans
  __shared__ ulonglong2 part2[32];
  __shared__ int s_maxseg, s_tiles;
  if (threadIdx.x == 0) {
    s_maxseg = 0;
    s_tiles = 0;
    if (tag) *tag = tag_value;
  }
  __syncthreads();
  for (int p = threadIdx.x; p < PN; p += kSchedThreads) {
    const int2 pr = patch_range(offN, p, nN, status);
    pieces[p] = (pr.y - pr.x + kTileRows - 1) / kTileRows;
    int sacc = 0;
    for (int r0 = 0; r0 < R; r0 += 8) {
      int k0[8], kn[8];
      source_ranges8(topk, p, R, r0, offM, PM, nM, status, k0, kn);
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (kn[u] > 0) sacc += (kn[u] + kTileRows - 1) / kTileRows;
    }
    nsegs[p] = sacc;
    atomicMax(&s_maxseg, sacc);
    atomicAdd(&s_tiles, pieces[p]);
  }
  __syncthreads();
  // row tiles ordered by decreasing segment count, so that the forward's
  // alternating walk over bands of tiles balances the CTAs
  const int ntile = s_tiles < 65536 ? sorted_tile_scan(pieces, nsegs, PN, s_maxseg, tbase, part2)
                                    : block_scan(pieces, PN, tbase, part);
  const int nseg = block_scan(nsegs, PN, sbase, part);
  for (int p = threadIdx.x; p < PN; p += kSchedThreads) {
    const int2 pr = patch_range(offN, p, nN, status);
    const int r0 = pr.x, rows = pr.y - pr.x;
    const int sb = sbase[p];
    const int ns = max(0, min(nsegs[p], seg_cap - sb));
    if (ns < nsegs[p]) atomicOr(status, kStatusBadIndex);
    for (int t = 0, i = 0; t < rows; t += kTileRows, ++i) {
      if (tbase[p] + i >= tile_cap) {
        atomicOr(status, kStatusBadIndex);
        break;
      }
      tiles[tbase[p] + i] = RowTile{r0 + t, min(kTileRows, rows - t), sb, ns};
    }
    int sidx = sb;
    for (int r0 = 0; r0 < R; r0 += 8) {
      int k0[8], kn[8];
      source_ranges8(topk, p, R, r0, offM, PM, nM, status, k0, kn);
#pragma unroll
      for (int u = 0; u < 8; ++u)
        for (int v = 0; v < kn[u] && sidx < sb + ns; v += kTileRows)
          segs[sidx++] = KeySeg{k0[u] + v, min(kTileRows, kn[u] - v)};
    }
  }
  const int m = min(ntile, tile_cap);
  if (threadIdx.x == 0) {
    counts[0] = m;
    counts[1] = min(nseg, seg_cap);
  }
  __syncthreads();  // the tile list is complete
  // prefix[t] = segments of tiles[0..t)
  const int per = (m + kSchedThreads - 1) / kSchedThreads;
  const int lo = min(m, (int)threadIdx.x * per), hi = min(m, lo + per);
  int sacc = 0;
  for (int i = lo; i < hi; ++i) sacc += tiles[i].nseg;
  int total;
  int r = block_exclusive(sacc, part, &total);
  for (int i = lo; i < hi; ++i) {
    prefix[i] = r;
    r += tiles[i].nseg;
  }
  if (threadIdx.x == 0) prefix[m] = total;
}

__global__ void inv_count_kernel(const int* __restrict__ topk, int n, int PM, int* __restrict__ cnt) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const int q = topk[i];
    if (q >= 0 && q < PM) atomicAdd(cnt + q, 1);
  }
}
__global__ void inv_fill_kernel(const int* __restrict__ topk, int PN, int R, int PM,
                                int* __restrict__ cursor, int* __restrict__ inv_p) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < PN * R; i += gridDim.x * blockDim.x) {
    const int q = topk[i];
    if (q >= 0 && q < PM) inv_p[atomicAdd(cursor + q, 1)] = i / R;
  }
}
__global__ void inv_sort_kernel(const int* __restrict__ inv_off, int PM, int* __restrict__ inv_p) {
  for (int q = blockIdx.x * blockDim.x + threadIdx.x; q < PM; q += gridDim.x * blockDim.x) {
    const int b = inv_off[q], e = inv_off[q + 1];
    for (int i = b + 1; i < e; ++i) {
      int x = inv_p[i], j = i - 1;
      while (j >= b && inv_p[j] > x) {
        inv_p[j + 1] = inv_p[j];
        --j;
      }
      inv_p[j + 1] = x;
    }
  }
}
__global__ void copy_offsets_kernel(const int* __restrict__ base, const int* __restrict__ totals,
                                    int m, int* __restrict__ off, int* __restrict__ cursor) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i <= m; i += gridDim.x * blockDim.x) {
    const int v = i < m ? base[i] : totals[0];
    off[i] = v;
    if (i < m) cursor[i] = v;
  }
}

int grid_for(long work, int per_block) {
  long b = (work + per_block - 1) / per_block;
  return (int)std::max<long>(1, std::min<long>(b, 148L * 16));
}

}  // namespace

cudaError_t launch_gather_rows_bf16(const void* in, int in_ld, int in_f32, const int* map, int rows,
                                    int src_rows, int cols, __nv_bfloat16* out, int out_ld,
                                    unsigned* status, cudaStream_t st, int ones_col) {
  if (rows <= 0) return cudaSuccess;
  const int g = grid_for(rows, 8);
  if (in_f32) {
    gather_bf16_from_f32<<<g, 256, 0, st>>>(static_cast<const float*>(in), in_ld, map, rows,
                                            src_rows, cols, out, out_ld, status);
    count_launch();
  } else {
    // 2: rows 16-byte aligned on both sides, 1: 8-byte aligned, 0: element copies
    const uintptr_t ia = reinterpret_cast<uintptr_t>(in), oa = reinterpret_cast<uintptr_t>(out);
    const int vec_ok = (in_ld % 8 == 0 && out_ld % 8 == 0 && ia % 16 == 0 && oa % 16 == 0)
                           ? 2
                           : (in_ld % 4 == 0 && out_ld % 4 == 0 && ia % 8 == 0 && oa % 8 == 0) ? 1 : 0;
    if (vec_ok) {
      const long long total = (long long)rows * (out_ld / (vec_ok == 2 ? 8 : 4));
      const int gb = (int)std::max<long long>(1, std::min<long long>((total + 255) / 256, 148LL * 16));
      const auto* ib = static_cast<const __nv_bfloat16*>(in);
      prof_launch_begin(st);
      if (vec_ok == 2)
        gather_bf16_pieces<8><<<gb, 256, 0, st>>>(ib, in_ld, map, rows, src_rows, cols, out, out_ld,
                                                  ones_col, status);
      else
        gather_bf16_pieces<4><<<gb, 256, 0, st>>>(ib, in_ld, map, rows, src_rows, cols, out, out_ld,
                                                  ones_col, status);
      prof_launch_end(st, SSC_PROF_GATHER);
      count_launch();
      return cudaGetLastError();
    }
    gather_bf16_from_bf16<<<g, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(in), in_ld, map,
                                             rows, src_rows, cols, out, out_ld, vec_ok, ones_col,
                                             status);
    count_launch();
  }
  return cudaGetLastError();
}

__global__ void scatter_rows_f32_kernel(const float* __restrict__ in, int in_ld,
                                        const int* __restrict__ map, int rows, int dst_rows,
                                        int cols, float* __restrict__ out, int out_ld, int vec_ok,
                                        unsigned* status) {
  const int warps = gridDim.x * (blockDim.x >> 5);
  const int lane = threadIdx.x & 31;
  if (vec_ok && cols <= 128) {
    // 4 rows per warp and step, one float4 per lane and row: the map entries,
    // then all four rows' loads, then the stores
    const int w = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    const int c4n = cols >> 2;
    for (int r0 = 4 * w; r0 < rows; r0 += 4 * warps) {
      int dst[4];
      float4 v[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) dst[u] = r0 + u < rows ? checked_src(map, r0 + u, dst_rows, status) : -1;
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (dst[u] >= 0 && lane < c4n)
          v[u] = __ldg(reinterpret_cast<const float4*>(in + (size_t)(r0 + u) * in_ld) + lane);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        if (dst[u] < 0) continue;
        float* o = out + (size_t)dst[u] * out_ld;
        if (lane < c4n) reinterpret_cast<float4*>(o)[lane] = v[u];
        for (int c = 4 * c4n + lane; c < cols; c += 32) o[c] = in[(size_t)(r0 + u) * in_ld + c];
      }
    }
    return;
  }
  for (int r = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += warps) {
    const int dst = checked_src(map, r, dst_rows, status);
    if (dst < 0) continue;
    const float* a = in + (size_t)r * in_ld;
    float* o = out + (size_t)dst * out_ld;
    if (vec_ok) {
      for (int v = lane; v < (cols >> 2); v += 32)
        reinterpret_cast<float4*>(o)[v] = __ldg(reinterpret_cast<const float4*>(a) + v);
      for (int c = ((cols >> 2) << 2) + lane; c < cols; c += 32) o[c] = a[c];
    } else {
      for (int c = lane; c < cols; c += 32) o[c] = a[c];
    }
  }
}

cudaError_t launch_scatter_rows_f32(const float* in, int in_ld, const int* map, int rows,
                                    int dst_rows, int cols, float* out, int out_ld,
                                    unsigned* status, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  const int vec_ok = in_ld % 4 == 0 && out_ld % 4 == 0 && reinterpret_cast<uintptr_t>(in) % 16 == 0 &&
                     reinterpret_cast<uintptr_t>(out) % 16 == 0;
  const int g = grid_for(rows, vec_ok && cols <= 128 ? 32 : 8);
  scatter_rows_f32_kernel<<<g, 256, 0, st>>>(in, in_ld, map, rows, dst_rows, cols, out, out_ld,
                                             vec_ok, status);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_gather3_bf16(const __nv_bfloat16* const in[3], const int in_ld[3],
                                const int* const map[3], const int rows[3], const int src_rows[3],
                                const int cols[3], __nv_bfloat16* const out[3], const int out_ld[3],
                                unsigned* status, cudaStream_t st) {
  GatherJobs jobs;
  long long total = 0;
  bool small = true;
  for (int j = 0; j < 3; ++j) {
    GatherJob& g = jobs.j[j];
    const uintptr_t ia = reinterpret_cast<uintptr_t>(in[j]), oa = reinterpret_cast<uintptr_t>(out[j]);
    const bool out16 = out_ld[j] % 8 == 0 && oa % 16 == 0;
    const bool in16 = in_ld[j] % 8 == 0 && ia % 16 == 0;
    const bool in8 = in_ld[j] % 4 == 0 && ia % 8 == 0;
    g.split = out16 && !in16 && in8;
    g.vec = (out16 && (in16 || in8))                                         ? 8
            : (in8 && out_ld[j] % 4 == 0 && oa % 8 == 0)                     ? 4
                                                                             : 1;
    g.in = in[j];
    g.map = map[j];
    g.out = out[j];
    g.in_ld = in_ld[j];
    g.rows = rows[j];
    g.src_rows = src_rows[j];
    g.cols = cols[j];
    g.out_ld = out_ld[j];
    g.pieces = out_ld[j] / g.vec;
    g.magic = g.pieces > 0 ? (1ull << 40) / (unsigned long long)g.pieces + 1 : 0;
    if (g.pieces >= 512) small = false;
    total += (long long)rows[j] * g.pieces;
  }
  if (total == 0) return cudaSuccess;
  if (total >= (1LL << 30) || !small) {
    // too many pieces for 32-bit indices (or rows too long for the inverse):
    // one launch per matrix
    for (int j = 0; j < 3; ++j) {
      const cudaError_t e = launch_gather_rows_bf16(in[j], in_ld[j], 0, map[j], rows[j], src_rows[j],
                                                    cols[j], out[j], out_ld[j], status, st);
      if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
  }
  const long long begin = total;
  const int blocks = (int)std::max<long long>(1, std::min<long long>((begin + 1023) / 1024, 148LL * 8));
  prof_launch_begin(st);
  gather_jobs_kernel<<<blocks, 256, 0, st>>>(jobs, status);
  prof_launch_end(st, SSC_PROF_GATHER);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_gather_rows_f32(const float* in, int in_ld, const int* map, int rows,
                                   int src_rows, int cols, float* out, int out_ld, unsigned* status,
                                   cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  gather_f32_kernel<<<grid_for(rows, 8), 256, 0, st>>>(in, in_ld, map, rows, src_rows, cols, out,
                                                        out_ld, status);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_bwd_prep(const float* dO, int lddo, const float* O, int ldo, const float* lse,
                            const int* map, int rows, int src_rows, int k, __nv_bfloat16* dOb,
                            int ldb, float* dOf, int ldf, float* D, float* lse_out,
                            unsigned* status, cudaStream_t st) {
  if (rows <= 0) return cudaSuccess;
  // 16-byte row pieces of dO and O (and 8-byte bf16 / 16-byte fp32 output pieces)
  const auto a16 = [](const void* q) { return reinterpret_cast<uintptr_t>(q) % 16 == 0; };
  const int vec4 = lddo % 4 == 0 && ldo % 4 == 0 && a16(dO) && a16(O) &&
                   (!dOb || (ldb % 4 == 0 && reinterpret_cast<uintptr_t>(dOb) % 8 == 0)) &&
                   (!dOf || (ldf % 4 == 0 && a16(dOf)));
  bwd_prep_kernel<<<grid_for(rows, vec4 && k <= 256 ? 16 : 8), 256, 0, st>>>(
      dO, lddo, O, ldo, lse, map, rows, src_rows, k, dOb, ldb, dOf, ldf, D, lse_out, vec4, status);
  count_launch();
  return cudaGetLastError();
}

int dense_num_tiles(int nN) { return (nN + kTileRows - 1) / kTileRows; }
int dense_num_segs(int nM) { return (nM + kTileRows - 1) / kTileRows; }

cudaError_t launch_dense_schedule(int nN, int nM, RowTile* tiles, KeySeg* segs, int* prefix,
                                  cudaStream_t st) {
  const int m = std::max(dense_num_tiles(nN), dense_num_segs(nM)) + 1;
  dense_schedule_kernel<<<grid_for(m, 256), 256, 0, st>>>(nN, nM, tiles, segs, prefix);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_batched_schedule(int batch, int nN, int nM, RowTile* tiles, KeySeg* segs,
                                    int* prefix, cudaStream_t st) {
  const long m = (long)batch * std::max(dense_num_tiles(nN), dense_num_segs(nM)) + 1;
  batched_schedule_kernel<<<grid_for(m, 256), 256, 0, st>>>(batch, nN, nM, tiles, segs, prefix);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_concat_tables(const int* off, const int* mem, int P, int n, int batch,
                                 int* off_out, int* mem_out, unsigned* status, cudaStream_t st) {
  const long m = (long)batch * std::max(P, n) + 1;
  concat_tables_kernel<<<grid_for(m, 256), 256, 0, st>>>(off, mem, P, n, batch, off_out, mem_out,
                                                         status);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_concat_topk(const int* topk, int PN, int R, int PM, int batch, int* out,
                               unsigned* status, cudaStream_t st) {
  const long m = (long)batch * PN * R;
  concat_topk_kernel<<<grid_for(m, 256), 256, 0, st>>>(topk, PN, R, PM, batch, out, status);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_quantize_e4m3(const __nv_bfloat16* Q, int ldq, int nN, const __nv_bfloat16* K,
                                 int ldk, int nM, int d, uint8_t* Q8, uint8_t* K8,
                                 unsigned* amax2, float* qk_dequant, cudaStream_t st) {
  cudaError_t e;
  if ((e = cudaMemsetAsync(amax2, 0, 2 * sizeof(unsigned), st)) != cudaSuccess) return e;
  amax_kernel<<<grid_for((long)nN * d, 256), 256, 0, st>>>(Q, ldq, nN, d, amax2);
  amax_kernel<<<grid_for((long)nM * d, 256), 256, 0, st>>>(K, ldk, nM, d, amax2 + 1);
  quantize_e4m3_kernel<<<grid_for((long)nN * d, 256), 256, 0, st>>>(Q, ldq, nN, d, amax2, Q8);
  quantize_e4m3_kernel<<<grid_for((long)nM * d, 256), 256, 0, st>>>(K, ldk, nM, d, amax2 + 1, K8);
  dequant_factor_kernel<<<1, 1, 0, st>>>(amax2, qk_dequant);
  count_launch(5);
  return cudaGetLastError();
}

int geo_max_tiles(int nN, int PN) { return PN + (nN + kTileRows - 1) / kTileRows; }
int geo_max_segs(int nM, int PM, int PN, int R) {
  (void)PM;
  const long a = (long)PN * R + (long)PN * ((nM + kTileRows - 1) / kTileRows);
  return (int)std::min<long>(a, 0x7fffffffL);
}
size_t geo_schedule_scratch_ints(int PN) { return 4 * (size_t)PN + 2; }

cudaError_t launch_geo_schedule(const int* offN, int PN, int nN, const int* offM, int PM, int nM,
                                const int* topk, int R, RowTile* tiles, KeySeg* segs, int* counts,
                                int* prefix, int* scratch, unsigned* status, cudaStream_t st,
                                unsigned long long* tag, unsigned long long tag_value) {
  int* pieces = scratch;
  int* nsegs = scratch + PN;
  int* tbase = scratch + 2 * PN;
  int* sbase = scratch + 3 * PN;
  const int tile_cap = geo_max_tiles(nN, PN), seg_cap = geo_max_segs(nM, PM, PN, R);
  geo_schedule_kernel<<<1, kSchedThreads, 0, st>>>(offN, PN, nN, offM, PM, nM, topk, R, tiles, segs,
                                                   counts, prefix, pieces, nsegs, tbase, sbase,
                                                   tile_cap, seg_cap, tag, tag_value, status);
  count_launch();
  return cudaGetLastError();
}

namespace {
__global__ void check_tag_kernel(const unsigned long long* tag, unsigned long long expect,
                                 unsigned* status) {
  if (*tag != expect) atomicOr(status, kStatusBadIndex);
}
}  // namespace

cudaError_t launch_check_tag(const unsigned long long* tag, unsigned long long expect,
                             unsigned* status, cudaStream_t st) {
  check_tag_kernel<<<1, 1, 0, st>>>(tag, expect, status);
  count_launch();
  return cudaGetLastError();
}

size_t invert_topk_scratch_ints(int PM) { return 3 * (size_t)PM + 2; }

cudaError_t launch_invert_topk(const int* topk, int PN, int R, int PM, int* inv_off, int* inv_p,
                               int* scratch, cudaStream_t st) {
  int* cnt = scratch;            // [PM]
  int* base = scratch + PM;      // [PM]
  int* cursor = scratch + 2 * PM;  // [PM]
  int* totals = scratch + 3 * PM;  // [2]
  cudaError_t e = cudaMemsetAsync(cnt, 0, sizeof(int) * PM, st);
  if (e != cudaSuccess) return e;
  inv_count_kernel<<<grid_for((long)PN * R, 256), 256, 0, st>>>(topk, PN * R, PM, cnt);
  count_launch();
  scan2_kernel<<<1, 1024, 0, st>>>(cnt, nullptr, PM, base, nullptr, totals);
  count_launch();
  copy_offsets_kernel<<<grid_for(PM + 1, 256), 256, 0, st>>>(base, totals, PM, inv_off, cursor);
  count_launch();
  inv_fill_kernel<<<grid_for((long)PN * R, 256), 256, 0, st>>>(topk, PN, R, PM, cursor, inv_p);
  count_launch();
  inv_sort_kernel<<<grid_for(PM, 128), 128, 0, st>>>(inv_off, PM, inv_p);
  count_launch();
  return cudaGetLastError();
}

}  // namespace ssc
