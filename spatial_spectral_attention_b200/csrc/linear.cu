// linear.cu -- the linear-attention (ELU) coupling on 5th-generation tensor
// cores (sm_100a).
//
// Source: "Spatial-Spectral Coupling as Attention", project page, Table 1, row
// "Linear attention (ELU)" (the approximate coupling the exact ones are
// compared with) and the ai4snews digest, "Interpretation" (linear attention
// replaces the softmax with a low-rank feature map).  The pages do not print
// the map; this library takes the ELU feature map phi(x) = elu(x) + 1
// (x + 1 for x > 0, exp(x) otherwise), applied to every descriptor entry.
// The weight of the pair (i, j) is <phi(Q_i), phi(K_j)> and each target row is
// normalised by its weight sum, so with
//   KV = sum_j phi(K_j)^T V_j  [d x k],   z = sum_j phi(K_j)  [d],
//   O_i = phi(Q_i) KV / den_i,  den_i = <phi(Q_i), z>,
// and the cost is linear in the vertex counts.  Backward for dL/dO = dO, with
// D_i = <dO_i, O_i> and Y_i = [dO_i / den_i, -D_i / den_i]:
//   dphi(Q_i) = Y_i [KV | z]^T,   [dKV | dz] = sum_i phi(Q_i)^T Y_i,
//   dphi(K_j) = [V_j | 1] [dKV | dz]^T,   dV_j = phi(K_j) dKV,
//   dQ = dphi(Q) * phi'(Q),  dK = dphi(K) * phi'(K),  phi'(x) = 1 (x > 0), exp(x).
//
// Kernels (bandwidth-bound skinny contractions, all on tcgen05 with TMEM
// accumulators and TMA-staged operands):
//   lin_reduce_kernel  C[d x nb] = phi(X)^T B over all rows (split over the
//                      SMs, A and B MN-major views of row tiles; phi applied in
//                      shared memory; a column of ones in B delivers z).
//   lin_finish_kernel  sums the per-CTA partials in a fixed order and writes
//                      the bf16 weight matrix in both orientations.
//   lin_rows_kernel    per 128-row tile, one MMA against a resident weight
//                      matrix: the forward (O, den), dV, and dQ / dK (times
//                      phi' of the descriptors).
//   lin_prep_kernel    Y rows from dO, O and den.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>

#include <cooperative_groups.h>

#include "internal.h"
#include "ssc.h"

namespace cg = cooperative_groups;

namespace ssc {
namespace {

constexpr int kBox = 128 * 128;  // bytes of a 128-row x 64-column bf16 box
constexpr int kWCols = 256;      // columns of the bf16 weight matrix W [128 x 256]
constexpr int kRedCluster = 4;   // CTAs of the reduction that sum their partials through DSMEM
constexpr int kAccPitch = 260;   // floats per staged accumulator row (skews the banks)

struct LinMaps {
  CUtensorMap a;  // row tiles of A: box {64, 128}
  CUtensorMap b;  // reduce: row tiles of B, box {64, 128}; rows kernel: resident W or W^T
  CUtensorMap o;  // rows kernel: fp32 output, box {32, 32} (stores)
};

struct LinReduceParams {
  int n;         // rows of X and B
  int xch;       // X boxes loaded per tile (d / 64); the others are zero-filled
  int bch;       // B chunks per tile (nb / 64 rounded up)
  int bload;     // B chunks loaded by TMA (those starting inside B's width)
  int nb;        // N of the MMA (multiple of 16, <= 256)
  int d;
  int ones_col;  // >= 0: that column of the B tile is set to one on rows < n
  float* part;   // [gridDim.x / kRedCluster][128][256]
  WaitCtl ctl;
};

enum LinMode { kLinFwd = 0, kLinDv = 1, kLinWide = 2 };

struct LinRowsParams {
  int n;         // rows of A and of the output
  int d, k;
  int nmma;      // N of the MMA
  int ksteps;    // K steps of 16 (wide mode)
  int ach;       // A boxes per tile
  int aload;     // A boxes loaded by TMA
  int wrows;     // rows of the resident weight box (256 for W^T, 128 for W)
  int ones_col;  // wide mode on V: that column of the A tile is set to one on rows < n
  const __nv_bfloat16* X;  // wide mode: descriptors whose phi' scales the result
  int ldx;
  float* out;
  int ldout;
  float* den;  // forward: row normalisers
  int tma_out;  // outputs leave through TMA stores of staged 32 x 32 boxes
  WaitCtl ctl;
};

constexpr float kLog2e = 1.4426950408889634f;
constexpr int kWorkers = 256;  // threads of the transform / epilogue warps (warps 2-9)

// exp(x) for x <= 0 through the MUFU base-2 exponential (relative error near
// 2^-22, far below the bf16 rounding that follows); branch-free phi and phi'.
__device__ __forceinline__ float exp_nonpos(float x) { return ex2_approx(fminf(x, 0.f) * kLog2e); }
__device__ __forceinline__ float phi_elu1(float x) { return x > 0.f ? x + 1.0f : exp_nonpos(x); }
__device__ __forceinline__ float dphi_elu1(float x) { return x > 0.f ? 1.0f : exp_nonpos(x); }

__device__ __forceinline__ float2 bf2_to_f2(uint32_t w) {
  return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

// phi applied to the 8 bf16 values of a 16-byte piece.
__device__ __forceinline__ uint4 phi_piece(uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float2 f = bf2_to_f2(w[i]);
    o[i] = pack_bf16x2(phi_elu1(f.x), phi_elu1(f.y));
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// phi over the first `nload` 64-column boxes of a 128-row tile (element-wise,
// so the swizzle is irrelevant), zeros over the rest of its `nch` boxes; the
// pieces are split over the kWorkers threads, four loads ahead of the math.
__device__ __forceinline__ void phi_tile(uint8_t* tile, int nload, int nch, int tid) {
  const int total = nch * 1024;  // 16-byte pieces
  for (int i0 = tid; i0 < total; i0 += 4 * kWorkers) {
    uint4 v[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * kWorkers;
      v[u] = (i < total && (i >> 10) < nload) ? *reinterpret_cast<const uint4*>(tile + (size_t)i * 16)
                                               : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = i0 + u * kWorkers;
      if (i < total)
        *reinterpret_cast<uint4*>(tile + (size_t)i * 16) =
            (i >> 10) < nload ? phi_piece(v[u]) : make_uint4(0, 0, 0, 0);
    }
  }
}

// 2-D tiled store of a shared-memory box into global memory through the tensor
// map (elements outside the tensor are not written); x * 4 bytes must be a
// multiple of 16 and x, y must not be negative.  Tracked by bulk async-groups.
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* m, int x, int y, const void* smem_src) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
          reinterpret_cast<uint64_t>(m)),
      "r"(x), "r"(y), "r"(smem_u32(smem_src))
      : "memory");
}

// Writes 32 fp32 values as row `lane` of a 32 x 32 box staged with the 128-byte
// swizzle (16-byte piece q of row r at piece q ^ (r & 7)).
__device__ __forceinline__ void stage_row32(uint8_t* box, int lane, const float (&v)[32]) {
#pragma unroll
  for (int q = 0; q < 8; ++q)
    *reinterpret_cast<float4*>(box + lane * 128 + ((q ^ (lane & 7)) << 4)) =
        make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
}

// Byte offset of element (r, c) of a 128B-swizzled tile stored as 64-column
// boxes of `box_rows` rows.
__device__ __forceinline__ uint32_t sw128_offset(int r, int c, int box_rows) {
  const int b = c >> 6, cb = c & 63;
  return (uint32_t)(b * box_rows * 128 + r * 128 + ((((cb >> 3) ^ (r & 7)) << 4)) + (cb & 7) * 2);
}

// The fixups one thread makes to row r of a B (reduce) or A (wide) tile in
// shared memory: chunks [nload, nch) are zero-filled, and the ones column is
// set when the row is valid.
__device__ __forceinline__ void row_fixups(uint8_t* tile, int r, int nload, int nch, int ones_col,
                                           bool valid) {
  for (int c = nload; c < nch; ++c)
    for (int q0 = 0; q0 < 8; ++q0) {
      const int q = (q0 + r) & 7;  // spread the rows over the banks
      *reinterpret_cast<uint4*>(tile + c * kBox + r * 128 + q * 16) = make_uint4(0, 0, 0, 0);
    }
  if (ones_col >= 0 && valid)
    *reinterpret_cast<__nv_bfloat16*>(tile + sw128_offset(r, ones_col, 128)) = __float2bfloat16(1.0f);
}

// ------------------------------------------------------------------ reduce
// Roles: warp 0 TMA producer, warp 1 MMA issuer and TMEM owner, warps 2-9 the
// phi transform of each X tile, the B-tile fixups and the epilogue (TMEM lane
// = output row c; the two warps of a lane quarter take alternate 32-column
// chunks).
__global__ void __cluster_dims__(kRedCluster, 1, 1) __launch_bounds__(64 + kWorkers, 1)
    lin_reduce_kernel(const __grid_constant__ LinMaps tm, const LinReduceParams p) {
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_full[2], bar_xf[2], bar_empty[2], bar_done;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base_u = smem_u32(smem_raw);
  const uint32_t sbase = (base_u + 1023u) & ~1023u;
  auto gptr = [&](uint32_t sa) { return smem_raw + (sa - base_u); };
  const uint32_t xbytes = 2 * kBox;
  const uint32_t stage = xbytes + p.bch * kBox;
  const int ntiles = (p.n + 127) / 128;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_full[i], 1);
      mbar_init(&bar_xf[i], kWorkers / 32);
      mbar_init(&bar_empty[i], 1);
    }
    mbar_init(&bar_done, 1);
    s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem, 256);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm.a);
    tma_prefetch_desc(&tm.b);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort = &s_abort;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0;
      for (int t = blockIdx.x; t < ntiles && !*abort; t += gridDim.x, ++it) {
        const int st = it & 1;
        if (it >= 2 && !mbar_wait(&bar_empty[st], ((it >> 1) - 1) & 1, p.ctl, abort)) break;
        mbar_arrive_expect_tx(&bar_full[st], (uint32_t)(p.xch + p.bload) * kBox);
        uint8_t* sx = gptr(sbase + st * stage);
        for (int c = 0; c < p.xch; ++c) tma_load_2d(sx + c * kBox, &tm.a, 64 * c, 128 * t, &bar_full[st]);
        for (int c = 0; c < p.bload; ++c)
          tma_load_2d(sx + xbytes + c * kBox, &tm.b, 64 * c, 128 * t, &bar_full[st]);
      }
      if (*abort) {
        volatile int never = 0;
        for (uint32_t g = it >= 2 ? it - 2 : 0; g < it; ++g)
          mbar_wait(&bar_full[g & 1], (g >> 1) & 1, p.ctl, &never);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = make_idesc_bf16(128, p.nb, 1, 1);
      uint32_t it = 0;
      for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++it) {
        const int st = it & 1;
        if (!mbar_wait(&bar_xf[st], (it >> 1) & 1, p.ctl, abort)) break;
        tc_fence_after();
        const uint32_t sx = sbase + st * stage, sb = sx + xbytes;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem, make_sdesc(sx + kk * 2048, kBox, 1024, kSw128),
                 make_sdesc(sb + kk * 2048, kBox, 1024, kSw128), idesc, (it > 0 || kk > 0) ? 1u : 0u);
        mma_commit(&bar_empty[st]);
      }
      mma_commit(&bar_done);
      volatile int never = 0;
      mbar_wait(&bar_done, 0, p.ctl, &never);
    }
  } else {
    const int tid = threadIdx.x - 64;  // 0..kWorkers-1
    uint32_t it = 0;
    bool ok = true;
    for (int t = blockIdx.x; t < ntiles; t += gridDim.x, ++it) {
      const int st = it & 1;
      if (!mbar_wait(&bar_full[st], (it >> 1) & 1, p.ctl, abort)) {
        ok = false;
        break;
      }
      uint8_t* sx = gptr(sbase + st * stage);
      phi_tile(sx, p.xch, 2, tid);
      if (tid < 128) row_fixups(sx + xbytes, tid, p.bload, p.bch, p.ones_col, 128 * t + tid < p.n);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_xf[st]);
    }
    // stage this CTA's sum [128 x nb] in shared memory (the pipeline buffers
    // are idle once the last MMA has completed); a CTA without tiles stages zeros
    if (ok && mbar_wait(&bar_done, 0, p.ctl, abort)) {
      tc_fence_after();
      const int c = 32 * (warp & 3) + lane;  // TMEM lane = output row (channel)
      const int half = (warp - 2) >> 2;
      const bool has = (int)blockIdx.x < ntiles;
      float* row = reinterpret_cast<float*>(gptr(sbase)) + c * kAccPitch;
      const uint32_t ta = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
      for (int m0 = 32 * half; m0 < p.nb; m0 += 64) {
        uint32_t v[32];
        tmem_ld32(ta + m0, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(row + m0 + i) =
              has ? make_float4(__uint_as_float(v[i]), __uint_as_float(v[i + 1]),
                                __uint_as_float(v[i + 2]), __uint_as_float(v[i + 3]))
                  : make_float4(0.f, 0.f, 0.f, 0.f);
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
  // the kRedCluster CTAs of the cluster add their staged sums in rank order
  // through distributed shared memory; CTA `rank` writes rows [32 rank, +32)
  cluster_sync_all();
  if (warp >= 2) {
    cg::cluster_group cluster = cg::this_cluster();
    const int rank = (int)cluster.block_rank();
    const float* src[kRedCluster];
#pragma unroll
    for (int q = 0; q < kRedCluster; ++q)
      src[q] = cluster.map_shared_rank(reinterpret_cast<float*>(gptr(sbase)), q);
    const int nb4 = p.nb >> 2;
    float* dst = p.part + (size_t)(blockIdx.x / kRedCluster) * 128 * 256;
    for (int i = threadIdx.x - 64; i < 32 * nb4; i += kWorkers) {
      const int c = 32 * rank + i / nb4, m = 4 * (i % nb4);
      if (c >= p.d) continue;
      float4 acc = *reinterpret_cast<const float4*>(src[0] + c * kAccPitch + m);
#pragma unroll
      for (int q = 1; q < kRedCluster; ++q) {
        const float4 v = *reinterpret_cast<const float4*>(src[q] + c * kAccPitch + m);
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      *reinterpret_cast<float4*>(dst + (size_t)c * 256 + m) = acc;
    }
  }
  cluster_sync_all();  // no CTA leaves while another still reads its shared memory
}

// Sums the G partials in block order and writes W [128 x 256] and W^T
// [256 x 128] (bf16, zero outside d x nb), and the fp32 sum when W32 is given.
__global__ void lin_finish_kernel(const float* __restrict__ part, int G, int d, int nb,
                                  __nv_bfloat16* __restrict__ W, __nv_bfloat16* __restrict__ WT,
                                  float* __restrict__ W32) {
  const int idx = blockIdx.x * blockDim.x + threadIdx.x;
  if (idx >= 128 * kWCols) return;
  const int c = idx / kWCols, m = idx % kWCols;
  float s = 0.f;
  if (c < d && m < nb) {
    // block order; the loads run ahead of the (ordered) additions
#pragma unroll 8
    for (int g = 0; g < G; ++g) s += part[((size_t)g * 128 + c) * 256 + m];
  }
  const __nv_bfloat16 b = __float2bfloat16(s);
  W[idx] = b;
  WT[(size_t)m * 128 + c] = b;
  if (W32) W32[idx] = s;
}

// ------------------------------------------------------------------ rows
// Per 128-row tile of A: acc = A W (N = nmma) with W resident in shared memory.
//   kLinFwd: A = phi(X) (K = 128), W = [KV | z]^T; O = acc[0..k) / acc[k], den = acc[k].
//   kLinDv:  A = phi(K), W = dKV^T; dV = acc[0..k).
//   kLinWide: A = Y or [V | 1] (K = 16 ksteps), W = [KV | z] or [dKV | dz];
//             out = acc[0..d) * phi'(X row).
// Roles as in the reduce kernel; warps 2-9 transform tile i + 1 before they
// write tile i, so the tensor core works on one tile while they finish the
// other.  In the epilogue the two warps of a TMEM lane quarter take alternate
// 16-column chunks of their 32 rows.
template <int MODE>
__global__ void __launch_bounds__(64 + kWorkers, 1)
    lin_rows_kernel(const __grid_constant__ LinMaps tm, const LinRowsParams p) {
  constexpr int S = MODE == kLinWide ? 2 : 3;     // A ring depth
  constexpr int kStg = MODE == kLinWide ? 1 : 2;  // 4 KB output staging boxes per worker warp
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_w, bar_full[S], bar_xf[S], bar_empty[S], bar_acc_full[2],
      bar_acc_empty[2], bar_drain;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base_u = smem_u32(smem_raw);
  const uint32_t sbase = (base_u + 1023u) & ~1023u;
  auto gptr = [&](uint32_t sa) { return smem_raw + (sa - base_u); };
  const uint32_t wchunk = (uint32_t)p.wrows * 128;         // bytes of one 64-column W box
  const uint32_t wbytes = MODE == kLinWide ? 4 * wchunk : 2 * wchunk;
  const uint32_t abytes = (uint32_t)p.ach * kBox;
  const uint32_t sW = sbase, sA0 = sbase + wbytes, sStg = sA0 + S * abytes;
  const int ntiles = (p.n + 127) / 128;
  const uint32_t acc_cols = MODE == kLinWide ? 128 : 256;

  if (threadIdx.x == 0) {
    mbar_init(&bar_w, 1);
    for (int i = 0; i < S; ++i) {
      mbar_init(&bar_full[i], 1);
      mbar_init(&bar_xf[i], kWorkers / 32);
      mbar_init(&bar_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_acc_full[i], 1);
      mbar_init(&bar_acc_empty[i], kWorkers / 32);
    }
    mbar_init(&bar_drain, 1);
    s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm.a);
    tma_prefetch_desc(&tm.b);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort = &s_abort;

  if (warp == 0) {
    if (lane == 0) {
      const int nwb = MODE == kLinWide ? 4 : 2;
      mbar_arrive_expect_tx(&bar_w, wbytes);
      for (int c = 0; c < nwb; ++c) tma_load_2d(gptr(sW) + c * wchunk, &tm.b, 64 * c, 0, &bar_w);
      uint32_t it = 0;
      for (int t = blockIdx.x; t < ntiles && !*abort; t += gridDim.x, ++it) {
        const int st = it % S;
        if (it >= (uint32_t)S && !mbar_wait(&bar_empty[st], ((it / S) - 1) & 1, p.ctl, abort)) break;
        mbar_arrive_expect_tx(&bar_full[st], (uint32_t)p.aload * kBox);
        uint8_t* sa = gptr(sA0 + st * abytes);
        for (int c = 0; c < p.aload; ++c) tma_load_2d(sa + c * kBox, &tm.a, 64 * c, 128 * t, &bar_full[st]);
      }
      // every copy issued must land before the CTA may exit
      volatile int never = 0;
      mbar_wait(&bar_w, 0, p.ctl, &never);
      if (*abort)
        for (uint32_t g = it >= (uint32_t)S ? it - S : 0; g < it; ++g)
          mbar_wait(&bar_full[g % S], (g / S) & 1, p.ctl, &never);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = make_idesc_bf16(128, p.nmma, 0, 0);
      bool ok = mbar_wait(&bar_w, 0, p.ctl, abort);
      uint32_t it = 0;
      for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++it) {
        const int st = it % S, buf = it & 1;
        if (!mbar_wait(&bar_xf[st], (it / S) & 1, p.ctl, abort)) break;
        if (it >= 2 && !mbar_wait(&bar_acc_empty[buf], ((it >> 1) - 1) & 1, p.ctl, abort)) break;
        tc_fence_after();
        const uint32_t sa = sA0 + st * abytes;
        const uint32_t acc = tmem + buf * acc_cols;
        if (MODE == kLinWide) {
          for (int kk = 0; kk < p.ksteps; ++kk) {
            const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
            const uint32_t woff = (kk >> 2) * wchunk + (kk & 3) * 32;
            mma_ss(acc, make_sdesc(sa + off, 16, 1024, kSw128), make_sdesc(sW + woff, 16, 1024, kSw128),
                   idesc, kk > 0 ? 1u : 0u);
          }
        } else {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * kBox + (kk & 3) * 32;
            const uint32_t woff = (kk >> 2) * wchunk + (kk & 3) * 32;
            mma_ss(acc, make_sdesc(sa + off, 16, 1024, kSw128), make_sdesc(sW + woff, 16, 1024, kSw128),
                   idesc, kk > 0 ? 1u : 0u);
          }
        }
        mma_commit(&bar_empty[st]);
        mma_commit(&bar_acc_full[buf]);
      }
      mma_commit(&bar_drain);
      volatile int never = 0;
      mbar_wait(&bar_drain, 0, p.ctl, &never);
    }
  } else {
    const int tid = threadIdx.x - 64;
    const int r = 32 * (warp & 3) + lane;  // TMEM lane = row within the tile
    const int half = (warp - 2) >> 2;      // which alternate 16-column chunks
    const uint32_t ta = tmem + ((uint32_t)(32 * (warp & 3)) << 16);
    // prepare tile number `it` (t = its row tile) in ring stage it % S
    auto prepare = [&](uint32_t it, int t) -> bool {
      const int st = it % S;
      if (!mbar_wait(&bar_full[st], (it / S) & 1, p.ctl, abort)) return false;
      uint8_t* sa = gptr(sA0 + st * abytes);
      if (MODE != kLinWide) phi_tile(sa, p.aload, 2, tid);
      else if (tid < 128) row_fixups(sa, tid, p.aload, p.ach, p.ones_col, 128 * t + tid < p.n);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_xf[st]);
      return true;
    };
    // outputs: staged per warp as 32 x 32 fp32 boxes (128-byte swizzle) and
    // written by TMA stores, or stored from registers when the output's leading
    // dimension rules TMA out
    uint8_t* stg = gptr(sStg) + (warp - 2) * kStg * 4096;
    uint32_t nst = 0;
    auto put_box = [&](const float (&v)[32], int x, int y) {
      const int b = nst % kStg;
      if (nst >= (uint32_t)kStg) {
        if (lane == 0) bulk_wait_group_read<kStg - 1>();
        __syncwarp();
      }
      uint8_t* box = stg + b * 4096;
      stage_row32(box, lane, v);
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        tma_store_2d(&tm.o, x, y, box);
        bulk_commit_group();
      }
      ++nst;
    };
    auto put_direct = [&](const float (&v)[32], float* optr, int c0, int cols) {
      if ((p.ldout & 3) == 0 && c0 + 32 <= cols) {
#pragma unroll
        for (int i = 0; i < 32; i += 4)
          *reinterpret_cast<float4*>(optr + c0 + i) = make_float4(v[i], v[i + 1], v[i + 2], v[i + 3]);
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (c0 + i < cols) optr[c0 + i] = v[i];
      }
    };
    bool ok = true;
    uint32_t it = 0;
    if (blockIdx.x < (unsigned)ntiles) ok = prepare(0, blockIdx.x);
    for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x, ++it) {
      const int tn = t + (int)gridDim.x;
      if (tn < ntiles && !prepare(it + 1, tn)) break;
      const int buf = it & 1;
      const int row = 128 * t + r;
      const int ybox = 128 * t + 32 * (warp & 3);
      const bool live = row < p.n;
      float* optr = p.out + (size_t)(live ? row : 0) * p.ldout;
      // wide mode: this thread's descriptor entries (32-column boxes half,
      // half + 2), loaded before the wait
      uint4 xv[8];
      if (MODE == kLinWide) {
        const __nv_bfloat16* xrow = p.X + (size_t)row * p.ldx;
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int c0 = 32 * (2 * jj + half);
#pragma unroll
          for (int u = 0; u < 4; ++u)
            xv[4 * jj + u] = (live && c0 < p.d) ? *reinterpret_cast<const uint4*>(xrow + c0 + 8 * u)
                                                : make_uint4(0, 0, 0, 0);
        }
      }
      if (!mbar_wait(&bar_acc_full[buf], (it >> 1) & 1, p.ctl, abort)) break;
      tc_fence_after();
      const uint32_t acc = ta + buf * acc_cols;
      if (MODE == kLinWide) {
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int c0 = 32 * (2 * jj + half);
          if (c0 >= p.d) break;
          uint32_t a[32];
          tmem_ld32(acc + c0, a);
          tmem_ld_wait();
          float g[32];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint32_t w[4] = {xv[4 * jj + u].x, xv[4 * jj + u].y, xv[4 * jj + u].z,
                                   xv[4 * jj + u].w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 f = bf2_to_f2(w[i]);
              g[8 * u + 2 * i] = __uint_as_float(a[8 * u + 2 * i]) * dphi_elu1(f.x);
              g[8 * u + 2 * i + 1] = __uint_as_float(a[8 * u + 2 * i + 1]) * dphi_elu1(f.y);
            }
          }
          if (p.tma_out) {
            if (ybox < p.n) put_box(g, c0, ybox);  // a box past the last row is skipped
          }
          else if (live) put_direct(g, optr, c0, p.d);
        }
      } else {
        float inv = 1.0f;
        if (MODE == kLinFwd) {
          const float den = __uint_as_float(tmem_ld1(acc + p.k));
          tmem_ld_wait();
          inv = 1.0f / den;
          if (live && half == 0) p.den[row] = den;
        }
        for (int c0 = 32 * half; c0 < p.k; c0 += 64) {
          uint32_t a[32];
          tmem_ld32(acc + c0, a);
          tmem_ld_wait();
          float g[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) g[i] = __uint_as_float(a[i]) * inv;
          if (p.tma_out) {
            if (ybox < p.n) put_box(g, c0, ybox);  // a box past the last row is skipped
          }
          else if (live) put_direct(g, optr, c0, p.k);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar_acc_empty[buf]);
    }
    // the stores must have read their staging before the CTA's memory is released
    if (lane == 0) bulk_wait_group_all();
    __syncwarp();
  }
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ prep
// Row i (one warp): g = bf16(dO_i), D_i = <g, O_i>,
// Y_i = bf16([g / den_i, -D_i / den_i, 0 ...]) over ldy columns.
__global__ void lin_prep_kernel(const float* __restrict__ dO, int lddo, const float* __restrict__ O,
                                int ldo, const float* __restrict__ den, int n, int k,
                                __nv_bfloat16* __restrict__ Y, int ldy) {
  const int wpb = blockDim.x >> 5;
  const int lane = threadIdx.x & 31;
  for (int i = blockIdx.x * wpb + (threadIdx.x >> 5); i < n; i += gridDim.x * wpb) {
    const float* g = dO + (size_t)i * lddo;
    const float* o = O + (size_t)i * ldo;
    float D = 0.f;
    for (int m = lane; m < k; m += 32) D += __bfloat162float(__float2bfloat16(g[m])) * o[m];
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) D += __shfl_xor_sync(0xffffffffu, D, s);
    const float inv = 1.0f / den[i];
    __nv_bfloat16* y = Y + (size_t)i * ldy;
    for (int m = lane; m < ldy; m += 32) {
      float v = 0.f;
      if (m < k) v = __bfloat162float(__float2bfloat16(g[m])) * inv;
      else if (m == k) v = -D * inv;
      y[m] = __float2bfloat16(v);
    }
  }
}

// ------------------------------------------------------------------ host
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn lin_encode_fn() {
  static const EncodeTiledFn fn = [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(ptr);
    return static_cast<EncodeTiledFn>(nullptr);
  }();
  return fn;
}

// fp32 [rows, cols] with leading dimension ld (elements), box {32, 32},
// 128-byte swizzle (TMA stores of staged output boxes; nothing is written
// outside the tensor).
bool lin_map_out(CUtensorMap* m, const float* ptr, int rows, int cols, int ld) {
  EncodeTiledFn fn = lin_encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)ld * 4};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(ptr), gdim, gstride, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// bf16 [rows, cols] with leading dimension ld (elements), box {64, box_rows},
// 128-byte swizzle; elements outside the tensor read as zero.
bool lin_map(CUtensorMap* m, const void* ptr, int rows, int cols, int ld, int box_rows) {
  EncodeTiledFn fn = lin_encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), gdim, gstride, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int lin_num_sms() {
  static const int n = [] {
    int dev = 0, v = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev);
    return v > 0 ? v : 148;
  }();
  return n;
}

// Clusters of the reduction: one per kRedCluster row tiles, up to an SM's
// worth of CTAs and no more than can be resident at once (the occupancy query
// is made once per shared-memory size, under a lock).
int lin_reduce_clusters(int n, int smem) {
  static std::mutex mu;
  static int cached_smem = -1, cached = 0;
  int resident = lin_num_sms() / kRedCluster;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (smem != cached_smem) {
      cudaLaunchConfig_t q = {};
      q.gridDim = dim3(kRedCluster * resident);
      q.blockDim = dim3(64 + kWorkers);
      q.dynamicSmemBytes = smem;
      int nc = 0;
      if (cudaFuncSetAttribute(lin_reduce_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               smem) == cudaSuccess &&
          cudaOccupancyMaxActiveClusters(&nc, lin_reduce_kernel, &q) == cudaSuccess && nc > 0)
        cached = nc;
      else
        cached = resident;
      cudaGetLastError();
      cached_smem = smem;
    }
    resident = std::max(1, std::min(resident, cached));
  }
  const int ntiles = (n + 127) / 128;
  return std::max(1, std::min((ntiles + kRedCluster - 1) / kRedCluster, resident));
}

}  // namespace

int lin_kv(int k) { return (k + 1 + 15) / 16 * 16; }

int lin_reduce_grid(int n) {
  const int ntiles = (n + 127) / 128;
  return std::max(1, (std::min(ntiles, lin_num_sms()) + kRedCluster - 1) / kRedCluster);
}

cudaError_t launch_lin_reduce(const __nv_bfloat16* X, int ldx, const __nv_bfloat16* B, int ldb,
                              int n, int d, int bwidth, int nb, int ones_col, float* part,
                              LinWeights w, cudaStream_t st, const WaitCtl& ctl) {
  LinMaps tm;
  std::memset(&tm, 0, sizeof(tm));
  if (!lin_map(&tm.a, X, n, d, ldx, 128) || !lin_map(&tm.b, B, n, bwidth, ldb, 128))
    return cudaErrorInvalidValue;
  LinReduceParams p;
  p.n = n;
  p.d = d;
  p.xch = (d + 63) / 64;
  p.nb = nb;
  p.bch = (nb + 63) / 64;
  p.bload = std::min(p.bch, (bwidth + 63) / 64);
  p.ones_col = ones_col;
  p.part = part;
  p.ctl = ctl;
  // the pipeline's two stages, or the staged [128 x kAccPitch] fp32 sum
  const int smem = 1024 + std::max(2 * (2 * kBox + p.bch * kBox), 128 * kAccPitch * 4);
  const int nclusters = lin_reduce_clusters(n, smem);
  cudaError_t e = cudaFuncSetAttribute(lin_reduce_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  prof_launch_begin(st);
  lin_reduce_kernel<<<kRedCluster * nclusters, 64 + kWorkers, smem, st>>>(tm, p);
  prof_launch_end(st, SSC_PROF_LIN_REDUCE);
  count_launch();
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  lin_finish_kernel<<<128 * kWCols / 256, 256, 0, st>>>(part, nclusters, d, nb, w.W, w.WT, w.W32);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_lin_rows(int mode, const __nv_bfloat16* A, int lda, int awidth, int n,
                            const __nv_bfloat16* Wmat, int d, int k, int nmma, int ksteps,
                            int ones_col, const __nv_bfloat16* X, int ldx, float* out, int ldout,
                            float* den, cudaStream_t st, const WaitCtl& ctl) {
  LinMaps tm;
  std::memset(&tm, 0, sizeof(tm));
  LinRowsParams p;
  std::memset(&p, 0, sizeof(p));
  p.n = n;
  p.d = d;
  p.k = k;
  p.nmma = nmma;
  p.ksteps = ksteps;
  p.ones_col = ones_col;
  p.X = X;
  p.ldx = ldx;
  p.out = out;
  p.ldout = ldout;
  p.den = den;
  p.ctl = ctl;
  const bool wide = mode == kLinWide;
  p.ach = wide ? (ksteps + 3) / 4 : 2;
  p.aload = std::min(p.ach, (awidth + 63) / 64);
  p.wrows = wide ? 128 : 256;
  if (!lin_map(&tm.a, A, n, awidth, lda, 128)) return cudaErrorInvalidValue;
  p.tma_out = (ldout % 4 == 0 && (reinterpret_cast<uintptr_t>(out) & 15u) == 0) ? 1 : 0;
  if (p.tma_out && !lin_map_out(&tm.o, out, n, wide ? d : k, ldout)) return cudaErrorInvalidValue;
  if (wide ? !lin_map(&tm.b, Wmat, 128, kWCols, kWCols, 128) : !lin_map(&tm.b, Wmat, kWCols, 128, 128, 256))
    return cudaErrorInvalidValue;
  const int S = wide ? 2 : 3;
  const int wbytes = wide ? 4 * 128 * 128 : 2 * 256 * 128;
  const int stg = 8 * (wide ? 1 : 2) * 4096;  // output staging of the 8 worker warps
  const int smem = 1024 + wbytes + S * p.ach * kBox + stg;
  const int grid = std::max(1, std::min((n + 127) / 128, lin_num_sms()));
  auto kern = mode == kLinFwd ? lin_rows_kernel<kLinFwd>
              : mode == kLinDv ? lin_rows_kernel<kLinDv>
                               : lin_rows_kernel<kLinWide>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  prof_launch_begin(st);
  kern<<<grid, 64 + kWorkers, smem, st>>>(tm, p);
  prof_launch_end(st, SSC_PROF_LIN_ROWS);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_lin_prep(const float* dO, int lddo, const float* O, int ldo, const float* den,
                            int n, int k, __nv_bfloat16* Y, int ldy, cudaStream_t st) {
  const int blocks = std::max(1, std::min((n + 7) / 8, lin_num_sms() * 16));
  lin_prep_kernel<<<blocks, 256, 0, st>>>(dO, lddo, O, ldo, den, n, k, Y, ldy);
  count_launch();
  return cudaGetLastError();
}

}  // namespace ssc
