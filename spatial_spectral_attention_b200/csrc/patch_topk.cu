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
#include "ssc.h"

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

// Row-staged pooling (rows of d * esize bytes, a multiple of 16, 16-byte
// aligned): the block copies the patch's member rows into shared memory with
// cp.async (16-byte pieces, kPoolRows rows per buffer, two buffers), so every
// load of a chunk is in flight at once; each thread then adds its channels
// over the staged rows strictly in member order (bit-identical to pool_kernel).
constexpr int kPoolRows = 64;
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// One shape's pooling job: descriptors F [n, ld], patch tables off/mem, P
// patches, means mu [P, d].
struct PoolSet {
  const void* F;
  const int* off;
  const int* mem;
  double* mu;
  int ld, n, P;
};

// Blocks [0, set_a.P) pool the first shape, the next set_b.P blocks the second.
template <bool F32>
__global__ void __launch_bounds__(128) pool_rows_kernel(const PoolSet set_a, const PoolSet set_b,
                                                        int d, unsigned* status) {
  constexpr int kEsz = F32 ? 4 : 2;
  extern __shared__ __align__(16) uint8_t s_rows[];  // [2][kPoolRows][d * kEsz]
  __shared__ int s_mem[kPoolStage];
  const bool second = (int)blockIdx.x >= set_a.P;
  const PoolSet& S = second ? set_b : set_a;
  const int p = second ? blockIdx.x - set_a.P : blockIdx.x;
  const void* __restrict__ F = S.F;
  const int ld = S.ld, n = S.n;
  const int* __restrict__ off = S.off;
  const int* __restrict__ mem = S.mem;
  double* __restrict__ mu = S.mu;
  int b = off[p], e = off[p + 1];
  if (b < 0 || e <= b || e > n) {
    if (threadIdx.x == 0) atomicOr(status, kStatusBadIndex);
    b = min(max(b, 0), n);
    e = min(max(e, b), n);
  }
  const int rowb = d * kEsz;
  const int pieces = rowb / 16;
  const uint8_t* Fb = static_cast<const uint8_t*>(F);
  const uint32_t sbase = smem_u32(s_rows);
  const int c0 = threadIdx.x, c1 = threadIdx.x + 128;  // this thread's channels (d <= 256)
  double s0 = 0.0, s1 = 0.0;
  for (int r0 = b; r0 < e; r0 += kPoolStage) {
    const int nr = min(kPoolStage, e - r0);
    __syncthreads();  // the previous pass is done with s_mem and the row buffers
    for (int i = threadIdx.x; i < nr; i += blockDim.x) {
      int v = mem[r0 + i];
      if (v < 0 || v >= n) {
        atomicOr(status, kStatusBadIndex);
        v = -1;
      }
      s_mem[i] = v;
    }
    __syncthreads();
    const int nch = (nr + kPoolRows - 1) / kPoolRows;
    auto issue = [&](int k) {
      const uint32_t buf = sbase + (uint32_t)((k & 1) * kPoolRows * rowb);
      const int rows = min(kPoolRows, nr - k * kPoolRows);
      for (int i = threadIdx.x; i < rows * pieces; i += blockDim.x) {
        const int r = i / pieces, pc = i - r * pieces;
        const int v = s_mem[k * kPoolRows + r];
        if (v >= 0) cp_async16(buf + r * rowb + pc * 16, Fb + ((size_t)v * ld * kEsz + pc * 16));
      }
      cp_async_commit();
    };
    issue(0);
    for (int k = 0; k < nch; ++k) {
      if (k + 1 < nch) {
        issue(k + 1);
        cp_async_wait<1>();  // chunk k has landed (this thread's copies)
      } else {
        cp_async_wait<0>();
      }
      __syncthreads();  // ... and every thread's
      const uint8_t* buf = s_rows + (k & 1) * kPoolRows * rowb;
      const int rows = min(kPoolRows, nr - k * kPoolRows);
      auto elem = [&](int r, int c) -> double {
        const uint8_t* row = buf + r * rowb;
        if constexpr (F32) return (double)reinterpret_cast<const float*>(row)[c];
        else return (double)__bfloat162float(reinterpret_cast<const __nv_bfloat16*>(row)[c]);
      };
      // eight rows' values read ahead, then added strictly in row order
      for (int r0 = 0; r0 < rows; r0 += 8) {
        double x0[8], x1[8];
        bool ok[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int r = r0 + u;
          ok[u] = r < rows && s_mem[k * kPoolRows + r] >= 0;
          x0[u] = (ok[u] && c0 < d) ? elem(r, c0) : 0.0;
          x1[u] = (ok[u] && c1 < d) ? elem(r, c1) : 0.0;
        }
#pragma unroll
        for (int u = 0; u < 8; ++u)
          if (ok[u]) {
            if (c0 < d) s0 = __dadd_rn(s0, x0[u]);
            if (c1 < d) s1 = __dadd_rn(s1, x1[u]);
          }
      }
      __syncthreads();  // buffer k & 1 is refilled by issue(k + 2)
    }
  }
  const double cnt = (double)max(e - b, 1);
  if (c0 < d) mu[(size_t)p * d + c0] = __ddiv_rn(s0, cnt);
  if (c1 < d) mu[(size_t)p * d + c1] = __ddiv_rn(s1, cnt);
}

// fp32 -> fp64 from the bits, on the integer pipe (exact, like the
// conversion instruction): a normal number keeps its sign and mantissa and
// moves its exponent from the 127 to the 1023 bias; zeros, subnormals,
// infinities and NaNs take the conversion instruction.
__device__ __forceinline__ double widen_f32_bits(uint32_t u) {
  const uint32_t e = (u >> 23) & 0xffu;
  if (e - 1u < 254u)
    return __longlong_as_double((long long)(((unsigned long long)(u >> 31) << 63) |
                                            ((unsigned long long)(e + 896u) << 52) |
                                            ((unsigned long long)(u & 0x7fffffu) << 29)));
  return (double)__uint_as_float(u);
}

// Warp-sliced pooling for d = 32 CPL WPP: the WPP warps of a patch each take a
// slice of 32 CPL channels, and each lane sums its CPL channels as CPL
// independent chains, strictly in member order (bit-identical to
// pool_kernel).  A warp stages its slice of the member rows in shared memory
// with cp.async, kWarpRows rows per chunk and two chunks in flight; member
// indices go through shared memory too.  Four warps per block, both shapes in
// one launch.
constexpr int kWarpRows = 32;
template <bool F32, int CPL, int WPP>
__global__ void __launch_bounds__(128) pool_warp_kernel(const PoolSet set_a, const PoolSet set_b,
                                                        unsigned* status) {
  constexpr int kEsz = F32 ? 4 : 2;
  constexpr int kRowB = 32 * CPL * kEsz;    // bytes of this warp's slice of a row
  constexpr int kPieces = kRowB / 16;       // 16-byte pieces per slice
  constexpr int kChunkB = kWarpRows * kRowB;
  static_assert(kRowB % 16 == 0, "a slice is whole 16-byte pieces");
  extern __shared__ __align__(16) uint8_t s_pool[];  // [4 warps][2][kWarpRows][kRowB]
  __shared__ int s_idx[4][2][kWarpRows];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gw = blockIdx.x * 4 + warp;
  const int gp = gw / WPP, slice = gw % WPP;
  if (gp >= set_a.P + set_b.P) return;  // warp-uniform; no block barrier below
  const bool second = gp >= set_a.P;
  const PoolSet& S = second ? set_b : set_a;
  const int p = second ? gp - set_a.P : gp;
  const int n = S.n;
  const int* __restrict__ mem = S.mem;
  const uint8_t* Fb = static_cast<const uint8_t*>(S.F) + slice * kRowB;
  const size_t ldb = (size_t)S.ld * kEsz;
  int b = S.off[p], e = S.off[p + 1];
  if (b < 0 || e <= b || e > n) {
    if (lane == 0 && slice == 0) atomicOr(status, kStatusBadIndex);
    b = min(max(b, 0), n);
    e = min(max(e, b), n);
  }
  const int rows = e - b;
  const int nch = (rows + kWarpRows - 1) / kWarpRows;
  uint8_t* wbuf = s_pool + warp * 2 * kChunkB;
  const uint32_t wbase = smem_u32(wbuf);
  // the member indices of the first 8 chunks, all loaded up front
  constexpr int kPre = 8;
  int pre[kPre];
#pragma unroll
  for (int j = 0; j < kPre; ++j) {
    const int r = b + j * kWarpRows + lane;
    pre[j] = r < e ? mem[r] : -1;
  }
  auto issue = [&](int k) {
    const int r0 = b + k * kWarpRows;
    int v = -1;
    if (r0 + lane < e) {
      if (k < kPre) {
#pragma unroll
        for (int j = 0; j < kPre; ++j)
          if (j == k) v = pre[j];
      } else {
        v = mem[r0 + lane];
      }
      if (v < 0 || v >= n) {
        if (slice == 0) atomicOr(status, kStatusBadIndex);
        v = -1;
      }
    }
    s_idx[warp][k & 1][lane] = v;
    __syncwarp();
    const uint32_t buf = wbase + (k & 1) * kChunkB;
#pragma unroll
    for (int j = 0; j < kWarpRows * kPieces / 32; ++j) {
      const int i = lane + 32 * j;
      const int r = i / kPieces, pc = i % kPieces;
      const int vr = s_idx[warp][k & 1][r];
      if (vr >= 0) cp_async16(buf + r * kRowB + pc * 16, Fb + (size_t)vr * ldb + pc * 16);
    }
    cp_async_commit();
  };
  double acc[CPL];
#pragma unroll
  for (int c = 0; c < CPL; ++c) acc[c] = 0.0;
  if (nch > 0) issue(0);
  for (int k = 0; k < nch; ++k) {
    if (k + 1 < nch) {
      issue(k + 1);
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncwarp();  // every lane's copies of chunk k are visible
    const uint8_t* buf = wbuf + (k & 1) * kChunkB + lane * CPL * kEsz;
    const int nr = min(kWarpRows, rows - k * kWarpRows);
    for (int r0 = 0; r0 < nr; r0 += 8) {
      double x[8][CPL];
      bool ok[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int r = r0 + u;
        ok[u] = r < nr && s_idx[warp][k & 1][r] >= 0;  // the same for every lane
        // the element bits as fp32 (bf16 -> fp32 is exact: the bf16 bits are
        // the high half of the float), widened to fp64 exactly
        uint32_t h[CPL];
        if constexpr (F32) {
          if constexpr (CPL == 1) {
            h[0] = ok[u] ? *reinterpret_cast<const uint32_t*>(buf + r * kRowB) : 0u;
          } else {
            const uint2 t = ok[u] ? *reinterpret_cast<const uint2*>(buf + r * kRowB) : make_uint2(0u, 0u);
            h[0] = t.x;
            h[1] = t.y;
          }
        } else {
          if constexpr (CPL == 1) {
            h[0] = ok[u] ? (uint32_t)*reinterpret_cast<const uint16_t*>(buf + r * kRowB) << 16 : 0u;
          } else {
            const uint32_t w = ok[u] ? *reinterpret_cast<const uint32_t*>(buf + r * kRowB) : 0u;
            h[0] = w << 16;
            h[1] = w & 0xffff0000u;
          }
        }
#pragma unroll
        for (int c = 0; c < CPL; ++c) x[u][c] = widen_f32_bits(h[c]);
      }
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (ok[u]) {
#pragma unroll
          for (int c = 0; c < CPL; ++c) acc[c] = __dadd_rn(acc[c], x[u][c]);
        }
    }
    __syncwarp();  // chunk k's buffer is refilled by issue(k + 2)
  }
  const double cnt = (double)max(e - b, 1);
#pragma unroll
  for (int c = 0; c < CPL; ++c)
    S.mu[(size_t)p * 32 * CPL * WPP + slice * 32 * CPL + lane * CPL + c] = __ddiv_rn(acc[c], cnt);
}

constexpr int kST = 32;  // score tile (target x source patches)
constexpr int kSC = 128;  // channels staged per step (one load phase for d <= 128)

// scores[p, q] for a 32 x 32 tile per block; each thread owns 4 outputs and
// sums its products strictly in channel order.  blockIdx.z selects the pair of
// a batch (its means and score block follow the previous pair's).
__global__ void __launch_bounds__(256, 2) scores_kernel(const double* __restrict__ muN, int PN,
                                                     const double* __restrict__ muM, int PM, int d,
                                                     double* __restrict__ sc) {
  muN += (size_t)blockIdx.z * PN * d;
  muM += (size_t)blockIdx.z * PM * d;
  sc += (size_t)blockIdx.z * PN * PM;
  extern __shared__ double s_ab[];  // a[kST][kSC + 1], then b[kST][kSC + 1]
  double(*a)[kSC + 1] = reinterpret_cast<double(*)[kSC + 1]>(s_ab);
  double(*b)[kSC + 1] = reinterpret_cast<double(*)[kSC + 1]>(s_ab + kST * (kSC + 1));
  const int p0 = blockIdx.y * kST, q0 = blockIdx.x * kST;
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;  // 8 rows of threads
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
  for (int c0 = 0; c0 < d; c0 += kSC) {
    // all of this thread's loads in flight before the first store
    double va[kST * kSC / 256], vb[kST * kSC / 256];
#pragma unroll
    for (int j = 0; j < kST * kSC / 256; ++j) {
      const int i = threadIdx.x + 256 * j;
      const int r = i / kSC, cc = i % kSC;
      va[j] = (p0 + r < PN && c0 + cc < d) ? muN[(size_t)(p0 + r) * d + c0 + cc] : 0.0;
      vb[j] = (q0 + r < PM && c0 + cc < d) ? muM[(size_t)(q0 + r) * d + c0 + cc] : 0.0;
    }
#pragma unroll
    for (int j = 0; j < kST * kSC / 256; ++j) {
      const int i = threadIdx.x + 256 * j;
      a[i / kSC][i % kSC] = va[j];
      b[i / kSC][i % kSC] = vb[j];
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

// One warp per target patch, eight per block: round r scans the score row for
// the best candidate ranked after the round r-1 winner and the warp agrees on
// it by xor-shuffles (every lane ends with the winner), so no block barrier is
// needed.  Because each round only admits candidates ranked after the previous
// winner, no candidate needs marking.
// The lane's share of the row (q = lane + 32 i) is read once into registers
// when it fits (PM <= 32 kTopkRegs); otherwise every round re-reads the row.
constexpr int kTopkRegs = 40;
__global__ void __launch_bounds__(64) topk_warp_kernel(const double* __restrict__ sc, int PN, int PM,
                                                       int R, int* __restrict__ topk) {
  const int lane = threadIdx.x & 31;
  const int p = blockIdx.x * 2 + (threadIdx.x >> 5);
  if (p >= PN) return;  // warp-uniform
  const double* row = sc + (size_t)p * PM;
  const bool in_regs = PM <= 32 * kTopkRegs;
  double v[kTopkRegs];
  if (in_regs) {
#pragma unroll
    for (int i = 0; i < kTopkRegs; ++i) v[i] = lane + 32 * i < PM ? row[lane + 32 * i] : 0.0;
  }
  Pick prev{DBL_MAX, -1};
  for (int r = 0; r < R; ++r) {
    Pick mine{-DBL_MAX, INT_MAX};  // no candidate yet
    if (in_regs) {
#pragma unroll
      for (int i = 0; i < kTopkRegs; ++i) {
        const int q = lane + 32 * i;
        if (q >= PM) break;
        const Pick c{v[i], q};
        if (r > 0 && !pick_before(prev, c)) continue;
        if (mine.q == INT_MAX || pick_before(c, mine)) mine = c;
      }
    } else {
      for (int q = lane; q < PM; q += 32) {
        const Pick c{row[q], q};
        if (r > 0 && !pick_before(prev, c)) continue;
        if (mine.q == INT_MAX || pick_before(c, mine)) mine = c;
      }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      Pick x;
      x.s = __shfl_xor_sync(0xffffffffu, mine.s, o);
      x.q = __shfl_xor_sync(0xffffffffu, mine.q, o);
      if (x.q != INT_MAX && (mine.q == INT_MAX || pick_before(x, mine))) mine = x;
    }
    if (lane == 0) topk[(size_t)p * R + r] = mine.q;
    prev = mine;
  }
}

}  // namespace

size_t scores_topk_workspace_bytes(int PN, int PM, int d, int batch) {
  Carve c(nullptr);
  c.take<double>((size_t)batch * PN * d);
  c.take<double>((size_t)batch * PM * d);
  c.take<double>((size_t)batch * PN * PM);
  return c.used + 256;
}

cudaError_t launch_scores_topk(const void* FN, int ldn, int nN, const void* FM, int ldm, int nM,
                               int d, int dtype, const int* offN, const int* memN, int PN,
                               const int* offM, const int* memM, int PM, int R, int* topk,
                               double* scores, void* ws, unsigned* status, cudaStream_t st,
                               int batch) {
  Carve c(ws);
  double* muN = c.take<double>((size_t)batch * PN * d);
  double* muM = c.take<double>((size_t)batch * PM * d);
  double* sc_ws = c.take<double>((size_t)batch * PN * PM);
  double* sc = scores ? scores : sc_ws;
  const int pt = d >= 128 ? 128 : 64;
  const int esz = dtype == 1 ? 4 : 2;
  // rows staged through shared memory when they are whole 16-byte pieces
  auto staged = [&](const void* F, int ld) {
    return d <= 256 && (d * esz) % 16 == 0 && ((size_t)ld * esz) % 16 == 0 &&
           reinterpret_cast<uintptr_t>(F) % 16 == 0;
  };
  const int rows_smem = 2 * kPoolRows * d * esz;
  auto pool = [&](const void* F, int ld, int n, int P, const int* off, const int* mem, double* mu) {
    prof_launch_begin(st);
    if (dtype == 1) pool_kernel<true><<<P, pt, 0, st>>>(F, ld, n, d, off, mem, mu, status);
    else pool_kernel<false><<<P, pt, 0, st>>>(F, ld, n, d, off, mem, mu, status);
    prof_launch_end(st, SSC_PROF_POOL);
    count_launch();
    return cudaGetLastError();
  };
  cudaError_t pe;
  if ((d == 64 || d == 128) && staged(FN, ldn) && staged(FM, ldm)) {
    // one warp per patch, both shapes in one launch
    const PoolSet a{FN, offN, memN, muN, ldn, batch * nN, batch * PN};
    const PoolSet b{FM, offM, memM, muM, ldm, batch * nM, batch * PM};
    // bf16: one channel per lane (d / 32 warps per patch); fp32: two
    // (d / 64 warps per patch), slices of 64 and 256 bytes of each row
    const int cpl = dtype == 1 ? 2 : 1;
    const int wpp = d / (32 * cpl);
    const int smem = 4 * 2 * kWarpRows * 32 * cpl * esz;
    auto kern = dtype == 1 ? (d == 128 ? pool_warp_kernel<true, 2, 2> : pool_warp_kernel<true, 2, 1>)
                           : (d == 128 ? pool_warp_kernel<false, 1, 4> : pool_warp_kernel<false, 1, 2>);
    if ((pe = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
        cudaSuccess)
      return pe;
    const int total = batch * (PN + PM) * wpp;
    prof_launch_begin(st);
    kern<<<(total + 3) / 4, 128, smem, st>>>(a, b, status);
    prof_launch_end(st, SSC_PROF_POOL);
    count_launch();
    if ((pe = cudaGetLastError()) != cudaSuccess) return pe;
  } else if (staged(FN, ldn) && staged(FM, ldm)) {
    // both shapes in one launch, member rows staged through shared memory
    auto kern = dtype == 1 ? pool_rows_kernel<true> : pool_rows_kernel<false>;
    if ((pe = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, rows_smem)) !=
        cudaSuccess)
      return pe;
    const PoolSet a{FN, offN, memN, muN, ldn, batch * nN, batch * PN};
    const PoolSet b{FM, offM, memM, muM, ldm, batch * nM, batch * PM};
    prof_launch_begin(st);
    kern<<<batch * (PN + PM), 128, rows_smem, st>>>(a, b, d, status);
    prof_launch_end(st, SSC_PROF_POOL);
    count_launch();
    if ((pe = cudaGetLastError()) != cudaSuccess) return pe;
  } else {
    if ((pe = pool(FN, ldn, batch * nN, batch * PN, offN, memN, muN)) != cudaSuccess) return pe;
    if ((pe = pool(FM, ldm, batch * nM, batch * PM, offM, memM, muM)) != cudaSuccess) return pe;
  }
  dim3 grid((PM + kST - 1) / kST, (PN + kST - 1) / kST, batch);
  const int sc_smem = 2 * kST * (kSC + 1) * (int)sizeof(double);
  if ((pe = cudaFuncSetAttribute(scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 sc_smem)) != cudaSuccess)
    return pe;
  prof_launch_begin(st);
  scores_kernel<<<grid, 256, sc_smem, st>>>(muN, PN, muM, PM, d, sc);
  prof_launch_end(st, SSC_PROF_SCORES);
  count_launch();
  prof_launch_begin(st);
  topk_warp_kernel<<<(batch * PN + 1) / 2, 64, 0, st>>>(sc, batch * PN, PM, R, topk);
  prof_launch_end(st, SSC_PROF_TOPK);
  count_launch();
  return cudaGetLastError();
}

}  // namespace ssc
