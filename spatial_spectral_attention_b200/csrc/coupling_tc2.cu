// coupling_tc2.cu -- the dense forward coupling on CTA pairs (2-SM tcgen05 MMAs).
//
// Same operation as tc_fwd_kernel ("Spatial-Spectral Coupling as Attention",
// project page, "Spatial-spectral coupling is attention": O = softmax(s Q K^T) V
// with Q = F_N, K = F_M, V = Phi_M, plus lse), laid out for the B200's 2-SM
// tensor-core instructions.  A cluster of two CTAs owns a 256-row query tile;
// CTA r holds query rows [128 r, 128 r + 128) of it.  For every 128-key tile
// each CTA loads only half of the shared operands -- 64 key rows of K and half
// of the (32-padded) V columns -- and the even CTA issues M = 256 MMAs that read
// both halves:
//     S = Q K^T    SS, M = 256, N = 128 keys (each CTA: 64 keys of B)
//     O += P V     TS, P from each CTA's tensor memory, N = kp2 (V padded to a
//                  multiple of 32; each CTA supplies kp2/2 columns of B)
// Each CTA's tensor memory receives its own 128 rows of S and O, so the softmax
// warps of both CTAs run exactly as in the single-CTA kernel.  This halves the
// bytes every SM streams per key tile (K and V traffic is the limit of the
// single-CTA forward) and reduces the shared-memory operand reads per MMA.
//
// Barrier topology: operand "full" barriers and the P-ready barrier live in the
// even CTA (the MMA issuer); TMA loads of both CTAs complete on them.  Every
// "empty"/"ready" signal produced by the MMAs is a commit multicast to both
// CTAs.  All waits are bounded.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <vector>

#include "internal.h"
#include "ssc.h"

namespace ssc {
namespace {

constexpr int kChunk = 128 * 128;     // 128 rows x 64 bf16, 128B-swizzled
constexpr int kHalfChunk = 64 * 128;  // 64 rows x 64 bf16
constexpr int kKS = 4;                // K ring depth
constexpr int kVS = 3;                // V ring depth
constexpr int kNWG = 2;               // softmax warpgroups per CTA (a thread pair owns a row)
constexpr int kMaxPairs = 80;         // CTA pairs the partial-result workspace is sized for
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct PairMaps {
  CUtensorMap q;  // {d, nq}, box {64, 128}
  CUtensorMap k;  // {d, nk}, box {64, 64}: one CTA's half of a key tile
  CUtensorMap v;  // {k, nk}, box {64, 128}
};

struct PairParams {
  int nq, nk, d, k;
  int kp2;     // V columns padded to a multiple of 32 (MMA N of P V)
  int qch;     // d / 64
  int vh;      // V columns supplied by each CTA (kp2 / 2)
  int vbox;    // 64-column boxes per CTA per V tile
  int nkt;     // key tiles of 128
  int ntiles;  // query tiles of 256 rows
  int sum_col;  // V column holding ones (the row sum comes out of P V), or -1
  long long units;  // ntiles * nkt (query tile, key tile) units, split evenly over the pairs
  float scale_log2;
  float* O;
  int ldo;
  float* lse;
  float* part;  // partial results of query tiles split between pairs: 2 slots per pair
  WaitCtl ctl;
};

// Floats of one partial-result slot: unnormalised O [256][kp2], then the running
// max (log2 units) and sum of every row.
__host__ __device__ inline size_t part_slot_floats(int kp2) { return (size_t)256 * kp2 + 512; }

// The (query tile, key tile) units are numbered tile-major and pair c owns
// [c U / P, (c + 1) U / P); a run of consecutive units of one query tile is a
// segment [jb, je) of its key tiles.
__host__ __device__ inline long long pair_first_unit(int c, long long U, int npairs) {
  return (long long)c * U / npairs;
}
struct PairRange {
  long long u, u1;
};
__device__ __forceinline__ bool pair_next(PairRange& r, int nkt, int& t, int& jb, int& je) {
  if (r.u >= r.u1) return false;
  t = (int)(r.u / nkt);
  jb = (int)(r.u - (long long)t * nkt);
  je = (int)min((long long)nkt, jb + (r.u1 - r.u));
  r.u += je - jb;
  return true;
}

// Maximum of N values with the three-input max of sm_100 (N / 2 instructions
// instead of N - 1), as a tree.
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}
template <int N>
__device__ __forceinline__ float max_tree3(const float (&v)[N]) {
  if constexpr (N == 1) {
    return v[0];
  } else if constexpr (N == 2) {
    return fmaxf(v[0], v[1]);
  } else {
    constexpr int M = (N + 2) / 3;
    float w[M];
#pragma unroll
    for (int i = 0; i < N / 3; ++i) w[i] = fmax3(v[3 * i], v[3 * i + 1], v[3 * i + 2]);
    if constexpr (N % 3 == 1) w[N / 3] = v[N - 1];
    if constexpr (N % 3 == 2) w[N / 3] = fmaxf(v[N - 2], v[N - 1]);
    return max_tree3<M>(w);
  }
}

// D16 > 0 fixes d = 16 D16 at compile time so the S = Q K^T issue loop is fully
// unrolled (a run-time trip count slows the single issuing thread); D16 = 0
// takes d from the parameters.  kSumCol: V carries a column of ones at
// p.sum_col, so O's column sum_col is the softmax row sum (of the bf16 P that
// the MMA multiplies) and the softmax threads do not add it up.
template <int NWG, int D16, bool kSumCol>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(96 + 128 * NWG, 1)
    tc_fwd_pair_kernel(const __grid_constant__ PairMaps tm, const PairParams p) {
  const int d16 = D16 > 0 ? D16 : p.d / 16;
  constexpr int NSM = 128 * NWG;
  constexpr int kVWarp = 2 + 4 * NWG;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_q_full, bar_q_empty, bar_k_full[kKS], bar_k_empty[kKS], bar_v_full[kVS],
      bar_v_empty[kVS], bar_s_full[2], bar_p_full[2], bar_o_full[2], bar_drain;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const uint32_t base_u = smem_u32(smem_raw);
  const uint32_t sbase = (base_u + 1023u) & ~1023u;
  auto gptr = [&](uint32_t sa) { return smem_raw + (sa - base_u); };
  const int qbytes = p.qch * kChunk;
  const int kbytes = p.qch * kHalfChunk;
  const int vbytes = p.vbox * kChunk;
  const uint32_t sQ = sbase;
  const uint32_t sK0 = sQ + qbytes;
  const uint32_t sV0 = sK0 + kKS * kbytes;
  // barriers of the even CTA, as cluster addresses
  auto lead = [&](uint64_t* b) { return mapa_shared(smem_u32(b), 0); };

  if (threadIdx.x == 0) {
    mbar_init(&bar_q_full, 1);
    mbar_init(&bar_q_empty, 1);
    for (int i = 0; i < kKS; ++i) {
      mbar_init(&bar_k_full[i], 1);
      mbar_init(&bar_k_empty[i], 1);
    }
    for (int i = 0; i < kVS; ++i) {
      mbar_init(&bar_v_full[i], 1);
      mbar_init(&bar_v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_s_full[i], 1);
      mbar_init(&bar_p_full[i], 2 * (NSM / 32));  // one arrival per softmax warp of both CTAs
    }
    mbar_init(&bar_o_full[0], 1);
    mbar_init(&bar_o_full[1], 1);
    mbar_init(&bar_drain, 1);
    s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(&s_tmem, 512);
    tmem_relinquish_pair();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm.q);
    tma_prefetch_desc(&tm.k);
    tma_prefetch_desc(&tm.v);
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync_all();  // both CTAs' barriers exist before any remote operation
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort = &s_abort;
  const long long u_first = pair_first_unit(pair, p.units, npairs);
  const long long u_end = pair_first_unit(pair + 1, p.units, npairs);

  if (warp == 0) {
    // ---------------- Q and K producer (both CTAs)
    if (lane == 0) {
      uint32_t it = 0, tcount = 0;
      PairRange rr{u_first, u_end};
      int t, jb, je;
      for (; !*abort && pair_next(rr, p.nkt, t, jb, je); ++tcount) {
        const int row0 = t * 256 + 128 * (int)rank;
        if (tcount > 0 && !mbar_wait(&bar_q_empty, (tcount - 1) & 1, p.ctl, abort)) break;
        if (rank == 0) mbar_arrive_expect_tx(&bar_q_full, 2 * qbytes);
        for (int c = 0; c < p.qch; ++c)
          tma_load_2d_pair(gptr(sQ) + c * kChunk, &tm.q, 64 * c, row0, lead(&bar_q_full));
        bool ok = true;
        for (int j = jb; j < je; ++j, ++it) {
          const int st = it % kKS;
          if (it >= (uint32_t)kKS &&
              !mbar_wait(&bar_k_empty[st], ((it / kKS) - 1) & 1, p.ctl, abort)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&bar_k_full[st], 2 * kbytes);
          for (int c = 0; c < p.qch; ++c)
            tma_load_2d_pair(gptr(sK0) + st * kbytes + c * kHalfChunk, &tm.k, 64 * c,
                             j * 128 + 64 * (int)rank, lead(&bar_k_full[st]));
        }
        if (!ok) break;
      }
      if (*abort) __nanosleep(20000);  // let copies already in flight land
    }
  } else if (warp == kVWarp) {
    // ---------------- V producer (both CTAs): this CTA's kp2/2 columns
    if (lane == 0) {
      uint32_t it = 0;
      PairRange rr{u_first, u_end};
      int t, jb, je;
      while (!*abort && pair_next(rr, p.nkt, t, jb, je)) {
        bool ok = true;
        for (int j = jb; j < je; ++j, ++it) {
          const int st = it % kVS;
          if (it >= (uint32_t)kVS &&
              !mbar_wait(&bar_v_empty[st], ((it / kVS) - 1) & 1, p.ctl, abort)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&bar_v_full[st], 2 * vbytes);
          for (int b = 0; b < p.vbox; ++b)
            tma_load_2d_pair(gptr(sV0) + st * vbytes + b * kChunk, &tm.v,
                             p.vh * (int)rank + 64 * b, j * 128, lead(&bar_v_full[st]));
        }
        if (!ok) break;
      }
      if (*abort) __nanosleep(20000);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer (even CTA only)
    if (lane == 0 && rank == 0) {
      const uint32_t idesc_s = make_idesc_bf16(256, 128, 0, 0);
      const uint32_t idesc_pv = make_idesc_bf16(256, p.kp2, 0, 1);
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      auto issue_s = [&](uint32_t g) -> bool {
        const int st = g % kKS;
        if (!mbar_wait(&bar_k_full[st], (g / kKS) & 1, p.ctl, abort)) return false;
        tc_fence_after();
        const uint32_t sk = sK0 + st * kbytes;
        const uint32_t d_tmem = tmem + (g & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < d16; ++kk) {
          const uint32_t ch = kk >> 2, w = (kk & 3) * 32;
          mma_ss_pair(d_tmem, make_sdesc(sQ + ch * kChunk + w, 16, 1024, kSw128),
                      make_sdesc(sk + ch * kHalfChunk + w, 16, 1024, kSw128), idesc_s, kk > 0);
        }
        mma_commit_pair(&bar_s_full[g & 1]);
        mma_commit_pair(&bar_k_empty[st]);
        return true;
      };
      PairRange rr{u_first, u_end};
      int t, jb, je;
      for (; ok && pair_next(rr, p.nkt, t, jb, je); ++tcount) {
        const int nk = je - jb;
        if (!mbar_wait(&bar_q_full, tcount & 1, p.ctl, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int j = 0; j < std::min(2, nk) && ok; ++j) ok = issue_s(it + j);
        for (int j = 0; j < nk && ok; ++j) {
          const uint32_t g = it + j;
          const int buf = g & 1, vst = g % kVS;
          if (!mbar_wait_cluster(&bar_p_full[buf], (g >> 1) & 1, p.ctl, abort) ||
              !mbar_wait(&bar_v_full[vst], (g / kVS) & 1, p.ctl, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sv = sV0 + vst * vbytes;
          for (int kk = 0; kk < 8; ++kk)
            mma_ts_pair(tmem + 256, tmem + buf * 128 + kk * 8,
                        make_sdesc(sv + kk * 2048, kChunk, 1024, kSw128), idesc_pv,
                        (j > 0 || kk > 0) ? 1u : 0u);
          mma_commit_pair(&bar_v_empty[vst]);
          mma_commit_pair(&bar_o_full[g & 1]);
          if (j + 2 < nk) ok = issue_s(g + 2);
        }
        mma_commit_pair(&bar_q_empty);
        it += nk;
      }
      mma_commit_pair(&bar_drain);
      volatile int never = 0;
      mbar_wait(&bar_drain, 0, p.ctl, &never);
    }
  } else {
    // ---------------- softmax / correction / epilogue (both CTAs)
    // Two warpgroups share every 32-lane TMEM quarter: warpgroup w takes lanes
    // [16 w, 16 w + 16) of each quarter (.16x32bx2 accesses) and the two halves of
    // a warp split each of those rows' 128 columns, thread half h holding S
    // columns [64 h, 64 h + 64).  A row's max then takes one shuffle and no
    // exchange between warpgroups, and every SMSP runs two softmax warps.  O is
    // handled in 32-column chunks, half h taking the 16 columns at 32 c + 16 h.
    static_assert(NWG == 2, "the softmax layout below is for two warpgroups");
    const int wg = (warp - 2) >> 2;
    const int half = lane >> 4;
    const int lrow = 32 * (warp & 3) + 16 * wg + (lane & 15);  // TMEM lane = query row in the CTA
    const uint32_t tl = tmem + ((uint32_t)(32 * (warp & 3) + 16 * wg) << 16);
    const int nchunk2 = p.kp2 / 32;
    uint32_t it = 0, tcount = 0;
    PairRange rr{u_first, u_end};
    int t, jb, je;
    for (; pair_next(rr, p.nkt, t, jb, je); ++tcount) {
      const int row0 = t * 256 + 128 * (int)rank;
      const int nk = je - jb;
      float m = -INFINITY, l = 0.f;
      bool ok = true;
      int o_done = 0;  // P V of this segment's key tiles [0, o_done) waited for
      auto wait_pv = [&](int t2) {
        const uint32_t g2 = it + t2;
        return mbar_wait(&bar_o_full[g2 & 1], (g2 >> 1) & 1, p.ctl, abort);
      };
      for (int jj = 0; jj < nk; ++jj) {
        const uint32_t g = it + jj;
        const int buf = g & 1;
        const int nkeys = min(128, p.nk - 128 * (jb + jj));
        if (!mbar_wait(&bar_s_full[buf], (g >> 1) & 1, p.ctl, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        float x[64];  // S columns 64 half + i
        tmem_ld16x2_32<64>(tl + buf * 128, reinterpret_cast<uint32_t(&)[32]>(x[0]));
        tmem_ld16x2_32<64>(tl + buf * 128 + 32, reinterpret_cast<uint32_t(&)[32]>(x[32]));
        tmem_ld_wait();
        if (nkeys < 128) {
#pragma unroll
          for (int i = 0; i < 64; ++i)
            if (64 * half + i >= nkeys) x[i] = -INFINITY;
        }
        float mx = max_tree3<64>(x);
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 16));
        const float m_new = fmaxf(m, mx * p.scale_log2);
        const bool need = m_new > m + 8.0f;
        // O-complete waits.  The P V of key tile g commits to bar_o_full[g & 1];
        // a parity wait for it is exact while the P V two tiles later cannot have
        // completed yet, which holds for every P V before the current tile's
        // (that one needs this thread's P first).  Each P V is waited for once,
        // in order: normally two tiles behind, where it never blocks; rescaling O
        // needs the previous tile's P V complete first.
        if (jj > 0 && __any_sync(0xffffffffu, need)) {
          bool waited = true;
          for (; o_done < jj; ++o_done)
            if (!wait_pv(o_done)) {
              waited = false;
              break;
            }
          if (!waited) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float f = need ? ex2_approx(m - m_new) : 1.0f;
          for (int c = 0; c < nchunk2; ++c) {
            uint32_t o[16];
            tmem_ld16x2_16<16>(tl + 256 + 32 * c, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
            tmem_st16x2_16<16>(tl + 256 + 32 * c, o);
          }
          tmem_st_wait();
          l *= f;
          if (need) m = m_new;
        } else if (need) {
          m = m_new;
        }
        const float neg_m = -m;
        float rs[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t pk[2][16];  // P as bf16 pairs: words [32 half, 32 half + 32) of the row
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const float a0 = ex2_approx(fmaf(x[2 * i], p.scale_log2, neg_m));
          const float a1 = ex2_approx(fmaf(x[2 * i + 1], p.scale_log2, neg_m));
          if (!kSumCol) rs[i & 3] += a0 + a1;
          pk[i >> 4][i & 15] = pack_bf16x2(a0, a1);
        }
        l += (rs[0] + rs[1]) + (rs[2] + rs[3]);
        tmem_st16x2_16<32>(tl + buf * 128, pk[0]);
        tmem_st16x2_16<32>(tl + buf * 128 + 16, pk[1]);
        tmem_st_wait();
        if (o_done + 2 <= jj) {
          // the P V of two key tiles back
          if (!wait_pv(o_done)) {
            ok = false;
            break;
          }
          ++o_done;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (rank == 0) mbar_arrive(&bar_p_full[buf]);
          else mbar_arrive_remote(lead(&bar_p_full[buf]));
        }
      }
      if (!ok) break;
      // the remaining P V of the segment, in order, end with the last one
      for (; o_done < nk; ++o_done)
        if (!wait_pv(o_done)) {
          ok = false;
          break;
        }
      if (!ok) break;
      tc_fence_after();
      if (kSumCol) {
        // the row sum is O's column sum_col: read at split 1 from column
        // sum_col - 1 (half 0) and sum_col (half 1), which keeps the access
        // inside TMEM for every k, and taken from half 1
        const uint32_t lv = tmem_ld16x2_1<1>(tl + 256 + p.sum_col - 1);
        tmem_ld_wait();
        l = __shfl_sync(0xffffffffu, __uint_as_float(lv), (lane & 15) + 16);
      } else {
        l += __shfl_xor_sync(0xffffffffu, l, 16);
      }
      const int row = row0 + lrow;
      const bool live = row < p.nq;
      if (jb == 0 && je == p.nkt) {
        // every key tile of this query tile was processed here: O / l and lse
        float* optr = p.O + (size_t)(live ? row : 0) * p.ldo;
        const float inv = 1.0f / l;
        for (int c = 0; c < nchunk2; ++c) {
          uint32_t o[16];
          tmem_ld16x2_16<16>(tl + 256 + 32 * c, o);
          tmem_ld_wait();
          if (live) {
            const int c0 = 32 * c + 16 * half;
            if (c0 + 16 <= p.k && (p.ldo & 3) == 0) {
#pragma unroll
              for (int i = 0; i < 16; i += 4)
                *reinterpret_cast<float4*>(optr + c0 + i) =
                    make_float4(__uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv,
                                __uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i)
                if (c0 + i < p.k) optr[c0 + i] = __uint_as_float(o[i]) * inv;
            }
          }
        }
        if (live && half == 0) p.lse[row] = (m + log2f(l)) * kLn2;
      } else {
        // the query tile's key tiles are split between pairs: the unnormalised
        // O, the running max and the sum go to this pair's slot for the merge
        // (slot 0: the first query tile of the pair's range, 1: the last)
        const int slot = 2 * pair + ((long long)t == u_first / p.nkt ? 0 : 1);
        float* ps = p.part + (size_t)slot * part_slot_floats(p.kp2);
        const int prow = 128 * (int)rank + lrow;
        float* po = ps + (size_t)prow * p.kp2;
        for (int c = 0; c < nchunk2; ++c) {
          uint32_t o[16];
          tmem_ld16x2_16<16>(tl + 256 + 32 * c, o);
          tmem_ld_wait();
          const int c0 = 32 * c + 16 * half;
#pragma unroll
          for (int i = 0; i < 16; i += 4)
            *reinterpret_cast<float4*>(po + c0 + i) =
                make_float4(__uint_as_float(o[i]), __uint_as_float(o[i + 1]),
                            __uint_as_float(o[i + 2]), __uint_as_float(o[i + 3]));
        }
        if (half == 0) {
          ps[(size_t)256 * p.kp2 + prow] = m;
          ps[(size_t)256 * p.kp2 + 256 + prow] = l;
        }
      }
      it += nk;
    }
  }

  __syncthreads();
  cluster_sync_all();  // no CTA leaves while its peer's MMAs or signals may target it
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

// Merges the pieces of every query tile whose key tiles were split between
// pairs (the per-pair results are exact softmax-weighted sums over their key
// tiles, relative to their own running max m_q, log2 units):
//   m = max_q m_q,  l = sum_q l_q 2^(m_q - m),  O = sum_q O_q 2^(m_q - m) / l,
//   lse = (m + log2 l) ln 2.
// Block (c, y) looks at the boundary between pair c and pair c + 1; the first
// boundary inside a query tile merges that tile.  The block covers 32 of the
// tile's 256 rows; eight threads share a row, each taking every eighth float4
// of it, so the loads of a row are contiguous.
constexpr int kMergeRows = 32;
__global__ void __launch_bounds__(256) pair_merge_kernel(const PairParams p, int npairs) {
  const int c = blockIdx.x;
  const long long U = p.units;
  const long long b = pair_first_unit(c + 1, U, npairs);
  if (b >= U || b % p.nkt == 0) return;  // the boundary is not inside a query tile
  const int t = (int)(b / p.nkt);
  const long long t0 = (long long)t * p.nkt, t1 = t0 + p.nkt;
  if (pair_first_unit(c, U, npairs) > t0) return;  // an earlier boundary lies in this tile
  const int row = blockIdx.y * kMergeRows + (threadIdx.x >> 3);
  const int part = threadIdx.x & 7;
  const int grow = t * 256 + row;
  if (grow >= p.nq) return;
  int q0 = c;  // the pair holding the tile's first unit
  while (q0 > 0 && pair_first_unit(q0, U, npairs) > t0) --q0;
  const size_t slot_f = part_slot_floats(p.kp2);
  auto piece = [&](int q) -> const float* {
    const int slot = 2 * q + (pair_first_unit(q, U, npairs) / p.nkt == t ? 0 : 1);
    return p.part + (size_t)slot * slot_f;
  };
  const size_t stat = (size_t)256 * p.kp2;  // row maxima, then row sums
  float m = -INFINITY;
  for (int q = q0; q < npairs && pair_first_unit(q, U, npairs) < t1; ++q)
    m = fmaxf(m, piece(q)[stat + row]);
  float l = 0.f;
  for (int q = q0; q < npairs && pair_first_unit(q, U, npairs) < t1; ++q) {
    const float* ps = piece(q);
    l += ps[stat + 256 + row] * exp2f(ps[stat + row] - m);
  }
  const float inv = 1.0f / l;
  float* optr = p.O + (size_t)grow * p.ldo;
  constexpr int kMaxF4 = 8;  // kp2 <= 256: at most 8 float4 per thread
  float4 acc[kMaxF4];
#pragma unroll
  for (int i = 0; i < kMaxF4; ++i) acc[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int q = q0; q < npairs && pair_first_unit(q, U, npairs) < t1; ++q) {
    const float* ps = piece(q);
    const float w = exp2f(ps[stat + row] - m) * inv;
    const float4* src = reinterpret_cast<const float4*>(ps + (size_t)row * p.kp2);
#pragma unroll
    for (int i = 0; i < kMaxF4; ++i) {
      const int f4 = part + 8 * i;
      if (4 * f4 < p.k) {
        const float4 o = src[f4];
        acc[i].x = fmaf(o.x, w, acc[i].x);
        acc[i].y = fmaf(o.y, w, acc[i].y);
        acc[i].z = fmaf(o.z, w, acc[i].z);
        acc[i].w = fmaf(o.w, w, acc[i].w);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < kMaxF4; ++i) {
    const int c0 = 4 * (part + 8 * i);
    if (c0 >= p.k) continue;
    if (c0 + 4 <= p.k && (p.ldo & 3) == 0) {
      *reinterpret_cast<float4*>(optr + c0) = acc[i];
    } else {
      const float v[4] = {acc[i].x, acc[i].y, acc[i].z, acc[i].w};
      for (int j = 0; j < 4 && c0 + j < p.k; ++j) optr[c0 + j] = v[j];
    }
  }
  if (part == 0) p.lse[grow] = (m + log2f(l)) * kLn2;
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn2() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  }
  return fn;
}

bool map2(CUtensorMap* m, const void* ptr, int rows, int cols, int ld, int box_cols, int box_rows) {
  EncodeTiledFn fn = encode_fn2();
  if (!fn) return false;
  cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), gdim, gstride, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

bool tc_pair_supported(int d, int k) { return (d == 64 || d == 128) && k >= 1 && k <= 256; }

// CTA pairs of one kernel configuration that can be resident at once, per
// device (the occupancy query costs host time that would leave the GPU idle
// between the launches of a call, so its answer is kept).
int resident_pairs(int dev, const void* kern, cudaLaunchConfig_t cfg) {
  struct Entry {
    int dev;
    const void* kern;
    size_t smem;
    int pairs;
  };
  static std::mutex mu;
  static std::vector<Entry> cache;
  std::lock_guard<std::mutex> lock(mu);
  for (const Entry& e : cache)
    if (e.dev == dev && e.kern == kern && e.smem == cfg.dynamicSmemBytes) return e.pairs;
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cfg.gridDim = dim3(2 * std::max(1, sms / 2));
  int nclusters = 0;
  if (cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg) != cudaSuccess || nclusters < 1)
    nclusters = std::max(1, sms / 2);
  cudaGetLastError();
  cache.push_back({dev, kern, cfg.dynamicSmemBytes, nclusters});
  return nclusters;
}

size_t tc_pair_part_floats(int k) {
  return 2 * (size_t)kMaxPairs * part_slot_floats((k + 31) / 32 * 32);
}

cudaError_t launch_tc_fwd_pair(const __nv_bfloat16* Q, int ldq, const __nv_bfloat16* K, int ldk,
                               const __nv_bfloat16* V, int ldv, int nN, int nM, int d, int k,
                               float scale, float* O, int ldo, float* lse, float* part,
                               int sum_col, cudaStream_t st, const WaitCtl& ctl) {
  PairParams p;
  std::memset(&p, 0, sizeof(p));
  p.nq = nN;
  p.nk = nM;
  p.d = d;
  p.k = k;
  p.kp2 = (k + 31) / 32 * 32;
  p.qch = d / 64;
  p.vh = p.kp2 / 2;
  p.vbox = (p.vh + 63) / 64;
  p.nkt = (nM + 127) / 128;
  p.ntiles = (nN + 255) / 256;
  p.units = (long long)p.ntiles * p.nkt;
  p.scale_log2 = scale * kLog2e;
  p.O = O;
  p.ldo = ldo;
  p.lse = lse;
  p.part = part;
  p.sum_col = sum_col;
  p.ctl = ctl;
  if (!part) return cudaErrorInvalidValue;
  PairMaps tm;
  std::memset(&tm, 0, sizeof(tm));
  if (!map2(&tm.q, Q, nN, d, ldq, 64, 128) || !map2(&tm.k, K, nM, d, ldk, 64, 64) ||
      !map2(&tm.v, V, nM, sum_col >= 0 ? k + 1 : k, ldv, 64, 128))
    return cudaErrorInvalidValue;
  if (sum_col >= 0 && (sum_col != k || k + 1 > p.kp2)) return cudaErrorInvalidValue;
  auto kern = d == 128 ? (sum_col >= 0 ? tc_fwd_pair_kernel<kNWG, 8, true> : tc_fwd_pair_kernel<kNWG, 8, false>)
                       : (sum_col >= 0 ? tc_fwd_pair_kernel<kNWG, 0, true> : tc_fwd_pair_kernel<kNWG, 0, false>);
  const int smem = 1024 + p.qch * kChunk + kKS * p.qch * kHalfChunk + kVS * p.vbox * kChunk;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  int dev = 0;
  cudaGetDevice(&dev);
  const int threads = 96 + 128 * kNWG;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(threads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  const int nclusters = resident_pairs(dev, reinterpret_cast<const void*>(kern), cfg);
  // every resident pair gets an equal share of the units (at least one)
  const int pairs = (int)std::max<long long>(
      1, std::min<long long>(p.units, std::min(nclusters, kMaxPairs)));
  cfg.gridDim = dim3(2 * pairs);
  count_launch();
  prof_launch_begin(st);
  e = cudaLaunchKernelEx(&cfg, kern, tm, p);
  prof_launch_end(st, SSC_PROF_DENSE_FWD);
  if (e != cudaSuccess || pairs == 1) return e;
  pair_merge_kernel<<<dim3(pairs - 1, 256 / kMergeRows), 256, 0, st>>>(p, pairs);
  count_launch();
  return cudaGetLastError();
}

}  // namespace ssc
