// coupling_tc.cu -- the bf16 coupling on 5th-generation tensor cores (sm_100a).
//
// Operation ("Spatial-Spectral Coupling as Attention", project page, section
// "Spatial-spectral coupling is attention"): O = softmax(s Q K^T) V with
// Q = F_N, K = F_M, V = Phi_M, plus lse; its backward with recompute from lse
// (a training step, section "Results").  Geo-FlashAttention (section
// "Geo-FlashAttention") is the same kernel driven by a different tile
// schedule: each row tile of a target patch visits only the key rows of its
// selected source patches, which the patch-major gather made contiguous.
//
// Work unit: a RowTile (<= 128 query rows) and its list of KeySegs (<= 128
// key rows each).  CTAs are persistent (one per SM: the kernel claims all 512
// TMEM columns) and walk the tile list round-robin.
//
// Forward, per CTA (warp roles):
//   warp 0      TMA producer: Q tile once per row tile, K/V tiles into a
//               2-stage ring (128B-swizzled boxes of 64 columns; the k % 64
//               remainder of V in a 32B/64B-swizzled box).
//   warp 1      MMA issuer (one thread) and TMEM owner:
//                 S_j = Q K_j^T            (SS, K-major x K-major, M=N=128)
//                 O  += P_j V_j            (TS: P from TMEM, V MN-major)
//               with S double-buffered in TMEM columns [0,128) and [128,256)
//               and O in [256, 256+kp).
//   warps 2-5   softmax, one thread per query row (TMEM lane): row max, exp2,
//               row sum, P written back over S as packed bf16; O is rescaled in
//               TMEM only when the running max grows by more than 2^8
//               (otherwise the stale max is kept, which bounds P by 256);
//               epilogue O / l and lse.
// Backward (query-stationary, one row tile per pass, key tiles streamed):
//                 dP_j = dO V_j^T          (SS, K-major, K = kp)
//                 S_j  = Q K_j^T
//   compute     P = exp2(S s log2e - lse log2e), dS = P (dP - D) -> bf16 in a
//               128B-swizzled smem tile [q][keys]
//                 dQ  += dS K_j            (SS, dS K-major, K_j MN-major)
//                 dKp  = dS^T Q            (SS, both MN-major views)
//   compute     dKp (TMEM) -> scale -> fp32 vector atomics into dK
//   end         dQ (TMEM) -> scale -> store.
//   A second pass with kDV computes dV = P^T dO the same way when requested.
//
// Every mbarrier wait is bounded (globaltimer); on expiry the kernel records
// SSC timeout in the status word, every role leaves its loop, the MMA thread
// drains its tensor-core work and TMEM is freed before the CTA exits.
#include <algorithm>
#include <cmath>
#include <cstring>

#include "internal.h"
#include "ssc.h"

namespace ssc {
namespace {

constexpr int kChunk = 128 * 128;  // bytes of a 128-row x 64-col bf16 swizzled box
constexpr int kFwdSoftmaxGroups = 2;  // softmax warpgroups per forward CTA
constexpr int kBwdComputeGroups = 2;  // compute warpgroups per backward CTA
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct TensorMaps {
  CUtensorMap q;     // box {64, 128}, SW128
  CUtensorMap k;     // box {64, 128}, SW128
  CUtensorMap v;     // box {64, 128}, SW128
  CUtensorMap vr;    // box {vr, 128}, SW32/SW64 (remainder columns of V)
  CUtensorMap g;     // dO: box {64, 128}, SW128
  CUtensorMap gr;    // dO remainder
  CUtensorMap dk;    // dK fp32 [nk, d]: box {32, 32}, SW128 (TMA reductions of the partials)
};

struct TcParams {
  const RowTile* tiles;
  const KeySeg* segs;
  const int* ntiles_dev;
  int ntiles_host;
  const int* tile_prefix;  // [ntiles + 1]: units (key segments) before each row tile
  const int* row_map;
  const int* col_map;
  int d, k, kp, qch, vf, vr;
  int nq, nk;        // rows of Q (and of the outputs O, lse, dQ) and of K/V (dK, dV)
  int vstages;       // forward V ring depth
  float scale_log2;  // scale * log2(e)
  const float* qk_dequant;  // fp8 forward: device factor that turns the e4m3 product into Q K^T
  float scale;
  float* O;
  int ldo;
  float* lse;
  // backward
  const float* lse_in;  // row order of Q
  const float* Dvec;
  float* dQ;
  int lddq;
  float* dK;
  int lddk;
  float* dV;
  int lddv;
  const __nv_bfloat16* dOb;  // bf16 dO rows of kp columns (zero padded), row order of Q
  int lddob;
  int vec_atomics;
  int vec_atomics_dq;
  int dk_tma;  // partial dK reduced by TMA through tm.dk (key rows contiguous, no column map)
  int debug_stall;  // abort-path test hook: the MMA issuer waits on a barrier nothing arrives at
  WaitCtl ctl;
};

__device__ __forceinline__ uint32_t tmem_lane_addr(uint32_t base, int warp, uint32_t col) {
  return base + ((uint32_t)(32 * (warp & 3)) << 16) + col;
}

// Bytes of one V (or dO) tile in shared memory: vf full 64-col chunks plus the
// remainder box.
__host__ __device__ inline int vtile_bytes(int vf, int vr) { return vf * kChunk + 128 * vr * 2; }
__host__ __device__ inline uint32_t rem_swizzle(int vr) { return vr == 16 ? kSw32 : kSw64; }

// ------------------------------------------------------------------ forward
// Max of 32 values by a balanced tree (short dependency chain).
__device__ __forceinline__ float max32(const float (&x)[32]) {
  float t[16];
#pragma unroll
  for (int i = 0; i < 16; ++i) t[i] = fmaxf(x[i], x[i + 16]);
#pragma unroll
  for (int w = 8; w > 0; w >>= 1)
#pragma unroll
    for (int i = 0; i < w; ++i) t[i] = fmaxf(t[i], t[i + w]);
  return t[0];
}

// Row tile of this CTA's r-th pass: the tile list is cut into bands of
// gridDim.x tiles walked in alternate directions, so that with the tiles
// sorted by decreasing work (the Geo schedule does that) the passes pair
// long tiles with short ones.  Every index in [0, ntiles) belongs to exactly
// one (CTA, pass); a CTA is done at its first index >= ntiles.
__device__ __forceinline__ int snake_tile(int r) {
  const int G = gridDim.x, c = blockIdx.x;
  return r * G + ((r & 1) ? G - 1 - c : c);
}

// NWG softmax warpgroups split every query row's 128 key columns: thread
// (wg, lane row) owns columns [wg*CW, (wg+1)*CW) of the S tile, CW = 128/NWG.
// QCH > 0 fixes the operand shape at compile time (d = 64 QCH; V rows of VF
// full 64-column chunks plus VR remainder columns) so the MMA issue loops are
// fully unrolled; QCH = 0 reads the shape from the parameters.
//
// kFP8: Q and K arrive as e4m3 copies (d = 128: one 128-byte box per row) and
// S = Q K^T runs as kind::f8f6f4 MMAs (K = 32 per instruction); the product is
// multiplied back to Q K^T by the device factor p.qk_dequant, folded into the
// softmax's exponent scale.  P V stays bf16.
template <int NWG, int QCH, int VF, int VR, bool kFP8>
__global__ void __launch_bounds__(96 + 128 * NWG, 1)
    tc_fwd_kernel(const __grid_constant__ TensorMaps tm, const TcParams p) {
  constexpr bool kFixed = QCH > 0;
  const int qch = kFP8 ? 1 : (kFixed ? QCH : p.qch);
  const int vf = kFixed ? VF : p.vf;
  const int vr = kFixed ? VR : p.vr;
  const int d16 = kFixed ? 4 * QCH : p.d / 16;
  constexpr int CW = 128 / NWG;  // S columns per softmax thread
  constexpr int NC = CW / 32;    // 32-column TMEM loads per thread
  constexpr int NSM = 128 * NWG; // softmax threads
  constexpr int kVWarp = 2 + 4 * NWG;  // warp of the V producer
  // Fixed shape: V arrives as 16-column blocks in the 32-byte swizzle (4 KB
  // each, the layout of the remainder box), so that P.V is one MMA of
  // N = 64 VF + VR per K step instead of one per 64-column chunk plus one
  // N = 16 MMA for the remainder.
  constexpr bool kV32 = kFixed;
  constexpr int kVBlocks = (64 * VF + VR) / 16;
  extern __shared__ uint8_t smem_raw[];
  // A K stage is free when the S MMA that read it completes (bar_s_full of
  // the same index); a V stage when its P.V completes (bar_o_full of the
  // same index with two V stages, bar_v_empty with one).
  __shared__ uint64_t bar_q_full, bar_q_empty, bar_k_full[2], bar_v_full[2], bar_v_empty,
      bar_s_full[2], bar_p_full[2], bar_o_full[2], bar_drain, bar_xmax, bar_xsum, bar_never;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  // Partial row maxima / sums exchanged between the softmax warpgroups through
  // mbarriers (bounded waits, unlike a named barrier).
  __shared__ float s_pmax[2][NWG][128];  // partial row maxima, double-buffered by tile parity
  __shared__ float s_psum[NWG][128];     // partial row sums for the epilogue

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base_u = smem_u32(smem_raw);
  const uint32_t sbase = (base_u + 1023u) & ~1023u;
  auto gptr = [&](uint32_t sa) { return smem_raw + (sa - base_u); };
  const int qbytes = kFP8 ? 128 * 128 : qch * kChunk;  // e4m3: 128 rows x 128 bytes
  const int vbytes = vtile_bytes(vf, vr);
  const int VS = p.vstages;  // V ring depth (1 or 2); the K ring has 2 stages
  const uint32_t sQ = sbase;
  const uint32_t sK0 = sQ + qbytes;
  const uint32_t sV0 = sK0 + 2 * qbytes;
  // epilogue staging: 2 KB per softmax warp, after the V ring
  const uint32_t sStage = sV0 + p.vstages * vbytes;
  const int ntiles = p.ntiles_dev ? *p.ntiles_dev : p.ntiles_host;

  if (threadIdx.x == 0) {
    mbar_init(&bar_q_full, 1);
    mbar_init(&bar_q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_k_full[i], 1);
      mbar_init(&bar_v_full[i], 1);
      mbar_init(&bar_s_full[i], 1);
      mbar_init(&bar_p_full[i], NSM);
      mbar_init(&bar_o_full[i], 1);
    }
    mbar_init(&bar_v_empty, 1);
    mbar_init(&bar_drain, 1);
    mbar_init(&bar_never, 1);  // nothing arrives: the abort-path test hook waits here
    mbar_init(&bar_xmax, NSM);
    mbar_init(&bar_xsum, NSM);
    s_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm.q);
    tma_prefetch_desc(&tm.k);
    tma_prefetch_desc(&tm.v);
    if (vr) tma_prefetch_desc(&tm.vr);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort = &s_abort;

  if (warp == 0) {
    // ---------------- TMA producer: Q once per row tile, K tiles (2-stage ring
    // freed as soon as the S MMA that reads a stage completes)
    if (lane == 0) {
      uint32_t it = 0, tcount = 0;
      int q_issued = -1;
      for (int r = 0, t = snake_tile(0); t < ntiles && !*abort; t = snake_tile(++r), ++tcount) {
        const RowTile tile = p.tiles[t];
        if (tcount > 0 && !mbar_wait(&bar_q_empty, (tcount - 1) & 1, p.ctl, abort)) break;
        mbar_arrive_expect_tx(&bar_q_full, qbytes);
        for (int c = 0; c < qch; ++c)
          tma_load_2d(gptr(sQ) + c * kChunk, &tm.q, 64 * c, tile.row0, &bar_q_full);
        q_issued = (int)tcount;
        bool ok = true;
        for (int j = 0; j < tile.nseg; ++j, ++it) {
          const int key0 = p.segs[tile.seg0 + j].key0;
          const int st = it & 1;
          if (it >= 2 && !mbar_wait(&bar_s_full[st], ((it >> 1) - 1) & 1, p.ctl, abort)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar_k_full[st], qbytes);
          uint8_t* dk = gptr(sK0) + st * qbytes;
          for (int c = 0; c < qch; ++c)
            tma_load_2d(dk + c * kChunk, &tm.k, 64 * c, key0, &bar_k_full[st]);
        }
        if (!ok) break;
      }
      if (*abort) {
        // let the copies already issued land before the CTA can exit
        volatile int never = 0;
        if (q_issued >= 0) mbar_wait(&bar_q_full, q_issued & 1, p.ctl, &never);
        for (uint32_t g = it >= 2 ? it - 2 : 0; g < it; ++g)
          mbar_wait(&bar_k_full[g & 1], (g >> 1) & 1, p.ctl, &never);
      }
    }
  } else if (warp == kVWarp) {
    // ---------------- TMA producer: V tiles (ring freed when the P.V MMA that
    // reads a stage completes)
    if (lane == 0) {
      uint32_t it = 0;
      for (int r = 0, t = snake_tile(0); t < ntiles && !*abort; t = snake_tile(++r)) {
        const RowTile tile = p.tiles[t];
        bool ok = true;
        for (int j = 0; j < tile.nseg; ++j, ++it) {
          const int key0 = p.segs[tile.seg0 + j].key0;
          const int st = it % VS;
          if (it >= (uint32_t)VS && !mbar_wait(VS == 2 ? &bar_o_full[st] : &bar_v_empty,
                                               ((it / VS) - 1) & 1, p.ctl, abort)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar_v_full[st], vbytes);
          uint8_t* dv = gptr(sV0) + st * vbytes;
          if (kV32) {
#pragma unroll
            for (int c = 0; c < kVBlocks; ++c)
              tma_load_2d(dv + c * 4096, &tm.vr, 16 * c, key0, &bar_v_full[st]);
          } else {
            for (int c = 0; c < vf; ++c)
              tma_load_2d(dv + c * kChunk, &tm.v, 64 * c, key0, &bar_v_full[st]);
            if (vr) tma_load_2d(dv + vf * kChunk, &tm.vr, 64 * vf, key0, &bar_v_full[st]);
          }
        }
        if (!ok) break;
      }
      if (*abort) {
        volatile int never = 0;
        for (uint32_t g = it >= (uint32_t)VS ? it - VS : 0; g < it; ++g)
          mbar_wait(&bar_v_full[g % VS], (g / VS) & 1, p.ctl, &never);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = kFP8 ? make_idesc_e4m3(128, 128) : make_idesc_bf16(128, 128, 0, 0);
      const uint32_t idesc_pv = make_idesc_bf16(128, 64 * (vf > 0 ? vf : 1), 0, 1);
      const uint32_t idesc_pvr = make_idesc_bf16(128, vr > 0 ? vr : 16, 0, 1);
      const uint32_t idesc_pv32 = make_idesc_bf16(128, 16 * kVBlocks, 0, 1);
      const uint32_t o_col = tmem + 256;
      const uint32_t rsw = rem_swizzle(vr);
      const uint32_t rrow = (uint32_t)vr * 2;  // bytes per row of the remainder box
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      auto issue_s = [&](uint32_t g) -> bool {
        const int st = g & 1;
        if (!mbar_wait(&bar_k_full[st], (g >> 1) & 1, p.ctl, abort)) return false;
        tc_fence_after();
        const uint32_t sk = sK0 + st * qbytes;
        const uint32_t d_tmem = tmem + (g & 1) * 128;
        if (kFP8) {
          // 4 K-steps of 32 e4m3 values (32 bytes) along the 128-byte rows
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            mma_ss_e4m3(d_tmem, make_sdesc(sQ + kk * 32, 16, 1024, kSw128),
                        make_sdesc(sk + kk * 32, 16, 1024, kSw128), idesc_s, kk > 0);
        } else {
#pragma unroll
          for (int kk = 0; kk < d16; ++kk) {
            const uint32_t off = (kk >> 2) * kChunk + (kk & 3) * 32;
            mma_ss(d_tmem, make_sdesc(sQ + off, 16, 1024, kSw128), make_sdesc(sk + off, 16, 1024, kSw128),
                   idesc_s, kk > 0);
          }
        }
        mma_commit(&bar_s_full[g & 1]);
        return true;
      };
      for (int r = 0, t = snake_tile(0); t < ntiles && ok; t = snake_tile(++r), ++tcount) {
        const RowTile tile = p.tiles[t];
        const int nk = tile.nseg;
        if (!mbar_wait(&bar_q_full, tcount & 1, p.ctl, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int j = 0; j < std::min(2, nk) && ok; ++j) ok = issue_s(it + j);
        // Q is free once the tile's last S MMA completes: the next tile's Q
        // (and its first S MMAs) then overlap this tile's last P.V and epilogue
        if (ok && nk <= 2) mma_commit(&bar_q_empty);
        // abort-path test hook: the bounded wait gives up and raises *abort
        if (ok && p.debug_stall && tcount == 0) ok = mbar_wait(&bar_never, 0, p.ctl, abort);
        for (int j = 0; j < nk && ok; ++j) {
          const uint32_t g = it + j;
          const int buf = g & 1, vst = g % VS;
          if (!mbar_wait(&bar_p_full[buf], (g >> 1) & 1, p.ctl, abort) ||
              !mbar_wait(&bar_v_full[vst], (g / VS) & 1, p.ctl, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sv = sV0 + vst * vbytes;
          const uint32_t a_tmem = tmem + buf * 128;
          if (kV32) {
            // B = V: 16-column blocks 4 KB apart, 8-key groups 256 B apart
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ts(o_col, a_tmem + kk * 8, make_sdesc(sv + kk * 512, 4096, 256, kSw32), idesc_pv32,
                     (j > 0 || kk > 0) ? 1u : 0u);
          } else {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
              if (vf > 0)
                mma_ts(o_col, a_tmem + kk * 8, make_sdesc(sv + kk * 2048, kChunk, 1024, kSw128),
                       idesc_pv, acc);
              if (vr > 0)
                mma_ts(o_col + 64 * vf, a_tmem + kk * 8,
                       make_sdesc(sv + vf * kChunk + kk * 16 * rrow, 128 * rrow, 8 * rrow, rsw),
                       idesc_pvr, acc);
            }
          }
          if (VS == 1) mma_commit(&bar_v_empty);
          mma_commit(&bar_o_full[g & 1]);
          if (j + 2 < nk) {
            ok = issue_s(g + 2);
            if (ok && j + 3 == nk) mma_commit(&bar_q_empty);
          }
        }
        it += nk;
      }
      // drain: wait until every tensor-core op issued here has completed
      mma_commit(&bar_drain);
      volatile int never = 0;
      mbar_wait(&bar_drain, 0, p.ctl, &never);
    }
  } else if (warp >= 2 && warp < kVWarp) {
    // ---------------- softmax / correction / epilogue (NWG warpgroups)
    const int wg = (warp - 2) >> 2;
    const int lrow = 32 * (warp & 3) + lane;  // TMEM lane = row within the tile
    const int col0 = wg * CW;                 // first S column of this thread
    const int nchunk = p.kp / 16;             // 16-column chunks of O
    // exponent scale: s log2(e), times the e4m3 dequantisation factor in fp8 mode
    const float scale_log2 = kFP8 ? p.scale_log2 * *p.qk_dequant : p.scale_log2;
    uint32_t it = 0, tcount = 0;
    for (int r = 0, t = snake_tile(0); t < ntiles; t = snake_tile(++r), ++tcount) {
      const RowTile tile = p.tiles[t];
      const int nk = tile.nseg;
      float m = -INFINITY, l = 0.f;
      bool ok = true;
      int nkeys_next = nk > 0 ? p.segs[tile.seg0].nkeys : 0;
      // output row of this thread (read now, used by the epilogue)
      const int row = tile.row0 + lrow;
      int orow = (lrow < tile.nrows && row < p.nq) ? (p.row_map ? p.row_map[row] : row) : -1;
      for (int j = 0; j < nk; ++j) {
        const uint32_t g = it + j;
        const int buf = g & 1;
        const int nkeys = nkeys_next;
        if (j + 1 < nk) nkeys_next = p.segs[tile.seg0 + j + 1].nkeys;
        if (!mbar_wait(&bar_s_full[buf], (g >> 1) & 1, p.ctl, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // 32-column chunks wholly past the segment's last key (nkeys is uniform
        // over the tile, so these branches are warp-uniform): not loaded, no
        // exponentials, P = 0
        float x[NC][32];
        const uint32_t sa = tmem_lane_addr(tmem, warp, buf * 128 + col0);
#pragma unroll
        for (int c = 0; c < NC; ++c)
          if (col0 + 32 * c < nkeys) tmem_ld32(sa + 32 * c, reinterpret_cast<uint32_t(&)[32]>(x[c]));
        tmem_ld_wait();
        if (nkeys < 128) {
#pragma unroll
          for (int c = 0; c < NC; ++c)
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (col0 + 32 * c + i >= nkeys) x[c][i] = -INFINITY;
        }
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < NC; ++c)
          if (col0 + 32 * c < nkeys) mx = fmaxf(mx, max32(x[c]));
        if (NWG > 1) {
          s_pmax[g & 1][wg][lrow] = mx;
          mbar_arrive(&bar_xmax);
          if (!mbar_wait(&bar_xmax, g & 1, p.ctl, abort)) {
            ok = false;
            break;
          }
#pragma unroll
          for (int w = 0; w < NWG; ++w) mx = fmaxf(mx, s_pmax[g & 1][w][lrow]);
        }
        const float m_new = fmaxf(m, mx * scale_log2);
        const bool need = m_new > m + 8.0f;
        // PV_g completes on bar_o_full[g & 1] (its phase g >> 1 there).  O is
        // rescaled only after PV_{g-1} has completed; otherwise P_g is handed
        // over while PV_{g-1} may still run, so the tensor pipe always has the
        // next P.V queued.
        if (j > 0 && __any_sync(0xffffffffu, need)) {
          if (!mbar_wait(&bar_o_full[(g - 1) & 1], ((g - 1) >> 1) & 1, p.ctl, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const float f = need ? ex2_approx(m - m_new) : 1.0f;
          const uint32_t oa = tmem_lane_addr(tmem, warp, 256);
          for (int c = wg; c < nchunk; c += NWG) {
            uint32_t o[16];
            tmem_ld16(oa + 16 * c, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * f);
            tmem_st16(oa + 16 * c, o);
          }
          tmem_st_wait();
          l *= f;
          if (need) m = m_new;
        } else if (need) {
          m = m_new;
        }
        const float neg_m = -m;
        float rs[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t pk[NC][16];
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          if (col0 + 32 * c >= nkeys) {
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[c][i] = 0u;
            continue;
          }
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float a0 = ex2_approx(fmaf(x[c][2 * i], scale_log2, neg_m));
            const float a1 = ex2_approx(fmaf(x[c][2 * i + 1], scale_log2, neg_m));
            rs[i & 3] += a0 + a1;
            pk[c][i] = pack_bf16x2(a0, a1);
          }
        }
        l += (rs[0] + rs[1]) + (rs[2] + rs[3]);
        // P over this thread's columns: TMEM columns buf*128 + col0/2 ...
        const uint32_t pa = tmem_lane_addr(tmem, warp, buf * 128 + col0 / 2);
#pragma unroll
        for (int c = 0; c < NC; ++c) tmem_st16(pa + 16 * c, pk[c]);
        tmem_st_wait();
        // Keep this thread within one phase of bar_o_full[g & 1]: PV_{g-2} is
        // complete already (S_g, waited for above, was issued after it), so
        // this wait only advances the phase this thread has observed there.
        if (g >= 2 && !mbar_wait(&bar_o_full[g & 1], ((g - 2) >> 1) & 1, p.ctl, abort)) {
          ok = false;
          break;
        }
        tc_fence_before();
        mbar_arrive(&bar_p_full[buf]);
      }
      if (!ok) break;
      // epilogue: wait for the last PV, combine the partial row sums, O / l, lse
      const uint32_t glast = it + nk - 1;
      if (!mbar_wait(&bar_o_full[glast & 1], (glast >> 1) & 1, p.ctl, abort)) break;
      tc_fence_after();
      if (NWG > 1) {
        s_psum[wg][lrow] = l;
        mbar_arrive(&bar_xsum);
        if (!mbar_wait(&bar_xsum, tcount & 1, p.ctl, abort)) break;
        l = 0.f;
#pragma unroll
        for (int w = 0; w < NWG; ++w) l += s_psum[w][lrow];
      }
      if (orow >= p.nq) orow = -1;
      const bool live = orow >= 0;
      if (!live) orow = 0;
      const float inv = 1.0f / l;
      const uint32_t oa = tmem_lane_addr(tmem, warp, 256);
      // O / l goes out through a per-warp staging buffer: 32 rows x 16 columns,
      // 64-byte rows whose 16-byte units are XOR-swizzled by (row >> 1) & 3 (no
      // bank conflicts either way).  Each store instruction then writes 64
      // contiguous bytes of 8 rows instead of 16 bytes of 32 rows.
      float* stg = reinterpret_cast<float*>(gptr(sStage + (warp - 2) * 2048));
      const bool vec_ok = (p.ldo & 3) == 0;
      // the output rows of the 4 rows this lane stores per chunk
      int orow_r[4];
      bool live_r[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        orow_r[i] = __shfl_sync(0xffffffffu, orow, 8 * i + (lane >> 2));
        live_r[i] = __shfl_sync(0xffffffffu, live ? 1 : 0, 8 * i + (lane >> 2)) != 0;
      }
      // TMEM loads one chunk ahead of the stores
      uint32_t o[16], o_next[16];
      if (wg < nchunk) tmem_ld16(oa + 16 * wg, o_next);
      for (int c = wg; c < nchunk; c += NWG) {
        tmem_ld_wait(o_next);
#pragma unroll
        for (int i = 0; i < 16; ++i) o[i] = o_next[i];
        if (c + NWG < nchunk) tmem_ld16(oa + 16 * (c + NWG), o_next);
#pragma unroll
        for (int u = 0; u < 4; ++u)
          *reinterpret_cast<float4*>(stg + lane * 16 + (((u ^ (lane >> 1)) & 3) << 2)) =
              make_float4(__uint_as_float(o[4 * u]) * inv, __uint_as_float(o[4 * u + 1]) * inv,
                          __uint_as_float(o[4 * u + 2]) * inv, __uint_as_float(o[4 * u + 3]) * inv);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = 8 * i + (lane >> 2), u = lane & 3;
          const float4 v = *reinterpret_cast<const float4*>(stg + r * 16 + (((u ^ (r >> 1)) & 3) << 2));
          const int col = 16 * c + 4 * u;
          if (live_r[i]) {
            float* dst = p.O + (size_t)orow_r[i] * p.ldo + col;
            if (vec_ok && col + 4 <= p.k) {
              *reinterpret_cast<float4*>(dst) = v;
            } else {
              if (col < p.k) dst[0] = v.x;
              if (col + 1 < p.k) dst[1] = v.y;
              if (col + 2 < p.k) dst[2] = v.z;
              if (col + 3 < p.k) dst[3] = v.w;
            }
          }
        }
        __syncwarp();
      }
      if (live && wg == 0) p.lse[orow] = (m + log2f(l)) * kLn2;
      it += nk;
    }
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ backward
// Transpose a 4 x 4 block of float4 held by the 4 lanes of a quad (lane q holds
// row q, float4 columns 0..3) so that lane q ends with column q of rows 0..3 in
// v[0..3].  Two butterfly exchanges (lane distance 1, then 2), each moving half
// of the block; every lane of the warp must take part.
__device__ __forceinline__ float4 shfl_xor4(float4 a, int m) {
  return make_float4(__shfl_xor_sync(0xffffffffu, a.x, m), __shfl_xor_sync(0xffffffffu, a.y, m),
                     __shfl_xor_sync(0xffffffffu, a.z, m), __shfl_xor_sync(0xffffffffu, a.w, m));
}
__device__ __forceinline__ void quad_transpose4(float4 (&v)[4], int q) {
  {
    // distance 1: column pairs (0,1) and (2,3) swap their off-diagonal entries
    const bool odd = (q & 1) != 0;
    const float4 r0 = shfl_xor4(odd ? v[0] : v[1], 1);
    const float4 r1 = shfl_xor4(odd ? v[2] : v[3], 1);
    if (odd) {
      v[0] = r0;
      v[2] = r1;
    } else {
      v[1] = r0;
      v[3] = r1;
    }
  }
  {
    // distance 2: 2 x 2 blocks swap across the quad's halves
    const bool hi = (q & 2) != 0;
    const float4 r0 = shfl_xor4(hi ? v[0] : v[2], 2);
    const float4 r1 = shfl_xor4(hi ? v[1] : v[3], 2);
    if (hi) {
      v[0] = r0;
      v[1] = r1;
    } else {
      v[2] = r0;
      v[3] = r1;
    }
  }
}

// kDV = false: dQ (stored) and dK (atomics).  kDV = true: dV (atomics).
// The backward's work is the flat list of (row tile, key segment) units, in
// row-tile order; CTA c takes units [c U / G, (c + 1) U / G).  Every CTA gets
// the same amount of work (no tail wave), at the price that a row tile may be
// shared by two CTAs, which then reduce their dQ contributions atomically.
struct UnitRange {
  int t, j, left;  // current tile, first segment in it, units still to do
};
// Next run of consecutive segments [jb, je) of one tile t; false when done.
__device__ __forceinline__ bool next_segment(UnitRange& r, const RowTile* tiles, int ntiles, int& t,
                                             int& jb, int& je) {
  while (r.left > 0 && r.t < ntiles) {
    const int avail = tiles[r.t].nseg - r.j;
    if (avail <= 0) {
      ++r.t;
      r.j = 0;
      continue;
    }
    const int take = min(avail, r.left);
    t = r.t;
    jb = r.j;
    je = r.j + take;
    r.left -= take;
    ++r.t;
    r.j = 0;
    return true;
  }
  return false;
}

// NCG compute warpgroups split the key columns of S / dP (and the columns of
// the dK / dV / dQ flushes); every element is independent in the backward.
//
// QCH > 0 fixes the operand shape at compile time (d = 64 QCH; V and dO rows of
// VF full 64-column chunks plus VR remainder columns), so that every MMA issue
// loop has a constant trip count and is fully unrolled: a single issuing thread
// with run-time loop bounds cannot keep the tensor pipe busy at N = 128.
// QCH = 0 reads the shape from the parameters (any d, k).
template <bool kDV, int NCG, int QCH, int VF, int VR>
__global__ void __launch_bounds__(64 + 128 * NCG + 128, 1)
    tc_bwd_kernel(const __grid_constant__ TensorMaps tm, const TcParams p) {
  constexpr bool kFixed = QCH > 0;
  const int qch = kFixed ? QCH : p.qch;
  const int vf = kFixed ? VF : p.vf;
  const int vr = kFixed ? VR : p.vr;
  const int d16 = kFixed ? 4 * QCH : p.d / 16;
  constexpr int CW = 128 / NCG;  // key columns per compute thread
  constexpr int NC = CW / 32;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_qg_full, bar_qg_empty, bar_k_full, bar_k_empty, bar_v_full, bar_v_empty,
      bar_sdp_full, bar_ds_full, bar_dkp_full, bar_dkp_empty, bar_dq_full, bar_drain;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ int s_range[3];  // first tile, first segment in it, number of units

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base_u = smem_u32(smem_raw);
  const uint32_t sbase = (base_u + 1023u) & ~1023u;
  const int qbytes = qch * kChunk;
  const int vbytes = vtile_bytes(vf, vr);
  const uint32_t sQ = sbase;
  const uint32_t sG = sQ + qbytes;           // dO tile
  const uint32_t sK = sG + vbytes;
  const uint32_t sV = sK + qbytes;           // unused in the dV pass
  const uint32_t sS = sV + (kDV ? 0 : vbytes);  // dS (or P) tile [q][keys], 2 chunks
  auto gptr = [&](uint32_t s) { return smem_raw + (s - base_u); };
  const int ntiles = p.ntiles_dev ? *p.ntiles_dev : p.ntiles_host;

  if (threadIdx.x == 0) {
    mbar_init(&bar_qg_full, 1);
    mbar_init(&bar_qg_empty, 1);
    mbar_init(&bar_k_full, 1);
    mbar_init(&bar_k_empty, 1);
    mbar_init(&bar_v_full, 1);
    mbar_init(&bar_v_empty, 1);
    mbar_init(&bar_sdp_full, 1);
    mbar_init(&bar_ds_full, 128 * NCG);
    mbar_init(&bar_dkp_full, 1);
    mbar_init(&bar_dkp_empty, 128);
    mbar_init(&bar_dq_full, 1);
    mbar_init(&bar_drain, 1);
    s_abort = 0;
    fence_barrier_init();
    // this CTA's share of the (row tile, key segment) units
    const int U = p.tile_prefix[ntiles];
    const long long u0 = (long long)blockIdx.x * U / gridDim.x;
    const long long u1 = (long long)(blockIdx.x + 1) * U / gridDim.x;
    int lo = 0, hi = ntiles;  // largest t < ntiles with prefix[t] <= u0
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (p.tile_prefix[mid] <= u0) lo = mid;
      else hi = mid;
    }
    s_range[0] = lo;
    s_range[1] = ntiles > 0 ? (int)(u0 - p.tile_prefix[lo]) : 0;
    s_range[2] = ntiles > 0 ? (int)(u1 - u0) : 0;
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort = &s_abort;
  // TMEM columns
  const uint32_t c_s = 0, c_dp = 128, c_dq = 256, c_dkp = kDV ? 256 : 384;

  if (warp == 0) {
    if (lane == 0) {
      uint32_t it = 0, tcount = 0;
      int q_issued = -1, k_last = -1, v_last = -1;
      UnitRange ur{s_range[0], s_range[1], s_range[2]};
      int t, jb, je;
      while (!*abort && next_segment(ur, p.tiles, ntiles, t, jb, je)) {
        const RowTile tile = p.tiles[t];
        if (tcount > 0 && !mbar_wait(&bar_qg_empty, (tcount - 1) & 1, p.ctl, abort)) break;
        q_issued = (int)tcount;
        mbar_arrive_expect_tx(&bar_qg_full, qbytes + vbytes);
        for (int c = 0; c < qch; ++c)
          tma_load_2d(gptr(sQ) + c * kChunk, &tm.q, 64 * c, tile.row0, &bar_qg_full);
        for (int c = 0; c < vf; ++c)
          tma_load_2d(gptr(sG) + c * kChunk, &tm.g, 64 * c, tile.row0, &bar_qg_full);
        if (vr) tma_load_2d(gptr(sG) + vf * kChunk, &tm.gr, 64 * vf, tile.row0, &bar_qg_full);
        bool ok = true;
        for (int j = jb; j < je; ++j, ++it) {
          const KeySeg sg = p.segs[tile.seg0 + j];
          if (!kDV) {
            if (it >= 1 && !mbar_wait(&bar_v_empty, (it - 1) & 1, p.ctl, abort)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&bar_v_full, vbytes);
            for (int c = 0; c < vf; ++c)
              tma_load_2d(gptr(sV) + c * kChunk, &tm.v, 64 * c, sg.key0, &bar_v_full);
            if (vr) tma_load_2d(gptr(sV) + vf * kChunk, &tm.vr, 64 * vf, sg.key0, &bar_v_full);
            v_last = (int)it;
          }
          if (it >= 1 && !mbar_wait(&bar_k_empty, (it - 1) & 1, p.ctl, abort)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar_k_full, qbytes);
          for (int c = 0; c < qch; ++c)
            tma_load_2d(gptr(sK) + c * kChunk, &tm.k, 64 * c, sg.key0, &bar_k_full);
          k_last = (int)it;
        }
        ++tcount;
        if (!ok) break;
      }
      if (*abort) {
        // let the copies already issued land before the CTA can exit
        volatile int never = 0;
        if (q_issued >= 0) mbar_wait(&bar_qg_full, q_issued & 1, p.ctl, &never);
        if (k_last >= 0) mbar_wait(&bar_k_full, k_last & 1, p.ctl, &never);
        if (v_last >= 0) mbar_wait(&bar_v_full, v_last & 1, p.ctl, &never);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc_s = make_idesc_bf16(128, 128, 0, 0);
      const uint32_t idesc_dq = make_idesc_bf16(128, p.d, 0, 1);
      const uint32_t idesc_dkp = make_idesc_bf16(128, p.d, 1, 1);
      const uint32_t idesc_dv = make_idesc_bf16(128, 64 * (vf > 0 ? vf : 1), 1, 1);
      const uint32_t idesc_dvr = make_idesc_bf16(128, vr > 0 ? vr : 16, 1, 1);
      const uint32_t rsw = rem_swizzle(vr);
      const uint32_t rrow = (uint32_t)vr * 2;
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      UnitRange ur{s_range[0], s_range[1], s_range[2]};
      int t, jb, je;
      while (ok && next_segment(ur, p.tiles, ntiles, t, jb, je)) {
        if (!mbar_wait(&bar_qg_full, tcount & 1, p.ctl, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int j = jb; j < je && ok; ++j, ++it) {
          if (!kDV) {
            // dP = dO V^T (K = kp)
            if (!mbar_wait(&bar_v_full, it & 1, p.ctl, abort)) {
              ok = false;
              break;
            }
            tc_fence_after();
            int kk = 0;
#pragma unroll
            for (int c = 0; c < vf; ++c)
#pragma unroll
              for (int u = 0; u < 4; ++u, ++kk) {
                const uint32_t off = c * kChunk + u * 32;
                mma_ss(tmem + c_dp, make_sdesc(sG + off, 16, 1024, kSw128),
                       make_sdesc(sV + off, 16, 1024, kSw128), idesc_s, kk > 0);
              }
#pragma unroll
            for (int u = 0; u < vr / 16; ++u, ++kk) {
              const uint32_t off = vf * kChunk + u * 32;
              mma_ss(tmem + c_dp, make_sdesc(sG + off, 16, 8 * rrow, rsw),
                     make_sdesc(sV + off, 16, 8 * rrow, rsw), idesc_s, kk > 0);
            }
            mma_commit(&bar_v_empty);
          }
          // S = Q K^T
          if (!mbar_wait(&bar_k_full, it & 1, p.ctl, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < d16; ++kk) {
            const uint32_t off = (kk >> 2) * kChunk + (kk & 3) * 32;
            mma_ss(tmem + c_s, make_sdesc(sQ + off, 16, 1024, kSw128),
                   make_sdesc(sK + off, 16, 1024, kSw128), idesc_s, kk > 0);
          }
          mma_commit(&bar_sdp_full);
          // wait for dS (or P) in shared memory
          if (!mbar_wait(&bar_ds_full, it & 1, p.ctl, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (!kDV) {
            // dQ += dS K_j : A = dS [q][keys] K-major, B = K_j [keys][d] MN-major
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
              const uint32_t aoff = (kk >> 2) * kChunk + (kk & 3) * 32;
              mma_ss(tmem + c_dq, make_sdesc(sS + aoff, 16, 1024, kSw128),
                     make_sdesc(sK + kk * 2048, kChunk, 1024, kSw128), idesc_dq,
                     (j > jb || kk > 0) ? 1u : 0u);
            }
            mma_commit(&bar_k_empty);
            // the flush warpgroup has read the previous partial out of TMEM
            if (it >= 1 && !mbar_wait(&bar_dkp_empty, (it - 1) & 1, p.ctl, abort)) {
              ok = false;
              break;
            }
            tc_fence_after();
            // dKp = dS^T Q : A = dS viewed MN-major (M = keys), B = Q MN-major (N = d)
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ss(tmem + c_dkp, make_sdesc(sS + kk * 2048, kChunk, 1024, kSw128),
                     make_sdesc(sQ + kk * 2048, kChunk, 1024, kSw128), idesc_dkp, kk > 0);
          } else {
            mma_commit(&bar_k_empty);
            // the flush warpgroup has read the previous partial out of TMEM
            if (it >= 1 && !mbar_wait(&bar_dkp_empty, (it - 1) & 1, p.ctl, abort)) {
              ok = false;
              break;
            }
            tc_fence_after();
            // dVp = P^T dO : A = P viewed MN-major (M = keys), B = dO MN-major (N = k)
            for (int kk = 0; kk < 8; ++kk) {
              if (vf > 0)
                mma_ss(tmem + c_dkp, make_sdesc(sS + kk * 2048, kChunk, 1024, kSw128),
                       make_sdesc(sG + kk * 2048, kChunk, 1024, kSw128), idesc_dv, kk > 0);
              if (vr > 0)
                mma_ss(tmem + c_dkp + 64 * vf, make_sdesc(sS + kk * 2048, kChunk, 1024, kSw128),
                       make_sdesc(sG + vf * kChunk + kk * 16 * rrow, 128 * rrow, 8 * rrow, rsw),
                       idesc_dvr, kk > 0);
            }
          }
          mma_commit(&bar_dkp_full);
        }
        if (!ok) break;
        mma_commit(&bar_dq_full);
        mma_commit(&bar_qg_empty);
        ++tcount;
      }
      mma_commit(&bar_drain);
      volatile int never = 0;
      mbar_wait(&bar_drain, 0, p.ctl, &never);
    }
  } else if (warp < 2 + 4 * NCG) {
    // ---------------- softmax (NCG warpgroups): one thread per query row; the
    // warpgroups split the key columns of S / dP.  They also store dQ.
    const int wg = (warp - 2) >> 2;
    const int lrow = 32 * (warp & 3) + lane;
    const int col0 = wg * CW;
    uint32_t it = 0, tcount = 0;
    UnitRange ur{s_range[0], s_range[1], s_range[2]};
    int t, jb, je;
    for (; next_segment(ur, p.tiles, ntiles, t, jb, je); ++tcount) {
      const RowTile tile = p.tiles[t];
      const int qrow = tile.row0 + lrow;
      const bool live_row = lrow < tile.nrows && qrow < p.nq;
      const float lse2 = live_row ? p.lse_in[qrow] * kLog2e : 0.f;
      const float Di = (!kDV && live_row) ? p.Dvec[qrow] : 0.f;
      bool ok = true;
      KeySeg sg_next = p.segs[tile.seg0 + jb];
      for (int j = jb; j < je; ++j, ++it) {
        const KeySeg sg = sg_next;
        if (j + 1 < je) sg_next = p.segs[tile.seg0 + j + 1];
        // S / dP of this key tile; the commit behind it also covers the MMAs of
        // the previous tile that read the dS tile overwritten below
        if (!mbar_wait(&bar_sdp_full, it & 1, p.ctl, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ta = tmem_lane_addr(tmem, warp, 0);
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          uint32_t sv[32], dp[32];
          tmem_ld32(ta + c_s + col0 + 32 * c, sv);
          if (!kDV) tmem_ld32(ta + c_dp + col0 + 32 * c, dp);
          tmem_ld_wait();
          uint32_t pk[16];
          const int cbase = col0 + 32 * c;
          const bool full = live_row && cbase + 32 <= sg.nkeys;
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float v2[2];
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              float pr = ex2_approx(fmaf(__uint_as_float(sv[2 * i + h]), p.scale_log2, -lse2));
              if (!full && (cbase + 2 * i + h >= sg.nkeys || !live_row)) pr = 0.f;
              v2[h] = kDV ? pr : pr * (__uint_as_float(dp[2 * i + h]) - Di);
            }
            pk[i] = pack_bf16x2(v2[0], v2[1]);
          }
          // row lrow, keys [cbase, cbase+32): 64-key chunk cbase/64, 16-byte
          // units ((cbase%64)/8) + 0..3, swizzled by the row
          const uint32_t rowb = sS + (cbase >> 6) * kChunk + lrow * 128;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint32_t unit = (((cbase & 63) >> 3) + u) ^ (lrow & 7);
            asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(rowb + unit * 16),
                         "r"(pk[4 * u]), "r"(pk[4 * u + 1]), "r"(pk[4 * u + 2]), "r"(pk[4 * u + 3])
                         : "memory");
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bar_ds_full);
      }
      if (!ok) break;
      if (!mbar_wait(&bar_dq_full, tcount & 1, p.ctl, abort)) break;
      if (!kDV) {
        tc_fence_after();
        // TMEM loads are warp-collective: every lane loads, live rows store
        int orow = live_row ? (p.row_map ? p.row_map[qrow] : qrow) : -1;
        const bool store_row = orow >= 0 && orow < p.nq;
        const bool whole = jb == 0 && je == tile.nseg;  // all of the row tile's keys done here
        if (!store_row) orow = 0;
        float* dq = p.dQ + (size_t)orow * p.lddq;
        const uint32_t ta = tmem_lane_addr(tmem, warp, c_dq);
        for (int cc = wg; cc < d16; cc += NCG) {
          uint32_t o[16];
          tmem_ld16(ta + 16 * cc, o);
          tmem_ld_wait();
          if (!store_row) continue;
          if (!whole) {
            // the row tile's keys are split over several CTAs: reduce into dQ
            if (p.vec_atomics_dq) {
#pragma unroll
              for (int i = 0; i < 16; i += 4)
                atomicAdd(reinterpret_cast<float4*>(dq + 16 * cc + i),
                          make_float4(__uint_as_float(o[i]) * p.scale, __uint_as_float(o[i + 1]) * p.scale,
                                      __uint_as_float(o[i + 2]) * p.scale,
                                      __uint_as_float(o[i + 3]) * p.scale));
            } else {
#pragma unroll
              for (int i = 0; i < 16; ++i) atomicAdd(dq + 16 * cc + i, __uint_as_float(o[i]) * p.scale);
            }
          } else if ((p.lddq & 3) == 0) {
#pragma unroll
            for (int i = 0; i < 16; i += 4)
              *reinterpret_cast<float4*>(dq + 16 * cc + i) = make_float4(
                  __uint_as_float(o[i]) * p.scale, __uint_as_float(o[i + 1]) * p.scale,
                  __uint_as_float(o[i + 2]) * p.scale, __uint_as_float(o[i + 3]) * p.scale);
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) dq[16 * cc + i] = __uint_as_float(o[i]) * p.scale;
          }
        }
      }
    }
  } else {
    // ---------------- flush (one warpgroup): thread = key row of the partial
    // dK (or dV) in TMEM; reduces it into global memory while the softmax
    // warpgroups and the tensor cores work on the next key tile.
    const int lrow = 32 * (warp & 3) + lane;
    const int kt_out = kDV ? p.kp : p.d;  // columns of the partial
    const int nchunk_out = kt_out / 16;
    const int ldd = kDV ? p.lddv : p.lddk;
    float* const dbase = kDV ? p.dV : p.dK;
    const int ncols = kDV ? p.k : p.d;
    const float mul = kDV ? 1.0f : p.scale;
    const int qbase = lane & ~3;
    uint32_t it = 0;
    bool ok = true;
    UnitRange ur{s_range[0], s_range[1], s_range[2]};
    int t, jb, je;
    while (ok && next_segment(ur, p.tiles, ntiles, t, jb, je)) {
      const RowTile tile = p.tiles[t];
      for (int j = jb; j < je; ++j, ++it) {
        const KeySeg sg = p.segs[tile.seg0 + j];
        const int krow = sg.key0 + lrow;
        int okey = (lrow < sg.nkeys && krow < p.nk) ? (p.col_map ? p.col_map[krow] : krow) : -1;
        if (okey >= p.nk) okey = -1;
        const bool live_key = okey >= 0;
        if (!live_key) okey = 0;
        float* dst = dbase + (size_t)okey * ldd;
        // Rows of this thread's lane quad (destination row, liveness): the
        // vector path transposes each quad's 4 x 16 values so that one
        // reduction instruction covers 64 contiguous bytes of each of 8 rows.
        int qkey[4];
        bool qlive[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          qkey[m] = __shfl_sync(0xffffffffu, okey, qbase + m);
          qlive[m] = __shfl_sync(0xffffffffu, live_key ? 1 : 0, qbase + m) != 0;
        }
        if (!mbar_wait(&bar_dkp_full, it & 1, p.ctl, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ta = tmem_lane_addr(tmem, warp, c_dkp);
        // four 16-column chunks per TMEM round trip; the partial's columns are
        // released to the MMA issuer as soon as the last load has landed
        for (int g0 = 0; g0 < nchunk_out; g0 += 4) {
          uint32_t o[4][16];
#pragma unroll
          for (int q = 0; q < 4; ++q)
            if (g0 + q < nchunk_out) tmem_ld16(ta + 16 * (g0 + q), o[q]);
          tmem_ld_wait();
          if (g0 + 4 >= nchunk_out) {
            tc_fence_before();
            mbar_arrive(&bar_dkp_empty);
          }
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int c0 = 16 * (g0 + q);
            if (g0 + q >= nchunk_out) break;
            if (p.vec_atomics && c0 + 16 <= ncols) {
              float4 v[4];
#pragma unroll
              for (int c = 0; c < 4; ++c)
                v[c] = make_float4(__uint_as_float(o[q][4 * c]) * mul,
                                   __uint_as_float(o[q][4 * c + 1]) * mul,
                                   __uint_as_float(o[q][4 * c + 2]) * mul,
                                   __uint_as_float(o[q][4 * c + 3]) * mul);
              quad_transpose4(v, lane & 3);
              // v[m] = columns [c0 + 4 (lane & 3), +4) of quad row m
#pragma unroll
              for (int m = 0; m < 4; ++m)
                if (qlive[m])
                  atomicAdd(reinterpret_cast<float4*>(dbase + (size_t)qkey[m] * ldd + c0 +
                                                      4 * (lane & 3)),
                            v[m]);
            } else if (live_key) {
#pragma unroll
              for (int i = 0; i < 16; ++i)
                if (c0 + i < ncols) atomicAdd(dst + c0 + i, __uint_as_float(o[q][i]) * mul);
            }
          }
        }
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ backward, dQ and dK
// Query-stationary backward for dQ and dK (the dV pass keeps tc_bwd_kernel).
// 128 (2 + NCG) threads in four warpgroups:
//   WG0   warp 0: TMA producer (Q once per row tile; K_j into a 2-stage ring;
//         V_j); warp 1: MMA issuer and TMEM owner; warps 2-3 idle.
//   WG1.. (NCG softmax warpgroups): thread = query row (TMEM lane); the
//         warpgroups split the key columns.  They write the row tile's dO into
//         TMEM once per row tile.
//   last  (flush): thread = key row; reduces every key tile's partial dK into
//         global memory while the other roles move on, and at the end of each
//         run of a row tile's key tiles reads dQ out of TMEM (handing the
//         columns back to the MMA issuer at once) and stores it, so that the
//         softmax warpgroups go on to the next row tile meanwhile.
// TMEM columns: [0,128) S_j and then dP_j of the same key tile (dP is issued
// once the softmax has read S, so its MMAs run under the softmax's exp2);
// [128, 128 + kp/2) dO as bf16 pairs, the A operand of dP; [256, 256 + d) dQ;
// [384, 384 + d) the partial dK.  Per key tile j:
//   S_j  = Q K_j^T      (SS)                -> softmax: P = exp2(S s log2e - lse log2e)
//   dP_j = dO V_j^T     (TS, A = dO)        -> softmax: dS = P (dP - D) -> bf16 smem
//   dQ  += dS K_j       (SS, K_j MN-major)
//   dKp  = dS^T Q       (SS, MN-major views) -> flush warpgroup -> dK
// Shared memory: Q, two K stages, V, dS (no dO tile), which leaves room for
// the second K stage; a key tile's K load overlaps the previous tile's work.
template <int NCG, int QCH, int VF, int VR, bool kNoDK, bool kDqFlush>
__global__ void __launch_bounds__(128 * (2 + NCG), 1)
    tc_bwd_dqk_kernel(const __grid_constant__ TensorMaps tm, const TcParams p) {
  static_assert(NCG == 2, "the register split assumes two softmax warpgroups");
  constexpr bool kFixed = QCH > 0;
  const int qch = kFixed ? QCH : p.qch;
  const int vf = kFixed ? VF : p.vf;
  const int vr = kFixed ? VR : p.vr;
  const int d16 = kFixed ? 4 * QCH : p.d / 16;
  constexpr int CW = 128 / NCG;  // key columns per softmax thread
  constexpr int NC = CW / 32;
  constexpr int kFlushWarp = 4 + 4 * NCG;
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_q_full, bar_q_empty, bar_k_full[2], bar_k_empty[2], bar_v_full,
      bar_v_empty, bar_s_full, bar_s_read, bar_dp_full, bar_ds_full, bar_do_full, bar_dkp_full,
      bar_dkp_empty, bar_dq_full, bar_dq_empty, bar_drain, bar_dp_read, bar_never;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ int s_range[3];  // first tile, first segment in it, number of units

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base_u = smem_u32(smem_raw);
  const uint32_t sbase = (base_u + 1023u) & ~1023u;
  const int qbytes = qch * kChunk;
  const int vbytes = vtile_bytes(vf, vr);
  const uint32_t sQ = sbase;
  const uint32_t sK0 = sQ + qbytes;  // K stage s at sK0 + s * qbytes
  const uint32_t sV = sK0 + 2 * qbytes;
  const uint32_t sS = sV + vbytes;   // dS tile [q][keys], 2 chunks
  const uint32_t sStage = sS + 2 * kChunk;  // 32 KB: two 4 KB staging boxes per flush warp (TMA path)
  auto gptr = [&](uint32_t s) { return smem_raw + (s - base_u); };
  const int ntiles = p.ntiles_dev ? *p.ntiles_dev : p.ntiles_host;

  if (threadIdx.x == 0) {
    mbar_init(&bar_q_full, 1);
    mbar_init(&bar_q_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_k_full[i], 1);
      mbar_init(&bar_k_empty[i], 1);
    }
    mbar_init(&bar_v_full, 1);
    mbar_init(&bar_v_empty, 1);
    mbar_init(&bar_s_full, 1);
    mbar_init(&bar_s_read, 128 * NCG);
    mbar_init(&bar_dp_full, 1);
    mbar_init(&bar_ds_full, 128 * NCG);
    mbar_init(&bar_dp_read, 128 * NCG);
    mbar_init(&bar_do_full, 128 * NCG);
    mbar_init(&bar_dkp_full, 1);
    mbar_init(&bar_dkp_empty, 128);
    mbar_init(&bar_dq_full, 1);
    mbar_init(&bar_dq_empty, 128);
    mbar_init(&bar_drain, 1);
    mbar_init(&bar_never, 1);  // nothing arrives: the abort-path test hook waits here
    s_abort = 0;
    fence_barrier_init();
    // this CTA's share of the (row tile, key segment) units
    const int U = p.tile_prefix[ntiles];
    const long long u0 = (long long)blockIdx.x * U / gridDim.x;
    const long long u1 = (long long)(blockIdx.x + 1) * U / gridDim.x;
    int lo = 0, hi = ntiles;  // largest t < ntiles with prefix[t] <= u0
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (p.tile_prefix[mid] <= u0) lo = mid;
      else hi = mid;
    }
    s_range[0] = lo;
    s_range[1] = ntiles > 0 ? (int)(u0 - p.tile_prefix[lo]) : 0;
    s_range[2] = ntiles > 0 ? (int)(u1 - u0) : 0;
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort = &s_abort;
  const uint32_t c_sp = 0, c_do = 128, c_dq = 256, c_dkp = 384;

  if (warp < 4) {
    warpgroup_reg_dealloc<80>();
    if (warp == 0 && lane == 0) {
      // ---------------- TMA producer
      uint32_t it = 0, tcount = 0;
      int q_last = -1, v_last = -1;
      int k_last[2] = {-1, -1};  // phase index of the last load issued per K stage
      UnitRange ur{s_range[0], s_range[1], s_range[2]};
      int t, jb, je;
      while (!*abort && next_segment(ur, p.tiles, ntiles, t, jb, je)) {
        const RowTile tile = p.tiles[t];
        if (tcount > 0 && !mbar_wait(&bar_q_empty, (tcount - 1) & 1, p.ctl, abort)) break;
        mbar_arrive_expect_tx(&bar_q_full, qbytes);
        for (int c = 0; c < qch; ++c)
          tma_load_2d(gptr(sQ) + c * kChunk, &tm.q, 64 * c, tile.row0, &bar_q_full);
        q_last = (int)tcount;
        bool ok = true;
        for (int j = jb; j < je; ++j, ++it) {
          const KeySeg sg = p.segs[tile.seg0 + j];
          const int st = it & 1;
          if (it >= 2 && !mbar_wait(&bar_k_empty[st], ((it >> 1) - 1) & 1, p.ctl, abort)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar_k_full[st], qbytes);
          for (int c = 0; c < qch; ++c)
            tma_load_2d(gptr(sK0 + st * qbytes) + c * kChunk, &tm.k, 64 * c, sg.key0, &bar_k_full[st]);
          k_last[st] = (int)(it >> 1);
          if (it >= 1 && !mbar_wait(&bar_v_empty, (it - 1) & 1, p.ctl, abort)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar_v_full, vbytes);
          for (int c = 0; c < vf; ++c)
            tma_load_2d(gptr(sV) + c * kChunk, &tm.v, 64 * c, sg.key0, &bar_v_full);
          if (vr) tma_load_2d(gptr(sV) + vf * kChunk, &tm.vr, 64 * vf, sg.key0, &bar_v_full);
          v_last = (int)it;
        }
        ++tcount;
        if (!ok) break;
      }
      if (*abort) {
        // let the copies already issued land before the CTA can exit
        volatile int never = 0;
        if (q_last >= 0) mbar_wait(&bar_q_full, q_last & 1, p.ctl, &never);
        for (int s2 = 0; s2 < 2; ++s2)
          if (k_last[s2] >= 0) mbar_wait(&bar_k_full[s2], k_last[s2] & 1, p.ctl, &never);
        if (v_last >= 0) mbar_wait(&bar_v_full, v_last & 1, p.ctl, &never);
      }
    } else if (warp == 1 && lane == 0) {
      // ---------------- MMA issuer
      const uint32_t idesc_s = make_idesc_bf16(128, 128, 0, 0);  // S and dP: N = 128 keys
      const uint32_t idesc_dq = make_idesc_bf16(128, p.d, 0, 1);
      const uint32_t idesc_dkp = make_idesc_bf16(128, p.d, 1, 1);
      const uint32_t rsw = rem_swizzle(vr);
      const uint32_t rrow = (uint32_t)vr * 2;
      uint32_t it = 0, tcount = 0;
      bool ok = true;
      UnitRange ur{s_range[0], s_range[1], s_range[2]};
      int t, jb, je;
      while (ok && next_segment(ur, p.tiles, ntiles, t, jb, je)) {
        if (!mbar_wait(&bar_q_full, tcount & 1, p.ctl, abort) ||
            !mbar_wait(&bar_do_full, tcount & 1, p.ctl, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // S = Q K_j^T into the S/dP columns (K stage it & 1)
        auto issue_s = [&](uint32_t u) -> bool {
          const uint32_t sK = sK0 + (u & 1) * qbytes;
          if (!mbar_wait(&bar_k_full[u & 1], (u >> 1) & 1, p.ctl, abort)) return false;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < d16; ++kk) {
            const uint32_t off = (kk >> 2) * kChunk + (kk & 3) * 32;
            mma_ss(tmem + c_sp, make_sdesc(sQ + off, 16, 1024, kSw128),
                   make_sdesc(sK + off, 16, 1024, kSw128), idesc_s, kk > 0);
          }
          mma_commit(&bar_s_full);
          return true;
        };
        ok = issue_s(it);
        // abort-path test hook: the bounded wait gives up and raises *abort
        if (ok && p.debug_stall && tcount == 0) ok = mbar_wait(&bar_never, 0, p.ctl, abort);
        // Per key tile the tensor pipe runs dP_j, S_{j+1}, dQ_j, dKp_j: the next
        // tile's S is issued as soon as the softmax has read dP_j and runs while
        // it computes dS_j; the softmax then works on S_{j+1} while dQ_j and dKp_j
        // run.  dP_{j+1} is committed after dKp_j, so its barrier also tells the
        // softmax that dS_j has been consumed.
        for (int j = jb; j < je && ok; ++j, ++it) {
          const int st = it & 1;
          const uint32_t sK = sK0 + st * qbytes;
          // dP = dO V^T into the same columns, once the softmax has read S
          if (!mbar_wait(&bar_s_read, it & 1, p.ctl, abort) ||
              !mbar_wait(&bar_v_full, it & 1, p.ctl, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          {
            int kk = 0;
#pragma unroll
            for (int c = 0; c < vf; ++c)
#pragma unroll
              for (int u = 0; u < 4; ++u, ++kk)
                mma_ts(tmem + c_sp, tmem + c_do + 8 * kk,
                       make_sdesc(sV + c * kChunk + u * 32, 16, 1024, kSw128), idesc_s, kk > 0);
#pragma unroll
            for (int u = 0; u < vr / 16; ++u, ++kk)
              mma_ts(tmem + c_sp, tmem + c_do + 8 * kk,
                     make_sdesc(sV + vf * kChunk + u * 32, 16, 8 * rrow, rsw), idesc_s, kk > 0);
          }
          mma_commit(&bar_v_empty);
          mma_commit(&bar_dp_full);
          // the softmax has read dP: the next S goes into the columns while it
          // computes dS
          if (!mbar_wait(&bar_dp_read, it & 1, p.ctl, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (j + 1 < je && !issue_s(it + 1)) {
            ok = false;
            break;
          }
          // dS in shared memory
          if (!mbar_wait(&bar_ds_full, it & 1, p.ctl, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // dQ += dS K_j : A = dS [q][keys] K-major, B = K_j [keys][d] MN-major; the
          // run's first one overwrites the columns once the flush warpgroup has
          // read the previous run's dQ out of them
          if (kDqFlush && j == jb && tcount > 0 &&
              !mbar_wait(&bar_dq_empty, (tcount - 1) & 1, p.ctl, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t aoff = (kk >> 2) * kChunk + (kk & 3) * 32;
            mma_ss(tmem + c_dq, make_sdesc(sS + aoff, 16, 1024, kSw128),
                   make_sdesc(sK + kk * 2048, kChunk, 1024, kSw128), idesc_dq,
                   (j > jb || kk > 0) ? 1u : 0u);
          }
          mma_commit(&bar_k_empty[st]);
          if (!kNoDK) {
            // the flush warpgroup has read the previous partial out of TMEM
            if (it >= 1 && !mbar_wait(&bar_dkp_empty, (it - 1) & 1, p.ctl, abort)) {
              ok = false;
              break;
            }
            tc_fence_after();
            // dKp = dS^T Q : A = dS viewed MN-major (M = keys), B = Q MN-major (N = d)
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ss(tmem + c_dkp, make_sdesc(sS + kk * 2048, kChunk, 1024, kSw128),
                     make_sdesc(sQ + kk * 2048, kChunk, 1024, kSw128), idesc_dkp, kk > 0);
            mma_commit(&bar_dkp_full);
          }
        }
        if (!ok) break;
        mma_commit(&bar_dq_full);
        mma_commit(&bar_q_empty);
        ++tcount;
      }
      mma_commit(&bar_drain);
      volatile int never = 0;
      mbar_wait(&bar_drain, 0, p.ctl, &never);
    }
  } else if (warp < kFlushWarp) {
    // ---------------- softmax (NCG warpgroups): thread = query row
    warpgroup_reg_alloc<128>();
    const int wg = (warp - 4) >> 2;
    const int lrow = 32 * (warp & 3) + lane;
    const int col0 = wg * CW;
    const int kp16 = p.kp / 16;  // 8-column TMEM pieces of the dO row
    uint32_t it = 0, tcount = 0;
    UnitRange ur{s_range[0], s_range[1], s_range[2]};
    int t, jb, je;
    for (; next_segment(ur, p.tiles, ntiles, t, jb, je); ++tcount) {
      const RowTile tile = p.tiles[t];
      const int qrow = tile.row0 + lrow;
      const bool live_row = lrow < tile.nrows && qrow < p.nq;
      const float lse2 = live_row ? p.lse_in[qrow] * kLog2e : 0.f;
      const float Di = live_row ? p.Dvec[qrow] : 0.f;
      // this row tile's dO row into TMEM (the previous row tile's MMAs are
      // complete: its dQ was waited for below before getting here)
      {
        // all of this thread's pieces are loaded before the first TMEM store, so
        // their latencies overlap (kp <= 256: at most 8 pieces of 16 columns)
        const uint4* src = reinterpret_cast<const uint4*>(p.dOb + (size_t)(live_row ? qrow : 0) * p.lddob);
        const uint32_t da = tmem_lane_addr(tmem, warp, c_do);
        uint4 piece[16];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int pc = wg + NCG * i;
          piece[2 * i] = piece[2 * i + 1] = make_uint4(0u, 0u, 0u, 0u);
          if (live_row && pc < kp16) {
            piece[2 * i] = __ldg(src + 2 * pc);
            piece[2 * i + 1] = __ldg(src + 2 * pc + 1);
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int pc = wg + NCG * i;
          if (pc >= kp16) break;
          const uint4 a = piece[2 * i], b = piece[2 * i + 1];
          const uint32_t r[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
          tmem_st8(da + 8 * pc, r);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bar_do_full);
      }
      bool ok = true;
      KeySeg sg_next = p.segs[tile.seg0 + jb];
      for (int j = jb; j < je; ++j, ++it) {
        const KeySeg sg = sg_next;
        if (j + 1 < je) sg_next = p.segs[tile.seg0 + j + 1];
        if (!mbar_wait(&bar_s_full, it & 1, p.ctl, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ta = tmem_lane_addr(tmem, warp, c_sp + col0);
        uint32_t sv[NC][32];
#pragma unroll
        for (int c = 0; c < NC; ++c) tmem_ld32(ta + 32 * c, sv[c]);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&bar_s_read);  // the S columns may now receive dP
        // P = exp2(S s log2e - lse log2e); keys past the segment and dead rows -> 0
        float pr[NC][32];
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          const int cbase = col0 + 32 * c;
          const bool full = live_row && cbase + 32 <= sg.nkeys;
          if (kFixed && cbase >= sg.nkeys) {  // wholly past the segment's last key: no exponentials
#pragma unroll
            for (int i = 0; i < 32; ++i) pr[c][i] = 0.f;
            continue;
          }
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            float v = ex2_approx(fmaf(__uint_as_float(sv[c][i]), p.scale_log2, -lse2));
            if (!full && (cbase + i >= sg.nkeys || !live_row)) v = 0.f;
            pr[c][i] = v;
          }
        }
        // dP of this key tile; its commit also covers the MMAs of the previous
        // key tile that read the dS tile overwritten below
        if (!mbar_wait(&bar_dp_full, it & 1, p.ctl, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t dp[NC][32];
#pragma unroll
        for (int c = 0; c < NC; ++c) tmem_ld32(ta + 32 * c, dp[c]);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&bar_dp_read);  // the S/dP columns may now receive the next S
#pragma unroll
        for (int c = 0; c < NC; ++c) {
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i)
            pk[i] = pack_bf16x2(pr[c][2 * i] * (__uint_as_float(dp[c][2 * i]) - Di),
                                pr[c][2 * i + 1] * (__uint_as_float(dp[c][2 * i + 1]) - Di));
          // row lrow, keys [cbase, cbase+32): 64-key chunk cbase/64, 16-byte
          // units ((cbase%64)/8) + 0..3, swizzled by the row
          const int cbase = col0 + 32 * c;
          const uint32_t rowb = sS + (cbase >> 6) * kChunk + lrow * 128;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint32_t unit = (((cbase & 63) >> 3) + u) ^ (lrow & 7);
            asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(rowb + unit * 16),
                         "r"(pk[4 * u]), "r"(pk[4 * u + 1]), "r"(pk[4 * u + 2]), "r"(pk[4 * u + 3])
                         : "memory");
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(&bar_ds_full);
      }
      if (!ok) break;
      if constexpr (kDqFlush) {
        // the run's MMAs are complete (its dP read dO): the next run's dO may
        // be written; the flush warpgroup stores this run's dQ
        if (!mbar_wait(&bar_dq_full, tcount & 1, p.ctl, abort)) break;
        continue;
      }
      if (!mbar_wait(&bar_dq_full, tcount & 1, p.ctl, abort)) break;
      tc_fence_after();
      // dQ / s goes out through a 2 KB staging area inside this warp's own rows
      // of the dS tile (free: every MMA that read it is complete): 32 rows x
      // 16 columns per chunk, 16-byte units XOR-swizzled by (row >> 1) & 3, so
      // that each store or reduction covers 64 contiguous bytes of 8 rows.
      const bool whole = jb == 0 && je == tile.nseg;  // all of the row tile's keys done here
      float* stg = reinterpret_cast<float*>(gptr(sS + wg * kChunk + (warp & 3) * 4096));
      // output rows of the 4 rows this lane stores per chunk (row 8 i + lane / 4
      // of the warp's 32)
      int orow_r[4];
      bool live_r[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int lr = 32 * (warp & 3) + 8 * i + (lane >> 2);
        const int qr = tile.row0 + lr;
        int o_r = (lr < tile.nrows && qr < p.nq) ? (p.row_map ? p.row_map[qr] : qr) : -1;
        live_r[i] = o_r >= 0 && o_r < p.nq;
        orow_r[i] = live_r[i] ? o_r : 0;
      }
      const bool vec_ok = (p.lddq & 3) == 0 && (whole || p.vec_atomics_dq);
      const uint32_t qa = tmem_lane_addr(tmem, warp, c_dq);
      for (int cc = wg; cc < d16; cc += NCG) {
        uint32_t o[16];
        tmem_ld16(qa + 16 * cc, o);  // warp-collective: every lane loads
        tmem_ld_wait();
#pragma unroll
        for (int u = 0; u < 4; ++u)
          *reinterpret_cast<float4*>(stg + lane * 16 + (((u ^ (lane >> 1)) & 3) << 2)) = make_float4(
              __uint_as_float(o[4 * u]) * p.scale, __uint_as_float(o[4 * u + 1]) * p.scale,
              __uint_as_float(o[4 * u + 2]) * p.scale, __uint_as_float(o[4 * u + 3]) * p.scale);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int r = 8 * i + (lane >> 2), u = lane & 3;
          const float4 v = *reinterpret_cast<const float4*>(stg + r * 16 + (((u ^ (r >> 1)) & 3) << 2));
          if (!live_r[i]) continue;
          float* dst = p.dQ + (size_t)orow_r[i] * p.lddq + 16 * cc + 4 * u;
          if (vec_ok) {
            if (whole) *reinterpret_cast<float4*>(dst) = v;
            else atomicAdd(reinterpret_cast<float4*>(dst), v);  // the row tile's keys are split over CTAs
          } else if (whole) {
            dst[0] = v.x;
            dst[1] = v.y;
            dst[2] = v.z;
            dst[3] = v.w;
          } else {
            atomicAdd(dst, v.x);
            atomicAdd(dst + 1, v.y);
            atomicAdd(dst + 2, v.z);
            atomicAdd(dst + 3, v.w);
          }
        }
        __syncwarp();
      }
    }
  } else {
    // ---------------- flush (one warpgroup): thread = key row of the partial dK,
    // and at the end of each run the query row of its dQ
    warpgroup_reg_alloc<176>();
    const int lrow = 32 * (warp & 3) + lane;
    const int qbase = lane & ~3;
    const uint32_t wstage = sStage + (warp & 3) * 8192;  // this warp's two 4 KB boxes
    uint32_t it = 0, wblk = 0, rcount = 0;
    bool ok = true;
    UnitRange ur{s_range[0], s_range[1], s_range[2]};
    int t, jb, je;
    while (ok && (kDqFlush || !kNoDK) && next_segment(ur, p.tiles, ntiles, t, jb, je)) {
      const RowTile tile = p.tiles[t];
      for (int j = jb; j < je && !kNoDK; ++j, ++it) {
        const KeySeg sg = p.segs[tile.seg0 + j];
        const int krow = sg.key0 + lrow;
        int okey = (lrow < sg.nkeys && krow < p.nk) ? (p.col_map ? p.col_map[krow] : krow) : -1;
        if (okey >= p.nk) okey = -1;
        const bool live_key = okey >= 0;
        if (!live_key) okey = 0;
        float* dst = p.dK + (size_t)okey * p.lddk;
        // rows of this thread's lane quad (destination row, liveness): each
        // quad transposes its 4 x 16 values so that one reduction covers 64
        // contiguous bytes of each of 8 rows
        int qkey[4] = {0, 0, 0, 0};
        bool qlive[4] = {false, false, false, false};
        if (!p.dk_tma) {
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            qkey[m] = __shfl_sync(0xffffffffu, okey, qbase + m);
            qlive[m] = __shfl_sync(0xffffffffu, live_key ? 1 : 0, qbase + m) != 0;
          }
        }
        if (!mbar_wait(&bar_dkp_full, it & 1, p.ctl, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t ta = tmem_lane_addr(tmem, warp, c_dkp);
        // the whole partial (d <= 128 columns) in one TMEM round trip, then the
        // columns go back to the MMA issuer before the reductions start
        uint32_t o[8][16];
#pragma unroll
        for (int q = 0; q < 8; ++q)
          if (q < d16) tmem_ld16(ta + 16 * q, o[q]);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&bar_dkp_empty);
        if (p.dk_tma) {
          // Each warp adds its own 32 key rows: 32-column boxes of 32 rows (4 KB),
          // written into the warp's two staging buffers (unit u of a row at
          // u ^ (row & 7), the tensor map's 128-byte swizzle) and handed by lane 0
          // to the TMA unit.  The warp only waits for its own reductions, and the
          // CTA keeps eight of them in flight.
#pragma unroll
          for (int bq = 0; bq < 4; ++bq) {
            if (2 * bq >= d16) break;
            const uint32_t sbuf = wstage + (wblk & 1) * 4096;
            if (wblk >= 2) {
              if (lane == 0) bulk_wait_group_read<1>();  // the box written two rounds ago is read
              __syncwarp();
            }
#pragma unroll
            for (int u = 0; u < 8; ++u) {
              const uint32_t* src = &o[2 * bq + (u >> 2)][4 * (u & 3)];
              asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(
                               sbuf + lane * 128 + ((u ^ (lane & 7)) << 4)),
                           "r"(__float_as_uint(__uint_as_float(src[0]) * p.scale)),
                           "r"(__float_as_uint(__uint_as_float(src[1]) * p.scale)),
                           "r"(__float_as_uint(__uint_as_float(src[2]) * p.scale)),
                           "r"(__float_as_uint(__uint_as_float(src[3]) * p.scale))
                           : "memory");
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) {
              tma_reduce_add_2d(&tm.dk, 32 * bq, sg.key0 + 32 * (warp & 3), gptr(sbuf));
              bulk_commit_group();
            }
            ++wblk;
          }
          continue;
        }
#pragma unroll
        for (int q = 0; q < 8; ++q) {
          if (q >= d16) break;
          const int c0 = 16 * q;
          if (p.vec_atomics) {
            float4 v[4];
#pragma unroll
            for (int c = 0; c < 4; ++c)
              v[c] = make_float4(__uint_as_float(o[q][4 * c]) * p.scale,
                                 __uint_as_float(o[q][4 * c + 1]) * p.scale,
                                 __uint_as_float(o[q][4 * c + 2]) * p.scale,
                                 __uint_as_float(o[q][4 * c + 3]) * p.scale);
            quad_transpose4(v, lane & 3);
            // v[m] = columns [c0 + 4 (lane & 3), +4) of quad row m
#pragma unroll
            for (int m = 0; m < 4; ++m)
              if (qlive[m])
                atomicAdd(reinterpret_cast<float4*>(p.dK + (size_t)qkey[m] * p.lddk + c0 + 4 * (lane & 3)),
                          v[m]);
          } else if (live_key) {
#pragma unroll
            for (int i = 0; i < 16; ++i) atomicAdd(dst + c0 + i, __uint_as_float(o[q][i]) * p.scale);
          }
        }
      }
      if (!ok) break;
      if constexpr (!kDqFlush) continue;
      // dQ / s of this run: its MMAs are complete; the columns are read in one
      // TMEM round trip and handed back to the MMA issuer before the stores.
      // Stored when the run covers all of the row tile's keys, else added
      // (the row tile's keys are split over CTAs).
      if (!mbar_wait(&bar_dq_full, rcount & 1, p.ctl, abort)) break;
      tc_fence_after();
      {
        const uint32_t qa = tmem_lane_addr(tmem, warp, c_dq);
        const bool whole = jb == 0 && je == tile.nseg;
        const int qr = tile.row0 + lrow;
        int orow = (lrow < tile.nrows && qr < p.nq) ? (p.row_map ? p.row_map[qr] : qr) : -1;
        if (orow >= p.nq) orow = -1;
        const bool live = orow >= 0;
        if (!live) orow = 0;
        const bool vec = (p.lddq & 3) == 0 && (whole || p.vec_atomics_dq);
        // the output rows of this thread's lane quad
        int qrow[4];
        bool qlive[4];
#pragma unroll
        for (int m = 0; m < 4; ++m) {
          qrow[m] = __shfl_sync(0xffffffffu, orow, qbase + m);
          qlive[m] = __shfl_sync(0xffffffffu, live ? 1 : 0, qbase + m) != 0;
        }
        // 16 columns of dQ / s: with float4 access each lane quad transposes
        // its 4 x 16 values, so that a float4 of each lane covers 64
        // contiguous bytes of a row with the quad's other lanes
        auto put = [&](int q, const uint32_t (&o)[16]) {
          if (vec) {
            float4 v[4];
#pragma unroll
            for (int c = 0; c < 4; ++c)
              v[c] = make_float4(__uint_as_float(o[4 * c]) * p.scale, __uint_as_float(o[4 * c + 1]) * p.scale,
                                 __uint_as_float(o[4 * c + 2]) * p.scale,
                                 __uint_as_float(o[4 * c + 3]) * p.scale);
            quad_transpose4(v, lane & 3);
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              if (!qlive[m]) continue;
              float4* d4 = reinterpret_cast<float4*>(p.dQ + (size_t)qrow[m] * p.lddq + 16 * q + 4 * (lane & 3));
              if (whole) *d4 = v[m];
              else atomicAdd(d4, v[m]);
            }
          } else if (live) {
            float* dst = p.dQ + (size_t)orow * p.lddq + 16 * q;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float v = __uint_as_float(o[i]) * p.scale;
              if (whole) dst[i] = v;
              else atomicAdd(dst + i, v);
            }
          }
        };
        if constexpr (kFixed) {
          // all d = 128 columns in one TMEM round trip, handed back to the MMA
          // issuer before the stores
          uint32_t o[8][16];
#pragma unroll
          for (int q = 0; q < 8; ++q) tmem_ld16(qa + 16 * q, o[q]);
          tmem_ld_wait();
          tc_fence_before();
          mbar_arrive(&bar_dq_empty);
#pragma unroll
          for (int q = 0; q < 8; ++q) put(q, o[q]);
        } else {
          for (int q = 0; q < d16; ++q) {
            uint32_t o[16];
            tmem_ld16(qa + 16 * q, o);
            tmem_ld_wait();
            put(q, o);
          }
          tc_fence_before();
          mbar_arrive(&bar_dq_empty);
        }
      }
      ++rcount;
    }
    // the reductions still in flight must finish before the CTA exits
    if (lane == 0 && p.dk_tma) bulk_wait_group_all();
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ backward, dV (dense)
// Key-stationary dV = P^T dO for the dense coupling: a CTA holds one key tile
// K_j (128 keys) and streams the query row tiles i past it,
//   S^T = K_j Q_i^T                (SS, both K-major)   -> TMEM [0,128) / [128,256)
//   P^T = exp2(S^T s log2e - lse_i log2e)  per column i (the softmax of row i is
//         already normalised by its lse: no running max, no row sum)
//   dV_j += P^T dO_i               (TS: P^T from TMEM, dO_i MN-major) -> TMEM [256, 256 + kp)
// so dV accumulates on chip and leaves once per key tile; no partial dV per
// (row tile, key tile) goes through L2 reductions.  Units (key tile, row tile)
// are numbered key-tile-major and split evenly over the CTAs; a key tile whose
// row tiles two CTAs share is added into dV atomically by both.
// Warps: 0 producer (K_j once per key tile; Q_i into a 2-stage ring), 1 MMA
// issuer and TMEM owner, 2..2+4 NWG-1 the P^T warpgroups (thread = key row,
// the warpgroups split the 128 query columns and nothing orders them against
// each other, so each packs its bf16 P^T over its own S columns only),
// 2+4 NWG the dO producer, whose
// 32 lanes also stage lse_i log2e of the tile's rows in shared memory (+inf
// past the last row, which zeroes those columns of P^T).
struct DvRange {
  int t, j, left;  // key tile, first row tile in it, units still to do
};
__device__ __forceinline__ bool dv_next(DvRange& r, int nkt, int nrt, int& t, int& jb, int& je) {
  if (r.left <= 0 || r.t >= nkt) return false;
  const int take = min(nrt - r.j, r.left);
  t = r.t;
  jb = r.j;
  je = r.j + take;
  r.left -= take;
  ++r.t;
  r.j = 0;
  return true;
}

template <int NWG, int QCH, int VF, int VR>
__global__ void __launch_bounds__(96 + 128 * NWG, 1)
    tc_dv_kernel(const __grid_constant__ TensorMaps tm, const TcParams p) {
  constexpr bool kFixed = QCH > 0;
  const int qch = kFixed ? QCH : p.qch;
  const int vf = kFixed ? VF : p.vf;
  const int vr = kFixed ? VR : p.vr;
  const int d16 = kFixed ? 4 * QCH : p.d / 16;
  constexpr int CW = 128 / NWG;  // query columns per P^T thread
  constexpr int NC = CW / 32;
  constexpr int NSM = 128 * NWG;
  constexpr int kGWarp = 2 + 4 * NWG;  // dO producer
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_k_full, bar_k_empty, bar_q_full[2], bar_q_empty[2], bar_g_full[2],
      bar_g_empty[2], bar_l_full[2], bar_s_full[2], bar_p_full[2], bar_dv_full, bar_drain;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ __align__(16) float s_lse2[2][128];  // lse_i log2e of the stage's rows
  __shared__ int s_range[3];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base_u = smem_u32(smem_raw);
  const uint32_t sbase = (base_u + 1023u) & ~1023u;
  auto gptr = [&](uint32_t sa) { return smem_raw + (sa - base_u); };
  const int qbytes = qch * kChunk;
  const int gbytes = vtile_bytes(vf, vr);
  const uint32_t sK = sbase;             // the stationary key tile
  const uint32_t sQ0 = sK + qbytes;      // Q stage s at sQ0 + s * qbytes
  const uint32_t sG0 = sQ0 + 2 * qbytes; // dO stage s at sG0 + s * gbytes
  const int nkt = (p.nk + 127) / 128, nrt = (p.nq + 127) / 128;

  if (threadIdx.x == 0) {
    mbar_init(&bar_k_full, 1);
    mbar_init(&bar_k_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_q_full[i], 1);
      mbar_init(&bar_q_empty[i], 1);
      mbar_init(&bar_g_full[i], 1);
      mbar_init(&bar_g_empty[i], 1);
      mbar_init(&bar_l_full[i], 32);
      mbar_init(&bar_s_full[i], 1);
      mbar_init(&bar_p_full[i], NSM);
    }
    mbar_init(&bar_dv_full, 1);
    mbar_init(&bar_drain, 1);
    s_abort = 0;
    fence_barrier_init();
    const long long U = (long long)nkt * nrt;
    const long long u0 = (long long)blockIdx.x * U / gridDim.x;
    const long long u1 = (long long)(blockIdx.x + 1) * U / gridDim.x;
    s_range[0] = nrt > 0 ? (int)(u0 / nrt) : 0;
    s_range[1] = nrt > 0 ? (int)(u0 % nrt) : 0;
    s_range[2] = (int)(u1 - u0);
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm.q);
    tma_prefetch_desc(&tm.k);
    tma_prefetch_desc(&tm.g);
    if (vr) tma_prefetch_desc(&tm.gr);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort = &s_abort;

  if (warp == 0) {
    // ---------------- producer: K_j once per key tile, Q_i into a 2-stage ring
    if (lane == 0) {
      uint32_t g = 0, tcount = 0;
      int k_issued = -1;
      bool ok = true;
      DvRange r{s_range[0], s_range[1], s_range[2]};
      int t, jb, je;
      while (ok && !*abort && dv_next(r, nkt, nrt, t, jb, je)) {
        if (tcount > 0 && !mbar_wait(&bar_k_empty, (tcount - 1) & 1, p.ctl, abort)) break;
        mbar_arrive_expect_tx(&bar_k_full, qbytes);
        for (int c = 0; c < qch; ++c)
          tma_load_2d(gptr(sK) + c * kChunk, &tm.k, 64 * c, 128 * t, &bar_k_full);
        k_issued = (int)tcount;
        for (int j = jb; j < je; ++j, ++g) {
          const int st = g & 1;
          if (g >= 2 && !mbar_wait(&bar_q_empty[st], ((g >> 1) - 1) & 1, p.ctl, abort)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar_q_full[st], qbytes);
          for (int c = 0; c < qch; ++c)
            tma_load_2d(gptr(sQ0 + st * qbytes) + c * kChunk, &tm.q, 64 * c, 128 * j, &bar_q_full[st]);
        }
        ++tcount;
      }
      if (*abort) {
        // let the copies already issued land before the CTA can exit
        volatile int never = 0;
        if (k_issued >= 0) mbar_wait(&bar_k_full, k_issued & 1, p.ctl, &never);
        for (uint32_t h = g >= 2 ? g - 2 : 0; h < g; ++h)
          mbar_wait(&bar_q_full[h & 1], (h >> 1) & 1, p.ctl, &never);
      }
    }
  } else if (warp == kGWarp) {
    // ---------------- producer: dO_i into a 2-stage ring (lane 0) and the
    // stage's lse_i log2e (all lanes)
    uint32_t g = 0;
    bool ok = true;
    DvRange r{s_range[0], s_range[1], s_range[2]};
    int t, jb, je;
    while (ok && !*abort && dv_next(r, nkt, nrt, t, jb, je)) {
      for (int j = jb; j < je; ++j, ++g) {
        const int st = g & 1;
        if (g >= 2 && !mbar_wait(&bar_g_empty[st], ((g >> 1) - 1) & 1, p.ctl, abort)) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&bar_g_full[st], gbytes);
          uint8_t* dg = gptr(sG0 + st * gbytes);
          for (int c = 0; c < vf; ++c)
            tma_load_2d(dg + c * kChunk, &tm.g, 64 * c, 128 * j, &bar_g_full[st]);
          if (vr) tma_load_2d(dg + vf * kChunk, &tm.gr, 64 * vf, 128 * j, &bar_g_full[st]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int row = 128 * j + 32 * q + lane;
          s_lse2[st][32 * q + lane] = row < p.nq ? p.lse_in[row] * kLog2e : INFINITY;
        }
        mbar_arrive(&bar_l_full[st]);
      }
    }
    if (*abort && lane == 0) {
      volatile int never = 0;
      for (uint32_t h = g >= 2 ? g - 2 : 0; h < g; ++h)
        mbar_wait(&bar_g_full[h & 1], (h >> 1) & 1, p.ctl, &never);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = make_idesc_bf16(128, 128, 0, 0);
      const uint32_t idesc_pv = make_idesc_bf16(128, 64 * (vf > 0 ? vf : 1), 0, 1);
      const uint32_t idesc_pvr = make_idesc_bf16(128, vr > 0 ? vr : 16, 0, 1);
      const uint32_t dv_col = tmem + 256;
      const uint32_t rsw = rem_swizzle(vr);
      const uint32_t rrow = (uint32_t)vr * 2;  // bytes per row of the remainder box
      uint32_t g0 = 0, tcount = 0;
      bool ok = true;
      // S^T_g = K_j Q_g^T into S buffer g & 1 (Q stage g & 1)
      auto issue_s = [&](uint32_t g) -> bool {
        const int st = g & 1;
        if (!mbar_wait(&bar_q_full[st], (g >> 1) & 1, p.ctl, abort)) return false;
        tc_fence_after();
        const uint32_t sq = sQ0 + st * qbytes;
        const uint32_t d_tmem = tmem + st * 128;
#pragma unroll
        for (int kk = 0; kk < d16; ++kk) {
          const uint32_t off = (kk >> 2) * kChunk + (kk & 3) * 32;
          mma_ss(d_tmem, make_sdesc(sK + off, 16, 1024, kSw128), make_sdesc(sq + off, 16, 1024, kSw128),
                 idesc_s, kk > 0);
        }
        mma_commit(&bar_s_full[st]);
        mma_commit(&bar_q_empty[st]);
        return true;
      };
      DvRange r{s_range[0], s_range[1], s_range[2]};
      int t, jb, je;
      while (ok && dv_next(r, nkt, nrt, t, jb, je)) {
        const int nu = je - jb;
        if (!mbar_wait(&bar_k_full, tcount & 1, p.ctl, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int j = 0; j < min(2, nu) && ok; ++j) ok = issue_s(g0 + j);
        for (int j = 0; j < nu && ok; ++j) {
          const uint32_t g = g0 + j;
          const int buf = g & 1;
          if (!mbar_wait(&bar_p_full[buf], (g >> 1) & 1, p.ctl, abort) ||
              !mbar_wait(&bar_g_full[buf], (g >> 1) & 1, p.ctl, abort)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // dV += P^T dO_g : A = P^T (bf16 pairs, each warpgroup's CW query
          // columns packed at the start of its own CW S columns), B = dO_g MN-major
          const uint32_t sg = sG0 + buf * gbytes;
          const uint32_t a_tmem = tmem + buf * 128;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t acc = (j > 0 || kk > 0) ? 1u : 0u;
            const uint32_t pcol = 8 * kk + ((16 * kk) / CW) * (CW / 2);
            if (vf > 0)
              mma_ts(dv_col, a_tmem + pcol, make_sdesc(sg + kk * 2048, kChunk, 1024, kSw128),
                     idesc_pv, acc);
            if (vr > 0)
              mma_ts(dv_col + 64 * vf, a_tmem + pcol,
                     make_sdesc(sg + vf * kChunk + kk * 16 * rrow, 128 * rrow, 8 * rrow, rsw),
                     idesc_pvr, acc);
          }
          mma_commit(&bar_g_empty[buf]);
          if (j + 2 < nu) ok = issue_s(g + 2);
        }
        if (!ok) break;
        mma_commit(&bar_k_empty);
        mma_commit(&bar_dv_full);
        g0 += nu;
        ++tcount;
      }
      // drain: wait until every tensor-core op issued here has completed
      mma_commit(&bar_drain);
      volatile int never = 0;
      mbar_wait(&bar_drain, 0, p.ctl, &never);
    }
  } else if (warp >= 2 && warp < kGWarp) {
    // ---------------- P^T (NWG warpgroups): thread = key row (TMEM lane); the
    // warpgroups split the 128 query columns; epilogue dV per key tile
    const int wg = (warp - 2) >> 2;
    const int lrow = 32 * (warp & 3) + lane;
    const int col0 = wg * CW;
    const int nchunk = p.kp / 16;
    uint32_t g0 = 0, tcount = 0;
    bool ok = true;
    DvRange r{s_range[0], s_range[1], s_range[2]};
    int t, jb, je;
    while (ok && dv_next(r, nkt, nrt, t, jb, je)) {
      const int nu = je - jb;
      for (int j = 0; j < nu; ++j) {
        const uint32_t g = g0 + j;
        const int buf = g & 1;
        if (!mbar_wait(&bar_s_full[buf], (g >> 1) & 1, p.ctl, abort) ||
            !mbar_wait(&bar_l_full[buf], (g >> 1) & 1, p.ctl, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t x[NC][32];
        const uint32_t sa = tmem_lane_addr(tmem, warp, buf * 128 + col0);
#pragma unroll
        for (int c = 0; c < NC; ++c) tmem_ld32(sa + 32 * c, x[c]);
        tmem_ld_wait();
        // P^T = exp2(S^T s log2e - lse_i log2e); columns past the last query row
        // carry lse = +inf and give 0
        const float4* l4 = reinterpret_cast<const float4*>(&s_lse2[buf][col0]);
        uint32_t pk[NC][16];
#pragma unroll
        for (int c = 0; c < NC; ++c)
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 lv = l4[8 * c + q];
            const float a0 = ex2_approx(fmaf(__uint_as_float(x[c][4 * q]), p.scale_log2, -lv.x));
            const float a1 = ex2_approx(fmaf(__uint_as_float(x[c][4 * q + 1]), p.scale_log2, -lv.y));
            const float a2 = ex2_approx(fmaf(__uint_as_float(x[c][4 * q + 2]), p.scale_log2, -lv.z));
            const float a3 = ex2_approx(fmaf(__uint_as_float(x[c][4 * q + 3]), p.scale_log2, -lv.w));
            pk[c][2 * q] = pack_bf16x2(a0, a1);
            pk[c][2 * q + 1] = pack_bf16x2(a2, a3);
          }
        // packed into the first half of this warpgroup's own S columns (already
        // read by this thread): the other warpgroup may still be reading its S
        const uint32_t pa = tmem_lane_addr(tmem, warp, buf * 128 + col0);
#pragma unroll
        for (int c = 0; c < NC; ++c) tmem_st16(pa + 16 * c, pk[c]);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bar_p_full[buf]);
      }
      if (!ok) break;
      // epilogue: the key tile's dV rows; a key tile shared with another CTA is
      // added atomically (dV is zeroed by the caller)
      if (!mbar_wait(&bar_dv_full, tcount & 1, p.ctl, abort)) break;
      tc_fence_after();
      const int key = 128 * t + lrow;
      const bool live = key < p.nk;
      const bool whole = jb == 0 && je == nrt;
      float* dst = p.dV + (size_t)(live ? key : 0) * p.lddv;
      const uint32_t da = tmem_lane_addr(tmem, warp, 256);
      for (int c = wg; c < nchunk; c += NWG) {
        uint32_t o[16];
        tmem_ld16(da + 16 * c, o);
        tmem_ld_wait();
        if (!live) continue;
        const int c0 = 16 * c;
        if (c0 + 16 <= p.k && p.vec_atomics) {
#pragma unroll
          for (int i = 0; i < 16; i += 4) {
            const float4 v = make_float4(__uint_as_float(o[i]), __uint_as_float(o[i + 1]),
                                         __uint_as_float(o[i + 2]), __uint_as_float(o[i + 3]));
            if (whole) *reinterpret_cast<float4*>(dst + c0 + i) = v;
            else atomicAdd(reinterpret_cast<float4*>(dst + c0 + i), v);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i)
            if (c0 + i < p.k) {
              if (whole) dst[c0 + i] = __uint_as_float(o[i]);
              else atomicAdd(dst + c0 + i, __uint_as_float(o[i]));
            }
        }
      }
      g0 += nu;
      ++tcount;
    }
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ backward, dK (dense, deterministic)
// Key-stationary dK = scale dS^T Q for the dense coupling: a CTA keeps one key
// tile (K_j and V_j) and streams the query row tiles i past it,
//   S^T  = K_j Q_i^T          (SS, both K-major)            -> TMEM [0,128) / [128,256)
//   dP^T = V_j dO_i^T         (SS, both K-major, K = kp)     -> TMEM [256,384)
//   P^T  = exp2(S^T s log2e - lse_i log2e),  dS^T = P^T (dP^T - D_i)
//          -> bf16 pairs over this warpgroup's own S^T columns
//   dK_j += dS^T Q_i          (TS: dS^T from TMEM, Q_i MN-major) -> TMEM [384, 384 + d)
// The units (key tile, row tile) are numbered key-tile-major and split evenly
// over no more CTAs than there are key tiles, so a key tile is shared by at
// most two CTAs: the first atomic add into the zeroed dK is exact and the
// second commutes with it, so dK is the same bit for bit on every run.
// Warps: 0 producer (K_j and V_j once per key tile, Q_i into a 2-stage ring),
// 1 MMA issuer and TMEM owner, 2..2+4 NWG-1 the dS^T warpgroups (thread = key
// row; the warpgroups split the 128 query columns), 2+4 NWG the dO producer,
// whose lanes also stage lse_i log2e (+inf past the last row) and D_i.
// The MMA issuer runs dP^T_g, dK_{g-1}, S^T_{g+1} per row tile, so dP^T_g
// overlaps the dS^T work of row tile g-1.
template <int NWG, int QCH, int VF, int VR>
__global__ void __launch_bounds__(96 + 128 * NWG, 1)
    tc_dk_kernel(const __grid_constant__ TensorMaps tm, const TcParams p) {
  constexpr bool kFixed = QCH > 0;
  const int qch = kFixed ? QCH : p.qch;
  const int vf = kFixed ? VF : p.vf;
  const int vr = kFixed ? VR : p.vr;
  const int d16 = kFixed ? 4 * QCH : p.d / 16;
  constexpr int CW = 128 / NWG;  // query columns per dS^T thread
  constexpr int NC = CW / 32;
  constexpr int NSM = 128 * NWG;
  constexpr int kGWarp = 2 + 4 * NWG;  // dO producer
  extern __shared__ uint8_t smem_raw[];
  __shared__ uint64_t bar_kv_full, bar_kv_empty, bar_q_full[2], bar_q_empty[2], bar_g_full,
      bar_g_empty, bar_l_full[2], bar_l_empty[2], bar_s_full[2], bar_dp_full, bar_dp_read,
      bar_p_full[2], bar_dk_full, bar_dk_empty, bar_drain;
  __shared__ uint32_t s_tmem;
  __shared__ int s_abort;
  __shared__ __align__(16) float s_lse2[2][128];  // lse_i log2e of the stage's rows
  __shared__ __align__(16) float s_D[2][128];     // D_i of the stage's rows
  __shared__ int s_range[3];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t base_u = smem_u32(smem_raw);
  const uint32_t sbase = (base_u + 1023u) & ~1023u;
  auto gptr = [&](uint32_t sa) { return smem_raw + (sa - base_u); };
  const int qbytes = qch * kChunk;
  const int vbytes = vtile_bytes(vf, vr);
  const uint32_t sK = sbase;             // the stationary key tile
  const uint32_t sV = sK + qbytes;       // its V rows
  const uint32_t sQ0 = sV + vbytes;      // Q stage s at sQ0 + s * qbytes
  const int QS = p.vstages;                // Q ring depth (2, or 1 when k is large)
  const uint32_t sG = sQ0 + QS * qbytes;  // the dO tile (one stage)
  const int nkt = (p.nk + 127) / 128, nrt = (p.nq + 127) / 128;
  const uint32_t c_dp = 256, c_dk = 384;

  if (threadIdx.x == 0) {
    mbar_init(&bar_kv_full, 1);
    mbar_init(&bar_kv_empty, 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&bar_q_full[i], 1);
      mbar_init(&bar_q_empty[i], 1);
      mbar_init(&bar_l_full[i], 32);
      mbar_init(&bar_l_empty[i], NSM);
      mbar_init(&bar_s_full[i], 1);
      mbar_init(&bar_p_full[i], NSM);
    }
    mbar_init(&bar_g_full, 1);
    mbar_init(&bar_g_empty, 1);
    mbar_init(&bar_dp_full, 1);
    mbar_init(&bar_dp_read, NSM);
    mbar_init(&bar_dk_full, 1);
    mbar_init(&bar_dk_empty, NSM);
    mbar_init(&bar_drain, 1);
    s_abort = 0;
    fence_barrier_init();
    const long long U = (long long)nkt * nrt;
    const long long u0 = (long long)blockIdx.x * U / gridDim.x;
    const long long u1 = (long long)(blockIdx.x + 1) * U / gridDim.x;
    s_range[0] = nrt > 0 ? (int)(u0 / nrt) : 0;
    s_range[1] = nrt > 0 ? (int)(u0 % nrt) : 0;
    s_range[2] = (int)(u1 - u0);
  }
  if (warp == 1) {
    tmem_alloc(&s_tmem, 512);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tm.q);
    tma_prefetch_desc(&tm.k);
    tma_prefetch_desc(&tm.v);
    tma_prefetch_desc(&tm.g);
    if (vr) {
      tma_prefetch_desc(&tm.vr);
      tma_prefetch_desc(&tm.gr);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = s_tmem;
  volatile int* abort = &s_abort;

  if (warp == 0) {
    // ---------------- producer: K_j and V_j once per key tile, Q_i ring
    if (lane == 0) {
      uint32_t g = 0, tcount = 0;
      int kv_issued = -1;
      bool ok = true;
      DvRange r{s_range[0], s_range[1], s_range[2]};
      int t, jb, je;
      while (ok && !*abort && dv_next(r, nkt, nrt, t, jb, je)) {
        if (tcount > 0 && !mbar_wait(&bar_kv_empty, (tcount - 1) & 1, p.ctl, abort)) break;
        mbar_arrive_expect_tx(&bar_kv_full, qbytes + vbytes);
        for (int c = 0; c < qch; ++c)
          tma_load_2d(gptr(sK) + c * kChunk, &tm.k, 64 * c, 128 * t, &bar_kv_full);
        for (int c = 0; c < vf; ++c)
          tma_load_2d(gptr(sV) + c * kChunk, &tm.v, 64 * c, 128 * t, &bar_kv_full);
        if (vr) tma_load_2d(gptr(sV) + vf * kChunk, &tm.vr, 64 * vf, 128 * t, &bar_kv_full);
        kv_issued = (int)tcount;
        for (int j = jb; j < je; ++j, ++g) {
          const int st = g % QS;
          if (g >= (uint32_t)QS && !mbar_wait(&bar_q_empty[st], ((g / QS) - 1) & 1, p.ctl, abort)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bar_q_full[st], qbytes);
          for (int c = 0; c < qch; ++c)
            tma_load_2d(gptr(sQ0 + st * qbytes) + c * kChunk, &tm.q, 64 * c, 128 * j, &bar_q_full[st]);
        }
        ++tcount;
      }
      if (*abort) {
        // let the copies already issued land before the CTA can exit
        volatile int never = 0;
        if (kv_issued >= 0) mbar_wait(&bar_kv_full, kv_issued & 1, p.ctl, &never);
        for (uint32_t h = g >= (uint32_t)QS ? g - QS : 0; h < g; ++h)
          mbar_wait(&bar_q_full[h % QS], (h / QS) & 1, p.ctl, &never);
      }
    }
  } else if (warp == kGWarp) {
    // ---------------- producer: dO_i (one stage, lane 0) and the stage's
    // lse_i log2e and D_i (all lanes)
    uint32_t g = 0;
    bool ok = true;
    DvRange r{s_range[0], s_range[1], s_range[2]};
    int t, jb, je;
    while (ok && !*abort && dv_next(r, nkt, nrt, t, jb, je)) {
      for (int j = jb; j < je; ++j, ++g) {
        const int st = g & 1;
        // the dO stage is free once dP^T of the previous row tile is done; the
        // lse / D stage once the dS^T of two row tiles back has used it
        if ((g >= 1 && !mbar_wait(&bar_g_empty, (g - 1) & 1, p.ctl, abort)) ||
            (g >= 2 && !mbar_wait(&bar_l_empty[st], ((g >> 1) - 1) & 1, p.ctl, abort))) {
          ok = false;
          break;
        }
        if (lane == 0) {
          mbar_arrive_expect_tx(&bar_g_full, vbytes);
          for (int c = 0; c < vf; ++c)
            tma_load_2d(gptr(sG) + c * kChunk, &tm.g, 64 * c, 128 * j, &bar_g_full);
          if (vr) tma_load_2d(gptr(sG) + vf * kChunk, &tm.gr, 64 * vf, 128 * j, &bar_g_full);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int row = 128 * j + 32 * q + lane;
          s_lse2[st][32 * q + lane] = row < p.nq ? p.lse_in[row] * kLog2e : INFINITY;
          s_D[st][32 * q + lane] = row < p.nq ? p.Dvec[row] : 0.f;
        }
        mbar_arrive(&bar_l_full[st]);
      }
    }
    if (*abort && lane == 0 && g >= 1) {
      volatile int never = 0;
      mbar_wait(&bar_g_full, (g - 1) & 1, p.ctl, &never);
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s = make_idesc_bf16(128, 128, 0, 0);
      const uint32_t idesc_dk = make_idesc_bf16(128, p.d, 0, 1);
      const uint32_t rsw = rem_swizzle(vr);
      const uint32_t rrow = (uint32_t)vr * 2;  // bytes per row of the remainder box
      uint32_t g0 = 0, tcount = 0;
      bool ok = true;
      // S^T_g = K_j Q_g^T into S buffer g & 1 (Q stage g % QS)
      auto issue_s = [&](uint32_t g) -> bool {
        const int qs = g % QS;
        if (!mbar_wait(&bar_q_full[qs], (g / QS) & 1, p.ctl, abort)) return false;
        tc_fence_after();
        const uint32_t sq = sQ0 + qs * qbytes;
#pragma unroll
        for (int kk = 0; kk < d16; ++kk) {
          const uint32_t off = (kk >> 2) * kChunk + (kk & 3) * 32;
          mma_ss(tmem + (g & 1) * 128, make_sdesc(sK + off, 16, 1024, kSw128),
                 make_sdesc(sq + off, 16, 1024, kSw128), idesc_s, kk > 0);
        }
        mma_commit(&bar_s_full[g & 1]);
        return true;
      };
      // dK_j += dS^T_g Q_g : A = dS^T (bf16 pairs, each warpgroup's CW query
      // columns packed at the start of its own CW S columns), B = Q_g MN-major
      auto issue_dk = [&](uint32_t g, bool first) -> bool {
        const int st = g & 1, qs = g % QS;
        if (!mbar_wait(&bar_p_full[st], (g >> 1) & 1, p.ctl, abort)) return false;
        tc_fence_after();
        const uint32_t sq = sQ0 + qs * qbytes;
        const uint32_t a_tmem = tmem + st * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t pcol = 8 * kk + ((16 * kk) / CW) * (CW / 2);
          mma_ts(tmem + c_dk, a_tmem + pcol, make_sdesc(sq + kk * 2048, kChunk, 1024, kSw128), idesc_dk,
                 (!first || kk > 0) ? 1u : 0u);
        }
        mma_commit(&bar_q_empty[qs]);
        return true;
      };
      DvRange r{s_range[0], s_range[1], s_range[2]};
      int t, jb, je;
      while (ok && dv_next(r, nkt, nrt, t, jb, je)) {
        const int nu = je - jb;
        if (!mbar_wait(&bar_kv_full, tcount & 1, p.ctl, abort) ||
            (tcount > 0 && !mbar_wait(&bar_dk_empty, (tcount - 1) & 1, p.ctl, abort))) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int j = 0; j < min(QS, nu) && ok; ++j) ok = issue_s(g0 + j);
        for (int j = 0; j < nu && ok; ++j) {
          const uint32_t g = g0 + j;
          // dP^T_g = V_j dO_g^T once dO_g is in and dP^T_{g-1} has been read
          if (!mbar_wait(&bar_g_full, g & 1, p.ctl, abort) ||
              (g >= 1 && !mbar_wait(&bar_dp_read, (g - 1) & 1, p.ctl, abort))) {
            ok = false;
            break;
          }
          tc_fence_after();
          int kk = 0;
#pragma unroll
          for (int c = 0; c < vf; ++c)
#pragma unroll
            for (int u = 0; u < 4; ++u, ++kk) {
              const uint32_t off = c * kChunk + u * 32;
              mma_ss(tmem + c_dp, make_sdesc(sV + off, 16, 1024, kSw128),
                     make_sdesc(sG + off, 16, 1024, kSw128), idesc_s, kk > 0);
            }
#pragma unroll
          for (int u = 0; u < vr / 16; ++u, ++kk) {
            const uint32_t off = vf * kChunk + u * 32;
            mma_ss(tmem + c_dp, make_sdesc(sV + off, 16, 8 * rrow, rsw),
                   make_sdesc(sG + off, 16, 8 * rrow, rsw), idesc_s, kk > 0);
          }
          mma_commit(&bar_g_empty);
          mma_commit(&bar_dp_full);
          if (QS == 2) {
            // dK_{g-1}, then S^T_{g+1} into the S buffer dK_{g-1} reads (issued after it)
            if (j >= 1 && (!issue_dk(g - 1, j == 1) || (j + 1 < nu && !issue_s(g + 1)))) {
              ok = false;
              break;
            }
          } else {
            // one Q stage: dK_g must be done with Q_g before Q_{g+1} can load
            if (!issue_dk(g, j == 0) || (j + 1 < nu && !issue_s(g + 1))) {
              ok = false;
              break;
            }
          }
        }
        if (!ok) break;
        if (QS == 2 && !issue_dk(g0 + nu - 1, nu == 1)) {
          ok = false;
          break;
        }
        mma_commit(&bar_kv_empty);
        mma_commit(&bar_dk_full);
        g0 += nu;
        ++tcount;
      }
      // drain: wait until every tensor-core op issued here has completed
      mma_commit(&bar_drain);
      volatile int never = 0;
      mbar_wait(&bar_drain, 0, p.ctl, &never);
    }
  } else if (warp >= 2 && warp < kGWarp) {
    // ---------------- dS^T (NWG warpgroups): thread = key row (TMEM lane); the
    // warpgroups split the 128 query columns; epilogue dK per key tile
    const int wg = (warp - 2) >> 2;
    const int lrow = 32 * (warp & 3) + lane;
    const int col0 = wg * CW;
    uint32_t g0 = 0, tcount = 0;
    bool ok = true;
    DvRange r{s_range[0], s_range[1], s_range[2]};
    int t, jb, je;
    while (ok && dv_next(r, nkt, nrt, t, jb, je)) {
      const int nu = je - jb;
      for (int j = 0; j < nu; ++j) {
        const uint32_t g = g0 + j;
        const int buf = g & 1;
        if (!mbar_wait(&bar_s_full[buf], (g >> 1) & 1, p.ctl, abort) ||
            !mbar_wait(&bar_l_full[buf], (g >> 1) & 1, p.ctl, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t x[NC][32];
        const uint32_t sa = tmem_lane_addr(tmem, warp, buf * 128 + col0);
#pragma unroll
        for (int c = 0; c < NC; ++c) tmem_ld32(sa + 32 * c, x[c]);
        tmem_ld_wait();
        // P^T = exp2(S^T s log2e - lse_i log2e); columns past the last query row
        // carry lse = +inf and give 0
        const float4* l4 = reinterpret_cast<const float4*>(&s_lse2[buf][col0]);
        float pr[NC][32];
#pragma unroll
        for (int c = 0; c < NC; ++c)
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 lv = l4[8 * c + q];
            pr[c][4 * q] = ex2_approx(fmaf(__uint_as_float(x[c][4 * q]), p.scale_log2, -lv.x));
            pr[c][4 * q + 1] = ex2_approx(fmaf(__uint_as_float(x[c][4 * q + 1]), p.scale_log2, -lv.y));
            pr[c][4 * q + 2] = ex2_approx(fmaf(__uint_as_float(x[c][4 * q + 2]), p.scale_log2, -lv.z));
            pr[c][4 * q + 3] = ex2_approx(fmaf(__uint_as_float(x[c][4 * q + 3]), p.scale_log2, -lv.w));
          }
        if (!mbar_wait(&bar_dp_full, g & 1, p.ctl, abort)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t da = tmem_lane_addr(tmem, warp, c_dp + col0);
#pragma unroll
        for (int c = 0; c < NC; ++c) tmem_ld32(da + 32 * c, x[c]);
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive(&bar_dp_read);  // the dP columns may receive the next dP^T
        const float4* d4 = reinterpret_cast<const float4*>(&s_D[buf][col0]);
        uint32_t pk[NC][16];
#pragma unroll
        for (int c = 0; c < NC; ++c)
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            const float4 dv = d4[8 * c + q];
            pk[c][2 * q] = pack_bf16x2(pr[c][4 * q] * (__uint_as_float(x[c][4 * q]) - dv.x),
                                       pr[c][4 * q + 1] * (__uint_as_float(x[c][4 * q + 1]) - dv.y));
            pk[c][2 * q + 1] = pack_bf16x2(pr[c][4 * q + 2] * (__uint_as_float(x[c][4 * q + 2]) - dv.z),
                                           pr[c][4 * q + 3] * (__uint_as_float(x[c][4 * q + 3]) - dv.w));
          }
        mbar_arrive(&bar_l_empty[buf]);  // lse and D of this stage are no longer read
        // packed into the first half of this warpgroup's own S columns (already
        // read by this thread): the other warpgroup may still be reading its S
        const uint32_t pa = tmem_lane_addr(tmem, warp, buf * 128 + col0);
#pragma unroll
        for (int c = 0; c < NC; ++c) tmem_st16(pa + 16 * c, pk[c]);
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(&bar_p_full[buf]);
      }
      if (!ok) break;
      // epilogue: the key tile's dK rows; a key tile shared with another CTA is
      // added atomically (dK is zeroed by the caller; at most two adds, which
      // commute)
      if (!mbar_wait(&bar_dk_full, tcount & 1, p.ctl, abort)) break;
      tc_fence_after();
      const int key = 128 * t + lrow;
      const bool live = key < p.nk;
      const bool whole = jb == 0 && je == nrt;
      float* dst = p.dK + (size_t)(live ? key : 0) * p.lddk;
      const uint32_t ka = tmem_lane_addr(tmem, warp, c_dk);
      for (int c = wg; c < d16; c += NWG) {
        uint32_t o[16];
        tmem_ld16(ka + 16 * c, o);
        tmem_ld_wait();
        if (!live) continue;
        const int c0 = 16 * c;
        if (p.vec_atomics) {
#pragma unroll
          for (int i = 0; i < 16; i += 4) {
            const float4 v = make_float4(__uint_as_float(o[i]) * p.scale, __uint_as_float(o[i + 1]) * p.scale,
                                         __uint_as_float(o[i + 2]) * p.scale,
                                         __uint_as_float(o[i + 3]) * p.scale);
            if (whole) *reinterpret_cast<float4*>(dst + c0 + i) = v;
            else atomicAdd(reinterpret_cast<float4*>(dst + c0 + i), v);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            if (whole) dst[c0 + i] = __uint_as_float(o[i]) * p.scale;
            else atomicAdd(dst + c0 + i, __uint_as_float(o[i]) * p.scale);
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&bar_dk_empty);  // the dK columns may receive the next key tile
      g0 += nu;
      ++tcount;
    }
  }

  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

__global__ void wait_probe_kernel(WaitCtl ctl) {
  __shared__ uint64_t bar;
  __shared__ int s_abort;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    s_abort = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(&bar, 0, ctl, &s_abort);  // nothing ever arrives
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
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

// 2-D bf16 tensor [rows, cols] with leading dimension ld (elements); box of
// {box_cols, 128}; columns >= cols and rows >= rows read as zero.
bool make_map(CUtensorMap* m, const void* ptr, int rows, int cols, int ld, int box_cols,
              CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)ld * 2};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, 128};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), gdim, gstride, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D fp32 tensor [rows, cols] with leading dimension ld (elements), box
// {box_cols, box_rows}; elements outside the tensor are skipped by reductions.
bool make_map_f32(CUtensorMap* m, const void* ptr, int rows, int cols, int ld, int box_cols,
                  int box_rows, CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)ld * 4};
  cuuint32_t box[2] = {(cuuint32_t)box_cols, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(ptr), gdim, gstride, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

CUtensorMapSwizzle rem_sw_host(int vr) {
  return vr == 16 ? CU_TENSOR_MAP_SWIZZLE_32B : CU_TENSOR_MAP_SWIZZLE_64B;
}

int padded_k(int k) {
  int kp = (k + 15) / 16 * 16;
  if (kp % 64 == 48) kp += 16;
  return kp;
}

int num_sms() {
  static int n = 0;
  if (!n) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (n <= 0) n = 148;
  }
  return n;
}

int smem_optin() {
  static int v = 0;
  if (!v) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
    if (v <= 0) v = 232448;
  }
  return v;
}

std::atomic<int> g_stall_next{0};
// 1 for the launch that takes the armed abort-path hook of kernel `which`.
int take_stall(int which) {
  int expected = which;
  return g_stall_next.compare_exchange_strong(expected, 0) ? 1 : 0;
}

void fill_common(const TcArgs& a, TcParams& p) {
  std::memset(&p, 0, sizeof(p));
  p.tiles = a.tiles;
  p.segs = a.segs;
  p.ntiles_dev = a.ntiles_dev;
  p.ntiles_host = a.ntiles_host;
  p.tile_prefix = a.tile_prefix;
  p.row_map = a.row_map;
  p.col_map = a.col_map;
  p.d = a.d;
  p.k = a.k;
  p.nq = a.nQrows;
  p.nk = a.nKrows;
  p.kp = padded_k(a.k);
  p.qch = a.d / 64;
  p.vf = p.kp / 64;
  p.vr = p.kp % 64;
  p.scale = a.scale;
  p.scale_log2 = a.scale * kLog2e;
}

}  // namespace

bool tc_supported(int d, int k) { return (d == 64 || d == 128) && k >= 1 && k <= 256; }

void tc_debug_stall_next(int which) { g_stall_next.store(which); }

namespace {

// e4m3 [rows, cols] (one byte per element) with leading dimension ld bytes,
// box {128, 128}, 128-byte swizzle; rows past the end read as zero.
bool make_map_e4m3(CUtensorMap* m, const void* ptr, int rows, int cols, int ld) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t gdim[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {(cuuint64_t)ld};
  cuuint32_t box[2] = {128, 128};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), gdim, gstride, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// fp8: a.Q and a.K point to e4m3 copies (d = 128, ld in bytes) and qk_dequant
// to the device factor that turns their product into Q K^T.
cudaError_t launch_fwd_single(const TcArgs& a, float* O, int ldo, float* lse, cudaStream_t st,
                              const WaitCtl& ctl, bool fp8, const float* qk_dequant) {
  TcParams p;
  fill_common(a, p);
  p.O = O;
  p.ldo = ldo;
  p.lse = lse;
  p.ctl = ctl;
  p.qk_dequant = qk_dequant;
  TensorMaps tm;
  std::memset(&tm, 0, sizeof(tm));
  if (fp8) {
    if (a.d != 128 || !make_map_e4m3(&tm.q, a.Q, a.nQrows, a.d, a.ldq) ||
        !make_map_e4m3(&tm.k, a.K, a.nKrows, a.d, a.ldk))
      return cudaErrorInvalidValue;
  } else if (!make_map(&tm.q, a.Q, a.nQrows, a.d, a.ldq, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
             !make_map(&tm.k, a.K, a.nKrows, a.d, a.ldk, 64, CU_TENSOR_MAP_SWIZZLE_128B)) {
    return cudaErrorInvalidValue;
  }
  if (!make_map(&tm.v, a.V, a.nKrows, a.k, a.ldv, 64, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (p.vr && !make_map(&tm.vr, a.V, a.nKrows, a.k, a.ldv, p.vr, rem_sw_host(p.vr)))
    return cudaErrorInvalidValue;
  constexpr int NWG = kFwdSoftmaxGroups;
  const bool fixed = p.d == 128 && p.qch == 2 && p.vf == 3 && p.vr == 16;
  auto kern = fp8 ? (fixed ? tc_fwd_kernel<NWG, 2, 3, 16, true> : tc_fwd_kernel<NWG, 0, 0, 0, true>)
                 : (fixed ? tc_fwd_kernel<NWG, 2, 3, 16, false> : tc_fwd_kernel<NWG, 0, 0, 0, false>);
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  // two V stages when they fit next to Q and the two K stages, else one
  const int qtile = fp8 ? 128 * 128 : p.qch * kChunk;
  const int stage_bytes = 4 * NWG * 2048;  // epilogue staging, 2 KB per softmax warp
  p.vstages = 2;
  int smem = 1024 + qtile * 3 + p.vstages * vtile_bytes(p.vf, p.vr) + stage_bytes;
  if (smem + (int)fa.sharedSizeBytes > smem_optin()) {
    p.vstages = 1;
    smem = 1024 + qtile * 3 + vtile_bytes(p.vf, p.vr) + stage_bytes;
  }
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int work = a.ntiles_dev ? num_sms() : a.ntiles_host;
  const int grid = std::max(1, std::min(work, num_sms()));
  p.debug_stall = take_stall(1);
  prof_launch_begin(st);
  kern<<<grid, 96 + 128 * NWG, smem, st>>>(tm, p);
  prof_launch_end(st, SSC_PROF_FWD);
  count_launch();
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_tc_fwd(const TcArgs& a, float* O, int ldo, float* lse, cudaStream_t st,
                          const WaitCtl& ctl) {
  return launch_fwd_single(a, O, ldo, lse, st, ctl, false, nullptr);
}

cudaError_t launch_tc_fwd_e4m3(const TcArgs& a, const float* qk_dequant, float* O, int ldo,
                               float* lse, cudaStream_t st, const WaitCtl& ctl) {
  return launch_fwd_single(a, O, ldo, lse, st, ctl, true, qk_dequant);
}

cudaError_t launch_tc_bwd(const TcArgs& a, const __nv_bfloat16* dOb, int lddob, const float* lse,
                          const float* D, float* dQ, int lddq, float* dK, int lddk, float* dV,
                          int lddv, cudaStream_t st, const WaitCtl& ctl, float* dK_ord) {
  TcParams p;
  fill_common(a, p);
  p.lse_in = lse;
  p.Dvec = D;
  p.dQ = dQ;
  p.lddq = lddq;
  p.dK = dK;
  p.lddk = lddk;
  p.dV = dV;
  p.lddv = lddv;
  p.ctl = ctl;
  p.vec_atomics_dq = (lddq % 4 == 0) && (reinterpret_cast<uintptr_t>(dQ) % 16 == 0);
  TensorMaps tm;
  std::memset(&tm, 0, sizeof(tm));
  if (!make_map(&tm.q, a.Q, a.nQrows, a.d, a.ldq, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tm.k, a.K, a.nKrows, a.d, a.ldk, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tm.v, a.V, a.nKrows, a.k, a.ldv, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tm.g, dOb, a.nQrows, a.k, lddob, 64, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (p.vr && (!make_map(&tm.vr, a.V, a.nKrows, a.k, a.ldv, p.vr, rem_sw_host(p.vr)) ||
               !make_map(&tm.gr, dOb, a.nQrows, a.k, lddob, p.vr, rem_sw_host(p.vr))))
    return cudaErrorInvalidValue;
  const int vb = vtile_bytes(p.vf, p.vr);
  const int grid = num_sms();  // units are split evenly over every SM
  const bool fixed = p.d == 128 && p.qch == 2 && p.vf == 3 && p.vr == 16;
  p.dOb = dOb;
  p.lddob = lddob;
  {
    // dQ and dK: dO lives in TMEM, K is double-buffered, a warpgroup of its own
    // reduces the dK partials
    if (dK_ord) {
      // dK in the key order of K: contiguous rows, no column map
      p.col_map = nullptr;
      p.dK = dK_ord;
      p.lddk = a.d;
    }
    p.vec_atomics = (p.lddk % 4 == 0) && (reinterpret_cast<uintptr_t>(p.dK) % 16 == 0);
    // key rows contiguous in dK (no column map): partials go through TMA reductions
    p.dk_tma = !p.col_map && p.vec_atomics &&
               make_map_f32(&tm.dk, p.dK, a.nKrows, a.d, p.lddk, 32, 32, CU_TENSOR_MAP_SWIZZLE_128B);
    const int smem = 1024 + 3 * p.qch * kChunk + vb + 4 * kChunk;
    // dQ stored by the flush warpgroup when row tiles run over many key tiles
    // (dense: the softmax warpgroups then go straight on to the next row
    // tile); by the softmax warpgroups when runs are short (Geo: a dozen key
    // segments per row tile, where the flush warpgroup's extra stores would
    // hold up the dK partials)
    const bool dq_flush = a.ntiles_dev == nullptr;
    auto kern = fixed ? (dq_flush ? tc_bwd_dqk_kernel<kBwdComputeGroups, 2, 3, 16, false, true>
                                  : tc_bwd_dqk_kernel<kBwdComputeGroups, 2, 3, 16, false, false>)
                      : (dq_flush ? tc_bwd_dqk_kernel<kBwdComputeGroups, 0, 0, 0, false, true>
                                  : tc_bwd_dqk_kernel<kBwdComputeGroups, 0, 0, 0, false, false>);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    p.debug_stall = take_stall(2);
    prof_launch_begin(st);
    kern<<<grid, 128 * (2 + kBwdComputeGroups), smem, st>>>(tm, p);
    prof_launch_end(st, SSC_PROF_BWD_DQK);
    p.debug_stall = 0;
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (dV) {
    p.col_map = a.col_map;  // dV rows are scattered through the column map
    p.vec_atomics = (lddv % 4 == 0) && (reinterpret_cast<uintptr_t>(dV) % 16 == 0);
    const int smem = 1024 + 2 * p.qch * kChunk + vb + 2 * kChunk;
    auto kern = fixed ? tc_bwd_kernel<true, kBwdComputeGroups, 2, 3, 16>
                      : tc_bwd_kernel<true, kBwdComputeGroups, 0, 0, 0>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    prof_launch_begin(st);
    kern<<<grid, 64 + 128 * kBwdComputeGroups + 128, smem, st>>>(tm, p);
    prof_launch_end(st, SSC_PROF_BWD_DV);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_tc_dv_dense(const __nv_bfloat16* Q, int ldq, const __nv_bfloat16* K, int ldk,
                               const __nv_bfloat16* dOb, int lddob, const float* lse, int nN,
                               int nM, int d, int k, float scale, float* dV, int lddv,
                               cudaStream_t st, const WaitCtl& ctl, int max_ctas) {
  TcArgs a;
  std::memset(&a, 0, sizeof(a));
  a.Q = Q;
  a.K = K;
  a.ldq = ldq;
  a.ldk = ldk;
  a.nQrows = nN;
  a.nKrows = nM;
  a.d = d;
  a.k = k;
  a.scale = scale;
  TcParams p;
  fill_common(a, p);
  p.lse_in = lse;
  p.dV = dV;
  p.lddv = lddv;
  p.ctl = ctl;
  p.vec_atomics = (lddv % 4 == 0) && (reinterpret_cast<uintptr_t>(dV) % 16 == 0);
  TensorMaps tm;
  std::memset(&tm, 0, sizeof(tm));
  if (!make_map(&tm.q, Q, nN, d, ldq, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tm.k, K, nM, d, ldk, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tm.g, dOb, nN, k, lddob, 64, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (p.vr && !make_map(&tm.gr, dOb, nN, k, lddob, p.vr, rem_sw_host(p.vr))) return cudaErrorInvalidValue;
  const bool fixed = p.d == 128 && p.qch == 2 && p.vf == 3 && p.vr == 16;
  auto kern = fixed ? tc_dv_kernel<2, 2, 3, 16> : tc_dv_kernel<2, 0, 0, 0>;
  cudaFuncAttributes fa;
  cudaError_t e = cudaFuncGetAttributes(&fa, kern);
  if (e != cudaSuccess) return e;
  // K tile, two Q stages, two dO stages (at most 230,400 bytes for d = 128, k = 256)
  const int smem = 1024 + 3 * p.qch * kChunk + 2 * vtile_bytes(p.vf, p.vr);
  if (smem + (int)fa.sharedSizeBytes > smem_optin()) return cudaErrorInvalidValue;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  const int grid = std::max(1, max_ctas > 0 ? std::min(max_ctas, num_sms()) : num_sms());
  prof_launch_begin(st);
  kern<<<grid, 96 + 128 * 2, smem, st>>>(tm, p);
  prof_launch_end(st, SSC_PROF_BWD_DV);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_tc_bwd_deterministic(const __nv_bfloat16* Q, int ldq, const __nv_bfloat16* K,
                                        int ldk, const __nv_bfloat16* V, int ldv,
                                        const __nv_bfloat16* dOb, int lddob, const float* lse,
                                        const float* D, const RowTile* tiles, const KeySeg* segs,
                                        const int* prefix, int nN, int nM, int d, int k,
                                        float scale, float* dQ, int lddq, float* dK, int lddk,
                                        float* dV, int lddv, cudaStream_t st, const WaitCtl& ctl) {
  TcArgs a;
  std::memset(&a, 0, sizeof(a));
  a.Q = Q;
  a.K = K;
  a.V = V;
  a.ldq = ldq;
  a.ldk = ldk;
  a.ldv = ldv;
  a.nQrows = nN;
  a.nKrows = nM;
  a.d = d;
  a.k = k;
  a.scale = scale;
  a.tiles = tiles;
  a.segs = segs;
  a.ntiles_host = (nN + 127) / 128;
  a.tile_prefix = prefix;
  TcParams p;
  fill_common(a, p);
  p.lse_in = lse;
  p.Dvec = D;
  p.dQ = dQ;
  p.lddq = lddq;
  p.dK = dK;
  p.lddk = lddk;
  p.ctl = ctl;
  p.dOb = dOb;
  p.lddob = lddob;
  p.vec_atomics_dq = (lddq % 4 == 0) && (reinterpret_cast<uintptr_t>(dQ) % 16 == 0);
  p.vec_atomics = (lddk % 4 == 0) && (reinterpret_cast<uintptr_t>(dK) % 16 == 0);
  TensorMaps tm;
  std::memset(&tm, 0, sizeof(tm));
  if (!make_map(&tm.q, Q, nN, d, ldq, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tm.k, K, nM, d, ldk, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tm.v, V, nM, k, ldv, 64, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map(&tm.g, dOb, nN, k, lddob, 64, CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorInvalidValue;
  if (p.vr && (!make_map(&tm.vr, V, nM, k, ldv, p.vr, rem_sw_host(p.vr)) ||
               !make_map(&tm.gr, dOb, nN, k, lddob, p.vr, rem_sw_host(p.vr))))
    return cudaErrorInvalidValue;
  const int vb = vtile_bytes(p.vf, p.vr);
  const bool fixed = p.d == 128 && p.qch == 2 && p.vf == 3 && p.vr == 16;
  const int nrt = (nN + 127) / 128, nkt = (nM + 127) / 128;
  cudaError_t e;
  {
    // dQ: no more CTAs than row tiles, so a row tile's dQ gets at most two adds
    const int smem = 1024 + 3 * p.qch * kChunk + vb + 4 * kChunk;
    auto kern = fixed ? tc_bwd_dqk_kernel<kBwdComputeGroups, 2, 3, 16, true, true>
                      : tc_bwd_dqk_kernel<kBwdComputeGroups, 0, 0, 0, true, true>;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
        cudaSuccess)
      return e;
    prof_launch_begin(st);
    kern<<<std::max(1, std::min(num_sms(), nrt)), 128 * (2 + kBwdComputeGroups), smem, st>>>(tm, p);
    prof_launch_end(st, SSC_PROF_BWD_DQK);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  {
    // dK: key-stationary, no more CTAs than key tiles
    auto kern = fixed ? tc_dk_kernel<2, 2, 3, 16> : tc_dk_kernel<2, 0, 0, 0>;
    cudaFuncAttributes fa;
    if ((e = cudaFuncGetAttributes(&fa, kern)) != cudaSuccess) return e;
    // K and V tiles, two Q stages (one when V rows are long), one dO stage
    p.vstages = 2;
    int smem = 1024 + 3 * p.qch * kChunk + 2 * vb;
    if (smem + (int)fa.sharedSizeBytes > smem_optin()) {
      p.vstages = 1;
      smem = 1024 + 2 * p.qch * kChunk + 2 * vb;
    }
    if (smem + (int)fa.sharedSizeBytes > smem_optin()) return cudaErrorInvalidValue;
    if ((e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) !=
        cudaSuccess)
      return e;
    prof_launch_begin(st);
    kern<<<std::max(1, std::min(num_sms(), nkt)), 96 + 128 * 2, smem, st>>>(tm, p);
    prof_launch_end(st, SSC_PROF_BWD_DK);
    count_launch();
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  if (!dV) return cudaSuccess;
  return launch_tc_dv_dense(Q, ldq, K, ldk, dOb, lddob, lse, nN, nM, d, k, scale, dV, lddv, st, ctl,
                            nkt);
}

cudaError_t launch_wait_timeout_probe(cudaStream_t st, const WaitCtl& ctl) {
  wait_probe_kernel<<<1, 32, 0, st>>>(ctl);
  count_launch();
  return cudaGetLastError();
}

}  // namespace ssc
