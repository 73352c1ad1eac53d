// internal.h -- launch interfaces between the C ABI (ssc_api.cu) and the
// kernel files.  Host-side only types; no torch, no allocation.
#pragma once
#include <cstddef>
#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include <atomic>

#include "common.cuh"

namespace ssc {

// Number of kernels this library has launched (all devices, all streams).
inline std::atomic<unsigned long long> g_launches{0};
inline void count_launch(unsigned n = 1) { g_launches.fetch_add(n, std::memory_order_relaxed); }

// One unit of coupling work: query rows [row0, row0+nrows) (nrows <= 128) of
// the (possibly patch-major) Q buffer attend to the key segments
// segs[seg0 .. seg0+nseg).
struct RowTile {
  int row0, nrows, seg0, nseg;
};
// A run of consecutive key rows [key0, key0+nkeys), nkeys <= 128.
struct KeySeg {
  int key0, nkeys;
};

constexpr int kTileRows = 128;

// Round x up to a multiple of a.
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Sequential carve-out of a caller workspace (256-byte aligned pieces).
struct Carve {
  char* base;
  size_t used = 0;
  explicit Carve(void* b) : base(static_cast<char*>(b)) {}
  template <class T>
  T* take(size_t count) {
    used = round_up(used, 256);
    T* p = base ? reinterpret_cast<T*>(base + used) : nullptr;
    used += count * sizeof(T);
    return p;
  }
};

// The wait control every call passes to its kernels: the library's device
// status word on the current device and the current wait limit (ssc_api.cu).
WaitCtl library_wait_ctl();

// ------------------------------------------------------------ fps.cu
size_t fps_workspace_bytes(int n, int P);
// Test hook: 0 = pick the FPS cluster size from the device (16 where allowed,
// else 8); 8 or 16 forces that size for later calls.
void fps_force_cluster_size(int cl);
cudaError_t launch_fps_patches(const float* pts, int n, int P, int seed, int* centers, int* owner,
                               int* offsets, int* members, void* ws, cudaStream_t st,
                               const WaitCtl& ctl);
// Patch tables from owner [n] (every entry in [0, P)): offsets [P+1] and
// members [n] grouped by patch, ascending vertex id within a patch; counts and
// cursor are [P] scratch.
cudaError_t launch_patch_tables(const int* owner, int n, int P, int* offsets, int* members,
                                int* counts, int* cursor, cudaStream_t st);

// ------------------------------------------------------------ fps_mesh.cu
size_t fps_mesh_workspace_bytes(int n, int P);
// Geodesic FPS + nearest-centre patches on a mesh graph (CSR off [n+1], adj
// [nnz], fp64 edge lengths w [nnz]), then the patch tables.
cudaError_t launch_fps_mesh(const int* off, const int* adj, const double* w, int n, int nnz, int P,
                            int seed, int* centers, int* owner, int* offsets, int* members,
                            void* ws, cudaStream_t st, const WaitCtl& ctl);

// ------------------------------------------------------------ patch_topk.cu
size_t scores_topk_workspace_bytes(int PN, int PM, int d, int batch = 1);
// batch > 1: FN, FM hold batch shapes back to back (batch nN, batch nM rows)
// and the tables are the concatenated ones (batch PN and batch PM patches);
// scores [batch][PN][PM] pair by pair, topk [batch][PN][R] local to the pair.
cudaError_t launch_scores_topk(const void* FN, int ldn, int nN, const void* FM, int ldm, int nM,
                               int d, int dtype, const int* offN, const int* memN, int PN,
                               const int* offM, const int* memM, int PM, int R, int* topk,
                               double* scores, void* ws, unsigned* status, cudaStream_t st,
                               int batch = 1);

// ------------------------------------------------------------ prep.cu
// out[r, 0..cols) = in[map ? map[r] : r, 0..cols) converted to bf16 (in is
// bf16 or fp32 per in_f32), zero-filled up to out_ld.
// A map entry outside [0, src_rows) yields a zero row and sets the
// bad-index bit of the status word.
// ones_col >= 0: that padding column of every output row is set to one.
cudaError_t launch_gather_rows_bf16(const void* in, int in_ld, int in_f32, const int* map, int rows,
                                    int src_rows, int cols, __nv_bfloat16* out, int out_ld,
                                    unsigned* status, cudaStream_t st, int ones_col = -1);
// Three such gathers (no column of ones) in one launch: job j copies rows[j]
// rows of in[j] (through map[j]) into out[j].
cudaError_t launch_gather3_bf16(const __nv_bfloat16* const in[3], const int in_ld[3],
                                const int* const map[3], const int rows[3], const int src_rows[3],
                                const int cols[3], __nv_bfloat16* const out[3], const int out_ld[3],
                                unsigned* status, cudaStream_t st);
// fp32 variant (check mode).
cudaError_t launch_gather_rows_f32(const float* in, int in_ld, const int* map, int rows,
                                   int src_rows, int cols, float* out, int out_ld, unsigned* status,
                                   cudaStream_t st);
// Backward preparation of row r (source row src = map ? map[r] : r):
//   dOb[r, 0..k) = bf16(dO[src]) (zero-padded to ldb) when dOb != nullptr,
//   dOf[r, 0..k) = dO[src] when dOf != nullptr,
//   D[r] = <dO'[src], O[src]> with dO' the bf16-rounded value on the bf16 path,
//   lse_out[r] = lse[src].
cudaError_t launch_bwd_prep(const float* dO, int lddo, const float* O, int ldo, const float* lse,
                            const int* map, int rows, int src_rows, int k, __nv_bfloat16* dOb,
                            int ldb, float* dOf, int ldf, float* D, float* lse_out,
                            unsigned* status, cudaStream_t st);
// Dense schedule: ceil(nN/128) row tiles, all pointing at ceil(nM/128) segments.
int dense_num_tiles(int nN);
int dense_num_segs(int nM);
// prefix [ntiles + 1] receives the prefix sums of the tiles' segment counts.
cudaError_t launch_dense_schedule(int nN, int nM, RowTile* tiles, KeySeg* segs, int* prefix,
                                  cudaStream_t st);
// Block-diagonal schedule of `batch` dense pairs stored back to back
// (batch * ceil(nN/128) row tiles, batch * ceil(nM/128) segments, prefix of
// batch * ceil(nN/128) + 1 entries).
cudaError_t launch_batched_schedule(int batch, int nN, int nM, RowTile* tiles, KeySeg* segs,
                                    int* prefix, cudaStream_t st);
// Per-shape patch tables (off [batch][P+1], mem [batch][n]) as the tables of one
// problem (off_out [batch P + 1], mem_out [batch n]); bad entries are made
// out of range and set the bad-index bit.
cudaError_t launch_concat_tables(const int* off, const int* mem, int P, int n, int batch,
                                 int* off_out, int* mem_out, unsigned* status, cudaStream_t st);
// Per-pair top-R lists [batch][PN][R] shifted to the concatenated source patches.
cudaError_t launch_concat_topk(const int* topk, int PN, int R, int PM, int batch, int* out,
                               unsigned* status, cudaStream_t st);
// Geo schedule: per target patch ceil(|p|/128) row tiles that share the list of
// 128-row pieces of the patch's selected source patches.  Writes the counts to
// counts[0] (tiles) and counts[1] (segments).  Upper bounds for sizing:
int geo_max_tiles(int nN, int PN);
int geo_max_segs(int nM, int PM, int PN, int R);
// topk entries outside [0, PM) are skipped and set the bad-index bit.
// Offsets outside [0, n] or decreasing are clamped and set the bad-index bit.
// tag: written with tag_value (a fingerprint of the call) when not null.
cudaError_t launch_geo_schedule(const int* offN, int PN, int nN, const int* offM, int PM, int nM,
                                const int* topk, int R, RowTile* tiles, KeySeg* segs, int* counts,
                                int* prefix, int* scratch, unsigned* status, cudaStream_t st,
                                unsigned long long* tag = nullptr,
                                unsigned long long tag_value = 0);
// Sets the bad-index bit of *status when *tag differs from expect.
cudaError_t launch_check_tag(const unsigned long long* tag, unsigned long long expect,
                             unsigned* status, cudaStream_t st);
size_t geo_schedule_scratch_ints(int PN);
// Transposed selection (for the key-stationary fp32 backward): for every
// source patch q the ascending list of target patches p with q in topk[p].
size_t invert_topk_scratch_ints(int PM);
cudaError_t launch_invert_topk(const int* topk, int PN, int R, int PM, int* inv_off, int* inv_p,
                               int* scratch, cudaStream_t st);

// ------------------------------------------------------------ coupling_simt.cu (fp32)
struct SimtArgs {
  const float* Q;
  const float* K;
  const float* V;
  int ldq, ldk, ldv;
  int nN, nM, d, k;
  float scale;
  const RowTile* tiles;
  const KeySeg* segs;
  const int* ntiles_dev;  // nullable: number of tiles read on the device
  int ntiles_host;        // used when ntiles_dev == nullptr
  const int* row_map;     // output row r -> vertex (nullable = identity)
  const int* col_map;     // key row j -> vertex (nullable = identity)
};
cudaError_t launch_simt_fwd(const SimtArgs& a, float* O, int ldo, float* lse, cudaStream_t st);
// dQ: query-stationary.  Needs D and lse in the (permuted) row order.
cudaError_t launch_simt_bwd_dq(const SimtArgs& a, const float* dO, int lddo, const float* lse,
                               const float* D, float* dQ, int lddq, cudaStream_t st);
// dK/dV: key-stationary.  Dense when inv_off == nullptr (every row attends);
// otherwise key row j of source patch q is seen by the rows of the target
// patches inv_p[inv_off[q] .. inv_off[q+1]).
struct SimtKeyArgs {
  const int* offM;     // source patch offsets (patch-major key rows), nullable for dense
  int PM;
  const int* offN;     // target patch offsets (patch-major query rows)
  const int* inv_off;
  const int* inv_p;
  unsigned* status;    // bad-index reports
};
cudaError_t launch_simt_bwd_dkdv(const SimtArgs& a, const SimtKeyArgs& g, const float* dO,
                                 int lddo, const float* lse, const float* D, float* dK, int lddk,
                                 float* dV, int lddv, cudaStream_t st);

// ------------------------------------------------------------ coupling_tc.cu (bf16, tcgen05)
struct TcArgs {
  const __nv_bfloat16* Q;  // [nQrows, ldq]
  const __nv_bfloat16* K;  // [nKrows, ldk]
  const __nv_bfloat16* V;  // [nKrows, ldv]
  int ldq, ldk, ldv;
  int nQrows, nKrows;
  int d, k;
  float scale;
  const RowTile* tiles;
  const KeySeg* segs;
  const int* ntiles_dev;  // nullable
  int ntiles_host;
  const int* tile_prefix;  // [ntiles + 1] prefix sums of the tiles' segment counts
  const int* row_map;
  const int* col_map;
};
// Launch timing record (profile.cu): bracket a kernel launch on stream st.
void prof_launch_begin(cudaStream_t st);
void prof_launch_end(cudaStream_t st, int kernel);

bool tc_supported(int d, int k);
// Abort-path test hook: the next launch of the forward (1) or dQ/dK backward
// (2) tensor-core kernel stalls its MMA issuer on a barrier nothing arrives at
// until the bounded wait gives up (0 disarms).
void tc_debug_stall_next(int which);
cudaError_t launch_tc_fwd(const TcArgs& a, float* O, int ldo, float* lse, cudaStream_t st,
                          const WaitCtl& ctl);
// The same forward with S = Q K^T on e4m3 tensor cores: a.Q and a.K point to
// e4m3 copies with d = 128 (ldq, ldk in bytes), qk_dequant to the device
// factor (scale of Q times scale of K) that restores Q K^T from their product.
cudaError_t launch_tc_fwd_e4m3(const TcArgs& a, const float* qk_dequant, float* O, int ldo,
                               float* lse, cudaStream_t st, const WaitCtl& ctl);
// e4m3 copies of bf16 Q [nN, ldq] and K [nM, ldk] (d columns, rows of d bytes):
// each tensor divided by its own scale amax / 448 (amax its largest magnitude),
// rounded to nearest with saturation; *qk_dequant = scale_Q * scale_K.  amax2
// is [2] scratch.
cudaError_t launch_quantize_e4m3(const __nv_bfloat16* Q, int ldq, int nN, const __nv_bfloat16* K,
                                 int ldk, int nM, int d, uint8_t* Q8, uint8_t* K8,
                                 unsigned* amax2, float* qk_dequant, cudaStream_t st);
// dQ written (scaled), dK accumulated with atomics (caller zeroes it).
// dOb: bf16 [nQrows, lddob] (k padded with zeros), lse/D in row order.
// dK_ord (optional): dK is reduced into this [a.nKrows, d] buffer in the key
// order of a.K (no column map, contiguous rows) instead of into dK; the caller
// scatters it.  The dV pass still uses a.col_map.
cudaError_t launch_tc_bwd(const TcArgs& a, const __nv_bfloat16* dOb, int lddob, const float* lse,
                          const float* D, float* dQ, int lddq, float* dK, int lddk, float* dV,
                          int lddv, cudaStream_t st, const WaitCtl& ctl, float* dK_ord = nullptr);
// Dense dV = P^T dO on tensor cores, key-stationary (dV accumulated per key tile
// on chip; no partial-dV reductions).  dOb: bf16 dO rows of kp columns, zero
// padded; lse in row order; dV zeroed by the caller.
// max_ctas > 0 caps the grid (no more CTAs than key tiles gives every key
// tile at most two contributions, which makes the result run-to-run exact).
cudaError_t launch_tc_dv_dense(const __nv_bfloat16* Q, int ldq, const __nv_bfloat16* K, int ldk,
                               const __nv_bfloat16* dOb, int lddob, const float* lse, int nN,
                               int nM, int d, int k, float scale, float* dV, int lddv,
                               cudaStream_t st, const WaitCtl& ctl, int max_ctas = 0);
// The dense backward with results identical bit for bit from run to run:
// dQ query-stationary with each row tile shared by at most two CTAs, dK
// key-stationary with each key tile shared by at most two CTAs (two fp32 adds
// into a zeroed output commute), dV likewise.  dQ, dK (and dV) are zeroed by
// the caller; dOb, lse, D and the dense tile schedule as for launch_tc_bwd.
cudaError_t launch_tc_bwd_deterministic(const __nv_bfloat16* Q, int ldq, const __nv_bfloat16* K,
                                        int ldk, const __nv_bfloat16* V, int ldv,
                                        const __nv_bfloat16* dOb, int lddob, const float* lse,
                                        const float* D, const RowTile* tiles, const KeySeg* segs,
                                        const int* prefix, int nN, int nM, int d, int k,
                                        float scale, float* dQ, int lddq, float* dK, int lddk,
                                        float* dV, int lddv, cudaStream_t st, const WaitCtl& ctl);
// out[map[r]] = in[r] for r < rows (map entries outside [0, dst_rows) are dropped
// and set the bad-index bit).
cudaError_t launch_scatter_rows_f32(const float* in, int in_ld, const int* map, int rows,
                                    int dst_rows, int cols, float* out, int out_ld,
                                    unsigned* status, cudaStream_t st);

// ------------------------------------------------------------ coupling_tc2.cu (bf16, CTA pairs)
// Dense forward on clusters of two CTAs issuing 2-SM MMAs (query tiles of 256).
bool tc_pair_supported(int d, int k);
// Partial-result workspace (floats) of the dense pair forward: query tiles whose
// key tiles are split between CTA pairs are merged from it.  sum_col >= 0: V
// holds ones in that column (V is read with k + 1 columns), so the softmax row
// sum comes out of the P V product; -1: the softmax threads add it up.
size_t tc_pair_part_floats(int k);
cudaError_t launch_tc_fwd_pair(const __nv_bfloat16* Q, int ldq, const __nv_bfloat16* K, int ldk,
                               const __nv_bfloat16* V, int ldv, int nN, int nM, int d, int k,
                               float scale, float* O, int ldo, float* lse, float* part,
                               int sum_col, cudaStream_t st, const WaitCtl& ctl);

// ------------------------------------------------------------ linear.cu (ELU linear attention)
// Columns of the bf16 operands that carry [V | 1] and Y: k + 1 rounded to 16.
int lin_kv(int k);
// Upper bound on the partial sums the reduction over n rows leaves (its
// workspace holds that many [128 x 256] fp32 blocks, one per CTA cluster).
int lin_reduce_grid(int n);
// The weight matrix a reduction produces: W [128 x 256] and W^T [256 x 128]
// in bf16 (zero outside d x nb), and the fp32 W when W32 != nullptr.
struct LinWeights {
  __nv_bfloat16* W;
  __nv_bfloat16* WT;
  float* W32;
};
// W = phi(X)^T B over n rows: X [n, ldx] with d columns, B [n, ldb] with bwidth
// columns (read as zero beyond), nb = N (multiple of 16, <= 256); ones_col >= 0
// sets that column of B to one on every row.
cudaError_t launch_lin_reduce(const __nv_bfloat16* X, int ldx, const __nv_bfloat16* B, int ldb,
                              int n, int d, int bwidth, int nb, int ones_col, float* part,
                              LinWeights w, cudaStream_t st, const WaitCtl& ctl);
// Row-tile products against a resident weight matrix (mode 0: forward
// O = phi(A) W^T / den; 1: dV = phi(A) W^T; 2: out = (A W) * phi'(X)).
cudaError_t launch_lin_rows(int mode, const __nv_bfloat16* A, int lda, int awidth, int n,
                            const __nv_bfloat16* Wmat, int d, int k, int nmma, int ksteps,
                            int ones_col, const __nv_bfloat16* X, int ldx, float* out, int ldout,
                            float* den, cudaStream_t st, const WaitCtl& ctl);
// Y rows [g / den, -<g, O> / den, 0 ...] with g = bf16(dO), ldy columns.
cudaError_t launch_lin_prep(const float* dO, int lddo, const float* O, int ldo, const float* den,
                            int n, int k, __nv_bfloat16* Y, int ldy, cudaStream_t st);

// Test hook: a kernel that waits on a barrier nothing arrives on.
cudaError_t launch_wait_timeout_probe(cudaStream_t st, const WaitCtl& ctl);

}  // namespace ssc
