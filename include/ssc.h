/*
 * ssc.h -- C ABI of the spatial-spectral coupling library (libssc.so), sm_100a.
 *
 * The library evaluates the spatial-spectral coupling of deep functional maps,
 *     O = Pi_NM Phi_M = softmax(s * F_N F_M^T) Phi_M,
 * as scaled dot-product attention with Q = F_N (target descriptors),
 * K = F_M (source descriptors) and V = Phi_M (source Laplace-Beltrami
 * eigenbasis) without ever storing the n_N x n_M map Pi_NM
 * ("Spatial-Spectral Coupling as Attention", project page, sections "The
 * bottleneck" and "Spatial-spectral coupling is attention").  It also provides
 * Geo-FlashAttention (same page, section "Geo-FlashAttention"): both shapes are
 * partitioned into geodesic patches, patch-mean descriptors are scored, each
 * target patch keeps its top R source patches, and the exact softmax runs over
 * the vertices of those patches only.
 *
 * Conventions shared by every call
 *  - Every pointer argument is a DEVICE pointer owned by the caller, unless a
 *    comment says otherwise.  The library never allocates device memory: each
 *    call that needs scratch space has a *_workspace_size query, and the caller
 *    passes a device buffer `ws` of at least that many bytes (256-byte aligned).
 *  - Work is enqueued on `stream` (a cudaStream_t, passed as void*) and runs
 *    asynchronously; no call synchronises the host.  Device-side failures
 *    (a bounded wait that ran out) are recorded in a library status word that
 *    ssc_device_status() reads back.
 *  - Some launches that do not depend on the work just before them (the Geo
 *    patch-major gather, the zeroing of the backward's accumulators) run on a
 *    side stream of the library: one per host thread and device, created on
 *    that thread's first call outside stream capture.  It waits for `stream`
 *    before its launches and `stream` waits for it afterwards (events), so
 *    the call's work is ordered on `stream` as a whole; a call inside stream
 *    capture brings the side stream into the capture and joins it back.  When
 *    the side stream cannot be made, everything runs on `stream`.
 *  - Matrices are row-major with an explicit leading dimension (`ld*`, in
 *    elements, >= the row length).  bf16 Q and K need 16-byte aligned base
 *    pointers and leading dimensions that are multiples of 8 elements (the
 *    tensor-memory-accelerator reads them in place); bf16 V may have any
 *    stride (it is re-packed into the workspace when its rows are not 16-byte
 *    aligned); fp32 inputs need 4-byte alignment; fp32 outputs need 16-byte
 *    aligned base pointers.
 *  - Index tables that are inconsistent (an index out of range, offsets that
 *    decrease or exceed n, repeated top-R entries) never cause an out-of-range
 *    access: the offending entries are dropped, results are unspecified and
 *    ssc_device_status() reports SSC_ERR_INVALID_ARG.
 *  - `dtype` selects the input type of Q, K, V: SSC_BF16 (bf16 inputs, tensor
 *    cores, fp32 accumulation) or SSC_F32 (fp32 inputs on CUDA cores, a check
 *    mode held to a 1e-4 tolerance).  Outputs are always fp32.
 *  - Sizes: n >= 1, d in {64, 128}, 1 <= k <= 256, 1 <= R <= P <= n,
 *    P <= 65535.  Violations return SSC_ERR_INVALID_ARG or SSC_ERR_UNSUPPORTED
 *    before any work is enqueued; outputs are then untouched.
 *  - Vertex indices and patch tables are int32.
 */
#ifndef SSC_H_
#define SSC_H_

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef void* ssc_stream_t; /* a cudaStream_t; NULL = the legacy default stream */

enum ssc_status_code {
  SSC_OK = 0,
  SSC_ERR_INVALID_ARG = 1,  /* bad size, null pointer, bad index table */
  SSC_ERR_UNSUPPORTED = 2,  /* d or k outside what the kernels implement */
  SSC_ERR_ALIGNMENT = 3,    /* base pointer or leading dimension misaligned */
  SSC_ERR_WORKSPACE = 4,    /* workspace missing or smaller than the query */
  SSC_ERR_CUDA = 5,         /* a CUDA runtime/driver call failed */
  SSC_ERR_TIMEOUT = 6       /* a device-side wait hit its limit (see ssc_device_status) */
};

enum ssc_dtype { SSC_BF16 = 0, SSC_F32 = 1 };

/* Human-readable text for a status code (static storage, never NULL). */
const char* ssc_status_string(int status);

/* Library version, (major << 16) | minor. */
int ssc_version(void);

/* Running count of the CUDA kernels this library has enqueued (host-side
 * counter, all devices and streams); lets a caller attribute launches. */
unsigned long long ssc_kernel_launches(void);

/* Synchronises `stream`, then stores into *status the device status word that
 * kernels set when a bounded wait ran out (SSC_OK or SSC_ERR_TIMEOUT) and, if
 * `clear` is non-zero, resets it.  Returns SSC_ERR_CUDA if the sync failed. */
int ssc_device_status(ssc_stream_t stream, int clear, int* status);

/* Sets the time limit of every device-side wait, in nanoseconds (default
 * 2e9).  Intended for tests; 0 restores the default. */
int ssc_set_wait_limit_ns(unsigned long long ns);

/* Test hook of the bounded-wait machinery: launches one block that waits on a
 * barrier nothing will ever arrive on.  The wait gives up after `limit_ns`,
 * records SSC_ERR_TIMEOUT in the device status word and the kernel returns.
 * No GPU fault, trap or hang is involved. */
int ssc_debug_wait_timeout(unsigned long long limit_ns, ssc_stream_t stream);

/* Test hook of the abort path of the tensor-core coupling kernels.  which = 1:
 * the next launch of the forward kernel (Geo forward, and the dense forward
 * on fp8 tensor cores); which = 2: the next launch of the dQ/dK backward
 * kernel (dense and Geo).  In that launch the MMA issuer, after its first S
 * MMAs, waits on a barrier nothing arrives at.  The bounded wait gives up
 * after the wait limit (ssc_set_wait_limit_ns), records SSC_ERR_TIMEOUT in the
 * device status word and raises the kernel's abort flag: every role leaves its
 * loop, the producers wait for their copies in flight, the issued MMAs drain
 * and TMEM is freed before the CTAs exit, so the context stays usable.  The
 * outputs of that launch are undefined.  No GPU fault, trap or hang is
 * involved.  which = 0 disarms; other values return SSC_ERR_INVALID_ARG. */
int ssc_debug_stall_next_launch(int which);

/* ------------------------------------------------------------------------ */
/* Geodesic patches.                                                        */
/* Source: digest "Interpretation" (geodesic farthest-point sampling) and    */
/* project page "Geo-FlashAttention" (partition each surface into geodesic   */
/* patches).  On the unit sphere the geodesic distance is the great-circle   */
/* distance, a decreasing function of the dot product, so every ranking is   */
/* made on the fp64 dot ((x0*y0 + x1*y1) + x2*y2) of the fp32 coordinates.   */
/* ------------------------------------------------------------------------ */

/* Scratch bytes ssc_fps_patches needs for n points and P patches. */
size_t ssc_fps_patches_workspace_size(int n, int P);

/* Farthest-point sampling plus nearest-centre (Voronoi) assignment.
 *   pts      [n,3] fp32 unit vectors, row-major, contiguous
 *   seed_vertex  first centre (the synthetic workloads use vertex 0)
 * Outputs (all int32, caller-allocated):
 *   centers  [P]   centre t = the not-yet-chosen vertex whose largest dot to
 *                  centres 0..t-1 is smallest; ties -> lowest vertex index
 *   owner    [n]   patch of each vertex = index of its nearest centre (largest
 *                  dot), ties -> lowest patch index; a centre owns itself
 *   offsets  [P+1] patch p holds members[offsets[p] .. offsets[p+1])
 *   members  [n]   vertices grouped by patch, ascending vertex id in a patch
 * Results are bit-identical to the fp64 definition.  Requires 1 <= P <= n,
 * P <= 65535, n <= 2^24. */
int ssc_fps_patches(const float* pts, int n, int P, int seed_vertex,
                    int* centers, int* owner, int* offsets, int* members,
                    void* ws, size_t ws_bytes, ssc_stream_t stream);

/* Geodesic patches on a triangle mesh (the digest's "Interpretation":
 * geodesic farthest-point sampling; project page "Geo-FlashAttention":
 * geodesic patches), with the geodesic distance read as the shortest path
 * along mesh edges: edge lengths added in fp64 from the source outward,
 * minimised over paths.
 *   adj_off  [n+1] int32, adj [nnz] int32: the edge graph in CSR form (each
 *            undirected edge listed from both ends; adj_off[0] = 0,
 *            adj_off[n] = nnz)
 *   edge_len [nnz] fp64: length of each listed edge (>= 0)
 * Outputs as ssc_fps_patches: centre t = the vertex farthest from its nearest
 * centre among 0..t-1 (ties -> lowest vertex index; a vertex no centre
 * reaches is at +inf, so every connected part receives a centre before any
 * part receives a second); owner = nearest centre (ties -> lowest patch
 * index); offsets/members the patch tables.  When P is smaller than the
 * number of connected parts, vertices no centre reaches keep owner -1 and
 * are listed in members after the last patch (from offsets[P] to n, in
 * ascending order), so members is always a permutation of the vertices.
 * Distances are bit-identical to
 * Dijkstra's in fp64, so every index is exact.  Requires 1 <= P <= n,
 * P <= 65535.  Edges with a negative or NaN length or an endpoint out of
 * range, and offsets out of [0, nnz] or decreasing, are skipped and reported
 * as SSC_ERR_INVALID_ARG in the device status word. */
size_t ssc_fps_patches_mesh_workspace_size(int n, int P);

int ssc_fps_patches_mesh(const int* adj_off, const int* adj, const double* edge_len, int n,
                         int nnz, int P, int seed_vertex, int* centers, int* owner,
                         int* offsets, int* members, void* ws, size_t ws_bytes,
                         ssc_stream_t stream);

/* The same patches without a workspace argument, for callers that cannot
 * allocate device memory at all (for instance code embedded in a host program
 * that owns every device allocation and hands over only input and output
 * buffers).  The pages have no counterpart of this call; it exists for such
 * callers only.  Results equal ssc_fps_patches bit for bit.
 *   Limits: n <= SSC_FPS_NOALLOC_MAX_N, P <= SSC_FPS_NOALLOC_MAX_P; larger
 *   sizes return SSC_ERR_UNSUPPORTED before any work is enqueued.
 *   Scratch: a fixed 3 MiB array in the library's own device memory, held by
 *   every GPU that loads the library until the process exits.  The first
 *   call on a device looks up the array's device address (with that device
 *   current); make that first call before capturing any stream into a graph.
 *   Every call shares the array: calls that overlap on the GPU (different
 *   streams or host threads) race and must be serialised by the caller; each
 *   call clears the counters it needs zeroed.  No device allocation is made.
 *   The looked-up address is kept for the rest of the process, so a program
 *   that resets a device's primary context (cudaDeviceReset) must not call
 *   this entry point on that device afterwards. */
#define SSC_FPS_NOALLOC_MAX_N 262144
#define SSC_FPS_NOALLOC_MAX_P 65535
int ssc_fps_patches_noalloc(const float* pts, int n, int P, int seed_vertex,
                            int* centers, int* owner, int* offsets, int* members,
                            ssc_stream_t stream);

/* Test hook of the FPS launch (the pages have no counterpart): 8 or 16 forces
 * the thread-block cluster size of later ssc_fps_patches* calls (16 still
 * falls back to 8 where the device cannot hold such a cluster); 0 restores
 * the automatic choice.  With 8 CTAs, point counts above 8 x 16384 take the
 * path that keeps the per-point state in the workspace instead of on chip.
 * Other values are SSC_ERR_INVALID_ARG.  Results do not depend on it. */
int ssc_debug_fps_cluster_size(int cl);

/* Launch timing (a measurement hook; the pages have no counterpart).
 * ssc_profile_enable(1) clears the record and starts recording: every later
 * launch of a tracked coupling kernel is bracketed by two CUDA events on the
 * stream it is launched on.  ssc_profile_enable(0) stops recording (the
 * record is kept), ssc_profile_enable(2) resumes it without clearing; other
 * values are SSC_ERR_INVALID_ARG.  ssc_profile_read waits for the recorded launches of one
 * kernel to finish and returns their summed device time in milliseconds and
 * their count.  Host-side event objects only; no device memory is allocated.
 * Errors: SSC_ERR_INVALID_ARG for a null pointer or an unknown kernel id,
 * SSC_ERR_CUDA if an event cannot be read. */
#define SSC_PROF_DENSE_FWD 0 /* dense forward on CTA pairs (tc_fwd_pair_kernel) */
#define SSC_PROF_FWD 1       /* single-CTA forward (Geo, and dense when pairs are not used) */
#define SSC_PROF_BWD_DQK 2   /* backward dQ/dK kernel (tc_bwd_dqk_kernel) */
#define SSC_PROF_BWD_DV 3    /* optional dV pass (tc_dv_kernel dense, tc_bwd_kernel Geo) */
#define SSC_PROF_FPS 4       /* FPS rounds (fps_cluster_kernel / fps_cluster_mem_kernel) */
#define SSC_PROF_POOL 5      /* patch-mean pooling, one launch per shape */
#define SSC_PROF_SCORES 6    /* patch score matrix */
#define SSC_PROF_TOPK 7      /* top-R selection */
#define SSC_PROF_GATHER 8    /* bf16 row gathers (patch-major Q, K, V; V re-pack) */
#define SSC_PROF_LIN_REDUCE 9 /* linear coupling: phi(X)^T B reductions */
#define SSC_PROF_LIN_ROWS 10  /* linear coupling: row-tile products (O, dQ, dK, dV) */
#define SSC_PROF_BWD_DK 11    /* deterministic backward: key-stationary dK (tc_dk_kernel) */
#define SSC_PROF_KERNELS 12
int ssc_profile_enable(int on);
int ssc_profile_read(int kernel, double* total_ms, int* launches);

/* Scratch bytes ssc_patch_scores_topk needs. */
size_t ssc_patch_scores_topk_workspace_size(int PN, int PM, int d);

/* Pool, score and select (project page "Geo-FlashAttention": pool source
 * keys, score source patches using descriptors, keep the top R per target).
 *   FN [nN, ldn], FM [nM, ldm]   descriptors (bf16 or fp32 per dtype)
 *   offN/memN, offM/memM          patch tables from ssc_fps_patches
 * Computes in fp64, in a fixed order (bit-exact):
 *   mu_N(p) = mean over members of p of F_N (ascending vertex order, one divide)
 *   score(p,q) = sum_{c=0..d-1} mu_N(p)_c * mu_M(q)_c  (in order, no FMA)
 * Outputs: topk [PN,R] int32, per row the R best q by (score desc, q asc);
 * scores [PN,PM] fp64 (nullable; when NULL the matrix lives in `ws`). */
int ssc_patch_scores_topk(const void* FN, int ldn, int nN, const void* FM, int ldm, int nM,
                          int d, int dtype,
                          const int* offN, const int* memN, int PN,
                          const int* offM, const int* memM, int PM,
                          int R, int* topk, double* scores,
                          void* ws, size_t ws_bytes, ssc_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Dense coupling (project page, "Spatial-spectral coupling is attention").  */
/*   S = scale * Q K^T, Pi = row softmax of S, O = Pi V,                     */
/*   lse_i = ln sum_j exp(S_ij) (natural log).                               */
/* Q [nN, ldq], K [nM, ldk], V [nM, ldv] in `dtype`; O [nN, ldo] fp32 and    */
/* lse [nN] fp32.                                                            */
/* ------------------------------------------------------------------------ */

size_t ssc_dense_coupling_workspace_size(int nN, int nM, int d, int k, int dtype);

int ssc_dense_coupling_fwd(const void* Q, int ldq, const void* K, int ldk,
                           const void* V, int ldv, int nN, int nM, int d, int k,
                           float scale, int dtype, float* O, int ldo, float* lse,
                           void* ws, size_t ws_bytes, ssc_stream_t stream);

/* Backward of a loss L with dL/dO = dO (fp32 [nN, lddo]), given the forward's
 * O and lse.  Textbook softmax-matmul gradient with recompute from lse:
 *   D_i = <dO_i, O_i>, P_ij = exp(S_ij - lse_i), dP_ij = <dO_i, V_j>,
 *   dS_ij = P_ij (dP_ij - D_i), dQ = scale dS K, dK = scale dS^T Q, dV = P^T dO.
 * On the bf16 path dO is rounded to bf16 once and that value is used
 * throughout (D included).  dV may be NULL (the eigenbasis is not learned);
 * dQ [nN, lddq], dK [nM, lddk], dV [nM, lddv] fp32 are overwritten. */
int ssc_dense_coupling_bwd(const void* Q, int ldq, const void* K, int ldk,
                           const void* V, int ldv, int nN, int nM, int d, int k,
                           float scale, int dtype, const float* O, int ldo,
                           const float* lse, const float* dO, int lddo,
                           float* dQ, int lddq, float* dK, int lddk,
                           float* dV, int lddv,
                           void* ws, size_t ws_bytes, ssc_stream_t stream);

/* The dense forward with S = Q K^T on fp8 tensor cores (e4m3 inputs, fp32
 * accumulation; the pages have no counterpart: a lower-precision variant
 * whose error against the exact coupling is measured, not a replacement for
 * the bf16 path).  Q and K (bf16, d = 128) are each divided by their own
 * scale amax / 448 (amax = largest magnitude of the tensor) and rounded to
 * e4m3 with saturation; the product is multiplied back by both scales before
 * the softmax.  P V stays bf16 x bf16.  Same arguments and outputs as
 * ssc_dense_coupling_fwd (bf16 only, d must be 128, else
 * SSC_ERR_UNSUPPORTED); its own workspace query. */
size_t ssc_dense_coupling_fwd_e4m3_workspace_size(int nN, int nM, int d, int k);

int ssc_dense_coupling_fwd_e4m3(const void* Q, int ldq, const void* K, int ldk,
                                const void* V, int ldv, int nN, int nM, int d, int k,
                                float scale, float* O, int ldo, float* lse,
                                void* ws, size_t ws_bytes, ssc_stream_t stream);

/* ssc_dense_coupling_bwd with results that are the same bit for bit on
 * every run (same arguments, same workspace size).  The default backward adds
 * the dK partials of every query tile in whatever order the reductions
 * arrive, so its last bits vary from run to run.  This one runs three passes:
 * dQ query-stationary (the dK work dropped), dK key-stationary (a CTA keeps a
 * key tile and streams the query tiles past it, recomputing S^T, dP^T and
 * dS^T), dV key-stationary; each pass uses no more CTAs than there are tiles
 * of its output, so an output tile receives at most two fp32 additions into
 * the zeroed result, and two additions commute.  Costs about 1.6x the
 * flops of the default backward (S and dP are computed twice).  Results
 * equal the default backward's within the bf16 tolerances.  The fp32 check
 * mode is already deterministic and is run as is. */
int ssc_dense_coupling_bwd_deterministic(const void* Q, int ldq, const void* K, int ldk,
                                         const void* V, int ldv, int nN, int nM, int d, int k,
                                         float scale, int dtype, const float* O, int ldo,
                                         const float* lse, const float* dO, int lddo,
                                         float* dQ, int lddq, float* dK, int lddk,
                                         float* dV, int lddv,
                                         void* ws, size_t ws_bytes, ssc_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Geo-FlashAttention (project page, "Geo-FlashAttention"; digest,           */
/* "Interpretation": each target patch computes the exact softmax over only  */
/* its highest-scoring source patches).  Row i of target patch p attends to  */
/* U(p) = union of the members of source patches topk[p, 0..R-1]; the        */
/* softmax is normalised over U(p).  Patch tables as from ssc_fps_patches,   */
/* topk as from ssc_patch_scores_topk (entries must be distinct).  Outputs   */
/* are in vertex order, like the dense calls.                                */
/* ------------------------------------------------------------------------ */

size_t ssc_geo_coupling_workspace_size(int nN, int nM, int d, int k, int PN, int PM,
                                       int R, int dtype);

int ssc_geo_coupling_fwd(const void* Q, int ldq, const void* K, int ldk,
                         const void* V, int ldv, int nN, int nM, int d, int k,
                         float scale, int dtype,
                         const int* offN, const int* memN, int PN,
                         const int* offM, const int* memM, int PM,
                         const int* topk, int R,
                         float* O, int ldo, float* lse,
                         void* ws, size_t ws_bytes, ssc_stream_t stream);

int ssc_geo_coupling_bwd(const void* Q, int ldq, const void* K, int ldk,
                         const void* V, int ldv, int nN, int nM, int d, int k,
                         float scale, int dtype,
                         const int* offN, const int* memN, int PN,
                         const int* offM, const int* memM, int PM,
                         const int* topk, int R,
                         const float* O, int ldo, const float* lse,
                         const float* dO, int lddo,
                         float* dQ, int lddq, float* dK, int lddk,
                         float* dV, int lddv,
                         void* ws, size_t ws_bytes, ssc_stream_t stream);

/* ssc_geo_coupling_bwd without rebuilding what ssc_geo_coupling_fwd left in  */
/* the workspace: the patch-major copies of Q, K and V and the tile schedule  */
/* (the saved state a training step keeps from its forward; the pages have   */
/* no counterpart).  Same arguments and results as ssc_geo_coupling_bwd.     */
/* Contract: ws is the workspace of a completed or earlier-enqueued           */
/* ssc_geo_coupling_fwd call on the same stream with the same Q, K, V, sizes, */
/* dtype and patch tables, and nothing wrote to ws or to those inputs in      */
/* between.  The forward leaves a fingerprint of its call (sizes, dtype and   */
/* the addresses of Q, K, V and the tables) in the workspace and this call    */
/* compares it on the device: a workspace of another call sets the bad-      */
/* argument bit of the device status word (ssc_device_status then reports    */
/* SSC_ERR_INVALID_ARG) and the gradients are undefined.  Changed contents   */
/* at the same addresses are not detected.                                   */
/* The backward itself overwrites only the workspace's backward buffers, so   */
/* it can be called again on the same forward state.                         */
int ssc_geo_coupling_bwd_reuse(const void* Q, int ldq, const void* K, int ldk,
                               const void* V, int ldv, int nN, int nM, int d, int k,
                               float scale, int dtype,
                               const int* offN, const int* memN, int PN,
                               const int* offM, const int* memM, int PM,
                               const int* topk, int R,
                               const float* O, int ldo, const float* lse,
                               const float* dO, int lddo,
                               float* dQ, int lddq, float* dK, int lddk,
                               float* dV, int lddv,
                               void* ws, size_t ws_bytes, ssc_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Batches of shape pairs (a training step of a functional-map pipeline       */
/* evaluates the coupling for every pair of its batch; project page, Table 1, */
/* "One ULRSSM training step", and "Only the evaluation of PiPhi changes").   */
/* `batch` independent pairs of equal sizes are stored back to back: Q        */
/* [batch][nN][ldq], K [batch][nM][ldk], V [batch][nM][ldv], O [batch][nN]    */
/* [ldo], lse [batch][nN], dO, dQ like O/Q, dK, dV like K/V (pair b starts    */
/* b nN rows, resp. b nM rows, after pair 0).  Patch tables per pair:         */
/* offN [batch][PN+1], memN [batch][nN], offM [batch][PM+1], memM [batch][nM] */
/* with vertex ids local to the pair, topk [batch][PN][R] with source patches */
/* local to the pair.  One launch of each kernel covers every pair: the       */
/* dense calls run a block-diagonal tile schedule (row tiles of pair b visit  */
/* only the key tiles of pair b), the Geo calls shift the tables of pair b by */
/* b nN / b nM vertices and b PN / b PM patches into one problem.  Results    */
/* equal those of the single-pair calls on each pair (the bf16 dense forward  */
/* uses the single-CTA kernel, so its rounding order differs from the pair    */
/* kernel's).  Table entries outside their pair's range are dropped and set   */
/* SSC_ERR_INVALID_ARG in the device status word; they never reach another    */
/* pair.  Limits: batch nN, batch nM <= 2^30; Geo: batch PN, batch PM <=      */
/* 65535.  The fp32 check mode of the dense calls runs pair after pair.       */
/*                                                                            */
/* The reverse coupling Pi_MN Phi_N = softmax(s F_M F_N^T) Phi_N, which       */
/* pipelines use to map in the other direction, is the same call with the     */
/* roles swapped: Q = F_M, K = F_N, V = Phi_N (and, for Geo, the M tables as  */
/* the target tables, with top-R lists scored from F_M against F_N).  A batch */
/* may hold pairs of both directions when their sizes agree.                  */
/* ------------------------------------------------------------------------ */

size_t ssc_dense_coupling_batched_workspace_size(int batch, int nN, int nM, int d, int k,
                                                 int dtype);

int ssc_dense_coupling_fwd_batched(int batch, const void* Q, int ldq, const void* K, int ldk,
                                   const void* V, int ldv, int nN, int nM, int d, int k,
                                   float scale, int dtype, float* O, int ldo, float* lse,
                                   void* ws, size_t ws_bytes, ssc_stream_t stream);

int ssc_dense_coupling_bwd_batched(int batch, const void* Q, int ldq, const void* K, int ldk,
                                   const void* V, int ldv, int nN, int nM, int d, int k,
                                   float scale, int dtype, const float* O, int ldo,
                                   const float* lse, const float* dO, int lddo,
                                   float* dQ, int lddq, float* dK, int lddk,
                                   float* dV, int lddv,
                                   void* ws, size_t ws_bytes, ssc_stream_t stream);

size_t ssc_geo_coupling_batched_workspace_size(int batch, int nN, int nM, int d, int k, int PN,
                                               int PM, int R, int dtype);

int ssc_geo_coupling_fwd_batched(int batch, const void* Q, int ldq, const void* K, int ldk,
                                 const void* V, int ldv, int nN, int nM, int d, int k, float scale,
                                 int dtype, const int* offN, const int* memN, int PN,
                                 const int* offM, const int* memM, int PM, const int* topk, int R,
                                 float* O, int ldo, float* lse,
                                 void* ws, size_t ws_bytes, ssc_stream_t stream);

int ssc_geo_coupling_bwd_batched(int batch, const void* Q, int ldq, const void* K, int ldk,
                                 const void* V, int ldv, int nN, int nM, int d, int k, float scale,
                                 int dtype, const int* offN, const int* memN, int PN,
                                 const int* offM, const int* memM, int PM, const int* topk, int R,
                                 const float* O, int ldo, const float* lse,
                                 const float* dO, int lddo,
                                 float* dQ, int lddq, float* dK, int lddk,
                                 float* dV, int lddv,
                                 void* ws, size_t ws_bytes, ssc_stream_t stream);

/* Pooling, scores and top-R for a batch: FN [batch][nN][ldn], FM
 * [batch][nM][ldm], tables as above; topk [batch][PN][R] (local source
 * patches), scores [batch][PN][PM] (nullable).  Bit-identical, pair by pair,
 * to ssc_patch_scores_topk. */
size_t ssc_patch_scores_topk_batched_workspace_size(int batch, int nN, int nM, int PN, int PM,
                                                    int d);

int ssc_patch_scores_topk_batched(int batch, const void* FN, int ldn, int nN, const void* FM,
                                  int ldm, int nM, int d, int dtype, const int* offN,
                                  const int* memN, int PN, const int* offM, const int* memM, int PM,
                                  int R, int* topk, double* scores,
                                  void* ws, size_t ws_bytes, ssc_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Linear-attention (ELU) coupling: the approximate coupling of the project   */
/* page's Table 1 (row "Linear attention (ELU)"); the digest's               */
/* "Interpretation" describes linear attention as replacing the softmax with */
/* a low-rank feature map.  Feature map phi(x) = elu(x) + 1 (x + 1 for x > 0,  */
/* exp(x) otherwise) on every descriptor entry; weights <phi(Q_i), phi(K_j)>, */
/* each row normalised by its weight sum:                                    */
/*   O_i = sum_j <phi(Q_i), phi(K_j)> V_j / den_i,                            */
/*   den_i = sum_j <phi(Q_i), phi(K_j)>,                                      */
/* evaluated as phi(Q_i) (sum_j phi(K_j)^T V_j) / <phi(Q_i), sum_j phi(K_j)>, */
/* linear in nN + nM.  There is no scale (the map has none).                 */
/* Q [nN, ldq], K [nM, ldk], V [nM, ldv] bf16 (Q and K 16-byte aligned with  */
/* ldq, ldk multiples of 8; V any stride, re-packed when needed); d in       */
/* {64, 128}, 1 <= k <= 255.  phi(Q), phi(K), the d x (k+1) sums and dO/den  */
/* are rounded to bf16 for the tensor cores, accumulation is fp32.  Outputs  */
/* fp32: O [nN, ldo] (16-byte aligned), den [nN].                            */
/* ------------------------------------------------------------------------ */

size_t ssc_linear_coupling_workspace_size(int nN, int nM, int d, int k);

int ssc_linear_coupling_fwd(const void* Q, int ldq, const void* K, int ldk,
                            const void* V, int ldv, int nN, int nM, int d, int k,
                            float* O, int ldo, float* den,
                            void* ws, size_t ws_bytes, ssc_stream_t stream);

/* Backward for dL/dO = dO (fp32 [nN, lddo]), given the forward's O and den:
 *   D_i = <dO_i, O_i>, dW_ij = (<dO_i, V_j> - D_i) / den_i for the weights
 *   W_ij = <phi(Q_i), phi(K_j)>, dQ_i = phi'(Q_i) * sum_j dW_ij phi(K_j),
 *   dK_j = phi'(K_j) * sum_i dW_ij phi(Q_i), dV_j = sum_i W_ij dO_i / den_i,
 * with phi'(x) = 1 for x > 0 and exp(x) otherwise; evaluated in the same
 * factored form as the forward.  dO is rounded to bf16 once.  dV may be NULL;
 * dQ [nN, lddq], dK [nM, lddk], dV [nM, lddv] fp32 (16-byte aligned) are
 * overwritten. */
int ssc_linear_coupling_bwd(const void* Q, int ldq, const void* K, int ldk,
                            const void* V, int ldv, int nN, int nM, int d, int k,
                            const float* O, int ldo, const float* den,
                            const float* dO, int lddo,
                            float* dQ, int lddq, float* dK, int lddk,
                            float* dV, int lddv,
                            void* ws, size_t ws_bytes, ssc_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SSC_H_ */
