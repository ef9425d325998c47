/*
 * svg.h -- C ABI of the B200 semantic-aware top-p sparse attention library
 * (libsvg.so, built for sm_100a).
 *
 * The five calls are the stages of the method described on the page
 * "Sparse VideoGen2: Accelerate Video Generation with Sparse Attention via
 * Semantic-Aware Permutation" (technical summary, section 2):
 *
 *   svg_kmeans       section 2(a) "Clustering" + 2(c) "Centroid cache"
 *   svg_permute      section 2(a) "Permutation"
 *   svg_select_topp  section 2(b) "Centroid approximation" + "Top-p strategy"
 *   svg_sparse_attn  section 2(c) "Customized attention kernel"
 *   svg_unpermute    section 2(a) "Mathematical equivalence"
 *
 * svg_sparse_attn_unpermuted is the last two in one kernel (the
 * un-permutation done by the attention kernel's store).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Tensors are head-major: a [BH, N, D] tensor holds BH = batch*heads
 *    independent heads of N tokens with D channels, row-major, contiguous.
 *    Q/K/V and outputs are bfloat16 (raw 16-bit storage), centroids float32,
 *    indices int32.  D must be 64 or 128.
 *  - Every pointer argument is a DEVICE pointer owned by the caller, except
 *    the pointer arrays `src`/`dst` of svg_permute, which are host arrays
 *    holding device pointers.  The library never allocates or frees device
 *    memory: scratch space comes from the caller as `ws`/`ws_bytes`, sized
 *    with the matching *_workspace_size() call.  Workspaces need 256-byte
 *    alignment and may be reused between calls on the same stream.
 *  - Device pointers to bf16 tensors need 16-byte alignment.
 *  - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *    default stream).  Arguments are checked on the host before anything is
 *    launched; a bad argument returns SVG_ERR_INVALID_ARG / _UNSUPPORTED /
 *    _WORKSPACE and launches nothing.  A launch failure returns SVG_ERR_CUDA.
 *  - Kernels never trap.  Every wait inside a kernel is bounded in time
 *    (svg_set_wait_timeout_ns); when a bound is hit or a device-side check
 *    fails the kernel records a code in a device error word and returns.
 *    svg_get_error() reads and clears that word.
 *  - Nothing throws across this boundary.
 */
#ifndef SVG_H_
#define SVG_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st *svg_stream_t; /* same type as cudaStream_t */

typedef enum svg_status {
  SVG_OK = 0,
  SVG_ERR_INVALID_ARG = 1,  /* null/misaligned pointer, bad size, p out of range, C > N ... */
  SVG_ERR_UNSUPPORTED = 2,  /* head dimension other than 64/128, sizes beyond int32 ranges */
  SVG_ERR_WORKSPACE = 3,    /* ws smaller than the *_workspace_size() result */
  SVG_ERR_CUDA = 4,         /* a CUDA runtime/driver call failed (launch, tensor map) */
  SVG_ERR_TIMEOUT = 5,      /* a bounded in-kernel wait expired (device error word) */
  SVG_ERR_DEVICE_CHECK = 6  /* a device-side consistency check failed (device error word) */
} svg_status;

/* Human-readable name of a status code (static string). */
const char *svg_status_string(svg_status s);

/* The last CUDA failure that made a call return SVG_ERR_CUDA: what failed
 * (kernel or CUDA call) and CUDA's own message; "" if none yet.  The string
 * belongs to the library and stays valid in the calling thread until its
 * next call of this function. */
const char *svg_last_cuda_error(void);

/* ------------------------------------------------------------------------ k-means
 * Lloyd's k-means on every head independently (section 2(a) "Clustering":
 * Q and K are clustered independently into C_q and C_k clusters).
 *
 *   x          [BH, N, D] bf16   tokens (Q or K of one layer)
 *   centroids  [BH, C, D] fp32   in: initial centroids (seeding tokens, or the
 *                                previous denoising step's centroids = the
 *                                "centroid cache" of section 2(c));
 *                                out: centroids after `iters` rounds
 *   assign     [BH, N]    int32  out: cluster of every token, from the last
 *                                assign step
 *   counts     [BH, C]    int32  out: tokens per cluster for `assign`
 *
 * One round = assign (a_n = argmin_c ||x_n - mu_c||^2, ties to the lowest c)
 * then update (mu_c = mean of its tokens, rounded once to fp32; an empty
 * cluster keeps its centroid).  Sums run in fp64, where every partial sum of
 * bf16 values of ordinary range is exact, so the summation order does not
 * change the result.  The returned centroids are the means of the returned
 * assignment.  Requires iters >= 1, 1 <= C <= N,
 * C <= 1024.  Distances run on the tensor cores with the centroids split
 * into a bf16 high and low part (about 16 significant bits).
 */
size_t svg_kmeans_workspace_size(int BH, int N, int D, int C);
svg_status svg_kmeans(const void *x, int BH, int N, int D, int C, int iters, float *centroids,
                      int32_t *assign, int32_t *counts, void *ws, size_t ws_bytes,
                      svg_stream_t stream);

/* ------------------------------------------------------------------------ permutation
 * Semantic-aware permutation (section 2(a) "Permutation"): a stable counting
 * sort of the tokens of every head by cluster id, then a row gather.
 *
 *   assign   [BH, N]    int32  cluster ids in [0, C)
 *   perm     [BH, N]    int32  out: perm[r] = source token of permuted row r;
 *                              inside a cluster tokens keep ascending order
 *   offsets  [BH, C+1]  int32  out: cluster c = rows [offsets[c], offsets[c+1])
 *   src/dst  host arrays of `ntensors` (0..3) device pointers to [BH, N, D]
 *            bf16 tensors; dst[t][h][r] = src[t][h][perm[h][r]].  Q uses the
 *            Q permutation; K and V share the K permutation (call once with
 *            ntensors = 2).  dst must not alias src.
 * A device-side range check of `assign` records SVG_ERR_DEVICE_CHECK.
 */
size_t svg_permute_workspace_size(int BH, int N, int C);
svg_status svg_permute(const int32_t *assign, int BH, int N, int C, int32_t *perm, int32_t *offsets,
                       int ntensors, const void *const *src, void *const *dst, int D, void *ws,
                       size_t ws_bytes, svg_stream_t stream);

/* ------------------------------------------------------------------------ top-p selection
 * Centroid-based top-p block selection (section 2(b)).  For every head h and
 * q-cluster i with n_q[h,i] > 0:
 *     logit_j = scale * mu_q[h,i] . mu_k[h,j]
 *     w_j     = n_k[h,j] * exp(logit_j - max) / sum      (live j: n_k > 0)
 * k-clusters are sorted by w descending (ties: lower j) and the shortest
 * prefix whose cumulative weight reaches p is kept (p >= 1: every live j).
 *
 *   mu_q [BH, Cq, D] fp32, n_q [BH, Cq] int32, mu_k [BH, Ck, D] fp32, n_k [BH, Ck] int32
 *   sel_count [BH, Cq]     int32  out: number of selected k-clusters (0 for empty rows)
 *   sel_cols  [BH, Cq, Ck] int32  out: row (h,i) holds its selected k-cluster ids in
 *                                 ascending order in its first sel_count entries;
 *                                 the remaining entries are left untouched
 * Requires 0 < p, Ck <= 1024; scale <= 0 selects 1/sqrt(D) (formed in
 * float64).  The cut turns weights into an integer set, so logits, weights
 * and prefix masses are evaluated in float64 (products of fp32 centroid
 * channels are exact there); a float64 evaluation can differ from the exact
 * cut only when a prefix mass lies within about 1e-12 of p.
 */
svg_status svg_select_topp(const float *mu_q, const int32_t *n_q, const float *mu_k,
                           const int32_t *n_k, int BH, int Cq, int Ck, int D, float p, float scale,
                           int32_t *sel_count, int32_t *sel_cols, svg_stream_t stream);

/* ------------------------------------------------------------------------ sparse attention
 * Attention over the selected variable-size blocks (section 2(c) "Customized
 * attention kernel"): permuted query rows of q-cluster i attend, with exact
 * softmax and no causal mask, to the union of the permuted key rows of the
 * k-clusters selected for i.
 *
 *   qp, kp, vp  [BH, N, D] bf16  permuted Q (Q permutation), K and V (K permutation)
 *   q_off       [BH, Cq+1] int32 q-cluster row ranges (svg_permute offsets)
 *   k_off       [BH, Ck+1] int32 k-cluster row ranges
 *   sel_count, sel_cols          svg_select_topp output
 *   op          [BH, N, D] bf16  out: permuted output rows
 *   lse         [BH, N]    fp32  optional out (NULL to skip): natural-log
 *                                sum_j exp(scale * q.k_j) per row
 * Rows of empty q-clusters do not exist; every other row is written.  A row
 * whose cluster selected no key is left untouched and flagged with
 * SVG_ERR_DEVICE_CHECK, and so is a sel_count outside [0, Ck] (it is clamped
 * before any block list entry is read).  Requires Ck <= 1024
 * (SVG_ERR_UNSUPPORTED otherwise).  scale <= 0 selects 1/sqrt(D).
 */
size_t svg_sparse_attn_workspace_size(int BH, int N, int Cq);
svg_status svg_sparse_attn(const void *qp, const void *kp, const void *vp, int BH, int N, int D,
                           const int32_t *q_off, int Cq, const int32_t *k_off, int Ck,
                           const int32_t *sel_count, const int32_t *sel_cols, float scale, void *op,
                           float *lse, void *ws, size_t ws_bytes, svg_stream_t stream);

/* The same attention with the un-permutation (section 2(a) "Mathematical
 * equivalence": O[perm_q[r]] = O'[r]) fused into the kernel's store: row r
 * of a head's result goes to row perm_q[r] of o, so o is in the original token
 * order and no permuted copy of the output exists.
 *
 *   perm_q  [BH, N]    int32  the Q permutation (svg_permute), required
 *   o       [BH, N, D] bf16   out: attention output in token order; must not
 *                             alias qp, kp or vp
 *   lse     [BH, N]    fp32   optional out, also in token order
 * Other arguments, the workspace and the result are those of svg_sparse_attn
 * followed by svg_unpermute.  A perm_q entry outside [0, N) is skipped and
 * flagged with SVG_ERR_DEVICE_CHECK.
 */
svg_status svg_sparse_attn_unpermuted(const void *qp, const void *kp, const void *vp, int BH,
                                      int N, int D, const int32_t *q_off, int Cq,
                                      const int32_t *k_off, int Ck, const int32_t *sel_count,
                                      const int32_t *sel_cols, float scale, const int32_t *perm_q,
                                      void *o, float *lse, void *ws, size_t ws_bytes,
                                      svg_stream_t stream);

/* Attention with K and V in token order (section 2(c) "Customized attention
 * kernel": the selected key rows are loaded sparsely from where they are and
 * computed on densely): the kernel fetches permuted key row r of head h from
 * row perm_k[h][r] of k and v with 16-byte asynchronous copies, so no
 * permuted copy of K or V exists.  Q is permuted (dense query tiles).
 *
 *   qp      [BH, N, D] bf16   Q permuted by the Q permutation
 *   k, v    [BH, N, D] bf16   K and V in token order
 *   perm_k  [BH, N]    int32  the K permutation (svg_permute of the K
 *                             clusters with ntensors = 0): perm_k[h][r] = token
 *                             of permuted key row r; k_off its offsets
 *   perm_q  [BH, N]    int32  optional: with it o (and lse) are stored in
 *                             token order as in svg_sparse_attn_unpermuted;
 *                             NULL stores Q-permuted rows as svg_sparse_attn
 *   o       [BH, N, D] bf16   out; must not alias k or v (nor qp with perm_q)
 * The other arguments, the workspace and the result are those of
 * svg_sparse_attn (with perm_q: svg_sparse_attn_unpermuted).  A perm_k entry
 * outside [0, N) is replaced by 0 and flagged with SVG_ERR_DEVICE_CHECK.
 */
svg_status svg_sparse_attn_gather(const void *qp, const void *k, const void *v, const int32_t *perm_k,
                                  int BH, int N, int D, const int32_t *q_off, int Cq,
                                  const int32_t *k_off, int Ck, const int32_t *sel_count,
                                  const int32_t *sel_cols, float scale, const int32_t *perm_q,
                                  void *o, float *lse, void *ws, size_t ws_bytes,
                                  svg_stream_t stream);

/* ------------------------------------------------------------------------ 8-bit Q K^T
 * Low-bit attention in the spirit of the page "TurboDiffusion" (section
 * "SageAttention: low-bit quantization": attention on quantised operands to
 * cut memory traffic and compute).  The page fixes no format; here Q and K
 * are FP8 E4M3 (bias 7, 3 mantissa bits, largest finite 448; round to
 * nearest, ties to even, saturating at +-448), the logits are
 * scale * (q8 . k8) * s_q[row] * s_k[head], and P and V stay bf16.
 *
 * svg_quantize_e4m3: x [BH, N, D] bf16 -> x8 [BH, N, D] E4M3 bytes and float32
 * scales, x8 = E4M3(x / s) with the division in float32 and
 * s = amax|x| / 448 (1 where amax is 0):
 *   per_row = 1   one scale per row, scales [BH * N]   (for Q)
 *   per_row = 0   one scale per head over all N*D values, scales [BH]  (for K)
 * D = 64 or 128.  x and x8 16-byte aligned, not aliased.  The per-head form
 * zeroes `scales` (stream-ordered) before reducing into it.
 * perm [BH, N] int32 is optional: with it the rows are gathered on the way,
 * x8[h][i] = E4M3(x[h][perm[h][i]] / s) (per-row scales follow the output
 * row; a head's scale does not depend on the order), so the permuted Q and K
 * of svg_permute need not be written in bf16 first.  A perm entry outside
 * [0, N) gives a zero row and is flagged with SVG_ERR_DEVICE_CHECK.
 *
 * svg_sparse_attn_fp8: svg_sparse_attn / svg_sparse_attn_unpermuted with
 * q8 [BH, N, D] and k8 [BH, N, D] E4M3 in permuted row order (svg_quantize_e4m3
 * of q and k through perm_q and perm_k, or of the permuted qp and kp),
 * q_scale [BH * N] and k_scale [BH] their scales, vp bf16.  perm_q optional: with it o (and lse) are in token order, else in
 * the Q-permuted order.  D must be 128 (SVG_ERR_UNSUPPORTED otherwise).  The
 * workspace is svg_sparse_attn_workspace_size(BH, N, Cq) bytes; other
 * arguments and the error behaviour are those of svg_sparse_attn.
 */
svg_status svg_quantize_e4m3(const void *x, const int32_t *perm, int BH, int N, int D, int per_row, void *x8,
                             float *scales, svg_stream_t stream);
svg_status svg_sparse_attn_fp8(const void *q8, const float *q_scale, const void *k8, const float *k_scale,
                               const void *vp, int BH, int N, int D, const int32_t *q_off, int Cq,
                               const int32_t *k_off, int Ck, const int32_t *sel_count, const int32_t *sel_cols,
                               float scale, const int32_t *perm_q, void *o, float *lse, void *ws,
                               size_t ws_bytes, svg_stream_t stream);

/* ------------------------------------------------------------------------ DynamicRad block masks
 * Block masks of the page "DynamicRad: Content-Adaptive Sparse Attention for
 * Long Video Diffusion", section 2(a) (radial candidate set; static-ratio and
 * dynamic-threshold modes), written in the block-list format of
 * svg_select_topp so svg_sparse_attn runs them on Q, K and V in token order
 * (q_off = k_off = offsets; no permutation).
 *
 * Tokens are frame-major: token n = t*S + s with S = N / frames.  A block is
 * `block` consecutive tokens of one frame: a frame has nb = ceil(S / block)
 * blocks (the last one ragged), block id c = t*nb + b.  Key block (t2, b2) is
 * a candidate of query block (t1, b1) iff |b1 - b2| <= w(|t1 - t2|),
 * w(d) = floor(w0 * gamma^d) (gamma^d formed by d successive float64
 * multiplications).  Modes:
 *   SVG_DYNRAD_CANDIDATES  every candidate;
 *   SVG_DYNRAD_STATIC      per key frame the max(1, ceil(rho(d) * m)) candidates
 *                          nearest to b1 (ties to the lower b2), m = candidates
 *                          in that frame, rho(d) = min(1, rho0 * gamma^d);
 *   SVG_DYNRAD_DYNAMIC     candidates whose proxy scale * mean(q rows of the
 *                          query block) . mean(k rows of the key block)
 *                          (float64) is >= theta; a query block keeping none
 *                          keeps its highest-proxy candidate (ties: lower id).
 *
 *   q, k       [BH, N, D] bf16 (read in dynamic mode only; may be NULL otherwise)
 *   offsets    [BH, Cb+1] int32  out: first token of every block, then N
 *   sel_count  [BH, Cb]   int32  out: kept key blocks per query block (>= 1)
 *   sel_cols   [BH, Cb, Cb] int32 out: kept key block ids, ascending
 *   ws         dynamic mode: svg_dynrad_workspace_size bytes (the float64
 *              block means); unused otherwise
 * Cb = svg_dynrad_num_blocks(N, frames, block) (0 when frames does not divide
 * N or an argument is not positive).  Requires Cb <= 1024
 * (SVG_ERR_UNSUPPORTED), w0 >= 0, gamma >= 0, rho0 > 0 in static mode, and
 * D = 64 or 128 in dynamic mode.  scale <= 0 selects 1/sqrt(D).
 */
enum { SVG_DYNRAD_CANDIDATES = 0, SVG_DYNRAD_STATIC = 1, SVG_DYNRAD_DYNAMIC = 2 };
int svg_dynrad_num_blocks(int N, int frames, int block);
size_t svg_dynrad_workspace_size(int BH, int N, int D, int frames, int block);
svg_status svg_dynrad_select(const void *q, const void *k, int BH, int N, int D, int frames, int block, int mode,
                             float w0, float gamma, float rho0, float theta, float scale, int32_t *offsets,
                             int32_t *sel_count, int32_t *sel_cols, void *ws, size_t ws_bytes,
                             svg_stream_t stream);

/* ------------------------------------------------------------------------ sparse attention, no allocation
 * No counterpart on the pages: this is a service for callers that cannot hand
 * the library a scratch buffer.  Some callers have no way to obtain device
 * memory at the point where they call: a plug-in running inside a host
 * framework that owns every allocation, an inference loop whose memory budget
 * is fixed when it starts, or a runtime that forbids device allocation after
 * initialisation.  This call takes the same inputs and outputs as
 * svg_sparse_attn and computes the same result, but its scratch space is a
 * fixed array compiled into the library (SVG_NOALLOC_SCRATCH_BYTES, 4 MiB) that
 * every GPU which loads the library holds until the process exits.
 *
 *  - Limit: svg_sparse_attn_workspace_size(BH, N, Cq), about
 *    16*BH*(ceil(N/256) + Cq) + 16*BH*Cq bytes plus 2.5 MiB of per-CTA key
 *    ranges, must not exceed SVG_NOALLOC_SCRATCH_BYTES (e.g. 80 heads x 75,600
 *    tokens x 200 q-clusters needs 3.5 MB); larger sizes return
 *    SVG_ERR_WORKSPACE before anything is launched.
 *  - It allocates and frees nothing (no cudaMalloc, no cudaFree, no
 *    allocating library routine).
 *  - The first call on each device looks up the device address of the array
 *    (cudaGetSymbolAddress, with that device current) and caches it; make that
 *    first call before any stream capture.
 *  - All calls share the one array and it keeps the previous call's contents;
 *    the call rewrites every scratch entry it reads, so nothing needs
 *    clearing, but calls whose executions overlap on the GPU (different
 *    streams, or host threads) race on the array: order them on one stream.
 */
#define SVG_NOALLOC_SCRATCH_BYTES (4u << 20)
svg_status svg_sparse_attn_noalloc(const void *qp, const void *kp, const void *vp, int BH, int N,
                                   int D, const int32_t *q_off, int Cq, const int32_t *k_off,
                                   int Ck, const int32_t *sel_count, const int32_t *sel_cols,
                                   float scale, void *op, float *lse, svg_stream_t stream);

/* ------------------------------------------------------------------------ un-permutation
 * Inverse permutation (section 2(a) "Mathematical equivalence"):
 * x[h][perm[h][r]] = xp[h][r] for every row r.  x must not alias xp.
 */
svg_status svg_unpermute(const void *xp, const int32_t *perm, int BH, int N, int D, void *x,
                         svg_stream_t stream);

/* ------------------------------------------------------------------------ errors and limits
 * svg_get_error synchronises `stream`, then returns and clears the device
 * error word of the current device (SVG_OK when nothing was recorded;
 * SVG_ERR_CUDA when the synchronisation itself failed).
 * svg_set_wait_timeout_ns sets the bound of every in-kernel wait for the
 * following launches (default 2e9 ns; 0 restores the default).
 */
svg_status svg_get_error(svg_stream_t stream);
void svg_set_wait_timeout_ns(uint64_t ns);

/* Where the first recorded device error came from (the site field of the
 * device error word). */
typedef enum svg_error_site {
  SVG_SITE_NONE = 0,
  SVG_SITE_ATTN_PRODUCER = 1,   /* attention: item loader or TMA producer warp */
  SVG_SITE_ATTN_MMA = 2,        /* attention: an MMA issuer warp */
  SVG_SITE_ATTN_SOFTMAX = 3,    /* attention: a softmax warp */
  SVG_SITE_ATTN_DRAIN = 4,      /* attention: waiting for copies in flight after an abort */
  SVG_SITE_ATTN_EMPTY_ROW = 5,  /* attention planning: bad k-cluster id or no keys selected */
  SVG_SITE_PERMUTE_RANGE = 6,   /* permute: cluster id outside [0, C) */
  SVG_SITE_KMEANS_MMA = 7,      /* k-means assign: MMA issuer warp */
  SVG_SITE_KMEANS_EPI = 8,      /* k-means assign: epilogue warps */
  SVG_SITE_KMEANS_RANGE = 9,    /* k-means update: cluster id outside [0, C) */
  SVG_SITE_KMEANS_DRAIN = 10    /* k-means assign: waiting for copies in flight after an abort */
} svg_error_site;

/* Same as svg_get_error (synchronises, returns and clears the error word),
 * and also reports where the error came from: *site (an svg_error_site) and
 * *block (the low 16 bits of the recording CTA's blockIdx.x); both 0 when
 * nothing was recorded.  Either pointer may be NULL. */
svg_status svg_get_error_detail(svg_stream_t stream, int32_t *site, int32_t *block);

/* Test hook for failure detection (no GPU fault involved): fault = 1 makes
 * the following svg_sparse_attn launches skip loading their query tiles, so
 * the kernel's bounded waits run out, it records SVG_ERR_TIMEOUT, waits for
 * its own in-flight copies, frees its tensor memory and returns; fault = 0
 * restores normal operation.  Outputs of a faulted launch are undefined. */
void svg_debug_set_fault(int fault);

/* ------------------------------------------------------------------------ kernel timing
 * Live per-kernel timing for benchmarks.  While enabled, the library records
 * a pair of CUDA events on the caller's stream around every launch of its two
 * heavy kernels: kernel 0 = the k-means assign kernel (inside svg_kmeans),
 * kernel 1 = the block-sparse attention kernel (inside svg_sparse_attn and
 * svg_sparse_attn_unpermuted, without their planning kernels).  Events come from a fixed pool created on
 * the first enable (up to 1024 launches between reads; later launches are not
 * timed and are reported in `dropped`).  svg_profile_read waits for the
 * recorded events, returns the summed milliseconds and the number of timed
 * launches of one kernel since the previous read, and resets that kernel's
 * record.  Timing adds two event records per launch and nothing else. */
svg_status svg_profile_enable(int on);
svg_status svg_profile_read(int kernel, double *ms, int *launches, int *dropped);

/* While profiling is enabled, every attention launch also counts the
 * (128-row query tile, 128-key tile) pairs it issues tensor-core work for: one
 * S = Q K^T chain and one O += P V chain each, i.e. 4 * 128 * 128 * D
 * multiply-add FLOPs including masked padding rows and columns.  This call
 * waits for the device, returns the count accumulated since the previous call
 * and resets it.  Issued FLOPs against the selected blocks' FLOPs give the
 * padding waste of the variable-size blocks. */
svg_status svg_profile_attn_pairs(uint64_t *pairs);

/* Library version, e.g. "svg-b200 0.2 (sm_100a)". */
const char *svg_version(void);

#ifdef __cplusplus
}
#endif
#endif /* SVG_H_ */
