/*
 * prism.h -- C ABI of the B200 (sm_100a) implementation of Prism's dynamic
 * block-sparse video self-attention ("Prism: Dynamic Sparse Attention for
 * Native 2K Joint Video-Audio Generation Model Training", arXiv 2610.05416).
 *
 * The path, in call order (forward):
 *   prism_zone_indicator -> prism_assign_blocks -> prism_permute (Q, K, V)
 *   -> prism_block_select -> prism_bsa_fwd -> prism_unpermute (O)
 * and backward:
 *   prism_permute (dO) -> prism_bsa_bwd -> prism_unpermute (dQ, dK, dV)
 *
 * Conventions shared by every entry point
 *   - All pointers are DEVICE pointers unless a comment says otherwise; the
 *     caller owns every buffer.  No entry point allocates device memory:
 *     scratch comes in through (workspace, ws_bytes), sized by
 *     prism_workspace_size().
 *   - Every call is asynchronous on `stream` (a cudaStream_t; NULL is the
 *     legacy default stream).  Counts produced on the device (the number of
 *     blocks, the number of selected pairs) stay on the device; buffers are
 *     sized by the upper bounds stated below so that no call needs a host sync.
 *   - Return value: PRISM_OK, or a negative status for errors found on the
 *     host before launch (PRISM_EINVAL, PRISM_ECUDA).  Errors found by a
 *     kernel (capacity overflow, a bounded wait that timed out, an index out of
 *     range) are latched in a device status word that prism_device_status()
 *     returns and clears.  prism_last_error() gives a message for the last
 *     non-zero status of the calling thread.  Nothing traps or aborts.
 *   - Layouts.  Natural token order n = (t*H + y)*W + x.  "Natural" tensors
 *     are [N, heads, head_dim]; "permuted" tensors are [heads, N, head_dim]
 *     with the tokens in zone-local block order (see prism_permute), so every
 *     block of every head is one contiguous [B, head_dim] tile.
 *   - Sizes.  Z = N/512 zones; a zone holds 512/B blocks with B in
 *     {64,128,256}, so the block count nblk <= NBLK_CAP = 8*Z.  Per-head block
 *     arrays are strided by NBLK_CAP.
 */
#ifndef PRISM_H
#define PRISM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* status codes */
#define PRISM_OK 0
#define PRISM_EINVAL (-1)    /* bad argument: null, misaligned, unsupported size */
#define PRISM_ECAPACITY (-2) /* selected pairs exceed col_capacity (device-reported) */
#define PRISM_ECUDA (-3)     /* a CUDA runtime call failed */
#define PRISM_ETIMEOUT (-4)  /* a bounded device wait gave up (device-reported) */
#define PRISM_EBOUNDS (-5)   /* a device index check failed (device-reported) */

/* element types */
#define PRISM_BF16 0
#define PRISM_F32 1

/* workspace kinds for prism_workspace_size */
#define PRISM_WS_INDICATOR 0
#define PRISM_WS_SELECT 1
#define PRISM_WS_FWD 2
#define PRISM_WS_BWD 3

typedef void *prism_stream; /* cudaStream_t */

/*
 * Problem statement (Method, and the knobs of the selection):
 *   T, H, W   token grid; each a positive multiple of the 8x8x8 macro-zone
 *             (Key ideas, "Macro-Zone Partitioning").
 *   heads, head_dim   attention heads and per-head width; head_dim 64 or 128.
 *   tau128, tau256    density thresholds of Method §2 (0.5 and 0.25).
 *   eps       the epsilon of the composite indicator g_d (Method §1); 1e-4.
 *   top_k     minimum number of key blocks per query block (Method §3), >= 1.
 *   top_p     cumulative probability mass to keep (Method §3), in (0, 1].
 *   scale     softmax scale for block scores and attention; 0 means
 *             1/sqrt(head_dim).
 * The two variants of the Prism repository's configuration table (its README):
 *   fixed_shape  PRISM_DYNAMIC_SHAPES (0): the dynamic assignment of Method §2.
 *             PRISM_FIXED_SHAPE(s) (s + 1, s a canonical shape index 0..15):
 *             every zone takes shape s and g, rho are not read.  With the
 *             dynamic assignment switched off (enable_ivpq_dynamic_block
 *             false) the README's blocks are 4x4x4: PRISM_FIXED_444.
 *   sparsity  0: k = top_k.  In (0, 1]: the README's ratio form bsa_sparsity,
 *             the share of key blocks a query block skips, so
 *             k = max(1, ceil((1 - sparsity) * nblk)) (formed in double from
 *             this float) and top_k is not read.
 * A zero-initialised tail (both 0) gives the method as the paper states it.
 */
typedef struct {
  int32_t T, H, W;
  int32_t heads, head_dim;
  float tau128, tau256;
  float eps;
  int32_t top_k;
  float top_p;
  float scale;
  int32_t fixed_shape;
  float sparsity;
} prism_params;

#define PRISM_DYNAMIC_SHAPES 0
#define PRISM_FIXED_SHAPE(s) ((s) + 1)
#define PRISM_FIXED_444 PRISM_FIXED_SHAPE(3)

/* One block of the zone-local layout: permuted rows [start, start+size) of
 * every head, inside zone `zone`, of canonical shape index `shape`. */
typedef struct {
  int32_t start, size, zone, shape;
} prism_block;

/* Bytes of workspace an entry point needs (kind = PRISM_WS_*).  For
 * PRISM_WS_SELECT the amount is the minimum (one head of block scores at a
 * time); more lets more heads run per pass, up to `*bytes_all_heads`.
 * col_capacity matters for PRISM_WS_BWD only.  Host-only; returns a status. */
int prism_workspace_size(const prism_params *p, int kind, int64_t col_capacity,
                         size_t *bytes, size_t *bytes_all_heads);

/*
 * Method §1, the indicator's audio input: a_n = ||h_n||_2, the Euclidean norm
 * of each video token's audio-to-video cross-attention output over all of its
 * channels (heads * head_dim of that layer, all heads together).  The pages
 * cache these norms from the preceding layer; this is the producer.
 *   h      [N, C] row-major, PRISM_BF16 or PRISM_F32, 16-byte aligned; C > 0 a
 *          multiple of 8 (bf16) or 4 (f32).  Squares are summed in float.
 *   a      out [N] float.
 * N = 0 launches nothing.  Host-detected errors return PRISM_EINVAL.
 */
int prism_audio_norms(const void *h, int h_dtype, int64_t N, int C, float *a, prism_stream stream);

/*
 * Method §1 and the density of §2: per macro-zone m, the directional video
 * variances sigma^2_{v,d}(m) of the mean-pooled V along T, H and W (averaged
 * over all heads*head_dim channels), r_{v,d} = sigma^2_{v,d}/sum, the audio
 * coupling abar(m) = zone mean of a / global max of a, the normalised audio
 * directional variance vhat_{a,d} (a pooled like V), the composite indicator
 * g_d = r_{v,d} + abar*vhat_{a,d} + eps and the density
 * rho(m) = (info(m)/max info + abar(m))/2 with info = sum_d sigma^2_{v,d}.
 *   V      natural [N, heads, head_dim], dtype PRISM_BF16 or PRISM_F32,
 *          16-byte aligned.
 *   audio  [N] float, nullable: NULL (first layer, no cached norms) means
 *          abar = vhat = 0.
 *   g      out [Z, 3] float (T, H, W);  rho  out [Z] float.
 *   debug  out, nullable: [Z, 8] float = sigma2_v[3], info, abar, vhat_a[3].
 *   workspace  >= prism_workspace_size(PRISM_WS_INDICATOR) bytes.
 */
int prism_zone_indicator(const prism_params *p, const void *V, int v_dtype, const float *audio,
                         float *g, float *rho, float *debug, void *workspace, size_t ws_bytes,
                         prism_stream stream);

/*
 * The indicator in two halves, for a grid whose tokens are spread over several
 * GPUs by T-slabs (slabs of whole 8-frame zone layers; a slab is a grid of its
 * own and its zones are the full grid's zones m0 .. m0+Z_slab-1, in order):
 *
 * prism_zone_records: per zone of the grid described by p (a slab), the
 *   record of PRISM_ZONE_RECORD doubles
 *     [sigma2_v,T  sigma2_v,H  sigma2_v,W  info  mean(a)  sigma2_a,T
 *      sigma2_a,H  sigma2_a,W  max(a)]
 *   (Method §1: channel-averaged axis variances of the mean-pooled V, their
 *   sum, and the same pooling of the audio norms; zeros where audio is NULL).
 *   V, audio, workspace as in prism_zone_indicator; records out [Z, 9].
 * prism_zone_finalize: from the records of ALL zones of the whole grid
 *   (p describes the whole grid; the slabs' records concatenated in slab
 *   order), the grid maxima of info and max(a), then g, rho and debug exactly
 *   as prism_zone_indicator computes them.  has_audio: nonzero if audio norms
 *   were given.
 * prism_zone_records on the whole grid followed by prism_zone_finalize gives
 * bit for bit the result of prism_zone_indicator.
 */
#define PRISM_ZONE_RECORD 9
int prism_zone_records(const prism_params *p, const void *V, int v_dtype, const float *audio,
                       double *records, void *workspace, size_t ws_bytes, prism_stream stream);
int prism_zone_finalize(const prism_params *p, const double *records, int has_audio, float *g, float *rho,
                        float *debug, prism_stream stream);

/*
 * prism_zone_indicator without any workspace: the same computation, with its
 * scratch (per-zone partial sums) held in a fixed device array inside the
 * library.  It is for callers that cannot allocate device memory at the
 * point of the call: plugins that run inside another framework's execution
 * (which hands them only the input and output buffers), allocator-free or
 * real-time runtimes that must not block on cudaMalloc's implicit device
 * synchronisation, and code that otherwise would have to keep a workspace
 * alive between calls.  The pages have no counterpart; it is a deployment aid.
 *   Limits: at most PRISM_NOALLOC_MAX_ZONES macro-zones and at most
 *   PRISM_NOALLOC_MAX_CHANNELS channels (heads * head_dim); larger problems
 *   return PRISM_EINVAL without launching anything.
 *   The fixed array (about 1.8 MiB) is reserved on every GPU that loads the
 *   library until the process exits.  The first call on each device looks up
 *   the array's device address (cudaGetSymbolAddress) with that device
 *   current; make that first call before any stream capture.  The address is
 *   kept until the process exits; cudaDeviceReset would load the library's
 *   device code again, possibly elsewhere, so this entry point is not
 *   supported on a device after cudaDeviceReset.  All calls share
 *   the one array: calls that overlap on the GPU (different streams, or
 *   different host threads, without ordering between them) race on it.
 *   Every other argument, layout and error behaves as in prism_zone_indicator.
 */
#define PRISM_NOALLOC_MAX_ZONES 4096
#define PRISM_NOALLOC_MAX_CHANNELS 4096
int prism_zone_indicator_noalloc(const prism_params *p, const void *V, int v_dtype, const float *audio,
                                 float *g, float *rho, float *debug, prism_stream stream);

/*
 * Method §2: block volume B(m) (rho >= tau128 -> 64, tau256 <= rho < tau128 ->
 * 128, else 256), optimal log2 edges l*_d = -1/2 log2 g_d + 1/3(S + 1/2 sum
 * log2 g), and the nearest of the 16 candidate shapes (edges in {2,4,8},
 * product B; canonical order volume then (bT,bH,bW) ascending; distance ties
 * within 1e-9 go to the lowest index).  Decisions are taken in double.
 *   g [Z,3], rho [Z]        in (as produced by prism_zone_indicator); not
 *                           read, and may be NULL, when p->fixed_shape names a
 *                           fixed shape
 *   shape_id [Z]            out, canonical shape index
 *   zone_blk_base [Z+1]     out, first block of each zone (exclusive scan)
 *   blocks [8Z]             out, block table in zone-local order
 *   nblk [1]                out, number of blocks
 */
int prism_assign_blocks(const prism_params *p, const float *g, const float *rho, uint8_t *shape_id,
                        int32_t *zone_blk_base, prism_block *blocks, int32_t *nblk,
                        prism_stream stream);

/*
 * Zone-local token permutation with fused block mean-pooling (Method §3's
 * block representatives).  Zone m owns permuted rows [512m, 512m+512); inside
 * it the blocks follow raster order over the (8/bT, 8/bH, 8/bW) block grid and
 * the tokens of a block follow raster (t, y, x).
 *   x        natural [N, heads, head_dim], PRISM_BF16 or PRISM_F32, 16-B aligned
 *   x_perm   out, permuted [heads, N, head_dim] bf16
 *   pooled   out, nullable: [heads, 8Z, head_dim] float, mean of each block's
 *            rows (computed from x in its own precision)
 */
int prism_permute(const prism_params *p, const uint8_t *shape_id, const int32_t *zone_blk_base,
                  const void *x, int x_dtype, void *x_perm, float *pooled, prism_stream stream);

/* Inverse of prism_permute: permuted [heads, N, head_dim] (in_dtype) ->
 * natural [N, heads, head_dim] (out_dtype). */
int prism_unpermute(const prism_params *p, const uint8_t *shape_id, const void *x_perm,
                    int in_dtype, void *x, int out_dtype, prism_stream stream);

/*
 * Method §3: block scores s_ij = scale * Qbar_i . Kbar_j (float), block
 * probabilities P_i = softmax_j over the head's blocks, and the hybrid set
 * S_i = Top-k(P_i, k) U Top-p(P_i, p): key blocks ranked by (score
 * descending, index ascending); S_i is the longest of the first min(k, nblk)
 * and the shortest prefix whose mass reaches p (mass summed in 2^-40 fixed
 * point; p >= 1 keeps the whole row, the only prefix of mass 1 in exact
 * arithmetic).  k is p->top_k, or comes from p->sparsity and nblk on the device
 * when that is set.  Output is a CSR per head over rows h*8Z + i, columns
 * ascending.
 *   nblk [1]              in (device), from prism_assign_blocks
 *   q_pooled, k_pooled    in [heads, 8Z, head_dim] float
 *   row_ptr               out [heads*8Z + 1] int32 (rows i >= nblk are empty)
 *   col                   out [col_capacity] int32
 *   nnz [1]               out (device) int64, total selected pairs.  If it
 *                         exceeds col_capacity nothing is written to col and
 *                         the device status becomes PRISM_ECAPACITY.
 *   workspace             >= the PRISM_WS_SELECT minimum
 */
int prism_block_select(const prism_params *p, const int32_t *nblk, const float *q_pooled,
                       const float *k_pooled, int32_t *row_ptr, int32_t *col, int64_t col_capacity,
                       int64_t *nnz, void *workspace, size_t ws_bytes, prism_stream stream);

/*
 * Method §3: block-sparse attention forward, online softmax, bidirectional:
 * for each query row r of block i, O_r = softmax(scale q_r K^T) V over the
 * tokens of the key blocks in S_i; LSE_r = natural log of the softmax
 * denominator (including the max).
 *   blocks, nblk          from prism_assign_blocks; zone_blk_base likewise
 *   q, k, v               permuted [heads, N, head_dim] bf16, 16-B aligned
 *   row_ptr, col          CSR from prism_block_select
 *   o                     out permuted [heads, N, head_dim] bf16
 *   o_res                 out, nullable: permuted [heads, N, head_dim] bf16, the
 *                         rounding residual O_fp32 - O_bf16.  Training passes it
 *                         to prism_bsa_bwd so that D = rowsum(dO o O) sees O to
 *                         about 16 significant bits instead of 8.
 *   lse                   out [heads, N] float
 *   workspace             >= prism_workspace_size(PRISM_WS_FWD), 16-B aligned
 *                         (head_dim 128: the per-head max |v| and a copy of V
 *                         in fp16 scaled by a power of two per head, so that
 *                         O += P V runs with P in fp16; 0 bytes for head_dim 64)
 */
int prism_bsa_fwd(const prism_params *p, const prism_block *blocks, const int32_t *zone_blk_base,
                  const int32_t *nblk, const void *q, const void *k, const void *v,
                  const int32_t *row_ptr, const int32_t *col, void *o, void *o_res, float *lse,
                  void *workspace, size_t ws_bytes, prism_stream stream);

/*
 * Backward of prism_bsa_fwd for the fixed selection: with P the attention
 * probabilities, dV = P^T dO, dP = dO V^T, D_r = rowsum(dO o O),
 * dS = P (dP - D), dQ = scale dS K, dK = scale dS^T Q.
 *   o, dout               permuted [heads, N, head_dim] bf16 (forward output, its gradient)
 *   o_res                 nullable: the residual written by prism_bsa_fwd
 *   lse                   [heads, N] float from prism_bsa_fwd
 *   nnz, col_capacity     as returned to / given to prism_block_select
 *   dq, dk, dv            out permuted [heads, N, head_dim] bf16
 *   workspace             >= prism_workspace_size(PRISM_WS_BWD, col_capacity)
 *                         (head_dim 128 adds fp16 copies of V and dO and an
 *                         fp32 dQ accumulator: heads * N * 128 * 8 bytes)
 * head_dim 128 on the tensor cores runs one kernel per key tile that forms dK,
 * dV and each query tile's part of dQ, summed into the fp32 accumulator by
 * atomic reductions: dQ may then differ run to run in its last bits (the order
 * of the fp32 additions is not fixed); dK and dV are reproducible.  Its
 * dP and dV products take fp16 copies of V and dO scaled per head by powers
 * of two (exact for bf16 inputs; entries of magnitude 2^75 or more are outside
 * that range), the others bf16.  It needs O
 * and lse from the tensor-core forward, whose truncated fp16 probabilities it
 * reproduces (the rows of dS then sum to zero as they do in exact arithmetic).
 */
int prism_bsa_bwd(const prism_params *p, const prism_block *blocks, const int32_t *zone_blk_base,
                  const int32_t *nblk, const void *q, const void *k, const void *v, const void *o,
                  const void *o_res, const void *dout, const float *lse, const int32_t *row_ptr, const int32_t *col,
                  const int64_t *nnz, int64_t col_capacity, void *dq, void *dk, void *dv,
                  void *workspace, size_t ws_bytes, prism_stream stream);

/* Process-wide options (host-only; set while no call is in flight).
 *   PRISM_OPT_ATTN_BACKEND  0 (default): tcgen05/TMEM/TMA attention kernels for
 *                           head_dim 128, warp-level MMA kernels otherwise;
 *                           1: warp-level MMA kernels always (cross-checking).
 *   PRISM_OPT_WAIT_LIMIT    polls before a device-side wait gives up and
 *                           latches PRISM_ETIMEOUT; 0 restores the default.
 *   PRISM_OPT_DEBUG_STALL   test hook: when 1 the forward kernel never signals
 *                           its first probability tile (nor the tensor-core
 *                           backward its first P^T tile), so a bounded wait
 *                           must time out (PRISM_ETIMEOUT), with no trap or hang.
 * Returns PRISM_EINVAL for an unknown option. */
#define PRISM_OPT_ATTN_BACKEND 0
#define PRISM_OPT_WAIT_LIMIT 1
#define PRISM_OPT_DEBUG_STALL 2
int prism_set_option(int option, int64_t value);

/* Kernel-launch trace hook.  When set, the library calls
 *   fn(user, kernel_name, 0, stream) just before and
 *   fn(user, kernel_name, 1, stream) just after
 * every kernel it launches, on the calling thread, so that a caller can
 * record CUDA events around each kernel and count launches.  NULL disables.
 * The hook is process-wide; set it while no other thread is calling in. */
typedef void (*prism_trace_fn)(void *user, const char *kernel, int end, prism_stream stream);
int prism_set_trace(prism_trace_fn fn, void *user);

/* Synchronises `stream`, returns the latched device status (PRISM_OK or one
 * of PRISM_ECAPACITY / PRISM_ETIMEOUT / PRISM_EBOUNDS) and clears it. */
int prism_device_status(prism_stream stream);

/* Message for the last non-zero status returned to the calling thread. */
const char *prism_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* PRISM_H */
