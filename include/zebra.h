/*
 * zebra.h — C ABI of the Zebra3D multi-view global-attention library (sm_100a).
 *
 * Source of the method: the page "How Hybrid Attention Lets Feed-Forward 3D
 * Models Scale to Many Views" (wispaper.ai), sections
 *   "Linear-centered stages plus tile-sparse stages"   (tile-sparse stage, xL/yS)
 *   "A closed-form fit avoids retraining from scratch"  (centered affine correction)
 *   "Speedup scales with the number of input views"     (fused Q/K normalisation,
 *       positional rotation and channel-softmax feature map; tile-major K/V packing)
 *
 * Token layout (all entry points). A layer sees V views; view v holds
 * L = n_special + grid_h*grid_w tokens at token indices [v*L, (v+1)*L): first the
 * n_special special tokens (camera, registers), then the patch grid in row-major
 * order. Tokens are tiled per view into 8x8 patch blocks anchored at grid (0,0);
 * bottom/right edge tiles are partial. Tile index
 *   u = v*T_v + (row/8)*ceil(grid_w/8) + col/8,  T_v = ceil(grid_h/8)*ceil(grid_w/8),
 * T = V*T_v tiles in all. Inside a tile, tokens are numbered row-major, 0..n_u-1.
 *
 * Q, K, V and outputs are [N, H, d] tensors: element (n, h, c) of a tensor with
 * layout {tok_stride, head_stride} sits at ptr[n*tok_stride + h*head_stride + c]
 * (strides in elements; channels contiguous). A NULL layout means contiguous
 * [N, H, d] (tok_stride = H*d, head_stride = d). Outputs are always contiguous.
 *
 * Conventions.
 *  - Ownership: the caller owns every buffer; all data pointers are DEVICE
 *    pointers unless stated. The library allocates and frees no memory; scratch
 *    comes from the caller's workspace (size: zebra_workspace_bytes; base
 *    256-byte aligned, as cudaMalloc returns).
 *  - Streams: each call enqueues its kernels on `stream` (a cudaStream_t passed
 *    as void*; NULL = legacy default stream) and returns without synchronising.
 *  - Errors: argument errors return a nonzero status before anything is enqueued;
 *    zebra_last_error() then describes the failure (thread-local). Launch errors
 *    return ZEBRA_ERR_CUDA. Device-side failures (a bounded wait that ran out,
 *    a failed numerical check) set a sticky device status word, read by
 *    zebra_sync_status().
 *  - Inputs are never modified. Outputs are written completely.
 */
#ifndef ZEBRA_H
#define ZEBRA_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define ZEBRA_API __attribute__((visibility("default")))
#else
#define ZEBRA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Status codes returned by every int-valued entry point. */
#define ZEBRA_OK 0
#define ZEBRA_ERR_INVALID_ARG 1   /* null pointer, bad size, y outside [0,1), ... */
#define ZEBRA_ERR_UNSUPPORTED 2   /* d != 64, tile != 8, too many tiles, no sm_100 device */
#define ZEBRA_ERR_WORKSPACE 3     /* workspace smaller than zebra_workspace_bytes() or not 256-byte aligned */
#define ZEBRA_ERR_CUDA 4          /* a CUDA runtime or cuBLASLt call failed */
#define ZEBRA_ERR_TIMEOUT 5       /* a device-side bounded wait gave up (sticky) */
#define ZEBRA_ERR_NUMERIC 6       /* a device-side numerical check failed (sticky): the affine
                                     fit's system was not positive definite */

/* Element types of Q/K/V/out. bf16 is the production type; fp32 is accepted
 * by the stage entry points for small, CPU-checkable runs. */
typedef enum { ZEBRA_F32 = 0, ZEBRA_BF16 = 1 } zebra_dtype;

/* Layer geometry. Constraints: views >= 0, grid_h >= 1, grid_w >= 1,
 * 0 <= n_special <= 64, tile == 8, heads >= 1, head_dim == 64. */
typedef struct zebra_geom {
  int32_t views;
  int32_t grid_h;
  int32_t grid_w;
  int32_t n_special;
  int32_t tile;
  int32_t heads;
  int32_t head_dim;
} zebra_geom;

/* Strides (in elements) of a strided [N, H, d] input. */
typedef struct zebra_layout {
  int64_t tok_stride;
  int64_t head_stride;
} zebra_layout;

/* Layer kinds of zebra_hybrid_layer ("xL/yS" allocation, section
 * "Linear-centered stages plus tile-sparse stages"). */
#define ZEBRA_LAYER_LINEAR 0
#define ZEBRA_LAYER_SPARSE 1
#define ZEBRA_LAYER_DENSE 2

/* Operation ids of zebra_workspace_bytes. */
#define ZEBRA_OP_SELECT 0
#define ZEBRA_OP_SPARSE 1
#define ZEBRA_OP_LINEAR 2
#define ZEBRA_OP_HYBRID_LINEAR 3
#define ZEBRA_OP_HYBRID_SPARSE 4
#define ZEBRA_OP_HYBRID_DENSE 5
#define ZEBRA_OP_AFFINE 6         /* zebra_affine_moments */

/* Number of kept key tiles per query tile for sparsity y in [0,1):
 * k = clamp(ceil((1-y)*T - 1e-6), 1, T) — the selector "retains a key-tile
 * fraction of 1 minus y" (section "Linear-centered stages plus tile-sparse
 * stages"); the ceiling and the 1e-6 guard are this library's reading.
 * Returns -1 for y outside [0,1) or n_tiles < 1. Host only, no CUDA call. */
ZEBRA_API int32_t zebra_keep_count(double y, int32_t n_tiles);

/* Tile pooling and tile-major packing (sections "Linear-centered stages plus
 * tile-sparse stages": omitted tiles become mean key/value landmarks; "Speedup
 * scales with the number of input views": K/V packed in tile-major order).
 *   x           [N, H, d] of type dt, strided by `layout` (NULL = contiguous)
 *   x_mean      out [H, T, d] fp32: mean of each tile's n_u actual tokens (required)
 *   x_packed    out [H, T, 64, d] of type dt, or NULL: tile u's tokens in row-major
 *               tile order at rows 0..n_u-1, rows n_u..63 zero
 *   tile_counts out [T] int32 n_u, or NULL
 * T = 0 (views == 0) is a no-op. */
ZEBRA_API int zebra_tile_pool(const zebra_geom* g, zebra_dtype dt, const void* x, const zebra_layout* layout,
                    float* x_mean, void* x_packed, int32_t* tile_counts, void* stream);

/* Per-query-tile key-tile selector (section "Linear-centered stages plus
 * tile-sparse stages"). Scores key tile u for query tile t by the dot
 * q_mean[h,t] . k_mean[h,u] over all T tiles (own tile included), to fp32
 * accuracy (tensor cores on the means' bf16 parts, fp32 accumulation; equal
 * key means give equal scores), and keeps the top k = zebra_keep_count(y, T);
 * equal scores go to the lower tile index.
 *   q_mean, k_mean [H, T, d] fp32 (from zebra_tile_pool)
 *   mask      out [H, T, W] uint32, W = ceil(T/32): bit (u%32) of word u/32 of
 *             row (h, t) is set iff key tile u is kept for query tile t
 *   near_tie  out [H, T] uint8 or NULL: 1 where the k-th and (k+1)-th scores
 *             differ by a relative gap < 1e-5 (0 when k == T)
 *   k_out     HOST int32 out or NULL: the keep count
 *   workspace device scratch of zebra_workspace_bytes(g, ZEBRA_OP_SELECT, ..) bytes
 * Requires T <= 49152. */
ZEBRA_API int zebra_tile_select(const zebra_geom* g, const float* q_mean, const float* k_mean, double y,
                      uint32_t* mask, uint8_t* near_tie, int32_t* k_out,
                      void* workspace, size_t ws_bytes, void* stream);

/* Tile-sparse softmax attention of one layer (section "Linear-centered stages
 * plus tile-sparse stages"). Per head, a patch query of tile t attends with
 * scale 1/sqrt(d):
 *   - every token of each kept key tile, exactly;
 *   - every special-token key, exactly;
 *   - its own key exactly, when its own tile t is not kept;
 *   - one landmark per other unkept tile u: key = mean K, value = mean V of the
 *     tile's tokens, logit q.k_mean/sqrt(d) + ln(m), m = n_u; for the own tile
 *     (when unkept) the landmark covers its n_t - 1 other tokens (omitted if 0).
 * Special-token queries attend all N keys densely.
 *   q, k, v   [N, H, d] of type dt, strided by `layout` (NULL = contiguous)
 *   y         sparsity in [0,1); y = 0 keeps every tile (dense attention)
 *   mask      [H, T, W] selection from zebra_tile_select, or NULL to select here
 *   out       [N, H, d] of type dt, contiguous
 *   workspace zebra_workspace_bytes(g, ZEBRA_OP_SPARSE, dt, y) bytes
 * In bf16 the patch rows go out as ceil(T*H / (4 * SMs)) kernel launches of
 * one resident wave each, all on `stream` (each becomes a node when the call
 * is captured into a CUDA graph). Requires T*H*64 < 2^31 (ZEBRA_ERR_UNSUPPORTED
 * otherwise) and, without a mask, T <= 49152. */
ZEBRA_API int zebra_sparse_attn(const zebra_geom* g, zebra_dtype dt, const void* q, const void* k, const void* v,
                      const zebra_layout* layout, double y, const uint32_t* mask, void* out,
                      void* workspace, size_t ws_bytes, void* stream);

/* Linear global attention with the per-head centered affine correction
 * (sections "Speedup scales with the number of input views" and "A closed-form
 * fit avoids retraining from scratch"). Per head h and token n:
 *   f(x) = phi(rope2d(x / sqrt(mean(x^2) + eps))), phi = softmax over the d channels,
 *   rope2d turns channel pairs (j, j+16) of channels 0-31 by patch row * base^(-j/16)
 *   and of channels 32-63 by patch column * base^(-j/16); special tokens unrotated;
 *   S = sum_m f(k_m) v_m^T (d x d), z = sum_m f(k_m), over all N tokens;
 *   out_n = A_h (S^T f(q_n) / (z . f(q_n))) + b_h.
 *   A    [H, d, d] fp32 row-major (A[h][i][j] multiplies o_j into y_i), or NULL = identity
 *   b    [H, d] fp32, or NULL = zero
 *   out  [N, H, d] of type dt, contiguous
 *   workspace zebra_workspace_bytes(g, ZEBRA_OP_LINEAR, dt, 0) bytes */
ZEBRA_API int zebra_linear_attn(const zebra_geom* g, zebra_dtype dt, const void* q, const void* k, const void* v,
                      const zebra_layout* layout, const float* A, const float* b, float rope_base,
                      float eps, void* out, void* workspace, size_t ws_bytes, void* stream);

/* The linear stage of zebra_linear_attn (same arguments and checks) for
 * callers that cannot allocate device memory: code whose device memory is
 * owned by another framework's allocator or a fixed reservation (so a
 * cudaMalloc of a workspace would fail or fragment it), latency-critical paths
 * that must not risk an allocation stalling the device, and thin C or FFI
 * clients with no allocator at hand. The paper has no counterpart of this
 * entry point; it only changes where the scratch memory comes from.
 * Scratch: a built-in device array of 16 MiB (every GPU that loads the
 * library holds it until the process exits); no cudaMalloc, cudaFree or
 * allocating library routine is called. Geometries whose per-head state and
 * one chunk's partials do not fit in it return ZEBRA_ERR_UNSUPPORTED (at 16
 * heads any token count fits). The token chunks are those of
 * zebra_linear_attn while their partials fit (at 16 heads: up to 124,928
 * tokens), and then the result is bit-identical to it; beyond that the chunks
 * grow to fit, and the result differs from zebra_linear_attn only by the order
 * of the fp32 sums. The first call on a device looks up the array's device
 * address (cudaGetSymbolAddress) and caches it; make that first call before
 * any stream capture. cudaDeviceReset invalidates the cached address: do not
 * call this entry point after a reset. Every call uses the same array, so
 * calls that overlap on the GPU (e.g. on two streams) race; serialise them.
 * Nothing in the array has to start at zero: each call overwrites what it
 * reads. */
ZEBRA_API int zebra_linear_attn_noalloc(const zebra_geom* g, zebra_dtype dt, const void* q, const void* k,
                                        const void* v, const zebra_layout* layout, const float* A, const float* b,
                                        float rope_base, float eps, void* out, void* stream);

/* One stacked global-attention layer, bf16 only (section "Linear-centered
 * stages plus tile-sparse stages": preserved QKV/output projections,
 * normalisation and positional encoding):
 *   x_out = x + concat_heads(Attn(Q, K, V)) W_o^T,  [Q|K|V] = x W_qkv^T,
 * where Attn is the linear stage (kind ZEBRA_LAYER_LINEAR, with A, b), or the
 * tile-sparse stage at sparsity y (ZEBRA_LAYER_SPARSE), or dense softmax
 * attention (ZEBRA_LAYER_DENSE); the sparse and dense kinds first apply the
 * RMS norm and 2D rotation of zebra_linear_attn to Q and K.
 *   x      [N, D] bf16, D = heads*head_dim
 *   w_qkv  [3D, D] bf16 row-major; w_o [D, D] bf16 row-major
 *   x_out  [N, D] bf16 (may equal x)
 *   workspace zebra_workspace_bytes(g, ZEBRA_OP_HYBRID_*, ZEBRA_BF16, y) bytes */
ZEBRA_API int zebra_hybrid_layer(const zebra_geom* g, int kind, const void* x, const void* w_qkv, const void* w_o,
                       const float* A, const float* b, double y, float rope_base, float eps, void* x_out,
                       void* workspace, size_t ws_bytes, void* stream);

/* Workspace bytes needed by operation `op` (ZEBRA_OP_*) for this geometry,
 * element type and sparsity. Returns 0 and sets the last error on an invalid
 * geometry or op. Host only. */
ZEBRA_API size_t zebra_workspace_bytes(const zebra_geom* g, int op, zebra_dtype dt, double y);

/* Description of the last error of the calling thread ("" if none). */
ZEBRA_API const char* zebra_last_error(void);

/* Synchronises `stream`, then reads and clears the device status words of the
 * current device. Returns ZEBRA_OK, ZEBRA_ERR_TIMEOUT, ZEBRA_ERR_NUMERIC or
 * ZEBRA_ERR_CUDA. */
ZEBRA_API int zebra_sync_status(void* stream);

/* Test hook of the error path (no counterpart in the paper; for tests of the
 * library only). On the current device it sets the limit of every bounded
 * wait of the bf16 sparse attention kernel to `wait_ns` nanoseconds (0 = the
 * default of 2 s) and, when `block` >= 0, makes that kernel's copy producer
 * stop before the block of index `block` of each query tile's block stream,
 * so that the tensor-core warp's wait for that block's keys runs out: the
 * kernel then records ZEBRA_ERR_TIMEOUT in the sticky status word, lets its
 * copies and MMAs in flight land (each wait bounded again), frees its tensor
 * memory and exits, leaving the outputs of the affected rows undefined. The
 * same call sets the wait limit of the bf16 linear stage's state kernel and,
 * when `block` >= 0, makes it leave out the tensor-core MMAs of block `block`
 * (64 tokens) of each token chunk, so that its wait for their completion runs
 * out the same way (the stage's outputs are then undefined).
 * zebra_sync_status() reports the timeout. zebra_debug_inject(-1, 0) restores
 * normal operation. Every wait stays bounded, so no setting can hang the GPU.
 * Returns ZEBRA_OK, ZEBRA_ERR_CUDA or ZEBRA_ERR_UNSUPPORTED (no sm_100 device). */
ZEBRA_API int zebra_debug_inject(int32_t block, uint64_t wait_ns);

/* Number of kernels this library has launched in this process (all devices). */
ZEBRA_API uint64_t zebra_launch_count(void);

/* ---------------------------------------------------------------------------
 * Closed-form centred affine fit of the linear stage's output correction.
 *
 * Section "A closed-form fit avoids retraining from scratch": teacher (dense
 * softmax) outputs and converted linear outputs are accumulated across scenes,
 * tokens, heads and views, and a centred affine correction is fitted by a
 * regularised least-squares solve in float64. One sample is the pair (x, y) of
 * 64-vectors at one (token, head): x the linear stage's output before the
 * correction (zebra_linear_attn with A = b = NULL), y the teacher's output.
 * Samples of all heads are pooled into one fit (per_head = 0), or each head is
 * fitted on its own (per_head = 1).
 *
 * `moments` (device, float64, caller-owned) holds, per group (1 group pooled,
 * H groups per head), ZEBRA_AFFINE_GROUP_DOUBLES values in this order: the
 * sample count, sum x [64], sum y [64], sum x x^T [64 x 64, row-major],
 * sum x y^T [64 x 64, row-major; entry (i, j) = sum x_i y_j], sum |y|^2 [1].
 * Zero it before the first call of a fit; each zebra_affine_moments call (one
 * scene) adds its samples. The additions are deterministic (fixed order).
 * ------------------------------------------------------------------------- */
#define ZEBRA_AFFINE_GROUP_DOUBLES 8322

/* Adds the moments of the samples x, y ([N, H, 64] of dtype dt, both with
 * `layout`, NULL = contiguous) to `moments`.
 *   workspace  device scratch of zebra_workspace_bytes(g, ZEBRA_OP_AFFINE, ..)
 *              bytes (per-CTA partial moments)
 * Errors: ZEBRA_ERR_INVALID_ARG (null or misaligned pointers, bad strides),
 * ZEBRA_ERR_WORKSPACE, ZEBRA_ERR_CUDA. */
ZEBRA_API int zebra_affine_moments(const zebra_geom* g, zebra_dtype dt, const void* x, const void* y,
                                   const zebra_layout* layout, int per_head, double* moments, void* workspace,
                                   size_t ws_bytes, void* stream);

/* Solves the centred ridge fit of every group of `moments`:
 *   mu_x = sum x / n, mu_y = sum y / n,
 *   C_xx = sum x x^T / n - mu_x mu_x^T,  C_xy = sum x y^T / n - mu_x mu_y^T,
 *   A^T = (C_xx + lam I)^-1 C_xy (Cholesky, float64),  b = mu_y - A mu_x,
 * and writes A [H, 64, 64] and b [H, 64] as float32, the layout
 * zebra_linear_attn takes (the same A, b for every head when pooled).
 * lam >= 0 (the page gives no value). If C_xx + lam I is not positive definite
 * or a group holds no sample, that group's A and b are NaN and
 * zebra_sync_status() returns ZEBRA_ERR_NUMERIC.
 * Errors: ZEBRA_ERR_INVALID_ARG (null pointers, lam < 0 or not finite). */
ZEBRA_API int zebra_affine_solve(const zebra_geom* g, const double* moments, int per_head, double lam, float* A,
                                 float* b, void* stream);

/* Attention-concentration diagnostic (section "Sensitive stages also
 * concentrate their attention": the stages that resist linear conversion are
 * the ones whose attention mass is concentrated). For every row of the sampled
 * patch query tiles and every head, dense softmax attention over all N keys
 * (scale 1/sqrt(d)) is evaluated, and its mass is split into
 *   selected_mass  the sum of the probabilities of the tokens of the key tiles
 *                  that `mask` keeps for the row's tile (what the sparse
 *                  stage keeps exact), and
 *   special_mass   the sum over the special-token keys.
 *   q, k          [N, H, d] bf16, strided by `layout` (NULL = contiguous);
 *                 ZEBRA_ERR_UNSUPPORTED for other types
 *   mask          [H, T, W] selection (zebra_tile_select)
 *   query_tiles   HOST [n_query_tiles] int32 tile indices in [0, T),
 *                 1 <= n_query_tiles <= 1024
 *   selected_mass, special_mass  out [n_query_tiles, H, 64] fp32: entry
 *                 (i, h, a) for row a (row-major inside the tile) of tile
 *                 query_tiles[i]; rows a >= n_t of a partial tile are 0
 *   workspace     zebra_coverage_workspace_bytes(g, n_query_tiles) bytes
 * Deterministic (fixed-order combines). */
ZEBRA_API int zebra_coverage(const zebra_geom* g, zebra_dtype dt, const void* q, const void* k,
                             const zebra_layout* layout, const uint32_t* mask, const int32_t* query_tiles,
                             int32_t n_query_tiles, float* selected_mass, float* special_mass, void* workspace,
                             size_t ws_bytes, void* stream);
/* Workspace bytes of zebra_coverage (0 and an error message for invalid
 * arguments). Host only. */
ZEBRA_API size_t zebra_coverage_workspace_bytes(const zebra_geom* g, int32_t n_query_tiles);

/* Single-stage linear-conversion error (section "Linear-centered stages plus
 * tile-sparse stages": stages are ranked by the error of converting them
 * alone to linear attention). For every group of `moments` (accumulated by
 * zebra_affine_moments; 1 group pooled, H per head) writes
 *   err[g] = mean over the group's samples of |A x + b - y|^2
 *          = (tr(A Sxx A^T) + 2 b.(A sx) - 2 tr(A Sxy) + n|b|^2 - 2 b.sy + sum|y|^2) / n
 * in float64, with A, b the correction of zebra_affine_solve's layout
 * ([H, 64, 64] and [H, 64] fp32; a pooled group uses head 0's). An empty group
 * gives NaN. err: device, float64, one value per group.
 * Errors: ZEBRA_ERR_INVALID_ARG (null or misaligned pointers). */
ZEBRA_API int zebra_affine_residual(const zebra_geom* g, const double* moments, int per_head, const float* A,
                                    const float* b, double* err, void* stream);

/* Layer allocation for a linear fraction x (section "Linear-centered stages
 * plus tile-sparse stages": the xL/yS setting converts the fraction x of
 * stages with the lowest single-stage linear-conversion error to linear
 * attention and the rest to tile-sparse attention). Host only, no CUDA call.
 *   errors     HOST [n_layers] float64 (e.g. from zebra_affine_residual)
 *   is_linear  HOST out [n_layers] int32: 1 = linear, 0 = sparse
 * The count is floor(x * n_layers + 1/2); layers are ranked by error with
 * ties (and NaN errors, which rank last) in index order. Returns the count,
 * or -1 for n_layers < 0, x outside [0, 1] or a null pointer with
 * n_layers > 0. */
ZEBRA_API int32_t zebra_allocate_layers(const double* errors, int32_t n_layers, double linear_fraction,
                                        int32_t* is_linear);

/* Optional per-kernel timing. zebra_profile_enable(1) clears the record and
 * from then on brackets every kernel this library launches (or, for the sparse
 * attention kernel, the sequence of launches of one call) with two CUDA events
 * on the launching stream; it also zeroes the device counters of visible
 * attention logits. zebra_profile_enable(0) stops recording. Returns a status. */
ZEBRA_API int zebra_profile_enable(int on);

/* Waits for the recorded events and writes a text report into buf (at most len
 * bytes, NUL-terminated): one line "kernel <name> <records> <total ms>
 * <launches>" per kernel name in first-launch order (records = bracketed
 * intervals, launches = kernel launches inside them), then
 * "logits sparse_rows <n>" and
 * "logits special_rows <n>", the number of unmasked query-key logits the
 * attention kernels evaluated (4*d FLOPs each: QK^T and PV). Returns the full
 * report length. Host pointer. */
ZEBRA_API long long zebra_profile_report(char* buf, size_t len);

/* Library version string. */
ZEBRA_API const char* zebra_version(void);

#ifdef __cplusplus
}
#endif

#endif /* ZEBRA_H */
