/*
 * gs.h -- C ABI of the B200 (sm_100a) differentiable EWA Gaussian-splatting
 * library (libgs_b200.so).
 *
 * The calls follow the pipeline the pages state: project the 3D Gaussians,
 * assign them to tiles and depth-sort, blend per pixel, and differentiate it
 * ("Better Gaussian Splatting in Julia", pwwt.cn, sec. 3.2-3.3 and 5.4; the
 * second Julia page, lshu.cn, sec. 3.2 `rasterize` pseudocode and sec. 1
 * capability table), accumulate the plain and absolute view-space gradients
 * used for densification (jsqmd.com, sec. 2 table and sec. 3.1), and take one
 * Adam step over every parameter (lshu.cn sec. 3.3 and 5.3).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - Every array argument is a DEVICE pointer owned by the caller, except the
 *    camera array, the background colour and the Adam group table, which are
 *    HOST pointers read before the call returns. The library never allocates
 *    or frees device memory and keeps no state between calls.
 *  - `stream` is a cudaStream_t passed as void* (NULL = legacy default
 *    stream). Every call only enqueues work on that stream and returns
 *    without synchronising, except gs_get_status.
 *  - Argument errors are detected on the host before anything is enqueued and
 *    returned at once (GS_ERR_INVALID_ARG, GS_ERR_OVERFLOW). A failed launch
 *    returns GS_ERR_CUDA. Conditions only the device can see are OR-ed into
 *    the status word at the start of a workspace (the GS_STATUS_BIT_* bits
 *    below) and read back by gs_get_status: pair capacity exceeded, a
 *    bounded wait that gave up, an index or range out of bounds (clipped,
 *    never dereferenced), a Gaussian culled for non-finite values. The calls
 *    with a device wait or an index to check (gs_project, gs_bin_sort,
 *    gs_rasterize_fwd, gs_rasterize_bwd) take that workspace; the
 *    gs_bin_sort workspace serves all of them.
 *  - Pixel (x, y) has its centre at (x + 0.5, y + 0.5); tiles are 16 x 16
 *    pixels; tile index within a view is ty * tiles_x + tx, and the global
 *    tile index of view v is v * tiles_per_view + tile.
 *  - All views of one call share width and height.
 */
#ifndef GS_B200_H
#define GS_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define GS_ABI_VERSION 4
#define GS_TILE 16            /* tile edge in pixels */
#define GS_MAX_VIEWS 32       /* views per call */
#define GS_RECORD_FLOATS 16   /* floats per projected record */
#define GS_GRAD2D_FLOATS 12   /* floats per screen-space gradient record */
#define GS_MAX_PAIR_CAPACITY ((int64_t)1 << 31) /* pair positions are 32-bit */

/* Bits of the device status word (the first 4 bytes of a workspace). */
#define GS_STATUS_BIT_CAPACITY 1u   /* more pairs than pair_capacity: nothing emitted */
#define GS_STATUS_BIT_TIMEOUT 2u    /* a bounded device-side wait gave up */
#define GS_STATUS_BIT_BOUNDS 4u     /* an index or range out of bounds was clipped */
#define GS_STATUS_BIT_NONFINITE 8u  /* a Gaussian with a non-finite value was culled */

typedef enum gs_status {
  GS_OK = 0,
  GS_ERR_INVALID_ARG = 1,     /* bad pointer, size, degree, view count, layout */
  GS_ERR_CAPACITY = 2,        /* more Gaussian x tile pairs than pair_capacity */
  GS_ERR_OVERFLOW = 3,        /* a size exceeds a 32-bit field it must fit */
  GS_ERR_DEVICE_TIMEOUT = 4,  /* a bounded device-side wait gave up */
  GS_ERR_NONFINITE = 5,       /* a Gaussian with a non-finite parameter or colour was culled */
  GS_ERR_CUDA = 6             /* a CUDA runtime call or launch failed */
} gs_status;

/* Sort strategy of gs_bin_sort; both give bit-identical per-tile lists. */
typedef enum gs_sort_mode {
  /* Emit one 64-bit key (global tile << 32 | float bits of depth) per
   * Gaussian x tile pair and radix-sort the keys (least significant digit
   * first, 8-bit digits, single-sweep passes). */
  GS_SORT_FULL64 = 0,
  /* Radix-sort the Gaussians of each view once by (view << 32 | depth bits),
   * emit the pairs in that order, then radix-sort the pairs stably by global
   * tile alone. Same order as FULL64, fewer bytes per pair. */
  GS_SORT_PRESORT = 1
} gs_sort_mode;

/* Pinhole camera (lshu.cn sec. 3.2: "camera intrinsics and extrinsics").
 * viewmat: row-major 3x4 [R | t] mapping world to camera coordinates
 * (x right, y down, z forward). u = fx * x / z + cx, v = fy * y / z + cy.
 * campos: camera centre in world coordinates (origin of the SH view
 * direction). 88 bytes. */
typedef struct gs_camera {
  float viewmat[12];
  float fx, fy, cx, cy;
  int32_t width, height;
  float campos[3];
  float reserved;
} gs_camera;

/* Raw (un-activated) Gaussian parameters, structure of arrays
 * (pwwt.cn sec. 1.1 and 3.1; lshu.cn sec. 3.1 table):
 *   means          float [n][4]  x, y, z, (pad, ignored)
 *   log_scales     float [n][4]  log of the per-axis scale, (pad, ignored)
 *   quats          float [n][4]  rotation quaternion w, x, y, z (normalised
 *                                inside; need not be unit)
 *   opacity_logit  float [n]     opacity = sigmoid(logit)
 *   sh             float [n][(sh_degree+1)^2][3]  real SH colour coefficients
 *   sh_quant       the same coefficients as quantised codes (gs_sh_quant,
 *                  below) instead: exactly one of sh and sh_quant is
 *                  non-NULL. The calls that read the coefficients
 *                  (gs_project, gs_project_bwd, gs_rasterize_bwd with
 *                  gradients) then decode each code where they use it, to the
 *                  float gs_sh_dequantize would give, so their results equal
 *                  those of the float path on the decoded SH bit for bit;
 *                  sh_quant->n must equal n and sh_quant->k3 3 (sh_degree+1)^2.
 * The float4 arrays must be 16-byte aligned. */
struct gs_sh_quant;
typedef struct gs_params {
  const float* means;
  const float* log_scales;
  const float* quats;
  const float* opacity_logit;
  const float* sh;
  int32_t sh_degree;  /* 0..3 */
  int32_t reserved;
  int64_t n;          /* number of Gaussians, 0 <= n < 2^31 */
  const struct gs_sh_quant* sh_quant;
} gs_params;

/* Gradients of the raw parameters: same layouts as gs_params (pad lanes are
 * written as 0). Overwritten, not accumulated, by gs_rasterize_bwd. */
typedef struct gs_grads {
  float* means;
  float* log_scales;
  float* quats;
  float* opacity_logit;
  float* sh;
} gs_grads;

/* Output of gs_project, per view v and Gaussian i (record index v*n + i):
 * records [n_views][n][16] floats, 16-byte aligned (what the rasteriser reads).
 * The 2D Gaussian (mean (u, v), conic = inverse 2D covariance, opacity o) is
 * stored in the form the rasteriser evaluates, every field computed in double
 * precision and rounded to float once:
 *   0 uh      1 vh       u and v rounded to float
 *   2 w1x     3 w1y      rows of the 2x2 matrix W = diag(k1, k2) E^T, E the
 *   5 w2x     6 w2y      unit eigenvectors of the 2D covariance (largest
 *                        eigenvalue lambda1 first), k_i = sqrt(log2(e) / (2
 *                        lambda_i)); W^T W = (log2(e) / 2) conic
 *   4 c1      7 c2       c_i = -(w_i . (u - uh, v - vh)) with the float rows:
 *                        the part of the mean below float precision
 *   8 nlo                -log2(255 o)
 *   9 r  10 g  11 b      colour
 *  12 hx     13 hy       half-widths of a box around the ellipse where
 *                        alpha >= 1/255 (q <= Q = 2 ln(255 o)): sqrt(Qp
 *                        cov_xx) + 0.01 and sqrt(Qp cov_yy) + 0.01 with
 *                        Qp = Q + 0.002 |Q| + 1e-4; -1 when Qp <= 0
 *  14 o                  activated opacity
 *  15 zero
 * For the pixel centre P and d = P - (uh, vh), p_i = w_i . d + c_i and
 * zq = p1^2 + p2^2 + nlo equal (log2(e)/2) q - log2(255 o) with
 * q = (P - mean)^T conic (P - mean): alpha_raw = o exp(-q/2) = 2^-zq / 255,
 * and alpha_raw >= 1/255 exactly when zq <= 0. (The eigen form is a sum of
 * squares, so it keeps its relative accuracy for elongated splats, where the
 * conic form a dx^2 + 2 b dx dy + c dy^2 loses it to cancellation.)
 * bins [n_views][n][4] floats, 16-byte aligned (what the binning reads):
 *   0 depth key: camera-space z as the float fma chain
 *     fma(W20, x, fma(W21, y, fma(W22, z, t2))) of the float inputs
 *   1 tile_x  (bits) tx0 | tx1 << 16   inclusive tile range touched
 *   2 tile_y  (bits) ty0 | ty1 << 16   (tx0 > tx1 marks a culled Gaussian)
 *   3 zero
 * radii [n_views][n] int32: ceil(3 sqrt(lambda_max)) of the 2D covariance,
 *   0 when culled (the densification visibility filter). */
typedef struct gs_projected {
  float* records;
  float* bins;
  int32_t* radii;
} gs_projected;

/* Output of gs_bin_sort.
 *   ids     uint32 [pair_capacity]  Gaussian index (within its view) of each
 *           pair, ordered by global tile, then depth key, then index
 *   ranges  int64 [n_views * tiles_per_view][2]  [start, end) of each tile's
 *           slice of ids (start == end for an empty tile)
 *   n_pairs int64 [1]  number of pairs (always written, also on overflow) */
typedef struct gs_binned {
  uint32_t* ids;
  int64_t* ranges;
  int64_t* n_pairs;
  int64_t pair_capacity;
} gs_binned;

/* One Adam parameter group (lshu.cn sec. 3.3 per-group learning rates). */
typedef struct gs_adam_group {
  float* param;
  const float* grad;
  float* exp_avg;     /* first moment m */
  float* exp_avg_sq;  /* second moment v */
  int64_t count;      /* floats in the group */
  float lr;
  float reserved;
} gs_adam_group;

/* ABI version of the loaded library (GS_ABI_VERSION). */
int32_t gs_abi_version(void);

/* Static text for a status code. */
const char* gs_status_string(gs_status status);

/* Bytes of workspace gs_bin_sort needs for n Gaussians, n_views views of
 * cams[0]'s size, pair_capacity pairs and the given sort mode. Returns 0 for
 * invalid arguments, pair_capacity above GS_MAX_PAIR_CAPACITY included. The
 * workspace must be 256-byte aligned; its first 256
 * bytes hold the device status word and counters; zero them once (e.g.
 * cudaMemset) before the workspace is first used. */
size_t gs_workspace_size(int64_t n, int32_t n_views, const gs_camera* cams,
                         int64_t pair_capacity, int32_t sort_mode);

/* How gs_bin_sort will order the pairs of a request (host only, no CUDA call):
 *   path             GS_PATH_TILE_ID (64-bit (tile, depth) keys in full-64
 *                    mode, or presorted pairs sorted by tile id),
 *                    GS_PATH_COLUMNS (presorted pairs emitted by tile column,
 *                    then sorted by row) or GS_PATH_TILES (presorted pairs
 *                    placed straight at their positions, no pair sort);
 *   presort_passes   radix passes over the per-Gaussian depth keys (0 in
 *                    full-64 mode);
 *   pair_passes      radix passes over the pair keys (0 on GS_PATH_TILES);
 *   pair_single_sweep  1 if those passes are single-sweep (one digit-count
 *                    kernel, then one kernel per pass: the 64-bit keys of
 *                    full-64 mode), 0 if reduce-then-scan (three kernels per
 *                    pass: the 32-bit keys of the other paths);
 *   ranges_from_counts  1 if the tile ranges come from per-tile pair counts
 *                    (a difference array of the rectangles' corners per
 *                    view, two kernels) rather than from a read of the
 *                    sorted keys, whose last pass then writes no keys:
 *                    GS_PATH_COLUMNS and full-64 mode on grids whose
 *                    (tiles_x + 1) (tiles_y + 1) counters fit 160 KiB;
 *   pair_key_bytes   bytes per pair key: 8 in full-64 mode, 4 on
 *                    GS_PATH_TILE_ID and on GS_PATH_COLUMNS when the ranges
 *                    are read off the keys (row << column bits | column);
 *                    on GS_PATH_COLUMNS with ranges_from_counts the keys are
 *                    the rows alone: 1 byte up to 256 rows (views x tile
 *                    rows), 2 up to 65536; 0 on GS_PATH_TILES (no keys);
 *   gaussians_per_block, blocks_per_view  the Gaussian blocks of
 *                    GS_PATH_TILES (0 otherwise).
 * Returns GS_ERR_INVALID_ARG for a request gs_workspace_size rejects. */
enum { GS_PATH_TILE_ID = 0, GS_PATH_COLUMNS = 1, GS_PATH_TILES = 2 };
typedef struct gs_sort_plan {
  int32_t path;
  int32_t presort_passes;
  int32_t pair_passes;
  int32_t gaussians_per_block;
  int32_t pair_single_sweep;
  int32_t ranges_from_counts;
  int64_t blocks_per_view;
  int32_t pair_key_bytes;
  int32_t reserved;
} gs_sort_plan;
gs_status gs_bin_sort_plan(int64_t n, int32_t n_views, const gs_camera* cams,
                           int32_t sort_mode, gs_sort_plan* plan);

/* EWA projection (pwwt.cn sec. 3.2 `project_gaussian`: world -> camera ->
 * pixel with division by depth, covariance through the Jacobian of that map;
 * lshu.cn sec. 3.2). Per view and Gaussian: R from the normalised quaternion,
 * Sigma = R diag(exp(2 s)) R^T, t = W mu + T, J = [[fx/z, 0, -fx x/z^2],
 * [0, fy/z, -fy y/z^2]], cov2d = J W Sigma W^T J^T + 0.3 I, conic = cov2d^-1,
 * radius = ceil(3 sqrt(lambda_max)), colour = max(0, sum_k Y_k(d) sh_k + 0.5)
 * with d = normalize(mu - campos), opacity = sigmoid(logit), tile rectangle
 * floor((u -+ radius)/16) clamped to the grid. Culled when z < 0.2, the 2D
 * covariance is not positive definite, or the rectangle is empty.
 * Geometry (camera-space mean, covariance, radius, rectangle, depth key) is
 * evaluated in double precision and rounded to float at the end; colour in
 * float. A Gaussian with a non-finite mean, log-scale, quaternion, logit or
 * colour (a non-finite SH coefficient), or a zero quaternion, is culled in
 * every view and its depth key marked; gs_bin_sort on those records raises
 * GS_ERR_NONFINITE in its status word (the rest of the frame is unaffected).
 * Writes out->records, out->bins and out->radii for all n_views * n records.
 * `ws` is a workspace (e.g. gs_bin_sort's) whose status word receives
 * GS_STATUS_BIT_TIMEOUT if the staging of a block's SH coefficients into
 * shared memory did not complete in time (the block then reads them from
 * global memory, so the output is still exact). */
gs_status gs_project(const gs_params* params, const gs_camera* cams, int32_t n_views,
                     gs_projected* out, void* ws, void* stream);

/* Tile binning with depth sort (pwwt.cn sec. 3.3 steps 1-2 and 4.3 tiles;
 * lshu.cn sec. 3.2 `assign_to_tiles` and `sort_by_depth!`). Every Gaussian
 * with a non-empty rectangle emits one pair per tile it touches; the pairs
 * are ordered by global tile, then by the float bits of its depth key, then
 * by Gaussian index (the order of a stable sort on the 64-bit key
 * tile << 32 | depth bits over pairs emitted in index order).
 * `n` is the per-view Gaussian count used by gs_project. `ws` must hold
 * gs_workspace_size(n, n_views, cams, out->pair_capacity, sort_mode) bytes.
 * If more than pair_capacity pairs are needed, nothing is emitted, n_pairs
 * still receives the count, every range is empty and GS_ERR_CAPACITY is
 * raised in the status word. */
gs_status gs_bin_sort(const gs_projected* proj, const gs_camera* cams, int32_t n_views,
                      int64_t n, int32_t sort_mode, gs_binned* out, void* ws,
                      size_t ws_bytes, void* stream);

/* Size of the fixed scratch array that gs_bin_sort_noalloc uses. */
#define GS_NOALLOC_SCRATCH_BYTES (32u << 20)

/* gs_bin_sort for callers that must not allocate device memory. (The pages
 * have no counterpart; this is a library convenience.) Some callers cannot
 * call cudaMalloc: code that runs inside a host application owning the
 * device's memory budget (a plug-in or an engine's render thread), or a loop
 * that cannot afford the device-wide synchronisation and the late
 * out-of-memory failure a fresh allocation can bring. This entry point takes
 * the same inputs and outputs as gs_bin_sort but no workspace: its scratch is
 * a fixed array of GS_NOALLOC_SCRATCH_BYTES inside the library, which every
 * GPU that uses this entry point holds from its first call until the process
 * exits (with eager module loading, CUDA_MODULE_LOADING=EAGER, every context
 * that loads the library holds it, whether or not it calls this entry
 * point). Each call looks up the array's device address on the current
 * device (cudaGetSymbolAddress, a host-side query), so the address stays
 * right after a cudaDeviceReset; make the first call on a device before any
 * stream capture. Requests whose gs_workspace_size exceeds GS_NOALLOC_SCRATCH_BYTES
 * are rejected with GS_ERR_INVALID_ARG before anything is enqueued. All calls
 * share the one array: calls whose work overlaps on the GPU (for example on
 * two streams) race and corrupt each other's results; serialise them.
 * Each call starts with a cleared status word; if `device_status` (a device
 * int32, may be NULL) is given, the call's device-side status bits (1 pair
 * capacity exceeded, 2 a bounded wait gave up, 4 an index out of range) are
 * copied there at the end, in stream order: the GS_STATUS_BIT_* bits (1 pair
 * capacity exceeded, 2 a bounded wait gave up, 4 an index or range out of
 * bounds was clipped, 8 a Gaussian culled for non-finite values was met). */
gs_status gs_bin_sort_noalloc(const gs_projected* proj, const gs_camera* cams, int32_t n_views,
                              int64_t n, int32_t sort_mode, gs_binned* out,
                              int32_t* device_status, void* stream);

/* Forward rasterisation, one 16x16 tile per thread block and one thread per
 * pixel (pwwt.cn sec. 5.4 tile mode; lshu.cn sec. 3.2 `blend`, sec. 7.3).
 * For each pixel, front to back over its tile's list:
 *   alpha = min(0.99, o exp(-q/2)), q = d^T conic d, d = pixel centre - mean;
 *   skip when alpha < 1/255; T' = T (1 - alpha); stop (without adding it)
 *   when T' < 1e-4; C += colour * alpha * T; T = T'.
 * Then C += T * bg[c]. Outputs (device):
 *   image     float [n_views][3][H][W]
 *   final_T   float [n_views][H][W]  transmittance after the last contributor
 *   n_contrib uint32 [n_views][H][W] 1 + position in the tile's list of the
 *             last contributing Gaussian (0 if none)
 *   warp_masks (optional, NULL skips it) uint8 [pair_capacity], by pair
 *             position: for every list entry the forward examined, bit w
 *             (0..3) set if the entry's alpha >= 1/255 ellipse reaches the
 *             tile's 8x8 pixel block w (blocks in row-major order within the
 *             tile); entries past a tile's early stop are not written.
 *             gs_rasterize_bwd reads it instead of testing every entry again.
 * `bg` is a host pointer to 3 floats. The test alpha_raw >= 1/255 is taken as
 * zq <= 0 on the record's evaluation form (see gs_projected) and alpha_raw
 * as 2^-zq / 255 with the SFU exp2. `ws` (device, 256-byte aligned, its
 * status word zeroed once, e.g. the gs_bin_sort workspace) receives
 * GS_STATUS_BIT_BOUNDS for a list entry naming a Gaussian >= n or a tile
 * range outside the ids buffer (the entry reads record 0 and reaches no
 * pixel; the range renders as empty), and GS_STATUS_BIT_TIMEOUT if a record
 * batch's copy into shared memory did not complete in time (that tile's
 * pixels keep what they had composited). */
gs_status gs_rasterize_fwd(const gs_projected* proj, const gs_binned* bins,
                           const gs_camera* cams, int32_t n_views, int64_t n,
                           const float* bg, float* image, float* final_T,
                           uint32_t* n_contrib, uint8_t* warp_masks, void* ws, void* stream);

/* Backward of gs_rasterize_fwd and gs_project (lshu.cn sec. 1
 * "differentiable rasterisation"). Given dL/dimage [n_views][3][H][W] and the
 * forward's final_T and n_contrib, replays each pixel's list back to front
 * and writes, per view and Gaussian, grad2d [n_views][n][12]:
 *   0 dL/du  1 dL/dv  2 dL/dconic_a  3 dL/dconic_b  4 dL/dconic_c
 *   5 dL/dopacity  6..8 dL/d(r, g, b)
 *   9 sum over pixels of ||(dL/du, dL/dv)|| (the absolute view-space
 *     gradient, jsqmd.com sec. 2 table)   10, 11 zero
 * (0 and 1 together are the view's plain view-space gradient), then the
 * gradients of the raw parameters summed over views into *grads
 * (overwritten; see gs_project_bwd). grad2d is overwritten. With
 * grads == NULL only grad2d is computed. warp_masks: NULL, or the forward's
 * (same binned lists and records): the backward then takes each entry's
 * block mask from it (the entries it replays all lie before the forward's
 * stop). `ws` as for gs_rasterize_fwd (the same conditions are reported; a
 * tile whose batch copy timed out adds nothing further to grad2d). */
gs_status gs_rasterize_bwd(const gs_params* params, const gs_projected* proj,
                           const gs_binned* bins, const gs_camera* cams, int32_t n_views,
                           const float* bg, const float* dL_dimage, const float* final_T,
                           const uint32_t* n_contrib, const uint8_t* warp_masks,
                           float* grad2d, gs_grads* grads, void* ws, void* stream);

/* Projection backward alone (the second half of gs_rasterize_bwd): the
 * gradients of the raw parameters from the screen-space gradients grad2d
 * [n_views][n][12] (fields 0..8 as written by gs_rasterize_bwd), summed over
 * the views in which radii[v][i] > 0, by the chain rule of gs_project:
 * conic -> 2D covariance -> (J W, R, scale) -> log-scale, quaternion (through
 * its normalisation), mean (through J and the pixel coordinates); colour ->
 * SH coefficients and, through the view direction, the mean; opacity ->
 * logit. *grads is overwritten. */
gs_status gs_project_bwd(const gs_params* params, const gs_camera* cams, int32_t n_views,
                         const int32_t* radii, const float* grad2d, gs_grads* grads,
                         void* stream);

/* The single-GPU training step's tail in one pass (lshu.cn sec. 3.3 Adam with
 * per-group learning rates; jsqmd.com sec. 2 densification statistics): the
 * projection backward of gs_project_bwd, then, instead of writing gradients,
 * the Adam step of gs_adam_step applied to every parameter of every Gaussian
 * (padding lanes included, with gradient 0) and the statistics of
 * gs_densify_stats, all from the values in registers. The parameters of
 * *params are updated IN PLACE (its arrays must be writable device memory);
 * exp_avg / exp_avg_sq are the moments in the gs_params layouts (updated);
 * lr[5] the learning rates of means, log-scales, quaternions, opacity logits
 * and SH; beta1, beta2, eps, step as gs_adam_step. accum_plain, accum_abs
 * (float [n]) and denom (int32 [n]) receive the statistics as
 * gs_densify_stats adds them; all three NULL skips them. Parameters, moments
 * and statistics equal those of gs_project_bwd + gs_densify_stats +
 * gs_adam_step over the same groups, bit for bit. Float SH only
 * (params->sh_quant NULL); the SH arrays of params, exp_avg and exp_avg_sq
 * 16-byte aligned. Argument errors as those calls. One launch. */
gs_status gs_project_bwd_adam(const gs_params* params, const gs_camera* cams, int32_t n_views,
                              const int32_t* radii, const float* grad2d, gs_grads* exp_avg,
                              gs_grads* exp_avg_sq, const float* lr, float beta1, float beta2,
                              float eps, int64_t step, float* accum_plain, float* accum_abs,
                              int32_t* denom, void* stream);

/* Densification statistics (jsqmd.com sec. 2 table and sec. 3.1
 * `add_densification_stats`): for each view v and Gaussian i with
 * radii[v][i] > 0, accumulate
 *   accum_plain[i] += ||(grad2d[v][i][0], grad2d[v][i][1])||,
 *   accum_abs[i]   += grad2d[v][i][9],
 *   denom[i]       += 1.
 * The three outputs accumulate across calls (the caller zeroes them). */
gs_status gs_densify_stats(const float* grad2d, const int32_t* radii, int32_t n_views,
                           int64_t n, float* accum_plain, float* accum_abs,
                           int32_t* denom, void* stream);

/* Adam step over up to 8 groups (lshu.cn sec. 3.3 and 5.3; Kingma and Ba):
 * m = b1 m + (1-b1) g; v = b2 v + (1-b2) g^2;
 * p -= lr * (m / (1 - b1^step)) / (sqrt(v / (1 - b2^step)) + eps).
 * `groups` is a host array; step >= 1. Each group's arrays must be 16-byte
 * aligned. */
gs_status gs_adam_step(const gs_adam_group* groups, int32_t n_groups, float beta1,
                       float beta2, float eps, int64_t step, void* stream);

/* Thresholds of gs_densify_and_prune. The pages fix only the gradient
 * threshold (0.0002 in the absolute-gradient tutorial's configuration); the
 * other cut-offs are the caller's. Scale and opacity tests are taken on the
 * raw parameters, so they are given as a log-scale and a logit. */
typedef struct gs_densify_params {
  float grad_threshold;     /* densify when accum > grad_threshold * denom, denom > 0 */
  float log_scale_split;    /* a densifying Gaussian whose largest log-scale exceeds
                               this is split, else cloned */
  float logit_min_opacity;  /* prune when the opacity logit is below this */
  float log_max_scale;      /* prune when the largest log-scale exceeds this */
  float log_split_shrink;   /* a child's log-scales: the parent's minus this (ln 1.6) */
  int32_t reserved;
} gs_densify_params;

/* The thresholds of gs_densify_and_prune from cut-offs in the units a user
 * states them in (host only, no CUDA call): the gradient threshold as is, the
 * scales as scales (log-scale = ln s), the minimum opacity as an opacity
 * (logit = ln(o / (1 - o))) and the split shrink factor (ln of it; 1.6 in
 * the usual configuration). Each conversion is taken in double precision and
 * rounded to float once. GS_ERR_INVALID_ARG unless scale_split, max_scale and
 * split_shrink are > 0, 0 < min_opacity < 1 and out is not NULL. */
gs_status gs_densify_params_from_cutoffs(double grad_threshold, double scale_split,
                                         double min_opacity, double max_scale,
                                         double split_shrink, gs_densify_params* out);

/* Bytes of workspace gs_densify_and_prune needs for n Gaussians (256-byte
 * aligned; the first 256 bytes hold the status word, as for gs_bin_sort). */
size_t gs_densify_workspace_size(int64_t n);

/* densify_and_prune (jsqmd.com sec. 1 and 3.3; pwwt.cn sec. 4.2). With the
 * float32 decisions of gs_densify_params, Gaussian i (index order) becomes:
 *   pruned (logit < logit_min_opacity or largest log-scale > log_max_scale;
 *     pruning wins): nothing;
 *   kept (not densifying): itself, with its Adam moments;
 *   cloned (densifying, largest log-scale <= log_scale_split): itself with its
 *     moments, then an exact copy with zero moments;
 *   split (densifying, larger): two children with zero moments: child c's
 *     mean is mean + R (exp(log-scale) * z[i][c]) (R the rotation of the
 *     normalised quaternion, z the caller's standard normal draws,
 *     float [n][2][3]); its log-scales are the parent's minus
 *     log_split_shrink; quaternion, logit and SH are copied.
 * The output Gaussians are compacted in that order into `out`, `m_out`,
 * `v_out` (the layouts of gs_params, out_capacity Gaussians each; padding
 * lanes copied); *n_out (device int64) always receives their number. If it
 * exceeds out_capacity nothing is written and GS_ERR_CAPACITY is raised in
 * the status word. accum is the view-space gradient accumulator of
 * gs_densify_stats (plain or absolute), denom its visibility count. codes, if
 * not NULL, receives int8 [n]: 0 pruned, 1 kept, 2 cloned, 3 split. With
 * quantised SH (in->sh_quant set) the SH blocks are not touched here (the sh
 * fields of out, m_out, v_out may be NULL) and codes must not be NULL:
 * gs_densify_sh_quant then builds the output's SH state from them. Outputs
 * must not overlap the inputs. */
gs_status gs_densify_and_prune(const gs_params* in, const gs_grads* m_in, const gs_grads* v_in,
                               const float* accum, const int32_t* denom, const float* z,
                               const gs_densify_params* dp, gs_grads* out, gs_grads* m_out,
                               gs_grads* v_out, int64_t out_capacity, int64_t* n_out,
                               int8_t* codes, void* ws, size_t ws_bytes, void* stream);

/* Bytes of workspace gs_l1_dssim needs for n_views views (sums and a block
 * counter; 8-byte aligned). */
size_t gs_l1_dssim_workspace_size(int32_t n_views);

/* Photometric loss and its gradient (second Julia page, lshu.cn, sec. 3.3):
 *   L_v = (1 - lambda) mean|x - y| + lambda (1 - mean SSIM(x, y))
 * per view v, the means over its 3 x height x width values. SSIM follows its
 * own definition (Wang et al. 2004), which the page does not restate: an
 * 11 x 11 Gaussian window of sigma 1.5 normalised to 1, C1 = 0.01^2,
 * C2 = 0.03^2 (dynamic range 1), the map taken at every pixel with the
 * planes zero outside the image.
 * image, target: float [n_views][3][height][width] (the layout of
 *   gs_rasterize_fwd's colour), device memory, not overlapping dL_dimage.
 * terms: device double [n_views][3] receives (L_v, mean L1, mean SSIM).
 * dL_dimage: device float, image's layout, receives dL_v / dimage (the
 *   L1 subgradient taken as 0 where x == y); NULL skips the gradient.
 * ws: device workspace of gs_l1_dssim_workspace_size(n_views) bytes,
 *   8-byte aligned; owned by the caller and overwritten.
 * n_views 0 returns GS_OK with nothing done; n_views > 21845, an empty image,
 * a height above 2,097,120, lambda outside [0, 1] or a NULL pointer is
 * GS_ERR_INVALID_ARG. One launch on `stream`. */
gs_status gs_l1_dssim(const float* image, const float* target, int32_t n_views, int32_t height,
                      int32_t width, float lambda, double* terms, float* dL_dimage, void* ws,
                      size_t ws_bytes, void* stream);

/* ---- quantised SH state (Spirula VRAM page, sec. 魔法一) ----------------
 * SH coefficients kept as 8- or 16-bit codes, every 256 Gaussians of one
 * coefficient sharing a (min, max) pair; the Adam moments of those values are
 * bfloat16. With n_pad = n rounded up to a multiple of GS_QUANT_GROUP and
 * k3 = 3 (degree + 1)^2, value j of Gaussian i (j = 3 coefficient + channel)
 * lives, by layout:
 *   GS_QUANT_PLANAR  codes uint8 (bits 8) or uint16 (bits 16) [k3][n_pad],
 *       the code at j * n_pad + i; the moments are two separate uint16
 *       (bfloat16) arrays [k3][n_pad] passed beside the state;
 *   GS_QUANT_PACKED  the page's packed optimiser block: codes is uint16
 *       [k3][n_pad / 32][3][32]; the block (j, i / 32) holds the 32 codes of
 *       Gaussians 32 (i / 32) .. + 31 (a 16-bit word each, also for 8-bit
 *       codes), then their 32 first moments, then their 32 second moments
 *       (bfloat16): 192 bytes, so the 32 lanes of a warp that update 32
 *       consecutive values touch two cache lines.
 *   bounds  float [k3][n_pad / 256][2]: the (min, max) of group (j, i / 256);
 *   a code q decodes to min + q (max - min) / (2^bits - 1), in float32 as
 *   fma(q, (max - min) / (2^bits - 1), min) with each operation rounded.
 * Encoding takes each group's min and max over its real Gaussians and rounds
 * t = (x - min) * ((2^bits - 1) / (max - min)) in float32 to nearest-even
 * (rounding 0) or to floor(t + u) (rounding 1, u in [0, 1) from SplitMix64
 * output number step * 2^37 + j * 2^31 + i + 1 of `seed`, top 24 bits);
 * a group with max == min gets code 0. Padding lanes are never written. */
#define GS_QUANT_GROUP 256
enum { GS_QUANT_PLANAR = 0, GS_QUANT_PACKED = 1 };

typedef struct gs_sh_quant {
  void* codes;      /* see above; device memory, caller-owned, 4-byte (8-bit
                       planar codes) or 8-byte aligned */
  float* bounds;    /* see above; device memory, caller-owned */
  int64_t n;        /* Gaussians, 0 <= n < 2^31 */
  int32_t k3;       /* values per Gaussian: 3, 12, 27 or 48 */
  int32_t bits;     /* 8 or 16 */
  int32_t layout;   /* GS_QUANT_PLANAR or GS_QUANT_PACKED */
  int32_t reserved;
} gs_sh_quant;

/* Encode float SH [n][k3] (the gs_params layout) into q (nearest rounding).
 * Only codes and bounds are written (packed blocks keep their moments). */
gs_status gs_sh_quantize(const float* sh, const gs_sh_quant* q, void* stream);

/* Decode q into float SH [n][k3] (float32: fma(q, (max - min) / (2^bits - 1), min)). */
gs_status gs_sh_dequantize(const gs_sh_quant* q, float* sh, void* stream);

/* One Adam step on the quantised SH, fused: decode each value, update its
 * bfloat16 moments (round to nearest-even) with the float32 gradient grad_sh
 * ([n][k3], the gs_grads layout), take the step of gs_adam_step (lr, beta1,
 * beta2, eps, bias corrections of `step`), then re-encode the group with its
 * new min and max (rounding as above). Planar: the moments are exp_avg /
 * exp_avg_sq ([k3][n_pad], 8-byte aligned). Packed: they are in the blocks
 * and exp_avg / exp_avg_sq must be NULL. Both layouts give the same codes,
 * bounds and moments. Argument errors as gs_adam_step, plus rounding not
 * 0/1, bits not 8/16, k3 not 3/12/27/48, an unknown layout. */
gs_status gs_adam_step_sh_quant(const gs_sh_quant* q, const float* grad_sh, uint16_t* exp_avg,
                                uint16_t* exp_avg_sq, float lr, float beta1, float beta2,
                                float eps, int64_t step, int32_t rounding, uint64_t seed,
                                void* stream);

/* densify_and_prune for quantised SH (jsqmd.com sec. 1 and 3.3, with the
 * Spirula page's quantised state). `decisions` are the int8 codes
 * gs_densify_and_prune wrote for the same n Gaussians (0 pruned, 1 kept,
 * 2 cloned, 3 split); out->n must be their output count (1 per kept, 2 per
 * cloned or split Gaussian). Output Gaussian o takes the SH values of the
 * input it comes from (decoded), in gs_densify_and_prune's order, and its
 * groups are encoded anew with nearest rounding, so out equals gs_sh_quantize
 * of the decoded input SH gathered in that order. Moments: a kept Gaussian
 * and a clone's first copy keep theirs; a clone's copy and split children
 * get zeros. in and out have the same k3, bits and layout; planar moments
 * are m_in / v_in -> m_out / v_out ([k3][n_pad] each), packed ones travel
 * in the blocks (the four pointers NULL). ws: device workspace of
 * gs_densify_sh_quant_workspace_size(in->n, out->n) bytes, 256-byte aligned
 * (the first 256 bytes hold the status word). The output must not overlap
 * the input. Four launches on `stream`. */
size_t gs_densify_sh_quant_workspace_size(int64_t n_in, int64_t n_out);
gs_status gs_densify_sh_quant(const gs_sh_quant* in, const uint16_t* m_in, const uint16_t* v_in,
                              const int8_t* decisions, const gs_sh_quant* out, uint16_t* m_out,
                              uint16_t* v_out, void* ws, size_t ws_bytes, void* stream);

/* Test hook for the timeout path (the pages have no counterpart). Every
 * device-side wait of the library (an mbarrier phase in gs_project and the
 * rasteriser, a look-back flag in gs_bin_sort's emission and radix passes)
 * gives up after a time limit, sets GS_STATUS_BIT_TIMEOUT and lets its kernel
 * finish. This call makes one such wait run out on purpose, without faulting
 * anything:
 *   GS_STALL_RASTER_FWD / GS_STALL_RASTER_BWD  global tile `index` of the
 *     next rasteriser calls issues no record copies and waits in vain for
 *     its first batch (its pixels keep the background / add no gradient);
 *   GS_STALL_EMIT_LOOKBACK  emission block `index` of gs_bin_sort's
 *     look-back scan (GS_SORT_FULL64, and GS_SORT_PRESORT on grids that
 *     sort by tile id) never publishes its prefix, so its successors' waits
 *     run out;
 *   GS_STALL_SORT_LOOKBACK  partition `index` (of 4096 keys) of gs_bin_sort's
 *     single-sweep radix passes (the depth keys of GS_SORT_PRESORT, the pair
 *     keys of GS_SORT_FULL64) publishes neither its digit counts nor its
 *     prefix in any pass, so the waits of the partitions after it run out;
 *   GS_STALL_NONE  back to normal.
 * wait_limit_s (> 0) replaces the default limit of 2 s for every wait while
 * the setting holds; 0 keeps the default. Process-wide, not thread-safe
 * against concurrent calls of the library; meant for tests only. */
enum { GS_STALL_NONE = 0, GS_STALL_EMIT_LOOKBACK = 1, GS_STALL_RASTER_FWD = 2,
       GS_STALL_RASTER_BWD = 3, GS_STALL_SORT_LOOKBACK = 4 };
gs_status gs_debug_stall(int32_t site, int64_t index, double wait_limit_s);

/* Synchronise `stream`, return the status word accumulated in workspace `ws`
 * by device-side checks since the last call, and clear it. Several conditions
 * report the most severe: GS_ERR_DEVICE_TIMEOUT, then GS_ERR_OVERFLOW (an
 * index out of range was clipped), GS_ERR_CAPACITY, GS_ERR_NONFINITE. */
gs_status gs_get_status(void* ws, void* stream);

#ifdef __cplusplus
}  /* extern "C" */
#endif

#endif  /* GS_B200_H */
