/*
 * gs.h - C ABI of the B200 differentiable Gaussian-splatting tile rasterizer (libgs.so).
 *
 * The library is the data-parallel hot path of 3D Gaussian Splatting: per-Gaussian
 * projection, tile binning with a (tile_id << 32 | depth) radix sort, front-to-back
 * alpha compositing per 16x16 tile, its reverse pass, the chain back to the Gaussian
 * parameters, and the Adam update.  The three stages are the ones named in the gsplat
 * guide (lmnt.cn/news/262699) §2.1 -- "3D transform (R, t, scale, rot)", "depth and
 * screen-space projection", "differentiable alpha-blending rasterization" -- and the
 * split into a forward call and a standalone backward call follows the same guide
 * §2.2 (rasterize_gaussians / rasterize_gaussians_backward).
 *
 * Conventions for every call
 *   - Plain C.  Every call returns a gs_status; GS_OK is 0.  On failure,
 *     gs_last_error_detail() returns a thread-local description.
 *   - The library allocates nothing.  The caller owns every buffer.  Pointers are
 *     device pointers unless the name ends in _host.  `stream` is a cudaStream_t
 *     (NULL = the legacy default stream); calls enqueue work on it and return
 *     without waiting, except gs_bin_sort, which reads the instance count back
 *     to the host (one device-to-host copy and a stream synchronisation).
 *   - Arguments are checked on the host before anything is launched: NULL
 *     pointers, negative sizes and misaligned buffers (alignment as stated per
 *     array) return GS_ERR_INVALID_ARG; an SH degree above 3 or an image side
 *     outside 1..16384 returns GS_ERR_UNSUPPORTED.  A CUDA launch or copy error
 *     returns GS_ERR_CUDA.  No kernel traps or asserts.
 *   - Gradient outputs are accumulated (+=): callers zero them, and several views
 *     can add into the same buffers.  (The backward calls with Adam are the
 *     exception: their gradient buffer receives the step's gradient, written over.)
 *   - Arrays are structure-of-arrays, read with 128-bit loads: an array written
 *     "[n][4]" is n consecutive float4 records (16-byte aligned).
 *   - n (Gaussians) up to 2^31 - 1; instance counts up to 2^32 - 1; tiles up to 2^20.
 */
#ifndef GS_H
#define GS_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef int32_t gs_status;
#define GS_OK 0
#define GS_ERR_INVALID_ARG 1
#define GS_ERR_UNSUPPORTED 2
#define GS_ERR_CAPACITY 3
#define GS_ERR_CUDA 4

#define GS_TILE 16 /* tile side in pixels */

/* Pinhole camera.  x_cam = R x_world + t (R row-major, world to camera), OpenCV
 * axes (x right, y down, z forward).  Pixel (x, y) samples the image plane at
 * (x + 0.5, y + 0.5).  Gaussians with camera depth <= near_plane are culled; eps2d
 * is added to both diagonal entries of every projected 2D covariance (the
 * screen-space low-pass of the original 3DGS rasterizer, 0.3).
 *
 * tile_cull (0 or 1; anything else is GS_ERR_INVALID_ARG) selects the tiles the
 * binning calls put a visible Gaussian into:
 *   0  every tile of its tile rectangle (tiles_touched of them);
 *   1  only the tiles of the rectangle whose box of pixel centres, widened by
 *      1/1024 px, meets the region where o e^-sigma >= 1/255 (alpha can pass
 *      the compositing's skip test there), that bound taken with a margin of
 *      1e-4 (|ln(255 o)| + 1): the culling stage of the MUSA co-design article
 *      (qwbw.cn/news/278220 §1).  A conic that is not positive definite keeps
 *      its whole rectangle; an opacity below about 1/255 gets no tile.
 * The two give the same image, final_T and gradients (a dropped instance is
 * skipped at every pixel of its tile); n_contrib counts positions in the
 * lists actually binned.  The projection ignores the flag; a culled binning
 * needs 36 bytes more workspace per Gaussian (gs_bin_sort_workspace_bytes). */
typedef struct gs_camera {
    float R[9];
    float t[3];
    float fx, fy, cx, cy;
    int32_t width, height;
    float near_plane;
    float eps2d;
    int32_t tile_cull;
} gs_camera;

/* Gaussian parameters, stored pre-activation as the gsplat guide §3.3 sets
 * them up: scale = exp(log_scale), opacity = sigmoid(logit), rotation = the
 * normalised quaternion (w, x, y, z).
 *   means          [n][4]  x, y, z, unused        (16-byte aligned)
 *   quats          [n][4]  w, x, y, z             (16-byte aligned)
 *   log_scales     [n][4]  x, y, z, unused        (16-byte aligned)
 *   opacity_logits [n]                            (4-byte aligned)
 *   sh             [P][n][4] with P = gs_sh_planes(sh_degree): the Gaussian's
 *                  3*(d+1)^2 SH coefficients, coefficient-major and channel-minor
 *                  (c0.r c0.g c0.b c1.r ...), cut into float4 planes; plane j of
 *                  Gaussian i is sh[(j*n + i)*4 .. +3]; unused tail lanes are zero.
 *                  (16-byte aligned) */
typedef struct gs_params {
    const float* means;
    const float* quats;
    const float* log_scales;
    const float* opacity_logits;
    const float* sh;
    int32_t sh_degree;
    int64_t n;
} gs_params;

/* Gradients of the same parameters, same layouts; written with +=. */
typedef struct gs_param_grads {
    float* means;
    float* quats;
    float* log_scales;
    float* opacity_logits;
    float* sh;
} gs_param_grads;

/* Per-Gaussian projection results (written by gs_project, read by the later
 * calls).  A culled Gaussian has radius 0, tiles_touched 0 and zero features.
 *   xy            [n][2]  pixel position (u, v) of the mean        (8-byte aligned)
 *   depth         [n]     camera-space z                           (4-byte aligned)
 *   conic_opacity [n][4]  A, B, C of the inverse 2D covariance, so that
 *                         sigma = 1/2 (A dx^2 + C dy^2) + B dx dy, and the
 *                         opacity o                                 (16-byte aligned)
 *   rgb           [n][4]  colour r, g, b, 0                        (16-byte aligned)
 *   radius        [n]     ceil(3 sqrt(largest eigenvalue)) in pixels
 *   rect          [n][4]  tile rectangle xmin, ymin, xmax, ymax (max exclusive),
 *                         uint16                                   (8-byte aligned)
 *   tiles_touched [n]     (xmax - xmin) * (ymax - ymin)            (4-byte aligned) */
typedef struct gs_projected {
    float* xy;
    float* depth;
    float* conic_opacity;
    float* rgb;
    int32_t* radius;
    uint16_t* rect;
    uint32_t* tiles_touched;
} gs_projected;

/* Gradients with respect to the projected features, written by gs_raster_bwd (+=):
 *   xy            [n][2]  dL/du, dL/dv                              (8-byte aligned)
 *   conic_opacity [n][4]  dL/dA, dL/dB, dL/dC, dL/do                (16-byte aligned)
 *   rgb           [n][4]  dL/dr, dL/dg, dL/db, 0                    (16-byte aligned)
 *   xy_abs        [n][2]  NULL, or the absolute gradient (the absgrad option of
 *                         the gsplat guide §4.1): the sum over pixels of the
 *                         absolute value of each pixel's contribution to dL/du
 *                         and to dL/dv                               (8-byte aligned)
 * When xy_abs is set, the densification statistic of the backward calls
 * through the projection accumulates |xy_abs| instead of |xy|. */
typedef struct gs_grad2d {
    float* xy;
    float* conic_opacity;
    float* rgb;
    float* xy_abs;
} gs_grad2d;

/* Text for a status code (static storage). */
const char* gs_status_string(gs_status status);

/* Description of the last failure on the calling thread ("" if none). */
const char* gs_last_error_detail(void);

/* Number of float4 planes of the SH array for a degree (1, 3, 7, 12 for 0..3;
 * 0 for an unsupported degree). */
int32_t gs_sh_planes(int32_t sh_degree);

/* Tile grid of a camera: ceil(width / 16) x ceil(height / 16). */
gs_status gs_tile_grid(const gs_camera* cam, int32_t* tiles_x_host, int32_t* tiles_y_host);

/* gs_project -- stages 1 and 2 of the pipeline (gsplat guide §2.1) for every
 * Gaussian: camera-space mean, 3D covariance R S S^T R^T from the normalised
 * quaternion and exp(log_scale), EWA projection J W Sigma W^T J^T + eps2d I with
 * the perspective Jacobian J (x/z and y/z clamped to 1.3 times the half field of
 * view), its inverse (conic), the 3-sigma radius and tile rectangle, sigmoid
 * opacity, and the colour from real spherical harmonics of the viewing direction
 * (mean minus camera centre), offset by 0.5 and clamped at 0.  Culled: non-finite
 * parameters, a zero quaternion, depth <= near_plane, a non-positive 2D
 * determinant, an empty rectangle, a non-finite colour.
 * Arithmetic is double precision; outputs are rounded to float32. */
gs_status gs_project(const gs_params* params, const gs_camera* cam, gs_projected* out, void* stream);

/* gs_project_views -- gs_project for num_views (1..GS_MAX_VIEWS) views of the same
 * Gaussians in one launch: outs[v] receives, bit for bit, what gs_project writes
 * for cams[v].  The view-independent part of stages 1-2 of the gsplat guide §2.1
 * (the 3D covariance from quaternion and scales, the opacity) and the reading of
 * the parameters are shared by the views instead of repeated per view.  sh_half:
 * NULL, or the 16-bit copy of the SH planes that gs_project_sh16 reads (params->sh
 * is then not read).  Every outs[v] as gs_project's out; the views' arrays must
 * not overlap.  Asynchronous. */
gs_status gs_project_views(const gs_params* params, int32_t num_views, const gs_camera* cams, gs_projected* outs,
                           const uint16_t* sh_half, void* stream);

/* Bytes of device workspace gs_bin_sort needs for n Gaussians and up to `capacity`
 * instances (16-byte aligned buffer, owned by the caller), with the camera's
 * tile_cull (cam may be NULL: no culling). */
size_t gs_bin_sort_workspace_bytes(int64_t n, int64_t capacity, const gs_camera* cam);

/* gs_bin_sort -- tile binning.  Every visible Gaussian emits one instance per tile
 * of its rectangle (with the camera's tile_cull, per tile of the rectangle that its
 * footprint reaches: gs_camera), key = (ty * tiles_x + tx) << 32 | float32 bits of its depth,
 * value = Gaussian index; the instances are sorted by key, equal keys keeping
 * ascending Gaussian index, and tile_ranges[2t], [2t+1] receive the [begin, end)
 * of tile t in the sorted list ([0, 0) when empty).  Method: a stable LSD radix
 * sort of the Gaussians by depth bits, instances emitted in that order, then a
 * stable LSD radix sort by tile id (ceil(log2(tiles)) bits); the last pass writes
 * the 64-bit keys.
 *   keys [capacity] (8-byte aligned), vals [capacity] (4-byte aligned),
 *   tile_ranges [tiles][2] uint32 (8-byte aligned), workspace as sized above.
 * *num_instances_host receives K, the instance count.  K > capacity returns
 * GS_ERR_CAPACITY with keys and vals untouched and every tile range empty; call
 * again with a larger buffer.  The call waits for K (one 8-byte device-to-host
 * copy); gs_bin_sort_async does not. */
gs_status gs_bin_sort(const gs_projected* proj, int64_t n, const gs_camera* cam, void* workspace,
                      size_t workspace_bytes, uint64_t* keys, uint32_t* vals, int64_t capacity,
                      int64_t* num_instances_host, uint32_t* tile_ranges, void* stream);

/* gs_bin_sort_async -- gs_bin_sort without waiting: the passes over instances
 * are launched for `capacity` and read K on the device, and K is written to
 * *num_instances_dev (one uint64 on the device, 8-byte aligned) instead of the
 * host.  If K > capacity nothing is emitted or sorted and every tile range is
 * empty, so the later raster calls see no instances; the caller reads K when it
 * synchronises anyway and repeats the view with larger buffers. */
gs_status gs_bin_sort_async(const gs_projected* proj, int64_t n, const gs_camera* cam, void* workspace,
                            size_t workspace_bytes, uint64_t* keys, uint32_t* vals, int64_t capacity,
                            uint64_t* num_instances_dev, uint32_t* tile_ranges, void* stream);

/* Bytes of device workspace gs_depth_order_views needs for n Gaussians seen
 * from num_views views (about 16 bytes per Gaussian and view). */
size_t gs_depth_order_workspace_bytes(int64_t n, int32_t num_views);

/* gs_depth_order_views -- the first half of gs_bin_sort for several views of the
 * same Gaussians at once: for each view v (1..GS_MAX_VIEWS views, projs[v] as
 * written by gs_project; tiles_touched and depth are read), the stable order of
 * the Gaussians by the float32 bits of their depth, culled Gaussians last,
 * written to order[v * n ... v * n + n - 1] (uint32, 4-byte aligned).  One launch
 * per radix pass serves every view.  Asynchronous; workspace (16-byte aligned,
 * caller-owned) as sized above. */
gs_status gs_depth_order_views(const gs_projected* projs, int32_t num_views, int64_t n, void* workspace,
                               size_t workspace_bytes, uint32_t* order, void* stream);

/* gs_bin_sort_ordered_async -- gs_bin_sort_async from a depth order computed by
 * gs_depth_order_views (order [n], this view's row): emission of the instances
 * in that order, the stable passes by tile id, the ranges.  Same arguments,
 * results and capacity behaviour as gs_bin_sort_async otherwise (the same
 * workspace size). */
gs_status gs_bin_sort_ordered_async(const gs_projected* proj, int64_t n, const uint32_t* order, const gs_camera* cam,
                                    void* workspace, size_t workspace_bytes, uint64_t* keys, uint32_t* vals,
                                    int64_t capacity, uint64_t* num_instances_dev, uint32_t* tile_ranges,
                                    void* stream);

/* gs_bin_sort_ordered_views_async -- gs_bin_sort_ordered_async for num_views
 * (1..GS_MAX_VIEWS) views of the same n Gaussians and the same image size, every
 * kernel launched once for all of them (grid rows = views): view v has
 * projs[v], its depth order orders + v * n (the rows gs_depth_order_views
 * writes), cams[v] (only the image size is read; all views must have the same),
 * workspaces[v] of workspace_bytes[v] bytes, keys[v], vals[v], capacities[v],
 * num_instances_dev[v] and tile_ranges[v] -- host arrays of device pointers and
 * sizes.  Each view's results and capacity behaviour are gs_bin_sort_ordered_async's
 * bit for bit; one launch per kernel instead of one per view and kernel removes
 * the launch gaps and the partly filled last wave of every small launch.  The
 * views' buffers must not overlap.  Errors (nothing launched): those of
 * gs_bin_sort_ordered_async for any view, GS_ERR_INVALID_ARG for num_views
 * outside 1..GS_MAX_VIEWS or image sizes that differ. */
gs_status gs_bin_sort_ordered_views_async(const gs_projected* projs, int32_t num_views, int64_t n,
                                          const uint32_t* orders, const gs_camera* cams, void* const* workspaces,
                                          const size_t* workspace_bytes, uint64_t* const* keys, uint32_t* const* vals,
                                          const int64_t* capacities, uint64_t* const* num_instances_dev,
                                          uint32_t* const* tile_ranges, void* stream);

/* Size of the device array gs_bin_sort_static uses as its workspace (32 MiB). */
#define GS_STATIC_SCRATCH_BYTES ((size_t)32 << 20)

/* gs_bin_sort_static -- gs_bin_sort for callers that cannot allocate device
 * memory.  The paper has no counterpart: it is an interface for hosts that own
 * the whole device budget, frame loops where a cudaMalloc would stall every
 * stream, and foreign runtimes that can pass device pointers but cannot
 * allocate.  Same arguments and results as gs_bin_sort minus the workspace,
 * which is a library-owned device array of GS_STATIC_SCRATCH_BYTES held on
 * every device that loads the library until the process exits.
 *   - n and capacity whose workspace (gs_bin_sort_workspace_bytes) exceeds
 *     GS_STATIC_SCRATCH_BYTES return GS_ERR_UNSUPPORTED (the workspace is
 *     about 16 bytes per slot of max(capacity, n): about 2 million).
 *   - Every call looks up the array's address in the current context
 *     (cudaGetSymbolAddress, no allocation), so it stays valid after a
 *     cudaDeviceReset and in contexts the host creates itself.  The first call
 *     in a context loads the library's module there, which is when the array
 *     comes into being: make that first call before any stream capture.
 *   - All calls share the array.  Calls whose GPU work overlaps (other streams,
 *     other threads on the same device) race on it: serialise them.  No state
 *     carries over between calls; nothing in it needs clearing.
 *   - Allocates nothing (no cudaMalloc / cudaFree, no allocating library call). */
gs_status gs_bin_sort_static(const gs_projected* proj, int64_t n, const gs_camera* cam, uint64_t* keys,
                             uint32_t* vals, int64_t capacity, int64_t* num_instances_host, uint32_t* tile_ranges,
                             void* stream);

/* gs_tile_order -- the tiles ordered by decreasing length of their sorted lists
 * (tile_ranges as written by gs_bin_sort; tile_order [tiles] uint32, 4-byte
 * aligned).  Passed to the raster calls it starts the longest tiles first, so
 * that the end of each launch is not held by a few long tiles; results do not
 * depend on the order. */
gs_status gs_tile_order(const uint32_t* tile_ranges, const gs_camera* cam, uint32_t* tile_order, void* stream);

/* gs_tile_order_views -- gs_tile_order for num_views (1..GS_MAX_VIEWS) views of
 * the same tile grid (cam's image size) in one launch: tile_ranges[v] and
 * tile_orders[v] are view v's (host arrays of device pointers). */
gs_status gs_tile_order_views(int32_t num_views, const uint32_t* const* tile_ranges, const gs_camera* cam,
                              uint32_t* const* tile_orders, void* stream);

/* gs_raster_fwd -- stage 3 (gsplat guide §2.1) over 16x16 tiles.  For each
 * pixel, front to back over its tile's sorted list: sigma as above with
 * d = (u, v) - pixel centre; entries with sigma < 0 are skipped;
 * alpha = min(0.99, o exp(-sigma)); entries with alpha < 1/255 are skipped; if
 * T (1 - alpha) < 1e-4 the pixel stops without blending that entry; otherwise
 * C += rgb alpha T and T *= 1 - alpha.  sigma is evaluated in float32, for
 * conics with an eigenvalue ratio above 8 in the factored form
 * 1/2 A t^2 + 1/2 (det/A) dy^2, t = dx + (B/A) dy, which keeps a few ulps of
 * relative accuracy at any ratio; for a positive-definite conic sigma >= 0
 * holds and is not tested.
 *   tile_order  optional processing order from gs_tile_order (NULL: tile order)
 *   image   [H][W][3] = C + T bg (bg_host: 3 floats read during the call)
 *   final_T [H][W]    transmittance after the last blended entry
 *   n_contrib [H][W]  1 + list position of the last blended entry (0 if none) */
gs_status gs_raster_fwd(const gs_projected* proj, const uint32_t* vals, const uint32_t* tile_ranges,
                        const uint32_t* tile_order, const gs_camera* cam, const float* bg_host, float* image,
                        float* final_T, int32_t* n_contrib, void* stream);

/* gs_raster_fwd_l1 -- gs_raster_fwd followed by gs_l1_loss_grad on the image it
 * renders, in one kernel: the compositing writes image, final_T and n_contrib as
 * gs_raster_fwd does, and each pixel then takes its L1 term against target
 * ([H][W][3] float, 4-byte aligned): dL_dimage ([H][W][3], 4-byte aligned) =
 * sign(image - target) / (3 H W) (sign(0) = 0), and *loss_dev (one double, 8-byte
 * aligned) += mean |image - target|.  Image, final_T, n_contrib and dL_dimage equal
 * the two calls' bit for bit; the loss is their sum up to the order of its double
 * additions.  Saves the image's second read, the L1 kernel and its launch. */
gs_status gs_raster_fwd_l1(const gs_projected* proj, const uint32_t* vals, const uint32_t* tile_ranges,
                           const uint32_t* tile_order, const gs_camera* cam, const float* bg_host, const float* target,
                           float* image, float* final_T, int32_t* n_contrib, float* dL_dimage, double* loss_dev,
                           void* stream);

/* gs_raster_bwd -- the reverse of gs_raster_fwd for an upstream dL/dimage
 * [H][W][3]: per pixel, back to front from n_contrib, the transmittance in front
 * of each blended entry is recovered from final_T, and with S the colour blended
 * behind the entry (normalised by the transmittance just behind it):
 *   dL/drgb   += alpha T g
 *   dL/dalpha  = sum_c g_c (T (rgb_c - S_c) - final_T bg_c / (1 - alpha))
 * then through alpha = o exp(-sigma) (nothing when alpha was clamped at 0.99) to
 * o, to (u, v) and to (A, B, C).  Per-Gaussian sums are reduced across each warp
 * with shuffles before one vector atomic add per warp.  grad2d is accumulated.
 * tile_order as for gs_raster_fwd. */
gs_status gs_raster_bwd(const gs_projected* proj, const uint32_t* vals, const uint32_t* tile_ranges,
                        const uint32_t* tile_order, const gs_camera* cam, const float* bg_host, const float* final_T,
                        const int32_t* n_contrib, const float* dL_dimage, gs_grad2d* grad2d, void* stream);

/* gs_project_bwd -- chain grad2d through gs_project to the parameters (+= into
 * grads), in double precision: colour to SH coefficients (zero where the colour
 * was clamped) and to the mean through the viewing direction; (u, v) to the mean;
 * the conic through the 2x2 inverse, the EWA product and the Jacobian to the mean,
 * the log-scales and the quaternion (through its normalisation); opacity to its
 * logit.  Culled Gaussians get nothing.  When densify_accum and densify_count are
 * non-NULL, every visible Gaussian also gets densify_accum += |(dL/du, dL/dv)| and
 * densify_count += 1 (the screen-space mean-gradient statistic that adaptive
 * density control thresholds, gsplat guide §4.1).  [n] floats / int32.  When
 * densify_max_radius [n] int32 is non-NULL it becomes the largest of itself and
 * the view's radius (the screen-size statistic that gs_densify_plan prunes on). */
gs_status gs_project_bwd(const gs_params* params, const gs_camera* cam, const gs_projected* proj,
                         const gs_grad2d* grad2d, gs_param_grads* grads, float* densify_accum,
                         int32_t* densify_count, int32_t* densify_max_radius, void* stream);

/* Most views one multi-view backward call takes. */
#define GS_MAX_VIEWS 16

/* gs_project_bwd_views -- gs_project_bwd for num_views (1..GS_MAX_VIEWS) views of
 * the same Gaussians in one pass: cams, projs and grad2d are host arrays of
 * num_views structs (of projs only `radius` is read: a Gaussian counts as
 * visible in a view when its radius there is > 0).  Every Gaussian reads its
 * parameters once, adds every visible view's contribution in registers and
 * accumulates the sum over views into grads (+=); densify statistics as in
 * gs_project_bwd, summed (the largest radius: maximised) over views.  Equal, up
 * to rounding, to num_views calls of gs_project_bwd. */
gs_status gs_project_bwd_views(const gs_params* params, int32_t num_views, const gs_camera* cams,
                               const gs_projected* projs, const gs_grad2d* grad2d, gs_param_grads* grads,
                               float* densify_accum, int32_t* densify_count, int32_t* densify_max_radius,
                               void* stream);

/* gs_project_bwd_views_adam -- gs_project_bwd_views followed by the Adam step of
 * gs_adam for all five parameter groups (gsplat guide §4.2: lr_host[5] for
 * means, quats, log_scales, opacity_logits, sh; shared betas, eps and step).
 * params_inout holds the same arrays as params and is updated in place; adam_m
 * and adam_v are the first and second moments in the parameter layout.
 *
 * grads receives the step's summed gradient, written over (not added to): zero
 * for a Gaussian visible in none of the views, and the w lane of each means
 * entry holds the number of views in which the Gaussian is visible.  With grads
 * the chain and the Adam step are two launches (the chain, then one Adam launch
 * over all five groups) that pass the gradient through it; grads must not overlap
 * params, adam_m or adam_v.  grads may be NULL with up to
 * GS_ADAM_ONE_PASS_MAX_VIEWS views: the chain and the step then run as one
 * kernel and the gradient never reaches memory (slower: the step's memory round
 * trips wait on the chain's).
 *
 * With sparse_adam = 0 every Gaussian is updated, visible or not, as gs_adam
 * updates every element.  With sparse_adam = 1 (the sparse_grad option of the
 * gsplat guide §4.1) a Gaussian visible in none of the views keeps its
 * parameters and moments unchanged (no decay of the moments), as a sparse Adam
 * skips absent rows; the bias correction still uses `step`.  Errors (nothing
 * launched): those of gs_project_bwd_views, and GS_ERR_INVALID_ARG for grads
 * NULL with more than GS_ADAM_ONE_PASS_MAX_VIEWS views. */
#define GS_ADAM_ONE_PASS_MAX_VIEWS 2
gs_status gs_project_bwd_views_adam(const gs_params* params, int32_t num_views, const gs_camera* cams,
                                    const gs_projected* projs, const gs_grad2d* grad2d, gs_param_grads* params_inout,
                                    gs_param_grads* adam_m, gs_param_grads* adam_v, const float* lr_host,
                                    float beta1, float beta2, float eps, int32_t step, gs_param_grads* grads,
                                    float* densify_accum, int32_t* densify_count, int32_t* densify_max_radius,
                                    int32_t sparse_adam, void* stream);

/* The packed layout (the packed option of rasterize_gaussians, gsplat guide
 * §4.1): a view's projected features are stored only for the Gaussians it keeps
 * (radius > 0), contiguously in ascending Gaussian order.  Slot k holds
 * Gaussian gaussian_ids[k]; slot_of[i] is the slot of Gaussian i, or -1.  Every
 * later call takes the packed arrays as it takes gs_project's, with n replaced
 * by the capacity: the binning's values, the raster calls' 2D gradients and the
 * instance lists are then indexed by slot.  Because slots ascend with the
 * Gaussian id, the sort keys and the order of equal keys are those of the
 * unpacked layout with every value v replaced by gaussian_ids[v], the images are
 * the same bit for bit, and the 2D gradients are the same sums (added in an order
 * the atomics choose, as in the unpacked layout).
 *
 * gs_project_packed_workspace_bytes -- device workspace for n Gaussians (about
 * 60 bytes per Gaussian: gs_project's outputs for all of them, before packing).
 *
 * gs_project_packed -- gs_project of every Gaussian into the workspace, then
 * the order-preserving compaction into `capacity` packed slots:
 *   packed         gs_projected arrays of `capacity` entries (the alignments of
 *                  gs_projected);
 *   gaussian_ids   [capacity] uint32, 0xffffffff for an unused slot;
 *   slot_of        [params->n] int32;
 *   num_visible_dev  one uint64 on the device: the number V of Gaussians kept.
 * Slots V..capacity-1 hold culled entries (radius 0, tiles_touched 0, zero
 * features), so the later calls skip them.  V > capacity is not an error of the
 * call: slots up to capacity are filled, slot_of is -1 for the Gaussians that got
 * none, and the caller compares V (read when convenient) with the capacity and
 * repeats with more room before using the results.  Asynchronous, no host wait.
 * Errors (nothing launched): GS_ERR_INVALID_ARG for a NULL or misaligned pointer,
 * a capacity outside 0..2^31-1 or a workspace smaller than
 * gs_project_packed_workspace_bytes(params->n); GS_ERR_UNSUPPORTED as gs_project. */
size_t gs_project_packed_workspace_bytes(int64_t n);
gs_status gs_project_packed(const gs_params* params, const gs_camera* cam, void* workspace, size_t workspace_bytes,
                            gs_projected* packed, int64_t capacity, uint32_t* gaussian_ids, int32_t* slot_of,
                            uint64_t* num_visible_dev, void* stream);

/* gs_project_bwd_views_packed, gs_project_bwd_views_adam_packed --
 * gs_project_bwd_views and gs_project_bwd_views_adam for views in the packed
 * layout: projs[v] and grad2d[v] are view v's packed arrays and slot_of[v]
 * (a host array of num_views device pointers) its slot map; a Gaussian is in
 * view v when slot_of[v][i] >= 0.  Parameters, gradients and the densification
 * statistics stay indexed by Gaussian.  Results equal those of the unpacked
 * calls given the same per-Gaussian 2D gradients. */
gs_status gs_project_bwd_views_packed(const gs_params* params, int32_t num_views, const gs_camera* cams,
                                      const gs_projected* projs, const int32_t* const* slot_of,
                                      const gs_grad2d* grad2d, gs_param_grads* grads, float* densify_accum,
                                      int32_t* densify_count, int32_t* densify_max_radius, void* stream);
gs_status gs_project_bwd_views_adam_packed(const gs_params* params, int32_t num_views, const gs_camera* cams,
                                           const gs_projected* projs, const int32_t* const* slot_of,
                                           const gs_grad2d* grad2d, gs_param_grads* params_inout,
                                           gs_param_grads* adam_m, gs_param_grads* adam_v, const float* lr_host,
                                           float beta1, float beta2, float eps, int32_t step, gs_param_grads* grads,
                                           float* densify_accum, int32_t* densify_count, int32_t* densify_max_radius,
                                           int32_t sparse_adam, void* stream);

/* 16-bit SH storage (the guides' FP16 mode: FP16 parameters for rendering, mixed
 * precision in training).  The SH coefficients are kept as IEEE binary16 in the
 * float4-plane layout of gs_params.sh: [planes][n][4] halves, 8-byte aligned.
 * All arithmetic stays double / float32; widening a half is exact, so every
 * result equals the float32 path's on the rounded coefficients.
 *
 * gs_to_half -- out[i] = x[i] rounded to the nearest binary16, ties to even
 * (magnitudes past 65504 round to infinity, as IEEE 754 rounds); count floats,
 * x 16-byte and out 8-byte aligned.
 *
 * gs_project_sh16 -- gs_project with the SH coefficients read from sh_half
 * instead of params->sh (which may be NULL).  A coefficient that rounded to
 * infinity makes the colour non-finite, and the Gaussian is culled.
 *
 * gs_project_bwd_views_adam_sh16 -- gs_project_bwd_views_adam for views
 * projected by gs_project_sh16: the colour chain uses the half-precision
 * coefficients in sh_half (the values the forward pass used), Adam updates the
 * float32 coefficients params_inout->sh (the master copy), and each updated
 * float32 coefficient is written, rounded as by gs_to_half, to sh_half_out
 * (which may be sh_half itself).  Unpacked views only.
 *
 * Errors (nothing launched): GS_ERR_INVALID_ARG for a negative count, a NULL or
 * misaligned pointer (sh_half and sh_half_out 8-byte aligned when n > 0), and
 * otherwise as the float32 calls. */
gs_status gs_to_half(const float* x, int64_t count, uint16_t* out, void* stream);
gs_status gs_project_sh16(const gs_params* params, const uint16_t* sh_half, const gs_camera* cam, gs_projected* out,
                          void* stream);
gs_status gs_project_bwd_views_adam_sh16(const gs_params* params, int32_t num_views, const gs_camera* cams,
                                         const gs_projected* projs, const gs_grad2d* grad2d,
                                         const uint16_t* sh_half, uint16_t* sh_half_out, gs_param_grads* params_inout,
                                         gs_param_grads* adam_m, gs_param_grads* adam_v, const float* lr_host,
                                         float beta1, float beta2, float eps, int32_t step, gs_param_grads* grads,
                                         float* densify_accum, int32_t* densify_count, int32_t* densify_max_radius,
                                         int32_t sparse_adam, void* stream);

/* Adaptive density control (gsplat guide §4.1: every 100 steps,
 * densify_and_prune with a gradient threshold of 0.0002, a minimum opacity of
 * 0.005, an extent of 0.01 and a maximum screen size of 0.02; 3DGS deploy guide
 * §3.2: --densify_grad_threshold 0.0002).  Per Gaussian, in this order:
 *   prune   unless sigmoid(logit) >= min_opacity, or when max_screen_radius > 0
 *           and the largest radius it reached (densify_max_radius of the
 *           backward calls) exceeds max_screen_radius pixels;
 *   densify when densify_count > 0 and densify_accum / densify_count >=
 *           grad_threshold: clone (the Gaussian and an exact copy) when its
 *           largest scale exp(log_scale) <= scale_threshold, else split it into
 *           two children with means mu + R(q) (exp(log_scale) * z_j), z_j the
 *           caller's N(0, I) draws, log-scales reduced by log(1.6), the same
 *           rotation, opacity and SH;
 *   keep    otherwise.
 * Decisions are taken in double precision from the float32 values. */
typedef struct gs_densify_config {
    float grad_threshold;       /* units of densify_accum (pixels) */
    float scale_threshold;      /* world units */
    float min_opacity;
    int32_t max_screen_radius;  /* pixels; <= 0 disables the screen test */
} gs_densify_config;

#define GS_DENSIFY_PRUNE 0
#define GS_DENSIFY_KEEP 1
#define GS_DENSIFY_CLONE 2
#define GS_DENSIFY_SPLIT 3

/* Bytes of device workspace the densify calls need for n Gaussians (a few KB). */
size_t gs_densify_workspace_bytes(int64_t n);

/* gs_densify_plan -- the decisions and the output count.
 *   densify_accum [n] float, densify_count [n] int32 (as accumulated by the
 *   backward calls), densify_max_radius [n] int32 or NULL (then no screen test),
 *   decision [n] uint8 receives GS_DENSIFY_*, *num_out_dev (one uint64 on the
 *   device, 8-byte aligned) the number of output Gaussians: 1 per kept, 2 per
 *   cloned or split Gaussian.  workspace (16-byte aligned, caller-owned) carries
 *   the plan to gs_densify_apply and must not be touched in between.  Asynchronous. */
gs_status gs_densify_plan(const gs_params* params, const float* densify_accum, const int32_t* densify_count,
                          const int32_t* densify_max_radius, const gs_densify_config* cfg, void* workspace,
                          size_t workspace_bytes, uint8_t* decision, uint64_t* num_out_dev, void* stream);

/* gs_densify_apply -- write the planned Gaussians into new arrays, in input
 * order: a kept Gaussian once, a cloned one itself then its copy, a split one
 * child 0 then child 1.  out_params holds n_out Gaussians in the layout of
 * gs_params (SH planes of n_out rows).  adam_m / adam_v (the moments, laid out as
 * params) and out_m / out_v are all set or all NULL: surviving Gaussians keep
 * their moments, new ones (copies, children) start at zero.  split_noise [n][6]
 * float holds z_0 then z_1 for every Gaussian (read only for split ones).
 * n_out must equal the planned count (the call reads it from the workspace,
 * one 8-byte copy and wait, and returns GS_ERR_INVALID_ARG otherwise).  The
 * output arrays must not overlap the inputs. */
gs_status gs_densify_apply(const gs_params* params, const gs_params* adam_m, const gs_params* adam_v,
                           const float* split_noise, const uint8_t* decision, const void* workspace,
                           size_t workspace_bytes, int64_t n_out, gs_param_grads* out_params, gs_param_grads* out_m,
                           gs_param_grads* out_v, void* stream);

/* gs_adam -- one bias-corrected Adam step on `count` floats (gsplat guide §4.2:
 * one call per parameter group with its own lr; betas 0.9, 0.99; eps 1e-15):
 *   m = beta1 m + (1 - beta1) g;  v = beta2 v + (1 - beta2) g^2;
 *   param -= lr (m / (1 - beta1^step)) / (sqrt(v / (1 - beta2^step)) + eps).
 * step >= 1.  All four arrays 16-byte aligned. */
gs_status gs_adam(float* param, const float* grad, float* m, float* v, int64_t count, float lr, float beta1,
                  float beta2, float eps, int32_t step, void* stream);

/* gs_l1_loss_grad -- the L1 photometric term of the gsplat guide §4.1 over `count`
 * values: dL_dimage = sign(image - target) / count (sign(0) = 0), and
 * *loss_dev += mean |image - target| (one double on the device).
 * image, target, dL_dimage 16-byte aligned; loss_dev 8-byte aligned. */
gs_status gs_l1_loss_grad(const float* image, const float* target, int64_t count, float* dL_dimage,
                          double* loss_dev, void* stream);

/* Bytes of device workspace gs_l1_dssim_loss_grad needs for a width x height
 * image (72 bytes per pixel). */
size_t gs_l1_dssim_workspace_bytes(int32_t width, int32_t height);

/* gs_l1_dssim_loss_grad -- the L1 + D-SSIM photometric loss of the gsplat guide
 * §4.1, loss = l1_weight mean|image - target| + ssim_weight (1 - ssim(image,
 * target)) (the guide trains with weights 1 and 0.2), added to *loss_dev (one
 * double on the device), and its gradient with respect to the image written to
 * dL_dimage.  The pages do not define ssim: it is the standard structural
 * similarity, per channel and pixel with an 11x11 Gaussian window of standard
 * deviation 1.5 (normalised), C1 = 0.01^2, C2 = 0.03^2, the images zero outside
 * their bounds, averaged over all pixels and channels; the L1 term's gradient
 * is sign(image - target) / count with sign(0) = 0.  Double precision inside.
 *   image, target, dL_dimage [height][width][3] float (4-byte aligned);
 *   workspace (16-byte aligned, caller-owned) as sized above; loss_dev 8-byte
 *   aligned.  Asynchronous. */
gs_status gs_l1_dssim_loss_grad(const float* image, const float* target, int32_t width, int32_t height,
                                float l1_weight, float ssim_weight, void* workspace, size_t workspace_bytes,
                                float* dL_dimage, double* loss_dev, void* stream);

/* ------------------------------------------------------------ measurement
 * Diagnostics for the roofline of the compositing kernels; not part of the
 * pipeline.  The compositing stage is the one the gsplat guide §2.1 calls the
 * performance black hole; it is bound by arithmetic issue rather than by HBM,
 * so its denominators are measured instruction throughputs and its numerator
 * the work the method actually does. */

/* gs_raster_fwd_counted / gs_raster_bwd_counted -- gs_raster_fwd / gs_raster_bwd
 * (same arguments, same results, bit for bit) that also add work counters to
 * counts[0..4] (uint64 on the device, 8-byte aligned, +=):
 *   counts[0]  (pixel, entry) pairs evaluated: entries that reached a warp's
 *              pixel box (its 16x16 tile, or a 16x8 half of it) times the box's
 *              pixels (pixels outside the image included);
 *   counts[1]  pairs that did the method's work: in the forward pass the
 *              entries a pixel blended, in the reverse pass the entries a pixel
 *              takes a gradient from (the same blended set);
 *   counts[2]  list entries staged into shared memory, summed over warps;
 *   counts[3]  entries that reached a warp's box, summed over warps;
 *   counts[4]  forward pass: the pairs the method's per-pixel loop visits, for
 *              every pixel of the image its tile's list up to and including the
 *              entry at which it stops, or the whole list; reverse pass: 0 (its
 *              loop visits sum(n_contrib) pairs).
 * One atomic add per warp and counter at the warp's end. */
gs_status gs_raster_fwd_counted(const gs_projected* proj, const uint32_t* vals, const uint32_t* tile_ranges,
                                const uint32_t* tile_order, const gs_camera* cam, const float* bg_host, float* image,
                                float* final_T, int32_t* n_contrib, uint64_t* counts, void* stream);
gs_status gs_raster_bwd_counted(const gs_projected* proj, const uint32_t* vals, const uint32_t* tile_ranges,
                                const uint32_t* tile_order, const gs_camera* cam, const float* bg_host,
                                const float* final_T, const int32_t* n_contrib, const float* dL_dimage,
                                gs_grad2d* grad2d, uint64_t* counts, void* stream);

/* Instruction classes gs_alu_probe measures. */
#define GS_PROBE_FFMA 0  /* float32 fma, one per lane per instruction */
#define GS_PROBE_FFMA2 1 /* paired float32 fma of sm_100, two per lane per instruction */
#define GS_PROBE_EX2 2   /* ex2.approx.ftz.f32 (special-function unit) */
#define GS_PROBE_RCP 3   /* rcp.approx.ftz.f32 (special-function unit) */

/* Number of floats gs_alu_probe writes (one per thread of its grid). */
int64_t gs_alu_probe_slots(void);

/* gs_alu_probe -- one launch that executes `iters` (1..2^30) iterations of 8
 * independent dependency chains of instruction class `op` in every thread of a
 * grid of 8 blocks x 256 threads per SM, all in registers.  *ops_host receives
 * the operations the launch performs (flops for the fma forms, an fma counting
 * two; instructions x lanes for ex2 and rcp); the caller times the launch with
 * events on `stream`.  out: gs_alu_probe_slots() floats (4-byte aligned), the
 * chains' final values.  Asynchronous; op outside GS_PROBE_* or iters out of
 * range -> GS_ERR_INVALID_ARG. */
gs_status gs_alu_probe(int32_t op, int64_t iters, float* out, int64_t out_count, double* ops_host, void* stream);

/* Number of CUDA kernels this library has launched in the calling process
 * (a diagnostic counter, incremented on the host at every launch). */
uint64_t gs_kernel_launches(void);

/* gs_zero -- set `bytes` bytes at `ptr` to zero on the stream (clears the
 * accumulated gradient outputs between steps; a memset, nothing allocated). */
gs_status gs_zero(void* ptr, size_t bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* GS_H */
