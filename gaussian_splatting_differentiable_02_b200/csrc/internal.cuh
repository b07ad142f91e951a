// Internal declarations shared by the kernels and the C-ABI layer of libgs.so.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "gs.h"

namespace gsk {

constexpr int kTile = GS_TILE;              // 16x16 pixel tiles
constexpr int kTilePixels = kTile * kTile;  // 256
constexpr int kNumSMs = 148;                // B200

// Camera with the derived quantities every kernel needs, computed once on the
// host in double precision from the float32 fields.
struct CamArgs {
    double R[9], t[3];
    double fx, fy, cx, cy, near_plane, eps2d;
    double limx, limy;  // 1.3 x half field of view, in x/z and y/z
    double cc[3];       // camera centre -R^T t
    int W, H, TX, TY;
    int tile_cull;  // the binning emits only the tiles each footprint reaches (tile_reach.cuh)
};

CamArgs make_cam(const gs_camera& c);

inline int sh_planes(int deg) {
    switch (deg) {
        case 0: return 1;
        case 1: return 3;
        case 2: return 7;
        case 3: return 12;
        default: return 0;
    }
}

inline int tile_bits(int64_t tiles) {
    int b = 0;
    while ((int64_t(1) << b) < tiles) ++b;
    return b;
}

// ------------------------------------------------------------------ launchers
// Each returns the launch's cudaGetLastError().

// sh_half: null, or a 16-bit copy of the SH planes read instead of p.sh
cudaError_t launch_project_fwd(const gs_params& p, const CamArgs& cam, const gs_projected& out, cudaStream_t s,
                               const uint16_t* sh_half = nullptr);

// Several views (1..GS_MAX_VIEWS) of the same Gaussians in one pass; view v's
// outputs are launch_project_fwd's with cams[v] bit for bit.
cudaError_t launch_project_views(const gs_params& p, int V, const CamArgs* cams, const gs_projected* outs,
                                 cudaStream_t s, const uint16_t* sh_half = nullptr);

// float32 -> IEEE half (round to nearest even), count values
cudaError_t launch_to_half(const float* x, int64_t count, uint16_t* out, cudaStream_t s);

// One Adam step fused into the backward pass (parameters updated in place).
struct AdamStep {
    const gs_param_grads* params;  // the parameter arrays (same as gs_params), written
    const gs_param_grads* m;
    const gs_param_grads* v;
    float lr[5];  // means, quats, log_scales, opacity_logits, sh
    float beta1, beta2, eps;
    int step;
    bool sparse;  // skip Gaussians visible in no view (parameters and moments untouched)
    // 16-bit SH: the chain reads sh_half (the values the forward used) instead of the
    // float32 SH, and the updated float32 SH is written back rounded into sh_half_out
    const uint16_t* sh_half = nullptr;
    uint16_t* sh_half_out = nullptr;
};

// The packed projection: every Gaussian projected into `full` (workspace), then
// the visible ones compacted in ascending order into `capacity` packed slots.
struct PackWorkspace {
    gs_projected full;                 // [n] projection of every Gaussian
    unsigned long long* chunk_counts;  // [blocks]
    unsigned long long* total;         // [1] visible count
    int blocks;
    int64_t chunk;
};
size_t pack_workspace_layout(int64_t n, void* base, PackWorkspace* ws);
cudaError_t launch_project_packed(const gs_params& p, const CamArgs& cam, const PackWorkspace& ws,
                                  const gs_projected& packed, int64_t capacity, uint32_t* ids, int32_t* slot_of,
                                  unsigned long long* num_visible_dev, cudaStream_t s);

// Backward through the projection for V <= GS_MAX_VIEWS views of the same
// Gaussians; grads (+=) may be null when adam is given.  slots: null (projs and
// g2d indexed by Gaussian), or per view the slot of every Gaussian in the packed
// projs and g2d (-1: not in the view).
cudaError_t launch_project_bwd_views(const gs_params& p, int V, const CamArgs* cams, const gs_camera* raw,
                                     const gs_projected* projs, const int32_t* const* slots, const gs_grad2d* g2d,
                                     const gs_param_grads* grads,
                                     float* densify_accum, int32_t* densify_count, int32_t* densify_max_radius,
                                     const AdamStep* adam, cudaStream_t s);

struct SortWorkspace {
    unsigned long long* block_sums;  // [nb_emit]
    unsigned long long* total;       // [1]
    uint32_t* tkey[2];               // [max(capacity, n)] 32-bit keys, ping-pong
    uint32_t* tval[2];               // [max(capacity, n)] Gaussian indices, ping-pong
    uint32_t* hist;                  // [256][nb_sort]
    uint32_t* digit_totals;          // [256]
    uint32_t* runs;                  // culled binning (gs_camera.tile_cull), else null: [n][8] runs of tiles
    uint32_t* cnt;                   // culled binning: [n] instances per Gaussian, depth order
    int64_t nb_emit, nb_sort;
};
size_t sort_workspace_layout(int64_t n, int64_t capacity, bool cull, void* base, SortWorkspace* ws);

// Enqueues the whole binning and sort; the instance count stays on the device
// (ws.total, and *count_out when given).  K > capacity: nothing emitted, ranges empty.
cudaError_t launch_bin_sort(const gs_projected& proj, int64_t n, const CamArgs& cam, const SortWorkspace& ws,
                            uint64_t* keys, uint32_t* vals, int64_t capacity, uint32_t* ranges,
                            unsigned long long* count_out, cudaStream_t s);

// The rest of the binning from a given depth order of the Gaussians (order [n]):
// emission, the passes by tile id, ranges.
cudaError_t launch_bin_sort_ordered(const gs_projected& proj, int64_t n, const uint32_t* order, const CamArgs& cam,
                                    const SortWorkspace& ws, uint64_t* keys, uint32_t* vals, int64_t capacity,
                                    uint32_t* ranges, unsigned long long* count_out, cudaStream_t s);

// launch_bin_sort_ordered for several views (at most GS_MAX_VIEWS) of the same n
// Gaussians and tile grid in one launch per kernel: view v's projection, depth
// order, workspace, outputs and capacity at index v.
cudaError_t launch_bin_sort_ordered_views(int views, const gs_projected* projs, int64_t n,
                                          const uint32_t* const* orders, const CamArgs& cam, const SortWorkspace* ws,
                                          uint64_t* const* keys, uint32_t* const* vals, const int64_t* capacity,
                                          uint32_t* const* ranges, unsigned long long* const* count_out,
                                          cudaStream_t s);

// Stable depth order of the Gaussians of several views (at most GS_MAX_VIEWS) in
// one launch per radix pass: order [views][n].
struct DepthOrderWorkspace {
    uint32_t* key[2];        // [views][n], ping-pong
    uint32_t* val[2];        // [views][n], ping-pong
    uint32_t* hist;          // [views][256][nb]
    uint32_t* digit_totals;  // [views][256]
    int64_t nb;
};
size_t depth_order_workspace_layout(int64_t n, int views, void* base, DepthOrderWorkspace* ws);
cudaError_t launch_depth_order(const gs_projected* projs, int views, int64_t n, const DepthOrderWorkspace& ws,
                               uint32_t* order, cudaStream_t s);

cudaError_t launch_tile_order(const uint32_t* ranges, int tiles, uint32_t* order, cudaStream_t s);
cudaError_t launch_tile_order_views(int views, const uint32_t* const* ranges, int tiles, uint32_t* const* order,
                                    cudaStream_t s);

// The L1 term fused into the forward pass (gs_raster_fwd_l1).
struct L1Out {
    const float* target;  // [H][W][3]
    float* dL_dimage;     // [H][W][3]
    double* loss;         // += mean |image - target|
};

cudaError_t launch_raster_fwd(const gs_projected& proj, const uint32_t* vals, const uint32_t* ranges,
                              const uint32_t* order, const CamArgs& cam, const float bg[3], float* image,
                              float* final_T, int32_t* n_contrib, cudaStream_t s,
                              unsigned long long* counts = nullptr, const L1Out* l1 = nullptr);

cudaError_t launch_raster_bwd(const gs_projected& proj, const uint32_t* vals, const uint32_t* ranges,
                              const uint32_t* order, const CamArgs& cam, const float bg[3], const float* final_T,
                              const int32_t* n_contrib, const float* dL_dimage, const gs_grad2d& g2,
                              cudaStream_t s, unsigned long long* counts = nullptr);

cudaError_t launch_adam(float* param, const float* grad, float* m, float* v, int64_t count, float lr, float beta1,
                        float beta2, float eps, int32_t step, cudaStream_t s);

cudaError_t launch_l1(const float* image, const float* target, int64_t count, float* dL, double* loss,
                      cudaStream_t s);

struct DensifyWorkspace {
    unsigned long long* chunk_counts;  // [blocks]: output count per chunk, then its offset
    unsigned long long* total;         // [1]
    int blocks;
    int64_t chunk;
};
size_t densify_workspace_layout(int64_t n, void* base, DensifyWorkspace* ws);

cudaError_t launch_densify_plan(const gs_params& p, const float* accum, const int32_t* count,
                                const int32_t* max_radius, const gs_densify_config& cfg,
                                const DensifyWorkspace& ws, uint8_t* decision, uint64_t* num_out_dev,
                                cudaStream_t s);

cudaError_t launch_densify_apply(const gs_params& p, const gs_params* m, const gs_params* v, const float* noise,
                                 const uint8_t* decision, const DensifyWorkspace& ws, int64_t n_out,
                                 const gs_param_grads& op, const gs_param_grads* om, const gs_param_grads* ov,
                                 double log_split, cudaStream_t s);

// maps: [9][H][W] doubles of workspace
cudaError_t launch_l1_dssim(const float* image, const float* target, int W, int H, float l1_weight,
                            float ssim_weight, double* maps, float* dL, double* loss, cudaStream_t s);

// host-side count of kernel launches (gs_kernel_launches)
void count_launches(int k);

// record a failure for gs_last_error_detail() and return `st`
gs_status fail_detail(gs_status st, const char* fmt, ...);

// grid size: a multiple of the SM count, capped by the work
inline unsigned grid_for(int64_t work, int block, int per_sm = 8) {
    int64_t g = (work + block - 1) / block;
    int64_t cap = int64_t(kNumSMs) * per_sm;
    if (g > cap) g = cap;
    if (g < 1) g = 1;
    return unsigned(g);
}

}  // namespace gsk
