// C-ABI entry points of libgs.so (declared in gs.h): argument checks on the
// host, then the kernel launches.  Nothing here allocates device memory.
#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "internal.cuh"

namespace gsk {

namespace {
std::atomic<uint64_t> g_launches{0};
}

void count_launches(int k) { g_launches.fetch_add(uint64_t(k), std::memory_order_relaxed); }

CamArgs make_cam(const gs_camera& c) {
    CamArgs k;
    for (int i = 0; i < 9; ++i) k.R[i] = c.R[i];
    for (int i = 0; i < 3; ++i) k.t[i] = c.t[i];
    k.fx = c.fx;
    k.fy = c.fy;
    k.cx = c.cx;
    k.cy = c.cy;
    k.near_plane = c.near_plane;
    k.eps2d = c.eps2d;
    k.W = c.width;
    k.H = c.height;
    k.TX = (c.width + kTile - 1) / kTile;
    k.TY = (c.height + kTile - 1) / kTile;
    k.tile_cull = c.tile_cull;
    k.limx = 1.3 * (0.5 * double(c.width) / k.fx);
    k.limy = 1.3 * (0.5 * double(c.height) / k.fy);
    for (int j = 0; j < 3; ++j) k.cc[j] = -((k.R[0 + j] * k.t[0] + k.R[3 + j] * k.t[1]) + k.R[6 + j] * k.t[2]);
    return k;
}

}  // namespace gsk

namespace {

thread_local char g_detail[512] = "";

gs_status fail(gs_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_detail, sizeof g_detail, fmt, ap);
    va_end(ap);
    return st;
}

gs_status ok() {
    g_detail[0] = '\0';
    return GS_OK;
}

}  // namespace

gs_status gsk::fail_detail(gs_status st, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_detail, sizeof g_detail, fmt, ap);
    va_end(ap);
    return st;
}

namespace {

gs_status cuda_status(cudaError_t e, const char* where) {
    if (e == cudaSuccess) return ok();
    return fail(GS_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

#define CHECK_PTR(p, align)                                                                      \
    do {                                                                                         \
        if ((p) == nullptr) return fail(GS_ERR_INVALID_ARG, "%s: %s is NULL", fn, #p);           \
        if (!aligned((p), (align)))                                                              \
            return fail(GS_ERR_INVALID_ARG, "%s: %s is not %d-byte aligned", fn, #p, int(align)); \
    } while (0)

gs_status check_camera(const char* fn, const gs_camera* cam) {
    if (!cam) return fail(GS_ERR_INVALID_ARG, "%s: camera is NULL", fn);
    if (cam->width <= 0 || cam->height <= 0 || cam->width > 16384 || cam->height > 16384)
        return fail(GS_ERR_UNSUPPORTED, "%s: image %dx%d outside 1..16384", fn, cam->width, cam->height);
    const float f[] = {cam->fx, cam->fy, cam->cx, cam->cy, cam->near_plane, cam->eps2d};
    for (float v : f)
        if (!std::isfinite(v)) return fail(GS_ERR_INVALID_ARG, "%s: non-finite camera intrinsics", fn);
    for (int i = 0; i < 9; ++i)
        if (!std::isfinite(cam->R[i])) return fail(GS_ERR_INVALID_ARG, "%s: non-finite camera rotation", fn);
    for (int i = 0; i < 3; ++i)
        if (!std::isfinite(cam->t[i])) return fail(GS_ERR_INVALID_ARG, "%s: non-finite camera translation", fn);
    if (!(cam->fx > 0.f) || !(cam->fy > 0.f)) return fail(GS_ERR_INVALID_ARG, "%s: focal lengths must be > 0", fn);
    if (!(cam->near_plane > 0.f)) return fail(GS_ERR_INVALID_ARG, "%s: near_plane must be > 0", fn);
    if (!(cam->eps2d >= 0.f)) return fail(GS_ERR_INVALID_ARG, "%s: eps2d must be >= 0", fn);
    if (cam->tile_cull != 0 && cam->tile_cull != 1)
        return fail(GS_ERR_INVALID_ARG, "%s: tile_cull must be 0 or 1", fn);
    return GS_OK;
}

gs_status check_params(const char* fn, const gs_params* p, bool need_sh = true) {
    if (!p) return fail(GS_ERR_INVALID_ARG, "%s: params is NULL", fn);
    if (p->n < 0 || p->n > 0x7fffffffLL) return fail(GS_ERR_INVALID_ARG, "%s: n = %lld out of range", fn, (long long)p->n);
    if (p->sh_degree < 0 || p->sh_degree > 3)
        return fail(GS_ERR_UNSUPPORTED, "%s: SH degree %d (0..3 supported)", fn, int(p->sh_degree));
    if (p->n == 0) return GS_OK;
    CHECK_PTR(p->means, 16);
    CHECK_PTR(p->quats, 16);
    CHECK_PTR(p->log_scales, 16);
    CHECK_PTR(p->opacity_logits, 4);
    if (need_sh) CHECK_PTR(p->sh, 16);
    return GS_OK;
}

gs_status check_projected(const char* fn, const gs_projected* o, int64_t n, bool need_all) {
    if (!o) return fail(GS_ERR_INVALID_ARG, "%s: projected is NULL", fn);
    if (n == 0) return GS_OK;
    CHECK_PTR(o->xy, 8);
    CHECK_PTR(o->conic_opacity, 16);
    CHECK_PTR(o->rgb, 16);
    CHECK_PTR(o->radius, 4);
    if (need_all) {
        CHECK_PTR(o->depth, 4);
        CHECK_PTR(o->rect, 8);
        CHECK_PTR(o->tiles_touched, 4);
    }
    return GS_OK;
}

}  // namespace

extern "C" {

const char* gs_status_string(gs_status s) {
    switch (s) {
        case GS_OK: return "GS_OK";
        case GS_ERR_INVALID_ARG: return "GS_ERR_INVALID_ARG: invalid argument";
        case GS_ERR_UNSUPPORTED: return "GS_ERR_UNSUPPORTED: unsupported configuration";
        case GS_ERR_CAPACITY: return "GS_ERR_CAPACITY: instance buffer too small";
        case GS_ERR_CUDA: return "GS_ERR_CUDA: CUDA error";
        default: return "unknown gs_status";
    }
}

const char* gs_last_error_detail(void) { return g_detail; }

int32_t gs_sh_planes(int32_t sh_degree) { return gsk::sh_planes(sh_degree); }

gs_status gs_tile_grid(const gs_camera* cam, int32_t* tiles_x_host, int32_t* tiles_y_host) {
    const char* fn = "gs_tile_grid";
    gs_status st = check_camera(fn, cam);
    if (st != GS_OK) return st;
    if (!tiles_x_host || !tiles_y_host) return fail(GS_ERR_INVALID_ARG, "%s: NULL output", fn);
    *tiles_x_host = (cam->width + GS_TILE - 1) / GS_TILE;
    *tiles_y_host = (cam->height + GS_TILE - 1) / GS_TILE;
    return ok();
}

gs_status gs_project_sh16(const gs_params* params, const uint16_t* sh_half, const gs_camera* cam, gs_projected* out,
                          void* stream) {
    const char* fn = "gs_project_sh16";
    gs_status st;
    if ((st = check_params(fn, params, false)) != GS_OK) return st;
    if ((st = check_camera(fn, cam)) != GS_OK) return st;
    if ((st = check_projected(fn, out, params->n, true)) != GS_OK) return st;
    if (params->n > 0) CHECK_PTR(sh_half, 8);
    const gsk::CamArgs c = gsk::make_cam(*cam);
    return cuda_status(gsk::launch_project_fwd(*params, c, *out, static_cast<cudaStream_t>(stream), sh_half), fn);
}

gs_status gs_to_half(const float* x, int64_t count, uint16_t* out, void* stream) {
    const char* fn = "gs_to_half";
    if (count < 0) return fail(GS_ERR_INVALID_ARG, "%s: count < 0", fn);
    if (count == 0) return ok();
    CHECK_PTR(x, 16);
    CHECK_PTR(out, 8);
    return cuda_status(gsk::launch_to_half(x, count, out, static_cast<cudaStream_t>(stream)), fn);
}

gs_status gs_project(const gs_params* params, const gs_camera* cam, gs_projected* out, void* stream) {
    const char* fn = "gs_project";
    gs_status st;
    if ((st = check_params(fn, params)) != GS_OK) return st;
    if ((st = check_camera(fn, cam)) != GS_OK) return st;
    if ((st = check_projected(fn, out, params->n, true)) != GS_OK) return st;
    const gsk::CamArgs c = gsk::make_cam(*cam);
    return cuda_status(gsk::launch_project_fwd(*params, c, *out, static_cast<cudaStream_t>(stream)), fn);
}

gs_status gs_project_views(const gs_params* params, int32_t num_views, const gs_camera* cams, gs_projected* outs,
                           const uint16_t* sh_half, void* stream) {
    const char* fn = "gs_project_views";
    gs_status st;
    if ((st = check_params(fn, params, sh_half == nullptr)) != GS_OK) return st;
    if (num_views < 1 || num_views > GS_MAX_VIEWS)
        return fail(GS_ERR_INVALID_ARG, "%s: num_views %d outside 1..%d", fn, int(num_views), GS_MAX_VIEWS);
    if (!cams || !outs) return fail(GS_ERR_INVALID_ARG, "%s: cams or outs is NULL", fn);
    if (sh_half && params->n > 0) CHECK_PTR(sh_half, 8);
    gsk::CamArgs c[GS_MAX_VIEWS];
    for (int v = 0; v < num_views; ++v) {
        if ((st = check_camera(fn, cams + v)) != GS_OK) return st;
        if ((st = check_projected(fn, outs + v, params->n, true)) != GS_OK) return st;
        c[v] = gsk::make_cam(cams[v]);
    }
    return cuda_status(
        gsk::launch_project_views(*params, num_views, c, outs, static_cast<cudaStream_t>(stream), sh_half), fn);
}

size_t gs_bin_sort_workspace_bytes(int64_t n, int64_t capacity, const gs_camera* cam) {
    if (n < 0) n = 0;
    if (capacity < 0) capacity = 0;
    return gsk::sort_workspace_layout(n, capacity, cam && cam->tile_cull == 1, nullptr, nullptr);
}

}  // extern "C"

namespace {

// Checks and launch of the binning + sort.  With num_instances_host the call
// waits for K and reports GS_ERR_CAPACITY; with count_dev it returns at once.
gs_status bin_sort_impl(const char* fn, const gs_projected* proj, int64_t n, const gs_camera* cam, void* workspace,
                        size_t workspace_bytes, uint64_t* keys, uint32_t* vals, int64_t capacity,
                        int64_t* num_instances_host, unsigned long long* count_dev, uint32_t* tile_ranges,
                        void* stream, const uint32_t* order = nullptr) {
    gs_status st;
    if (n < 0 || n > 0x7fffffffLL) return fail(GS_ERR_INVALID_ARG, "%s: n out of range", fn);
    if (capacity < 0 || capacity > 0xffffffffLL) return fail(GS_ERR_INVALID_ARG, "%s: capacity out of range", fn);
    if ((st = check_camera(fn, cam)) != GS_OK) return st;
    if ((st = check_projected(fn, proj, n, true)) != GS_OK) return st;
    if (!num_instances_host && !count_dev) return fail(GS_ERR_INVALID_ARG, "%s: instance count output is NULL", fn);
    if (count_dev) CHECK_PTR(count_dev, 8);
    CHECK_PTR(workspace, 16);
    CHECK_PTR(tile_ranges, 8);
    if (capacity > 0) {
        CHECK_PTR(keys, 8);
        CHECK_PTR(vals, 4);
    }
    const size_t need = gsk::sort_workspace_layout(n, capacity, cam->tile_cull == 1, nullptr, nullptr);
    if (workspace_bytes < need)
        return fail(GS_ERR_INVALID_ARG, "%s: workspace of %zu bytes, %zu needed", fn, workspace_bytes, need);
    const int64_t tiles = int64_t((cam->width + GS_TILE - 1) / GS_TILE) * ((cam->height + GS_TILE - 1) / GS_TILE);
    if (tiles > (int64_t(1) << 20)) return fail(GS_ERR_UNSUPPORTED, "%s: more than 2^20 tiles", fn);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    gsk::SortWorkspace ws;
    gsk::sort_workspace_layout(n, capacity, cam->tile_cull == 1, workspace, &ws);
    const gsk::CamArgs c = gsk::make_cam(*cam);
    cudaError_t e = order ? gsk::launch_bin_sort_ordered(*proj, n, order, c, ws, keys, vals, capacity, tile_ranges,
                                                         count_dev, s)
                          : gsk::launch_bin_sort(*proj, n, c, ws, keys, vals, capacity, tile_ranges, count_dev, s);
    if (e != cudaSuccess) return cuda_status(e, fn);
    if (!num_instances_host) return ok();
    unsigned long long K = 0;
    e = cudaMemcpyAsync(&K, ws.total, sizeof K, cudaMemcpyDeviceToHost, s);
    if (e == cudaSuccess) e = cudaStreamSynchronize(s);
    if (e != cudaSuccess) return cuda_status(e, fn);
    *num_instances_host = int64_t(K);
    if (int64_t(K) > capacity)
        return fail(GS_ERR_CAPACITY, "%s: %llu instances, capacity %lld", fn, K, (long long)capacity);
    return ok();
}

}  // namespace

extern "C" {

gs_status gs_bin_sort(const gs_projected* proj, int64_t n, const gs_camera* cam, void* workspace,
                      size_t workspace_bytes, uint64_t* keys, uint32_t* vals, int64_t capacity,
                      int64_t* num_instances_host, uint32_t* tile_ranges, void* stream) {
    if (!num_instances_host) return fail(GS_ERR_INVALID_ARG, "gs_bin_sort: num_instances_host is NULL");
    return bin_sort_impl("gs_bin_sort", proj, n, cam, workspace, workspace_bytes, keys, vals, capacity,
                         num_instances_host, nullptr, tile_ranges, stream);
}

gs_status gs_bin_sort_async(const gs_projected* proj, int64_t n, const gs_camera* cam, void* workspace,
                            size_t workspace_bytes, uint64_t* keys, uint32_t* vals, int64_t capacity,
                            uint64_t* num_instances_dev, uint32_t* tile_ranges, void* stream) {
    if (!num_instances_dev) return fail(GS_ERR_INVALID_ARG, "gs_bin_sort_async: num_instances_dev is NULL");
    return bin_sort_impl("gs_bin_sort_async", proj, n, cam, workspace, workspace_bytes, keys, vals, capacity,
                         nullptr, reinterpret_cast<unsigned long long*>(num_instances_dev), tile_ranges, stream);
}

gs_status gs_bin_sort_ordered_async(const gs_projected* proj, int64_t n, const uint32_t* order, const gs_camera* cam,
                                    void* workspace, size_t workspace_bytes, uint64_t* keys, uint32_t* vals,
                                    int64_t capacity, uint64_t* num_instances_dev, uint32_t* tile_ranges,
                                    void* stream) {
    const char* fn = "gs_bin_sort_ordered_async";
    if (!num_instances_dev) return fail(GS_ERR_INVALID_ARG, "%s: num_instances_dev is NULL", fn);
    if (n > 0 && !order) return fail(GS_ERR_INVALID_ARG, "%s: order is NULL", fn);
    if (n > 0) CHECK_PTR(order, 4);
    return bin_sort_impl(fn, proj, n, cam, workspace, workspace_bytes, keys, vals, capacity, nullptr,
                         reinterpret_cast<unsigned long long*>(num_instances_dev), tile_ranges, stream,
                         n > 0 ? order : nullptr);
}

gs_status gs_bin_sort_ordered_views_async(const gs_projected* projs, int32_t num_views, int64_t n,
                                          const uint32_t* orders, const gs_camera* cams, void* const* workspaces,
                                          const size_t* workspace_bytes, uint64_t* const* keys, uint32_t* const* vals,
                                          const int64_t* capacities, uint64_t* const* num_instances_dev,
                                          uint32_t* const* tile_ranges, void* stream) {
    const char* fn = "gs_bin_sort_ordered_views_async";
    if (num_views < 1 || num_views > GS_MAX_VIEWS)
        return fail(GS_ERR_INVALID_ARG, "%s: num_views = %d (1..%d)", fn, int(num_views), GS_MAX_VIEWS);
    if (!projs || !cams || !workspaces || !workspace_bytes || !keys || !vals || !capacities || !num_instances_dev ||
        !tile_ranges)
        return fail(GS_ERR_INVALID_ARG, "%s: a per-view array is NULL", fn);
    if (n < 0 || n > 0x7fffffffLL) return fail(GS_ERR_INVALID_ARG, "%s: n out of range", fn);
    if (n > 0) {
        if (!orders) return fail(GS_ERR_INVALID_ARG, "%s: orders is NULL", fn);
        CHECK_PTR(orders, 4);
    }
    gs_status st;
    gsk::SortWorkspace ws[GS_MAX_VIEWS];
    const uint32_t* ord[GS_MAX_VIEWS];
    unsigned long long* cnt[GS_MAX_VIEWS];
    for (int v = 0; v < num_views; ++v) {
        const int64_t capacity = capacities[v];
        if (capacity < 0 || capacity > 0xffffffffLL)
            return fail(GS_ERR_INVALID_ARG, "%s: capacity of view %d out of range", fn, v);
        if ((st = check_camera(fn, cams + v)) != GS_OK) return st;
        if (cams[v].width != cams[0].width || cams[v].height != cams[0].height)
            return fail(GS_ERR_INVALID_ARG, "%s: view %d has another image size than view 0", fn, v);
        if ((st = check_projected(fn, projs + v, n, true)) != GS_OK) return st;
        CHECK_PTR(num_instances_dev[v], 8);
        CHECK_PTR(workspaces[v], 16);
        CHECK_PTR(tile_ranges[v], 8);
        if (capacity > 0) {
            CHECK_PTR(keys[v], 8);
            CHECK_PTR(vals[v], 4);
        }
        const bool cull = cams[v].tile_cull == 1;
        const size_t need = gsk::sort_workspace_layout(n, capacity, cull, nullptr, nullptr);
        if (workspace_bytes[v] < need)
            return fail(GS_ERR_INVALID_ARG, "%s: workspace of view %d has %zu bytes, %zu needed", fn, v,
                        workspace_bytes[v], need);
        gsk::sort_workspace_layout(n, capacity, cull, workspaces[v], &ws[v]);
        ord[v] = n > 0 ? orders + int64_t(v) * n : nullptr;
        cnt[v] = reinterpret_cast<unsigned long long*>(num_instances_dev[v]);
    }
    const gs_camera* cam = cams;
    const int64_t tiles = int64_t((cam->width + GS_TILE - 1) / GS_TILE) * ((cam->height + GS_TILE - 1) / GS_TILE);
    if (tiles > (int64_t(1) << 20)) return fail(GS_ERR_UNSUPPORTED, "%s: more than 2^20 tiles", fn);
    const gsk::CamArgs c = gsk::make_cam(*cam);
    return cuda_status(gsk::launch_bin_sort_ordered_views(num_views, projs, n, ord, c, ws, keys, vals, capacities,
                                                          tile_ranges, cnt, static_cast<cudaStream_t>(stream)),
                       fn);
}

size_t gs_depth_order_workspace_bytes(int64_t n, int32_t num_views) {
    if (n < 0) n = 0;
    if (num_views < 1) num_views = 1;
    return gsk::depth_order_workspace_layout(n, num_views, nullptr, nullptr);
}

gs_status gs_depth_order_views(const gs_projected* projs, int32_t num_views, int64_t n, void* workspace,
                               size_t workspace_bytes, uint32_t* order, void* stream) {
    const char* fn = "gs_depth_order_views";
    if (num_views < 1 || num_views > GS_MAX_VIEWS)
        return fail(GS_ERR_INVALID_ARG, "%s: num_views = %d (1..%d)", fn, int(num_views), GS_MAX_VIEWS);
    if (n < 0 || n > 0x7fffffffLL) return fail(GS_ERR_INVALID_ARG, "%s: n out of range", fn);
    if (!projs) return fail(GS_ERR_INVALID_ARG, "%s: projs is NULL", fn);
    CHECK_PTR(workspace, 16);
    if (workspace_bytes < gs_depth_order_workspace_bytes(n, num_views))
        return fail(GS_ERR_INVALID_ARG, "%s: workspace of %zu bytes, %zu needed", fn, workspace_bytes,
                    gs_depth_order_workspace_bytes(n, num_views));
    if (n > 0) {
        CHECK_PTR(order, 4);
        for (int v = 0; v < num_views; ++v) {
            CHECK_PTR(projs[v].tiles_touched, 4);
            CHECK_PTR(projs[v].depth, 4);
        }
    }
    gsk::DepthOrderWorkspace ws;
    gsk::depth_order_workspace_layout(n, num_views, workspace, &ws);
    return cuda_status(gsk::launch_depth_order(projs, num_views, n, ws, order, static_cast<cudaStream_t>(stream)), fn);
}

gs_status gs_tile_order(const uint32_t* tile_ranges, const gs_camera* cam, uint32_t* tile_order, void* stream) {
    const char* fn = "gs_tile_order";
    gs_status st;
    if ((st = check_camera(fn, cam)) != GS_OK) return st;
    CHECK_PTR(tile_ranges, 8);
    CHECK_PTR(tile_order, 4);
    const gsk::CamArgs c = gsk::make_cam(*cam);
    return cuda_status(gsk::launch_tile_order(tile_ranges, c.TX * c.TY, tile_order, static_cast<cudaStream_t>(stream)),
                       fn);
}

gs_status gs_tile_order_views(int32_t num_views, const uint32_t* const* tile_ranges, const gs_camera* cam,
                              uint32_t* const* tile_orders, void* stream) {
    const char* fn = "gs_tile_order_views";
    gs_status st;
    if (num_views < 1 || num_views > GS_MAX_VIEWS)
        return fail(GS_ERR_INVALID_ARG, "%s: num_views = %d (1..%d)", fn, int(num_views), GS_MAX_VIEWS);
    if ((st = check_camera(fn, cam)) != GS_OK) return st;
    if (!tile_ranges || !tile_orders) return fail(GS_ERR_INVALID_ARG, "%s: a per-view array is NULL", fn);
    for (int v = 0; v < num_views; ++v) {
        CHECK_PTR(tile_ranges[v], 8);
        CHECK_PTR(tile_orders[v], 4);
    }
    const gsk::CamArgs c = gsk::make_cam(*cam);
    return cuda_status(gsk::launch_tile_order_views(num_views, tile_ranges, c.TX * c.TY, tile_orders,
                                                    static_cast<cudaStream_t>(stream)),
                       fn);
}

}  // extern "C"

namespace {

gs_status raster_fwd_common(const char* fn, const gs_projected* proj, const uint32_t* vals,
                            const uint32_t* tile_ranges, const uint32_t* tile_order, const gs_camera* cam,
                            const float* bg_host, float* image, float* final_T, int32_t* n_contrib,
                            unsigned long long* counts, void* stream, const gsk::L1Out* l1 = nullptr) {
    gs_status st;
    if ((st = check_camera(fn, cam)) != GS_OK) return st;
    if ((st = check_projected(fn, proj, 1, false)) != GS_OK) return st;
    if (!bg_host) return fail(GS_ERR_INVALID_ARG, "%s: bg_host is NULL", fn);
    CHECK_PTR(vals, 4);
    CHECK_PTR(tile_ranges, 8);
    if (tile_order) CHECK_PTR(tile_order, 4);
    CHECK_PTR(image, 4);
    CHECK_PTR(final_T, 4);
    CHECK_PTR(n_contrib, 4);
    if (l1) {
        CHECK_PTR(l1->target, 4);
        CHECK_PTR(l1->dL_dimage, 4);
        CHECK_PTR(l1->loss, 8);
    }
    const gsk::CamArgs c = gsk::make_cam(*cam);
    return cuda_status(gsk::launch_raster_fwd(*proj, vals, tile_ranges, tile_order, c, bg_host, image, final_T,
                                              n_contrib, static_cast<cudaStream_t>(stream), counts, l1),
                       fn);
}

gs_status raster_bwd_common(const char* fn, const gs_projected* proj, const uint32_t* vals,
                            const uint32_t* tile_ranges, const uint32_t* tile_order, const gs_camera* cam,
                            const float* bg_host, const float* final_T, const int32_t* n_contrib,
                            const float* dL_dimage, gs_grad2d* grad2d, unsigned long long* counts, void* stream) {
    gs_status st;
    if ((st = check_camera(fn, cam)) != GS_OK) return st;
    if ((st = check_projected(fn, proj, 1, false)) != GS_OK) return st;
    if (!bg_host) return fail(GS_ERR_INVALID_ARG, "%s: bg_host is NULL", fn);
    if (!grad2d) return fail(GS_ERR_INVALID_ARG, "%s: grad2d is NULL", fn);
    CHECK_PTR(vals, 4);
    CHECK_PTR(tile_ranges, 8);
    if (tile_order) CHECK_PTR(tile_order, 4);
    CHECK_PTR(final_T, 4);
    CHECK_PTR(n_contrib, 4);
    CHECK_PTR(dL_dimage, 4);
    CHECK_PTR(grad2d->xy, 8);
    CHECK_PTR(grad2d->conic_opacity, 16);
    CHECK_PTR(grad2d->rgb, 16);
    if (grad2d->xy_abs) CHECK_PTR(grad2d->xy_abs, 8);
    const gsk::CamArgs c = gsk::make_cam(*cam);
    return cuda_status(gsk::launch_raster_bwd(*proj, vals, tile_ranges, tile_order, c, bg_host, final_T, n_contrib,
                                              dL_dimage, *grad2d, static_cast<cudaStream_t>(stream), counts),
                       fn);
}

}  // namespace

extern "C" {

gs_status gs_raster_fwd(const gs_projected* proj, const uint32_t* vals, const uint32_t* tile_ranges,
                        const uint32_t* tile_order, const gs_camera* cam, const float* bg_host, float* image,
                        float* final_T, int32_t* n_contrib, void* stream) {
    return raster_fwd_common("gs_raster_fwd", proj, vals, tile_ranges, tile_order, cam, bg_host, image, final_T,
                             n_contrib, nullptr, stream);
}

gs_status gs_raster_fwd_l1(const gs_projected* proj, const uint32_t* vals, const uint32_t* tile_ranges,
                           const uint32_t* tile_order, const gs_camera* cam, const float* bg_host, const float* target,
                           float* image, float* final_T, int32_t* n_contrib, float* dL_dimage, double* loss_dev,
                           void* stream) {
    const gsk::L1Out l1{target, dL_dimage, loss_dev};
    return raster_fwd_common("gs_raster_fwd_l1", proj, vals, tile_ranges, tile_order, cam, bg_host, image, final_T,
                             n_contrib, nullptr, stream, &l1);
}

gs_status gs_raster_bwd(const gs_projected* proj, const uint32_t* vals, const uint32_t* tile_ranges,
                        const uint32_t* tile_order, const gs_camera* cam, const float* bg_host, const float* final_T,
                        const int32_t* n_contrib, const float* dL_dimage, gs_grad2d* grad2d, void* stream) {
    return raster_bwd_common("gs_raster_bwd", proj, vals, tile_ranges, tile_order, cam, bg_host, final_T, n_contrib,
                             dL_dimage, grad2d, nullptr, stream);
}

gs_status gs_raster_fwd_counted(const gs_projected* proj, const uint32_t* vals, const uint32_t* tile_ranges,
                                const uint32_t* tile_order, const gs_camera* cam, const float* bg_host, float* image,
                                float* final_T, int32_t* n_contrib, uint64_t* counts, void* stream) {
    const char* fn = "gs_raster_fwd_counted";
    CHECK_PTR(counts, 8);
    return raster_fwd_common(fn, proj, vals, tile_ranges, tile_order, cam, bg_host, image, final_T, n_contrib,
                             reinterpret_cast<unsigned long long*>(counts), stream);
}

gs_status gs_raster_bwd_counted(const gs_projected* proj, const uint32_t* vals, const uint32_t* tile_ranges,
                                const uint32_t* tile_order, const gs_camera* cam, const float* bg_host,
                                const float* final_T, const int32_t* n_contrib, const float* dL_dimage,
                                gs_grad2d* grad2d, uint64_t* counts, void* stream) {
    const char* fn = "gs_raster_bwd_counted";
    CHECK_PTR(counts, 8);
    return raster_bwd_common(fn, proj, vals, tile_ranges, tile_order, cam, bg_host, final_T, n_contrib, dL_dimage,
                             grad2d, reinterpret_cast<unsigned long long*>(counts), stream);
}

}  // extern "C"

namespace {

gs_status check_grad_arrays(const char* fn, const gs_param_grads* g, const char* what) {
    if (!g) return fail(GS_ERR_INVALID_ARG, "%s: %s is NULL", fn, what);
    CHECK_PTR(g->means, 16);
    CHECK_PTR(g->quats, 16);
    CHECK_PTR(g->log_scales, 16);
    CHECK_PTR(g->opacity_logits, 4);
    CHECK_PTR(g->sh, 16);
    return GS_OK;
}

// Shared checks and launch of the (multi-view) backward through the projection.
gs_status project_bwd_common(const char* fn, const gs_params* params, int32_t num_views, const gs_camera* cams,
                             const gs_projected* projs, const gs_grad2d* grad2d, gs_param_grads* grads,
                             float* densify_accum, int32_t* densify_count, int32_t* densify_max_radius,
                             const gsk::AdamStep* adam, void* stream, const int32_t* const* slots = nullptr,
                             bool packed = false) {
    gs_status st;
    if ((st = check_params(fn, params)) != GS_OK) return st;
    if (num_views < 1 || num_views > GS_MAX_VIEWS)
        return fail(GS_ERR_INVALID_ARG, "%s: num_views = %d (1..%d)", fn, int(num_views), GS_MAX_VIEWS);
    if (!cams || !projs || !grad2d) return fail(GS_ERR_INVALID_ARG, "%s: cams, projs or grad2d is NULL", fn);
    if ((densify_accum == nullptr) != (densify_count == nullptr))
        return fail(GS_ERR_INVALID_ARG, "%s: densify_accum and densify_count must both be set or both NULL", fn);
    if (!grads && !adam) return fail(GS_ERR_INVALID_ARG, "%s: grads is NULL", fn);
    gsk::CamArgs c[GS_MAX_VIEWS];
    for (int v = 0; v < num_views; ++v) {
        if ((st = check_camera(fn, cams + v)) != GS_OK) return st;
        c[v] = gsk::make_cam(cams[v]);
        if (params->n > 0) {
            if (packed) {
                if (!slots) return fail(GS_ERR_INVALID_ARG, "%s: slot_of is NULL", fn);
                CHECK_PTR(slots[v], 4);
            }
            CHECK_PTR(projs[v].radius, 4);
            CHECK_PTR(grad2d[v].xy, 8);
            CHECK_PTR(grad2d[v].conic_opacity, 16);
            CHECK_PTR(grad2d[v].rgb, 16);
            if (grad2d[v].xy_abs) CHECK_PTR(grad2d[v].xy_abs, 8);
        }
    }
    if (params->n > 0) {
        if (grads && (st = check_grad_arrays(fn, grads, "grads")) != GS_OK) return st;
        if (densify_accum) {
            CHECK_PTR(densify_accum, 4);
            CHECK_PTR(densify_count, 4);
        }
        if (densify_max_radius) CHECK_PTR(densify_max_radius, 4);
        if (adam) {
            if ((st = check_grad_arrays(fn, adam->params, "params_inout")) != GS_OK) return st;
            if ((st = check_grad_arrays(fn, adam->m, "adam_m")) != GS_OK) return st;
            if ((st = check_grad_arrays(fn, adam->v, "adam_v")) != GS_OK) return st;
        }
    }
    return cuda_status(gsk::launch_project_bwd_views(*params, num_views, c, cams, projs, packed ? slots : nullptr,
                                                     grad2d, grads, densify_accum,
                                                     densify_count, densify_max_radius, adam,
                                                     static_cast<cudaStream_t>(stream)),
                       fn);
}

gs_status check_adam_hyper(const char* fn, float lr, float beta1, float beta2, float eps, int32_t step) {
    if (step < 1) return fail(GS_ERR_INVALID_ARG, "%s: step must be >= 1", fn);
    if (!std::isfinite(lr) || !(beta1 >= 0.f && beta1 < 1.f) || !(beta2 >= 0.f && beta2 < 1.f) || !(eps >= 0.f))
        return fail(GS_ERR_INVALID_ARG, "%s: invalid hyper-parameters", fn);
    return GS_OK;
}

}  // namespace

extern "C" {

gs_status gs_project_bwd(const gs_params* params, const gs_camera* cam, const gs_projected* proj,
                         const gs_grad2d* grad2d, gs_param_grads* grads, float* densify_accum,
                         int32_t* densify_count, int32_t* densify_max_radius, void* stream) {
    const char* fn = "gs_project_bwd";
    if (!grads) return fail(GS_ERR_INVALID_ARG, "%s: grads is NULL", fn);
    return project_bwd_common(fn, params, 1, cam, proj, grad2d, grads, densify_accum, densify_count,
                              densify_max_radius, nullptr, stream);
}

gs_status gs_project_bwd_views(const gs_params* params, int32_t num_views, const gs_camera* cams,
                               const gs_projected* projs, const gs_grad2d* grad2d, gs_param_grads* grads,
                               float* densify_accum, int32_t* densify_count, int32_t* densify_max_radius,
                               void* stream) {
    const char* fn = "gs_project_bwd_views";
    if (!grads) return fail(GS_ERR_INVALID_ARG, "%s: grads is NULL", fn);
    return project_bwd_common(fn, params, num_views, cams, projs, grad2d, grads, densify_accum, densify_count,
                              densify_max_radius, nullptr, stream);
}

}  // extern "C"

namespace {

gs_status project_bwd_adam_common(const char* fn, const gs_params* params, int32_t num_views, const gs_camera* cams,
                                  const gs_projected* projs, const int32_t* const* slots, bool packed,
                                  const gs_grad2d* grad2d, gs_param_grads* params_inout, gs_param_grads* adam_m,
                                  gs_param_grads* adam_v, const float* lr_host, float beta1, float beta2, float eps,
                                  int32_t step, gs_param_grads* grads, float* densify_accum, int32_t* densify_count,
                                  int32_t* densify_max_radius, int32_t sparse_adam, void* stream,
                                  const uint16_t* sh_half = nullptr, uint16_t* sh_half_out = nullptr,
                                  bool sh16 = false) {
    if (sparse_adam != 0 && sparse_adam != 1) return fail(GS_ERR_INVALID_ARG, "%s: sparse_adam must be 0 or 1", fn);
    if (sh16 && params && params->n > 0) {
        CHECK_PTR(sh_half, 8);
        CHECK_PTR(sh_half_out, 8);
    }
    if (!lr_host) return fail(GS_ERR_INVALID_ARG, "%s: lr_host is NULL", fn);
    gsk::AdamStep a;
    gs_status st;
    for (int g = 0; g < 5; ++g) {
        if ((st = check_adam_hyper(fn, lr_host[g], beta1, beta2, eps, step)) != GS_OK) return st;
        a.lr[g] = lr_host[g];
    }
    if (!params_inout || !adam_m || !adam_v) return fail(GS_ERR_INVALID_ARG, "%s: Adam arrays are NULL", fn);
    if (!grads && num_views > GS_ADAM_ONE_PASS_MAX_VIEWS)
        return fail(GS_ERR_INVALID_ARG, "%s: grads is NULL (required for more than %d views: the gradient passes "
                    "through it to the Adam step)", fn, GS_ADAM_ONE_PASS_MAX_VIEWS);
    if (params && (params_inout->means != params->means || params_inout->sh != params->sh))
        return fail(GS_ERR_INVALID_ARG, "%s: params_inout must be the arrays of params", fn);
    a.params = params_inout;
    a.m = adam_m;
    a.v = adam_v;
    a.beta1 = beta1;
    a.beta2 = beta2;
    a.eps = eps;
    a.step = step;
    a.sparse = sparse_adam == 1;
    if (sh16) {
        a.sh_half = sh_half;
        a.sh_half_out = sh_half_out;
    }
    return project_bwd_common(fn, params, num_views, cams, projs, grad2d, grads, densify_accum, densify_count,
                              densify_max_radius, &a, stream, slots, packed);
}

}  // namespace

extern "C" {

gs_status gs_project_bwd_views_adam(const gs_params* params, int32_t num_views, const gs_camera* cams,
                                    const gs_projected* projs, const gs_grad2d* grad2d, gs_param_grads* params_inout,
                                    gs_param_grads* adam_m, gs_param_grads* adam_v, const float* lr_host,
                                    float beta1, float beta2, float eps, int32_t step, gs_param_grads* grads,
                                    float* densify_accum, int32_t* densify_count, int32_t* densify_max_radius,
                                    int32_t sparse_adam, void* stream) {
    return project_bwd_adam_common("gs_project_bwd_views_adam", params, num_views, cams, projs, nullptr, false,
                                   grad2d, params_inout, adam_m, adam_v, lr_host, beta1, beta2, eps, step, grads,
                                   densify_accum, densify_count, densify_max_radius, sparse_adam, stream);
}

gs_status gs_project_bwd_views_adam_packed(const gs_params* params, int32_t num_views, const gs_camera* cams,
                                           const gs_projected* projs, const int32_t* const* slot_of,
                                           const gs_grad2d* grad2d, gs_param_grads* params_inout,
                                           gs_param_grads* adam_m, gs_param_grads* adam_v, const float* lr_host,
                                           float beta1, float beta2, float eps, int32_t step, gs_param_grads* grads,
                                           float* densify_accum, int32_t* densify_count, int32_t* densify_max_radius,
                                           int32_t sparse_adam, void* stream) {
    return project_bwd_adam_common("gs_project_bwd_views_adam_packed", params, num_views, cams, projs, slot_of, true,
                                   grad2d, params_inout, adam_m, adam_v, lr_host, beta1, beta2, eps, step, grads,
                                   densify_accum, densify_count, densify_max_radius, sparse_adam, stream);
}

gs_status gs_project_bwd_views_adam_sh16(const gs_params* params, int32_t num_views, const gs_camera* cams,
                                         const gs_projected* projs, const gs_grad2d* grad2d,
                                         const uint16_t* sh_half, uint16_t* sh_half_out, gs_param_grads* params_inout,
                                         gs_param_grads* adam_m, gs_param_grads* adam_v, const float* lr_host,
                                         float beta1, float beta2, float eps, int32_t step, gs_param_grads* grads,
                                         float* densify_accum, int32_t* densify_count, int32_t* densify_max_radius,
                                         int32_t sparse_adam, void* stream) {
    return project_bwd_adam_common("gs_project_bwd_views_adam_sh16", params, num_views, cams, projs, nullptr, false,
                                   grad2d, params_inout, adam_m, adam_v, lr_host, beta1, beta2, eps, step, grads,
                                   densify_accum, densify_count, densify_max_radius, sparse_adam, stream, sh_half,
                                   sh_half_out, true);
}

gs_status gs_project_bwd_views_packed(const gs_params* params, int32_t num_views, const gs_camera* cams,
                                      const gs_projected* projs, const int32_t* const* slot_of,
                                      const gs_grad2d* grad2d, gs_param_grads* grads, float* densify_accum,
                                      int32_t* densify_count, int32_t* densify_max_radius, void* stream) {
    const char* fn = "gs_project_bwd_views_packed";
    if (!grads) return fail(GS_ERR_INVALID_ARG, "%s: grads is NULL", fn);
    return project_bwd_common(fn, params, num_views, cams, projs, grad2d, grads, densify_accum, densify_count,
                              densify_max_radius, nullptr, stream, slot_of, true);
}

size_t gs_project_packed_workspace_bytes(int64_t n) {
    if (n < 0) n = 0;
    return gsk::pack_workspace_layout(n, nullptr, nullptr);
}

gs_status gs_project_packed(const gs_params* params, const gs_camera* cam, void* workspace, size_t workspace_bytes,
                            gs_projected* packed, int64_t capacity, uint32_t* gaussian_ids, int32_t* slot_of,
                            uint64_t* num_visible_dev, void* stream) {
    const char* fn = "gs_project_packed";
    gs_status st;
    if ((st = check_params(fn, params)) != GS_OK) return st;
    if ((st = check_camera(fn, cam)) != GS_OK) return st;
    if (capacity < 0 || capacity > 0x7fffffffLL) return fail(GS_ERR_INVALID_ARG, "%s: capacity out of range", fn);
    if ((st = check_projected(fn, packed, capacity, true)) != GS_OK) return st;
    CHECK_PTR(num_visible_dev, 8);
    CHECK_PTR(workspace, 16);
    if (capacity > 0) CHECK_PTR(gaussian_ids, 4);
    if (params->n > 0) CHECK_PTR(slot_of, 4);
    const size_t need = gsk::pack_workspace_layout(params->n, nullptr, nullptr);
    if (workspace_bytes < need)
        return fail(GS_ERR_INVALID_ARG, "%s: workspace of %zu bytes, %zu needed", fn, workspace_bytes, need);
    gsk::PackWorkspace ws;
    gsk::pack_workspace_layout(params->n, workspace, &ws);
    const gsk::CamArgs c = gsk::make_cam(*cam);
    return cuda_status(gsk::launch_project_packed(*params, c, ws, *packed, capacity, gaussian_ids, slot_of,
                                                  reinterpret_cast<unsigned long long*>(num_visible_dev),
                                                  static_cast<cudaStream_t>(stream)),
                       fn);
}

size_t gs_l1_dssim_workspace_bytes(int32_t width, int32_t height) {
    if (width <= 0 || height <= 0) return 0;
    return (size_t(width) * size_t(height) * 9 * sizeof(double) + 255) & ~size_t(255);
}

gs_status gs_l1_dssim_loss_grad(const float* image, const float* target, int32_t width, int32_t height,
                                float l1_weight, float ssim_weight, void* workspace, size_t workspace_bytes,
                                float* dL_dimage, double* loss_dev, void* stream) {
    const char* fn = "gs_l1_dssim_loss_grad";
    if (width <= 0 || height <= 0 || width > 16384 || height > 16384)
        return fail(GS_ERR_UNSUPPORTED, "%s: image %d x %d (1..16384 supported)", fn, int(width), int(height));
    if (!std::isfinite(l1_weight) || !std::isfinite(ssim_weight))
        return fail(GS_ERR_INVALID_ARG, "%s: non-finite weight", fn);
    CHECK_PTR(image, 4);
    CHECK_PTR(target, 4);
    CHECK_PTR(dL_dimage, 4);
    CHECK_PTR(loss_dev, 8);
    CHECK_PTR(workspace, 16);
    if (workspace_bytes < gs_l1_dssim_workspace_bytes(width, height))
        return fail(GS_ERR_INVALID_ARG, "%s: workspace of %zu bytes, %zu needed", fn, workspace_bytes,
                    gs_l1_dssim_workspace_bytes(width, height));
    return cuda_status(gsk::launch_l1_dssim(image, target, width, height, l1_weight, ssim_weight,
                                            static_cast<double*>(workspace), dL_dimage, loss_dev,
                                            static_cast<cudaStream_t>(stream)),
                       fn);
}

size_t gs_densify_workspace_bytes(int64_t n) {
    if (n < 0) n = 0;
    return gsk::densify_workspace_layout(n, nullptr, nullptr);
}

gs_status gs_densify_plan(const gs_params* params, const float* densify_accum, const int32_t* densify_count,
                          const int32_t* densify_max_radius, const gs_densify_config* cfg, void* workspace,
                          size_t workspace_bytes, uint8_t* decision, uint64_t* num_out_dev, void* stream) {
    const char* fn = "gs_densify_plan";
    gs_status st;
    if ((st = check_params(fn, params)) != GS_OK) return st;
    if (!cfg) return fail(GS_ERR_INVALID_ARG, "%s: cfg is NULL", fn);
    if (!std::isfinite(cfg->grad_threshold) || !std::isfinite(cfg->scale_threshold) ||
        !std::isfinite(cfg->min_opacity))
        return fail(GS_ERR_INVALID_ARG, "%s: non-finite threshold", fn);
    CHECK_PTR(workspace, 16);
    CHECK_PTR(num_out_dev, 8);
    if (workspace_bytes < gs_densify_workspace_bytes(params->n))
        return fail(GS_ERR_INVALID_ARG, "%s: workspace of %zu bytes, %zu needed", fn, workspace_bytes,
                    gs_densify_workspace_bytes(params->n));
    if (params->n > 0) {
        CHECK_PTR(densify_accum, 4);
        CHECK_PTR(densify_count, 4);
        CHECK_PTR(decision, 1);
        if (densify_max_radius) CHECK_PTR(densify_max_radius, 4);
    }
    gsk::DensifyWorkspace ws;
    gsk::densify_workspace_layout(params->n, workspace, &ws);
    return cuda_status(gsk::launch_densify_plan(*params, densify_accum, densify_count, densify_max_radius, *cfg, ws,
                                                decision, num_out_dev, static_cast<cudaStream_t>(stream)),
                       fn);
}

gs_status gs_densify_apply(const gs_params* params, const gs_params* adam_m, const gs_params* adam_v,
                           const float* split_noise, const uint8_t* decision, const void* workspace,
                           size_t workspace_bytes, int64_t n_out, gs_param_grads* out_params, gs_param_grads* out_m,
                           gs_param_grads* out_v, void* stream) {
    const char* fn = "gs_densify_apply";
    gs_status st;
    if ((st = check_params(fn, params)) != GS_OK) return st;
    const bool moments = adam_m || adam_v || out_m || out_v;
    if (moments && !(adam_m && adam_v && out_m && out_v))
        return fail(GS_ERR_INVALID_ARG, "%s: adam_m, adam_v, out_m and out_v must all be set or all NULL", fn);
    if (moments) {
        for (const gs_params* g : {adam_m, adam_v}) {
            if (g->n != params->n || g->sh_degree != params->sh_degree)
                return fail(GS_ERR_INVALID_ARG, "%s: moments differ from params in n or SH degree", fn);
            if ((st = check_params(fn, g)) != GS_OK) return st;
        }
    }
    if (n_out < 0 || n_out > 2 * params->n) return fail(GS_ERR_INVALID_ARG, "%s: n_out = %lld", fn, (long long)n_out);
    CHECK_PTR(workspace, 16);
    if (workspace_bytes < gs_densify_workspace_bytes(params->n))
        return fail(GS_ERR_INVALID_ARG, "%s: workspace of %zu bytes, %zu needed", fn, workspace_bytes,
                    gs_densify_workspace_bytes(params->n));
    if (params->n > 0) {
        CHECK_PTR(split_noise, 4);
        CHECK_PTR(decision, 1);
    }
    if (n_out > 0) {
        if ((st = check_grad_arrays(fn, out_params, "out_params")) != GS_OK) return st;
        if (moments) {
            if ((st = check_grad_arrays(fn, out_m, "out_m")) != GS_OK) return st;
            if ((st = check_grad_arrays(fn, out_v, "out_v")) != GS_OK) return st;
        }
    }
    gsk::DensifyWorkspace ws;
    gsk::densify_workspace_layout(params->n, const_cast<void*>(workspace), &ws);
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    unsigned long long planned = 0;
    if (cudaMemcpyAsync(&planned, ws.total, sizeof(planned), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return cuda_status(cudaGetLastError(), fn);
    if ((long long)planned != n_out)
        return fail(GS_ERR_INVALID_ARG, "%s: n_out = %lld but the plan has %llu", fn, (long long)n_out, planned);
    return cuda_status(gsk::launch_densify_apply(*params, adam_m, adam_v, split_noise, decision, ws, n_out,
                                                 out_params ? *out_params : gs_param_grads{}, out_m, out_v,
                                                 std::log(1.6), s),
                       fn);
}

gs_status gs_adam(float* param, const float* grad, float* m, float* v, int64_t count, float lr, float beta1,
                  float beta2, float eps, int32_t step, void* stream) {
    const char* fn = "gs_adam";
    if (count < 0) return fail(GS_ERR_INVALID_ARG, "%s: count < 0", fn);
    if (step < 1) return fail(GS_ERR_INVALID_ARG, "%s: step must be >= 1", fn);
    if (!std::isfinite(lr) || !(beta1 >= 0.f && beta1 < 1.f) || !(beta2 >= 0.f && beta2 < 1.f) || !(eps >= 0.f))
        return fail(GS_ERR_INVALID_ARG, "%s: invalid hyper-parameters", fn);
    if (count == 0) return ok();
    CHECK_PTR(param, 16);
    CHECK_PTR(grad, 16);
    CHECK_PTR(m, 16);
    CHECK_PTR(v, 16);
    return cuda_status(gsk::launch_adam(param, grad, m, v, count, lr, beta1, beta2, eps, step,
                                        static_cast<cudaStream_t>(stream)),
                       fn);
}

gs_status gs_l1_loss_grad(const float* image, const float* target, int64_t count, float* dL_dimage,
                          double* loss_dev, void* stream) {
    const char* fn = "gs_l1_loss_grad";
    if (count < 0) return fail(GS_ERR_INVALID_ARG, "%s: count < 0", fn);
    if (count == 0) return ok();
    CHECK_PTR(image, 16);
    CHECK_PTR(target, 16);
    CHECK_PTR(dL_dimage, 16);
    CHECK_PTR(loss_dev, 8);
    return cuda_status(gsk::launch_l1(image, target, count, dL_dimage, loss_dev, static_cast<cudaStream_t>(stream)),
                       fn);
}

uint64_t gs_kernel_launches(void) { return gsk::g_launches.load(std::memory_order_relaxed); }

gs_status gs_zero(void* ptr, size_t bytes, void* stream) {
    const char* fn = "gs_zero";
    if (bytes == 0) return ok();
    if (!ptr) return fail(GS_ERR_INVALID_ARG, "%s: ptr is NULL", fn);
    return cuda_status(cudaMemsetAsync(ptr, 0, bytes, static_cast<cudaStream_t>(stream)), fn);
}

}  // extern "C"
