// gs_project_packed: the projection in the packed layout (the packed option of
// rasterize_gaussians in the gsplat guide, lmnt.cn/news/262699 §4.1): only the
// Gaussians the view keeps (radius > 0) get feature entries, stored
// contiguously in ascending Gaussian order, with the Gaussian id of every slot
// and the slot of every Gaussian.  The rest of the path runs unchanged on the
// packed arrays: the binning's values become slots, and since slots ascend
// with the Gaussian id the stable sorts put equal keys in the same order.
//
// Launches: the projection of all Gaussians into workspace arrays, then an
// order-preserving compaction over contiguous chunks (compact.cuh): a count of
// the chunk's visible Gaussians, the chunk offsets, the copy of every visible
// Gaussian's features into its slot, and a pass that marks the slots past the
// visible count as culled entries.  Streaming work, bound by HBM bandwidth.
#include <cuda_runtime.h>

#include "compact.cuh"
#include "internal.cuh"

namespace gsk {
namespace {

using compact::kBlock;

struct PackArgs {
    // the projection of every Gaussian
    const float2* xy;
    const float* depth;
    const float4* conic_op;
    const float4* rgb;
    const int32_t* radius;
    const uint2* rect;
    const uint32_t* touched;
    // the packed arrays, `capacity` slots
    float2* pxy;
    float* pdepth;
    float4* pconic_op;
    float4* prgb;
    int32_t* pradius;
    uint2* prect;
    uint32_t* ptouched;
    uint32_t* ids;      // [capacity] Gaussian of each slot
    int32_t* slot_of;   // [n] slot of each Gaussian, -1 when it has none
    unsigned long long* chunk_counts;  // counts, then offsets
    const unsigned long long* visible;  // total visible count (device)
    int64_t n, capacity, chunk;
};

__global__ void __launch_bounds__(kBlock) pack_plan_kernel(const PackArgs a) {
    const int64_t begin = int64_t(blockIdx.x) * a.chunk;
    const int64_t end = begin + a.chunk < a.n ? begin + a.chunk : a.n;
    unsigned long long total = 0;
    for (int64_t base = begin; base < end; base += kBlock) {
        const int64_t i = base + threadIdx.x;
        total += unsigned(__syncthreads_count(i < end && __ldg(a.radius + i) > 0));
    }
    if (threadIdx.x == 0) a.chunk_counts[blockIdx.x] = total;
}

__global__ void __launch_bounds__(kBlock) pack_apply_kernel(const PackArgs a) {
    __shared__ unsigned warp_tot[kBlock / 32];
    const int64_t begin = int64_t(blockIdx.x) * a.chunk;
    const int64_t end = begin + a.chunk < a.n ? begin + a.chunk : a.n;
    unsigned long long run = a.chunk_counts[blockIdx.x];
    for (int64_t base = begin; base < end; base += kBlock) {
        const int64_t i = base + threadIdx.x;
        const unsigned vis = (i < end && __ldg(a.radius + i) > 0) ? 1u : 0u;
        unsigned tile_total;
        const unsigned incl = compact::block_inclusive_scan(vis, warp_tot, tile_total);
        const int64_t k = int64_t(run + (incl - vis));
        run += tile_total;
        if (i >= end) continue;
        const bool kept = vis && k < a.capacity;
        a.slot_of[i] = kept ? int32_t(k) : -1;
        if (!kept) continue;
        a.ids[k] = uint32_t(i);
        a.pxy[k] = __ldg(a.xy + i);
        a.pdepth[k] = __ldg(a.depth + i);
        a.pconic_op[k] = __ldg(a.conic_op + i);
        a.prgb[k] = __ldg(a.rgb + i);
        a.pradius[k] = __ldg(a.radius + i);
        a.prect[k] = __ldg(a.rect + i);
        a.ptouched[k] = __ldg(a.touched + i);
    }
}

// Slots [visible, capacity): culled entries (what gs_project writes for a culled
// Gaussian) with the id 0xffffffff.
__global__ void __launch_bounds__(256) pack_tail_kernel(const PackArgs a) {
    const unsigned long long v = *a.visible;
    const int64_t first = v < static_cast<unsigned long long>(a.capacity) ? int64_t(v) : a.capacity;
    for (int64_t k = first + blockIdx.x * int64_t(blockDim.x) + threadIdx.x; k < a.capacity;
         k += int64_t(gridDim.x) * blockDim.x) {
        a.ids[k] = 0xffffffffu;
        a.pxy[k] = make_float2(0.f, 0.f);
        a.pdepth[k] = 0.f;
        a.pconic_op[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        a.prgb[k] = make_float4(0.f, 0.f, 0.f, 0.f);
        a.pradius[k] = 0;
        a.prect[k] = make_uint2(0u, 0u);
        a.ptouched[k] = 0u;
    }
}

size_t align_256(size_t b) { return (b + 255) & ~size_t(255); }

}  // namespace

size_t pack_workspace_layout(int64_t n, void* base, PackWorkspace* ws) {
    const size_t m = size_t(n > 0 ? n : 1);
    char* b = static_cast<char*>(base);
    size_t off = 0;
    PackWorkspace w;
    w.full.xy = reinterpret_cast<float*>(b + off);
    off += align_256(8 * m);
    w.full.depth = reinterpret_cast<float*>(b + off);
    off += align_256(4 * m);
    w.full.conic_opacity = reinterpret_cast<float*>(b + off);
    off += align_256(16 * m);
    w.full.rgb = reinterpret_cast<float*>(b + off);
    off += align_256(16 * m);
    w.full.radius = reinterpret_cast<int32_t*>(b + off);
    off += align_256(4 * m);
    w.full.rect = reinterpret_cast<uint16_t*>(b + off);
    off += align_256(8 * m);
    w.full.tiles_touched = reinterpret_cast<uint32_t*>(b + off);
    off += align_256(4 * m);
    const compact::Chunking ch = compact::chunking(n);
    w.chunk_counts = reinterpret_cast<unsigned long long*>(b + off);
    w.total = w.chunk_counts + ch.blocks;
    w.blocks = ch.blocks;
    w.chunk = ch.chunk;
    off += compact::workspace_bytes(n);
    if (ws) *ws = w;
    return off;
}

cudaError_t launch_project_packed(const gs_params& p, const CamArgs& cam, const PackWorkspace& ws,
                                  const gs_projected& packed, int64_t capacity, uint32_t* ids, int32_t* slot_of,
                                  unsigned long long* num_visible_dev, cudaStream_t s) {
    cudaError_t e = launch_project_fwd(p, cam, ws.full, s);
    if (e != cudaSuccess) return e;
    PackArgs a;
    a.xy = reinterpret_cast<const float2*>(ws.full.xy);
    a.depth = ws.full.depth;
    a.conic_op = reinterpret_cast<const float4*>(ws.full.conic_opacity);
    a.rgb = reinterpret_cast<const float4*>(ws.full.rgb);
    a.radius = ws.full.radius;
    a.rect = reinterpret_cast<const uint2*>(ws.full.rect);
    a.touched = ws.full.tiles_touched;
    a.pxy = reinterpret_cast<float2*>(packed.xy);
    a.pdepth = packed.depth;
    a.pconic_op = reinterpret_cast<float4*>(packed.conic_opacity);
    a.prgb = reinterpret_cast<float4*>(packed.rgb);
    a.pradius = packed.radius;
    a.prect = reinterpret_cast<uint2*>(packed.rect);
    a.ptouched = packed.tiles_touched;
    a.ids = ids;
    a.slot_of = slot_of;
    a.chunk_counts = ws.chunk_counts;
    a.visible = ws.total;
    a.n = p.n;
    a.capacity = capacity;
    a.chunk = ws.chunk;
    if (p.n > 0) {
        pack_plan_kernel<<<ws.blocks, kBlock, 0, s>>>(a);
        count_launches(1);
    } else {
        e = cudaMemsetAsync(ws.chunk_counts, 0, sizeof(unsigned long long) * ws.blocks, s);
        if (e != cudaSuccess) return e;
    }
    compact::chunk_offsets_kernel<<<1, 1024, 0, s>>>(ws.chunk_counts, ws.blocks, ws.total, num_visible_dev);
    count_launches(1);
    if (p.n > 0) {
        pack_apply_kernel<<<ws.blocks, kBlock, 0, s>>>(a);
        count_launches(1);
    }
    if (capacity > 0) {
        pack_tail_kernel<<<grid_for(capacity, 256, 4), 256, 0, s>>>(a);
        count_launches(1);
    }
    return cudaGetLastError();
}

}  // namespace gsk
