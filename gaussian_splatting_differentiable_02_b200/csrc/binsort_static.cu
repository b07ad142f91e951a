// gs_bin_sort_static: gs_bin_sort with its workspace in a fixed device array
// owned by the library, for callers that cannot allocate device memory.
//
// Who cannot allocate: a host application that owns the whole device-memory
// budget and hands plugins nothing but its own buffers; code that runs where a
// cudaMalloc would stall every stream of the device (a frame loop that must
// not synchronise); bindings from runtimes that can pass device pointers in but
// have no allocator of their own.  They still pass inputs and outputs; only the
// sort's scratch moves into this array.
//
// The array is a file-scope __device__ variable, so every device that loads
// the library holds GS_STATIC_SCRATCH_BYTES of it until the process exits.  In
// host code its name is a host-side shadow, not a device address: the address
// comes from cudaGetSymbolAddress, looked up on every call in the current
// device's current context.  An address belongs to a context, not to a device
// number: after cudaDeviceReset, or in a host that creates its own contexts,
// a cached one would point at memory the new context never mapped.  The lookup
// allocates nothing; the first one in a context loads the library's module
// there (which is when the array itself comes into being).
//
// All calls share the one array and it keeps whatever the previous call left:
// every word the sort reads is written earlier in the same call (block sums,
// total, histograms, digit totals, the ping-pong copy), so nothing needs to be
// cleared first.  Calls whose work overlaps on the GPU (different streams,
// or threads racing on one device) corrupt each other's scratch: serialise them.
#include "internal.cuh"

namespace {

__device__ __align__(256) unsigned char g_static_scratch[GS_STATIC_SCRATCH_BYTES];

// Device address of the scratch array in the current context.
cudaError_t scratch_address(void** out) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess) return e;
    *out = p;
    return cudaSuccess;
}

}  // namespace

extern "C" gs_status gs_bin_sort_static(const gs_projected* proj, int64_t n, const gs_camera* cam, uint64_t* keys,
                                        uint32_t* vals, int64_t capacity, int64_t* num_instances_host,
                                        uint32_t* tile_ranges, void* stream) {
    const size_t need = gsk::sort_workspace_layout(n < 0 ? 0 : n, capacity < 0 ? 0 : capacity,
                                                   cam && cam->tile_cull == 1, nullptr, nullptr);
    if (n >= 0 && capacity >= 0 && need > size_t(GS_STATIC_SCRATCH_BYTES))
        return gsk::fail_detail(GS_ERR_UNSUPPORTED,
                                "gs_bin_sort_static: n = %lld and capacity = %lld need %zu bytes of scratch; the "
                                "static scratch holds %zu (use gs_bin_sort with a caller-owned workspace)",
                                (long long)n, (long long)capacity, need, size_t(GS_STATIC_SCRATCH_BYTES));
    void* ws = nullptr;
    const cudaError_t e = scratch_address(&ws);
    if (e != cudaSuccess)
        return gsk::fail_detail(GS_ERR_CUDA, "gs_bin_sort_static: scratch address: %s", cudaGetErrorString(e));
    return gs_bin_sort(proj, n, cam, ws, size_t(GS_STATIC_SCRATCH_BYTES), keys, vals, capacity, num_instances_host,
                       tile_ranges, stream);
}
