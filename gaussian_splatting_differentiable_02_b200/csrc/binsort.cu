// gs_bin_sort: tile binning with a (tile_id << 32 | depth) key and a stable LSD
// radix sort (the "culling and reordering" stage the MUSA co-design article,
// qwbw.cn/news/278220 §1, lists among the four 3DGS bottlenecks; the packed
// screen-space ordering of the gsplat guide, lmnt.cn/news/262699 §4.1).
//
// Kernels (no kernel waits on another block, so nothing here can spin):
//   count_kernel      per-block sum of tiles_touched
//   scan_blocks       one CTA: exclusive scan of the block sums, total K
//   emit_kernel       per block: in-block scan, then every visible Gaussian
//                     writes its (key, gid) instances, row-major over its rect
//   upsweep_kernel    per-block 256-bin digit histogram of one 8-bit digit
//   scan_hist_kernel  per digit: exclusive scan of the block histograms
//   downsweep_kernel  stable rank of every element among equal digits of its
//                     block (warp match + per-warp counters), scatter
//   ranges_kernel     [begin, end) of each tile in the sorted keys
#include "internal.cuh"

namespace gsk {
namespace {

constexpr int kEmitBlock = 256;
constexpr int kEmitPerThread = 8;
constexpr int kEmitChunk = kEmitBlock * kEmitPerThread;  // Gaussians per emit block

constexpr int kSortBlock = 256;
constexpr int kSortWarps = kSortBlock / 32;
constexpr int kSortPerThread = 16;
constexpr int kSortTile = kSortBlock * kSortPerThread;  // elements per sort block
constexpr int kWarpSpan = 32 * kSortPerThread;           // elements per warp

__device__ __forceinline__ unsigned long long warp_incl_scan(unsigned long long v) {
    const int lane = threadIdx.x & 31;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        unsigned long long t = __shfl_up_sync(0xffffffffu, v, d);
        if (lane >= d) v += t;
    }
    return v;
}

// Exclusive scan of one value per thread over the block (blockDim.x <= 1024).
// Returns the exclusive prefix; *total receives the block sum.
__device__ unsigned long long block_excl_scan(unsigned long long v, unsigned long long* total) {
    __shared__ unsigned long long warp_sums[32];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = (blockDim.x + 31) >> 5;
    const unsigned long long inc = warp_incl_scan(v);
    if (lane == 31) warp_sums[warp] = inc;
    __syncthreads();
    if (warp == 0) {
        unsigned long long s = lane < nw ? warp_sums[lane] : 0ull;
        s = warp_incl_scan(s);
        if (lane < nw) warp_sums[lane] = s;
    }
    __syncthreads();
    const unsigned long long before = warp == 0 ? 0ull : warp_sums[warp - 1];
    *total = warp_sums[nw - 1];
    __syncthreads();
    return before + inc - v;
}

__global__ void __launch_bounds__(kEmitBlock) count_kernel(const uint32_t* __restrict__ touched, int64_t n,
                                                           unsigned long long* block_sums) {
    const int64_t base = int64_t(blockIdx.x) * kEmitChunk;
    unsigned long long s = 0;
    for (int k = threadIdx.x; k < kEmitChunk; k += kEmitBlock) {
        const int64_t i = base + k;
        if (i < n) s += __ldg(touched + i);
    }
    unsigned long long tot;
    block_excl_scan(s, &tot);
    if (threadIdx.x == 0) block_sums[blockIdx.x] = tot;
}

__global__ void __launch_bounds__(1024) scan_blocks_kernel(unsigned long long* block_sums, int64_t nb,
                                                           unsigned long long* total) {
    unsigned long long carry = 0;
    for (int64_t base = 0; base < nb; base += 1024) {
        const int64_t i = base + threadIdx.x;
        const unsigned long long v = i < nb ? block_sums[i] : 0ull;
        unsigned long long tot;
        const unsigned long long ex = block_excl_scan(v, &tot);
        if (i < nb) block_sums[i] = carry + ex;
        carry += tot;
    }
    if (threadIdx.x == 0) *total = carry;
}

__global__ void __launch_bounds__(kEmitBlock) emit_kernel(const uint32_t* __restrict__ touched,
                                                          const uint2* __restrict__ rect,
                                                          const float* __restrict__ depth, int64_t n, int tiles_x,
                                                          const unsigned long long* __restrict__ block_offsets,
                                                          uint64_t* __restrict__ keys, uint32_t* __restrict__ vals) {
    const int64_t first = int64_t(blockIdx.x) * kEmitChunk + int64_t(threadIdx.x) * kEmitPerThread;
    unsigned long long mine = 0;
#pragma unroll
    for (int k = 0; k < kEmitPerThread; ++k)
        if (first + k < n) mine += __ldg(touched + first + k);
    unsigned long long tot;
    unsigned long long off = block_excl_scan(mine, &tot) + block_offsets[blockIdx.x];
    for (int k = 0; k < kEmitPerThread; ++k) {
        const int64_t i = first + k;
        if (i >= n) break;
        if (__ldg(touched + i) == 0u) continue;
        const uint2 r = __ldg(rect + i);
        const uint32_t x0 = r.x & 0xffffu, y0 = r.x >> 16, x1 = r.y & 0xffffu, y1 = r.y >> 16;
        const uint64_t zb = __float_as_uint(__ldg(depth + i));
        for (uint32_t ty = y0; ty < y1; ++ty)
            for (uint32_t tx = x0; tx < x1; ++tx) {
                keys[off] = (uint64_t(ty * uint32_t(tiles_x) + tx) << 32) | zb;
                vals[off] = uint32_t(i);
                ++off;
            }
    }
}

__global__ void __launch_bounds__(kSortBlock) upsweep_kernel(const uint64_t* __restrict__ keys, int64_t K, int shift,
                                                             uint32_t* __restrict__ hist, int64_t nb) {
    __shared__ uint32_t h[kSortWarps][256];
    const int warp = threadIdx.x >> 5;
    for (int k = threadIdx.x; k < kSortWarps * 256; k += kSortBlock) (&h[0][0])[k] = 0u;
    __syncthreads();
    const int64_t base = int64_t(blockIdx.x) * kSortTile;
#pragma unroll 4
    for (int k = 0; k < kSortPerThread; ++k) {
        const int64_t e = base + int64_t(k) * kSortBlock + threadIdx.x;
        if (e < K) atomicAdd(&h[warp][uint32_t(__ldg(keys + e) >> shift) & 0xffu], 1u);
    }
    __syncthreads();
    for (int d = threadIdx.x; d < 256; d += kSortBlock) {
        uint32_t s = 0;
#pragma unroll
        for (int w = 0; w < kSortWarps; ++w) s += h[w][d];
        hist[int64_t(d) * nb + blockIdx.x] = s;
    }
}

// One CTA per digit: exclusive scan over the blocks' counts of that digit.
__global__ void __launch_bounds__(1024) scan_hist_kernel(uint32_t* hist, int64_t nb, uint32_t* digit_totals) {
    uint32_t* row = hist + int64_t(blockIdx.x) * nb;
    unsigned long long carry = 0;
    for (int64_t base = 0; base < nb; base += 1024) {
        const int64_t i = base + threadIdx.x;
        const unsigned long long v = i < nb ? row[i] : 0ull;
        unsigned long long tot;
        const unsigned long long ex = block_excl_scan(v, &tot);
        if (i < nb) row[i] = uint32_t(carry + ex);
        carry += tot;
    }
    if (threadIdx.x == 0) digit_totals[blockIdx.x] = uint32_t(carry);
}

__global__ void __launch_bounds__(kSortBlock) downsweep_kernel(const uint64_t* __restrict__ keys_in,
                                                               const uint32_t* __restrict__ vals_in,
                                                               uint64_t* __restrict__ keys_out,
                                                               uint32_t* __restrict__ vals_out, int64_t K, int shift,
                                                               const uint32_t* __restrict__ hist, int64_t nb,
                                                               const uint32_t* __restrict__ digit_totals) {
    __shared__ uint32_t wcount[kSortWarps][256];
    __shared__ uint32_t gbase[256];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int k = threadIdx.x; k < kSortWarps * 256; k += kSortBlock) (&wcount[0][0])[k] = 0u;
    // digit base: exclusive prefix of the digit totals plus this block's offset
    {
        unsigned long long tot;
        const unsigned long long ex = block_excl_scan(threadIdx.x < 256 ? digit_totals[threadIdx.x] : 0u, &tot);
        if (threadIdx.x < 256) gbase[threadIdx.x] = uint32_t(ex) + hist[int64_t(threadIdx.x) * nb + blockIdx.x];
    }
    __syncthreads();

    const int64_t base = int64_t(blockIdx.x) * kSortTile + int64_t(warp) * kWarpSpan;
    const uint32_t lt_mask = (1u << lane) - 1u;
    uint64_t key[kSortPerThread];
    uint32_t val[kSortPerThread];
    uint32_t rank[kSortPerThread];
#pragma unroll
    for (int r = 0; r < kSortPerThread; ++r) {
        const int64_t e = base + r * 32 + lane;
        const bool in = e < K;
        key[r] = in ? __ldg(keys_in + e) : 0ull;
        val[r] = in ? __ldg(vals_in + e) : 0u;
        const uint32_t digit = in ? (uint32_t(key[r] >> shift) & 0xffu) : 256u;
        const uint32_t peers = __match_any_sync(0xffffffffu, digit);
        const uint32_t before = in ? wcount[warp][digit] : 0u;
        __syncwarp();
        if (in && (lane == __ffs(peers) - 1)) wcount[warp][digit] = before + __popc(peers);
        __syncwarp();
        rank[r] = before + __popc(peers & lt_mask);
    }
    __syncthreads();
    // exclusive prefix over warps for each digit
    for (int d = threadIdx.x; d < 256; d += kSortBlock) {
        uint32_t run = 0;
#pragma unroll
        for (int w = 0; w < kSortWarps; ++w) {
            const uint32_t c = wcount[w][d];
            wcount[w][d] = run;
            run += c;
        }
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < kSortPerThread; ++r) {
        const int64_t e = base + r * 32 + lane;
        if (e < K) {
            const uint32_t digit = uint32_t(key[r] >> shift) & 0xffu;
            const uint32_t pos = gbase[digit] + wcount[warp][digit] + rank[r];
            keys_out[pos] = key[r];
            vals_out[pos] = val[r];
        }
    }
}

__global__ void __launch_bounds__(256) ranges_kernel(const uint64_t* __restrict__ keys, int64_t K,
                                                     uint2* __restrict__ ranges) {
    for (int64_t k = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; k < K; k += int64_t(gridDim.x) * blockDim.x) {
        const uint32_t t = uint32_t(__ldg(keys + k) >> 32);
        if (k == 0 || uint32_t(__ldg(keys + k - 1) >> 32) != t) ranges[t].x = uint32_t(k);
        if (k == K - 1 || uint32_t(__ldg(keys + k + 1) >> 32) != t) ranges[t].y = uint32_t(k + 1);
    }
}

size_t align_up(size_t x) { return (x + 255) & ~size_t(255); }

}  // namespace

size_t sort_workspace_layout(int64_t n, int64_t capacity, void* base, SortWorkspace* ws) {
    const int64_t nb_emit = (n + kEmitChunk - 1) / kEmitChunk;
    const int64_t nb_sort = (capacity + kSortTile - 1) / kSortTile;
    size_t off = 0;
    char* b = static_cast<char*>(base);
    SortWorkspace w;
    w.nb_emit = nb_emit;
    w.nb_sort = nb_sort;
    w.block_sums = reinterpret_cast<unsigned long long*>(b + off);
    off += align_up(sizeof(unsigned long long) * size_t(nb_emit > 0 ? nb_emit : 1));
    w.total = reinterpret_cast<unsigned long long*>(b + off);
    off += align_up(sizeof(unsigned long long));
    w.keys_alt = reinterpret_cast<uint64_t*>(b + off);
    off += align_up(sizeof(uint64_t) * size_t(capacity > 0 ? capacity : 1));
    w.vals_alt = reinterpret_cast<uint32_t*>(b + off);
    off += align_up(sizeof(uint32_t) * size_t(capacity > 0 ? capacity : 1));
    w.hist = reinterpret_cast<uint32_t*>(b + off);
    off += align_up(sizeof(uint32_t) * 256 * size_t(nb_sort > 0 ? nb_sort : 1));
    w.digit_totals = reinterpret_cast<uint32_t*>(b + off);
    off += align_up(sizeof(uint32_t) * 256);
    if (ws) *ws = w;
    return off;
}

cudaError_t launch_count_instances(const gs_projected& proj, int64_t n, const SortWorkspace& ws, cudaStream_t s) {
    if (n > 0) {
        count_kernel<<<unsigned(ws.nb_emit), kEmitBlock, 0, s>>>(proj.tiles_touched, n, ws.block_sums);
        scan_blocks_kernel<<<1, 1024, 0, s>>>(ws.block_sums, ws.nb_emit, ws.total);
        count_launches(2);
    } else {
        cudaMemsetAsync(ws.total, 0, sizeof(unsigned long long), s);
    }
    return cudaGetLastError();
}

cudaError_t launch_emit_sort_ranges(const gs_projected& proj, int64_t n, const CamArgs& cam, const SortWorkspace& ws,
                                    uint64_t* keys, uint32_t* vals, int64_t K, uint32_t* ranges, cudaStream_t s) {
    const int64_t T = int64_t(cam.TX) * cam.TY;
    cudaError_t e = cudaMemsetAsync(ranges, 0, sizeof(uint32_t) * 2 * size_t(T), s);
    if (e != cudaSuccess || K == 0) return e;
    const int key_bits = 32 + tile_bits(T);
    const int passes = (key_bits + 7) / 8;
    // emit into the buffer that makes the last pass land in `keys`
    uint64_t* k_cur = (passes & 1) ? ws.keys_alt : keys;
    uint32_t* v_cur = (passes & 1) ? ws.vals_alt : vals;
    uint64_t* k_oth = (passes & 1) ? keys : ws.keys_alt;
    uint32_t* v_oth = (passes & 1) ? vals : ws.vals_alt;
    emit_kernel<<<unsigned(ws.nb_emit), kEmitBlock, 0, s>>>(proj.tiles_touched, reinterpret_cast<const uint2*>(proj.rect),
                                                            proj.depth, n, cam.TX, ws.block_sums, k_cur, v_cur);
    count_launches(1);
    const int64_t nb = (K + kSortTile - 1) / kSortTile;
    for (int p = 0; p < passes; ++p) {
        const int shift = 8 * p;
        upsweep_kernel<<<unsigned(nb), kSortBlock, 0, s>>>(k_cur, K, shift, ws.hist, nb);
        scan_hist_kernel<<<256, 1024, 0, s>>>(ws.hist, nb, ws.digit_totals);
        downsweep_kernel<<<unsigned(nb), kSortBlock, 0, s>>>(k_cur, v_cur, k_oth, v_oth, K, shift, ws.hist, nb,
                                                             ws.digit_totals);
        count_launches(3);
        uint64_t* tk = k_cur; k_cur = k_oth; k_oth = tk;
        uint32_t* tv = v_cur; v_cur = v_oth; v_oth = tv;
    }
    ranges_kernel<<<grid_for(K, 256, 8), 256, 0, s>>>(keys, K, reinterpret_cast<uint2*>(ranges));
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace gsk
