// gs_bin_sort / gs_bin_sort_async: tile binning with a (tile_id << 32 | depth)
// key (the "culling and reordering" stage the MUSA co-design article,
// qwbw.cn/news/278220 §1, lists among the four 3DGS bottlenecks; the
// screen-space ordering of the gsplat guide, lmnt.cn/news/262699 §4.1).
//
// The result is the list of instances sorted by (key, Gaussian index).  It is
// produced without sorting 64-bit keys: the Gaussians are first sorted by depth
// (a stable LSD radix sort of N 32-bit keys, culled Gaussians last), instances
// are emitted in that order as 32-bit (tile, gid) pairs, and a stable LSD radix
// sort over the tile bits alone finishes the job, since a stable sort by tile
// of a sequence ordered by (depth, gid) is ordered by (tile, depth, gid).  The
// last tile pass writes the 64-bit key, taking the depth bits from the
// Gaussian.  This moves about a third of the bytes of a 64-bit key sort.
//
// The instance count K stays on the device: the passes over instances are
// launched for the caller's capacity and read K when they start, so nothing
// waits for the host.  When K exceeds the capacity nothing is emitted or
// sorted and every tile range is left empty.
//
// Kernels (no kernel waits on another block, so nothing here can spin):
//   depth_keys        key = float32 bits of the depth (culled: 0xffffffff), val = gid
//   upsweep           per-block 256-bin histogram of one 8-bit digit
//   scan_hist         per digit: exclusive scan of the block histograms
//   downsweep         stable rank of every element among equal digits of its
//                     block (warp votes + per-warp counters), reorder in shared
//                     memory, coalesced scatter; the final tile pass writes
//                     64-bit keys
//   count_sorted      per-block sum of tiles_touched in depth order (culled
//                     binning: of the tiles each footprint reaches, with the
//                     runs of tiles of its first rows kept for emit)
//   scan_blocks       one CTA: exclusive scan of the block sums, total K
//   emit              every visible Gaussian, in depth order, writes its
//                     instances (row-major over its tile rectangle, or its
//                     runs of tiles)
//   ranges            [begin, end) of each tile in the sorted keys
#include "internal.cuh"
#include "tile_reach.cuh"

namespace gsk {
namespace {

constexpr int kEmitBlock = 256;
#ifndef GS_EMIT_ITEMS
#define GS_EMIT_ITEMS 2
#endif
constexpr int kEmitPerThread = GS_EMIT_ITEMS;
constexpr int kEmitChunk = kEmitBlock * kEmitPerThread;  // Gaussians per emit block
static_assert((kEmitChunk & (kEmitChunk - 1)) == 0, "the emit binary search halves a power of two");
// rows of a culled Gaussian whose runs of tiles the count pass keeps for the
// emission (32 bytes a Gaussian; 96% of the 1080p instances of the 1M mixture
// belong to Gaussians of at most 8 rows)
constexpr int kRunRows = 8;
static_assert(kRunRows % 4 == 0, "the emission loads runs as uint4");

#ifndef GS_SORT_ITEMS
#define GS_SORT_ITEMS 8
#endif
// downsweep blocks per SM the register budget is cut for (48 registers, no spill
// to speak of: 80 registers held it to 3 blocks; 16 views of 10M instances at
// 1080p 6.82 -> 5.83 ms of binning, 8 blocks with spills 6.72 ms)
#ifndef GS_SORT_MIN_BLOCKS
#define GS_SORT_MIN_BLOCKS 5
#endif
constexpr int kSortBlock = 256;
constexpr int kSortWarps = kSortBlock / 32;
constexpr int kSortPerThread = GS_SORT_ITEMS;
constexpr int kSortTile = kSortBlock * kSortPerThread;  // elements per sort block
constexpr int kWarpSpan = 32 * kSortPerThread;           // elements per warp

// Number of elements a pass covers: a host count, or the device instance count
// (0 when it exceeds the capacity).
struct Count {
    int64_t host;
    const unsigned long long* dev;
    int64_t limit;
    __device__ __forceinline__ int64_t get() const {
        if (!dev) return host;
        const unsigned long long k = *dev;
        return k <= static_cast<unsigned long long>(limit) ? static_cast<int64_t>(k) : 0;
    }
};

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

// The depth keys of several views at once: view blockIdx.y fills segment
// blockIdx.y (n elements) of keys and vals.
struct ViewDepths {
    const uint32_t* touched[GS_MAX_VIEWS];
    const float* depth[GS_MAX_VIEWS];
};

__global__ void __launch_bounds__(256) depth_keys_views_kernel(const ViewDepths src, int64_t n,
                                                               uint32_t* __restrict__ keys,
                                                               uint32_t* __restrict__ vals) {
    const int v = blockIdx.y;
    const uint32_t* touched = src.touched[v];
    const float* depth = src.depth[v];
    keys += int64_t(v) * n;
    vals += int64_t(v) * n;
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
        keys[i] = __ldg(touched + i) > 0u ? __float_as_uint(__ldg(depth + i)) : 0xffffffffu;
        vals[i] = uint32_t(i);
    }
}

// Radix passes over several independent segments at once (one per view): block
// row blockIdx.y works on segment blockIdx.y, with its own keys, values, element
// count, block histograms and digit totals.
struct PassSeg {
    const uint32_t* kin;
    const uint32_t* vin;
    uint32_t* kout;    // non-final passes
    uint64_t* kout64;  // the final tile pass: key32 << 32 | depth bits of the Gaussian
    uint32_t* vout;
    uint32_t* hist;          // [256][nb]
    uint32_t* digit_totals;  // [256]
    const float* depth;      // final tile pass: the Gaussians' depths
    Count cnt;
    int64_t nb;  // blocks of this segment (the rest of the grid row returns)
};
struct PassArgs {
    PassSeg seg[GS_MAX_VIEWS];
    int shift;
    int digit_bits;  // how many of the digit's 8 bits can be set (the last tile pass has fewer)
};

__global__ void __launch_bounds__(kSortBlock) upsweep_kernel(const __grid_constant__ PassArgs a) {
    __shared__ uint32_t h[kSortWarps][256];
    const PassSeg& g = a.seg[blockIdx.y];
    if (int64_t(blockIdx.x) >= g.nb) return;  // block-uniform
    const int64_t count = g.cnt.get();
    const int warp = threadIdx.x >> 5;
    for (int k = threadIdx.x; k < kSortWarps * 256; k += kSortBlock) (&h[0][0])[k] = 0u;
    __syncthreads();
    const int64_t base = int64_t(blockIdx.x) * kSortTile;
#pragma unroll 4
    for (int k = 0; k < kSortPerThread; ++k) {
        const int64_t e = base + int64_t(k) * kSortBlock + threadIdx.x;
        if (e < count) atomicAdd(&h[warp][(__ldg(g.kin + e) >> a.shift) & 0xffu], 1u);
    }
    __syncthreads();
    for (int d = threadIdx.x; d < 256; d += kSortBlock) {
        uint32_t sum = 0;
#pragma unroll
        for (int w = 0; w < kSortWarps; ++w) sum += h[w][d];
        g.hist[int64_t(d) * g.nb + blockIdx.x] = sum;
    }
}

// One CTA per digit and segment: exclusive scan over the blocks' counts of that digit.
__global__ void __launch_bounds__(1024) scan_hist_kernel(const __grid_constant__ PassArgs a) {
    const PassSeg& g = a.seg[blockIdx.y];
    uint32_t* row = g.hist + int64_t(blockIdx.x) * g.nb;
    unsigned long long carry = 0;
    for (int64_t base = 0; base < g.nb; base += 1024) {
        const int64_t i = base + threadIdx.x;
        const unsigned long long v = i < g.nb ? row[i] : 0ull;
        unsigned long long tot;
        const unsigned long long ex = block_excl_scan(v, &tot);
        if (i < g.nb) row[i] = uint32_t(carry + ex);
        carry += tot;
    }
    if (threadIdx.x == 0) g.digit_totals[blockIdx.x] = uint32_t(carry);
}

template <bool kFinal>
__global__ void __launch_bounds__(kSortBlock, GS_SORT_MIN_BLOCKS) downsweep_kernel(const __grid_constant__ PassArgs a) {
    __shared__ uint32_t wcount[kSortWarps][256];
    __shared__ uint32_t gbase[256];   // global start of each digit's run from this block
    __shared__ uint32_t lstart[256];  // start of each digit's run within the block
    __shared__ uint32_t sk[kSortTile];
    __shared__ uint32_t sv[kSortTile];
    const PassSeg& g = a.seg[blockIdx.y];
    if (int64_t(blockIdx.x) >= g.nb) return;  // block-uniform
    const int64_t count = g.cnt.get();
    const int64_t tile0 = int64_t(blockIdx.x) * kSortTile;
    if (tile0 >= count) return;  // block-uniform: launched for the capacity
    const int shift = a.shift;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    for (int k = threadIdx.x; k < kSortWarps * 256; k += kSortBlock) (&wcount[0][0])[k] = 0u;
    {
        unsigned long long tot;
        const unsigned long long ex = block_excl_scan(threadIdx.x < 256 ? g.digit_totals[threadIdx.x] : 0u, &tot);
        if (threadIdx.x < 256) gbase[threadIdx.x] = uint32_t(ex) + g.hist[int64_t(threadIdx.x) * g.nb + blockIdx.x];
    }
    __syncthreads();

    const int64_t base = tile0 + int64_t(warp) * kWarpSpan;
    const uint32_t lt_mask = (1u << lane) - 1u;
    uint32_t key[kSortPerThread], val[kSortPerThread], rank[kSortPerThread];
#pragma unroll
    for (int r = 0; r < kSortPerThread; ++r) {
        const int64_t e = base + r * 32 + lane;
        const bool in = e < count;
        key[r] = in ? __ldg(g.kin + e) : 0u;
        val[r] = in ? __ldg(g.vin + e) : 0u;
        const uint32_t digit = in ? ((key[r] >> shift) & 0xffu) : 256u;
        // the lanes holding the same digit, from one vote per digit bit and one for
        // validity (cheaper than a match instruction here: 0.41 -> 0.38 ms per 1080p view)
        uint32_t peers = __ballot_sync(0xffffffffu, in);
        peers = in ? peers : ~peers;
#pragma unroll
        for (int bit = 0; bit < 8; ++bit) {
            if (bit >= a.digit_bits) break;  // warp-uniform
            const bool set = (digit >> bit) & 1u;
            const uint32_t vb = __ballot_sync(0xffffffffu, set);
            peers &= set ? vb : ~vb;
        }
        const uint32_t before = in ? wcount[warp][digit] : 0u;
        __syncwarp();
        if (in && (lane == __ffs(peers) - 1)) wcount[warp][digit] = before + __popc(peers);
        __syncwarp();
        rank[r] = before + __popc(peers & lt_mask);
    }
    __syncthreads();
    // per digit: block total, then the exclusive prefix over warps
    uint32_t dtot = 0;
    if (threadIdx.x < 256) {
#pragma unroll
        for (int w = 0; w < kSortWarps; ++w) {
            const uint32_t c = wcount[w][threadIdx.x];
            wcount[w][threadIdx.x] = dtot;
            dtot += c;
        }
    }
    {
        unsigned long long tot;
        const unsigned long long ex = block_excl_scan(dtot, &tot);
        if (threadIdx.x < 256) lstart[threadIdx.x] = uint32_t(ex);
    }
    __syncthreads();
    // reorder by digit inside the block (stable), then write runs out coalesced
#pragma unroll
    for (int r = 0; r < kSortPerThread; ++r) {
        const int64_t e = base + r * 32 + lane;
        if (e < count) {
            const uint32_t digit = (key[r] >> shift) & 0xffu;
            const uint32_t p = lstart[digit] + wcount[warp][digit] + rank[r];
            sk[p] = key[r];
            sv[p] = val[r];
        }
    }
    __syncthreads();
    const int in_block = int(min(int64_t(kSortTile), count - tile0));
    for (int p = threadIdx.x; p < in_block; p += kSortBlock) {
        const uint32_t k = sk[p], v = sv[p];
        const uint32_t digit = (k >> shift) & 0xffu;
        const uint32_t o = gbase[digit] + (uint32_t(p) - lstart[digit]);
        if (kFinal) {
            g.kout64[o] = (uint64_t(k) << 32) | __float_as_uint(__ldg(g.depth + v));
        } else {
            g.kout[o] = k;
        }
        g.vout[o] = v;
    }
}

// The emission of several views at once (one per block row): each view's
// projection, depth order, workspace and outputs.
struct EmitSeg {
    const uint32_t* touched;
    const uint2* rect;
    const float2* xy;  // culled binning: the footprints (tile_reach.cuh)
    const float4* con;
    uint32_t* runs;    // culled binning (else null): [n][kRunRows] runs of the first rows, depth order
    uint32_t* cnt;     // culled binning: [n] instances of each Gaussian, depth order
    const uint32_t* order;           // [n] the view's depth order
    unsigned long long* block_sums;  // [nb_emit]
    unsigned long long* total;       // the view's instance count K
    unsigned long long* count_out;   // nullable: a copy of K for the caller
    Count inst;                      // K, or 0 when it exceeds the view's capacity
    uint32_t* tkey;                  // emitted (tile, gid) pairs
    uint32_t* tval;
    const uint64_t* keys;            // the sorted keys (ranges)
    uint2* ranges;                   // [tiles]
};
struct EmitArgs {
    EmitSeg seg[GS_MAX_VIEWS];
    int64_t n;        // Gaussians, the same in every view
    int64_t nb_emit;  // chunks of kEmitChunk Gaussians
    int tiles_x;
    int64_t tiles;
};

// The culled binning's counts for one chunk of kEmitChunk depth-ordered
// Gaussians, in halves of one Gaussian per thread: each thread sets up its
// Gaussian's footprint bound (tile_reach.cuh) in shared memory, a block scan
// numbers the rows of all the half's rectangles, and the block's threads then
// take those rows round-robin (so that no warp waits on its tallest
// Gaussian's rows), adding each row's run length to its Gaussian's count in
// shared memory and writing the runs of the first kRunRows rows as (first
// column << 16 | length) for the emission.  A Gaussian whose conic is not
// positive definite counts its whole rectangle, one that reaches nothing 0.
// Returns this thread's share of the chunk's instances.
__device__ unsigned long long culled_counts(const EmitArgs& a, const EmitSeg& g, int64_t base) {
    constexpr int kHalf = kEmitBlock;
    __shared__ TileReach s_tr[kHalf];
    __shared__ uint2 s_rect[kHalf];
    __shared__ uint32_t s_roff[kHalf + 1];
    __shared__ uint32_t s_cnt[kHalf];
    unsigned long long sum = 0;
    const int t = threadIdx.x;
    for (int half = 0; half < kEmitChunk / kHalf; ++half) {
        const int64_t i = base + int64_t(half) * kHalf + t;
        uint32_t rows = 0, direct = 0;
        if (i < a.n) {
            const uint32_t gid = __ldg(g.order + i);
            if (__ldg(g.touched + gid)) {
                const uint2 r = __ldg(g.rect + gid);
                const uint32_t w = (r.y & 0xffffu) - (r.x & 0xffffu), h = (r.y >> 16) - (r.x >> 16);
                const TileReach R = tile_reach_setup(__ldg(g.xy + gid), __ldg(g.con + gid));
                s_tr[t] = R;
                s_rect[t] = r;
                if (R.mode == 1) rows = h;
                else if (R.mode == 2) direct = w * h;
                // runs past the rectangle's last row read as empty
                uint32_t* out = g.runs + i * kRunRows;
                for (int k = int(rows); k < kRunRows; ++k) out[k] = 0u;
            }
        }
        s_cnt[t] = direct;
        unsigned long long tot;
        const uint32_t off = uint32_t(block_excl_scan(rows, &tot));
        s_roff[t] = off;
        if (t == 0) s_roff[kHalf] = uint32_t(tot);
        __syncthreads();
        for (uint32_t q = t; q < uint32_t(tot); q += kEmitBlock) {
            // the last Gaussian whose first row is <= q (it has at least one row)
            int lo = 0;
#pragma unroll
            for (int step = kHalf / 2; step > 0; step >>= 1)
                if (s_roff[lo + step] <= q) lo += step;
            const int k = int(q - s_roff[lo]);
            const uint2 r = s_rect[lo];
            const int x0 = int(r.x & 0xffffu), y0 = int(r.x >> 16), x1 = int(r.y & 0xffffu);
            int c0, c1;
            tile_reach_row(s_tr[lo], y0 + k, x0, x1, &c0, &c1);
            if (c1 > c0) atomicAdd(&s_cnt[lo], uint32_t(c1 - c0));
            if (k < kRunRows)
                g.runs[(base + int64_t(half) * kHalf + lo) * kRunRows + k] = (uint32_t(c0) << 16) | uint32_t(c1 - c0);
        }
        __syncthreads();
        if (i < a.n) {
            g.cnt[i] = s_cnt[t];
            sum += s_cnt[t];
        }
        __syncthreads();  // the shared arrays are reused by the next half
    }
    return sum;
}

// Per block of kEmitChunk depth-ordered Gaussians, the sum of their instance
// counts: tiles_touched, or in the culled binning the counts of culled_counts
// (stored with the runs for the emission).
__global__ void __launch_bounds__(kEmitBlock) count_sorted_kernel(const __grid_constant__ EmitArgs a) {
    const EmitSeg& g = a.seg[blockIdx.y];
    const int64_t base = int64_t(blockIdx.x) * kEmitChunk;
    unsigned long long sum = 0;
    if (g.runs) {
        sum = culled_counts(a, g, base);
    } else {
        for (int k = threadIdx.x; k < kEmitChunk; k += kEmitBlock) {
            const int64_t i = base + k;
            if (i < a.n) sum += __ldg(g.touched + __ldg(g.order + i));
        }
    }
    unsigned long long tot;
    block_excl_scan(sum, &tot);
    if (threadIdx.x == 0) g.block_sums[blockIdx.x] = tot;
}

// One CTA per view: exclusive scan of the view's block sums, its total K.
__global__ void __launch_bounds__(1024) scan_blocks_kernel(const __grid_constant__ EmitArgs a) {
    const EmitSeg& g = a.seg[blockIdx.x];
    unsigned long long carry = 0;
    for (int64_t base = 0; base < a.nb_emit; base += 1024) {
        const int64_t i = base + threadIdx.x;
        const unsigned long long v = i < a.nb_emit ? g.block_sums[i] : 0ull;
        unsigned long long tot;
        const unsigned long long ex = block_excl_scan(v, &tot);
        if (i < a.nb_emit) g.block_sums[i] = carry + ex;
        carry += tot;
    }
    if (threadIdx.x == 0) {
        *g.total = carry;
        if (g.count_out) *g.count_out = carry;
    }
}

// Instances of the block's Gaussians (depth order), load-balanced: the block's
// output slots [0, total) are dealt to its threads round-robin, and each slot
// finds its Gaussian by a binary search over the block's exclusive offsets in
// shared memory, then its tile: from its index inside the Gaussian's tile
// rectangle (row-major) when the Gaussian covers all of it, else (culled
// binning) from the runs of tiles count_sorted kept for its first rows, and
// past those rows from tile_reach_row again.  Consecutive slots are written by
// consecutive threads.
__global__ void __launch_bounds__(kEmitBlock) emit_kernel(const __grid_constant__ EmitArgs a) {
    __shared__ uint32_t s_start[kEmitChunk];
    __shared__ uint32_t s_gid[kEmitChunk];
    __shared__ uint2 s_rect[kEmitChunk];
    __shared__ unsigned char s_walk[kEmitChunk];
    __shared__ uint4 s_runs[kEmitChunk][kRunRows / 4];
    const EmitSeg& g = a.seg[blockIdx.y];
    if (g.inst.get() == 0) return;  // nothing fits: emit nothing
    const int64_t first = int64_t(blockIdx.x) * kEmitChunk + int64_t(threadIdx.x) * kEmitPerThread;
    uint32_t gid[kEmitPerThread], tt[kEmitPerThread];
    unsigned long long mine = 0;
#pragma unroll
    for (int k = 0; k < kEmitPerThread; ++k) {
        gid[k] = first + k < a.n ? __ldg(g.order + first + k) : 0u;
        tt[k] = first + k < a.n ? (g.runs ? __ldg(g.cnt + first + k) : __ldg(g.touched + gid[k])) : 0u;
        mine += tt[k];
    }
    unsigned long long total;
    uint32_t run = uint32_t(block_excl_scan(mine, &total));
    const unsigned long long base = g.block_sums[blockIdx.x];
#pragma unroll
    for (int k = 0; k < kEmitPerThread; ++k) {
        const int idx = threadIdx.x * kEmitPerThread + k;
        s_start[idx] = run;
        s_gid[idx] = gid[k];
        const uint2 r = tt[k] ? __ldg(g.rect + gid[k]) : make_uint2(0u, 0u);
        s_rect[idx] = r;
        const uint32_t area = ((r.y & 0xffffu) - (r.x & 0xffffu)) * ((r.y >> 16) - (r.x >> 16));
        const bool walk = g.runs && tt[k] != 0u && tt[k] != area;
        s_walk[idx] = walk;
        if (walk) {
            const uint4* src = reinterpret_cast<const uint4*>(g.runs + (first + k) * kRunRows);
#pragma unroll
            for (int q = 0; q < kRunRows / 4; ++q) s_runs[idx][q] = __ldg(src + q);
        }
        run += tt[k];
    }
    __syncthreads();
    for (uint32_t slot = threadIdx.x; slot < uint32_t(total); slot += kEmitBlock) {
        // the last Gaussian whose first slot is <= slot (it has at least one instance)
        int lo = 0;
#pragma unroll
        for (int step = kEmitChunk / 2; step > 0; step >>= 1)
            if (s_start[lo + step] <= slot) lo += step;
        const uint32_t j = slot - s_start[lo];
        const uint2 r = s_rect[lo];
        const int x0 = int(r.x & 0xffffu), y0 = int(r.x >> 16), x1 = int(r.y & 0xffffu), y1 = int(r.y >> 16);
        uint32_t tx, ty;
        if (!s_walk[lo]) {
            const uint32_t w = uint32_t(x1 - x0);
            ty = uint32_t(y0) + j / w;
            tx = uint32_t(x0) + j % w;
        } else {
            // a count that matches no walk (tiles_touched written under another
            // rule) leaves tile 0: a valid tile id, never a range written out of bounds
            tx = 0u;
            ty = 0u;
            uint32_t rest = j;
            bool found = false;
            const uint32_t* rr = reinterpret_cast<const uint32_t*>(s_runs[lo]);
#pragma unroll
            for (int k = 0; k < kRunRows; ++k) {
                const uint32_t m = rr[k] & 0xffffu;  // 0 past the rectangle's last row
                if (!found && rest < m) {
                    tx = (rr[k] >> 16) + rest;
                    ty = uint32_t(y0 + k);
                    found = true;
                }
                if (!found) rest -= m;
            }
            if (!found && y1 - y0 > kRunRows) {
                const uint32_t gg = s_gid[lo];
                const TileReach R = tile_reach_setup(__ldg(g.xy + gg), __ldg(g.con + gg));
                for (int y = y0 + kRunRows; y < y1; ++y) {
                    int c0, c1;
                    tile_reach_row(R, y, x0, x1, &c0, &c1);
                    const uint32_t m = uint32_t(c1 - c0);
                    if (rest < m) {
                        tx = uint32_t(c0) + rest;
                        ty = uint32_t(y);
                        break;
                    }
                    rest -= m;
                }
            }
        }
        g.tkey[base + slot] = ty * uint32_t(a.tiles_x) + tx;
        g.tval[base + slot] = s_gid[lo];
    }
}

// Every view's tile ranges empty: [0, 0).
__global__ void __launch_bounds__(256) zero_ranges_kernel(const __grid_constant__ EmitArgs a) {
    const EmitSeg& g = a.seg[blockIdx.y];
    for (int64_t t = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; t < a.tiles; t += int64_t(gridDim.x) * blockDim.x)
        g.ranges[t] = make_uint2(0u, 0u);
}

// Four consecutive keys per thread: a tile starts at k when the key before k has
// another tile, and ends after k when the key after k does.
__global__ void __launch_bounds__(256) ranges_kernel(const __grid_constant__ EmitArgs a) {
    const EmitSeg& g = a.seg[blockIdx.y];
    const int64_t K = g.inst.get();
    for (int64_t k0 = 4 * (blockIdx.x * int64_t(blockDim.x) + threadIdx.x); k0 < K;
         k0 += 4 * int64_t(gridDim.x) * blockDim.x) {
        uint32_t t[6];  // tiles of keys k0 - 1 .. k0 + 4 (0xffffffff past either end)
#pragma unroll
        for (int i = 0; i < 6; ++i) {
            const int64_t k = k0 - 1 + i;
            t[i] = k >= 0 && k < K ? uint32_t(__ldg(g.keys + k) >> 32) : 0xffffffffu;
        }
#pragma unroll
        for (int i = 1; i < 5; ++i) {
            if (k0 - 1 + i >= K) break;
            if (t[i - 1] != t[i]) g.ranges[t[i]].x = uint32_t(k0 - 1 + i);
            if (t[i + 1] != t[i]) g.ranges[t[i]].y = uint32_t(k0 + i);
        }
    }
}

size_t align_up(size_t x) { return (x + 255) & ~size_t(255); }

// One LSD pass over every segment of `a` (a.shift and a.digit_bits set for the
// pass): the grid covers the segment with the most blocks.
void radix_pass(const PassArgs& a, int segments, bool final, cudaStream_t s) {
    int64_t nb = 0;
    for (int v = 0; v < segments; ++v) nb = a.seg[v].nb > nb ? a.seg[v].nb : nb;
    if (nb == 0 || segments == 0) return;
    const dim3 grid(static_cast<unsigned>(nb), static_cast<unsigned>(segments));
    upsweep_kernel<<<grid, kSortBlock, 0, s>>>(a);
    scan_hist_kernel<<<dim3(256, unsigned(segments)), 1024, 0, s>>>(a);
    if (final)
        downsweep_kernel<true><<<grid, kSortBlock, 0, s>>>(a);
    else
        downsweep_kernel<false><<<grid, kSortBlock, 0, s>>>(a);
    count_launches(3);
}

int64_t sort_blocks(int64_t slots) { return (slots + kSortTile - 1) / kSortTile; }

}  // namespace

size_t sort_workspace_layout(int64_t n, int64_t capacity, bool cull, void* base, SortWorkspace* ws) {
    const int64_t nb_emit = (n + kEmitChunk - 1) / kEmitChunk;
    const int64_t slots = capacity > n ? capacity : n;  // the depth sort borrows the tile buffers
    const int64_t nb_sort = (slots + kSortTile - 1) / kSortTile;
    size_t off = 0;
    char* b = static_cast<char*>(base);
    SortWorkspace w;
    w.nb_emit = nb_emit;
    w.nb_sort = nb_sort;
    w.block_sums = reinterpret_cast<unsigned long long*>(b + off);
    off += align_up(sizeof(unsigned long long) * size_t(nb_emit > 0 ? nb_emit : 1));
    w.total = reinterpret_cast<unsigned long long*>(b + off);
    off += align_up(sizeof(unsigned long long));
    for (int r = 0; r < 2; ++r) {
        w.tkey[r] = reinterpret_cast<uint32_t*>(b + off);
        off += align_up(sizeof(uint32_t) * size_t(slots > 0 ? slots : 1));
        w.tval[r] = reinterpret_cast<uint32_t*>(b + off);
        off += align_up(sizeof(uint32_t) * size_t(slots > 0 ? slots : 1));
    }
    w.hist = reinterpret_cast<uint32_t*>(b + off);
    off += align_up(sizeof(uint32_t) * 256 * size_t(nb_sort > 0 ? nb_sort : 1));
    w.digit_totals = reinterpret_cast<uint32_t*>(b + off);
    off += align_up(sizeof(uint32_t) * 256);
    w.runs = nullptr;
    w.cnt = nullptr;
    if (cull) {
        w.runs = reinterpret_cast<uint32_t*>(b + off);
        off += align_up(sizeof(uint32_t) * kRunRows * size_t(n > 0 ? n : 1));
        w.cnt = reinterpret_cast<uint32_t*>(b + off);
        off += align_up(sizeof(uint32_t) * size_t(n > 0 ? n : 1));
    }
    if (ws) *ws = w;
    return off;
}

size_t depth_order_workspace_layout(int64_t n, int views, void* base, DepthOrderWorkspace* ws) {
    const int64_t total = n * views;
    const int64_t nb = (n + kSortTile - 1) / kSortTile;
    size_t off = 0;
    char* b = static_cast<char*>(base);
    DepthOrderWorkspace w;
    w.nb = nb;
    for (int r = 0; r < 2; ++r) {
        w.key[r] = reinterpret_cast<uint32_t*>(b + off);
        off += align_up(sizeof(uint32_t) * size_t(total > 0 ? total : 1));
        w.val[r] = reinterpret_cast<uint32_t*>(b + off);
        off += align_up(sizeof(uint32_t) * size_t(total > 0 ? total : 1));
    }
    w.hist = reinterpret_cast<uint32_t*>(b + off);
    off += align_up(sizeof(uint32_t) * 256 * size_t(nb > 0 ? nb : 1) * size_t(views > 0 ? views : 1));
    w.digit_totals = reinterpret_cast<uint32_t*>(b + off);
    off += align_up(sizeof(uint32_t) * 256 * size_t(views > 0 ? views : 1));
    if (ws) *ws = w;
    return off;
}

cudaError_t launch_depth_order(const gs_projected* projs, int views, int64_t n, const DepthOrderWorkspace& ws,
                               uint32_t* order, cudaStream_t s) {
    if (n == 0 || views == 0) return cudaSuccess;
    ViewDepths src;
    for (int v = 0; v < views; ++v) {
        src.touched[v] = projs[v].tiles_touched;
        src.depth[v] = projs[v].depth;
    }
    const dim3 kgrid(grid_for(n, 256, 8), static_cast<unsigned>(views));
    depth_keys_views_kernel<<<kgrid, 256, 0, s>>>(src, n, ws.key[0], ws.val[0]);
    count_launches(1);
    // four stable 8-bit passes A -> B -> A -> B -> (A, order), every view a segment
    for (int p = 0; p < 4; ++p) {
        const int b = p & 1;
        PassArgs a;
        a.shift = 8 * p;
        a.digit_bits = 8;
        for (int v = 0; v < views; ++v) {
            const int64_t o = int64_t(v) * n;
            PassSeg& g = a.seg[v];
            g.kin = ws.key[b] + o;
            g.vin = ws.val[b] + o;
            g.kout = ws.key[b ^ 1] + o;
            g.kout64 = nullptr;
            g.vout = (p == 3 ? order : ws.val[b ^ 1]) + o;
            g.hist = ws.hist + int64_t(v) * 256 * ws.nb;
            g.digit_totals = ws.digit_totals + int64_t(v) * 256;
            g.depth = nullptr;
            g.cnt = Count{n, nullptr, 0};
            g.nb = ws.nb;
        }
        radix_pass(a, views, false, s);
    }
    return cudaGetLastError();
}

cudaError_t launch_bin_sort(const gs_projected& proj, int64_t n, const CamArgs& cam, const SortWorkspace& ws,
                            uint64_t* keys, uint32_t* vals, int64_t capacity, uint32_t* ranges,
                            unsigned long long* count_out, cudaStream_t s) {
    if (n > 0) {
        // depth order of the Gaussians: 4 passes from buffer 1 back into buffer 1, so
        // that tval[1] holds the order while the instances are emitted into buffer 0
        ViewDepths src;
        src.touched[0] = proj.tiles_touched;
        src.depth[0] = proj.depth;
        depth_keys_views_kernel<<<dim3(grid_for(n, 256, 8), 1), 256, 0, s>>>(src, n, ws.tkey[1], ws.tval[1]);
        count_launches(1);
        for (int p = 0; p < 4; ++p) {
            const int b = (p & 1) ? 0 : 1;
            PassArgs a;
            a.shift = 8 * p;
            a.digit_bits = 8;
            PassSeg& g = a.seg[0];
            g.kin = ws.tkey[b];
            g.vin = ws.tval[b];
            g.kout = ws.tkey[b ^ 1];
            g.kout64 = nullptr;
            g.vout = ws.tval[b ^ 1];
            g.hist = ws.hist;
            g.digit_totals = ws.digit_totals;
            g.depth = nullptr;
            g.cnt = Count{n, nullptr, 0};
            g.nb = sort_blocks(n);
            radix_pass(a, 1, false, s);
        }
    }
    return launch_bin_sort_ordered_views(1, &proj, n, &ws.tval[1], cam, &ws, &keys, &vals, &capacity, &ranges,
                                         &count_out, s);
}

cudaError_t launch_bin_sort_ordered(const gs_projected& proj, int64_t n, const uint32_t* order, const CamArgs& cam,
                                    const SortWorkspace& ws, uint64_t* keys, uint32_t* vals, int64_t capacity,
                                    uint32_t* ranges, unsigned long long* count_out, cudaStream_t s) {
    return launch_bin_sort_ordered_views(1, &proj, n, &order, cam, &ws, &keys, &vals, &capacity, &ranges, &count_out,
                                         s);
}

cudaError_t launch_bin_sort_ordered_views(int views, const gs_projected* projs, int64_t n,
                                          const uint32_t* const* orders, const CamArgs& cam, const SortWorkspace* ws,
                                          uint64_t* const* keys, uint32_t* const* vals, const int64_t* capacity,
                                          uint32_t* const* ranges, unsigned long long* const* count_out,
                                          cudaStream_t s) {
    if (views == 0) return cudaSuccess;
    const int64_t T = int64_t(cam.TX) * cam.TY;
    EmitArgs e;
    e.n = n;
    e.nb_emit = ws[0].nb_emit;  // n alone sets it: the same in every view
    e.tiles_x = cam.TX;
    e.tiles = T;
    int64_t cap_max = 0;
    for (int v = 0; v < views; ++v) {
        EmitSeg& g = e.seg[v];
        g.touched = projs[v].tiles_touched;
        g.rect = reinterpret_cast<const uint2*>(projs[v].rect);
        g.xy = reinterpret_cast<const float2*>(projs[v].xy);
        g.con = reinterpret_cast<const float4*>(projs[v].conic_opacity);
        g.runs = ws[v].runs;
        g.cnt = ws[v].cnt;
        g.order = orders[v];
        g.block_sums = ws[v].block_sums;
        g.total = ws[v].total;
        g.count_out = count_out[v];
        g.inst = Count{0, ws[v].total, capacity[v]};
        g.tkey = ws[v].tkey[0];
        g.tval = ws[v].tval[0];
        g.keys = keys[v];
        g.ranges = reinterpret_cast<uint2*>(ranges[v]);
        cap_max = capacity[v] > cap_max ? capacity[v] : cap_max;
    }
    const unsigned V = static_cast<unsigned>(views);
    zero_ranges_kernel<<<dim3(grid_for(T, 256, 2), V), 256, 0, s>>>(e);
    count_launches(1);
    if (e.nb_emit > 0)
        count_sorted_kernel<<<dim3(unsigned(e.nb_emit), V), kEmitBlock, 0, s>>>(e);
    scan_blocks_kernel<<<V, 1024, 0, s>>>(e);  // n = 0: every K is 0
    count_launches(e.nb_emit > 0 ? 2 : 1);
    if (n == 0) return cudaGetLastError();
    // instances: launched for the capacities, K read on the device
    emit_kernel<<<dim3(unsigned(e.nb_emit), V), kEmitBlock, 0, s>>>(e);
    count_launches(1);
    const int bits = tile_bits(T);
    const int passes = bits > 0 ? (bits + 7) / 8 : 1;
    int cur = 0;
    for (int p = 0; p < passes; ++p) {
        const bool last = p == passes - 1;
        PassArgs a;
        a.shift = 8 * p;
        a.digit_bits = last ? bits - 8 * p : 8;
        for (int v = 0; v < views; ++v) {
            PassSeg& g = a.seg[v];
            g.kin = ws[v].tkey[cur];
            g.vin = ws[v].tval[cur];
            g.kout = last ? nullptr : ws[v].tkey[cur ^ 1];
            g.kout64 = last ? keys[v] : nullptr;
            g.vout = last ? vals[v] : ws[v].tval[cur ^ 1];
            g.hist = ws[v].hist;
            g.digit_totals = ws[v].digit_totals;
            g.depth = projs[v].depth;
            g.cnt = e.seg[v].inst;
            g.nb = sort_blocks(capacity[v]);
        }
        radix_pass(a, views, last, s);
        cur ^= 1;
    }
    if (cap_max > 0) {
        ranges_kernel<<<dim3(grid_for((cap_max + 3) / 4, 256, 8), V), 256, 0, s>>>(e);
        count_launches(1);
    }
    return cudaGetLastError();
}

}  // namespace gsk
