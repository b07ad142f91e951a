// Order-preserving compaction over contiguous chunks of elements, shared by the
// densification (parameters and moments into new arrays) and the packed
// projection (visible Gaussians into packed feature arrays).
//
// A "plan" launch gives one block per chunk and counts the chunk's outputs; the
// offsets launch below turns the counts into exclusive offsets; an "apply"
// launch over the same chunks recovers every element's output slot from a
// block-wide scan of the per-element output counts.  The chunking is a function
// of the element count alone, so the plan and the apply launches agree.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "internal.cuh"

namespace gsk {
namespace compact {

constexpr int kBlock = 128;
constexpr int kMaxChunks = kNumSMs * 8;

struct Chunking {
    int64_t chunk;  // elements per block, a multiple of kBlock
    int blocks;
};

inline Chunking chunking(int64_t n) {
    int64_t tiles = (n + kBlock - 1) / kBlock;
    int64_t blocks = tiles < kMaxChunks ? tiles : kMaxChunks;
    if (blocks < 1) blocks = 1;
    const int64_t tiles_per_block = (tiles + blocks - 1) / blocks;
    blocks = tiles_per_block > 0 ? (tiles + tiles_per_block - 1) / tiles_per_block : 1;
    if (blocks < 1) blocks = 1;
    return {tiles_per_block * kBlock, int(blocks)};
}

// Device workspace of a compaction: the chunk counts (then offsets) and the total.
inline size_t workspace_bytes(int64_t n) {
    const size_t bytes = (size_t(chunking(n).blocks) + 1) * sizeof(unsigned long long);
    return (bytes + 255) & ~size_t(255);
}

// Inclusive block-wide sum scan of one value per thread (kBlock threads);
// block_total receives the sum over the block.
__device__ __forceinline__ unsigned block_inclusive_scan(unsigned x, unsigned* warp_tot, unsigned& block_total) {
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
        const unsigned y = __shfl_up_sync(0xffffffffu, x, d);
        if (lane >= d) x += y;
    }
    if (lane == 31) warp_tot[w] = x;
    __syncthreads();
    if (w == 0) {
        unsigned t = lane < kBlock / 32 ? warp_tot[lane] : 0u;
#pragma unroll
        for (int d = 1; d < 32; d <<= 1) {
            const unsigned y = __shfl_up_sync(0xffffffffu, t, d);
            if (lane >= d) t += y;
        }
        if (lane < kBlock / 32) warp_tot[lane] = t;
    }
    __syncthreads();
    const unsigned before = w > 0 ? warp_tot[w - 1] : 0u;
    block_total = warp_tot[kBlock / 32 - 1];
    __syncthreads();
    return x + before;
}

namespace {  // one copy of the kernel per translation unit that launches it

// Exclusive scan of the chunk counts in place (one block of 1024 threads, each
// owning a contiguous run), the total to *total and *total_copy (nullable).
__global__ void __launch_bounds__(1024) chunk_offsets_kernel(unsigned long long* counts, int nb,
                                                             unsigned long long* total,
                                                             unsigned long long* total_copy) {
    __shared__ unsigned long long part[1024];
    const int per = (nb + 1023) / 1024;
    const int b0 = threadIdx.x * per;
    const int b1 = b0 + per < nb ? b0 + per : nb;
    unsigned long long s = 0;
    for (int b = b0; b < b1; ++b) s += counts[b];
    part[threadIdx.x] = s;
    __syncthreads();
    for (int d = 1; d < 1024; d <<= 1) {
        const unsigned long long y = threadIdx.x >= d ? part[threadIdx.x - d] : 0ull;
        __syncthreads();
        part[threadIdx.x] += y;
        __syncthreads();
    }
    unsigned long long run = part[threadIdx.x] - s;
    for (int b = b0; b < b1; ++b) {
        const unsigned long long c = counts[b];
        counts[b] = run;
        run += c;
    }
    if (threadIdx.x == 1023) {
        *total = part[1023];
        if (total_copy) *total_copy = part[1023];
    }
}

}  // namespace
}  // namespace compact
}  // namespace gsk
