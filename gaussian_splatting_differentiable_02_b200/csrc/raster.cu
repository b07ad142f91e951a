// gs_raster_fwd / gs_raster_bwd: stage 3 of the pipeline, differentiable
// front-to-back alpha blending per 16x16 tile (gsplat guide, lmnt.cn/news/262699
// §2.1: shared-memory prefetch of the tile's Gaussians, SoA features, warp-level
// synchronisation; §2.2: a standalone backward entry).
//
// Work decomposition: one warp per pixel box of a tile, one warp per block, blocks
// launched in the tile order of gs_tile_order when one is given; each lane owns a
// column segment of PX pixels (lane & 15 selects the column, lane >> 4 the upper
// or lower half of the box).  The backward on large tile grids takes PX = 8, a
// box per tile, so that the per-entry work of the warp (its shared-memory reads,
// the gradient sums, the branches) is spread over 256 pixels, on small grids
// PX = 4, two boxes per tile, for twice the warps; the forward takes PX = 4 on
// every grid (Layout below).  The warp walks its
// tile's sorted list in batches of 32 entries: every lane gathers one entry's
// 40 bytes (xy, conic + opacity, colour) by Gaussian index into shared memory
// with cp.async, double-buffered so the next batch is in flight while the
// current one is composited; the lane that gathered an entry also derives its
// per-entry constants and tests the entry against the warp's whole box (an
// entry whose smallest sigma over the box leaves alpha below 1/255 is dropped,
// and the constants of the others are compacted, so the warp's loop visits only
// entries that can reach its box).  Every lane then reads each entry once
// (broadcast loads) and
// applies it to its PX pixels, whose terms that depend only on dx are shared;
// the pixels go in pairs through the paired float32 instructions of sm_100
// (fma/mul/add on two floats at once).  No block-wide barrier is used: warps
// synchronise with __syncwarp and finish independently.
//
// Forward: a warp stops as soon as all of its pixels have terminated (warp vote
// per entry).  Backward: back to front from the largest n_contrib of the box,
// the transmittance in front of each entry recovered with rcp(1 - alpha) and
// g . S (S the colour blended behind) tracked per pixel; each lane sums its
// pixels' contributions as 9 moments of the entry (dL/dsigma against 1, dx,
// dy, ... and the colour terms), stashes them in shared memory, and every 8
// entries the warp adds the stashed moments up across its lanes, turns each
// entry's sums into its Gaussian's gradients with the entry's conic, and one
// lane per entry issues a float2 and two float4 atomic adds (batched atomics,
// MUSA co-design article qwbw.cn/news/278220 §2.2; EntrySums below).
//
// Both passes evaluate alpha with the same inline code built from explicit
// rounding intrinsics, so the backward pass repeats the forward pass's skip and
// clamp decisions exactly.
//
// Conditioning: sigma = 1/2 (A dx^2 + C dy^2) + B dx dy cancels badly far along
// the long axis of a needle-shaped Gaussian (the terms grow with the condition
// number of the conic).  Entries whose conic has an eigenvalue ratio above 8
// use the factored form sigma = 1/2 A t^2 + 1/2 D dy^2 with t = dx + (B/A) dy
// and D = det / A: both terms are non-negative, and t is formed with B/A split
// into two floats, so the float32 evaluation keeps a relative error of a few
// ulps whatever the conditioning; dsigma/du = A t and dsigma/dv = B t + D dy.
// The factors are derived once per entry in double.
#include <type_traits>

#include "internal.cuh"

namespace gsk {
namespace {

constexpr float kAlphaMax = 0.99f;
constexpr float kAlphaMin = 1.0f / 255.0f;
constexpr float kTMin = 1e-4f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr double kLog2eD = 1.4426950408889634;
// trace^2 / det = kappa + 1/kappa + 2 for the eigenvalue ratio kappa; kappa = 8 -> 10.125
constexpr float kCondMaxTraceSqOverDet = 10.125f;

// Warp layouts: a warp composites a box 16 pixels wide and 2 PX tall, each lane a
// column segment of PX pixels (lane & 15 selects the column, lane >> 4 the upper
// or lower half of the box); one warp per block, so that a block retires with its
// own box.  PX = 8: the box is the whole tile, and the warp's per-entry work (its
// shared-memory reads, the gradient reduction, the branches) is spread over 256
// pixels; PX = 4: two warps a tile, which culls entries against half tiles and
// gives twice the warps.  The backward uses PX = 8 on grids of at least
// kWideLayoutTiles tiles and PX = 4 on smaller ones; the forward uses PX = 4 on
// grids below kWideLayoutTilesFwd (every grid by default).  Measured (forward /
// backward ms per view) over the rectangle binning's lists: 16 1080p views of the
// 1M mixture (8160 tiles) PX = 8 at 14 / 16 blocks an SM 0.589 / 1.067, PX = 4 at
// 20 / 20 blocks 0.606 / 1.166; the 1296x840 view (4293 tiles) PX = 8 0.454 /
// 0.856, PX = 4 0.404 / 0.806 (two warps a block, 10 blocks: 0.622 / 1.144 at
// 1080p; PX = 8 at 12 / 14 / 20 blocks slower).  Over the culled binning's lists,
// which hold about half the entries and so halve the staging PX = 4 pays twice,
// at 1080p: PX = 8 0.504 / 0.970, PX = 4 0.463 / 1.012.
constexpr int kBoxW = 16;               // width of a warp's pixel box
constexpr int kWarps = 1;               // warps per block
#ifndef GS_WIDE_LAYOUT_TILES
#define GS_WIDE_LAYOUT_TILES 6144
#endif
constexpr int64_t kWideLayoutTiles = GS_WIDE_LAYOUT_TILES;
#ifndef GS_WIDE_LAYOUT_TILES_FWD
#define GS_WIDE_LAYOUT_TILES_FWD (int64_t(1) << 40)
#endif
constexpr int64_t kWideLayoutTilesFwd = GS_WIDE_LAYOUT_TILES_FWD;
#ifndef GS_FWD_PX
#define GS_FWD_PX 4  // the forward's layout below kWideLayoutTilesFwd
#endif
#ifndef GS_RASTER_FWD_BLOCKS2
#define GS_RASTER_FWD_BLOCKS2 32
#endif
#ifndef GS_RASTER_BWD_BLOCKS8
#define GS_RASTER_BWD_BLOCKS8 16
#endif
template <int PX>
struct Layout {
    static_assert(PX % 2 == 0 && kTile % (2 * PX) == 0, "pixel pairs; boxes tile the 16x16 tile");
    static constexpr int kPairs = PX / 2;                // pixel pairs per lane
    static constexpr int kBoxH = 2 * PX;                 // height of a warp's box
    static constexpr int kSub = kTile / kBoxH;           // warps per tile
    // resident blocks per SM the register allocation is sized for (launch bounds)
    static constexpr int kFwdMinBlocks = PX == 8 ? 14 : (PX == 4 ? 20 : GS_RASTER_FWD_BLOCKS2);
    static constexpr int kBwdMinBlocks = PX == 8 ? GS_RASTER_BWD_BLOCKS8 : 20;
};
constexpr int kBatch = 32;  // list entries staged per warp per batch
constexpr unsigned kFull = 0xffffffffu;

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp_approx(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ void cp_async16(void* smem, const void* gmem) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 16;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async8(void* smem, const void* gmem) {
    const unsigned s = static_cast<unsigned>(__cvta_generic_to_shared(smem));
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8;\n" ::"r"(s), "l"(gmem));
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;\n" ::); }

// Per-warp staging area: raw gathered features (double-buffered) and the
// per-entry constants derived from them.
// Evaluation of an entry (WarpStage::pb.w).
constexpr float kPlain = 0.f;          // expanded quadratic form in float32
constexpr float kSkip = 2.f;           // misses every pixel of the warp's box
constexpr float kFactored = 3.f;       // factored form 1/2 A t^2 + 1/2 D dy^2 in float32 (D > 0)
constexpr float kFactoredIndef = 4.f;  // the same with D <= 0 (a float32 conic that rounded to indefinite):
                                       // sigma can be negative, and such pixels are skipped
constexpr int kMayClampBit = 32;       // WarpStage::idx: the entry's alpha can reach the 0.99 clamp

struct WarpStage {
    float2 xy[2][kBatch];
    float4 con[2][kBatch];  // A, B, C, o
    float4 rgb[2][kBatch];
    uint32_t gid[2][kBatch];
    // per-entry constants of the batch's entries that reach the warp's box, compacted
    // in list order; idx is the entry's index in the batch
    float4 pa[kBatch];  // u, v, log2(o), 1/o
    float4 pb[kBatch];  // plain: -log2e A/2, -log2e B, -log2e C/2; factored: B/A (high, low part), D; flag
    float2 pc[kBatch];  // factored: -log2e A/2, -log2e D/2
    int idx[kBatch];
};

// Lane l < count gathers list entry first + l (reverse: first + count - 1 - l).
template <bool kReverse>
__device__ __forceinline__ void gather(WarpStage& S, int buf, const uint32_t* __restrict__ vals,
                                       const float2* __restrict__ xy, const float4* __restrict__ con,
                                       const float4* __restrict__ rgb, uint32_t first, int count, int lane) {
    if (lane < count) {
        const uint32_t e = kReverse ? first + uint32_t(count - 1 - lane) : first + uint32_t(lane);
        const uint32_t g = __ldg(vals + e);
        S.gid[buf][lane] = g;
        cp_async8(&S.xy[buf][lane], xy + g);
        cp_async16(&S.con[buf][lane], con + g);
        cp_async16(&S.rgb[buf][lane], rgb + g);
    }
    cp_async_commit();
}

// Smallest sigma = 1/2 (A dx^2 + 2 B dx dy + C dy^2) with dx fixed and dy in
// [dylo, dyhi] (a positive definite form is minimised at dy = -B dx / C).
template <class R>
__device__ __forceinline__ R edge_min(R A, R B, R C, R dx, R dylo, R dyhi) {
    const R dy = fmin(fmax(-B * dx / C, dylo), dyhi);
    return R(0.5) * (A * dx * dx + R(2) * B * dx * dy + C * dy * dy);
}

// Smallest sigma over the box [bx0, bx1] x [by0, by1] of pixel centres: 0 with
// the mean inside, else the smallest of the four edge minima.
template <class R>
__device__ __forceinline__ R box_min(R A, R B, R C, R u, R v, R bx0, R bx1, R by0, R by1) {
    if (u >= bx0 && u <= bx1 && v >= by0 && v <= by1) return R(0);
    const R dxlo = u - bx1, dxhi = u - bx0, dylo = v - by1, dyhi = v - by0;
    R m = fmin(edge_min(A, B, C, dxlo, dylo, dyhi), edge_min(A, B, C, dxhi, dylo, dyhi));
    m = fmin(m, edge_min(C, B, A, dylo, dxlo, dxhi));
    return fmin(m, edge_min(C, B, A, dyhi, dxlo, dxhi));
}

// Lane l < count derives the constants of staged entry l.  pb.w selects the
// evaluation (kPlain, kFactored, kFactoredIndef) or kSkip: the smallest sigma over
// this warp's pixel box [bx0, bx0 + kBoxW - 1] x [by0, by0 + kBoxH - 1] (pixel
// centres) puts alpha below 1/255 everywhere in it, with a margin far above
// the rounding of either evaluation, so no pixel of the warp would blend it.
// The bound is computed in float32 for well-conditioned conics and in double
// for the others (never for an indefinite one).  The entries not skipped are
// written compacted, in batch order, to S.pa / S.pb / S.pc with their batch index
// in S.idx (bits 0-4) and kMayClamp (bit 5) when the entry's opacity is high
// enough for its alpha to reach the 0.99 clamp; returns their number.  Called by
// the whole warp.
template <bool kNegRgb, int PX>
__device__ __forceinline__ int prep(WarpStage& S, int buf, int count, int lane, float bx0, float by0) {
    constexpr int kBoxH = Layout<PX>::kBoxH;
    float4 pa = make_float4(0.f, 0.f, 0.f, 0.f), pb = make_float4(0.f, 0.f, 0.f, kSkip);
    float2 pc = make_float2(0.f, 0.f);
    bool may_clamp = false;
    if (lane < count) {
        if (kNegRgb) {  // the forward pass blends with -alpha T weights
            const float4 c = S.rgb[buf][lane];
            S.rgb[buf][lane] = make_float4(-c.x, -c.y, -c.z, c.w);
        }
        const float2 xy = S.xy[buf][lane];
        const float4 c = S.con[buf][lane];
        const float tr = __fadd_rn(c.x, c.z);
        const float det = __fsub_rn(__fmul_rn(c.x, c.z), __fmul_rn(c.y, c.y));
        const bool ill = !(det > 0.f) || (__fmul_rn(tr, tr) > __fmul_rn(kCondMaxTraceSqOverDet, det));
        const float lo = log2f(c.w);
        // alpha >= 1/255 needs sigma <= ln(255 o) = ln 255 + lo ln 2
        const float cut = 5.541263545158426f + lo * 0.6931471805599453f;
        const float bx1 = bx0 + float(kBoxW - 1), by1 = by0 + float(kBoxH - 1);
        if (!ill) {
            const float smin = box_min<float>(c.x, c.y, c.z, xy.x, xy.y, bx0, bx1, by0, by1);
            const float flag = smin * (1.f - 1e-4f) > cut + 1e-4f ? kSkip : kPlain;
            pb = make_float4(__fmul_rn(-0.5f * kLog2e, c.x), __fmul_rn(-kLog2e, c.y), __fmul_rn(-0.5f * kLog2e, c.z),
                             flag);
        } else {
            const double A = c.x, B = c.y, C = c.z;
            if (A > 0.0) {
                const double D = (A * C - B * B) / A;  // A C and B^2 are exact in double
                const double r = B / A;
                const float rh = __double2float_rn(r);
                float flag = kFactoredIndef;
                if (D > 0.0) {
                    const double smin = box_min<double>(A, B, C, xy.x, xy.y, bx0, bx1, by0, by1);
                    flag = smin * (1.0 - 1e-4) > double(cut) + 1e-4 ? kSkip : kFactored;
                }
                pb = make_float4(rh, __double2float_rn(r - double(rh)), float(D), flag);
                pc = make_float2(__double2float_rn(-0.5 * kLog2eD * A), __double2float_rn(-0.5 * kLog2eD * D));
            } else {
                // A = Sigma'_yy / det > 0 for every conic the projection writes; a
                // non-positive one has no meaningful footprint
                pb = make_float4(0.f, 0.f, 0.f, kSkip);
            }
        }
        pa = make_float4(xy.x, xy.y, lo, 1.f / c.w);
        // o e^-sigma evaluates to at most o (1 + a few 1e-7) (ex2.approx and the
        // rounding of the exponent near the mean), so an opacity 1e-5 below 0.99
        // never reaches the clamp: such entries skip the clamp and its gate
        may_clamp = c.w > kAlphaMax * (1.f - 1e-5f);
    }
    const unsigned keep = __ballot_sync(kFull, pb.w != kSkip);
    if (pb.w != kSkip) {
        const int k = __popc(keep & ((1u << lane) - 1u));
        S.pa[k] = pa;
        S.pb[k] = pb;
        S.pc[k] = pc;
        S.idx[k] = lane | (may_clamp ? kMayClampBit : 0);
    }
    return __popc(keep);
}

// Pairs of pixels go through the paired float32 instructions of sm_100
// (two IEEE operations per instruction, rounded as two scalar ones).
using f2 = float2;
__device__ __forceinline__ f2 splat(float v) { return make_float2(v, v); }
__device__ __forceinline__ f2 fma2(f2 a, f2 b, f2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ f2 mul2(f2 a, f2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ f2 add2(f2 a, f2 b) { return __fadd2_rn(a, b); }

// One entry at the lane's pixels: -alpha per pixel (pairs 2p, 2p + 1; 0 where the
// pixel fails sigma >= 0 or alpha >= 1/255, so that it does not blend the entry),
// the offsets dx (shared) and dy of the mean from the pixel centres, t = dx +
// (B/A) dy for a factored entry, and (backward pass) a gate that is 0 where alpha
// was clamped at 0.99 and 1 elsewhere.  The masks are floats rather than bits: a
// pixel that does not take an entry runs the same paired instructions with alpha
// 0, and a clamped pixel's dL/dsigma is multiplied by 0.
template <int PX>
struct Alpha {
    f2 nal[PX / 2];
    f2 dy[PX / 2];
    f2 t[PX / 2];
    f2 gate[PX / 2];  // 0 where alpha was clamped at 0.99, else 1 (backward pass)
    float dx;
};

// -alpha at one pixel, 0 for a pixel that does not blend the entry (sigma < 0 or
// alpha < 1/255); with kMayClamp alpha is clamped at 0.99 and (kGate) gate = 0 when
// it was, else 1; without, alpha cannot reach the clamp and no gate is formed.
// 1.0f where a >= b, else 0.0f: one compare that writes a float (the ALU pipe is
// the busier one in these loops, and the mask's product runs on the FMA pipe)
__device__ __forceinline__ float mask_ge(float a, float b) {
    float m;
    asm("set.ge.f32.f32 %0, %1, %2;" : "=f"(m) : "f"(a), "f"(b));
    return m;
}

template <bool kGate, bool kMayClamp>
__device__ __forceinline__ void alpha_at(float e, bool sign_ok, float& nal, float& gate) {
    const float a = ex2_approx(e);
    // min(a, 0.99) >= 1/255 exactly when a >= 1/255; a pixel that fails it (or the
    // sign test) gets -alpha = -0, which leaves every sum as it was
    const float m = sign_ok ? mask_ge(a, kAlphaMin) : 0.f;
    nal = (kMayClamp ? fmaxf(-a, -kAlphaMax) : -a) * m;  // -min(a, 0.99), or 0
    if (kGate && kMayClamp) gate = a > kAlphaMax ? 0.f : 1.f;
}

// nyc[p]: minus the centres' y of the lane's pixels 2p and 2p + 1.
template <bool kGate, bool kMayClamp, int PX>
__device__ __forceinline__ void eval_alpha(const float4& pa, const float4& pb, const float2& pc, const float4& con,
                                           float px, const f2 (&nyc)[PX / 2], Alpha<PX>& r) {
    constexpr int kPairs = PX / 2;
    const f2 vy = splat(pa.y);
    if (pb.w >= kFactored) {
        const bool indef = pb.w == kFactoredIndef;
        r.dx = __fsub_rn(pa.x, px);
        const f2 dx2 = splat(r.dx), rh = splat(pb.x), rl = splat(pb.y), ka = splat(pc.x), kd = splat(pc.y);
#pragma unroll
        for (int p = 0; p < kPairs; ++p) {
            r.dy[p] = add2(vy, nyc[p]);
            r.t[p] = fma2(rl, r.dy[p], fma2(rh, r.dy[p], dx2));
            const f2 sv = fma2(mul2(ka, r.t[p]), r.t[p], mul2(mul2(kd, r.dy[p]), r.dy[p]));
            const f2 e = add2(sv, splat(pa.z));
            // sigma >= 0 by construction unless the conic is indefinite
            alpha_at<kGate, kMayClamp>(e.x, !indef || sv.x <= 0.f, r.nal[p].x, r.gate[p].x);
            alpha_at<kGate, kMayClamp>(e.y, !indef || sv.y <= 0.f, r.nal[p].y, r.gate[p].y);
        }
    } else {
        r.dx = __fsub_rn(pa.x, px);
        // the terms that depend only on dx, with log2(o) added once per entry
        const f2 a0 = splat(__fadd_rn(__fmul_rn(__fmul_rn(pb.x, r.dx), r.dx), pa.z));
        const f2 c1 = splat(__fmul_rn(pb.y, r.dx));
        const f2 cz = splat(pb.z);
#pragma unroll
        for (int p = 0; p < kPairs; ++p) {
            r.dy[p] = add2(vy, nyc[p]);
            // a positive-definite form has sigma >= 0; the float32 value can round
            // below zero only within rounding of the mean, where alpha is o either way
            const f2 e = fma2(r.dy[p], fma2(cz, r.dy[p], c1), a0);
            alpha_at<kGate, kMayClamp>(e.x, true, r.nal[p].x, r.gate[p].x);
            alpha_at<kGate, kMayClamp>(e.y, true, r.nal[p].y, r.gate[p].y);
        }
    }
}

struct FwdArgs {
    const float2* xy;
    const float4* con;
    const float4* rgb;
    const uint32_t* vals;
    const uint2* ranges;
    const uint32_t* order;  // tile processing order (nullable)
    int W, H, TX, tiles;
    float bg0, bg1, bg2;
    float* image;
    float* final_T;
    int32_t* n_contrib;
    unsigned long long* counts;  // kCount only: work counters (gs_raster_fwd_counted)
    // kL1 only (gs_raster_fwd_l1): the L1 term of every rendered value against target
    const float* target;
    float* dL_dimage;
    double* loss;
    float inv_count;
    double inv_count_d;
};

// Work counters of the counted variants (one atomic per warp at its end): pairs
// the warp evaluated (entries that reach its box x its pixels), pairs that did
// the method's work (blended in the forward pass, took a gradient in the
// reverse pass), list entries staged, entries that reached the box, and (the
// forward pass) the pairs the method's per-pixel loop visits: for each pixel of
// the image, its tile's list up to the entry at which it stops, or all of it.
__device__ __forceinline__ void add_counts(unsigned long long* counts, int evaluated_entries, int work_pairs,
                                           int staged, int lane, int box_pixels, int visited = 0) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        work_pairs += __shfl_xor_sync(kFull, work_pairs, o);
        visited += __shfl_xor_sync(kFull, visited, o);
    }
    if (lane == 0) {
        atomicAdd(counts + 0, (unsigned long long)evaluated_entries * box_pixels);
        atomicAdd(counts + 1, (unsigned long long)work_pairs);
        atomicAdd(counts + 2, (unsigned long long)staged);
        atomicAdd(counts + 3, (unsigned long long)evaluated_entries);
        atomicAdd(counts + 4, (unsigned long long)visited);
    }
}

// kL1: the pixels' L1 terms against the target in the epilogue (gs_raster_fwd_l1):
// dL/dimage = sign(image - target) / count, and the warp's sum of |image - target|
// added to the loss with one double atomic, the arithmetic of gs_l1_loss_grad.
template <int PX, bool kCount, bool kL1>
__global__ void __launch_bounds__(kWarps * 32, Layout<PX>::kFwdMinBlocks) raster_fwd_kernel(const FwdArgs a) {
    constexpr int kPx = PX, kPairs = Layout<PX>::kPairs, kBoxH = Layout<PX>::kBoxH, kSub = Layout<PX>::kSub;
    __shared__ WarpStage stage[kWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gw = blockIdx.x * kWarps + warp;
    const int slot = gw / kSub, sub = gw % kSub;
    if (slot >= a.tiles) return;
    const int tile = a.order ? int(__ldg(a.order + slot)) : slot;  // longest lists first when ordered
    WarpStage& S = stage[warp];
    const int xb = (tile % a.TX) * kTile;  // this warp's pixel box
    const int yb = (tile / a.TX) * kTile + sub * kBoxH;
    const int x = xb + lane % kBoxW;
    const int y0 = yb + (lane / kBoxW) * kPx;
    const float px = float(x) + 0.5f;
    const float bx0 = float(xb) + 0.5f, by0 = float(yb) + 0.5f;  // box corner (pixel centre)
    const uint2 range = a.ranges[tile];
    const int n = int(range.y - range.x);

    f2 nyc[kPairs], T[kPairs], Cr[kPairs], Cg[kPairs], Cb[kPairs];
    int last[kPx];
    f2 on[kPairs];  // 1 while the pixel composites, 0 once it has stopped (or lies outside the image)
#pragma unroll
    for (int p = 0; p < kPairs; ++p) {
        nyc[p] = make_float2(-(float(y0 + 2 * p) + 0.5f), -(float(y0 + 2 * p + 1) + 0.5f));
        T[p] = splat(1.f);
        Cr[p] = Cg[p] = Cb[p] = splat(0.f);
        on[p] = splat(1.f);
    }
#pragma unroll
    for (int i = 0; i < kPx; ++i) {
        last[i] = 0;
        if (x >= a.W || y0 + i >= a.H) {
            if (i & 1)
                on[i / 2].y = 0.f;
            else
                on[i / 2].x = 0.f;
        }
    }
    const f2 one = splat(1.f);
    int c_eval = 0, c_work = 0, c_staged = 0;  // kCount only
    int stop[kCount ? kPx : 1];                // kCount: 1-based position of the entry a pixel stopped at, or 0
#pragma unroll
    for (int i = 0; i < (kCount ? kPx : 1); ++i) stop[i] = 0;

    const int nb = (n + kBatch - 1) / kBatch;
    if (n > 0) gather<false>(S, 0, a.vals, a.xy, a.con, a.rgb, range.x, min(n, kBatch), lane);
    for (int b = 0; b < nb; ++b) {
        const int buf = b & 1;
        const int cnt = min(n - b * kBatch, kBatch);
        cp_async_wait_all();
        __syncwarp();
        if (b + 1 < nb)
            gather<false>(S, buf ^ 1, a.vals, a.xy, a.con, a.rgb, range.x + uint32_t((b + 1) * kBatch),
                          min(n - (b + 1) * kBatch, kBatch), lane);
        const int live = prep<true, PX>(S, buf, cnt, lane, bx0, by0);
        __syncwarp();
        if (kCount) c_staged += cnt;
        bool finished = false;
        for (int e = 0; e < live; ++e) {  // the batch's entries that reach this warp's box
            f2 alive = on[0];  // nonzero while some pixel of the lane composites
#pragma unroll
            for (int p = 1; p < kPairs; ++p) alive = add2(alive, on[p]);
            if (__all_sync(kFull, alive.x + alive.y == 0.f)) {
                finished = true;
                break;
            }
            if (kCount) ++c_eval;
            const int ij = S.idx[e];
            const int j = ij & (kBatch - 1);
            const float4 pa = S.pa[e], pb = S.pb[e];
            const float4 con = S.con[buf][j];
            const float4 nc = S.rgb[buf][j];  // minus the colour
            Alpha<PX> r;
            const int pos = b * kBatch + j + 1;
            const f2 ncr = splat(nc.x), ncg = splat(nc.y), ncb = splat(nc.z);
            if (ij & kMayClampBit)
                eval_alpha<false, true, PX>(pa, pb, S.pc[e], con, px, nyc, r);
            else
                eval_alpha<false, false, PX>(pa, pb, S.pc[e], con, px, nyc, r);
            // branch-free with float masks: -alpha is 0 for a pixel that does not blend
            // the entry or has stopped (on 0), so T (1 - alpha) = T and -alpha T = 0
            // leave it exactly as it was; T (1 - alpha) < 1e-4 then only happens for a
            // pixel that blends, which stops there without taking the entry
#pragma unroll
            for (int p = 0; p < kPairs; ++p) {
                f2 na = mul2(r.nal[p], on[p]);
                const f2 Tn = mul2(T[p], add2(one, na));  // T (1 - alpha)
                // 1 while T (1 - alpha) >= 1e-4; a pixel that reaches 0 stops there
                // without the entry: its -alpha becomes 0, so T (1 - 0) = T exactly
                const f2 keep = make_float2(mask_ge(Tn.x, kTMin), mask_ge(Tn.y, kTMin));
                na = mul2(na, keep);
                const f2 nw = mul2(na, T[p]);  // -alpha T
                Cr[p] = fma2(ncr, nw, Cr[p]);
                Cg[p] = fma2(ncg, nw, Cg[p]);
                Cb[p] = fma2(ncb, nw, Cb[p]);
                T[p] = mul2(T[p], add2(one, na));
                if (kCount) {
                    if (on[p].x != 0.f && keep.x == 0.f) stop[2 * p] = pos;
                    if (on[p].y != 0.f && keep.y == 0.f) stop[2 * p + 1] = pos;
                }
                on[p] = mul2(on[p], keep);
                last[2 * p] = na.x != 0.f ? pos : last[2 * p];
                last[2 * p + 1] = na.y != 0.f ? pos : last[2 * p + 1];
                if (kCount) c_work += int(na.x != 0.f) + int(na.y != 0.f);
            }
        }
        __syncwarp();
        if (finished) break;
    }
    cp_async_wait_all();
    if (kCount) {
        int visited = 0;
#pragma unroll
        for (int i = 0; i < kPx; ++i)
            if (x < a.W && y0 + i < a.H) visited += stop[i] ? stop[i] : n;
        add_counts(a.counts, c_eval, c_work, c_staged, lane, 32 * kPx, visited);
    }
    double l1 = 0.0;  // kL1: this lane's sum of |image - target|
    if (x < a.W) {
#pragma unroll
        for (int i = 0; i < kPx; ++i) {
            if (y0 + i < a.H) {
                const int64_t pix = int64_t(y0 + i) * a.W + x;
                const float Ti = i & 1 ? T[i / 2].y : T[i / 2].x;
                const float im[3] = {__fmaf_rn(Ti, a.bg0, i & 1 ? Cr[i / 2].y : Cr[i / 2].x),
                                     __fmaf_rn(Ti, a.bg1, i & 1 ? Cg[i / 2].y : Cg[i / 2].x),
                                     __fmaf_rn(Ti, a.bg2, i & 1 ? Cb[i / 2].y : Cb[i / 2].x)};
#pragma unroll
                for (int c = 0; c < 3; ++c) a.image[3 * pix + c] = im[c];
                a.final_T[pix] = Ti;
                a.n_contrib[pix] = last[i];
                if (kL1) {
#pragma unroll
                    for (int c = 0; c < 3; ++c) {
                        const float tg = __ldg(a.target + 3 * pix + c);
                        const float d = im[c] - tg;
                        l1 += fabs(double(im[c]) - double(tg));
                        a.dL_dimage[3 * pix + c] = d > 0.f ? a.inv_count : (d < 0.f ? -a.inv_count : 0.f);
                    }
                }
            }
        }
    }
    if (kL1) {
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) l1 += __shfl_xor_sync(kFull, l1, o);
        if (lane == 0) atomicAdd(a.loss, l1 * a.inv_count_d);
    }
}

struct BwdArgs {
    const float2* xy;
    const float4* con;
    const float4* rgb;
    const uint32_t* vals;
    const uint2* ranges;
    const uint32_t* order;  // tile processing order (nullable)
    int W, H, TX, tiles;
    float bg0, bg1, bg2;
    const float* final_T;
    const int32_t* n_contrib;
    const float* dL_dimage;
    float2* g_xy;
    float4* g_con;
    float4* g_rgb;
    float2* g_xy_abs;  // absgrad: sums of |per-pixel dL/du|, |per-pixel dL/dv| (kAbs only)
    unsigned long long* counts;  // kCount only: work counters (gs_raster_bwd_counted)
};

// The reverse pass's per-entry sums, taken in batches: each lane stashes its
// kVals partial moments of an entry in shared memory (slot s, column
// lane ^ swz(s)), and once kSlots entries are stashed the warp sums them
// transposed: lanes s * kL .. s * kL + kL - 1 (kL = 32 / kSlots) each add kSlots
// of the slot's 32 columns with float4 loads, two shuffle-add levels (kSlots = 8)
// finish the sums, and the first of them turns the slot's moments into the
// Gaussian's gradients (with the entry's conic, read from the batch's staging)
// and adds them with one vector atomic per record.  The slots are emptied at the
// end of every batch, while its staged entries are still in place.  Per entry that costs kVals shared stores
// and about two loads a value, against a five-level shuffle reduce-scatter, and
// the conic algebra runs once per entry instead of in every lane.
// swz(s) = 4 (s & 1) keeps the float4 loads of the two slots a wavefront serves
// on different banks.
//
// The moments, per lane (sums over its pixels of q = dL/dsigma times): X = dx s0
// (or, for an entry evaluated in the factored form, sum q t), s1 = sum q dy,
// dx^2 s0, dx s1, sum q dy^2, s0 = sum q, and the colour sums; with them
// dL/du = A X + B s1 (factored: A X), dL/dv = B X + C s1 (factored: B X + D s1),
// dL/dA = dx^2 s0 / 2, dL/dB = dx s1, dL/dC = sum q dy^2 / 2, dL/do = -s0 / o.
template <int kSlots, int kVals>
struct EntrySums {
    static constexpr int kL = 32 / kSlots;  // lanes that sum one slot
    float v[kVals][kSlots * 32];
    int e[kSlots];  // the slot's entry: its index among the batch's compacted entries
};

template <int kSlots, int kVals>
__device__ __forceinline__ void stash_entry(EntrySums<kSlots, kVals>& R, int slot, int lane, int e,
                                            const float (&v)[kVals]) {
    const int col = slot * 32 + (lane ^ (4 * (slot & 1)));
#pragma unroll
    for (int q = 0; q < kVals; ++q) R.v[q][col] = v[q];
    if (lane == 0) R.e[slot] = e;
}

template <int kSlots, int kVals>
__device__ __forceinline__ void flush_entries(const EntrySums<kSlots, kVals>& R, const WarpStage& S, int buf,
                                              int count, int lane, const BwdArgs& a) {
    constexpr int kL = EntrySums<kSlots, kVals>::kL;
    const int sl = lane / kL, part = lane % kL;
    const int swz = 4 * (sl & 1);
    float sum[kVals];
#pragma unroll
    for (int q = 0; q < kVals; ++q) {
        float acc = 0.f;
#pragma unroll
        for (int g = 0; g < kSlots / 4; ++g) {
            const float4 f =
                *reinterpret_cast<const float4*>(&R.v[q][sl * 32 + ((part * kSlots + 4 * g) ^ swz)]);
            acc += (f.x + f.y) + (f.z + f.w);
        }
        sum[q] = acc;
    }
#pragma unroll
    for (int o = 1; o < kL; o <<= 1)
#pragma unroll
        for (int q = 0; q < kVals; ++q) sum[q] += __shfl_xor_sync(kFull, sum[q], o);
    if (part == 0 && sl < count) {
        const int e = R.e[sl];
        const int j = S.idx[e] & (kBatch - 1);
        const uint32_t gid = S.gid[buf][j];
        const float4 con = S.con[buf][j];
        const float4 pb = S.pb[e];
        // plain: dL/du = A X + B s1, dL/dv = B X + C s1; factored: A X, B X + D s1
        const bool factored = pb.w >= kFactored;
        const float du = fmaf(con.x, sum[0], factored ? 0.f : con.y * sum[1]);
        const float dv = fmaf(con.y, sum[0], (factored ? pb.z : con.z) * sum[1]);
        atomicAdd(a.g_xy + gid, make_float2(du, dv));
        atomicAdd(a.g_con + gid, make_float4(0.5f * sum[2], sum[3], 0.5f * sum[4], -sum[5] * S.pa[e].w));
        atomicAdd(a.g_rgb + gid, make_float4(-sum[6], -sum[7], -sum[8], 0.f));
        if (kVals > 9) atomicAdd(a.g_xy_abs + gid, make_float2(sum[9], sum[kVals > 9 ? 10 : 0]));
    }
}

// kBg: the background is not black.  With a black one (every workload here) the
// background term of dL/dalpha is 0 and neither it nor its per-pixel factor is
// formed, which saves a paired instruction per pixel pair and eight registers.
template <int PX, bool kAbs, bool kCount, bool kBg>
__global__ void __launch_bounds__(kWarps * 32, Layout<PX>::kBwdMinBlocks) raster_bwd_kernel(const BwdArgs a) {
    constexpr int kPx = PX, kPairs = Layout<PX>::kPairs, kBoxH = Layout<PX>::kBoxH, kSub = Layout<PX>::kSub;
    // entries summed per batch: 8 with one warp per tile, 4 with two (whose 20 blocks
    // an SM the larger stash would not let fit in shared memory)
    constexpr int kSlots = PX == 8 ? 8 : 4;
    constexpr int kVals = kAbs ? 11 : 9;
    __shared__ WarpStage stage[kWarps];
    __shared__ __align__(16) EntrySums<kSlots, kVals> sums[kWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gw = blockIdx.x * kWarps + warp;
    const int slot = gw / kSub, sub = gw % kSub;
    if (slot >= a.tiles) return;
    const int tile = a.order ? int(__ldg(a.order + slot)) : slot;  // longest lists first when ordered
    WarpStage& S = stage[warp];
    EntrySums<kSlots, kVals>& R = sums[warp];
    int stashed = 0;  // entries in R not yet added (the same in every lane)
    const int xb = (tile % a.TX) * kTile;  // this warp's pixel box
    const int yb = (tile / a.TX) * kTile + sub * kBoxH;
    const int x = xb + lane % kBoxW;
    const int y0 = yb + (lane / kBoxW) * kPx;
    const float px = float(x) + 0.5f;
    const float bx0 = float(xb) + 0.5f, by0 = float(yb) + 0.5f;  // box corner (pixel centre)
    const uint2 range = a.ranges[tile];

    // per pixel pair: transmittance, minus g . S (S the colour blended behind),
    // dL/dimage, -final_T (bg . g)
    f2 nyc[kPairs], T[kPairs], nP[kPairs], gr[kPairs], gg[kPairs], gb[kPairs], ngb[kBg ? kPairs : 1];
    int last[kPx];
    int lmax = 0;
#pragma unroll
    for (int i = 0; i < kPx; ++i) {
        float Ti = 1.f, r = 0.f, g = 0.f, bb = 0.f;
        last[i] = 0;
        if (x < a.W && y0 + i < a.H) {
            const int64_t pix = int64_t(y0 + i) * a.W + x;
            Ti = a.final_T[pix];
            last[i] = a.n_contrib[pix];
            r = a.dL_dimage[3 * pix + 0];
            g = a.dL_dimage[3 * pix + 1];
            bb = a.dL_dimage[3 * pix + 2];
        }
        const float nb = -Ti * (a.bg0 * r + a.bg1 * g + a.bg2 * bb);
        const float ny = -(float(y0 + i) + 0.5f);
        if (i & 1) {
            T[i / 2].y = Ti; gr[i / 2].y = r; gg[i / 2].y = g; gb[i / 2].y = bb; nyc[i / 2].y = ny;
            if (kBg) ngb[i / 2].y = nb;
        } else {
            T[i / 2].x = Ti; gr[i / 2].x = r; gg[i / 2].x = g; gb[i / 2].x = bb; nyc[i / 2].x = ny;
            if (kBg) ngb[i / 2].x = nb;
        }
        lmax = max(lmax, last[i]);
    }
#pragma unroll
    for (int p = 0; p < kPairs; ++p) nP[p] = splat(0.f);
    const f2 one = splat(1.f), zero = splat(0.f);
    // entries past every pixel's last are never needed; never read past the list
    const int total = min(__reduce_max_sync(kFull, lmax), int(range.y - range.x));
    const int nb = (total + kBatch - 1) / kBatch;
    int c_eval = 0, c_work = 0, c_staged = 0;  // kCount only
    if (total > 0) {
        const int c0 = min(total, kBatch);
        gather<true>(S, 0, a.vals, a.xy, a.con, a.rgb, range.x + uint32_t(total - c0), c0, lane);
    }
    for (int b = 0; b < nb; ++b) {
        const int buf = b & 1;
        const int hi = total - b * kBatch;  // this batch covers positions [hi - cnt, hi)
        const int cnt = min(hi, kBatch);
        cp_async_wait_all();
        __syncwarp();
        if (b + 1 < nb) {
            const int nhi = hi - kBatch, ncnt = min(nhi, kBatch);
            gather<true>(S, buf ^ 1, a.vals, a.xy, a.con, a.rgb, range.x + uint32_t(nhi - ncnt), ncnt, lane);
        }
        const int live = prep<false, PX>(S, buf, cnt, lane, bx0, by0);
        __syncwarp();
        if (kCount) {
            c_staged += cnt;
            c_eval += live;
        }
        for (int e = 0; e < live; ++e) {  // the batch's entries that reach this warp's box
            const int ij = S.idx[e];
            const int j = ij & (kBatch - 1);
            const int pos = hi - 1 - j;  // 0-based list position of this entry
            const float4 pa = S.pa[e], pb = S.pb[e];
            const float4 con = S.con[buf][j];
            const float4 c = S.rgb[buf][j];
            // the entry at the lane's pixels; kMC: its alpha can reach the 0.99 clamp,
            // whose gate then multiplies dL/dsigma (else the gate is 1 and not formed)
            const auto entry = [&](auto may_clamp) {
                constexpr bool kMC = decltype(may_clamp)::value;
                Alpha<PX> r;
                eval_alpha<true, kMC, PX>(pa, pb, S.pc[e], con, px, nyc, r);
                const f2 cr = splat(c.x), cg = splat(c.y), cb = splat(c.z);
                f2 ndr = zero, ndg = zero, ndb = zero, nmo = zero, s1 = zero, s2 = zero, nm[kPairs];
                // branch-free: every pixel runs the same instructions, inactive ones
                // with alpha 0, so T, P and every sum stay unchanged
#pragma unroll
                for (int p = 0; p < kPairs; ++p) {
                    // -alpha, 0 where the pixel does not blend the entry or has not reached it
                    const f2 nae = make_float2(pos < last[2 * p] ? r.nal[p].x : 0.f,
                                               pos < last[2 * p + 1] ? r.nal[p].y : 0.f);
                    if (kCount) c_work += int(nae.x != 0.f) + int(nae.y != 0.f);
                    const f2 om = add2(one, nae);                                                  // 1 - alpha
                    const f2 rom = make_float2(rcp_approx(om.x), rcp_approx(om.y));
                    T[p] = mul2(T[p], rom);  // transmittance in front of this entry
                    const f2 nw = mul2(nae, T[p]);
                    ndr = fma2(nw, gr[p], ndr);
                    ndg = fma2(nw, gg[p], ndg);
                    ndb = fma2(nw, gb[p], ndb);
                    // only g . S enters the gradient: P = g . S with S <- c alpha + (1 - alpha) S
                    const f2 xg = add2(fma2(gr[p], cr, fma2(gg[p], cg, mul2(gb[p], cb))), nP[p]);  // g . c - P
                    const f2 dLda = kBg ? fma2(T[p], xg, mul2(ngb[p], rom)) : mul2(T[p], xg);
                    nP[p] = fma2(nae, xg, nP[p]);
                    // -dL/dalpha alpha = dL/dsigma, zero where alpha was clamped (times a 0/1 gate)
                    f2 q = mul2(dLda, nae);
                    if (kMC) q = mul2(q, r.gate[p]);
                    nm[p] = q;
                    nmo = add2(nmo, q);
                    s1 = fma2(q, r.dy[p], s1);
                    s2 = fma2(mul2(q, r.dy[p]), r.dy[p], s2);
                }
                // no vote on whether any pixel took the entry: 9 in 10 entries that reach
                // the box take a gradient somewhere in it, and the test costs more than the
                // reductions of zeros it would save
                const float s0 = nmo.x + nmo.y, m1 = s1.x + s1.y;
                const float dxs0 = r.dx * s0;
                float X;  // dx s0, or sum q t in the factored form
                float au = 0.f, av = 0.f;  // absgrad: sums of |per-pixel dL/du|, |per-pixel dL/dv|
                if (pb.w >= kFactored) {
                    // dsigma/du = A t, dsigma/dv = B t + D dy
                    f2 st = zero;
#pragma unroll
                    for (int p = 0; p < kPairs; ++p) st = fma2(nm[p], r.t[p], st);
                    X = st.x + st.y;
                    if (kAbs) {
#pragma unroll
                        for (int p = 0; p < kPairs; ++p) {
                            const f2 pu = mul2(nm[p], mul2(splat(con.x), r.t[p]));
                            const f2 pv = mul2(nm[p], fma2(splat(con.y), r.t[p], mul2(splat(pb.z), r.dy[p])));
                            au += fabsf(pu.x) + fabsf(pu.y);
                            av += fabsf(pv.x) + fabsf(pv.y);
                        }
                    }
                } else {
                    X = dxs0;
                    if (kAbs) {
                        // per pixel dsigma/du = A dx + B dy, dsigma/dv = B dx + C dy
                        const f2 adx = splat(con.x * r.dx), bdx = splat(con.y * r.dx);
#pragma unroll
                        for (int p = 0; p < kPairs; ++p) {
                            const f2 pu = mul2(nm[p], fma2(splat(con.y), r.dy[p], adx));
                            const f2 pv = mul2(nm[p], fma2(splat(con.z), r.dy[p], bdx));
                            au += fabsf(pu.x) + fabsf(pu.y);
                            av += fabsf(pv.x) + fabsf(pv.y);
                        }
                    }
                }
                float v[kVals];
                v[0] = X;
                v[1] = m1;
                v[2] = r.dx * dxs0;
                v[3] = r.dx * m1;
                v[4] = s2.x + s2.y;
                v[5] = s0;
                v[6] = ndr.x + ndr.y;
                v[7] = ndg.x + ndg.y;
                v[8] = ndb.x + ndb.y;
                if (kAbs) {
                    v[kAbs ? 9 : 0] = au;
                    v[kAbs ? 10 : 0] = av;
                }
                stash_entry(R, stashed, lane, e, v);
                if (++stashed == kSlots) {
                    __syncwarp();
                    flush_entries(R, S, buf, kSlots, lane, a);
                    __syncwarp();
                    stashed = 0;
                }
            };
            if (ij & kMayClampBit)
                entry(std::true_type{});
            else
                entry(std::false_type{});
        }
        if (stashed) {  // the batch's last entries, while its staging is in place
            __syncwarp();
            flush_entries(R, S, buf, stashed, lane, a);
            stashed = 0;
        }
        __syncwarp();
    }
    cp_async_wait_all();
    if (kCount) add_counts(a.counts, c_eval, c_work, c_staged, lane, 32 * kPx);
}

// Tiles ordered by decreasing list length (bucketed by floor(sqrt(length)),
// 256 buckets; order inside a bucket unspecified), so that the longest tiles
// start first and the kernel's tail holds short ones.  One CTA per view.
struct TileOrderArgs {
    const uint2* ranges[GS_MAX_VIEWS];
    uint32_t* order[GS_MAX_VIEWS];
    int tiles;
};

__global__ void __launch_bounds__(1024) tile_order_kernel(const __grid_constant__ TileOrderArgs a) {
    __shared__ uint32_t count[256];
    __shared__ uint32_t start[256];
    const uint2* ranges = a.ranges[blockIdx.x];
    uint32_t* order = a.order[blockIdx.x];
    for (int b = threadIdx.x; b < 256; b += blockDim.x) count[b] = 0u;
    __syncthreads();
    auto bucket = [&](int t) {
        const uint2 r = __ldg(ranges + t);
        const float len = float(r.y - r.x);
        return 255u - min(255u, uint32_t(sqrtf(len)));  // longest first
    };
    for (int t = threadIdx.x; t < a.tiles; t += blockDim.x) atomicAdd(&count[bucket(t)], 1u);
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t run = 0;
        for (int b = 0; b < 256; ++b) {
            start[b] = run;
            run += count[b];
        }
    }
    __syncthreads();
    for (int t = threadIdx.x; t < a.tiles; t += blockDim.x) order[atomicAdd(&start[bucket(t)], 1u)] = uint32_t(t);
}

}  // namespace

cudaError_t launch_tile_order_views(int views, const uint32_t* const* ranges, int tiles, uint32_t* const* order,
                                    cudaStream_t s) {
    if (tiles <= 0 || views <= 0) return cudaSuccess;
    TileOrderArgs a;
    for (int v = 0; v < views; ++v) {
        a.ranges[v] = reinterpret_cast<const uint2*>(ranges[v]);
        a.order[v] = order[v];
    }
    a.tiles = tiles;
    tile_order_kernel<<<unsigned(views), 1024, 0, s>>>(a);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_tile_order(const uint32_t* ranges, int tiles, uint32_t* order, cudaStream_t s) {
    return launch_tile_order_views(1, &ranges, tiles, &order, s);
}

cudaError_t launch_raster_fwd(const gs_projected& proj, const uint32_t* vals, const uint32_t* ranges,
                              const uint32_t* order, const CamArgs& cam, const float bg[3], float* image,
                              float* final_T, int32_t* n_contrib, cudaStream_t s, unsigned long long* counts,
                              const L1Out* l1) {
    FwdArgs a;
    a.xy = reinterpret_cast<const float2*>(proj.xy);
    a.con = reinterpret_cast<const float4*>(proj.conic_opacity);
    a.rgb = reinterpret_cast<const float4*>(proj.rgb);
    a.vals = vals;
    a.ranges = reinterpret_cast<const uint2*>(ranges);
    a.order = order;
    a.W = cam.W;
    a.H = cam.H;
    a.TX = cam.TX;
    a.tiles = cam.TX * cam.TY;
    a.bg0 = bg[0];
    a.bg1 = bg[1];
    a.bg2 = bg[2];
    a.image = image;
    a.final_T = final_T;
    a.n_contrib = n_contrib;
    a.counts = counts;
    a.target = l1 ? l1->target : nullptr;
    a.dL_dimage = l1 ? l1->dL_dimage : nullptr;
    a.loss = l1 ? l1->loss : nullptr;
    const int64_t count = int64_t(3) * cam.W * cam.H;
    a.inv_count = float(1.0 / double(count));
    a.inv_count_d = 1.0 / double(count);
    if (a.tiles >= kWideLayoutTilesFwd) {
        const unsigned grid = unsigned(a.tiles * Layout<8>::kSub);
        if (counts)
            raster_fwd_kernel<8, true, false><<<grid, kWarps * 32, 0, s>>>(a);
        else if (l1)
            raster_fwd_kernel<8, false, true><<<grid, kWarps * 32, 0, s>>>(a);
        else
            raster_fwd_kernel<8, false, false><<<grid, kWarps * 32, 0, s>>>(a);
    } else {
        constexpr int P = GS_FWD_PX;
        const unsigned grid = unsigned(a.tiles * Layout<P>::kSub);
        if (counts)
            raster_fwd_kernel<P, true, false><<<grid, kWarps * 32, 0, s>>>(a);
        else if (l1)
            raster_fwd_kernel<P, false, true><<<grid, kWarps * 32, 0, s>>>(a);
        else
            raster_fwd_kernel<P, false, false><<<grid, kWarps * 32, 0, s>>>(a);
    }
    count_launches(1);
    return cudaGetLastError();
}

namespace {
template <int PX, bool kBg>
void launch_raster_bwd_bg(const BwdArgs& a, bool counted, cudaStream_t s) {
    // the reverse pass keeps its entry sums in shared memory: ask for the largest
    // shared-memory carveout, so that its blocks an SM are set by registers alone
    static const bool carveout = [] {
        const int c = cudaSharedmemCarveoutMaxShared;
        const cudaFuncAttribute at = cudaFuncAttributePreferredSharedMemoryCarveout;
        bool ok = cudaFuncSetAttribute(raster_bwd_kernel<PX, false, false, kBg>, at, c) == cudaSuccess;
        ok = cudaFuncSetAttribute(raster_bwd_kernel<PX, true, false, kBg>, at, c) == cudaSuccess && ok;
        ok = cudaFuncSetAttribute(raster_bwd_kernel<PX, false, true, kBg>, at, c) == cudaSuccess && ok;
        ok = cudaFuncSetAttribute(raster_bwd_kernel<PX, true, true, kBg>, at, c) == cudaSuccess && ok;
        if (!ok) cudaGetLastError();  // a hint only: a refusal leaves the default carveout
        return ok;
    }();
    (void)carveout;
    const unsigned grid = unsigned(a.tiles * Layout<PX>::kSub);
    if (counted) {
        if (a.g_xy_abs)
            raster_bwd_kernel<PX, true, true, kBg><<<grid, kWarps * 32, 0, s>>>(a);
        else
            raster_bwd_kernel<PX, false, true, kBg><<<grid, kWarps * 32, 0, s>>>(a);
    } else if (a.g_xy_abs) {
        raster_bwd_kernel<PX, true, false, kBg><<<grid, kWarps * 32, 0, s>>>(a);
    } else {
        raster_bwd_kernel<PX, false, false, kBg><<<grid, kWarps * 32, 0, s>>>(a);
    }
}

template <int PX>
void launch_raster_bwd_layout(const BwdArgs& a, bool counted, cudaStream_t s) {
    if (a.bg0 != 0.f || a.bg1 != 0.f || a.bg2 != 0.f)
        launch_raster_bwd_bg<PX, true>(a, counted, s);
    else
        launch_raster_bwd_bg<PX, false>(a, counted, s);
}
}  // namespace

cudaError_t launch_raster_bwd(const gs_projected& proj, const uint32_t* vals, const uint32_t* ranges,
                              const uint32_t* order, const CamArgs& cam, const float bg[3], const float* final_T,
                              const int32_t* n_contrib, const float* dL_dimage, const gs_grad2d& g2,
                              cudaStream_t s, unsigned long long* counts) {
    BwdArgs a;
    a.xy = reinterpret_cast<const float2*>(proj.xy);
    a.con = reinterpret_cast<const float4*>(proj.conic_opacity);
    a.rgb = reinterpret_cast<const float4*>(proj.rgb);
    a.vals = vals;
    a.ranges = reinterpret_cast<const uint2*>(ranges);
    a.order = order;
    a.W = cam.W;
    a.H = cam.H;
    a.TX = cam.TX;
    a.tiles = cam.TX * cam.TY;
    a.bg0 = bg[0];
    a.bg1 = bg[1];
    a.bg2 = bg[2];
    a.final_T = final_T;
    a.n_contrib = n_contrib;
    a.dL_dimage = dL_dimage;
    a.g_xy = reinterpret_cast<float2*>(g2.xy);
    a.g_con = reinterpret_cast<float4*>(g2.conic_opacity);
    a.g_rgb = reinterpret_cast<float4*>(g2.rgb);
    a.g_xy_abs = reinterpret_cast<float2*>(g2.xy_abs);
    a.counts = counts;
    if (a.tiles >= kWideLayoutTiles)
        launch_raster_bwd_layout<8>(a, counts != nullptr, s);
    else
        launch_raster_bwd_layout<4>(a, counts != nullptr, s);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace gsk
