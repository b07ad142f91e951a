// gs_raster_fwd / gs_raster_bwd: stage 3 of the pipeline, differentiable
// front-to-back alpha blending per 16x16 tile (gsplat guide, lmnt.cn/news/262699
// §2.1: shared-memory prefetch of the tile's Gaussians, SoA features, warp-level
// synchronisation; §2.2: a standalone backward entry).
//
// Work decomposition: one warp per tile, each lane owns a column of 8 pixels
// (lane & 15 selects the column, lane >> 4 the upper or lower half), four tiles
// per block.  The warp walks its tile's sorted list in batches of 32 entries:
// every lane gathers one entry's 40 bytes (xy, conic + opacity, colour) by
// Gaussian index into shared memory with cp.async, double-buffered so the next
// batch is in flight while the current one is composited; the lane that
// gathered an entry also derives its per-entry constants.  Every lane then
// reads each entry once (broadcast loads) and applies it to its 8 pixels, whose
// terms that depend only on dx are shared.  No block-wide barrier is used:
// warps synchronise with __syncwarp and finish independently.
//
// Forward: a warp stops as soon as all 256 pixels have terminated (warp vote
// per entry).  Backward: back to front from the largest n_contrib of the tile;
// each lane sums its 8 pixels' contributions, the 9 per-Gaussian sums are
// reduce-scattered across the warp (18 shuffles) and three lanes issue one
// float2 / float4 atomic add each (batched atomics, MUSA co-design article
// qwbw.cn/news/278220 §2.2).  The gradient with respect to (u, v, A, B, C) is
// accumulated as three moments of dL/dsigma over the lane's pixels, then
// combined with dx and the conic once per entry.
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

#ifndef GS_RASTER_PX
#define GS_RASTER_PX 4
#endif
#ifndef GS_RASTER_BOXW
#define GS_RASTER_BOXW 16
#endif
constexpr int kPx = GS_RASTER_PX;        // pixels per lane (a column segment)
constexpr int kBoxW = GS_RASTER_BOXW;    // width of a warp's pixel box (16 or 8)
constexpr int kLaneRows = 32 / kBoxW;    // lanes stacked vertically in the box
constexpr int kBoxH = kLaneRows * kPx;   // height of a warp's pixel box
constexpr int kSubX = kTile / kBoxW, kSubY = kTile / kBoxH;
constexpr int kSub = kSubX * kSubY;      // warps per tile
constexpr int kWarps = 4;                // warps per block
static_assert(kTile % kBoxW == 0 && kTile % kBoxH == 0, "warp boxes tile the 16x16 tile");
// resident blocks per SM the register allocation is sized for (launch bounds)
#ifndef GS_RASTER_FWD_MIN_BLOCKS
#define GS_RASTER_FWD_MIN_BLOCKS 6
#endif
#ifndef GS_RASTER_BWD_MIN_BLOCKS
#define GS_RASTER_BWD_MIN_BLOCKS 5
#endif
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
constexpr float kPlain = 0.f;     // expanded quadratic form in float32
constexpr float kDouble = 1.f;    // quadratic form in double (a conic that is not positive definite)
constexpr float kSkip = 2.f;      // misses every pixel of the warp's box
constexpr float kFactored = 3.f;  // factored form 1/2 A t^2 + 1/2 D dy^2 in float32

struct WarpStage {
    float2 xy[2][kBatch];
    float4 con[2][kBatch];  // A, B, C, o
    float4 rgb[2][kBatch];
    uint32_t gid[2][kBatch];
    float4 pa[kBatch];  // u, v, log2(o), 1/o
    float4 pb[kBatch];  // plain: -log2e A/2, -log2e B, -log2e C/2; factored: B/A (high, low part), D; flag
    float2 pc[kBatch];  // factored: -log2e A/2, -log2e D/2
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
// evaluation (kPlain, kFactored, kDouble) or kSkip: the smallest sigma over
// this warp's pixel box [bx0, bx0 + kBoxW - 1] x [by0, by0 + kBoxH - 1] (pixel
// centres) puts alpha below 1/255 everywhere in it, with a margin far above
// the rounding of either evaluation, so no pixel of the warp would blend it.
// The bound is computed in float32 for well-conditioned conics and in double
// for the others.
__device__ __forceinline__ void prep(WarpStage& S, int buf, int count, int lane, float bx0, float by0) {
    if (lane < count) {
        const float2 xy = S.xy[buf][lane];
        const float4 c = S.con[buf][lane];
        const float tr = __fadd_rn(c.x, c.z);
        const float det = __fsub_rn(__fmul_rn(c.x, c.z), __fmul_rn(c.y, c.y));
        const bool ill = !(det > 0.f) || (__fmul_rn(tr, tr) > __fmul_rn(kCondMaxTraceSqOverDet, det));
        const float lo = log2f(c.w);
        // alpha >= 1/255 needs sigma <= ln(255 o) = ln 255 + lo ln 2
        const float cut = 5.541263545158426f + lo * 0.6931471805599453f;
        const float bx1 = bx0 + float(kBoxW - 1), by1 = by0 + float(kBoxH - 1);
        float4 pb;
        float2 pc = make_float2(0.f, 0.f);
        if (!ill) {
            const float smin = box_min<float>(c.x, c.y, c.z, xy.x, xy.y, bx0, bx1, by0, by1);
            const float flag = smin * (1.f - 1e-4f) > cut + 1e-4f ? kSkip : kPlain;
            pb = make_float4(__fmul_rn(-0.5f * kLog2e, c.x), __fmul_rn(-kLog2e, c.y), __fmul_rn(-0.5f * kLog2e, c.z),
                             flag);
        } else {
            const double A = c.x, B = c.y, C = c.z;
            const double D = (A * C - B * B) / A;  // A C and B^2 are exact in double
            if (A > 0.0 && D > 0.0) {
                const double smin = box_min<double>(A, B, C, xy.x, xy.y, bx0, bx1, by0, by1);
                const double r = B / A;
                const float rh = __double2float_rn(r);
                pb = make_float4(rh, __double2float_rn(r - double(rh)), float(D),
                                 smin * (1.0 - 1e-4) > double(cut) + 1e-4 ? kSkip : kFactored);
                pc = make_float2(__double2float_rn(-0.5 * kLog2eD * A), __double2float_rn(-0.5 * kLog2eD * D));
            } else {
                pb = make_float4(0.f, 0.f, 0.f, kDouble);
            }
        }
        S.pa[lane] = make_float4(xy.x, xy.y, lo, 1.f / c.w);
        S.pb[lane] = pb;
        S.pc[lane] = pc;
    }
}

// alpha of one entry at the lane's pixels, and the offsets dx (shared) and
// dy[i] of the mean from the pixel centres (t[i] = dx + (B/A) dy[i] for a
// factored entry).  Bit i of `blend` is set when pixel i passes sigma >= 0 and
// alpha >= 1/255; bit i of `clamp` when alpha was clamped at 0.99.
__device__ __forceinline__ void eval_alpha(const float4& pa, const float4& pb, const float2& pc, const float4& con,
                                           float px, int y0, float (&alpha)[kPx], unsigned& blend, unsigned& clamp,
                                           float& dx, float (&dy)[kPx], float (&t)[kPx]) {
    blend = 0u;
    clamp = 0u;
    if (pb.w == kFactored) {
        dx = __fsub_rn(pa.x, px);
#pragma unroll
        for (int i = 0; i < kPx; ++i) {
            dy[i] = __fsub_rn(pa.y, __fadd_rn(float(y0 + i), 0.5f));
            t[i] = __fmaf_rn(pb.y, dy[i], __fmaf_rn(pb.x, dy[i], dx));
            const float s = __fmaf_rn(__fmul_rn(pc.x, t[i]), t[i], __fmul_rn(__fmul_rn(pc.y, dy[i]), dy[i]));
            const float a = ex2_approx(__fadd_rn(s, pa.z));
            const bool c = a > kAlphaMax;
            alpha[i] = c ? kAlphaMax : a;
            if (alpha[i] >= kAlphaMin) blend |= 1u << i;  // s <= 0 by construction
            if (c) clamp |= 1u << i;
        }
    } else if (pb.w == kDouble) {
        const double dxd = __dsub_rn(double(pa.x), double(px));
        dx = __double2float_rn(dxd);
        const double A = con.x, B = con.y, C = con.z;
        const double adx2 = __dmul_rn(__dmul_rn(A, dxd), dxd);
        const double bdx = __dmul_rn(B, dxd);
#pragma unroll
        for (int i = 0; i < kPx; ++i) {
            const double dyd = __dsub_rn(double(pa.y), double(y0 + i) + 0.5);
            const double sig = __dadd_rn(__dmul_rn(0.5, __dadd_rn(adx2, __dmul_rn(__dmul_rn(C, dyd), dyd))),
                                         __dmul_rn(bdx, dyd));
            const float s = __double2float_rn(__dmul_rn(-sig, kLog2eD));
            dy[i] = __double2float_rn(dyd);
            t[i] = 0.f;
            const float a = ex2_approx(__fadd_rn(s, pa.z));
            const bool c = a > kAlphaMax;
            alpha[i] = c ? kAlphaMax : a;
            if (s <= 0.f && alpha[i] >= kAlphaMin) blend |= 1u << i;
            if (c) clamp |= 1u << i;
        }
    } else {
        dx = __fsub_rn(pa.x, px);
        const float a0 = __fmul_rn(__fmul_rn(pb.x, dx), dx);
        const float c1 = __fmul_rn(pb.y, dx);
#pragma unroll
        for (int i = 0; i < kPx; ++i) {
            dy[i] = __fsub_rn(pa.y, __fadd_rn(float(y0 + i), 0.5f));
            t[i] = 0.f;
            const float s = __fmaf_rn(dy[i], __fmaf_rn(pb.z, dy[i], c1), a0);
            const float a = ex2_approx(__fadd_rn(s, pa.z));
            const bool c = a > kAlphaMax;
            alpha[i] = c ? kAlphaMax : a;
            if (s <= 0.f && alpha[i] >= kAlphaMin) blend |= 1u << i;
            if (c) clamp |= 1u << i;
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
};

__global__ void __launch_bounds__(kWarps * 32, GS_RASTER_FWD_MIN_BLOCKS) raster_fwd_kernel(const FwdArgs a) {
    __shared__ WarpStage stage[kWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gw = blockIdx.x * kWarps + warp;
    const int slot = gw / kSub, sub = gw % kSub;
    if (slot >= a.tiles) return;
    const int tile = a.order ? int(__ldg(a.order + slot)) : slot;  // longest lists first when ordered
    WarpStage& S = stage[warp];
    const int xb = (tile % a.TX) * kTile + (sub % kSubX) * kBoxW;  // this warp's pixel box
    const int yb = (tile / a.TX) * kTile + (sub / kSubX) * kBoxH;
    const int x = xb + lane % kBoxW;
    const int y0 = yb + (lane / kBoxW) * kPx;
    const float px = float(x) + 0.5f;
    const float bx0 = float(xb) + 0.5f, by0 = float(yb) + 0.5f;  // box corner (pixel centre)
    const uint2 range = a.ranges[tile];
    const int n = int(range.y - range.x);

    float T[kPx], Cr[kPx], Cg[kPx], Cb[kPx];
    int last[kPx];
    unsigned done = 0u;
#pragma unroll
    for (int i = 0; i < kPx; ++i) {
        T[i] = 1.f;
        Cr[i] = Cg[i] = Cb[i] = 0.f;
        last[i] = 0;
        if (x >= a.W || y0 + i >= a.H) done |= 1u << i;
    }
    constexpr unsigned kAll = (1u << kPx) - 1u;

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
        prep(S, buf, cnt, lane, bx0, by0);
        __syncwarp();
        bool finished = false;
        for (int j = 0; j < cnt; ++j) {
            if (__all_sync(kFull, done == kAll)) {
                finished = true;
                break;
            }
            const float4 pa = S.pa[j], pb = S.pb[j];
            if (pb.w == kSkip) continue;  // misses every pixel of this warp
            const float4 con = S.con[buf][j];
            const float4 c = S.rgb[buf][j];
            float al[kPx], dy[kPx], tt[kPx], dx;
            unsigned blend, clamp;
            eval_alpha(pa, pb, S.pc[j], con, px, y0, al, blend, clamp, dx, dy, tt);
            blend &= ~done;
            const int pos = b * kBatch + j + 1;
            // branch-free so the 8 independent pixel chains interleave; a pixel
            // that does not take the entry adds c * 0 (exactly nothing)
#pragma unroll
            for (int i = 0; i < kPx; ++i) {
                const bool act = (blend >> i) & 1u;
                const float Tn = __fmul_rn(T[i], __fsub_rn(1.f, al[i]));
                const bool low = Tn < kTMin;
                const bool take = act && !low;
                const float w = take ? __fmul_rn(al[i], T[i]) : 0.f;
                Cr[i] = __fmaf_rn(c.x, w, Cr[i]);
                Cg[i] = __fmaf_rn(c.y, w, Cg[i]);
                Cb[i] = __fmaf_rn(c.z, w, Cb[i]);
                T[i] = take ? Tn : T[i];
                last[i] = take ? pos : last[i];
                done |= (act && low) ? (1u << i) : 0u;
            }
        }
        __syncwarp();
        if (finished) break;
    }
    cp_async_wait_all();
    if (x < a.W) {
#pragma unroll
        for (int i = 0; i < kPx; ++i) {
            if (y0 + i < a.H) {
                const int64_t pix = int64_t(y0 + i) * a.W + x;
                a.image[3 * pix + 0] = __fmaf_rn(T[i], a.bg0, Cr[i]);
                a.image[3 * pix + 1] = __fmaf_rn(T[i], a.bg1, Cg[i]);
                a.image[3 * pix + 2] = __fmaf_rn(T[i], a.bg2, Cb[i]);
                a.final_T[pix] = T[i];
                a.n_contrib[pix] = last[i];
            }
        }
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
};

// Sum 9 per-lane values over the warp and add them to the Gaussian's three
// gradient records with one vector atomic each (lanes 0, 1, 2).
__device__ __forceinline__ void warp_reduce_and_add(float (&v)[8], float v8, int lane, uint32_t gid,
                                                    const BwdArgs& a) {
    // reduce-scatter of 8 values: after it, lanes 4k..4k+3 hold the total of value k
    {
        const bool hi = (lane >> 4) & 1;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const float send = hi ? v[k] : v[k + 4];
            const float keep = hi ? v[k + 4] : v[k];
            v[k] = keep + __shfl_xor_sync(kFull, send, 16);
        }
    }
    {
        const bool hi = (lane >> 3) & 1;
#pragma unroll
        for (int k = 0; k < 2; ++k) {
            const float send = hi ? v[k] : v[k + 2];
            const float keep = hi ? v[k + 2] : v[k];
            v[k] = keep + __shfl_xor_sync(kFull, send, 8);
        }
    }
    {
        const bool hi = (lane >> 2) & 1;
        const float send = hi ? v[0] : v[1];
        const float keep = hi ? v[1] : v[0];
        v[0] = keep + __shfl_xor_sync(kFull, send, 4);
    }
    v[0] += __shfl_xor_sync(kFull, v[0], 2);
    v[0] += __shfl_xor_sync(kFull, v[0], 1);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v8 += __shfl_xor_sync(kFull, v8, o);
    // gather: lane 0 <- values 0,1 (du, dv); lane 1 <- 2..5 (dA, dB, dC, do); lane 2 <- 6,7 (dr, dg) + v8 (db)
    const int i0 = lane == 0 ? 0 : (lane == 1 ? 2 : 6);
    const int i1 = i0 + 1;
    const int i2 = lane == 1 ? 4 : 0;
    const int i3 = lane == 1 ? 5 : 0;
    const float f0 = __shfl_sync(kFull, v[0], 4 * i0);
    const float f1 = __shfl_sync(kFull, v[0], 4 * i1);
    const float f2 = __shfl_sync(kFull, v[0], 4 * i2);
    const float f3 = __shfl_sync(kFull, v[0], 4 * i3);
    if (lane == 0) atomicAdd(a.g_xy + gid, make_float2(f0, f1));
    if (lane == 1) atomicAdd(a.g_con + gid, make_float4(f0, f1, f2, f3));
    if (lane == 2) atomicAdd(a.g_rgb + gid, make_float4(f0, f1, v8, 0.f));
}

__global__ void __launch_bounds__(kWarps * 32, GS_RASTER_BWD_MIN_BLOCKS) raster_bwd_kernel(const BwdArgs a) {
    __shared__ WarpStage stage[kWarps];
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gw = blockIdx.x * kWarps + warp;
    const int slot = gw / kSub, sub = gw % kSub;
    if (slot >= a.tiles) return;
    const int tile = a.order ? int(__ldg(a.order + slot)) : slot;  // longest lists first when ordered
    WarpStage& S = stage[warp];
    const int xb = (tile % a.TX) * kTile + (sub % kSubX) * kBoxW;  // this warp's pixel box
    const int yb = (tile / a.TX) * kTile + (sub / kSubX) * kBoxH;
    const int x = xb + lane % kBoxW;
    const int y0 = yb + (lane / kBoxW) * kPx;
    const float px = float(x) + 0.5f;
    const float bx0 = float(xb) + 0.5f, by0 = float(yb) + 0.5f;  // box corner (pixel centre)
    const uint2 range = a.ranges[tile];

    float T[kPx], P[kPx], gr[kPx], gg[kPx], gb[kPx], ngb[kPx];
    int last[kPx];
    int lmax = 0;
#pragma unroll
    for (int i = 0; i < kPx; ++i) {
        P[i] = 0.f;
        if (x < a.W && y0 + i < a.H) {
            const int64_t pix = int64_t(y0 + i) * a.W + x;
            T[i] = a.final_T[pix];
            last[i] = a.n_contrib[pix];
            gr[i] = a.dL_dimage[3 * pix + 0];
            gg[i] = a.dL_dimage[3 * pix + 1];
            gb[i] = a.dL_dimage[3 * pix + 2];
        } else {
            T[i] = 1.f;
            last[i] = 0;
            gr[i] = gg[i] = gb[i] = 0.f;
        }
        ngb[i] = -T[i] * (a.bg0 * gr[i] + a.bg1 * gg[i] + a.bg2 * gb[i]);
        lmax = max(lmax, last[i]);
    }
    // entries past every pixel's last are never needed; never read past the list
    const int total = min(__reduce_max_sync(kFull, lmax), int(range.y - range.x));
    const int nb = (total + kBatch - 1) / kBatch;
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
        prep(S, buf, cnt, lane, bx0, by0);
        __syncwarp();
        for (int j = 0; j < cnt; ++j) {
            const int pos = hi - 1 - j;  // 0-based list position of this entry
            const float4 pa = S.pa[j], pb = S.pb[j];
            if (pb.w == kSkip) continue;  // misses every pixel of this warp
            const float4 con = S.con[buf][j];
            const float4 c = S.rgb[buf][j];
            float al[kPx], dy[kPx], tt[kPx], m[kPx], dx;
            unsigned blend, clamp;
            eval_alpha(pa, pb, S.pc[j], con, px, y0, al, blend, clamp, dx, dy, tt);
            float dr = 0.f, dg = 0.f, db = 0.f, mo = 0.f, s1 = 0.f, s2 = 0.f, st = 0.f;
            bool any = false;
            // branch-free: every pixel runs the same instructions, inactive ones
            // with zero weight and unchanged state
#pragma unroll
            for (int i = 0; i < kPx; ++i) {
                const bool act = ((blend >> i) & 1u) && pos < last[i];
                any = any || act;
                // an inactive pixel runs the same instructions with alpha 0: T, S and
                // every sum stay unchanged
                const float ae = act ? al[i] : 0.f;
                const float rom = rcp_approx(__fsub_rn(1.f, ae));
                T[i] = T[i] * rom;  // transmittance in front of this entry
                const float w = ae * T[i];
                dr = fmaf(w, gr[i], dr);
                dg = fmaf(w, gg[i], dg);
                db = fmaf(w, gb[i], db);
                // only g . S enters the gradient: P = g . S with S <- c alpha + (1 - alpha) S
                const float x = fmaf(gr[i], c.x, fmaf(gg[i], c.y, gb[i] * c.z)) - P[i];
                const float dLda = fmaf(T[i], x, ngb[i] * rom);
                P[i] = fmaf(ae, x, P[i]);
                m[i] = ((clamp >> i) & 1u) ? 0.f : dLda * ae;  // dL/dsigma = -m, dL/do = m / o
                mo += m[i];
                s1 = fmaf(-m[i], dy[i], s1);
                s2 = fmaf(-m[i] * dy[i], dy[i], s2);
                st = fmaf(-m[i], tt[i], st);  // factored entries only (tt = 0 otherwise)
            }
            const float s0 = -mo;
            if (__any_sync(kFull, any)) {
                float du, dv;
                if (pb.w == kFactored) {
                    // dsigma/du = A t, dsigma/dv = B t + D dy
                    du = con.x * st;
                    dv = fmaf(con.y, st, pb.z * s1);
                } else if (pb.w == kDouble) {
                    // not positive definite: dsigma/du = A dx + B dy, dsigma/dv = B dx + C dy per pixel in double
                    const double dxd = __dsub_rn(double(pa.x), double(px));
                    du = dv = 0.f;
#pragma unroll
                    for (int i = 0; i < kPx; ++i) {
                        const double dyd = __dsub_rn(double(pa.y), double(y0 + i) + 0.5);
                        const float su = __double2float_rn(double(con.x) * dxd + double(con.y) * dyd);
                        const float sv = __double2float_rn(double(con.y) * dxd + double(con.z) * dyd);
                        du = fmaf(-m[i], su, du);
                        dv = fmaf(-m[i], sv, dv);
                    }
                } else {
                    du = fmaf(con.x * dx, s0, con.y * s1);
                    dv = fmaf(con.y * dx, s0, con.z * s1);
                }
                float v[8] = {du, dv, 0.5f * dx * dx * s0, dx * s1, 0.5f * s2, mo * pa.w, dr, dg};
                warp_reduce_and_add(v, db, lane, S.gid[buf][j], a);
            }
        }
        __syncwarp();
    }
    cp_async_wait_all();
}

// Tiles ordered by decreasing list length (bucketed by floor(sqrt(length)),
// 256 buckets; order inside a bucket unspecified), so that the longest tiles
// start first and the kernel's tail holds short ones.  One CTA.
__global__ void __launch_bounds__(1024) tile_order_kernel(const uint2* __restrict__ ranges, int tiles,
                                                         uint32_t* __restrict__ order) {
    __shared__ uint32_t count[256];
    __shared__ uint32_t start[256];
    for (int b = threadIdx.x; b < 256; b += blockDim.x) count[b] = 0u;
    __syncthreads();
    auto bucket = [&](int t) {
        const uint2 r = __ldg(ranges + t);
        const float len = float(r.y - r.x);
        return 255u - min(255u, uint32_t(sqrtf(len)));  // longest first
    };
    for (int t = threadIdx.x; t < tiles; t += blockDim.x) atomicAdd(&count[bucket(t)], 1u);
    __syncthreads();
    if (threadIdx.x == 0) {
        uint32_t run = 0;
        for (int b = 0; b < 256; ++b) {
            start[b] = run;
            run += count[b];
        }
    }
    __syncthreads();
    for (int t = threadIdx.x; t < tiles; t += blockDim.x) order[atomicAdd(&start[bucket(t)], 1u)] = uint32_t(t);
}

}  // namespace

cudaError_t launch_tile_order(const uint32_t* ranges, int tiles, uint32_t* order, cudaStream_t s) {
    if (tiles <= 0) return cudaSuccess;
    tile_order_kernel<<<1, 1024, 0, s>>>(reinterpret_cast<const uint2*>(ranges), tiles, order);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_raster_fwd(const gs_projected& proj, const uint32_t* vals, const uint32_t* ranges,
                              const uint32_t* order, const CamArgs& cam, const float bg[3], float* image,
                              float* final_T, int32_t* n_contrib, cudaStream_t s) {
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
    raster_fwd_kernel<<<unsigned((a.tiles * kSub + kWarps - 1) / kWarps), kWarps * 32, 0, s>>>(a);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_raster_bwd(const gs_projected& proj, const uint32_t* vals, const uint32_t* ranges,
                              const uint32_t* order, const CamArgs& cam, const float bg[3], const float* final_T,
                              const int32_t* n_contrib, const float* dL_dimage, const gs_grad2d& g2,
                              cudaStream_t s) {
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
    raster_bwd_kernel<<<unsigned((a.tiles * kSub + kWarps - 1) / kWarps), kWarps * 32, 0, s>>>(a);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace gsk
