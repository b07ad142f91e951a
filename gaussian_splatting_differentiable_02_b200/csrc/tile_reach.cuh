// The tiles of a Gaussian's tile rectangle that its footprint can reach: where
// alpha = o e^-sigma can be at least 1/255 (the skip threshold of the
// compositing) at some point of the tile's box of pixel centres.  Binning a
// Gaussian into those tiles only, instead of its whole 3-sigma rectangle, drops
// the instances every pixel of the tile would skip anyway (the "culling and
// reordering" stage the MUSA co-design article, qwbw.cn/news/278220 §1, counts
// among the four 3DGS bottlenecks): images, final_T and gradients stay the
// same, n_contrib counts list positions in the shorter lists.
//
// The region sigma <= s is an ellipse for a positive definite conic, and its
// intersection with a tile row's band of pixel centres is convex, so the tiles
// it reaches in a row are one run of columns.  The projection counts them
// (tiles_touched) and the emission of the binning walks the same runs, both
// through tile_reach_row; every operation below is a correctly rounded double
// operation written as its intrinsic (no contraction into FMAs) or an exact one
// (floor, ceil, min, max, conversions), and the one float32 logarithm is the
// hardware lg2, so the two kernels take the same decisions bit for bit
// whatever their compile flags.
//
// Conservative by construction: s = ln(255 o) + 1e-4 (|ln(255 o)| + 1) from
// a float32 log2 good to 1e-6, and every box widened by 1/1024 px on each side,
// so a tile where the float32 compositing could blend the Gaussian is always
// kept.  A conic that is not positive definite in double keeps its whole
// rectangle; an opacity below about 1/255 reaches no tile.
#pragma once

#include <stdint.h>

namespace gsk {

struct TileReach {
    float u, v;     // mean in pixels
    float A, B, C;  // conic
    int mode;       // 0: no tile, 1: runs per row, 2: the whole rectangle
    double det;     // A C - B^2 (A C and B^2 are exact in double)
    double iA;      // 1 / A
    double s;       // the sigma bound, margin included
    double ym;      // half height of the region sigma <= s: sqrt(2 A s / det)
    double xm;      // half width: sqrt(2 C s / det)
    double dyr;     // dy of its rightmost point, where dx = xm (the leftmost: -dyr, -xm)
};

__device__ __forceinline__ float lg2_approx(float x) {
    float y;
    asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ TileReach tile_reach_setup(float2 xy, float4 conic_op) {
    TileReach r;
    r.u = xy.x;
    r.v = xy.y;
    r.A = conic_op.x;
    r.B = conic_op.y;
    r.C = conic_op.z;
    const double A = r.A, B = r.B, C = r.C;
    r.det = __dsub_rn(__dmul_rn(A, C), __dmul_rn(B, B));
    r.iA = 0.0;
    r.s = 0.0;
    r.ym = 0.0;
    r.xm = 0.0;
    r.dyr = 0.0;
    if (!(A > 0.0) || !(C > 0.0) || !(r.det > 0.0) || !(fabsf(r.u) < 1e30f) || !(fabsf(r.v) < 1e30f)) {
        r.mode = 2;
        return r;
    }
    // ln(255 o) = (log2 255 + log2 o) ln 2
    const double l = __dmul_rn(__dadd_rn(7.994353436858858, double(lg2_approx(conic_op.w))), 0.6931471805599453);
    const double s = __dadd_rn(l, __dmul_rn(__dadd_rn(fabs(l), 1.0), 1e-4));  // l + 1e-4 (|l| + 1)
    if (!(s > 0.0)) {  // also a NaN or zero opacity
        r.mode = 0;
        return r;
    }
    r.s = s;
    r.iA = __drcp_rn(A);
    const double two_s = __dmul_rn(2.0, s);
    r.ym = __dsqrt_rn(__ddiv_rn(__dmul_rn(two_s, A), r.det));
    r.xm = __dsqrt_rn(__ddiv_rn(__dmul_rn(two_s, C), r.det));
    r.dyr = __ddiv_rn(__dmul_rn(-B, r.xm), C);
    r.mode = 1;
    return r;
}

// Columns [*c0, *c1) of tile row ty that the region reaches, within the
// rectangle's columns [x0, x1); an empty run has *c0 == *c1.
__device__ __forceinline__ void tile_reach_row(const TileReach& r, int ty, int x0, int x1, int* c0, int* c1) {
    if (r.mode != 1) {
        *c0 = x0;
        *c1 = r.mode == 2 ? x1 : x0;
        return;
    }
    constexpr double kWiden = 1.0 / 1024.0;
    const double yb = double(16 * ty);
    const double v = r.v;
    const double dylo = __dsub_rn(__dadd_rn(yb, 0.5 - kWiden), v);
    const double dyhi = __dsub_rn(__dadd_rn(yb, 15.5 + kWiden), v);
    const double lo = fmax(dylo, -r.ym), hi = fmin(dyhi, r.ym);
    if (!(lo <= hi)) {
        *c0 = *c1 = x0;
        return;
    }
    // x extent at dy: (-B dy +- sqrt(2 A s - det dy^2)) / A; the right end is
    // concave in dy (largest at dyr clamped to the band: xm when dyr lies in it),
    // the left end convex (smallest at -dyr clamped: -xm when -dyr lies in it)
    const double A = r.A, B = r.B, u = r.u;
    const double two_as = __dmul_rn(__dmul_rn(2.0, A), r.s);
    const double dy_r = fmin(fmax(r.dyr, lo), hi);
    const double dy_l = fmin(fmax(-r.dyr, lo), hi);
    double xr = r.xm, xl = -r.xm;
    if (dy_r != r.dyr) {
        const double q = fmax(__dsub_rn(two_as, __dmul_rn(r.det, __dmul_rn(dy_r, dy_r))), 0.0);
        xr = __dmul_rn(__dadd_rn(__dmul_rn(-B, dy_r), __dsqrt_rn(q)), r.iA);
    }
    if (dy_l != -r.dyr) {
        const double q = fmax(__dsub_rn(two_as, __dmul_rn(r.det, __dmul_rn(dy_l, dy_l))), 0.0);
        xl = __dmul_rn(__dsub_rn(__dmul_rn(-B, dy_l), __dsqrt_rn(q)), r.iA);
    }
    // tile tx reaches [u + xl, u + xr] when 16 tx + 0.5 - w <= u + xr and
    // 16 tx + 15.5 + w >= u + xl
    const double hi_t = floor(__dmul_rn(__dsub_rn(__dadd_rn(u, xr), 0.5 - kWiden), 0.0625));
    const double lo_t = ceil(__dmul_rn(__dsub_rn(__dadd_rn(u, xl), 15.5 + kWiden), 0.0625));
    const double a = fmax(lo_t, double(x0));
    const double b = fmin(hi_t + 1.0, double(x1));
    if (!(a < b)) {
        *c0 = *c1 = x0;
        return;
    }
    *c0 = int(a);
    *c1 = int(b);
}

// Number of rectangle tiles [x0, x1) x [y0, y1) the region reaches.
__device__ __forceinline__ uint32_t tile_reach_count(const TileReach& r, int x0, int y0, int x1, int y1) {
    if (r.mode == 2) return uint32_t(x1 - x0) * uint32_t(y1 - y0);
    if (r.mode == 0) return 0u;
    uint32_t n = 0;
    for (int ty = y0; ty < y1; ++ty) {
        int c0, c1;
        tile_reach_row(r, ty, x0, x1, &c0, &c1);
        n += uint32_t(c1 - c0);
    }
    return n;
}

}  // namespace gsk
