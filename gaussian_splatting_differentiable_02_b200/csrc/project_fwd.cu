// gs_project: per-Gaussian projection (stages 1-2 of the pipeline in the gsplat
// guide, lmnt.cn/news/262699 §2.1) in double precision.
//
// This file is compiled with -fmad=false: every product and sum rounds as
// written, so the integer decisions taken from floating point (culling, the
// 3-sigma radius, the tile rectangle) and the float32 depth used in the sort key
// come out the same on any IEEE double implementation that evaluates the same
// expressions in the same order.  The SH coefficients may come from a 16-bit
// (IEEE half) copy; widening a half is exact, so the result is the float32 path's
// on the rounded coefficients.  The projection is streaming work (about 290
// bytes per Gaussian) and sits far below the device's double-precision rate, so
// the wider arithmetic costs no time.
#include <cuda_fp16.h>

#include "internal.cuh"

namespace gsk {
namespace {

// Real spherical harmonics to degree 3 (orthonormal, Condon-Shortley phase),
// index l^2 + l + m.
constexpr double kY0 = 0.28209479177387814;
constexpr double kY1 = 0.4886025119029199;
__constant__ double kY2[5] = {1.0925484305920792, -1.0925484305920792, 0.31539156525252005, -1.0925484305920792,
                           0.5462742152960396};
__constant__ double kY3[7] = {-0.5900435899266435, 2.890611442640554, -0.4570457994644658, 0.3731763325901154,
                           -0.4570457994644658, 1.445305721320277, -0.5900435899266435};

struct FwdArgs {
    const float4* means;
    const float4* quats;
    const float4* log_scales;
    const float* logits;
    const float4* sh;
    const uint2* sh_half;  // 16-bit copy of the SH planes (four IEEE halves per element), or null
    int deg, planes;
    int64_t n;
    CamArgs cam;
    float2* xy;
    float* depth;
    float4* conic_op;
    float4* rgb;
    int32_t* radius;
    uint2* rect;
    uint32_t* tiles_touched;
};

__device__ __forceinline__ bool finite(double x) { return isfinite(x); }

__device__ void write_culled(const FwdArgs& a, int64_t i) {
    a.xy[i] = make_float2(0.f, 0.f);
    a.depth[i] = 0.f;
    a.conic_op[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    a.rgb[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    a.radius[i] = 0;
    a.rect[i] = make_uint2(0u, 0u);
    a.tiles_touched[i] = 0u;
}

// One float4 element of SH plane p: from the float32 array, or widened exactly from
// the 16-bit copy.
template <bool kHalf>
__device__ __forceinline__ float4 sh_element(const float4* sh, const uint2* sh_half, int64_t n, int p, int64_t i) {
    if (!kHalf) return __ldg(sh + int64_t(p) * n + i);
    const uint2 h = __ldg(sh_half + int64_t(p) * n + i);
    const float2 lo = __half22float2(*reinterpret_cast<const __half2*>(&h.x));
    const float2 hi = __half22float2(*reinterpret_cast<const __half2*>(&h.y));
    return make_float4(lo.x, lo.y, hi.x, hi.y);
}

// The part of the projection that does not depend on the camera: the mean, the 3D
// covariance R S S^T R^T of the normalised quaternion and exp(log_scale), and the
// opacity.  ok is false for a Gaussian culled whatever the view (a non-finite
// parameter, a zero quaternion).
struct Gauss3D {
    double mu[3];
    double S[3][3];
    double o;
    bool ok;
};

__device__ __forceinline__ Gauss3D gauss3d(const float4 m4, const float4 q4, const float4 s4, const float lg) {
    Gauss3D g;
    g.mu[0] = m4.x;
    g.mu[1] = m4.y;
    g.mu[2] = m4.z;
    const double q[4] = {q4.x, q4.y, q4.z, q4.w};
    const double ls[3] = {s4.x, s4.y, s4.z};
    const double logit = lg;
    g.ok = finite(g.mu[0]) && finite(g.mu[1]) && finite(g.mu[2]) && finite(q[0]) && finite(q[1]) &&
           finite(q[2]) && finite(q[3]) && finite(ls[0]) && finite(ls[1]) && finite(ls[2]) && finite(logit);
    // rotation of the normalised quaternion (w, x, y, z)
    const double qn2 = ((q[0] * q[0] + q[1] * q[1]) + q[2] * q[2]) + q[3] * q[3];
    g.ok = g.ok && qn2 > 0.0;
    const double qn = sqrt(qn2);
    const double w = q[0] / qn, x = q[1] / qn, y = q[2] / qn, z = q[3] / qn;
    double Rq[3][3];
    Rq[0][0] = 1.0 - 2.0 * (y * y + z * z);
    Rq[0][1] = 2.0 * (x * y - w * z);
    Rq[0][2] = 2.0 * (x * z + w * y);
    Rq[1][0] = 2.0 * (x * y + w * z);
    Rq[1][1] = 1.0 - 2.0 * (x * x + z * z);
    Rq[1][2] = 2.0 * (y * z - w * x);
    Rq[2][0] = 2.0 * (x * z - w * y);
    Rq[2][1] = 2.0 * (y * z + w * x);
    Rq[2][2] = 1.0 - 2.0 * (x * x + y * y);

    const double s[3] = {exp(ls[0]), exp(ls[1]), exp(ls[2])};
    double M[3][3];
#pragma unroll
    for (int r = 0; r < 3; ++r)
#pragma unroll
        for (int c = 0; c < 3; ++c) M[r][c] = Rq[r][c] * s[c];
#pragma unroll
    for (int r = 0; r < 3; ++r)
#pragma unroll
        for (int c = 0; c < 3; ++c) g.S[r][c] = (M[r][0] * M[c][0] + M[r][1] * M[c][1]) + M[r][2] * M[c][2];
    g.o = 1.0 / (1.0 + exp(-logit));
    return g;
}

// One view's outputs of a Gaussian.
struct ViewOut {
    float2 xy;
    float depth;
    float4 conic_op;
    float4 rgb;
    int32_t radius;
    uint2 rect;
    uint32_t tiles_touched;
};

// The camera-dependent part of the projection of g in one view: camera-space
// mean, the perspective Jacobian (x/z and y/z clamped to 1.3 x the half field of
// view), J W Sigma W^T J^T + eps2d I, its inverse, the 3-sigma radius and tile
// rectangle, and the colour of the SH coefficients (sh(p): plane p as a float4)
// in the unit viewing direction.  Returns false when the view culls g.
template <class ShFetch>
__device__ __forceinline__ bool project_view(const CamArgs& cam, const Gauss3D& g, int deg, int planes, ShFetch sh,
                                             ViewOut& out) {
    const double* mu = g.mu;
    double pc[3];
#pragma unroll
    for (int r = 0; r < 3; ++r)
        pc[r] = ((cam.R[3 * r + 0] * mu[0] + cam.R[3 * r + 1] * mu[1]) + cam.R[3 * r + 2] * mu[2]) + cam.t[r];
    if (!(pc[2] > cam.near_plane)) return false;

    double txz = pc[0] / pc[2], tyz = pc[1] / pc[2];
    if (txz < -cam.limx) txz = -cam.limx;
    if (txz > cam.limx) txz = cam.limx;
    if (tyz < -cam.limy) tyz = -cam.limy;
    if (tyz > cam.limy) tyz = cam.limy;
    const double tx = txz * pc[2], ty = tyz * pc[2];
    const double iz = 1.0 / pc[2];
    const double J00 = cam.fx * iz, J02 = -(cam.fx * tx) * (iz * iz);
    const double J11 = cam.fy * iz, J12 = -(cam.fy * ty) * (iz * iz);
    double Tm[2][3];
#pragma unroll
    for (int c = 0; c < 3; ++c) {
        Tm[0][c] = J00 * cam.R[0 + c] + J02 * cam.R[6 + c];
        Tm[1][c] = J11 * cam.R[3 + c] + J12 * cam.R[6 + c];
    }
    double X[2][3];
#pragma unroll
    for (int r = 0; r < 2; ++r)
#pragma unroll
        for (int c = 0; c < 3; ++c) X[r][c] = (Tm[r][0] * g.S[0][c] + Tm[r][1] * g.S[1][c]) + Tm[r][2] * g.S[2][c];
    const double ca = ((X[0][0] * Tm[0][0] + X[0][1] * Tm[0][1]) + X[0][2] * Tm[0][2]) + cam.eps2d;
    const double cb = (X[0][0] * Tm[1][0] + X[0][1] * Tm[1][1]) + X[0][2] * Tm[1][2];
    const double cc = ((X[1][0] * Tm[1][0] + X[1][1] * Tm[1][1]) + X[1][2] * Tm[1][2]) + cam.eps2d;
    const double det = ca * cc - cb * cb;
    if (!(det > 0.0)) return false;
    const double idet = 1.0 / det;

    const double mid = 0.5 * (ca + cc);
    const double lmax = mid + sqrt(fmax(0.1, mid * mid - det));
    const double r = ceil(3.0 * sqrt(lmax));

    const double u = cam.fx * (pc[0] / pc[2]) + cam.cx;
    const double v = cam.fy * (pc[1] / pc[2]) + cam.cy;
    if (!finite(u) || !finite(v) || !finite(r)) return false;

    const double TXd = cam.TX, TYd = cam.TY;
    const double xmin = fmin(fmax(floor((u - r) * 0.0625), 0.0), TXd);
    const double xmax = fmin(fmax(floor((u + r) * 0.0625) + 1.0, 0.0), TXd);
    const double ymin = fmin(fmax(floor((v - r) * 0.0625), 0.0), TYd);
    const double ymax = fmin(fmax(floor((v + r) * 0.0625) + 1.0, 0.0), TYd);
    if ((xmax - xmin) * (ymax - ymin) <= 0.0) return false;

    // colour from the SH of the unit viewing direction
    const double dvx = mu[0] - cam.cc[0], dvy = mu[1] - cam.cc[1], dvz = mu[2] - cam.cc[2];
    const double dn = sqrt((dvx * dvx + dvy * dvy) + dvz * dvz);
    const double ux = dvx / dn, uy = dvy / dn, uz = dvz / dn;
    double Y[16];
    Y[0] = kY0;
    if (deg >= 1) {
        Y[1] = -kY1 * uy;
        Y[2] = kY1 * uz;
        Y[3] = -kY1 * ux;
    }
    if (deg >= 2) {
        const double xx = ux * ux, yy = uy * uy, zz = uz * uz;
        Y[4] = kY2[0] * (ux * uy);
        Y[5] = kY2[1] * (uy * uz);
        Y[6] = kY2[2] * (2.0 * zz - xx - yy);
        Y[7] = kY2[3] * (ux * uz);
        Y[8] = kY2[4] * (xx - yy);
        if (deg >= 3) {
            Y[9] = kY3[0] * uy * (3.0 * xx - yy);
            Y[10] = kY3[1] * (ux * uy) * uz;
            Y[11] = kY3[2] * uy * (4.0 * zz - xx - yy);
            Y[12] = kY3[3] * uz * (2.0 * zz - 3.0 * xx - 3.0 * yy);
            Y[13] = kY3[4] * ux * (4.0 * zz - xx - yy);
            Y[14] = kY3[5] * uz * (xx - yy);
            Y[15] = kY3[6] * ux * (xx - 3.0 * yy);
        }
    }
    const int nc = (deg + 1) * (deg + 1);
    double col[3] = {0.0, 0.0, 0.0};
#pragma unroll
    for (int p = 0; p < 12; ++p) {
        if (p >= planes) break;
        const float4 c4 = sh(p);
        const float cv[4] = {c4.x, c4.y, c4.z, c4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int f = 4 * p + e;  // flat coefficient index = 3 k + channel
            const int k = f / 3;
            if (k < nc) col[f - 3 * k] += double(cv[e]) * Y[k];
        }
    }
    float rgbf[3];
    bool colour_ok = true;
#pragma unroll
    for (int ch = 0; ch < 3; ++ch) {
        const double c = col[ch] + 0.5;
        colour_ok = colour_ok && finite(c);
        rgbf[ch] = float(c < 0.0 ? 0.0 : c);
    }
    if (!colour_ok) return false;

    out.xy = make_float2(float(u), float(v));
    out.depth = float(pc[2]);
    out.conic_op = make_float4(float(cc * idet), float(-cb * idet), float(ca * idet), float(g.o));
    out.rgb = make_float4(rgbf[0], rgbf[1], rgbf[2], 0.f);
    out.radius = int32_t(r);
    const uint32_t x0 = uint32_t(xmin), y0 = uint32_t(ymin), x1 = uint32_t(xmax), y1 = uint32_t(ymax);
    out.rect = make_uint2(x0 | (y0 << 16), x1 | (y1 << 16));
    out.tiles_touched = (x1 - x0) * (y1 - y0);
    return true;
}

template <bool kHalf>
__global__ void __launch_bounds__(256) project_fwd_kernel(const FwdArgs a) {
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < a.n; i += int64_t(gridDim.x) * blockDim.x) {
        const float4 m4 = __ldg(a.means + i);
        const float4 q4 = __ldg(a.quats + i);
        const float4 s4 = __ldg(a.log_scales + i);
        const float lg = __ldg(a.logits + i);
        // the SH planes are read only after the covariance arithmetic: start moving
        // them into L2 now so that their loads do not wait on DRAM then
        for (int p = 0; p < a.planes; ++p) {
            if (kHalf)
                asm volatile("prefetch.global.L2 [%0];" ::"l"(a.sh_half + int64_t(p) * a.n + i));
            else
                asm volatile("prefetch.global.L2 [%0];" ::"l"(a.sh + int64_t(p) * a.n + i));
        }
        const Gauss3D g = gauss3d(m4, q4, s4, lg);
        ViewOut o;
        const auto sh = [&](int p) { return sh_element<kHalf>(a.sh, a.sh_half, a.n, p, i); };
        if (!g.ok || !project_view(a.cam, g, a.deg, a.planes, sh, o)) {
            write_culled(a, i);
            continue;
        }
        a.xy[i] = o.xy;
        a.depth[i] = o.depth;
        a.conic_op[i] = o.conic_op;
        a.rgb[i] = o.rgb;
        a.radius[i] = o.radius;
        a.rect[i] = o.rect;
        a.tiles_touched[i] = o.tiles_touched;
    }
}

// Several views of the same Gaussians in one pass: the parameters (236 bytes a
// Gaussian at SH degree 3) are read and the view-independent part computed once,
// then every view's outputs are written; the per-view arithmetic is
// project_view's, so each view's results are those of project_fwd_kernel bit for
// bit.
struct ViewOutPtrs {
    float2* xy;
    float* depth;
    float4* conic_op;
    float4* rgb;
    int32_t* radius;
    uint2* rect;
    uint32_t* tiles_touched;
};

struct ViewsArgs {
    const float4* means;
    const float4* quats;
    const float4* log_scales;
    const float* logits;
    const float4* sh;
    const uint2* sh_half;
    int deg, planes, V;
    int64_t n;
    CamArgs cam[GS_MAX_VIEWS];
    ViewOutPtrs out[GS_MAX_VIEWS];
};

#ifndef GS_PROJECT_VIEWS_PER_THREAD
#define GS_PROJECT_VIEWS_PER_THREAD 16
#endif
// views a thread projects (a grid row per group of views; 1, 2, 4, 8, 16 views per
// thread: 1.81, 1.32, 1.09, 1.00, 0.99 ms for 16 views of 1M Gaussians at 1080p,
// against 1.72 ms for 16 single-view launches)
constexpr int kViewsPerThread = GS_PROJECT_VIEWS_PER_THREAD;

// With the SH planes in shared memory the kernel fits 4 blocks per SM in 124
// registers (16 views of 1M Gaussians: 0.98 -> 0.745 ms; the planes in registers
// took 229 registers, 2 blocks per SM)
#ifndef GS_PROJECT_VIEWS_MIN_BLOCKS
#define GS_PROJECT_VIEWS_MIN_BLOCKS 4
#endif
template <bool kHalf>
__global__ void __launch_bounds__(128, GS_PROJECT_VIEWS_MIN_BLOCKS) project_views_kernel(const __grid_constant__ ViewsArgs a) {
    __shared__ float4 shs[12][128];  // this thread's SH planes, column threadIdx.x (not in registers)
    const int v0 = blockIdx.y * kViewsPerThread;
    const int v1 = min(a.V, v0 + kViewsPerThread);
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < a.n; i += int64_t(gridDim.x) * blockDim.x) {
        const Gauss3D g = gauss3d(__ldg(a.means + i), __ldg(a.quats + i), __ldg(a.log_scales + i),
                                  __ldg(a.logits + i));
#pragma unroll
        for (int p = 0; p < 12; ++p)
            if (p < a.planes) shs[p][threadIdx.x] = sh_element<kHalf>(a.sh, a.sh_half, a.n, p, i);
        const auto sh = [&](int p) { return shs[p][threadIdx.x]; };
        for (int v = v0; v < v1; ++v) {
            const ViewOutPtrs& w = a.out[v];
            ViewOut o;
            if (!g.ok || !project_view(a.cam[v], g, a.deg, a.planes, sh, o)) {
                w.xy[i] = make_float2(0.f, 0.f);
                w.depth[i] = 0.f;
                w.conic_op[i] = make_float4(0.f, 0.f, 0.f, 0.f);
                w.rgb[i] = make_float4(0.f, 0.f, 0.f, 0.f);
                w.radius[i] = 0;
                w.rect[i] = make_uint2(0u, 0u);
                w.tiles_touched[i] = 0u;
                continue;
            }
            w.xy[i] = o.xy;
            w.depth[i] = o.depth;
            w.conic_op[i] = o.conic_op;
            w.rgb[i] = o.rgb;
            w.radius[i] = o.radius;
            w.rect[i] = o.rect;
            w.tiles_touched[i] = o.tiles_touched;
        }
    }
}

}  // namespace

cudaError_t launch_project_fwd(const gs_params& p, const CamArgs& cam, const gs_projected& out, cudaStream_t s,
                               const uint16_t* sh_half) {
    FwdArgs a;
    a.means = reinterpret_cast<const float4*>(p.means);
    a.quats = reinterpret_cast<const float4*>(p.quats);
    a.log_scales = reinterpret_cast<const float4*>(p.log_scales);
    a.logits = p.opacity_logits;
    a.sh = reinterpret_cast<const float4*>(p.sh);
    a.sh_half = reinterpret_cast<const uint2*>(sh_half);
    a.deg = p.sh_degree;
    a.planes = sh_planes(p.sh_degree);
    a.n = p.n;
    a.cam = cam;
    a.xy = reinterpret_cast<float2*>(out.xy);
    a.depth = out.depth;
    a.conic_op = reinterpret_cast<float4*>(out.conic_opacity);
    a.rgb = reinterpret_cast<float4*>(out.rgb);
    a.radius = out.radius;
    a.rect = reinterpret_cast<uint2*>(out.rect);
    a.tiles_touched = out.tiles_touched;
    if (p.n == 0) return cudaSuccess;
    if (sh_half)
        project_fwd_kernel<true><<<grid_for(p.n, 256, 16), 256, 0, s>>>(a);
    else
        project_fwd_kernel<false><<<grid_for(p.n, 256, 16), 256, 0, s>>>(a);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_project_views(const gs_params& p, int V, const CamArgs* cams, const gs_projected* outs,
                                 cudaStream_t s, const uint16_t* sh_half) {
    ViewsArgs a;
    a.means = reinterpret_cast<const float4*>(p.means);
    a.quats = reinterpret_cast<const float4*>(p.quats);
    a.log_scales = reinterpret_cast<const float4*>(p.log_scales);
    a.logits = p.opacity_logits;
    a.sh = reinterpret_cast<const float4*>(p.sh);
    a.sh_half = reinterpret_cast<const uint2*>(sh_half);
    a.deg = p.sh_degree;
    a.planes = sh_planes(p.sh_degree);
    a.V = V;
    a.n = p.n;
    for (int v = 0; v < V; ++v) {
        a.cam[v] = cams[v];
        a.out[v].xy = reinterpret_cast<float2*>(outs[v].xy);
        a.out[v].depth = outs[v].depth;
        a.out[v].conic_op = reinterpret_cast<float4*>(outs[v].conic_opacity);
        a.out[v].rgb = reinterpret_cast<float4*>(outs[v].rgb);
        a.out[v].radius = outs[v].radius;
        a.out[v].rect = reinterpret_cast<uint2*>(outs[v].rect);
        a.out[v].tiles_touched = outs[v].tiles_touched;
    }
    if (p.n == 0 || V == 0) return cudaSuccess;
    const dim3 grid(grid_for(p.n, 128, 16), unsigned((V + kViewsPerThread - 1) / kViewsPerThread));
    if (sh_half)
        project_views_kernel<true><<<grid, 128, 0, s>>>(a);
    else
        project_views_kernel<false><<<grid, 128, 0, s>>>(a);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace gsk
