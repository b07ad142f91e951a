// gs_project_bwd, gs_project_bwd_views, gs_project_bwd_views_adam: chain the
// per-Gaussian 2D gradients of one or several views through the projection to
// the Gaussian parameters (the "gradients to position / covariance / colour /
// opacity" of one fused backward, MUSA co-design article qwbw.cn/news/278220
// §2.2), and optionally apply the Adam step of the gsplat guide
// (lmnt.cn/news/262699) §4.2 in the same pass.
//
// Every view in which a Gaussian is visible contributes to dL/dSigma (6 values),
// dL/dmean, dL/dlogit and the 48 SH gradients; the view-independent part
// (normalised quaternion, rotation, scales, M = R diag(s), Sigma = M M^T) and the
// chain from the summed dL/dSigma to the scales and the quaternion are shared.
// Two kernels:
//   * one or two views: one thread per Gaussian, the views in a loop, the 48 SH
//     sums in a second pass over the visible views (their masked colour
//     gradients kept in shared memory) so that they never share registers with
//     the geometric chain; with Adam and no gradient buffer, the step runs in the
//     same thread and the gradients never reach memory (0.675 ms for 1M Gaussians
//     seen by one view), with a buffer it is the second launch below (0.569 ms);
//   * three to 16 views: one thread per Gaussian, the views in a loop, the 48 SH
//     sums in shared memory; with Adam, the summed gradient is written to the
//     caller's gradient buffer (required here) and the Adam step of all five
//     groups follows as a second, streaming launch.  Fused into the chain, the step's 15 float4
//     read-modify-writes per Gaussian ran one memory round trip after another in
//     a kernel held to 12 warps per SM by its registers (2.06 ms for 16 views of
//     1M Gaussians); apart, the chain takes 1.2 ms and the step 0.3 ms at 82% of
//     the measured HBM bandwidth.
// In the packed layout (gs_project_packed) a view's features and 2D gradients
// are read at the Gaussian's slot, found through the view's slot map.  With
// 16-bit SH storage the colour chain takes the half-precision coefficients the
// forward pass used, Adam updates the float32 coefficients, and their rounding to
// half is written back.
//
// The geometric chain is double precision: the inverse of a 2x2 conic and the
// EWA product are badly conditioned for needle-shaped Gaussians.  The colour
// (SH) chain is float32 except the sign test of the raw colour, which repeats the
// forward pass's double-precision decision.
#include <cuda_fp16.h>

#include <type_traits>

#include "internal.cuh"

namespace gsk {
namespace {

constexpr double kY0 = 0.28209479177387814;
constexpr double kY1 = 0.4886025119029199;
__constant__ double kY2[5] = {1.0925484305920792, -1.0925484305920792, 0.31539156525252005, -1.0925484305920792,
                              0.5462742152960396};
__constant__ double kY3[7] = {-0.5900435899266435, 2.890611442640554, -0.4570457994644658, 0.3731763325901154,
                              -0.4570457994644658, 1.445305721320277, -0.5900435899266435};

constexpr int kMaxViews = GS_MAX_VIEWS;
constexpr int kBwdBlock = 128;

// A view as the backward pass needs it: the camera (float32 values, widened
// exactly), the clamp limits and centre in double as the forward pass computed
// them, and the view's visibility and 2D gradients.
struct ViewArgs {
    double limx, limy, cc[3], eps2d;
    float R[9], t[3], fx, fy;
    const int32_t* slot;  // packed layout: entry of each Gaussian (-1: none); else null
    const int32_t* radius;
    const float2* g_xy;
    const float2* g_xy_abs;  // absolute 2D gradient for the densification statistic (nullable)
    const float4* g_con;
    const float4* g_rgb;
};

struct Args {
    const float4* means;
    const float4* quats;
    const float4* log_scales;
    const float* logits;
    const float4* sh;
    const uint2* sh_half;  // kHalf: the 16-bit SH the forward used (four halves per element)
    uint2* sh_half_out;    // kHalf: the updated SH rounded to 16 bits (may alias sh_half)
    int deg, planes, V;
    int64_t n;
    ViewArgs view[kMaxViews];
    // gradient outputs (+=), any may be null together (all or none)
    float4* d_means;
    float4* d_quats;
    float4* d_log_scales;
    float* d_logits;
    float4* d_sh;
    float* densify_accum;
    int32_t* densify_count;
    int32_t* densify_max_radius;
    bool sparse;     // Adam: leave Gaussians visible in no view untouched
    bool overwrite;  // gradient outputs written (this step's gradient) instead of added to
    // Adam (kAdam): parameters updated in place, first and second moments
    float4* p_means;
    float4* p_quats;
    float4* p_log_scales;
    float* p_logits;
    float4* p_sh;
    float4* m_means;
    float4* m_quats;
    float4* m_log_scales;
    float* m_logits;
    float4* m_sh;
    float4* v_means;
    float4* v_quats;
    float4* v_log_scales;
    float* v_logits;
    float4* v_sh;
    float lr_t[5];  // lr / (1 - beta1^t) for means, quats, log_scales, logits, sh
    float inv_sqrt_bc2, b1, b2, eps;
};

// Real SH basis to degree 3 (orthonormal, Condon-Shortley phase kept) at the
// unit direction (x, y, z), index l^2 + l + m.
template <typename T>
__device__ __forceinline__ void sh_basis(int deg, T x, T y, T z, T* Y) {
    Y[0] = T(kY0);
    if (deg < 1) return;
    Y[1] = T(-kY1) * y;
    Y[2] = T(kY1) * z;
    Y[3] = T(-kY1) * x;
    if (deg < 2) return;
    const T xx = x * x, yy = y * y, zz = z * z;
    Y[4] = T(kY2[0]) * (x * y);
    Y[5] = T(kY2[1]) * (y * z);
    Y[6] = T(kY2[2]) * (T(2) * zz - xx - yy);
    Y[7] = T(kY2[3]) * (x * z);
    Y[8] = T(kY2[4]) * (xx - yy);
    if (deg < 3) return;
    Y[9] = T(kY3[0]) * y * (T(3) * xx - yy);
    Y[10] = T(kY3[1]) * (x * y) * z;
    Y[11] = T(kY3[2]) * y * (T(4) * zz - xx - yy);
    Y[12] = T(kY3[3]) * z * (T(2) * zz - T(3) * xx - T(3) * yy);
    Y[13] = T(kY3[4]) * x * (T(4) * zz - xx - yy);
    Y[14] = T(kY3[5]) * z * (xx - yy);
    Y[15] = T(kY3[6]) * x * (xx - T(3) * yy);
}

// g += sum_k w[k] dY_k/d(x, y, z) for the basis above.
__device__ __forceinline__ void sh_grad_dir(int deg, float x, float y, float z, const float* w, float* g) {
    if (deg < 1) return;
    const float c1 = float(kY1);
    g[0] += -c1 * w[3];
    g[1] += -c1 * w[1];
    g[2] += c1 * w[2];
    if (deg < 2) return;
    const float c20 = float(kY2[0]), c21 = float(kY2[1]), c22 = float(kY2[2]), c23 = float(kY2[3]),
                c24 = float(kY2[4]);
    g[0] += c20 * y * w[4] - 2.f * c22 * x * w[6] + c23 * z * w[7] + 2.f * c24 * x * w[8];
    g[1] += c20 * x * w[4] + c21 * z * w[5] - 2.f * c22 * y * w[6] - 2.f * c24 * y * w[8];
    g[2] += c21 * y * w[5] + 4.f * c22 * z * w[6] + c23 * x * w[7];
    if (deg < 3) return;
    const float xx = x * x, yy = y * y, zz = z * z;
    const float c30 = float(kY3[0]), c31 = float(kY3[1]), c32 = float(kY3[2]), c33 = float(kY3[3]),
                c34 = float(kY3[4]), c35 = float(kY3[5]), c36 = float(kY3[6]);
    g[0] += c30 * 6.f * x * y * w[9] + c31 * y * z * w[10] - c32 * 2.f * x * y * w[11] - c33 * 6.f * x * z * w[12] +
            c34 * (4.f * zz - 3.f * xx - yy) * w[13] + c35 * 2.f * x * z * w[14] + c36 * (3.f * xx - 3.f * yy) * w[15];
    g[1] += c30 * (3.f * xx - 3.f * yy) * w[9] + c31 * x * z * w[10] + c32 * (4.f * zz - xx - 3.f * yy) * w[11] -
            c33 * 6.f * y * z * w[12] - c34 * 2.f * x * y * w[13] - c35 * 2.f * y * z * w[14] - c36 * 6.f * x * y * w[15];
    g[2] += c31 * x * y * w[10] + c32 * 8.f * y * z * w[11] + c33 * (6.f * zz - 3.f * xx - 3.f * yy) * w[12] +
            c34 * 8.f * x * z * w[13] + c35 * (xx - yy) * w[14];
}

__device__ __forceinline__ float adam_one(float p, float g, float& m, float& v, float lr_t, const Args& a) {
    m = a.b1 * m + (1.f - a.b1) * g;
    v = a.b2 * v + (1.f - a.b2) * (g * g);
    return p - lr_t * m / (sqrtf(v) * a.inv_sqrt_bc2 + a.eps);
}

// One float4 element of a parameter with its two moments.  The fused step loads
// several of them before storing any: the parameter and moment arrays could alias
// as far as the compiler knows, so a load placed after a store has to wait for it,
// and each element would make its own round trip to memory.
struct AdamElem {
    float4 p, m, v;
};

__device__ __forceinline__ AdamElem adam_load(const float4* p, const float4* m, const float4* v, int64_t i) {
    return AdamElem{p[i], m[i], v[i]};
}

__device__ __forceinline__ void adam_apply(AdamElem& e, float4 g, float lr_t, const Args& a) {
    e.p.x = adam_one(e.p.x, g.x, e.m.x, e.v.x, lr_t, a);
    e.p.y = adam_one(e.p.y, g.y, e.m.y, e.v.y, lr_t, a);
    e.p.z = adam_one(e.p.z, g.z, e.m.z, e.v.z, lr_t, a);
    e.p.w = adam_one(e.p.w, g.w, e.m.w, e.v.w, lr_t, a);
}

__device__ __forceinline__ void adam_store(float4* p, float4* m, float4* v, int64_t i, const AdamElem& e) {
    p[i] = e.p;
    m[i] = e.m;
    v[i] = e.v;
}

__device__ __forceinline__ float4 widen(uint2 h) {
    const float2 lo = __half22float2(*reinterpret_cast<const __half2*>(&h.x));
    const float2 hi = __half22float2(*reinterpret_cast<const __half2*>(&h.y));
    return make_float4(lo.x, lo.y, hi.x, hi.y);
}

__device__ __forceinline__ uint2 narrow(float4 f) {
    const __half2 lo = __floats2half2_rn(f.x, f.y);
    const __half2 hi = __floats2half2_rn(f.z, f.w);
    uint2 w;
    w.x = *reinterpret_cast<const uint32_t*>(&lo);
    w.y = *reinterpret_cast<const uint32_t*>(&hi);
    return w;
}

__device__ __forceinline__ void add4(float4* d, int64_t i, float4 g) {
    float4 x = d[i];
    d[i] = make_float4(x.x + g.x, x.y + g.y, x.z + g.z, x.w + g.w);
}

// Index of Gaussian i's entry in a view's projected features and 2D gradients:
// i itself, or its slot in the packed layout.
template <bool kPacked>
__device__ __forceinline__ int64_t entry(const ViewArgs& w, int64_t i) {
    return kPacked ? int64_t(__ldg(w.slot + i)) : i;
}

// One view's contribution to a Gaussian's gradients: the per-view part of the
// chain, from the view's 2D gradients back to dL/dSigma, dL/dmean and dL/dlogit,
// and the colour gradient with the SH basis it multiplies.
struct ViewTerms {
    double gS[6];     // dL/dSigma (xx, xy, xz, yy, yz, zz)
    double gmu_p[3];  // dL/dmean through the camera-space position (projection and Jacobian)
    double gmu_c[3];  // dL/dmean through the SH viewing direction
    double glogit;    // dL/dlogit
    float gcol[3];    // dL/dcolour, zero for a channel the forward pass clamped
    float Y[16];      // SH basis at the viewing direction
    float dnorm;      // the densification statistic's norm of the view's 2D position gradient
};

// sh(q): the Gaussian's SH coefficient q = 3 k + channel (float32, as the forward used it).
template <class Sh>
__device__ __forceinline__ void view_terms(const ViewArgs& cam, const double mu[3], const double S6[6],
                                           double do_dlogit, int deg, int nc, const Sh& sh, float2 gxy, float4 gco,
                                           float4 grg, float2 sxy, ViewTerms& o) {
    const double fx = cam.fx, fy = cam.fy;
    double pc[3];
#pragma unroll
    for (int r = 0; r < 3; ++r)
        pc[r] = ((double(cam.R[3 * r]) * mu[0] + double(cam.R[3 * r + 1]) * mu[1]) + double(cam.R[3 * r + 2]) * mu[2]) +
                double(cam.t[r]);
    const double iz = 1.0 / pc[2];
    double txz = pc[0] * iz, tyz = pc[1] * iz;
    const bool clx = (txz < -cam.limx) || (txz > cam.limx);
    const bool cly = (tyz < -cam.limy) || (tyz > cam.limy);
    txz = fmin(fmax(txz, -cam.limx), cam.limx);
    tyz = fmin(fmax(tyz, -cam.limy), cam.limy);
    const double J00 = fx * iz, J02 = -fx * txz * iz;
    const double J11 = fy * iz, J12 = -fy * tyz * iz;
    double T0[3], T1[3];
#pragma unroll
    for (int c = 0; c < 3; ++c) {
        T0[c] = J00 * double(cam.R[c]) + J02 * double(cam.R[6 + c]);
        T1[c] = J11 * double(cam.R[3 + c]) + J12 * double(cam.R[6 + c]);
    }
    const double ST0[3] = {S6[0] * T0[0] + S6[1] * T0[1] + S6[2] * T0[2], S6[1] * T0[0] + S6[3] * T0[1] + S6[4] * T0[2],
                           S6[2] * T0[0] + S6[4] * T0[1] + S6[5] * T0[2]};
    const double ST1[3] = {S6[0] * T1[0] + S6[1] * T1[1] + S6[2] * T1[2], S6[1] * T1[0] + S6[3] * T1[1] + S6[4] * T1[2],
                           S6[2] * T1[0] + S6[4] * T1[1] + S6[5] * T1[2]};
    const double ca = T0[0] * ST0[0] + T0[1] * ST0[1] + T0[2] * ST0[2] + cam.eps2d;
    const double cb = T0[0] * ST1[0] + T0[1] * ST1[1] + T0[2] * ST1[2];
    const double cc = T1[0] * ST1[0] + T1[1] * ST1[1] + T1[2] * ST1[2] + cam.eps2d;
    const double det = ca * cc - cb * cb;

    // conic (A, B, C) = (c, -b, a) / det  ->  (a, b, c)
    const double gA = gco.x, gB = gco.y, gC = gco.z;
    const double id2 = 1.0 / (det * det);
    const double ga = (-cc * cc * gA + cb * cc * gB - cb * cb * gC) * id2;
    const double gb = (2.0 * cb * cc * gA - (ca * cc + cb * cb) * gB + 2.0 * ca * cb * gC) * id2;
    const double gc = (-cb * cb * gA + ca * cb * gB - ca * ca * gC) * id2;
    // dL/dSigma = ga T0 T0^T + gb/2 (T0 T1^T + T1 T0^T) + gc T1 T1^T
    o.gS[0] = ga * T0[0] * T0[0] + gb * T0[0] * T1[0] + gc * T1[0] * T1[0];
    o.gS[1] = ga * T0[0] * T0[1] + 0.5 * gb * (T0[0] * T1[1] + T1[0] * T0[1]) + gc * T1[0] * T1[1];
    o.gS[2] = ga * T0[0] * T0[2] + 0.5 * gb * (T0[0] * T1[2] + T1[0] * T0[2]) + gc * T1[0] * T1[2];
    o.gS[3] = ga * T0[1] * T0[1] + gb * T0[1] * T1[1] + gc * T1[1] * T1[1];
    o.gS[4] = ga * T0[1] * T0[2] + 0.5 * gb * (T0[1] * T1[2] + T1[1] * T0[2]) + gc * T1[1] * T1[2];
    o.gS[5] = ga * T0[2] * T0[2] + gb * T0[2] * T1[2] + gc * T1[2] * T1[2];
    // rows of T = J W, then J(x, y, z) and (u, v) = (fx x/z + cx, fy y/z + cy)
    double gpc[3];
    {
        double gT0[3], gT1[3];
#pragma unroll
        for (int c = 0; c < 3; ++c) {
            gT0[c] = 2.0 * ga * ST0[c] + gb * ST1[c];
            gT1[c] = gb * ST0[c] + 2.0 * gc * ST1[c];
        }
        const double gJ00 = gT0[0] * cam.R[0] + gT0[1] * cam.R[1] + gT0[2] * cam.R[2];
        const double gJ02 = gT0[0] * cam.R[6] + gT0[1] * cam.R[7] + gT0[2] * cam.R[8];
        const double gJ11 = gT1[0] * cam.R[3] + gT1[1] * cam.R[4] + gT1[2] * cam.R[5];
        const double gJ12 = gT1[0] * cam.R[6] + gT1[1] * cam.R[7] + gT1[2] * cam.R[8];
        gpc[0] = double(gxy.x) * fx * iz;
        gpc[1] = double(gxy.y) * fy * iz;
        gpc[2] = -(double(gxy.x) * fx * pc[0] + double(gxy.y) * fy * pc[1]) * iz * iz;
        gpc[2] += -(gJ00 * fx + gJ11 * fy) * iz * iz;
        if (clx) {
            gpc[2] += gJ02 * fx * txz * iz * iz;
        } else {
            gpc[0] += -gJ02 * fx * iz * iz;
            gpc[2] += gJ02 * 2.0 * fx * pc[0] * iz * iz * iz;
        }
        if (cly) {
            gpc[2] += gJ12 * fy * tyz * iz * iz;
        } else {
            gpc[1] += -gJ12 * fy * iz * iz;
            gpc[2] += gJ12 * 2.0 * fy * pc[1] * iz * iz * iz;
        }
    }
#pragma unroll
    for (int c = 0; c < 3; ++c)
        o.gmu_p[c] = double(cam.R[c]) * gpc[0] + double(cam.R[3 + c]) * gpc[1] + double(cam.R[6 + c]) * gpc[2];
    o.glogit = double(gco.w) * do_dlogit;

    // colour: SH of the unit viewing direction (float); the sign of the raw colour
    // decides the clamp and is re-taken in double when close to 0
    const double dvx = mu[0] - cam.cc[0], dvy = mu[1] - cam.cc[1], dvz = mu[2] - cam.cc[2];
    const double dn = sqrt(dvx * dvx + dvy * dvy + dvz * dvz);
    const double idn = 1.0 / dn;  // one division for the six uses below
    const double ux = dvx * idn, uy = dvy * idn, uz = dvz * idn;
    const float fx3 = float(ux), fy3 = float(uy), fz3 = float(uz);
    sh_basis<float>(deg, fx3, fy3, fz3, o.Y);
    float raw[3] = {0.5f, 0.5f, 0.5f};
#pragma unroll
    for (int k = 0; k < 16; ++k)
        if (k < nc) {
            raw[0] = fmaf(sh(3 * k + 0), o.Y[k], raw[0]);
            raw[1] = fmaf(sh(3 * k + 1), o.Y[k], raw[1]);
            raw[2] = fmaf(sh(3 * k + 2), o.Y[k], raw[2]);
        }
    if (fabsf(raw[0]) < 1e-5f || fabsf(raw[1]) < 1e-5f || fabsf(raw[2]) < 1e-5f) {
        double Yd[16];
        sh_basis<double>(deg, ux, uy, uz, Yd);
        double rd[3] = {0.5, 0.5, 0.5};
        for (int k = 0; k < nc; ++k)
            for (int ch = 0; ch < 3; ++ch) rd[ch] += double(sh(3 * k + ch)) * Yd[k];
        for (int ch = 0; ch < 3; ++ch) raw[ch] = rd[ch] < 0.0 ? -1.f : 1.f;
    }
    o.gcol[0] = raw[0] < 0.f ? 0.f : grg.x;
    o.gcol[1] = raw[1] < 0.f ? 0.f : grg.y;
    o.gcol[2] = raw[2] < 0.f ? 0.f : grg.z;
    float wk[16];
#pragma unroll
    for (int k = 0; k < 16; ++k)
        wk[k] = k < nc ? sh(3 * k) * o.gcol[0] + sh(3 * k + 1) * o.gcol[1] + sh(3 * k + 2) * o.gcol[2] : 0.f;
    float gdir[3] = {0.f, 0.f, 0.f};
    sh_grad_dir(deg, fx3, fy3, fz3, wk, gdir);
    const double dproj = gdir[0] * ux + gdir[1] * uy + gdir[2] * uz;
    o.gmu_c[0] = (gdir[0] - ux * dproj) * idn;
    o.gmu_c[1] = (gdir[1] - uy * dproj) * idn;
    o.gmu_c[2] = (gdir[2] - uz * dproj) * idn;
    o.dnorm = sqrtf(sxy.x * sxy.x + sxy.y * sxy.y);
}

// The view-independent part of a Gaussian: normalised quaternion, scales,
// Sigma = M M^T with M = R(q) diag(exp(log_scale)), and dsigmoid/dlogit.
struct Gauss3 {
    double qv[4], s3[3], qn, S6[6], do_dlogit;
};

__device__ __forceinline__ void rotation(const double q[4], double Rq[3][3]) {
    const double w = q[0], x = q[1], y = q[2], z = q[3];
    Rq[0][0] = 1.0 - 2.0 * (y * y + z * z); Rq[0][1] = 2.0 * (x * y - w * z); Rq[0][2] = 2.0 * (x * z + w * y);
    Rq[1][0] = 2.0 * (x * y + w * z); Rq[1][1] = 1.0 - 2.0 * (x * x + z * z); Rq[1][2] = 2.0 * (y * z - w * x);
    Rq[2][0] = 2.0 * (x * z - w * y); Rq[2][1] = 2.0 * (y * z + w * x); Rq[2][2] = 1.0 - 2.0 * (x * x + y * y);
}

__device__ __forceinline__ Gauss3 gauss3(float4 q4, float4 s4, double logit) {
    Gauss3 g;
    g.qn = sqrt(((double(q4.x) * q4.x + double(q4.y) * q4.y) + double(q4.z) * q4.z) + double(q4.w) * q4.w);
    g.qv[0] = q4.x / g.qn; g.qv[1] = q4.y / g.qn; g.qv[2] = q4.z / g.qn; g.qv[3] = q4.w / g.qn;
    g.s3[0] = exp(double(s4.x)); g.s3[1] = exp(double(s4.y)); g.s3[2] = exp(double(s4.z));
    double Rq[3][3];
    rotation(g.qv, Rq);
    double M[3][3];
#pragma unroll
    for (int r = 0; r < 3; ++r)
#pragma unroll
        for (int c = 0; c < 3; ++c) M[r][c] = Rq[r][c] * g.s3[c];
    const int rr[6] = {0, 0, 0, 1, 1, 2}, cc6[6] = {0, 1, 2, 1, 2, 2};
#pragma unroll
    for (int e = 0; e < 6; ++e)
        g.S6[e] = M[rr[e]][0] * M[cc6[e]][0] + M[rr[e]][1] * M[cc6[e]][1] + M[rr[e]][2] * M[cc6[e]][2];
    const double o = 1.0 / (1.0 + exp(-logit));
    g.do_dlogit = o * (1.0 - o);
    return g;
}

// Sigma = M M^T, M = Rq diag(s): dL/dM = 2 G M with G = dL/dSigma (symmetric), then
// the log-scales and the (unnormalised) quaternion.
__device__ __forceinline__ void sigma_chain(const Gauss3& g, const double gS[6], double gls[3], double gq[4]) {
    const double w = g.qv[0], x = g.qv[1], y = g.qv[2], z = g.qv[3];
    double Rq[3][3];
    rotation(g.qv, Rq);
    const double G[3][3] = {{gS[0], gS[1], gS[2]}, {gS[1], gS[3], gS[4]}, {gS[2], gS[4], gS[5]}};
    double gR[3][3];
#pragma unroll
    for (int c = 0; c < 3; ++c) {
        double acc = 0.0;
#pragma unroll
        for (int r = 0; r < 3; ++r) {
            const double gM = 2.0 * g.s3[c] * (G[r][0] * Rq[0][c] + G[r][1] * Rq[1][c] + G[r][2] * Rq[2][c]);
            acc += gM * Rq[r][c];
            gR[r][c] = gM * g.s3[c];
        }
        gls[c] = acc * g.s3[c];
    }
    const double gw = 2.0 * (-z * gR[0][1] + y * gR[0][2] + z * gR[1][0] - x * gR[1][2] - y * gR[2][0] + x * gR[2][1]);
    const double gx = 2.0 * (y * gR[0][1] + z * gR[0][2] + y * gR[1][0] - 2.0 * x * gR[1][1] - w * gR[1][2] +
                             z * gR[2][0] + w * gR[2][1] - 2.0 * x * gR[2][2]);
    const double gy = 2.0 * (-2.0 * y * gR[0][0] + x * gR[0][1] + w * gR[0][2] + x * gR[1][0] + z * gR[1][2] -
                             w * gR[2][0] + z * gR[2][1] - 2.0 * y * gR[2][2]);
    const double gz = 2.0 * (-2.0 * z * gR[0][0] - w * gR[0][1] + x * gR[0][2] + w * gR[1][0] - 2.0 * z * gR[1][1] +
                             y * gR[1][2] + x * gR[2][0] + y * gR[2][1]);
    const double qd = w * gw + x * gx + y * gy + z * gz;
    gq[0] = (gw - w * qd) / g.qn;
    gq[1] = (gx - x * qd) / g.qn;
    gq[2] = (gy - y * qd) / g.qn;
    gq[3] = (gz - z * qd) / g.qn;
}

// A gradient output element: added to (gs_project_bwd*) or written over (the
// Adam calls, whose buffer holds the step's gradient only).
__device__ __forceinline__ void out4(const Args& a, float4* d, int64_t i, float4 g) {
    if (a.overwrite)
        d[i] = g;
    else
        add4(d, i, g);
}

// Gradient outputs (when given) and the Adam step of one parameter group of a
// Gaussian: group 0 the means, 1 the quaternion, 2 the log-scales.
template <bool kAdam>
__device__ __forceinline__ void apply_group(const Args& a, int64_t i, int group, float4 g) {
    float4* d = group == 0 ? a.d_means : group == 1 ? a.d_quats : a.d_log_scales;
    if (a.d_means) out4(a, d, i, g);
    if (kAdam) {
        float4* p = group == 0 ? a.p_means : group == 1 ? a.p_quats : a.p_log_scales;
        float4* m = group == 0 ? a.m_means : group == 1 ? a.m_quats : a.m_log_scales;
        float4* v = group == 0 ? a.v_means : group == 1 ? a.v_quats : a.v_log_scales;
        AdamElem e = adam_load(p, m, v, i);
        adam_apply(e, make_float4(g.x, g.y, g.z, group == 0 ? 0.f : g.w), a.lr_t[group], a);
        adam_store(p, m, v, i, e);
    }
}

template <bool kAdam>
__device__ __forceinline__ void apply_logit(const Args& a, int64_t i, float g) {
    if (a.d_means) {
        if (a.overwrite)
            a.d_logits[i] = g;
        else
            a.d_logits[i] += g;
    }
    if (kAdam) {
        float mm = a.m_logits[i], vv = a.v_logits[i];
        a.p_logits[i] = adam_one(a.p_logits[i], g, mm, vv, a.lr_t[3], a);
        a.m_logits[i] = mm;
        a.v_logits[i] = vv;
    }
}

template <bool kAdam, bool kHalf>
__device__ __forceinline__ void apply_sh_plane(const Args& a, int64_t i, int p, float4 g) {
    const int64_t e = int64_t(p) * a.n + i;
    if (a.d_means) out4(a, a.d_sh, e, g);
    if (kAdam) {
        AdamElem x = adam_load(a.p_sh, a.m_sh, a.v_sh, e);
        adam_apply(x, g, a.lr_t[4], a);
        adam_store(a.p_sh, a.m_sh, a.v_sh, e, x);
        if (kHalf) a.sh_half_out[e] = narrow(x.p);
    }
}

// A Gaussian seen by no view in a call that writes its gradient over the buffer.
__device__ __forceinline__ void write_zero_grads(const Args& a, int64_t i) {
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    a.d_means[i] = z;
    a.d_quats[i] = z;
    a.d_log_scales[i] = z;
    a.d_logits[i] = 0.f;
    for (int p = 0; p < a.planes; ++p) a.d_sh[int64_t(p) * a.n + i] = z;
}

template <bool kHalf>
__device__ __forceinline__ float4 load_sh_plane(const Args& a, int p, int64_t i) {
    return kHalf ? widen(__ldg(a.sh_half + int64_t(p) * a.n + i)) : __ldg(a.sh + int64_t(p) * a.n + i);
}

// ---------------------------------------------------------------------------
// One or two views (kSplitMaxViews): one thread per Gaussian.  The view loop adds
// each view's terms to dL/dSigma, dL/dmean and dL/dlogit; the 48 SH gradient sums
// are formed in a second pass over the visible views from the masked colour
// gradients kept in shared memory, after the geometric chain has released its
// registers (4 blocks per SM).
constexpr int kSplitMaxViews = GS_ADAM_ONE_PASS_MAX_VIEWS;

template <bool kAdam, bool kPacked, bool kHalf>
__global__ void __launch_bounds__(kBwdBlock, 4) project_bwd_split_kernel(const __grid_constant__ Args a) {
    __shared__ float shs[48][kBwdBlock];                  // this thread's SH coefficients, column threadIdx.x
    __shared__ float gcs[3 * kSplitMaxViews][kBwdBlock];  // its masked colour gradient of every view
    __shared__ float smu[3][kBwdBlock];                   // its mean before the step
    const int t = threadIdx.x;
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + t; i < a.n; i += int64_t(gridDim.x) * blockDim.x) {
        unsigned vis = 0u;
        int rmax = 0;
        for (int v = 0; v < a.V; ++v) {
            const int64_t j = entry<kPacked>(a.view[v], i);
            const int r = j >= 0 ? __ldg(a.view[v].radius + j) : 0;
            if (r > 0) vis |= 1u << v;
            rmax = max(rmax, r);
        }
        if ((!kAdam || a.sparse) && vis == 0u) {  // nothing to add (sparse Adam: nothing to update)
            if (a.overwrite && a.d_means) write_zero_grads(a, i);
            continue;
        }
        if (a.densify_max_radius && rmax > a.densify_max_radius[i]) a.densify_max_radius[i] = rmax;
        if (kAdam) {
            // the moments, read after the long double-precision chain, start moving into L2 now
            asm volatile("prefetch.global.L2 [%0];" ::"l"(a.m_means + i));
            asm volatile("prefetch.global.L2 [%0];" ::"l"(a.v_means + i));
            asm volatile("prefetch.global.L2 [%0];" ::"l"(a.m_quats + i));
            asm volatile("prefetch.global.L2 [%0];" ::"l"(a.v_quats + i));
            asm volatile("prefetch.global.L2 [%0];" ::"l"(a.m_log_scales + i));
            asm volatile("prefetch.global.L2 [%0];" ::"l"(a.v_log_scales + i));
            for (int p = 0; p < a.planes; ++p) {
                asm volatile("prefetch.global.L2 [%0];" ::"l"(a.m_sh + int64_t(p) * a.n + i));
                asm volatile("prefetch.global.L2 [%0];" ::"l"(a.v_sh + int64_t(p) * a.n + i));
            }
        }
        double gS[6] = {0, 0, 0, 0, 0, 0};
        double gmu[3] = {0, 0, 0};
        double glogit = 0.0;
        float dacc = 0.f;
        int dcnt = 0;
        const int nc = (a.deg + 1) * (a.deg + 1);
        Gauss3 g3;
        if (vis) {
            const float4 m4 = __ldg(a.means + i);
            const double mu[3] = {m4.x, m4.y, m4.z};
            smu[0][t] = m4.x;
            smu[1][t] = m4.y;
            smu[2][t] = m4.z;
            for (int p = 0; p < a.planes; ++p) {
                const float4 c4 = load_sh_plane<kHalf>(a, p, i);
                shs[4 * p + 0][t] = c4.x;
                shs[4 * p + 1][t] = c4.y;
                shs[4 * p + 2][t] = c4.z;
                shs[4 * p + 3][t] = c4.w;
            }
            g3 = gauss3(__ldg(a.quats + i), __ldg(a.log_scales + i), __ldg(a.logits + i));
            const auto sh = [&](int q) { return shs[q][t]; };
            for (unsigned rest = vis; rest; rest &= rest - 1u) {
                const int v = __ffs(rest) - 1;
                const ViewArgs& cam = a.view[v];
                const int64_t j = entry<kPacked>(cam, i);
                const float2 gxy = __ldg(cam.g_xy + j);
                const float2 sxy = cam.g_xy_abs ? __ldg(cam.g_xy_abs + j) : gxy;
                ViewTerms o;
                view_terms(cam, mu, g3.S6, g3.do_dlogit, a.deg, nc, sh, gxy, __ldg(cam.g_con + j),
                           __ldg(cam.g_rgb + j), sxy, o);
#pragma unroll
                for (int e = 0; e < 6; ++e) gS[e] += o.gS[e];
#pragma unroll
                for (int c = 0; c < 3; ++c) gmu[c] += o.gmu_p[c];
                glogit += o.glogit;
#pragma unroll
                for (int c = 0; c < 3; ++c) gcs[3 * v + c][t] = o.gcol[c];
#pragma unroll
                for (int c = 0; c < 3; ++c) gmu[c] += o.gmu_c[c];
                dacc += o.dnorm;
                dcnt += 1;
            }
        }
        double gls[3] = {0, 0, 0}, gq[4] = {0, 0, 0, 0};
        if (vis) sigma_chain(g3, gS, gls, gq);
        apply_group<kAdam>(a, i, 0, make_float4(float(gmu[0]), float(gmu[1]), float(gmu[2]),
                                                a.overwrite ? float(__popc(vis)) : 0.f));
        apply_group<kAdam>(a, i, 1, make_float4(float(gq[0]), float(gq[1]), float(gq[2]), float(gq[3])));
        apply_group<kAdam>(a, i, 2, make_float4(float(gls[0]), float(gls[1]), float(gls[2]), 0.f));
        apply_logit<kAdam>(a, i, float(glogit));
        // the SH pass: dL/dc_k = sum over the visible views of Y_k(direction) x the masked
        // colour gradient, the basis recomputed as in the first pass from the mean as it
        // was before this step (the Adam step above has already overwritten it)
        float gsh[48];
#pragma unroll
        for (int k = 0; k < 48; ++k) gsh[k] = 0.f;
        if (vis) {
            const double mu[3] = {smu[0][t], smu[1][t], smu[2][t]};
            for (unsigned rest = vis; rest; rest &= rest - 1u) {
                const int v = __ffs(rest) - 1;
                const ViewArgs& cam = a.view[v];
                const double dvx = mu[0] - cam.cc[0], dvy = mu[1] - cam.cc[1], dvz = mu[2] - cam.cc[2];
                const double dn = sqrt(dvx * dvx + dvy * dvy + dvz * dvz);
                const double idn = 1.0 / dn;  // the direction exactly as the first pass formed it
                float Y[16];
                sh_basis<float>(a.deg, float(dvx * idn), float(dvy * idn), float(dvz * idn), Y);
                const float gcol[3] = {gcs[3 * v][t], gcs[3 * v + 1][t], gcs[3 * v + 2][t]};
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    if (k < nc) {
                        gsh[3 * k + 0] = fmaf(Y[k], gcol[0], gsh[3 * k + 0]);
                        gsh[3 * k + 1] = fmaf(Y[k], gcol[1], gsh[3 * k + 1]);
                        gsh[3 * k + 2] = fmaf(Y[k], gcol[2], gsh[3 * k + 2]);
                    }
                }
            }
        }
#pragma unroll
        for (int p = 0; p < 12; ++p)
            if (p < a.planes)
                apply_sh_plane<kAdam, kHalf>(a, i, p, make_float4(gsh[4 * p], gsh[4 * p + 1], gsh[4 * p + 2], gsh[4 * p + 3]));
        if (a.densify_accum && dcnt) {
            a.densify_accum[i] += dacc;
            a.densify_count[i] += dcnt;
        }
    }
}

// ---------------------------------------------------------------------------
// Three to 16 views: one thread per Gaussian, the visible views in a loop (the
// next view's 2D gradients loaded while the current one is processed), the 48 SH
// gradient sums accumulated view by view in shared memory.  The gradient is the
// kernel's only output: with Adam it is written to the caller's gradient buffer
// and the Adam step follows as its own launch (adam_groups_kernel), which keeps
// the parameter and moment traffic out of this latency-bound chain.
#ifndef GS_PBWD_MIN_BLOCKS
#define GS_PBWD_MIN_BLOCKS 3
#endif

template <bool kPacked, bool kHalf>
__global__ void __launch_bounds__(kBwdBlock, GS_PBWD_MIN_BLOCKS) project_bwd_loop_kernel(const __grid_constant__ Args a) {
    __shared__ float shs[48][kBwdBlock];  // this thread's SH coefficients, column threadIdx.x
    __shared__ float gcs[48][kBwdBlock];  // its 48 SH gradient sums
    const int t = threadIdx.x;
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + t; i < a.n; i += int64_t(gridDim.x) * blockDim.x) {
        unsigned vis = 0u;
        int rmax = 0;
        for (int v = 0; v < a.V; ++v) {
            const int64_t j = entry<kPacked>(a.view[v], i);
            const int r = j >= 0 ? __ldg(a.view[v].radius + j) : 0;
            if (r > 0) vis |= 1u << v;
            rmax = max(rmax, r);
        }
        if (vis == 0u) {  // no view sees it: nothing to add, or a zero gradient to write
            if (a.overwrite && a.d_means) write_zero_grads(a, i);
            continue;
        }
        if (a.densify_max_radius && rmax > a.densify_max_radius[i]) a.densify_max_radius[i] = rmax;
        // the visible views' 2D gradients start moving into L2 now
        for (unsigned rest = vis; rest; rest &= rest - 1u) {
            const ViewArgs& w = a.view[__ffs(rest) - 1];
            const int64_t j = entry<kPacked>(w, i);
            asm volatile("prefetch.global.L2 [%0];" ::"l"(w.g_xy + j));
            asm volatile("prefetch.global.L2 [%0];" ::"l"(w.g_con + j));
            asm volatile("prefetch.global.L2 [%0];" ::"l"(w.g_rgb + j));
        }
        double gS[6] = {0, 0, 0, 0, 0, 0};
        double gmu[3] = {0, 0, 0};
        double glogit = 0.0;
        float dacc = 0.f;
        const int nc = (a.deg + 1) * (a.deg + 1);
#pragma unroll
        for (int k = 0; k < 48; ++k) gcs[k][t] = 0.f;
        const float4 m4 = __ldg(a.means + i);
        const double mu[3] = {m4.x, m4.y, m4.z};
        for (int p = 0; p < a.planes; ++p) {
            const float4 c4 = load_sh_plane<kHalf>(a, p, i);
            shs[4 * p + 0][t] = c4.x;
            shs[4 * p + 1][t] = c4.y;
            shs[4 * p + 2][t] = c4.z;
            shs[4 * p + 3][t] = c4.w;
        }
        const Gauss3 g3 = gauss3(__ldg(a.quats + i), __ldg(a.log_scales + i), __ldg(a.logits + i));
        const auto sh = [&](int q) { return shs[q][t]; };
        int v = __ffs(vis) - 1;
        int64_t nj = entry<kPacked>(a.view[v], i);
        float2 nxy = __ldg(a.view[v].g_xy + nj);
        float4 nco = __ldg(a.view[v].g_con + nj);
        float4 nrg = __ldg(a.view[v].g_rgb + nj);
        while (v >= 0) {
            const ViewArgs& cam = a.view[v];
            const float2 gxy = nxy;
            const float4 gco = nco;
            const float4 grg = nrg;
            const int64_t cj = nj;
            const unsigned rest = vis & ~((2u << v) - 1u);
            const int vn = rest ? __ffs(rest) - 1 : -1;
            if (vn >= 0) {
                nj = entry<kPacked>(a.view[vn], i);
                nxy = __ldg(a.view[vn].g_xy + nj);
                nco = __ldg(a.view[vn].g_con + nj);
                nrg = __ldg(a.view[vn].g_rgb + nj);
            }
            const float2 sxy = cam.g_xy_abs ? __ldg(cam.g_xy_abs + cj) : gxy;
            ViewTerms o;
            view_terms(cam, mu, g3.S6, g3.do_dlogit, a.deg, nc, sh, gxy, gco, grg, sxy, o);
#pragma unroll
            for (int e = 0; e < 6; ++e) gS[e] += o.gS[e];
#pragma unroll
            for (int c = 0; c < 3; ++c) gmu[c] += o.gmu_p[c];
            glogit += o.glogit;
#pragma unroll
            for (int k = 0; k < 16; ++k) {
                if (k < nc) {
                    gcs[3 * k + 0][t] = fmaf(o.Y[k], o.gcol[0], gcs[3 * k + 0][t]);
                    gcs[3 * k + 1][t] = fmaf(o.Y[k], o.gcol[1], gcs[3 * k + 1][t]);
                    gcs[3 * k + 2][t] = fmaf(o.Y[k], o.gcol[2], gcs[3 * k + 2][t]);
                }
            }
#pragma unroll
            for (int c = 0; c < 3; ++c) gmu[c] += o.gmu_c[c];
            dacc += o.dnorm;
            v = vn;
        }
        double gls[3], gq[4];
        sigma_chain(g3, gS, gls, gq);
        const float4 gm = make_float4(float(gmu[0]), float(gmu[1]), float(gmu[2]), a.overwrite ? float(__popc(vis)) : 0.f);
        out4(a, a.d_means, i, gm);
        out4(a, a.d_quats, i, make_float4(float(gq[0]), float(gq[1]), float(gq[2]), float(gq[3])));
        out4(a, a.d_log_scales, i, make_float4(float(gls[0]), float(gls[1]), float(gls[2]), 0.f));
        if (a.overwrite)
            a.d_logits[i] = float(glogit);
        else
            a.d_logits[i] += float(glogit);
#pragma unroll
        for (int p = 0; p < 12; ++p)
            if (p < a.planes)
                out4(a, a.d_sh, int64_t(p) * a.n + i, make_float4(gcs[4 * p][t], gcs[4 * p + 1][t], gcs[4 * p + 2][t], gcs[4 * p + 3][t]));
        if (a.densify_accum) {
            a.densify_accum[i] += dacc;
            a.densify_count[i] += __popc(vis);
        }
    }
}

// ---------------------------------------------------------------------------
// The Adam step of all five groups in one launch, from the step's gradient
// (gsplat guide §4.2; the arithmetic of adam_one).  Block row y takes group y:
// means, quaternions, log-scales and the SH planes as float4 elements, the logits
// as floats.  Sparse: an element whose Gaussian no view saw (visible-view count 0
// in the w lane of its means gradient) keeps its parameter and moments.
struct AdamGroups {
    float4* p[5];
    float4* m[5];
    float4* v[5];
    const float4* g[5];
    int64_t count[5];  // elements of the group (float4s; floats for the logits, group 3)
    float lr_t[5];
    float inv_sqrt_bc2, b1, b2, eps;
    int64_t n;
    uint2* sh_half_out;  // kHalf: the updated SH rounded to 16 bits
};

__device__ __forceinline__ float adam_scalar(float p, float g, float& m, float& v, float lr_t, const AdamGroups& a) {
    m = a.b1 * m + (1.f - a.b1) * g;
    v = a.b2 * v + (1.f - a.b2) * (g * g);
    return p - lr_t * m / (sqrtf(v) * a.inv_sqrt_bc2 + a.eps);
}

template <bool kSparse, bool kHalf>
__global__ void __launch_bounds__(256) adam_groups_kernel(const __grid_constant__ AdamGroups a) {
    const int gr = blockIdx.y;
    const int64_t count = a.count[gr];
    const float lr_t = a.lr_t[gr];
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    if (gr == 3) {  // logits: one float per Gaussian
        float* p = reinterpret_cast<float*>(a.p[3]);
        float* m = reinterpret_cast<float*>(a.m[3]);
        float* v = reinterpret_cast<float*>(a.v[3]);
        const float* g = reinterpret_cast<const float*>(a.g[3]);
        for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < count; i += stride) {
            if (kSparse && __ldg(a.g[0] + i).w == 0.f) continue;
            float mm = m[i], vv = v[i];
            p[i] = adam_scalar(p[i], __ldg(g + i), mm, vv, lr_t, a);
            m[i] = mm;
            v[i] = vv;
        }
        return;
    }
    // two elements a thread per trip, every load before the first store: more bytes in
    // flight per thread (one element a trip ran at 66-68% of the DRAM peak)
    for (int64_t i0 = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i0 < count; i0 += 2 * stride) {
        float4 pp[2], mm[2], vv[2], gg[2];
        bool on[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int64_t i = i0 + u * stride;
            on[u] = i < count && !(kSparse && __ldg(a.g[0] + (gr == 4 ? i % a.n : i)).w == 0.f);
            if (on[u]) {
                pp[u] = a.p[gr][i];
                mm[u] = a.m[gr][i];
                vv[u] = a.v[gr][i];
                gg[u] = __ldg(a.g[gr] + i);
            }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            if (!on[u]) continue;
            const int64_t i = i0 + u * stride;
            if (gr == 0) gg[u].w = 0.f;  // the means' w lane carries the visible-view count
            pp[u].x = adam_scalar(pp[u].x, gg[u].x, mm[u].x, vv[u].x, lr_t, a);
            pp[u].y = adam_scalar(pp[u].y, gg[u].y, mm[u].y, vv[u].y, lr_t, a);
            pp[u].z = adam_scalar(pp[u].z, gg[u].z, mm[u].z, vv[u].z, lr_t, a);
            pp[u].w = adam_scalar(pp[u].w, gg[u].w, mm[u].w, vv[u].w, lr_t, a);
            a.p[gr][i] = pp[u];
            a.m[gr][i] = mm[u];
            a.v[gr][i] = vv[u];
            if (kHalf && gr == 4) a.sh_half_out[i] = narrow(pp[u]);
        }
    }
}

// Calls f with the compile-time form of the run-time flags (Adam, packed layout,
// half SH), for the combinations the entry points use.
template <class F>
void dispatch_flags(bool adam, bool packed, bool half, F&& f) {
    using T = std::true_type;
    using N = std::false_type;
    if (adam) {
        if (half)
            f(T{}, N{}, T{});
        else if (packed)
            f(T{}, T{}, N{});
        else
            f(T{}, N{}, N{});
    } else if (packed) {
        f(N{}, T{}, N{});
    } else {
        f(N{}, N{}, N{});
    }
}

void fill_views(Args& a, const CamArgs* cams, const gs_projected* projs, const int32_t* const* slots,
                const gs_grad2d* g2d, int V, const gs_camera* raw) {
    a.V = V;
    for (int v = 0; v < V; ++v) {
        ViewArgs& w = a.view[v];
        w.limx = cams[v].limx;
        w.limy = cams[v].limy;
        w.eps2d = cams[v].eps2d;
        for (int j = 0; j < 3; ++j) w.cc[j] = cams[v].cc[j];
        for (int j = 0; j < 9; ++j) w.R[j] = raw[v].R[j];
        for (int j = 0; j < 3; ++j) w.t[j] = raw[v].t[j];
        w.fx = raw[v].fx;
        w.fy = raw[v].fy;
        w.slot = slots ? slots[v] : nullptr;
        w.radius = projs[v].radius;
        w.g_xy = reinterpret_cast<const float2*>(g2d[v].xy);
        w.g_xy_abs = reinterpret_cast<const float2*>(g2d[v].xy_abs);
        w.g_con = reinterpret_cast<const float4*>(g2d[v].conic_opacity);
        w.g_rgb = reinterpret_cast<const float4*>(g2d[v].rgb);
    }
}

void fill_params(Args& a, const gs_params& p) {
    a.means = reinterpret_cast<const float4*>(p.means);
    a.quats = reinterpret_cast<const float4*>(p.quats);
    a.log_scales = reinterpret_cast<const float4*>(p.log_scales);
    a.logits = p.opacity_logits;
    a.sh = reinterpret_cast<const float4*>(p.sh);
    a.deg = p.sh_degree;
    a.planes = sh_planes(p.sh_degree);
    a.n = p.n;
}

void fill_grads(float4*& m, float4*& q, float4*& l, float*& o, float4*& s, const gs_param_grads* g) {
    m = g ? reinterpret_cast<float4*>(g->means) : nullptr;
    q = g ? reinterpret_cast<float4*>(g->quats) : nullptr;
    l = g ? reinterpret_cast<float4*>(g->log_scales) : nullptr;
    o = g ? g->opacity_logits : nullptr;
    s = g ? reinterpret_cast<float4*>(g->sh) : nullptr;
}

}  // namespace

cudaError_t launch_project_bwd_views(const gs_params& p, int V, const CamArgs* cams, const gs_camera* raw,
                                     const gs_projected* projs, const int32_t* const* slots, const gs_grad2d* g2d,
                                     const gs_param_grads* grads,
                                     float* densify_accum, int32_t* densify_count, int32_t* densify_max_radius,
                                     const AdamStep* adam, cudaStream_t s) {
    if (p.n == 0) return cudaSuccess;
    Args a;
    fill_params(a, p);
    fill_views(a, cams, projs, slots, g2d, V, raw);
    fill_grads(a.d_means, a.d_quats, a.d_log_scales, a.d_logits, a.d_sh, grads);
    a.densify_accum = densify_accum;
    a.densify_count = densify_count;
    a.densify_max_radius = densify_max_radius;
    a.sparse = adam && adam->sparse;
    if (adam) {
        fill_grads(a.p_means, a.p_quats, a.p_log_scales, a.p_logits, a.p_sh, adam->params);
        fill_grads(a.m_means, a.m_quats, a.m_log_scales, a.m_logits, a.m_sh, adam->m);
        fill_grads(a.v_means, a.v_quats, a.v_log_scales, a.v_logits, a.v_sh, adam->v);
        const double bc1 = 1.0 - pow(double(adam->beta1), double(adam->step));
        const double bc2 = 1.0 - pow(double(adam->beta2), double(adam->step));
        for (int g = 0; g < 5; ++g) a.lr_t[g] = float(double(adam->lr[g]) / bc1);
        a.inv_sqrt_bc2 = float(1.0 / sqrt(bc2));
        a.b1 = adam->beta1;
        a.b2 = adam->beta2;
        a.eps = adam->eps;
        a.sh_half = reinterpret_cast<const uint2*>(adam->sh_half);
        a.sh_half_out = reinterpret_cast<uint2*>(adam->sh_half_out);
    }
    const bool half = adam && adam->sh_half;
    // the Adam calls' gradient buffer receives the step's gradient (written over)
    a.overwrite = adam != nullptr;
    if (V <= kSplitMaxViews && !(adam && grads)) {
        // no views loop to speak of, and (with Adam) no buffer: the step in the same kernel
        const unsigned grid = grid_for(p.n, kBwdBlock, 16);
        dispatch_flags(adam != nullptr, slots != nullptr, half, [&](auto ad, auto pk, auto hf) {
            project_bwd_split_kernel<decltype(ad)::value, decltype(pk)::value, decltype(hf)::value>
                <<<grid, kBwdBlock, 0, s>>>(a);
        });
        count_launches(1);
        return cudaGetLastError();
    }
    // the gradient into the buffer, then the Adam launch
    const unsigned grid = grid_for(p.n, kBwdBlock, 16);
    if (V <= kSplitMaxViews) {
        if (slots)
            project_bwd_split_kernel<false, true, false><<<grid, kBwdBlock, 0, s>>>(a);
        else if (half)
            project_bwd_split_kernel<false, false, true><<<grid, kBwdBlock, 0, s>>>(a);
        else
            project_bwd_split_kernel<false, false, false><<<grid, kBwdBlock, 0, s>>>(a);
    } else if (slots)
        project_bwd_loop_kernel<true, false><<<grid, kBwdBlock, 0, s>>>(a);
    else if (half)
        project_bwd_loop_kernel<false, true><<<grid, kBwdBlock, 0, s>>>(a);
    else
        project_bwd_loop_kernel<false, false><<<grid, kBwdBlock, 0, s>>>(a);
    count_launches(1);
    if (adam) {
        AdamGroups g;
        float4* const ps[5] = {a.p_means, a.p_quats, a.p_log_scales, reinterpret_cast<float4*>(a.p_logits), a.p_sh};
        float4* const ms[5] = {a.m_means, a.m_quats, a.m_log_scales, reinterpret_cast<float4*>(a.m_logits), a.m_sh};
        float4* const vs[5] = {a.v_means, a.v_quats, a.v_log_scales, reinterpret_cast<float4*>(a.v_logits), a.v_sh};
        const float4* const gs[5] = {a.d_means, a.d_quats, a.d_log_scales, reinterpret_cast<const float4*>(a.d_logits),
                                     a.d_sh};
        for (int k = 0; k < 5; ++k) {
            g.p[k] = ps[k];
            g.m[k] = ms[k];
            g.v[k] = vs[k];
            g.g[k] = gs[k];
            g.lr_t[k] = a.lr_t[k];
        }
        g.count[0] = g.count[1] = g.count[2] = g.count[3] = p.n;
        g.count[4] = int64_t(a.planes) * p.n;
        g.inv_sqrt_bc2 = a.inv_sqrt_bc2;
        g.b1 = a.b1;
        g.b2 = a.b2;
        g.eps = a.eps;
        g.n = p.n;
        g.sh_half_out = a.sh_half_out;
        const dim3 agrid(grid_for(g.count[4], 256, 8), 5);
        if (a.sparse) {
            if (half)
                adam_groups_kernel<true, true><<<agrid, 256, 0, s>>>(g);
            else
                adam_groups_kernel<true, false><<<agrid, 256, 0, s>>>(g);
        } else {
            if (half)
                adam_groups_kernel<false, true><<<agrid, 256, 0, s>>>(g);
            else
                adam_groups_kernel<false, false><<<agrid, 256, 0, s>>>(g);
        }
        count_launches(1);
    }
    return cudaGetLastError();
}

}  // namespace gsk
