// gs_project_bwd, gs_project_bwd_views, gs_project_bwd_views_adam: chain the
// per-Gaussian 2D gradients of one or several views through the projection to
// the Gaussian parameters (the "gradients to position / covariance / colour /
// opacity" of one fused backward, MUSA co-design article qwbw.cn/news/278220
// §2.2), and optionally apply the Adam step of the gsplat guide
// (lmnt.cn/news/262699) §4.2 in the same pass.
//
// One thread per Gaussian.  The view-independent part (normalised quaternion,
// rotation, scales, M = R diag(s), Sigma = M M^T) is computed once; every view in
// which the Gaussian is visible then adds its contribution to dL/dSigma (6
// values), dL/dmean, dL/dlogit and the 48 SH gradients, all held in registers;
// the chain from dL/dSigma to the scales and the quaternion runs once at the end.
// With Adam fused the gradients never reach memory: parameters, moments and the
// views' 2D gradients each make exactly one pass through HBM.  For one or two
// views the 48 SH gradients are summed in a second pass over the visible views
// (their masked colour gradients kept in shared memory), which lets the kernel
// run at twice the occupancy.  In the packed
// layout (gs_project_packed) a view's features and 2D gradients are read at the
// Gaussian's slot, found through the view's slot map.  With 16-bit SH storage the
// colour chain takes the half-precision coefficients the forward pass used, Adam
// updates the float32 coefficients, and their rounding to half is written back.
//
// The geometric chain is double precision: the inverse of a 2x2 conic and the
// EWA product are badly conditioned for needle-shaped Gaussians.  The colour
// (SH) chain is float32 except the sign test of the raw colour, which repeats the
// forward pass's double-precision decision.
#include <cuda_fp16.h>

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
    bool sparse;  // Adam: leave Gaussians visible in no view untouched
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

__device__ __forceinline__ float4 adam4(float4* p, float4* m, float4* v, int64_t i, float4 g, float lr_t,
                                        const Args& a) {
    float4 pp = p[i], mm = m[i], vv = v[i];
    pp.x = adam_one(pp.x, g.x, mm.x, vv.x, lr_t, a);
    pp.y = adam_one(pp.y, g.y, mm.y, vv.y, lr_t, a);
    pp.z = adam_one(pp.z, g.z, mm.z, vv.z, lr_t, a);
    pp.w = adam_one(pp.w, g.w, mm.w, vv.w, lr_t, a);
    p[i] = pp;
    m[i] = mm;
    v[i] = vv;
    return pp;
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

#ifndef GS_PBWD_MIN_BLOCKS
#define GS_PBWD_MIN_BLOCKS 3
#endif
// Launches with at most this many views defer the SH gradient to a second pass
// (kSplit): the 48 accumulators then never share registers with the geometric
// chain, and the kernel runs at 4 blocks per SM instead of 2.  With many views the
// single pass is faster (the second pass recomputes every view's SH basis).
constexpr int kSplitMaxViews = 2;

template <bool kAdam, bool kPacked, bool kHalf, bool kSplit>
__global__ void __launch_bounds__(kBwdBlock, kSplit ? 4 : GS_PBWD_MIN_BLOCKS) project_bwd_kernel(const Args a) {
    __shared__ float shs[48][kBwdBlock];  // this thread's SH coefficients, column threadIdx.x
    // kSplit: this thread's masked colour gradient of every view, kept for the SH pass;
    // otherwise the 48 SH gradient sums, accumulated view by view in shared memory
    // rather than in registers (which keeps the one-pass kernel at 3 blocks per SM)
    __shared__ float gcs[kSplit ? 3 * kMaxViews : 48][kBwdBlock];
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
        if ((!kAdam || a.sparse) && vis == 0u) continue;  // nothing to add (sparse Adam: nothing to update)
        if (a.densify_max_radius && rmax > a.densify_max_radius[i]) a.densify_max_radius[i] = rmax;
#ifndef GS_PBWD_NO_PREFETCH
        // everything this Gaussian reads after the long double-precision chain (the
        // visible views' 2D gradients, the Adam moments) starts moving into L2 now
        for (unsigned rest = vis; rest; rest &= rest - 1u) {
            const ViewArgs& w = a.view[__ffs(rest) - 1];
            const int64_t j = entry<kPacked>(w, i);
            asm volatile("prefetch.global.L2 [%0];" ::"l"(w.g_xy + j));
            asm volatile("prefetch.global.L2 [%0];" ::"l"(w.g_con + j));
            asm volatile("prefetch.global.L2 [%0];" ::"l"(w.g_rgb + j));
        }
        if (kAdam) {
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
#endif

        double gS[6] = {0, 0, 0, 0, 0, 0};  // symmetric dL/dSigma: xx, xy, xz, yy, yz, zz
        double gmu[3] = {0, 0, 0};
        double glogit = 0.0;
        float gsh[kSplit ? 48 : 1];  // kSplit: the SH gradient sums (the second pass)
#pragma unroll
        for (int k = 0; k < (kSplit ? 48 : 1); ++k) gsh[k] = 0.f;
        if (!kSplit) {
#pragma unroll
            for (int k = 0; k < 48; ++k) gcs[k][t] = 0.f;
        }
        float dacc = 0.f;
        int dcnt = 0;
        double qv[4] = {1, 0, 0, 0}, s3[3] = {0, 0, 0}, qn = 1.0;
        const int nc = (a.deg + 1) * (a.deg + 1);

        if (vis) {
            const float4 m4 = __ldg(a.means + i);
            const float4 q4 = __ldg(a.quats + i);
            const float4 s4 = __ldg(a.log_scales + i);
            const double logit = __ldg(a.logits + i);
            const double mu[3] = {m4.x, m4.y, m4.z};
            for (int p = 0; p < a.planes; ++p) {
                const float4 c4 = kHalf ? widen(__ldg(a.sh_half + int64_t(p) * a.n + i))
                                        : __ldg(a.sh + int64_t(p) * a.n + i);
                shs[4 * p + 0][t] = c4.x;
                shs[4 * p + 1][t] = c4.y;
                shs[4 * p + 2][t] = c4.z;
                shs[4 * p + 3][t] = c4.w;
            }
            // ---- view-independent: Sigma = M M^T, M = R(q) diag(exp(log_scale))
            qn = sqrt(((double(q4.x) * q4.x + double(q4.y) * q4.y) + double(q4.z) * q4.z) + double(q4.w) * q4.w);
            qv[0] = q4.x / qn; qv[1] = q4.y / qn; qv[2] = q4.z / qn; qv[3] = q4.w / qn;
            s3[0] = exp(double(s4.x)); s3[1] = exp(double(s4.y)); s3[2] = exp(double(s4.z));
            double S6[6];
            {
                const double w = qv[0], x = qv[1], y = qv[2], z = qv[3];
                const double Rq[3][3] = {{1.0 - 2.0 * (y * y + z * z), 2.0 * (x * y - w * z), 2.0 * (x * z + w * y)},
                                         {2.0 * (x * y + w * z), 1.0 - 2.0 * (x * x + z * z), 2.0 * (y * z - w * x)},
                                         {2.0 * (x * z - w * y), 2.0 * (y * z + w * x), 1.0 - 2.0 * (x * x + y * y)}};
                double M[3][3];
#pragma unroll
                for (int r = 0; r < 3; ++r)
#pragma unroll
                    for (int c = 0; c < 3; ++c) M[r][c] = Rq[r][c] * s3[c];
                const int rr[6] = {0, 0, 0, 1, 1, 2}, cc6[6] = {0, 1, 2, 1, 2, 2};
#pragma unroll
                for (int e = 0; e < 6; ++e)
                    S6[e] = M[rr[e]][0] * M[cc6[e]][0] + M[rr[e]][1] * M[cc6[e]][1] + M[rr[e]][2] * M[cc6[e]][2];
            }
            const double o = 1.0 / (1.0 + exp(-logit));
            const double do_dlogit = o * (1.0 - o);

            // visible views in order; the next view's 2D gradients are loaded while
            // the current one is processed
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
                const double fx = cam.fx, fy = cam.fy;
                double pc[3];
#pragma unroll
                for (int r = 0; r < 3; ++r)
                    pc[r] = ((double(cam.R[3 * r]) * mu[0] + double(cam.R[3 * r + 1]) * mu[1]) +
                             double(cam.R[3 * r + 2]) * mu[2]) + double(cam.t[r]);
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
                const double ST0[3] = {S6[0] * T0[0] + S6[1] * T0[1] + S6[2] * T0[2],
                                       S6[1] * T0[0] + S6[3] * T0[1] + S6[4] * T0[2],
                                       S6[2] * T0[0] + S6[4] * T0[1] + S6[5] * T0[2]};
                const double ST1[3] = {S6[0] * T1[0] + S6[1] * T1[1] + S6[2] * T1[2],
                                       S6[1] * T1[0] + S6[3] * T1[1] + S6[4] * T1[2],
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
                // dL/dSigma += ga T0 T0^T + gb/2 (T0 T1^T + T1 T0^T) + gc T1 T1^T
                gS[0] += ga * T0[0] * T0[0] + gb * T0[0] * T1[0] + gc * T1[0] * T1[0];
                gS[1] += ga * T0[0] * T0[1] + 0.5 * gb * (T0[0] * T1[1] + T1[0] * T0[1]) + gc * T1[0] * T1[1];
                gS[2] += ga * T0[0] * T0[2] + 0.5 * gb * (T0[0] * T1[2] + T1[0] * T0[2]) + gc * T1[0] * T1[2];
                gS[3] += ga * T0[1] * T0[1] + gb * T0[1] * T1[1] + gc * T1[1] * T1[1];
                gS[4] += ga * T0[1] * T0[2] + 0.5 * gb * (T0[1] * T1[2] + T1[1] * T0[2]) + gc * T1[1] * T1[2];
                gS[5] += ga * T0[2] * T0[2] + gb * T0[2] * T1[2] + gc * T1[2] * T1[2];
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
                    gmu[c] += double(cam.R[c]) * gpc[0] + double(cam.R[3 + c]) * gpc[1] + double(cam.R[6 + c]) * gpc[2];
                glogit += double(gco.w) * do_dlogit;

                // colour: SH of the unit viewing direction (float); the sign of the raw
                // colour decides the clamp and is re-taken in double when close to 0
                const double dvx = mu[0] - cam.cc[0], dvy = mu[1] - cam.cc[1], dvz = mu[2] - cam.cc[2];
                const double dn = sqrt(dvx * dvx + dvy * dvy + dvz * dvz);
                const double idn = 1.0 / dn;  // one division for the six uses below
                const double ux = dvx * idn, uy = dvy * idn, uz = dvz * idn;
                const float fx3 = float(ux), fy3 = float(uy), fz3 = float(uz);
                float Y[16];
                sh_basis<float>(a.deg, fx3, fy3, fz3, Y);
                float raw[3] = {0.5f, 0.5f, 0.5f};
#pragma unroll
                for (int k = 0; k < 16; ++k)
                    if (k < nc) {
                        raw[0] = fmaf(shs[3 * k + 0][t], Y[k], raw[0]);
                        raw[1] = fmaf(shs[3 * k + 1][t], Y[k], raw[1]);
                        raw[2] = fmaf(shs[3 * k + 2][t], Y[k], raw[2]);
                    }
                if (fabsf(raw[0]) < 1e-5f || fabsf(raw[1]) < 1e-5f || fabsf(raw[2]) < 1e-5f) {
                    double Yd[16];
                    sh_basis<double>(a.deg, ux, uy, uz, Yd);
                    double rd[3] = {0.5, 0.5, 0.5};
                    for (int k = 0; k < nc; ++k)
                        for (int ch = 0; ch < 3; ++ch) rd[ch] += double(shs[3 * k + ch][t]) * Yd[k];
                    for (int ch = 0; ch < 3; ++ch) raw[ch] = rd[ch] < 0.0 ? -1.f : 1.f;
                }
                const float gcol[3] = {raw[0] < 0.f ? 0.f : grg.x, raw[1] < 0.f ? 0.f : grg.y,
                                       raw[2] < 0.f ? 0.f : grg.z};
                if (kSplit) {
                    gcs[3 * v + 0][t] = gcol[0];
                    gcs[3 * v + 1][t] = gcol[1];
                    gcs[3 * v + 2][t] = gcol[2];
                }
                float wk[16];
#pragma unroll
                for (int k = 0; k < 16; ++k) {
                    if (k < nc) {
                        const float s0 = shs[3 * k][t], s1 = shs[3 * k + 1][t], s2 = shs[3 * k + 2][t];
                        if (!kSplit) {
                            gcs[3 * k + 0][t] = fmaf(Y[k], gcol[0], gcs[3 * k + 0][t]);
                            gcs[3 * k + 1][t] = fmaf(Y[k], gcol[1], gcs[3 * k + 1][t]);
                            gcs[3 * k + 2][t] = fmaf(Y[k], gcol[2], gcs[3 * k + 2][t]);
                        }
                        wk[k] = s0 * gcol[0] + s1 * gcol[1] + s2 * gcol[2];
                    } else {
                        wk[k] = 0.f;
                    }
                }
                float gdir[3] = {0.f, 0.f, 0.f};
                sh_grad_dir(a.deg, fx3, fy3, fz3, wk, gdir);
                const double dproj = gdir[0] * ux + gdir[1] * uy + gdir[2] * uz;
                gmu[0] += (gdir[0] - ux * dproj) * idn;
                gmu[1] += (gdir[1] - uy * dproj) * idn;
                gmu[2] += (gdir[2] - uz * dproj) * idn;

                const float2 sxy = cam.g_xy_abs ? __ldg(cam.g_xy_abs + cj) : gxy;
                dacc += sqrtf(sxy.x * sxy.x + sxy.y * sxy.y);
                dcnt += 1;
                v = vn;
            }
        }

        // ---- Sigma = M M^T, M = Rq diag(s): dL/dM = 2 G M with G = dL/dSigma (symmetric)
        double gls[3] = {0, 0, 0}, gq[4] = {0, 0, 0, 0};
        if (vis) {
            const double w = qv[0], x = qv[1], y = qv[2], z = qv[3];
            const double Rq[3][3] = {{1.0 - 2.0 * (y * y + z * z), 2.0 * (x * y - w * z), 2.0 * (x * z + w * y)},
                                     {2.0 * (x * y + w * z), 1.0 - 2.0 * (x * x + z * z), 2.0 * (y * z - w * x)},
                                     {2.0 * (x * z - w * y), 2.0 * (y * z + w * x), 1.0 - 2.0 * (x * x + y * y)}};
            const double G[3][3] = {{gS[0], gS[1], gS[2]}, {gS[1], gS[3], gS[4]}, {gS[2], gS[4], gS[5]}};
            double gR[3][3];
#pragma unroll
            for (int c = 0; c < 3; ++c) {
                double acc = 0.0;
#pragma unroll
                for (int r = 0; r < 3; ++r) {
                    const double gM = 2.0 * s3[c] * (G[r][0] * Rq[0][c] + G[r][1] * Rq[1][c] + G[r][2] * Rq[2][c]);
                    acc += gM * Rq[r][c];
                    gR[r][c] = gM * s3[c];
                }
                gls[c] = acc * s3[c];
            }
            const double gw = 2.0 * (-z * gR[0][1] + y * gR[0][2] + z * gR[1][0] - x * gR[1][2] - y * gR[2][0] +
                                     x * gR[2][1]);
            const double gx = 2.0 * (y * gR[0][1] + z * gR[0][2] + y * gR[1][0] - 2.0 * x * gR[1][1] - w * gR[1][2] +
                                     z * gR[2][0] + w * gR[2][1] - 2.0 * x * gR[2][2]);
            const double gy = 2.0 * (-2.0 * y * gR[0][0] + x * gR[0][1] + w * gR[0][2] + x * gR[1][0] +
                                     z * gR[1][2] - w * gR[2][0] + z * gR[2][1] - 2.0 * y * gR[2][2]);
            const double gz = 2.0 * (-2.0 * z * gR[0][0] - w * gR[0][1] + x * gR[0][2] + w * gR[1][0] -
                                     2.0 * z * gR[1][1] + y * gR[1][2] + x * gR[2][0] + y * gR[2][1]);
            const double qd = w * gw + x * gx + y * gy + z * gz;
            gq[0] = (gw - w * qd) / qn;
            gq[1] = (gx - x * qd) / qn;
            gq[2] = (gy - y * qd) / qn;
            gq[3] = (gz - z * qd) / qn;
        }

        const float4 g_means = make_float4(float(gmu[0]), float(gmu[1]), float(gmu[2]), 0.f);
        const float4 g_quats = make_float4(float(gq[0]), float(gq[1]), float(gq[2]), float(gq[3]));
        const float4 g_ls = make_float4(float(gls[0]), float(gls[1]), float(gls[2]), 0.f);
        const float g_logit = float(glogit);
        if (a.d_means) {  // gradient outputs (+=)
            add4(a.d_means, i, g_means);
            add4(a.d_quats, i, g_quats);
            add4(a.d_log_scales, i, g_ls);
            a.d_logits[i] += g_logit;
        }
        if (kAdam) {
            adam4(a.p_means, a.m_means, a.v_means, i, g_means, a.lr_t[0], a);
            adam4(a.p_quats, a.m_quats, a.v_quats, i, g_quats, a.lr_t[1], a);
            adam4(a.p_log_scales, a.m_log_scales, a.v_log_scales, i, g_ls, a.lr_t[2], a);
            float mm = a.m_logits[i], vv = a.v_logits[i];
            a.p_logits[i] = adam_one(a.p_logits[i], g_logit, mm, vv, a.lr_t[3], a);
            a.m_logits[i] = mm;
            a.v_logits[i] = vv;
        }
        if (kSplit && vis) {
            // the SH pass, after the geometric chain has released its registers:
            // dL/dc_k = sum over the visible views of Y_k(direction) x the masked colour
            // gradient, the basis recomputed as in the first pass
            const float4 m4 = __ldg(a.means + i);
            const double mu[3] = {m4.x, m4.y, m4.z};
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
        // the SH gradient of plane p (four coefficients): from the registers of the
        // second pass, or from the shared-memory sums
        const auto sh_grad = [&](int p) {
            if (kSplit) return make_float4(gsh[4 * p], gsh[4 * p + 1], gsh[4 * p + 2], gsh[4 * p + 3]);
            return make_float4(gcs[4 * p][t], gcs[4 * p + 1][t], gcs[4 * p + 2][t], gcs[4 * p + 3][t]);
        };
        if (a.d_means) {
#pragma unroll
            for (int p = 0; p < 12; ++p)
                if (p < a.planes) add4(a.d_sh, int64_t(p) * a.n + i, sh_grad(p));
        }
        if (kAdam) {
#pragma unroll
            for (int p = 0; p < 12; ++p)
                if (p < a.planes)
                {
                    const float4 up = adam4(a.p_sh, a.m_sh, a.v_sh, int64_t(p) * a.n + i, sh_grad(p), a.lr_t[4], a);
                    if (kHalf) a.sh_half_out[int64_t(p) * a.n + i] = narrow(up);
                }
        }
        if (a.densify_accum && dcnt) {
            a.densify_accum[i] += dacc;
            a.densify_count[i] += dcnt;
        }
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
    const unsigned grid = grid_for(p.n, kBwdBlock, 16);
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
        if (adam->sh_half)
            project_bwd_kernel<true, false, true, false><<<grid, kBwdBlock, 0, s>>>(a);
        else if (slots)
            project_bwd_kernel<true, true, false, false><<<grid, kBwdBlock, 0, s>>>(a);
        else if (V <= kSplitMaxViews)
            project_bwd_kernel<true, false, false, true><<<grid, kBwdBlock, 0, s>>>(a);
        else
            project_bwd_kernel<true, false, false, false><<<grid, kBwdBlock, 0, s>>>(a);
    } else if (slots) {
        project_bwd_kernel<false, true, false, false><<<grid, kBwdBlock, 0, s>>>(a);
    } else if (V <= kSplitMaxViews) {
        project_bwd_kernel<false, false, false, true><<<grid, kBwdBlock, 0, s>>>(a);
    } else {
        project_bwd_kernel<false, false, false, false><<<grid, kBwdBlock, 0, s>>>(a);
    }
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace gsk
