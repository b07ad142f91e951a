// gs_project_bwd: chain the per-Gaussian 2D gradients through the projection to
// the Gaussian parameters (the "gradients to position / covariance / colour /
// opacity" of a single fused backward, MUSA co-design article
// qwbw.cn/news/278220 §2.2), in double precision.  Each thread recomputes its
// Gaussian's forward intermediates, so nothing but the projected radius is
// cached between the passes.  The inverse of a 2x2 conic and the EWA product are
// badly conditioned for needle-like Gaussians; double keeps the chain accurate.
#include "internal.cuh"

namespace gsk {
namespace {

constexpr double kY1 = 0.4886025119029199;
__constant__ double kY2[5] = {1.0925484305920792, -1.0925484305920792, 0.31539156525252005, -1.0925484305920792,
                           0.5462742152960396};
__constant__ double kY3[7] = {-0.5900435899266435, 2.890611442640554, -0.4570457994644658, 0.3731763325901154,
                           -0.4570457994644658, 1.445305721320277, -0.5900435899266435};
constexpr double kY0 = 0.28209479177387814;

struct BwdArgs {
    const float4* means;
    const float4* quats;
    const float4* log_scales;
    const float* logits;
    const float4* sh;
    int deg, planes;
    int64_t n;
    CamArgs cam;
    const int32_t* radius;
    const float2* g_xy;
    const float4* g_con;
    const float4* g_rgb;
    float4* d_means;
    float4* d_quats;
    float4* d_log_scales;
    float* d_logits;
    float4* d_sh;
    float* densify_accum;
    int32_t* densify_count;
};

// SH basis values and their gradients with respect to the (unit) direction.
__device__ void sh_basis_grad(int deg, double x, double y, double z, double* Y, double (*dY)[3]) {
    Y[0] = kY0;
    dY[0][0] = dY[0][1] = dY[0][2] = 0.0;
    if (deg < 1) return;
    Y[1] = -kY1 * y; dY[1][0] = 0.0;  dY[1][1] = -kY1; dY[1][2] = 0.0;
    Y[2] = kY1 * z;  dY[2][0] = 0.0;  dY[2][1] = 0.0;  dY[2][2] = kY1;
    Y[3] = -kY1 * x; dY[3][0] = -kY1; dY[3][1] = 0.0;  dY[3][2] = 0.0;
    if (deg < 2) return;
    const double xx = x * x, yy = y * y, zz = z * z;
    Y[4] = kY2[0] * x * y;            dY[4][0] = kY2[0] * y;         dY[4][1] = kY2[0] * x;         dY[4][2] = 0.0;
    Y[5] = kY2[1] * y * z;            dY[5][0] = 0.0;                dY[5][1] = kY2[1] * z;         dY[5][2] = kY2[1] * y;
    Y[6] = kY2[2] * (2 * zz - xx - yy); dY[6][0] = -2 * kY2[2] * x;  dY[6][1] = -2 * kY2[2] * y;    dY[6][2] = 4 * kY2[2] * z;
    Y[7] = kY2[3] * x * z;            dY[7][0] = kY2[3] * z;         dY[7][1] = 0.0;                dY[7][2] = kY2[3] * x;
    Y[8] = kY2[4] * (xx - yy);        dY[8][0] = 2 * kY2[4] * x;     dY[8][1] = -2 * kY2[4] * y;    dY[8][2] = 0.0;
    if (deg < 3) return;
    Y[9] = kY3[0] * y * (3 * xx - yy);
    dY[9][0] = kY3[0] * 6 * x * y;  dY[9][1] = kY3[0] * (3 * xx - 3 * yy);  dY[9][2] = 0.0;
    Y[10] = kY3[1] * x * y * z;
    dY[10][0] = kY3[1] * y * z;     dY[10][1] = kY3[1] * x * z;             dY[10][2] = kY3[1] * x * y;
    Y[11] = kY3[2] * y * (4 * zz - xx - yy);
    dY[11][0] = kY3[2] * (-2 * x * y); dY[11][1] = kY3[2] * (4 * zz - xx - 3 * yy); dY[11][2] = kY3[2] * 8 * y * z;
    Y[12] = kY3[3] * z * (2 * zz - 3 * xx - 3 * yy);
    dY[12][0] = kY3[3] * (-6 * x * z); dY[12][1] = kY3[3] * (-6 * y * z); dY[12][2] = kY3[3] * (6 * zz - 3 * xx - 3 * yy);
    Y[13] = kY3[4] * x * (4 * zz - xx - yy);
    dY[13][0] = kY3[4] * (4 * zz - 3 * xx - yy); dY[13][1] = kY3[4] * (-2 * x * y); dY[13][2] = kY3[4] * 8 * x * z;
    Y[14] = kY3[5] * z * (xx - yy);
    dY[14][0] = kY3[5] * 2 * x * z; dY[14][1] = kY3[5] * (-2 * y * z);      dY[14][2] = kY3[5] * (xx - yy);
    Y[15] = kY3[6] * x * (xx - 3 * yy);
    dY[15][0] = kY3[6] * (3 * xx - 3 * yy); dY[15][1] = kY3[6] * (-6 * x * y); dY[15][2] = 0.0;
}

__global__ void __launch_bounds__(128) project_bwd_kernel(const BwdArgs a) {
    const CamArgs& cam = a.cam;
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < a.n; i += int64_t(gridDim.x) * blockDim.x) {
        if (__ldg(a.radius + i) <= 0) continue;
        const float4 m4 = __ldg(a.means + i);
        const float4 q4 = __ldg(a.quats + i);
        const float4 s4 = __ldg(a.log_scales + i);
        const double logit = __ldg(a.logits + i);
        const float2 gxy = a.g_xy[i];
        const float4 gco = a.g_con[i];
        const float4 grg = a.g_rgb[i];
        const double mu[3] = {m4.x, m4.y, m4.z};

        // ---- forward recompute
        double pc[3];
        for (int r = 0; r < 3; ++r)
            pc[r] = ((cam.R[3 * r + 0] * mu[0] + cam.R[3 * r + 1] * mu[1]) + cam.R[3 * r + 2] * mu[2]) + cam.t[r];
        const double qn = sqrt(((double(q4.x) * q4.x + double(q4.y) * q4.y) + double(q4.z) * q4.z) + double(q4.w) * q4.w);
        const double w = q4.x / qn, x = q4.y / qn, y = q4.z / qn, z = q4.w / qn;
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
        const double s[3] = {exp(double(s4.x)), exp(double(s4.y)), exp(double(s4.z))};
        double M[3][3];
        for (int r = 0; r < 3; ++r)
            for (int c = 0; c < 3; ++c) M[r][c] = Rq[r][c] * s[c];
        double S[3][3];
        for (int r = 0; r < 3; ++r)
            for (int c = 0; c < 3; ++c) S[r][c] = M[r][0] * M[c][0] + M[r][1] * M[c][1] + M[r][2] * M[c][2];
        const double iz = 1.0 / pc[2];
        double txz = pc[0] * iz, tyz = pc[1] * iz;
        const bool clx = (txz < -cam.limx) || (txz > cam.limx);
        const bool cly = (tyz < -cam.limy) || (tyz > cam.limy);
        txz = fmin(fmax(txz, -cam.limx), cam.limx);
        tyz = fmin(fmax(tyz, -cam.limy), cam.limy);
        const double J00 = cam.fx * iz, J02 = -cam.fx * txz * iz;
        const double J11 = cam.fy * iz, J12 = -cam.fy * tyz * iz;
        const double* W0 = cam.R;
        const double* W1 = cam.R + 3;
        const double* W2 = cam.R + 6;
        double T0[3], T1[3];
        for (int c = 0; c < 3; ++c) {
            T0[c] = J00 * W0[c] + J02 * W2[c];
            T1[c] = J11 * W1[c] + J12 * W2[c];
        }
        double ST0[3], ST1[3];  // Sigma T0^T, Sigma T1^T
        for (int r = 0; r < 3; ++r) {
            ST0[r] = S[r][0] * T0[0] + S[r][1] * T0[1] + S[r][2] * T0[2];
            ST1[r] = S[r][0] * T1[0] + S[r][1] * T1[1] + S[r][2] * T1[2];
        }
        const double ca = T0[0] * ST0[0] + T0[1] * ST0[1] + T0[2] * ST0[2] + cam.eps2d;
        const double cb = T0[0] * ST1[0] + T0[1] * ST1[1] + T0[2] * ST1[2];
        const double cc = T1[0] * ST1[0] + T1[1] * ST1[1] + T1[2] * ST1[2] + cam.eps2d;
        const double det = ca * cc - cb * cb;
        const double o = 1.0 / (1.0 + exp(-logit));

        // ---- opacity
        const double g_logit = double(gco.w) * o * (1.0 - o);

        // ---- colour: SH coefficients and the viewing direction
        const double dvx = mu[0] - cam.cc[0], dvy = mu[1] - cam.cc[1], dvz = mu[2] - cam.cc[2];
        const double dn = sqrt(dvx * dvx + dvy * dvy + dvz * dvz);
        const double ux = dvx / dn, uy = dvy / dn, uz = dvz / dn;
        double Y[16], dY[16][3];
        sh_basis_grad(a.deg, ux, uy, uz, Y, dY);
        const int nc = (a.deg + 1) * (a.deg + 1);
        double raw[3] = {0.5, 0.5, 0.5};
        float shv[48];
        for (int p = 0; p < a.planes; ++p) {
            const float4 c4 = __ldg(a.sh + int64_t(p) * a.n + i);
            shv[4 * p + 0] = c4.x; shv[4 * p + 1] = c4.y; shv[4 * p + 2] = c4.z; shv[4 * p + 3] = c4.w;
        }
        for (int k = 0; k < nc; ++k)
            for (int ch = 0; ch < 3; ++ch) raw[ch] += double(shv[3 * k + ch]) * Y[k];
        double gcol[3] = {grg.x, grg.y, grg.z};
        for (int ch = 0; ch < 3; ++ch)
            if (raw[ch] < 0.0) gcol[ch] = 0.0;
        double gdir[3] = {0.0, 0.0, 0.0};
        for (int k = 1; k < nc; ++k) {
            const double wk = double(shv[3 * k]) * gcol[0] + double(shv[3 * k + 1]) * gcol[1] + double(shv[3 * k + 2]) * gcol[2];
            gdir[0] += wk * dY[k][0];
            gdir[1] += wk * dY[k][1];
            gdir[2] += wk * dY[k][2];
        }
        const double dproj = gdir[0] * ux + gdir[1] * uy + gdir[2] * uz;
        double gmu[3] = {(gdir[0] - ux * dproj) / dn, (gdir[1] - uy * dproj) / dn, (gdir[2] - uz * dproj) / dn};
        for (int p = 0; p < a.planes; ++p) {
            float4 d = a.d_sh[int64_t(p) * a.n + i];
            float dv[4] = {d.x, d.y, d.z, d.w};
            for (int e = 0; e < 4; ++e) {
                const int f = 4 * p + e, k = f / 3;
                if (k < nc) dv[e] += float(Y[k] * gcol[f - 3 * k]);
            }
            a.d_sh[int64_t(p) * a.n + i] = make_float4(dv[0], dv[1], dv[2], dv[3]);
        }

        // ---- pixel position (u, v) = (fx x/z + cx, fy y/z + cy)
        double gpc[3];
        gpc[0] = double(gxy.x) * cam.fx * iz;
        gpc[1] = double(gxy.y) * cam.fy * iz;
        gpc[2] = -(double(gxy.x) * cam.fx * pc[0] + double(gxy.y) * cam.fy * pc[1]) * iz * iz;

        // ---- conic (A, B, C) = (c, -b, a) / det  ->  (a, b, c)
        const double gA = gco.x, gB = gco.y, gC = gco.z;
        const double id2 = 1.0 / (det * det);
        const double ga = (-cc * cc * gA + cb * cc * gB - cb * cb * gC) * id2;
        const double gb = (2.0 * cb * cc * gA - (ca * cc + cb * cb) * gB + 2.0 * ca * cb * gC) * id2;
        const double gc = (-cb * cb * gA + ca * cb * gB - ca * ca * gC) * id2;

        // ---- (a, b, c) = rows of T Sigma T^T -> Sigma and T
        // symmetric dL/dSigma = ga T0 T0^T + gb/2 (T0 T1^T + T1 T0^T) + gc T1 T1^T
        double G[3][3];
        for (int r = 0; r < 3; ++r)
            for (int c = 0; c < 3; ++c)
                G[r][c] = ga * T0[r] * T0[c] + 0.5 * gb * (T0[r] * T1[c] + T1[r] * T0[c]) + gc * T1[r] * T1[c];
        double gT0[3], gT1[3];
        for (int c = 0; c < 3; ++c) {
            gT0[c] = 2.0 * ga * ST0[c] + gb * ST1[c];
            gT1[c] = gb * ST0[c] + 2.0 * gc * ST1[c];
        }
        // T0 = J00 W0 + J02 W2, T1 = J11 W1 + J12 W2
        const double gJ00 = gT0[0] * W0[0] + gT0[1] * W0[1] + gT0[2] * W0[2];
        const double gJ02 = gT0[0] * W2[0] + gT0[1] * W2[1] + gT0[2] * W2[2];
        const double gJ11 = gT1[0] * W1[0] + gT1[1] * W1[1] + gT1[2] * W1[2];
        const double gJ12 = gT1[0] * W2[0] + gT1[1] * W2[1] + gT1[2] * W2[2];
        // J00 = fx/z, J11 = fy/z, J02 = -fx tx/z^2 with tx = z clamp(x/z)
        gpc[2] += -gJ00 * cam.fx * iz * iz - gJ11 * cam.fy * iz * iz;
        if (clx) {
            gpc[2] += gJ02 * cam.fx * txz * iz * iz;
        } else {
            gpc[0] += -gJ02 * cam.fx * iz * iz;
            gpc[2] += gJ02 * 2.0 * cam.fx * pc[0] * iz * iz * iz;
        }
        if (cly) {
            gpc[2] += gJ12 * cam.fy * tyz * iz * iz;
        } else {
            gpc[1] += -gJ12 * cam.fy * iz * iz;
            gpc[2] += gJ12 * 2.0 * cam.fy * pc[1] * iz * iz * iz;
        }
        // means: pc = W mu + t
        for (int c = 0; c < 3; ++c) gmu[c] += W0[c] * gpc[0] + W1[c] * gpc[1] + W2[c] * gpc[2];

        // ---- Sigma = M M^T, M = Rq diag(s): dL/dM = 2 G M
        double gM[3][3];
        for (int r = 0; r < 3; ++r)
            for (int c = 0; c < 3; ++c) gM[r][c] = 2.0 * (G[r][0] * M[0][c] + G[r][1] * M[1][c] + G[r][2] * M[2][c]);
        double gls[3], gR[3][3];
        for (int c = 0; c < 3; ++c) {
            gls[c] = (gM[0][c] * Rq[0][c] + gM[1][c] * Rq[1][c] + gM[2][c] * Rq[2][c]) * s[c];
            for (int r = 0; r < 3; ++r) gR[r][c] = gM[r][c] * s[c];
        }
        // rotation matrix of (w, x, y, z)
        const double gw = 2.0 * (-z * gR[0][1] + y * gR[0][2] + z * gR[1][0] - x * gR[1][2] - y * gR[2][0] + x * gR[2][1]);
        const double gx = 2.0 * (y * gR[0][1] + z * gR[0][2] + y * gR[1][0] - 2.0 * x * gR[1][1] - w * gR[1][2] +
                                 z * gR[2][0] + w * gR[2][1] - 2.0 * x * gR[2][2]);
        const double gy = 2.0 * (-2.0 * y * gR[0][0] + x * gR[0][1] + w * gR[0][2] + x * gR[1][0] + z * gR[1][2] -
                                 w * gR[2][0] + z * gR[2][1] - 2.0 * y * gR[2][2]);
        const double gz = 2.0 * (-2.0 * z * gR[0][0] - w * gR[0][1] + x * gR[0][2] + w * gR[1][0] - 2.0 * z * gR[1][1] +
                                 y * gR[1][2] + x * gR[2][0] + y * gR[2][1]);
        // through the normalisation q / |q|
        const double qd = w * gw + x * gx + y * gy + z * gz;
        const double gq[4] = {(gw - w * qd) / qn, (gx - x * qd) / qn, (gy - y * qd) / qn, (gz - z * qd) / qn};

        // ---- accumulate
        float4 d;
        d = a.d_means[i];
        a.d_means[i] = make_float4(d.x + float(gmu[0]), d.y + float(gmu[1]), d.z + float(gmu[2]), d.w);
        d = a.d_quats[i];
        a.d_quats[i] = make_float4(d.x + float(gq[0]), d.y + float(gq[1]), d.z + float(gq[2]), d.w + float(gq[3]));
        d = a.d_log_scales[i];
        a.d_log_scales[i] = make_float4(d.x + float(gls[0]), d.y + float(gls[1]), d.z + float(gls[2]), d.w);
        a.d_logits[i] += float(g_logit);
        if (a.densify_accum) {
            a.densify_accum[i] += sqrtf(gxy.x * gxy.x + gxy.y * gxy.y);
            a.densify_count[i] += 1;
        }
    }
}

}  // namespace

cudaError_t launch_project_bwd(const gs_params& p, const CamArgs& cam, const gs_projected& proj,
                               const gs_grad2d& g2, const gs_param_grads& g, float* densify_accum,
                               int32_t* densify_count, cudaStream_t s) {
    BwdArgs a;
    a.means = reinterpret_cast<const float4*>(p.means);
    a.quats = reinterpret_cast<const float4*>(p.quats);
    a.log_scales = reinterpret_cast<const float4*>(p.log_scales);
    a.logits = p.opacity_logits;
    a.sh = reinterpret_cast<const float4*>(p.sh);
    a.deg = p.sh_degree;
    a.planes = sh_planes(p.sh_degree);
    a.n = p.n;
    a.cam = cam;
    a.radius = proj.radius;
    a.g_xy = reinterpret_cast<const float2*>(g2.xy);
    a.g_con = reinterpret_cast<const float4*>(g2.conic_opacity);
    a.g_rgb = reinterpret_cast<const float4*>(g2.rgb);
    a.d_means = reinterpret_cast<float4*>(g.means);
    a.d_quats = reinterpret_cast<float4*>(g.quats);
    a.d_log_scales = reinterpret_cast<float4*>(g.log_scales);
    a.d_logits = g.opacity_logits;
    a.d_sh = reinterpret_cast<float4*>(g.sh);
    a.densify_accum = densify_accum;
    a.densify_count = densify_count;
    if (p.n == 0) return cudaSuccess;
    project_bwd_kernel<<<grid_for(p.n, 128, 16), 128, 0, s>>>(a);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace gsk
