/*
 * CPU oracle of the differentiable 3D Gaussian Splatting tile rasterizer.
 *
 * TEST INFRASTRUCTURE ONLY.  The pytest suites, the smoke check and the
 * benchmark's CPU-baseline leg call this library to obtain expected values;
 * the product (the CUDA library and its Python binding) never links, loads or
 * calls it, and the two share no code.
 *
 * What it computes, plainly and slowly, in double precision:
 *   - orc_project:     per-Gaussian projection (stages 1-2 of the three-stage
 *                      pipeline in the gsplat guide, lmnt.cn/news/262699 §2.1):
 *                      activations (gsplat guide §3.3: exp of log-scales,
 *                      sigmoid of opacity logits, w-first quaternion),
 *                      Sigma = R S S^T R^T, EWA projection J W Sigma W^T J^T
 *                      plus a screen-space dilation, its inverse (the conic),
 *                      a 3-sigma radius, the 16x16-tile rectangle, and the
 *                      view-dependent colour from real spherical harmonics.
 *   - orc_keys:        every (Gaussian, tile) instance with key
 *                      (tile_id << 32 | depth bits), sorted by (key, gid), and
 *                      the per-tile ranges of the sorted list.
 *   - orc_render:      stage 3, per pixel: the pixel's candidate set (visible
 *                      Gaussians whose tile rectangle covers the pixel's tile),
 *                      a full depth sort of that set, then front-to-back alpha
 *                      compositing: alpha = min(0.99, o exp(-1/2 d^T S'^-1 d)),
 *                      entries with alpha < 1/255 skipped, stop (without
 *                      blending) once the transmittance would fall below 1e-4.
 *   - orc_render_bwd:  the reverse of that compositing, derived directly from
 *                      C = sum_i c_i a_i T_i + T_final bg, accumulated in double.
 *   - orc_project_bwd: the exact derivative of orc_project's outputs with respect
 *                      to every Gaussian parameter, by forward-mode dual numbers
 *                      over the same templated projection code (one pass per
 *                      parameter), contracted with the 2D gradients.
 *   - orc_adam, orc_l1: Adam (gsplat guide §4.2: betas 0.9/0.99, eps 1e-15) and
 *                      the L1 photometric loss (gsplat guide §4.1) with its gradient.
 *   - orc_ssim:        the structural similarity of the L1 + D-SSIM loss
 *                      (gsplat guide §4.1) and its gradient.
 *   - orc_densify:     adaptive density control (gsplat guide §4.1): prune,
 *                      clone or split each Gaussian from its accumulated
 *                      screen-space gradient statistic, opacity, scale and the
 *                      largest screen radius it reached.
 *
 * Readings where the pages are silent (pixel centres at +0.5, near plane and
 * dilation as camera fields, 1.3x Jacobian clamp, radius = ceil(3 sqrt(lmax)),
 * rectangle rule, termination order, SH sign convention) are the same ones the
 * CUDA path implements; they are listed with the design notes.
 *
 * Precision: everything in double.  With `quantize` set, orc_project rounds its
 * outputs to float32, the storage precision of the projected arrays the
 * compositing stage consumes, so that later stages are evaluated exactly on the
 * same stage inputs the CUDA path stores.
 */
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>
#include <omp.h>

#include <array>
#include <map>
#include <utility>

namespace {

/* ---------------------------------------------------------------- dual numbers */

struct Dual {
    double v, d;
    Dual(double v_ = 0.0, double d_ = 0.0) : v(v_), d(d_) {}
};
inline Dual operator+(Dual a, Dual b) { return {a.v + b.v, a.d + b.d}; }
inline Dual operator-(Dual a, Dual b) { return {a.v - b.v, a.d - b.d}; }
inline Dual operator-(Dual a) { return {-a.v, -a.d}; }
inline Dual operator*(Dual a, Dual b) { return {a.v * b.v, a.d * b.v + a.v * b.d}; }
inline Dual operator/(Dual a, Dual b) { return {a.v / b.v, (a.d * b.v - a.v * b.d) / (b.v * b.v)}; }
inline Dual exp(Dual a) { double e = std::exp(a.v); return {e, a.d * e}; }
inline Dual sqrt(Dual a) { double s = std::sqrt(a.v); return {s, a.d / (2.0 * s)}; }
inline double val(Dual a) { return a.v; }
inline double val(double a) { return a; }
inline double der(Dual a) { return a.d; }
using std::exp;
using std::sqrt;

/* ---------------------------------------------------------------- camera */

struct Camera {
    double R[9], t[3], fx, fy, cx, cy, near_plane, eps2d;
    int width, height;
    int tiles_x() const { return (width + 15) / 16; }
    int tiles_y() const { return (height + 15) / 16; }
};

}  // namespace

extern "C" {
/* Camera as passed from Python: R (row-major, world->camera), t, fx, fy, cx, cy,
 * near, eps2d as doubles, then width and height. */
typedef struct {
    double R[9], t[3], fx, fy, cx, cy, near_plane, eps2d;
    int32_t width, height;
} orc_camera;
}

namespace {

Camera to_cam(const orc_camera* c) {
    Camera k;
    std::memcpy(k.R, c->R, sizeof k.R);
    std::memcpy(k.t, c->t, sizeof k.t);
    k.fx = c->fx; k.fy = c->fy; k.cx = c->cx; k.cy = c->cy;
    k.near_plane = c->near_plane; k.eps2d = c->eps2d;
    k.width = c->width; k.height = c->height;
    return k;
}

/* ------------------------------------------------ real spherical harmonics
 * Orthonormal real SH with the Condon-Shortley phase kept, index
 * k = l^2 + l + m for m = -l..l:
 *   m = 0:  K(l,0) P_l(z)
 *   m > 0:  sqrt2 K(l,m) (-1)^m Re((x+iy)^m) P_l^(m)(z)
 *   m < 0:  sqrt2 K(l,|m|) (-1)^|m| Im((x+iy)^|m|) P_l^(|m|)(z)
 * with K(l,m) = sqrt((2l+1)/(4 pi) (l-m)!/(l+m)!) and P_l^(m) the m-th
 * derivative of the Legendre polynomial; (1-z^2)^(m/2) cos(m phi) is folded
 * into Re((x+iy)^m).  Coefficients of P_l come from the explicit sum
 * P_l(z) = 2^-l sum_k (-1)^k C(l,k) C(2l-2k,l) z^(l-2k).
 */
double binom(int n, int k) {
    double r = 1.0;
    for (int i = 1; i <= k; ++i) r = r * (n - k + i) / i;
    return r;
}
double fact(int n) { double r = 1.0; for (int i = 2; i <= n; ++i) r *= i; return r; }

struct SHTable {
    // poly[l][m][p]: coefficient of z^p in P_l^(m)(z); norm[l][m] = K(l,m) (times sqrt2 for m>0)
    double poly[4][4][4];
    double norm[4][4];
    SHTable() {
        std::memset(poly, 0, sizeof poly);
        for (int l = 0; l <= 3; ++l) {
            double c[4] = {0, 0, 0, 0};
            for (int k = 0; 2 * k <= l; ++k)
                c[l - 2 * k] += std::ldexp(1.0, -l) * ((k & 1) ? -1.0 : 1.0) * binom(l, k) * binom(2 * l - 2 * k, l);
            for (int m = 0; m <= l; ++m) {
                for (int p = 0; p <= 3; ++p) poly[l][m][p] = c[p];
                for (int p = 0; p + 1 <= 3; ++p) c[p] = (p + 1) * c[p + 1];  // differentiate
                c[3] = 0.0;
                double K = std::sqrt((2 * l + 1) / (4.0 * M_PI) * fact(l - m) / fact(l + m));
                norm[l][m] = (m == 0) ? K : std::sqrt(2.0) * K * ((m & 1) ? -1.0 : 1.0);
            }
        }
    }
};
const SHTable& sh_table() { static SHTable t; return t; }

template <class T>
void sh_basis(int deg, T x, T y, T z, T* Y) {
    const SHTable& tb = sh_table();
    // powers (x+iy)^m
    T re[4], im[4];
    re[0] = T(1.0); im[0] = T(0.0);
    for (int m = 1; m <= 3; ++m) {
        re[m] = re[m - 1] * x - im[m - 1] * y;
        im[m] = re[m - 1] * y + im[m - 1] * x;
    }
    for (int l = 0; l <= deg; ++l) {
        for (int m = 0; m <= l; ++m) {
            T p = T(0.0);
            for (int q = 3; q >= 0; --q) p = p * z + T(tb.poly[l][m][q]);
            T base = T(tb.norm[l][m]) * p;
            if (m == 0) {
                Y[l * l + l] = base;
            } else {
                Y[l * l + l + m] = base * re[m];
                Y[l * l + l - m] = base * im[m];
            }
        }
    }
}

/* ------------------------------------------------------------ projection */

template <class T>
struct Proj {
    bool visible = false;
    T u, v, A, B, C, o, rgb[3], z;
    int radius = 0;
    int rect[4] = {0, 0, 0, 0};   // xmin, ymin, xmax, ymax (tiles, max exclusive)
};

inline bool finite3(double a, double b, double c) { return std::isfinite(a) && std::isfinite(b) && std::isfinite(c); }

/* One Gaussian.  P holds the 11 + 3*nc parameters in the order
 * mean(3) quat(4, wxyz) log_scale(3) opacity_logit(1) sh(nc*3, coefficient-major). */
template <class T>
Proj<T> project_one(const T* P, int deg, const Camera& cam) {
    Proj<T> out;
    const T* mu = P;
    const T* q = P + 3;
    const T* ls = P + 7;
    const T logit = P[10];
    const T* sh = P + 11;
    const int nc = (deg + 1) * (deg + 1);

    for (int i = 0; i < 11; ++i)
        if (!std::isfinite(val(P[i]))) return out;

    // camera space: p = R mu + t
    T pc[3];
    for (int r = 0; r < 3; ++r)
        pc[r] = ((T(cam.R[3 * r + 0]) * mu[0] + T(cam.R[3 * r + 1]) * mu[1]) + T(cam.R[3 * r + 2]) * mu[2]) + T(cam.t[r]);
    if (!(val(pc[2]) > cam.near_plane)) return out;

    // rotation from the normalised quaternion (w, x, y, z)
    T qn2 = ((q[0] * q[0] + q[1] * q[1]) + q[2] * q[2]) + q[3] * q[3];
    if (!(val(qn2) > 0.0)) return out;
    T qn = sqrt(qn2);
    T w = q[0] / qn, x = q[1] / qn, y = q[2] / qn, z = q[3] / qn;
    T Rq[3][3];
    Rq[0][0] = T(1.0) - T(2.0) * (y * y + z * z);
    Rq[0][1] = T(2.0) * (x * y - w * z);
    Rq[0][2] = T(2.0) * (x * z + w * y);
    Rq[1][0] = T(2.0) * (x * y + w * z);
    Rq[1][1] = T(1.0) - T(2.0) * (x * x + z * z);
    Rq[1][2] = T(2.0) * (y * z - w * x);
    Rq[2][0] = T(2.0) * (x * z - w * y);
    Rq[2][1] = T(2.0) * (y * z + w * x);
    Rq[2][2] = T(1.0) - T(2.0) * (x * x + y * y);

    // Sigma = M M^T with M = Rq diag(exp(log_scale))
    T s[3] = {exp(ls[0]), exp(ls[1]), exp(ls[2])};
    T M[3][3];
    for (int i = 0; i < 3; ++i)
        for (int j = 0; j < 3; ++j) M[i][j] = Rq[i][j] * s[j];
    T S[3][3];
    for (int i = 0; i < 3; ++i)
        for (int j = 0; j < 3; ++j) S[i][j] = (M[i][0] * M[j][0] + M[i][1] * M[j][1]) + M[i][2] * M[j][2];

    // EWA: J (2x3) of the perspective map at p, the x/z and y/z used in J
    // clamped to 1.3x the half field of view
    const double limx = 1.3 * (0.5 * cam.width / cam.fx);
    const double limy = 1.3 * (0.5 * cam.height / cam.fy);
    T txz = pc[0] / pc[2], tyz = pc[1] / pc[2];
    if (val(txz) < -limx) txz = T(-limx);
    if (val(txz) > limx) txz = T(limx);
    if (val(tyz) < -limy) tyz = T(-limy);
    if (val(tyz) > limy) tyz = T(limy);
    T tx = txz * pc[2], ty = tyz * pc[2];
    T iz = T(1.0) / pc[2];
    T J00 = T(cam.fx) * iz, J02 = -(T(cam.fx) * tx) * (iz * iz);
    T J11 = T(cam.fy) * iz, J12 = -(T(cam.fy) * ty) * (iz * iz);
    // Tm = J W (W = camera rotation)
    T Tm[2][3];
    for (int j = 0; j < 3; ++j) {
        Tm[0][j] = J00 * T(cam.R[0 + j]) + J02 * T(cam.R[6 + j]);
        Tm[1][j] = J11 * T(cam.R[3 + j]) + J12 * T(cam.R[6 + j]);
    }
    // Sigma' = Tm S Tm^T + eps2d I
    T X[2][3];
    for (int i = 0; i < 2; ++i)
        for (int j = 0; j < 3; ++j) X[i][j] = (Tm[i][0] * S[0][j] + Tm[i][1] * S[1][j]) + Tm[i][2] * S[2][j];
    T a = ((X[0][0] * Tm[0][0] + X[0][1] * Tm[0][1]) + X[0][2] * Tm[0][2]) + T(cam.eps2d);
    T b = (X[0][0] * Tm[1][0] + X[0][1] * Tm[1][1]) + X[0][2] * Tm[1][2];
    T c = ((X[1][0] * Tm[1][0] + X[1][1] * Tm[1][1]) + X[1][2] * Tm[1][2]) + T(cam.eps2d);
    T det = a * c - b * b;
    if (!(val(det) > 0.0)) return out;
    T idet = T(1.0) / det;

    // 3-sigma radius of the larger eigenvalue (integer, no derivative)
    double mid = 0.5 * (val(a) + val(c));
    double lmax = mid + std::sqrt(std::max(0.1, mid * mid - val(det)));
    double r = std::ceil(3.0 * std::sqrt(lmax));

    // pixel coordinates of the mean
    T u = T(cam.fx) * (pc[0] / pc[2]) + T(cam.cx);
    T v = T(cam.fy) * (pc[1] / pc[2]) + T(cam.cy);
    if (!std::isfinite(val(u)) || !std::isfinite(val(v)) || !std::isfinite(r)) return out;

    // 16x16 tile rectangle [min, max)
    const double TX = cam.tiles_x(), TY = cam.tiles_y();
    auto clampd = [](double x, double lo, double hi) { return x < lo ? lo : (x > hi ? hi : x); };
    double xmin = clampd(std::floor((val(u) - r) * 0.0625), 0.0, TX);
    double xmax = clampd(std::floor((val(u) + r) * 0.0625) + 1.0, 0.0, TX);
    double ymin = clampd(std::floor((val(v) - r) * 0.0625), 0.0, TY);
    double ymax = clampd(std::floor((val(v) + r) * 0.0625) + 1.0, 0.0, TY);
    if ((xmax - xmin) * (ymax - ymin) <= 0.0) return out;

    // colour: real SH of the viewing direction from the camera centre -R^T t
    double cc[3];
    for (int j = 0; j < 3; ++j) cc[j] = -((cam.R[0 + j] * cam.t[0] + cam.R[3 + j] * cam.t[1]) + cam.R[6 + j] * cam.t[2]);
    T dv[3] = {mu[0] - T(cc[0]), mu[1] - T(cc[1]), mu[2] - T(cc[2])};
    T dn = sqrt((dv[0] * dv[0] + dv[1] * dv[1]) + dv[2] * dv[2]);
    T Y[16];
    sh_basis(deg, dv[0] / dn, dv[1] / dn, dv[2] / dn, Y);
    for (int ch = 0; ch < 3; ++ch) {
        T acc = T(0.0);
        for (int k = 0; k < nc; ++k) acc = acc + sh[3 * k + ch] * Y[k];
        acc = acc + T(0.5);
        if (!std::isfinite(val(acc))) return out;
        out.rgb[ch] = (val(acc) < 0.0) ? T(0.0) : acc;
    }

    out.A = c * idet;
    out.B = -b * idet;
    out.C = a * idet;
    out.o = T(1.0) / (T(1.0) + exp(-logit));
    out.u = u;
    out.v = v;
    out.z = pc[2];
    out.radius = (int)r;
    out.rect[0] = (int)xmin; out.rect[1] = (int)ymin; out.rect[2] = (int)xmax; out.rect[3] = (int)ymax;
    out.visible = true;
    return out;
}

void load_params(int64_t i, const double* means, const double* quats, const double* log_scales, const double* logits,
                 const double* sh, int nc, double* P) {
    for (int j = 0; j < 3; ++j) P[j] = means[3 * i + j];
    for (int j = 0; j < 4; ++j) P[3 + j] = quats[4 * i + j];
    for (int j = 0; j < 3; ++j) P[7 + j] = log_scales[3 * i + j];
    P[10] = logits[i];
    for (int j = 0; j < 3 * nc; ++j) P[11 + j] = sh[(int64_t)3 * nc * i + j];
}

inline double q32(double x, int quantize) { return quantize ? (double)(float)x : x; }

inline uint32_t f32_bits(double z) {
    float f = (float)z;
    uint32_t b;
    std::memcpy(&b, &f, 4);
    return b;
}

}  // namespace

extern "C" {

int orc_version(void) { return 1; }

/* Project n Gaussians (or the subset idx[0..nidx) when idx != NULL; outputs are
 * indexed by position in idx).  Parameters arrive as doubles (the float32 scene
 * values widened exactly, or true doubles for finite-difference pins).
 * Culled Gaussians get radius 0, an empty
 * rectangle, tiles_touched 0 and zero features. */
int orc_project(int64_t n, const double* means, const double* quats, const double* log_scales, const double* logits,
                const double* sh, int sh_degree, const orc_camera* ocam, int quantize,
                const int64_t* idx, int64_t nidx,
                double* xy, double* depth, double* conic, double* opac, double* rgb,
                int32_t* radius, int32_t* rect, uint32_t* tiles_touched) {
    if (sh_degree < 0 || sh_degree > 3) return 1;
    const Camera cam = to_cam(ocam);
    const int nc = (sh_degree + 1) * (sh_degree + 1);
    const int64_t cnt = idx ? nidx : n;
#pragma omp parallel for schedule(dynamic, 1024)
    for (int64_t k = 0; k < cnt; ++k) {
        const int64_t i = idx ? idx[k] : k;
        double P[11 + 48];
        load_params(i, means, quats, log_scales, logits, sh, nc, P);
        Proj<double> p = project_one<double>(P, sh_degree, cam);
        if (!p.visible) {
            xy[2 * k] = xy[2 * k + 1] = 0.0;
            depth[k] = 0.0;
            conic[3 * k] = conic[3 * k + 1] = conic[3 * k + 2] = 0.0;
            opac[k] = 0.0;
            rgb[3 * k] = rgb[3 * k + 1] = rgb[3 * k + 2] = 0.0;
            radius[k] = 0;
            rect[4 * k] = rect[4 * k + 1] = rect[4 * k + 2] = rect[4 * k + 3] = 0;
            tiles_touched[k] = 0;
            continue;
        }
        xy[2 * k] = q32(p.u, quantize);
        xy[2 * k + 1] = q32(p.v, quantize);
        depth[k] = q32(p.z, quantize);
        conic[3 * k] = q32(p.A, quantize);
        conic[3 * k + 1] = q32(p.B, quantize);
        conic[3 * k + 2] = q32(p.C, quantize);
        opac[k] = q32(p.o, quantize);
        for (int c = 0; c < 3; ++c) rgb[3 * k + c] = q32(p.rgb[c], quantize);
        radius[k] = p.radius;
        for (int j = 0; j < 4; ++j) rect[4 * k + j] = p.rect[j];
        tiles_touched[k] = (uint32_t)((p.rect[2] - p.rect[0]) * (p.rect[3] - p.rect[1]));
    }
    return 0;
}

/* All (Gaussian, tile) instances: key = (ty*TX + tx) << 32 | float32 bits of the
 * view depth, value = gid; sorted by (key, gid).  ranges[2*t] / [2*t+1] are the
 * [begin, end) of tile t in the sorted list ([0,0) when empty).
 * Returns K, or -K-1 (nothing written) when K exceeds capacity. */
int64_t orc_keys(int64_t n, const double* depth, const int32_t* rect, const int32_t* radius, int tiles_x, int tiles_y,
                 int64_t capacity, uint64_t* keys, uint32_t* vals, uint32_t* ranges) {
    int64_t K = 0;
    for (int64_t i = 0; i < n; ++i)
        if (radius[i] > 0) K += (int64_t)(rect[4 * i + 2] - rect[4 * i]) * (rect[4 * i + 3] - rect[4 * i + 1]);
    if (K > capacity) return -K - 1;
    std::vector<std::pair<uint64_t, uint32_t>> inst;
    inst.reserve((size_t)K);
    for (int64_t i = 0; i < n; ++i) {
        if (radius[i] <= 0) continue;
        const uint64_t zb = f32_bits(depth[i]);
        for (int ty = rect[4 * i + 1]; ty < rect[4 * i + 3]; ++ty)
            for (int tx = rect[4 * i]; tx < rect[4 * i + 2]; ++tx)
                inst.emplace_back(((uint64_t)((int64_t)ty * tiles_x + tx) << 32) | zb, (uint32_t)i);
    }
    std::sort(inst.begin(), inst.end());
    const int64_t T = (int64_t)tiles_x * tiles_y;
    for (int64_t t = 0; t < 2 * T; ++t) ranges[t] = 0;
    for (int64_t k = 0; k < K; ++k) {
        keys[k] = inst[k].first;
        vals[k] = inst[k].second;
        const uint64_t t = inst[k].first >> 32;
        if (k == 0 || (inst[k - 1].first >> 32) != t) ranges[2 * t] = (uint32_t)k;
        if (k == K - 1 || (inst[k + 1].first >> 32) != t) ranges[2 * t + 1] = (uint32_t)(k + 1);
    }
    return K;
}

}  // extern "C"

namespace {

/* ---------------------------------------------------------- compositing */

struct Features {
    const double *xy, *depth, *conic, *opac, *rgb;
    const int32_t *radius, *rect;
};

constexpr double ALPHA_MAX = 0.99;
constexpr double ALPHA_MIN = 1.0 / 255.0;
constexpr double T_MIN = 1e-4;

struct Blended {
    int64_t gid;
    double alpha, T, G, dx, dy;
    bool clamped;
};

/* Candidates of one tile: visible Gaussians whose rectangle covers it. */
std::vector<int64_t> tile_candidates(int64_t n, const Features& f, int tx, int ty) {
    std::vector<int64_t> c;
    for (int64_t i = 0; i < n; ++i) {
        if (f.radius[i] <= 0) continue;
        const int32_t* r = f.rect + 4 * i;
        if (tx >= r[0] && tx < r[2] && ty >= r[1] && ty < r[3]) c.push_back(i);
    }
    return c;
}

/* The candidates whose alpha at pixel (px, py) could reach the 1/255 threshold
 * under a relative perturbation of band_alpha (o exp(-sigma) >= (1 - band_alpha)
 * / 255, or a form so close to indefinite that its sign is not decided), i.e.
 * every Gaussian a float32 evaluation might blend there, before or after the
 * pixel's stop.  A Gaussian outside this set takes no gradient from the pixel
 * whatever the pixel's straddling decisions are. */
std::vector<int64_t> reachable(const Features& f, const std::vector<int64_t>& cand, int px, int py,
                               double band_alpha) {
    std::vector<int64_t> r;
    const double X = px + 0.5, Yp = py + 0.5;
    for (int64_t i : cand) {
        const double dx = f.xy[2 * i] - X, dy = f.xy[2 * i + 1] - Yp;
        const double A = f.conic[3 * i], B = f.conic[3 * i + 1], Cc = f.conic[3 * i + 2];
        const double sigma = 0.5 * (A * dx * dx + Cc * dy * dy) + B * dx * dy;
        const double scale = 0.5 * (std::fabs(A) * dx * dx + std::fabs(Cc) * dy * dy) + std::fabs(B * dx * dy);
        const double s = sigma <= 1e-6 * scale ? 0.0 : sigma;  // undecided sign: as if at the mean
        if (f.opac[i] * std::exp(-s) >= (1.0 - band_alpha) * ALPHA_MIN) r.push_back(i);
    }
    return r;
}

/* A decision of the compositing that float32 evaluation may legitimately take the
 * other way: entry k of the pixel's depth-sorted list and the test. */
enum StraddleKind { kSignTest = 1, kSkipTest = 2, kClampTest = 3, kStopTest = 4 };
struct Straddle {
    size_t k;
    int kind;
};

/* Composite one pixel front to back over its depth-sorted candidate list.
 * Returns the blended entries (for the reverse pass) and the ambiguity flags:
 *   bit 0: a skip/stop decision lay within the relative band of its threshold
 *          (alpha vs 1/255 or T(1-alpha) vs 1e-4, or the sign of a form this
 *          close to indefinite), so float32 evaluation may legitimately decide
 *          the other way;
 *   bit 1: an unclamped alpha lay within the band of the 0.99 clamp (gradients
 *          switch on or off there; values are continuous); those entries are
 *          appended to clamp_band when given.
 * Every such decision is appended to `straddles` when given; with `invert` the
 * one decision it names is taken the other way (the alternative result). */
int composite_pixel(const Features& f, std::vector<int64_t> cand, int px, int py, const double* bg,
                    double band_alpha, double band_T, double* color, double* finalT, int32_t* ncontrib,
                    std::vector<Blended>* blended, std::vector<int64_t>* clamp_band = nullptr,
                    std::vector<Straddle>* straddles = nullptr, const Straddle* invert = nullptr) {
    // full depth sort of this pixel's candidates: by float32 depth bits, then gid
    std::sort(cand.begin(), cand.end(), [&](int64_t a, int64_t b) {
        uint32_t za = f32_bits(f.depth[a]), zb = f32_bits(f.depth[b]);
        return za != zb ? za < zb : a < b;
    });
    const auto flipped = [&](size_t k, int kind) { return invert && invert->k == k && invert->kind == kind; };
    const auto record = [&](size_t k, int kind) {
        if (straddles) straddles->push_back({k, kind});
    };
    const double X = px + 0.5, Yp = py + 0.5;
    double T = 1.0, C[3] = {0, 0, 0};
    int32_t last = 0;
    int amb = 0;
    for (size_t k = 0; k < cand.size(); ++k) {
        const int64_t i = cand[k];
        const double dx = f.xy[2 * i] - X, dy = f.xy[2 * i + 1] - Yp;
        const double A = f.conic[3 * i], B = f.conic[3 * i + 1], Cc = f.conic[3 * i + 2];
        const double sigma = 0.5 * (A * dx * dx + Cc * dy * dy) + B * dx * dy;
        // a form this close to indefinite may round below zero in float32
        if (sigma <= 1e-6 * (0.5 * (std::fabs(A) * dx * dx + std::fabs(Cc) * dy * dy) + std::fabs(B * dx * dy)) &&
            sigma != 0.0) {
            amb |= 1;
            record(k, kSignTest);
        }
        if ((sigma < 0.0) != flipped(k, kSignTest)) continue;
        const double G = std::exp(-sigma);
        const double a = f.opac[i] * G;
        const double alpha = std::min(ALPHA_MAX, a);
        if (std::fabs(alpha - ALPHA_MIN) <= band_alpha * ALPHA_MIN) {
            amb |= 1;
            record(k, kSkipTest);
        }
        if ((alpha < ALPHA_MIN) != flipped(k, kSkipTest)) continue;
        if (std::fabs(a - ALPHA_MAX) <= band_alpha * ALPHA_MAX) {
            amb |= 2;
            if (clamp_band) clamp_band->push_back(i);
            record(k, kClampTest);
        }
        // the clamp changes alpha continuously; what a straddle decides is whether
        // alpha has a derivative with respect to o and sigma
        const bool clamped = (a > ALPHA_MAX) != flipped(k, kClampTest);
        const double Tn = T * (1.0 - alpha);
        if (std::fabs(Tn - T_MIN) <= band_T * T_MIN) {
            amb |= 1;
            record(k, kStopTest);
        }
        if ((Tn < T_MIN) != flipped(k, kStopTest)) break;
        for (int c = 0; c < 3; ++c) C[c] += f.rgb[3 * i + c] * alpha * T;
        if (blended) blended->push_back({i, alpha, T, G, dx, dy, clamped});
        T = Tn;
        last = (int32_t)(k + 1);
    }
    for (int c = 0; c < 3; ++c) color[c] = C[c] + T * bg[c];
    *finalT = T;
    *ncontrib = last;
    return amb;
}

/* The reverse pass of one pixel: the 9 gradient terms (u, v, A, B, C, o, r, g,
 * b) of every blended entry for the upstream g, derived directly from
 * C = sum_i c_i alpha_i T_i + T_final bg.  Appended to `out` as (gid, terms). */
void pixel_terms(const Features& f, const std::vector<Blended>& bl, double T_final, const double* g,
                 const double* bg, std::vector<std::pair<int64_t, std::array<double, 9>>>* out) {
    // S = colour accumulated behind the current entry, normalised by the
    // transmittance just behind it
    double S[3] = {0, 0, 0};
    for (int e = (int)bl.size() - 1; e >= 0; --e) {
        const Blended& b = bl[e];
        const int64_t i = b.gid;
        const double* c = f.rgb + 3 * i;
        std::array<double, 9> t9 = {0, 0, 0, 0, 0, 0, 0, 0, 0};
        double dL_dalpha = 0.0;
        for (int ch = 0; ch < 3; ++ch) {
            t9[6 + ch] = b.alpha * b.T * g[ch];
            dL_dalpha += g[ch] * (b.T * (c[ch] - S[ch]) - T_final * bg[ch] / (1.0 - b.alpha));
        }
        for (int ch = 0; ch < 3; ++ch) S[ch] = c[ch] * b.alpha + (1.0 - b.alpha) * S[ch];
        if (!b.clamped) {
            const double A = f.conic[3 * i], B = f.conic[3 * i + 1], Cc = f.conic[3 * i + 2];
            t9[5] = dL_dalpha * b.G;                        // d alpha / d o = G
            const double dL_dsigma = -dL_dalpha * b.alpha;  // d alpha / d sigma = -o G
            t9[0] = dL_dsigma * (A * b.dx + B * b.dy);      // d sigma / d u
            t9[1] = dL_dsigma * (B * b.dx + Cc * b.dy);     // d sigma / d v
            t9[2] = dL_dsigma * 0.5 * b.dx * b.dx;
            t9[3] = dL_dsigma * b.dx * b.dy;
            t9[4] = dL_dsigma * 0.5 * b.dy * b.dy;
        }
        out->push_back({i, t9});
    }
}

}  // namespace

extern "C" {

/* Render the pixels pix[0..npix) (indices y*W + x; NULL = every pixel in order).
 * Features are the orc_project outputs.  Writes image[3*k..], final_T[k],
 * n_contrib[k] (1 + position of the last blended entry in the tile's sorted
 * list, 0 if none) and ambiguous[k] (flags above). */
int orc_render(int64_t n, const double* xy, const double* depth, const double* conic, const double* opac,
               const double* rgb, const int32_t* radius, const int32_t* rect, const orc_camera* ocam,
               const double* bg, int64_t npix, const int64_t* pix, double band_alpha, double band_T,
               double* image, double* final_T, int32_t* n_contrib, uint8_t* ambiguous) {
    const Camera cam = to_cam(ocam);
    const Features f{xy, depth, conic, opac, rgb, radius, rect};
    const int64_t W = cam.width;
    const int64_t cnt = pix ? npix : W * cam.height;
    // group pixels by tile so each tile's candidate scan is done once
    std::vector<int64_t> order(cnt);
    for (int64_t k = 0; k < cnt; ++k) order[k] = k;
    auto tile_of = [&](int64_t k) {
        const int64_t p = pix ? pix[k] : k;
        return (p / W / 16) * cam.tiles_x() + (p % W) / 16;
    };
    std::stable_sort(order.begin(), order.end(), [&](int64_t a, int64_t b) { return tile_of(a) < tile_of(b); });
    std::vector<int64_t> starts;
    for (int64_t k = 0; k < cnt; ++k)
        if (k == 0 || tile_of(order[k]) != tile_of(order[k - 1])) starts.push_back(k);
    starts.push_back(cnt);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t s = 0; s < (int64_t)starts.size() - 1; ++s) {
        const int64_t t = tile_of(order[starts[s]]);
        const int tx = (int)(t % cam.tiles_x()), ty = (int)(t / cam.tiles_x());
        const std::vector<int64_t> cand = tile_candidates(n, f, tx, ty);
        for (int64_t j = starts[s]; j < starts[s + 1]; ++j) {
            const int64_t k = order[j];
            const int64_t p = pix ? pix[k] : k;
            ambiguous[k] = (uint8_t)composite_pixel(f, cand, (int)(p % W), (int)(p / W), bg, band_alpha, band_T,
                                                    image + 3 * k, final_T + k, n_contrib + k, nullptr);
        }
    }
    return 0;
}

/* Reverse pass for the pixels pix[0..npix) with upstream gradients
 * dL_dpix[3*k..] (all other pixels contribute nothing).  Accumulates (+=) into
 * grad2d[9*i..] = dL/d(u, v, A, B, C, o, r, g, b) and grad2d_abs (the sum of
 * the absolute values of the accumulated terms, a conditioning measure).
 * touched_amb[i] is set for the Gaussians whose gradient a straddling decision at
 * one of the pixels can change: with a skip/stop straddle (bit 0) every Gaussian
 * reachable at that pixel (it may blend there or not, and every blended entry's
 * T and S move with it); with only a clamp straddle (bit 1) the entries in the
 * clamp band (their alpha is continuous, only their own dalpha switches).
 * straddle (nullable, [n][9]) accumulates, over the pixels and over each of their
 * straddling decisions, |terms with that decision taken the other way - terms as
 * taken| per Gaussian and component: how far float32 evaluation that legitimately
 * decides a straddle the other way can move each 2D gradient. */
int orc_render_bwd(int64_t n, const double* xy, const double* depth, const double* conic, const double* opac,
                   const double* rgb, const int32_t* radius, const int32_t* rect, const orc_camera* ocam,
                   const double* bg, int64_t npix, const int64_t* pix, const double* dL_dpix, double band_alpha,
                   double band_T, double* grad2d, double* grad2d_abs, uint8_t* touched_amb, double* straddle) {
    const Camera cam = to_cam(ocam);
    const Features f{xy, depth, conic, opac, rgb, radius, rect};
    const int64_t W = cam.width;
    const int64_t cnt = pix ? npix : W * cam.height;
    std::vector<int64_t> order(cnt);
    for (int64_t k = 0; k < cnt; ++k) order[k] = k;
    auto tile_of = [&](int64_t k) {
        const int64_t p = pix ? pix[k] : k;
        return (p / W / 16) * cam.tiles_x() + (p % W) / 16;
    };
    std::stable_sort(order.begin(), order.end(), [&](int64_t a, int64_t b) { return tile_of(a) < tile_of(b); });
    std::vector<int64_t> starts;
    for (int64_t k = 0; k < cnt; ++k)
        if (k == 0 || tile_of(order[k]) != tile_of(order[k - 1])) starts.push_back(k);
    starts.push_back(cnt);
#pragma omp parallel for schedule(dynamic, 1)
    for (int64_t s = 0; s < (int64_t)starts.size() - 1; ++s) {
        const int64_t t = tile_of(order[starts[s]]);
        const int tx = (int)(t % cam.tiles_x()), ty = (int)(t / cam.tiles_x());
        const std::vector<int64_t> cand = tile_candidates(n, f, tx, ty);
        std::vector<Blended> bl, bl2;
        std::vector<int64_t> cb;
        std::vector<Straddle> events;
        std::vector<std::pair<int64_t, std::array<double, 9>>> terms, terms2;
        for (int64_t j = starts[s]; j < starts[s + 1]; ++j) {
            const int64_t k = order[j];
            const int64_t p = pix ? pix[k] : k;
            const int ppx = (int)(p % W), ppy = (int)(p / W);
            const double* g = dL_dpix + 3 * k;
            if (g[0] == 0.0 && g[1] == 0.0 && g[2] == 0.0) continue;
            bl.clear();
            cb.clear();
            events.clear();
            double color[3], T_final;
            int32_t nc;
            const int amb = composite_pixel(f, cand, ppx, ppy, bg, band_alpha, band_T, color, &T_final, &nc, &bl, &cb,
                                            &events);
            if (amb & 1) {
                for (int64_t i : reachable(f, cand, ppx, ppy, band_alpha)) {
#pragma omp atomic write
                    touched_amb[i] = 1;
                }
            } else if (amb & 2) {
                for (int64_t i : cb) {
#pragma omp atomic write
                    touched_amb[i] = 1;
                }
            }
            terms.clear();
            pixel_terms(f, bl, T_final, g, bg, &terms);
            for (const auto& it : terms) {
                for (int q = 0; q < 9; ++q) {
#pragma omp atomic
                    grad2d[9 * it.first + q] += it.second[q];
#pragma omp atomic
                    grad2d_abs[9 * it.first + q] += std::fabs(it.second[q]);
                }
            }
            if (!straddle) continue;
            // each straddling decision taken the other way: the difference of every
            // Gaussian's terms between the two results is what that decision can move
            for (const Straddle& ev : events) {
                bl2.clear();
                double color2[3], T_final2;
                int32_t nc2;
                composite_pixel(f, cand, ppx, ppy, bg, band_alpha, band_T, color2, &T_final2, &nc2, &bl2, nullptr,
                                nullptr, &ev);
                terms2.clear();
                pixel_terms(f, bl2, T_final2, g, bg, &terms2);
                std::map<int64_t, std::array<double, 9>> diff;
                for (const auto& it : terms2) {
                    auto& d = diff[it.first];
                    for (int q = 0; q < 9; ++q) d[q] += it.second[q];
                }
                for (const auto& it : terms) {
                    auto& d = diff[it.first];
                    for (int q = 0; q < 9; ++q) d[q] -= it.second[q];
                }
                for (const auto& it : diff) {
                    for (int q = 0; q < 9; ++q) {
#pragma omp atomic
                        straddle[9 * it.first + q] += std::fabs(it.second[q]);
                    }
                }
            }
        }
    }
    return 0;
}

/* Chain 2D gradients (grad2d[9*k..] for Gaussian idx[k], or k when idx is NULL)
 * to the Gaussian's parameters by forward-mode dual numbers through the same
 * projection code.  Accumulates (+=) g_means[3], g_quats[4], g_log_scales[3],
 * g_logits[1], g_sh[3*nc] per listed Gaussian (indexed by k).  When
 * densify_accum is given, visible Gaussians also get
 * densify_accum += |(dL/du, dL/dv)| and densify_count += 1. */
int orc_project_bwd(int64_t n, const double* means, const double* quats, const double* log_scales,
                    const double* logits, const double* sh, int sh_degree, const orc_camera* ocam, const int64_t* idx, int64_t nidx,
                    const double* grad2d, double* g_means, double* g_quats, double* g_log_scales, double* g_logits,
                    double* g_sh, double* densify_accum, int32_t* densify_count) {
    if (sh_degree < 0 || sh_degree > 3) return 1;
    const Camera cam = to_cam(ocam);
    const int nc = (sh_degree + 1) * (sh_degree + 1);
    const int np = 11 + 3 * nc;
    const int64_t cnt = idx ? nidx : n;
#pragma omp parallel for schedule(dynamic, 256)
    for (int64_t k = 0; k < cnt; ++k) {
        const int64_t i = idx ? idx[k] : k;
        double P[11 + 48];
        load_params(i, means, quats, log_scales, logits, sh, nc, P);
        const Proj<double> p0 = project_one<double>(P, sh_degree, cam);
        if (!p0.visible) continue;
        const double* g = grad2d + 9 * k;
        Dual D[11 + 48];
        for (int j = 0; j < np; ++j) D[j] = Dual(P[j], 0.0);
        double grad[11 + 48];
        for (int j = 0; j < np; ++j) {
            D[j].d = 1.0;
            const Proj<Dual> pd = project_one<Dual>(D, sh_degree, cam);
            D[j].d = 0.0;
            const double outs[9] = {der(pd.u), der(pd.v), der(pd.A), der(pd.B), der(pd.C), der(pd.o),
                                    der(pd.rgb[0]), der(pd.rgb[1]), der(pd.rgb[2])};
            double s = 0.0;
            for (int q = 0; q < 9; ++q) s += g[q] * outs[q];
            grad[j] = s;
        }
        for (int j = 0; j < 3; ++j) g_means[3 * k + j] += grad[j];
        for (int j = 0; j < 4; ++j) g_quats[4 * k + j] += grad[3 + j];
        for (int j = 0; j < 3; ++j) g_log_scales[3 * k + j] += grad[7 + j];
        g_logits[k] += grad[10];
        for (int j = 0; j < 3 * nc; ++j) g_sh[(int64_t)3 * nc * k + j] += grad[11 + j];
        if (densify_accum) {
            densify_accum[k] += std::sqrt(g[0] * g[0] + g[1] * g[1]);
            densify_count[k] += 1;
        }
    }
    return 0;
}

/* One Adam step (bias-corrected) on float32 storage, arithmetic in double:
 * m = b1 m + (1-b1) g;  v = b2 v + (1-b2) g^2;
 * p -= lr * (m / (1-b1^t)) / (sqrt(v / (1-b2^t)) + eps). */
int orc_adam(int64_t count, float* param, const float* grad, float* m, float* v, double lr, double b1, double b2,
             double eps, int step) {
    const double bc1 = 1.0 - std::pow(b1, step), bc2 = 1.0 - std::pow(b2, step);
    for (int64_t i = 0; i < count; ++i) {
        const double gi = grad[i];
        const double mi = b1 * m[i] + (1.0 - b1) * gi;
        const double vi = b2 * v[i] + (1.0 - b2) * gi * gi;
        const double upd = lr * (mi / bc1) / (std::sqrt(vi / bc2) + eps);
        m[i] = (float)mi;
        v[i] = (float)vi;
        param[i] = (float)(param[i] - upd);
    }
    return 0;
}

/* L1 loss mean|img - tgt| over count values and its gradient
 * sign(img - tgt) / count (sign(0) = 0) stored as float32. */
double orc_l1(int64_t count, const float* img, const float* tgt, float* grad) {
    double s = 0.0;
    const float inv = (float)(1.0 / (double)count);
    for (int64_t i = 0; i < count; ++i) {
        const double d = (double)img[i] - (double)tgt[i];
        s += std::fabs(d);
        grad[i] = d > 0.0 ? inv : (d < 0.0 ? -inv : 0.0f);
    }
    return s / (double)count;
}

/* Adaptive density control (gsplat guide, lmnt.cn/news/262699, §4.1: every
 * 100 steps densify_and_prune with a gradient threshold, a minimum opacity, a
 * spatial extent and a maximum screen size; 3DGS deploy guide, hmyw.cn/news/140031,
 * §3.2: --densify_grad_threshold 0.0002).  The pages give only the four
 * parameters; the decision per Gaussian i, in this order:
 *   prune  unless sigmoid(logit) >= min_opacity, or when max_screen_radius > 0
 *          and the largest radius seen max_radius[i] > max_screen_radius;
 *   densify when count[i] > 0 and accum[i] / count[i] >= grad_threshold:
 *          clone (the Gaussian and an exact copy) if its largest scale
 *          exp(log_scale) <= scale_threshold, else split it into two children
 *          with means mu + R(q) (s * z_j) (z_j = noise[i][j], N(0, I) draws
 *          passed in), log-scales log_scale - log(1.6), the same rotation,
 *          opacity and SH;
 *   keep   otherwise.
 * Outputs keep input order: input i contributes 0 (prune), 1 (keep), or 2
 * (clone: itself then the copy; split: child 0 then child 1) consecutive
 * Gaussians.  source[k] is the input of output k and fresh[k] = 1 marks a new
 * Gaussian (the copy, both children), whose optimizer state starts at zero.
 * Decisions and values in double; returns the output count. */
int64_t orc_densify(int64_t n, int nc, const double* means, const double* quats, const double* log_scales,
                    const double* logits, const double* sh, const double* accum, const int32_t* count,
                    const int32_t* max_radius, const double* noise, double grad_threshold, double scale_threshold,
                    double min_opacity, int32_t max_screen_radius, uint8_t* decision, int64_t* source,
                    uint8_t* fresh, double* out_means, double* out_quats, double* out_log_scales,
                    double* out_logits, double* out_sh) {
    const double log_split = std::log(1.6);
    int64_t k = 0;
    auto emit = [&](int64_t i, bool is_new) {
        source[k] = i;
        fresh[k] = is_new ? 1 : 0;
        for (int c = 0; c < 3; ++c) out_means[3 * k + c] = means[3 * i + c];
        for (int c = 0; c < 4; ++c) out_quats[4 * k + c] = quats[4 * i + c];
        for (int c = 0; c < 3; ++c) out_log_scales[3 * k + c] = log_scales[3 * i + c];
        out_logits[k] = logits[i];
        for (int c = 0; c < 3 * nc; ++c) out_sh[3 * nc * k + c] = sh[3 * nc * i + c];
        return k++;
    };
    for (int64_t i = 0; i < n; ++i) {
        const double opacity = 1.0 / (1.0 + std::exp(-logits[i]));
        const bool prune = !(opacity >= min_opacity) || (max_screen_radius > 0 && max_radius[i] > max_screen_radius);
        const bool densify = count[i] > 0 && accum[i] / count[i] >= grad_threshold;
        if (prune) {
            decision[i] = 0;
            continue;
        }
        if (!densify) {
            decision[i] = 1;
            emit(i, false);
            continue;
        }
        const double ls_max = std::max(log_scales[3 * i], std::max(log_scales[3 * i + 1], log_scales[3 * i + 2]));
        if (std::exp(ls_max) <= scale_threshold) {
            decision[i] = 2;
            emit(i, false);
            emit(i, true);
            continue;
        }
        decision[i] = 3;
        // rotation of the normalised quaternion (w, x, y, z)
        const double* q = quats + 4 * i;
        const double qn = std::sqrt(q[0] * q[0] + q[1] * q[1] + q[2] * q[2] + q[3] * q[3]);
        const double w = q[0] / qn, x = q[1] / qn, y = q[2] / qn, z = q[3] / qn;
        const double R[3][3] = {{1 - 2 * (y * y + z * z), 2 * (x * y - w * z), 2 * (x * z + w * y)},
                                {2 * (x * y + w * z), 1 - 2 * (x * x + z * z), 2 * (y * z - w * x)},
                                {2 * (x * z - w * y), 2 * (y * z + w * x), 1 - 2 * (x * x + y * y)}};
        for (int j = 0; j < 2; ++j) {
            const int64_t o = emit(i, true);
            double sz[3];
            for (int c = 0; c < 3; ++c) sz[c] = std::exp(log_scales[3 * i + c]) * noise[6 * i + 3 * j + c];
            for (int r = 0; r < 3; ++r)
                out_means[3 * o + r] = means[3 * i + r] + (R[r][0] * sz[0] + R[r][1] * sz[1] + R[r][2] * sz[2]);
            for (int c = 0; c < 3; ++c) out_log_scales[3 * o + c] = log_scales[3 * i + c] - log_split;
        }
    }
    return k;
}

/* Structural similarity of the L1 + D-SSIM photometric loss (gsplat guide,
 * lmnt.cn/news/262699, §4.1: loss = l1_loss + 0.2 * (1 - ssim(render, gt))).
 * The pages do not define ssim(); this is the standard structural similarity:
 * per channel and pixel p, with w an 11x11 Gaussian window (standard deviation
 * 1.5, normalised to sum 1) centred on p and the images taken as 0 outside
 * their bounds,
 *   mx = sum w x, my = sum w y, sxx = sum w x^2 - mx^2, syy = sum w y^2 - my^2,
 *   sxy = sum w x y - mx my,
 *   S(p) = (2 mx my + C1)(2 sxy + C2) / ((mx^2 + my^2 + C1)(sxx + syy + C2)),
 * C1 = 0.01^2, C2 = 0.03^2 (dynamic range 1), and ssim = the mean of S over
 * pixels and channels.  Images are [H][W][ch].  Returns ssim; `map` (nullable)
 * receives S; `grad` (nullable) receives d ssim / d x, from
 *   dS(p)/dmx = S (2 my / a - 2 my / b - 2 mx / c + 2 mx / d),
 *   dS(p)/d(sum w x^2) = -S / d,  dS(p)/d(sum w x y) = 2 S / b
 * (a, b, c, d the four factors above) and the window weights, summed over
 * every p whose window covers the pixel.  Plain sums over the 2D window. */
double orc_ssim(int H, int W, int ch, const double* x, const double* y, double* map, double* grad) {
    const int R = 5;
    double g[2 * R + 1], gs = 0.0;
    for (int k = -R; k <= R; ++k) gs += g[k + R] = std::exp(-(double)(k * k) / (2.0 * 1.5 * 1.5));
    for (int k = 0; k <= 2 * R; ++k) g[k] /= gs;
    const double C1 = 0.01 * 0.01, C2 = 0.03 * 0.03;
    const int64_t n = (int64_t)H * W * ch;
    std::vector<double> dmx(grad ? n : 0), dxx(grad ? n : 0), dxy(grad ? n : 0);
    double total = 0.0;
#pragma omp parallel for reduction(+ : total) schedule(static)
    for (int py = 0; py < H; ++py)
        for (int px = 0; px < W; ++px)
            for (int c = 0; c < ch; ++c) {
                double mx = 0, my = 0, exx = 0, eyy = 0, exy = 0;
                for (int dy = -R; dy <= R; ++dy)
                    for (int dx = -R; dx <= R; ++dx) {
                        const int qy = py + dy, qx = px + dx;
                        if (qy < 0 || qy >= H || qx < 0 || qx >= W) continue;
                        const double w = g[dy + R] * g[dx + R];
                        const double xv = x[((int64_t)qy * W + qx) * ch + c], yv = y[((int64_t)qy * W + qx) * ch + c];
                        mx += w * xv;
                        my += w * yv;
                        exx += w * xv * xv;
                        eyy += w * yv * yv;
                        exy += w * xv * yv;
                    }
                const double a = 2 * mx * my + C1, b = 2 * (exy - mx * my) + C2;
                const double cc = mx * mx + my * my + C1, d = (exx - mx * mx) + (eyy - my * my) + C2;
                const double S = a * b / (cc * d);
                const int64_t i = ((int64_t)py * W + px) * ch + c;
                if (map) map[i] = S;
                total += S;
                if (grad) {
                    dmx[i] = S * (2 * my / a - 2 * my / b - 2 * mx / cc + 2 * mx / d);
                    dxx[i] = -S / d;
                    dxy[i] = 2 * S / b;
                }
            }
    if (grad) {
#pragma omp parallel for schedule(static)
        for (int qy = 0; qy < H; ++qy)
            for (int qx = 0; qx < W; ++qx)
                for (int c = 0; c < ch; ++c) {
                    const int64_t q = ((int64_t)qy * W + qx) * ch + c;
                    double s = 0.0;
                    for (int dy = -R; dy <= R; ++dy)
                        for (int dx = -R; dx <= R; ++dx) {
                            const int py = qy + dy, px = qx + dx;
                            if (py < 0 || py >= H || px < 0 || px >= W) continue;
                            const double w = g[dy + R] * g[dx + R];
                            const int64_t p = ((int64_t)py * W + px) * ch + c;
                            s += w * (dmx[p] + 2.0 * x[q] * dxx[p] + y[q] * dxy[p]);
                        }
                    grad[q] = s / (double)n;
                }
    }
    return total / (double)n;
}

/* Real SH basis values at unit directions dirs[3*k..] (degree <= 3), for pins. */
int orc_sh_basis(int64_t count, const double* dirs, int deg, double* Y) {
    const int nc = (deg + 1) * (deg + 1);
    for (int64_t k = 0; k < count; ++k) {
        double tmp[16];
        sh_basis<double>(deg, dirs[3 * k], dirs[3 * k + 1], dirs[3 * k + 2], tmp);
        for (int j = 0; j < nc; ++j) Y[nc * k + j] = tmp[j];
    }
    return 0;
}

int orc_set_threads(int t) {
    if (t > 0) omp_set_num_threads(t);
    return omp_get_max_threads();
}

}  // extern "C"
