// L1 + D-SSIM photometric loss and its gradient with respect to the rendered
// image (gsplat guide, lmnt.cn/news/262699, §4.1: loss = l1_loss + 0.2 (1 - ssim)).
//
// ssim is the mean over pixels and channels of the structural similarity with
// an 11x11 Gaussian window (standard deviation 1.5), C1 = 0.01^2, C2 = 0.03^2,
// the images taken as zero outside their bounds.  Two stencil passes over
// 32x8 output tiles, each staging its tile plus a 5-pixel halo in shared memory
// and applying the separable window as a horizontal then a vertical 11-tap sum:
//   pass 1  the five windowed moments of every pixel and channel, S, and the
//           three partial derivatives of S (with respect to the windowed mean,
//           the windowed x^2 and the windowed x y), written to the workspace;
//           the loss terms reduced per block and added to the loss;
//   pass 2  the window applied to the partial-derivative maps (the adjoint of
//           the first pass's window sums; the window is symmetric), combined
//           with x and y into d ssim / d x, plus the L1 term's sign / count.
// Arithmetic is double precision: the moments cancel (var = E[x^2] - mean^2 at
// the scale of C2 = 9e-4) and the partial derivatives reach 1/C1 in dark
// regions, so float32 would lose several digits of the gradient.
#include <cmath>

#include "internal.cuh"

namespace gsk {
namespace {

constexpr int kR = 5;               // window radius
constexpr int kTaps = 2 * kR + 1;   // 11
constexpr int kTW = 32, kTH = 8;    // output tile
constexpr int kRW = kTW + 2 * kR;   // 42: tile plus halo
constexpr int kRH = kTH + 2 * kR;   // 18
constexpr int kThreads = kTW * kTH; // 256
constexpr double kC1 = 0.01 * 0.01, kC2 = 0.03 * 0.03;

struct SsimArgs {
    const float* x;  // image [H][W][3]
    const float* y;  // target
    int W, H;
    double g[kTaps];
    double inv_count;  // 1 / (3 H W)
    double l1_weight, ssim_weight;
    double* maps;  // [9][H][W]: plane 3 c + k, k = dS/dmean, dS/dE[x^2], dS/dE[xy] of channel c
    float* dL;
    double* loss;
};

__device__ __forceinline__ double block_sum(double v, double* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[w] = v;
    __syncthreads();
    double t = 0.0;
    if (threadIdx.x < 32) {
        t = lane < kThreads / 32 ? red[lane] : 0.0;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) t += __shfl_xor_sync(0xffffffffu, t, o);
    }
    return t;  // valid in thread 0
}

__global__ void __launch_bounds__(kThreads) ssim_moments_kernel(const SsimArgs a) {
    __shared__ float xs[3][kRH][kRW];
    __shared__ float ys[3][kRH][kRW];
    __shared__ double hs[5][kRH][kTW];
    __shared__ double red[kThreads / 32];
    const int x0 = blockIdx.x * kTW, y0 = blockIdx.y * kTH;
    // stage the tile and halo (zero outside the image), channel-interleaved rows
    for (int i = threadIdx.x; i < kRH * kRW * 3; i += kThreads) {
        const int r = i / (kRW * 3), k = i % (kRW * 3);
        const int col = k / 3, c = k % 3;
        const int gy = y0 - kR + r, gx = x0 - kR + col;
        const bool in = gy >= 0 && gy < a.H && gx >= 0 && gx < a.W;
        const int64_t off = (int64_t(gy) * a.W + gx) * 3 + c;
        xs[c][r][col] = in ? __ldg(a.x + off) : 0.f;
        ys[c][r][col] = in ? __ldg(a.y + off) : 0.f;
    }
    __syncthreads();
    const int tx = threadIdx.x % kTW, ty = threadIdx.x / kTW;
    const int px = x0 + tx, py = y0 + ty;
    const bool out_in = px < a.W && py < a.H;
    double s_sum = 0.0, l1_sum = 0.0;
    for (int c = 0; c < 3; ++c) {
        // horizontal window sums of x, y, x^2, y^2, x y
        for (int i = threadIdx.x; i < kRH * kTW; i += kThreads) {
            const int r = i / kTW, col = i % kTW;
            double m0 = 0, m1 = 0, m2 = 0, m3 = 0, m4 = 0;
#pragma unroll
            for (int k = 0; k < kTaps; ++k) {
                const double xv = xs[c][r][col + k], yv = ys[c][r][col + k], w = a.g[k];  // exact widening
                m0 = fma(w, xv, m0);
                m1 = fma(w, yv, m1);
                m2 = fma(w, xv * xv, m2);
                m3 = fma(w, yv * yv, m3);
                m4 = fma(w, xv * yv, m4);
            }
            hs[0][r][col] = m0;
            hs[1][r][col] = m1;
            hs[2][r][col] = m2;
            hs[3][r][col] = m3;
            hs[4][r][col] = m4;
        }
        __syncthreads();
        double mx = 0, my = 0, exx = 0, eyy = 0, exy = 0;
#pragma unroll
        for (int k = 0; k < kTaps; ++k) {
            const double w = a.g[k];
            mx = fma(w, hs[0][ty + k][tx], mx);
            my = fma(w, hs[1][ty + k][tx], my);
            exx = fma(w, hs[2][ty + k][tx], exx);
            eyy = fma(w, hs[3][ty + k][tx], eyy);
            exy = fma(w, hs[4][ty + k][tx], exy);
        }
        if (out_in) {
            const double A = 2.0 * mx * my + kC1, B = 2.0 * (exy - mx * my) + kC2;
            const double C = mx * mx + my * my + kC1, D = (exx - mx * mx) + (eyy - my * my) + kC2;
            const double S = A * B / (C * D);
            s_sum += S;
            const double xv = xs[c][ty + kR][tx + kR], yv = ys[c][ty + kR][tx + kR];
            l1_sum += fabs(xv - yv);
            const int64_t plane = int64_t(a.W) * a.H, pix = int64_t(py) * a.W + px;
            a.maps[(3 * c + 0) * plane + pix] = S * (2.0 * my / A - 2.0 * my / B - 2.0 * mx / C + 2.0 * mx / D);
            a.maps[(3 * c + 1) * plane + pix] = -S / D;
            a.maps[(3 * c + 2) * plane + pix] = 2.0 * S / B;
        }
        __syncthreads();
    }
    const double n_out = double(out_in ? 3 : 0);
    const double part = a.l1_weight * l1_sum + a.ssim_weight * (n_out - s_sum);
    const double tot = block_sum(part, red);
    if (threadIdx.x == 0) atomicAdd(a.loss, tot * a.inv_count);
}

__global__ void __launch_bounds__(kThreads) ssim_grad_kernel(const SsimArgs a) {
    __shared__ double fs[3][kRH][kRW];
    __shared__ double hs[3][kRH][kTW];
    const int x0 = blockIdx.x * kTW, y0 = blockIdx.y * kTH;
    const int tx = threadIdx.x % kTW, ty = threadIdx.x / kTW;
    const int px = x0 + tx, py = y0 + ty;
    const bool out_in = px < a.W && py < a.H;
    const int64_t plane = int64_t(a.W) * a.H;
    for (int c = 0; c < 3; ++c) {
        // this channel's three maps over the tile and halo (zero outside the image)
        for (int i = threadIdx.x; i < 3 * kRH * kRW; i += kThreads) {
            const int f = i / (kRH * kRW), rc = i % (kRH * kRW);
            const int r = rc / kRW, col = rc % kRW;
            const int gy = y0 - kR + r, gx = x0 - kR + col;
            const bool in = gy >= 0 && gy < a.H && gx >= 0 && gx < a.W;
            fs[f][r][col] = in ? a.maps[(3 * c + f) * plane + int64_t(gy) * a.W + gx] : 0.0;
        }
        __syncthreads();
        for (int i = threadIdx.x; i < kRH * kTW; i += kThreads) {
            const int r = i / kTW, col = i % kTW;
            double m0 = 0, m1 = 0, m2 = 0;
#pragma unroll
            for (int k = 0; k < kTaps; ++k) {
                const double w = a.g[k];
                m0 = fma(w, fs[0][r][col + k], m0);
                m1 = fma(w, fs[1][r][col + k], m1);
                m2 = fma(w, fs[2][r][col + k], m2);
            }
            hs[0][r][col] = m0;
            hs[1][r][col] = m1;
            hs[2][r][col] = m2;
        }
        __syncthreads();
        if (out_in) {
            double b0 = 0, b1 = 0, b2 = 0;
#pragma unroll
            for (int k = 0; k < kTaps; ++k) {
                const double w = a.g[k];
                b0 = fma(w, hs[0][ty + k][tx], b0);
                b1 = fma(w, hs[1][ty + k][tx], b1);
                b2 = fma(w, hs[2][ty + k][tx], b2);
            }
            const int64_t off = (int64_t(py) * a.W + px) * 3 + c;
            const double xv = __ldg(a.x + off), yv = __ldg(a.y + off);
            const double dssim = (b0 + 2.0 * xv * b1 + yv * b2) * a.inv_count;
            const double sgn = xv > yv ? 1.0 : (xv < yv ? -1.0 : 0.0);
            a.dL[off] = float(a.l1_weight * sgn * a.inv_count - a.ssim_weight * dssim);
        }
        __syncthreads();
    }
}

}  // namespace

cudaError_t launch_l1_dssim(const float* image, const float* target, int W, int H, float l1_weight,
                            float ssim_weight, double* maps, float* dL, double* loss, cudaStream_t s) {
    SsimArgs a;
    a.x = image;
    a.y = target;
    a.W = W;
    a.H = H;
    double sum = 0.0;
    for (int k = 0; k < kTaps; ++k) sum += a.g[k] = std::exp(-double((k - kR) * (k - kR)) / (2.0 * 1.5 * 1.5));
    for (int k = 0; k < kTaps; ++k) a.g[k] /= sum;
    a.inv_count = 1.0 / (3.0 * double(W) * double(H));
    a.l1_weight = l1_weight;
    a.ssim_weight = ssim_weight;
    a.maps = maps;
    a.dL = dL;
    a.loss = loss;
    const dim3 grid((W + kTW - 1) / kTW, (H + kTH - 1) / kTH);
    ssim_moments_kernel<<<grid, kThreads, 0, s>>>(a);
    ssim_grad_kernel<<<grid, kThreads, 0, s>>>(a);
    count_launches(2);
    return cudaGetLastError();
}

}  // namespace gsk
