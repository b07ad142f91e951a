// gs_raster_fwd / gs_raster_bwd: stage 3 of the pipeline, differentiable
// front-to-back alpha blending per 16x16 tile (gsplat guide, lmnt.cn/news/262699
// §2.1: shared-memory prefetch of the tile's Gaussians, SoA features, warp-level
// synchronisation; §2.2: a standalone backward entry).
//
// One CTA per tile, one pixel per thread.  Each batch of up to 256 list entries
// is gathered by Gaussian index into shared memory with cp.async (16-byte
// LDGSTS), double-buffered so the next batch is in flight while the current one
// is composited.  Both passes evaluate alpha with the same inline function and
// explicit rounding intrinsics, so the backward pass makes exactly the skip and
// clamp decisions the forward pass made.
//
// Conditioning: sigma = 1/2 (A dx^2 + C dy^2) + B dx dy cancels badly far along
// the long axis of a needle-shaped Gaussian (the terms grow with the condition
// number of the conic).  Entries whose conic has a condition number above
// kCondMax evaluate the quadratic form (and its derivatives in the backward pass)
// in double; the rest stay in float32, where the error is a few ulp of sigma.
#include "internal.cuh"

namespace gsk {
namespace {

constexpr float kAlphaMax = 0.99f;
constexpr float kAlphaMin = 1.0f / 255.0f;
constexpr float kTMin = 1e-4f;
constexpr float kLog2e = 1.4426950408889634f;
constexpr double kLog2eD = 1.4426950408889634;
// trace^2 / det = kappa + 1/kappa + 2 for the eigenvalue ratio kappa; 8 -> 10.125
constexpr float kCondMaxTraceSqOverDet = 10.125f;

constexpr int kBlock = kTilePixels;  // 256 threads, one pixel each

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
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

// Raw features of one list entry as gathered from global memory.
struct RawBuf {
    float2 xy[kBlock];
    float4 con[kBlock];  // A, B, C, o
    float4 rgb[kBlock];
    uint32_t gid[kBlock];
};

// Derived per-entry constants used by the per-pixel loop.
struct Prepped {
    float4 xyl;   // u, v, log2(o), ill-conditioned flag (0 or 1)
    float4 q;     // -log2e * A/2, -log2e * B, -log2e * C/2, 1/o
};

__device__ __forceinline__ Prepped prep(float2 xy, float4 con) {
    Prepped p;
    const float A = con.x, B = con.y, C = con.z, o = con.w;
    const float tr = A + C, det = A * C - B * B;
    const bool ill = !(det > 0.f) || (tr * tr > kCondMaxTraceSqOverDet * det);
    p.xyl = make_float4(xy.x, xy.y, log2f(o), ill ? 1.f : 0.f);
    p.q = make_float4(__fmul_rn(-0.5f * kLog2e, A), __fmul_rn(-kLog2e, B), __fmul_rn(-0.5f * kLog2e, C), 1.f / o);
    return p;
}

struct AlphaOut {
    float alpha;    // < kAlphaMin means "not blended"
    bool clamped;   // alpha hit 0.99
    float dx, dy;   // mean minus pixel centre
};

// alpha = min(0.99, o exp(-sigma)); 0 when sigma < 0.
__device__ __forceinline__ AlphaOut splat_alpha(const Prepped& p, const float4& con, float px, float py) {
    AlphaOut r;
    float s;  // -log2(e) * sigma
    if (p.xyl.w != 0.f) {
        const double dx = double(p.xyl.x) - double(px), dy = double(p.xyl.y) - double(py);
        const double sig = 0.5 * (double(con.x) * dx * dx + double(con.z) * dy * dy) + double(con.y) * dx * dy;
        s = float(-sig * kLog2eD);
        r.dx = float(dx);
        r.dy = float(dy);
    } else {
        r.dx = __fsub_rn(p.xyl.x, px);
        r.dy = __fsub_rn(p.xyl.y, py);
        const float qx = __fmaf_rn(p.q.y, r.dy, __fmul_rn(p.q.x, r.dx));
        s = __fmaf_rn(qx, r.dx, __fmul_rn(__fmul_rn(p.q.z, r.dy), r.dy));
    }
    if (s > 0.f) {
        r.alpha = 0.f;
        r.clamped = false;
        return r;
    }
    const float a = ex2_approx(__fadd_rn(s, p.xyl.z));
    r.clamped = a > kAlphaMax;
    r.alpha = r.clamped ? kAlphaMax : a;
    return r;
}

// Gather entries [first, first + count) of the sorted list into `buf`
// (entry e -> slot e - first, or reversed for the backward pass).
template <bool kReverse>
__device__ __forceinline__ void gather(RawBuf& buf, const uint32_t* __restrict__ vals, const float2* __restrict__ xy,
                                       const float4* __restrict__ con, const float4* __restrict__ rgb, uint32_t first,
                                       int count) {
    const int t = threadIdx.x;
    if (t < count) {
        const uint32_t e = kReverse ? first + uint32_t(count - 1 - t) : first + uint32_t(t);
        const uint32_t g = __ldg(vals + e);
        buf.gid[t] = g;
        cp_async8(&buf.xy[t], xy + g);
        cp_async16(&buf.con[t], con + g);
        cp_async16(&buf.rgb[t], rgb + g);
    }
    cp_async_commit();
}

struct FwdArgs {
    const float2* xy;
    const float4* con;
    const float4* rgb;
    const uint32_t* vals;
    const uint2* ranges;
    int W, H, TX;
    float bg0, bg1, bg2;
    float* image;
    float* final_T;
    int32_t* n_contrib;
};

__global__ void __launch_bounds__(kBlock) raster_fwd_kernel(const FwdArgs a) {
    __shared__ RawBuf buf[2];
    __shared__ Prepped pre[kBlock];
    const int tile = blockIdx.x;
    const int tx = tile % a.TX, ty = tile / a.TX;
    const int x = tx * kTile + (threadIdx.x & (kTile - 1));
    const int y = ty * kTile + (threadIdx.x >> 4);
    const bool inside = x < a.W && y < a.H;
    const float px = float(x) + 0.5f, py = float(y) + 0.5f;
    const uint2 range = a.ranges[tile];
    const int total = int(range.y - range.x);

    float T = 1.f, Cr = 0.f, Cg = 0.f, Cb = 0.f;
    int last = 0;
    bool done = !inside;

    int cur = 0;
    if (total > 0) gather<false>(buf[0], a.vals, a.xy, a.con, a.rgb, range.x, min(total, kBlock));
    for (int start = 0; start < total; start += kBlock) {
        const int count = min(total - start, kBlock);
        cp_async_wait_all();
        __syncthreads();  // batch `cur` landed; everyone finished reading `pre` and buf[cur ^ 1]
        if (__syncthreads_count(done) == kBlock) break;
        if (start + kBlock < total)
            gather<false>(buf[cur ^ 1], a.vals, a.xy, a.con, a.rgb, range.x + uint32_t(start + kBlock),
                          min(total - start - kBlock, kBlock));
        if (threadIdx.x < count) pre[threadIdx.x] = prep(buf[cur].xy[threadIdx.x], buf[cur].con[threadIdx.x]);
        __syncthreads();
        if (!done) {
            for (int j = 0; j < count; ++j) {
                const Prepped p = pre[j];
                const float4 con = buf[cur].con[j];
                const AlphaOut al = splat_alpha(p, con, px, py);
                if (al.alpha < kAlphaMin) continue;
                const float Tn = __fmul_rn(T, __fsub_rn(1.f, al.alpha));
                if (Tn < kTMin) {
                    done = true;
                    break;
                }
                const float4 c = buf[cur].rgb[j];
                const float w = __fmul_rn(al.alpha, T);
                Cr = __fmaf_rn(c.x, w, Cr);
                Cg = __fmaf_rn(c.y, w, Cg);
                Cb = __fmaf_rn(c.z, w, Cb);
                T = Tn;
                last = start + j + 1;
            }
        }
        cur ^= 1;
    }
    cp_async_wait_all();
    if (inside) {
        const int64_t pix = int64_t(y) * a.W + x;
        a.image[3 * pix + 0] = __fmaf_rn(T, a.bg0, Cr);
        a.image[3 * pix + 1] = __fmaf_rn(T, a.bg1, Cg);
        a.image[3 * pix + 2] = __fmaf_rn(T, a.bg2, Cb);
        a.final_T[pix] = T;
        a.n_contrib[pix] = last;
    }
}

struct BwdArgs {
    const float2* xy;
    const float4* con;
    const float4* rgb;
    const uint32_t* vals;
    const uint2* ranges;
    int W, H, TX;
    float bg0, bg1, bg2;
    const float* final_T;
    const int32_t* n_contrib;
    const float* dL_dimage;
    float2* g_xy;
    float4* g_con;
    float4* g_rgb;
};

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

__global__ void __launch_bounds__(kBlock) raster_bwd_kernel(const BwdArgs a) {
    __shared__ RawBuf buf[2];
    __shared__ Prepped pre[kBlock];
    __shared__ int max_last;
    const int tile = blockIdx.x;
    const int tx = tile % a.TX, ty = tile / a.TX;
    const int x = tx * kTile + (threadIdx.x & (kTile - 1));
    const int y = ty * kTile + (threadIdx.x >> 4);
    const bool inside = x < a.W && y < a.H;
    const float px = float(x) + 0.5f, py = float(y) + 0.5f;
    const uint2 range = a.ranges[tile];
    const int lane = threadIdx.x & 31;

    float T = 1.f, gr = 0.f, gg = 0.f, gb = 0.f, Tfinal = 1.f;
    int last = 0;
    if (inside) {
        const int64_t pix = int64_t(y) * a.W + x;
        Tfinal = a.final_T[pix];
        T = Tfinal;
        last = a.n_contrib[pix];
        gr = a.dL_dimage[3 * pix + 0];
        gg = a.dL_dimage[3 * pix + 1];
        gb = a.dL_dimage[3 * pix + 2];
    }
    const float bgg = a.bg0 * gr + a.bg1 * gg + a.bg2 * gb;
    float Sr = 0.f, Sg = 0.f, Sb = 0.f;

    if (threadIdx.x == 0) max_last = 0;
    __syncthreads();
    atomicMax(&max_last, last);
    __syncthreads();
    const int total = max_last;  // entries beyond every pixel's last blended one are never needed

    int cur = 0;
    // batches walk the list from the back: batch b covers positions [hi - count, hi)
    if (total > 0) {
        const int count0 = min(total, kBlock);
        gather<true>(buf[0], a.vals, a.xy, a.con, a.rgb, range.x + uint32_t(total - count0), count0);
    }
    for (int hi = total; hi > 0; hi -= kBlock) {
        const int count = min(hi, kBlock);
        cp_async_wait_all();
        __syncthreads();
        if (hi - kBlock > 0) {
            const int nhi = hi - kBlock, ncount = min(nhi, kBlock);
            gather<true>(buf[cur ^ 1], a.vals, a.xy, a.con, a.rgb, range.x + uint32_t(nhi - ncount), ncount);
        }
        if (threadIdx.x < count) pre[threadIdx.x] = prep(buf[cur].xy[threadIdx.x], buf[cur].con[threadIdx.x]);
        __syncthreads();
        for (int j = 0; j < count; ++j) {
            const int pos = hi - 1 - j;  // list position of this entry
            const Prepped p = pre[j];
            const float4 con = buf[cur].con[j];
            float g9[9] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            bool contrib = false;
            if (pos < last) {
                const AlphaOut al = splat_alpha(p, con, px, py);
                if (al.alpha >= kAlphaMin) {
                    contrib = true;
                    const float om = __fsub_rn(1.f, al.alpha);
                    const float rom = __frcp_rn(om);
                    T = __fmul_rn(T, rom);  // transmittance in front of this entry
                    const float4 c = buf[cur].rgb[j];
                    const float w = al.alpha * T;
                    g9[6] = w * gr;
                    g9[7] = w * gg;
                    g9[8] = w * gb;
                    const float dLda =
                        T * (gr * (c.x - Sr) + gg * (c.y - Sg) + gb * (c.z - Sb)) - Tfinal * bgg * rom;
                    Sr = __fmaf_rn(c.x, al.alpha, om * Sr);
                    Sg = __fmaf_rn(c.y, al.alpha, om * Sg);
                    Sb = __fmaf_rn(c.z, al.alpha, om * Sb);
                    if (!al.clamped) {
                        g9[5] = dLda * al.alpha * p.q.w;  // d alpha / d o = alpha / o
                        const float dLds = -dLda * al.alpha;
                        float su, sv;
                        if (p.xyl.w != 0.f) {
                            const double dx = double(p.xyl.x) - double(px), dy = double(p.xyl.y) - double(py);
                            su = float(double(con.x) * dx + double(con.y) * dy);
                            sv = float(double(con.y) * dx + double(con.z) * dy);
                        } else {
                            su = con.x * al.dx + con.y * al.dy;
                            sv = con.y * al.dx + con.z * al.dy;
                        }
                        g9[0] = dLds * su;
                        g9[1] = dLds * sv;
                        g9[2] = 0.5f * dLds * al.dx * al.dx;
                        g9[3] = dLds * al.dx * al.dy;
                        g9[4] = 0.5f * dLds * al.dy * al.dy;
                    }
                }
            }
            if (__any_sync(0xffffffffu, contrib)) {
#pragma unroll
                for (int q = 0; q < 9; ++q) g9[q] = warp_sum(g9[q]);
                if (lane == 0) {
                    const uint32_t gid = buf[cur].gid[j];
                    atomicAdd(a.g_xy + gid, make_float2(g9[0], g9[1]));
                    atomicAdd(a.g_con + gid, make_float4(g9[2], g9[3], g9[4], g9[5]));
                    atomicAdd(a.g_rgb + gid, make_float4(g9[6], g9[7], g9[8], 0.f));
                }
            }
        }
        cur ^= 1;
    }
    cp_async_wait_all();
}

}  // namespace

cudaError_t launch_raster_fwd(const gs_projected& proj, const uint32_t* vals, const uint32_t* ranges,
                              const CamArgs& cam, const float bg[3], float* image, float* final_T,
                              int32_t* n_contrib, cudaStream_t s) {
    FwdArgs a;
    a.xy = reinterpret_cast<const float2*>(proj.xy);
    a.con = reinterpret_cast<const float4*>(proj.conic_opacity);
    a.rgb = reinterpret_cast<const float4*>(proj.rgb);
    a.vals = vals;
    a.ranges = reinterpret_cast<const uint2*>(ranges);
    a.W = cam.W;
    a.H = cam.H;
    a.TX = cam.TX;
    a.bg0 = bg[0];
    a.bg1 = bg[1];
    a.bg2 = bg[2];
    a.image = image;
    a.final_T = final_T;
    a.n_contrib = n_contrib;
    raster_fwd_kernel<<<unsigned(cam.TX * cam.TY), kBlock, 0, s>>>(a);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_raster_bwd(const gs_projected& proj, const uint32_t* vals, const uint32_t* ranges,
                              const CamArgs& cam, const float bg[3], const float* final_T, const int32_t* n_contrib,
                              const float* dL_dimage, const gs_grad2d& g2, cudaStream_t s) {
    BwdArgs a;
    a.xy = reinterpret_cast<const float2*>(proj.xy);
    a.con = reinterpret_cast<const float4*>(proj.conic_opacity);
    a.rgb = reinterpret_cast<const float4*>(proj.rgb);
    a.vals = vals;
    a.ranges = reinterpret_cast<const uint2*>(ranges);
    a.W = cam.W;
    a.H = cam.H;
    a.TX = cam.TX;
    a.bg0 = bg[0];
    a.bg1 = bg[1];
    a.bg2 = bg[2];
    a.final_T = final_T;
    a.n_contrib = n_contrib;
    a.dL_dimage = dL_dimage;
    a.g_xy = reinterpret_cast<float2*>(g2.xy);
    a.g_con = reinterpret_cast<float4*>(g2.conic_opacity);
    a.g_rgb = reinterpret_cast<float4*>(g2.rgb);
    raster_bwd_kernel<<<unsigned(cam.TX * cam.TY), kBlock, 0, s>>>(a);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace gsk
