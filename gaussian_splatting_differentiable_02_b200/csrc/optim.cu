// gs_adam and gs_l1_loss_grad: the optimiser step and the L1 photometric term
// of the training loop in the gsplat guide (lmnt.cn/news/262699) §4.1-4.2; and
// gs_to_half, the float32 -> FP16 rounding of parameters (the guides' FP16
// parameter storage).  All are streaming kernels: 128-bit loads, grid a multiple
// of the SM count.
#include <cuda_fp16.h>

#include "internal.cuh"

namespace gsk {
namespace {

struct AdamArgs {
    float* param;
    const float* grad;
    float* m;
    float* v;
    int64_t count;
    float lr_t;        // lr / (1 - beta1^t)
    float inv_sqrt_bc2;  // 1 / sqrt(1 - beta2^t)
    float b1, b2, eps;
};

__device__ __forceinline__ void adam_one(float& p, float g, float& m, float& v, const AdamArgs& a) {
    m = a.b1 * m + (1.f - a.b1) * g;
    v = a.b2 * v + (1.f - a.b2) * (g * g);
    p -= a.lr_t * m / (sqrtf(v) * a.inv_sqrt_bc2 + a.eps);
}

__global__ void __launch_bounds__(256) adam_kernel(const AdamArgs a) {
    const int64_t n4 = a.count >> 2;
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    float4* p4 = reinterpret_cast<float4*>(a.param);
    const float4* g4 = reinterpret_cast<const float4*>(a.grad);
    float4* m4 = reinterpret_cast<float4*>(a.m);
    float4* v4 = reinterpret_cast<float4*>(a.v);
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n4; i += stride) {
        float4 p = p4[i], m = m4[i], v = v4[i];
        const float4 g = __ldg(g4 + i);
        adam_one(p.x, g.x, m.x, v.x, a);
        adam_one(p.y, g.y, m.y, v.y, a);
        adam_one(p.z, g.z, m.z, v.z, a);
        adam_one(p.w, g.w, m.w, v.w, a);
        p4[i] = p;
        m4[i] = m;
        v4[i] = v;
    }
    for (int64_t i = (n4 << 2) + blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < a.count; i += stride)
        adam_one(a.param[i], a.grad[i], a.m[i], a.v[i], a);
}

__global__ void __launch_bounds__(256) l1_kernel(const float* __restrict__ img, const float* __restrict__ tgt,
                                                 int64_t count, float inv_count, double inv_count_d,
                                                 float* __restrict__ dL, double* loss) {
    __shared__ double partial[8];
    double s = 0.0;
    const int64_t n4 = count >> 2;
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    const float4* i4 = reinterpret_cast<const float4*>(img);
    const float4* t4 = reinterpret_cast<const float4*>(tgt);
    float4* d4 = reinterpret_cast<float4*>(dL);
    auto one = [&](float a, float b) {
        const float d = a - b;
        s += fabs(double(a) - double(b));
        return d > 0.f ? inv_count : (d < 0.f ? -inv_count : 0.f);
    };
    for (int64_t i = blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < n4; i += stride) {
        const float4 a = __ldg(i4 + i), b = __ldg(t4 + i);
        d4[i] = make_float4(one(a.x, b.x), one(a.y, b.y), one(a.z, b.z), one(a.w, b.w));
    }
    for (int64_t i = (n4 << 2) + blockIdx.x * int64_t(blockDim.x) + threadIdx.x; i < count; i += stride)
        dL[i] = one(img[i], tgt[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if ((threadIdx.x & 31) == 0) partial[threadIdx.x >> 5] = s;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int w = 0; w < 8; ++w) t += partial[w];
        atomicAdd(loss, t * inv_count_d);
    }
}

// Round to nearest even into IEEE half: four values per thread and step, then the tail.
__global__ void __launch_bounds__(256) to_half_kernel(const float* __restrict__ x, int64_t count,
                                                      uint16_t* __restrict__ out) {
    const int64_t q = count / 4;
    const int64_t stride = int64_t(gridDim.x) * blockDim.x;
    const int64_t first = blockIdx.x * int64_t(blockDim.x) + threadIdx.x;
    for (int64_t i = first; i < q; i += stride) {
        const float4 v = __ldg(reinterpret_cast<const float4*>(x) + i);
        const __half2 lo = __floats2half2_rn(v.x, v.y);
        const __half2 hi = __floats2half2_rn(v.z, v.w);
        uint2 w;
        w.x = *reinterpret_cast<const uint32_t*>(&lo);
        w.y = *reinterpret_cast<const uint32_t*>(&hi);
        reinterpret_cast<uint2*>(out)[i] = w;
    }
    for (int64_t i = 4 * q + first; i < count; i += stride) {
        const __half h = __float2half_rn(__ldg(x + i));
        out[i] = *reinterpret_cast<const uint16_t*>(&h);
    }
}

}  // namespace

cudaError_t launch_to_half(const float* x, int64_t count, uint16_t* out, cudaStream_t s) {
    if (count == 0) return cudaSuccess;
    to_half_kernel<<<grid_for((count + 3) / 4, 256, 8), 256, 0, s>>>(x, count, out);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_adam(float* param, const float* grad, float* m, float* v, int64_t count, float lr, float beta1,
                        float beta2, float eps, int32_t step, cudaStream_t s) {
    if (count == 0) return cudaSuccess;
    AdamArgs a;
    a.param = param;
    a.grad = grad;
    a.m = m;
    a.v = v;
    a.count = count;
    const double bc1 = 1.0 - pow(double(beta1), double(step));
    const double bc2 = 1.0 - pow(double(beta2), double(step));
    a.lr_t = float(double(lr) / bc1);
    a.inv_sqrt_bc2 = float(1.0 / sqrt(bc2));
    a.b1 = beta1;
    a.b2 = beta2;
    a.eps = eps;
    adam_kernel<<<grid_for((count + 3) / 4, 256, 8), 256, 0, s>>>(a);
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_l1(const float* image, const float* target, int64_t count, float* dL, double* loss,
                      cudaStream_t s) {
    if (count == 0) return cudaSuccess;
    const double inv = 1.0 / double(count);
    l1_kernel<<<grid_for((count + 3) / 4, 256, 8), 256, 0, s>>>(image, target, count, float(inv), inv, dL, loss);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace gsk
