// gs_alu_probe: throughput of the instruction classes the compositing kernels
// are built from, measured on the device at hand rather than taken from a data
// sheet.  The raster kernels are bound by arithmetic issue, not by HBM, so their
// roofline needs these denominators: float32 FMA (scalar and the paired
// FFMA2 form of sm_100), and the two special-function instructions they use per
// pixel and entry, ex2.approx (the exponential of alpha) and rcp.approx (the
// transmittance recovery of the reverse pass).
//
// Each thread runs kChains independent dependency chains of one instruction
// for `iters` iterations, entirely in registers (the rcp chain adds 1 before
// each reciprocal, an add on the FMA pipe, so that no two reciprocals cancel);
// the grid is 8 blocks of 256 threads per SM, so every scheduler has many warps
// to hide the latency.  The chains' final values are written out so that
// nothing is optimised away.
#include "internal.cuh"

namespace gsk {
namespace {

constexpr int kChains = 8;
constexpr int kProbeBlock = 256;
constexpr int kProbeBlocksPerSM = 8;

__device__ __forceinline__ float probe_ex2(float x) {
    float y;
    asm volatile("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float probe_rcp(float x) {
    float y;
    asm volatile("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// kOp: 0 scalar FFMA, 1 paired FFMA2, 2 ex2.approx, 3 rcp.approx
template <int kOp>
__global__ void __launch_bounds__(kProbeBlock) alu_probe_kernel(int64_t iters, float* __restrict__ out) {
    const int tid = blockIdx.x * blockDim.x + threadIdx.x;
    const float seed = 1e-3f * float(threadIdx.x & 63);
    float acc = 0.f;
    if (kOp == 1) {
        float2 a[kChains];
#pragma unroll
        for (int i = 0; i < kChains; ++i) a[i] = make_float2(seed + float(i), seed - float(i));
        const float2 m = make_float2(0.9999f, 0.9998f), c = make_float2(1e-7f, 2e-7f);
        for (int64_t k = 0; k < iters; ++k) {
#pragma unroll
            for (int i = 0; i < kChains; ++i) a[i] = __ffma2_rn(a[i], m, c);
        }
#pragma unroll
        for (int i = 0; i < kChains; ++i) acc += a[i].x + a[i].y;
    } else {
        float a[kChains];
#pragma unroll
        for (int i = 0; i < kChains; ++i) a[i] = seed + 0.01f * float(i + 1);
        for (int64_t k = 0; k < iters; ++k) {
#pragma unroll
            for (int i = 0; i < kChains; ++i) {
                if (kOp == 0) a[i] = fmaf(a[i], 0.9999f, 1e-7f);
                if (kOp == 2) a[i] = probe_ex2(-a[i]);  // stays in [0.5, 1]
                if (kOp == 3) a[i] = probe_rcp(a[i] + 1.f);  // x -> 1/(1 + x) stays in [0.5, 1]
            }
        }
#pragma unroll
        for (int i = 0; i < kChains; ++i) acc += a[i];
    }
    out[tid] = acc;
}

}  // namespace

int64_t alu_probe_threads() { return int64_t(kNumSMs) * kProbeBlocksPerSM * kProbeBlock; }

// Operations one launch performs: flops for the FMA forms (an FMA counts as
// two), instructions x lanes for the special functions.
double alu_probe_ops(int op, int64_t iters) {
    const double per_thread_iter = op == 0 ? 2.0 * kChains : op == 1 ? 4.0 * kChains : double(kChains);
    return per_thread_iter * double(iters) * double(alu_probe_threads());
}

cudaError_t launch_alu_probe(int op, int64_t iters, float* out, cudaStream_t s) {
    const unsigned grid = unsigned(kNumSMs * kProbeBlocksPerSM);
    switch (op) {
        case 0: alu_probe_kernel<0><<<grid, kProbeBlock, 0, s>>>(iters, out); break;
        case 1: alu_probe_kernel<1><<<grid, kProbeBlock, 0, s>>>(iters, out); break;
        case 2: alu_probe_kernel<2><<<grid, kProbeBlock, 0, s>>>(iters, out); break;
        default: alu_probe_kernel<3><<<grid, kProbeBlock, 0, s>>>(iters, out); break;
    }
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace gsk

extern "C" gs_status gs_alu_probe(int32_t op, int64_t iters, float* out, int64_t out_count, double* ops_host,
                                  void* stream) {
    const char* fn = "gs_alu_probe";
    if (op < GS_PROBE_FFMA || op > GS_PROBE_RCP)
        return gsk::fail_detail(GS_ERR_INVALID_ARG, "%s: op %d is not a GS_PROBE_* value", fn, int(op));
    if (iters < 1 || iters > (int64_t(1) << 30))
        return gsk::fail_detail(GS_ERR_INVALID_ARG, "%s: iters %lld outside [1, 2^30]", fn, (long long)iters);
    if (!out || !ops_host) return gsk::fail_detail(GS_ERR_INVALID_ARG, "%s: out or ops_host is NULL", fn);
    if (out_count < gsk::alu_probe_threads())
        return gsk::fail_detail(GS_ERR_INVALID_ARG, "%s: out holds %lld floats, %lld needed", fn,
                                (long long)out_count, (long long)gsk::alu_probe_threads());
    *ops_host = gsk::alu_probe_ops(op, iters);
    const cudaError_t e = gsk::launch_alu_probe(op, iters, out, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return gsk::fail_detail(GS_ERR_CUDA, "%s: %s", fn, cudaGetErrorString(e));
    return GS_OK;
}

extern "C" int64_t gs_alu_probe_slots(void) { return gsk::alu_probe_threads(); }
