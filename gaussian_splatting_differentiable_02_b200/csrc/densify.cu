// Adaptive density control: per-Gaussian prune / keep / clone / split decisions
// from the accumulated screen-space gradient statistic, the opacity, the largest
// scale and the largest screen radius (gsplat guide, lmnt.cn/news/262699, §4.1:
// densify_and_prune with a gradient threshold, minimum opacity, extent and
// maximum screen size), then an order-preserving compaction of the parameters
// and their Adam moments into new arrays.
//
// Three launches:
//   plan     one block per contiguous chunk of Gaussians: decision per
//            Gaussian (uint8), and the chunk's output count;
//   offsets  one block: exclusive scan of the chunk counts, the total
//            (compact.cuh);
//   apply    the same chunks: block-wide scan of the per-Gaussian output counts
//            gives every Gaussian its output slot; parameters and moments are
//            copied (keep, clone), or the two split children are written.
// Memory-bound: the decision reads 32 bytes per Gaussian, the compaction moves
// the parameters and both moments (3 x 236 bytes at SH degree 3) in and out.
#include <cuda_runtime.h>

#include "compact.cuh"
#include "internal.cuh"

namespace gsk {
namespace {

using compact::block_inclusive_scan;
using compact::chunking;
using compact::Chunking;
using compact::kBlock;

struct PlanArgs {
    const float* logits;
    const float4* log_scales;
    const float* accum;
    const int32_t* count;
    const int32_t* max_radius;
    double grad_threshold, scale_threshold, min_opacity;
    int32_t max_screen_radius;
    int64_t n, chunk;
    uint8_t* decision;
    unsigned long long* chunk_counts;
};

// The larger of two values with a NaN first operand winning and a NaN second
// operand losing, as `a < b ? b : a` reads.
__device__ __forceinline__ double larger(double a, double b) { return a < b ? b : a; }

__device__ __forceinline__ int decide(const PlanArgs& a, int64_t i) {
    const double opacity = 1.0 / (1.0 + exp(-double(__ldg(a.logits + i))));
    const bool prune = !(opacity >= a.min_opacity) ||
                       (a.max_screen_radius > 0 && __ldg(a.max_radius + i) > a.max_screen_radius);
    if (prune) return GS_DENSIFY_PRUNE;
    const int c = __ldg(a.count + i);
    const bool densify = c > 0 && double(__ldg(a.accum + i)) / double(c) >= a.grad_threshold;
    if (!densify) return GS_DENSIFY_KEEP;
    const float4 ls = __ldg(a.log_scales + i);
    const double lmax = larger(double(ls.x), larger(double(ls.y), double(ls.z)));
    return exp(lmax) <= a.scale_threshold ? GS_DENSIFY_CLONE : GS_DENSIFY_SPLIT;
}

__device__ __forceinline__ int outputs_of(int d) { return d == GS_DENSIFY_PRUNE ? 0 : (d == GS_DENSIFY_KEEP ? 1 : 2); }

__global__ void __launch_bounds__(kBlock) densify_plan_kernel(const PlanArgs a) {
    __shared__ unsigned warp_tot[kBlock / 32];
    const int64_t begin = int64_t(blockIdx.x) * a.chunk;
    const int64_t end = begin + a.chunk < a.n ? begin + a.chunk : a.n;
    unsigned long long total = 0;
    for (int64_t base = begin; base < end; base += kBlock) {
        const int64_t i = base + threadIdx.x;
        unsigned c = 0;
        if (i < end) {
            const int d = decide(a, i);
            a.decision[i] = uint8_t(d);
            c = outputs_of(d);
        }
        unsigned tile_total;
        block_inclusive_scan(c, warp_tot, tile_total);
        total += tile_total;
    }
    if (threadIdx.x == 0) a.chunk_counts[blockIdx.x] = total;
}

struct Group {  // one set of parameter-shaped arrays
    const float4* means;
    const float4* quats;
    const float4* log_scales;
    const float* logits;
    const float4* sh;
};
struct OutGroup {
    float4* means;
    float4* quats;
    float4* log_scales;
    float* logits;
    float4* sh;
};

struct ApplyArgs {
    Group p, m, v;
    OutGroup op, om, ov;
    bool moments;
    const float* noise;  // [n][6]
    const uint8_t* decision;
    const unsigned long long* chunk_offsets;
    double log_split;
    int planes;
    int64_t n, n_out, chunk;
};

// One Gaussian's record of a parameter-shaped group, held in registers so that
// every load is issued before the first store.
struct Record {
    float4 means, quats, log_scales, sh[12];
    float logit;
};

__device__ __forceinline__ void load_record(const Group& g, int64_t i, int planes, int64_t n, Record& r) {
    r.means = __ldg(g.means + i);
    r.quats = __ldg(g.quats + i);
    r.log_scales = __ldg(g.log_scales + i);
    r.logit = __ldg(g.logits + i);
#pragma unroll
    for (int p = 0; p < 12; ++p)
        if (p < planes) r.sh[p] = __ldg(g.sh + int64_t(p) * n + i);
}

__device__ __forceinline__ void store_record(const OutGroup& o, int64_t k, int planes, int64_t n_out,
                                             const Record& r) {
    o.means[k] = r.means;
    o.quats[k] = r.quats;
    o.log_scales[k] = r.log_scales;
    o.logits[k] = r.logit;
#pragma unroll
    for (int p = 0; p < 12; ++p)
        if (p < planes) o.sh[int64_t(p) * n_out + k] = r.sh[p];
}

__device__ __forceinline__ void zero_group(const OutGroup& o, int64_t k, int planes, int64_t n_out) {
    const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
    o.means[k] = z;
    o.quats[k] = z;
    o.log_scales[k] = z;
    o.logits[k] = 0.f;
#pragma unroll
    for (int p = 0; p < 12; ++p)
        if (p < planes) o.sh[int64_t(p) * n_out + k] = z;
}

// Child j of a split from the parent's record: mean + R(q) (exp(log_scale) * z_j)
// and log_scale - log(1.6) (double precision, rounded once); the rotation,
// opacity and SH are the parent's.
__device__ __forceinline__ void store_child(const OutGroup& o, int64_t k, int planes, int64_t n_out,
                                            const Record& p, const float* z, double log_split) {
    const float4 mu = p.means, q4 = p.quats, ls = p.log_scales;
    const double qw = q4.x, qx = q4.y, qy = q4.z, qz = q4.w;
    const double qn = sqrt(((qw * qw + qx * qx) + qy * qy) + qz * qz);
    const double w = qw / qn, x = qx / qn, y = qy / qn, zz = qz / qn;
    const double R00 = 1.0 - 2.0 * (y * y + zz * zz), R01 = 2.0 * (x * y - w * zz), R02 = 2.0 * (x * zz + w * y);
    const double R10 = 2.0 * (x * y + w * zz), R11 = 1.0 - 2.0 * (x * x + zz * zz), R12 = 2.0 * (y * zz - w * x);
    const double R20 = 2.0 * (x * zz - w * y), R21 = 2.0 * (y * zz + w * x), R22 = 1.0 - 2.0 * (x * x + y * y);
    const double s0 = exp(double(ls.x)) * double(__ldg(z)), s1 = exp(double(ls.y)) * double(__ldg(z + 1)),
                 s2 = exp(double(ls.z)) * double(__ldg(z + 2));
    o.means[k] = make_float4(float(double(mu.x) + ((R00 * s0 + R01 * s1) + R02 * s2)),
                             float(double(mu.y) + ((R10 * s0 + R11 * s1) + R12 * s2)),
                             float(double(mu.z) + ((R20 * s0 + R21 * s1) + R22 * s2)), 0.f);
    o.log_scales[k] = make_float4(float(double(ls.x) - log_split), float(double(ls.y) - log_split),
                                  float(double(ls.z) - log_split), 0.f);
    o.quats[k] = q4;
    o.logits[k] = p.logit;
#pragma unroll
    for (int pl = 0; pl < 12; ++pl)
        if (pl < planes) o.sh[int64_t(pl) * n_out + k] = p.sh[pl];
}

__global__ void __launch_bounds__(kBlock) densify_apply_kernel(const ApplyArgs a) {
    __shared__ unsigned warp_tot[kBlock / 32];
    const int64_t begin = int64_t(blockIdx.x) * a.chunk;
    const int64_t end = begin + a.chunk < a.n ? begin + a.chunk : a.n;
    unsigned long long run = a.chunk_offsets[blockIdx.x];
    for (int64_t base = begin; base < end; base += kBlock) {
        const int64_t i = base + threadIdx.x;
        const int d = i < end ? int(a.decision[i]) : GS_DENSIFY_PRUNE;
        const unsigned c = outputs_of(d);
        unsigned tile_total;
        const unsigned incl = block_inclusive_scan(c, warp_tot, tile_total);
        const int64_t k = int64_t(run + (incl - c));
        run += tile_total;
        if (c == 0 || k + c > a.n_out) continue;
        Record r;
        load_record(a.p, i, a.planes, a.n, r);
        if (d == GS_DENSIFY_SPLIT) {
            store_child(a.op, k, a.planes, a.n_out, r, a.noise + 6 * i, a.log_split);
            store_child(a.op, k + 1, a.planes, a.n_out, r, a.noise + 6 * i + 3, a.log_split);
            if (a.moments) {
                zero_group(a.om, k, a.planes, a.n_out);
                zero_group(a.om, k + 1, a.planes, a.n_out);
                zero_group(a.ov, k, a.planes, a.n_out);
                zero_group(a.ov, k + 1, a.planes, a.n_out);
            }
            continue;
        }
        store_record(a.op, k, a.planes, a.n_out, r);
        if (d == GS_DENSIFY_CLONE) store_record(a.op, k + 1, a.planes, a.n_out, r);
        if (a.moments) {
            load_record(a.m, i, a.planes, a.n, r);
            store_record(a.om, k, a.planes, a.n_out, r);
            load_record(a.v, i, a.planes, a.n, r);
            store_record(a.ov, k, a.planes, a.n_out, r);
            if (d == GS_DENSIFY_CLONE) {
                zero_group(a.om, k + 1, a.planes, a.n_out);
                zero_group(a.ov, k + 1, a.planes, a.n_out);
            }
        }
    }
}

Group group_of(const gs_params& p) {
    return {reinterpret_cast<const float4*>(p.means), reinterpret_cast<const float4*>(p.quats),
            reinterpret_cast<const float4*>(p.log_scales), p.opacity_logits, reinterpret_cast<const float4*>(p.sh)};
}

OutGroup out_group_of(const gs_param_grads& g) {
    return {reinterpret_cast<float4*>(g.means), reinterpret_cast<float4*>(g.quats),
            reinterpret_cast<float4*>(g.log_scales), g.opacity_logits, reinterpret_cast<float4*>(g.sh)};
}

}  // namespace

size_t densify_workspace_layout(int64_t n, void* base, DensifyWorkspace* ws) {
    const Chunking ch = chunking(n);
    if (ws) {
        ws->chunk_counts = static_cast<unsigned long long*>(base);
        ws->total = ws->chunk_counts + ch.blocks;
        ws->blocks = ch.blocks;
        ws->chunk = ch.chunk;
    }
    return compact::workspace_bytes(n);
}

cudaError_t launch_densify_plan(const gs_params& p, const float* accum, const int32_t* count,
                                const int32_t* max_radius, const gs_densify_config& cfg,
                                const DensifyWorkspace& ws, uint8_t* decision, uint64_t* num_out_dev,
                                cudaStream_t s) {
    PlanArgs a;
    a.logits = p.opacity_logits;
    a.log_scales = reinterpret_cast<const float4*>(p.log_scales);
    a.accum = accum;
    a.count = count;
    a.max_radius = max_radius;
    a.grad_threshold = cfg.grad_threshold;
    a.scale_threshold = cfg.scale_threshold;
    a.min_opacity = cfg.min_opacity;
    a.max_screen_radius = max_radius ? cfg.max_screen_radius : 0;
    a.n = p.n;
    a.chunk = ws.chunk;
    a.decision = decision;
    a.chunk_counts = ws.chunk_counts;
    if (p.n > 0) {
        densify_plan_kernel<<<ws.blocks, kBlock, 0, s>>>(a);
        count_launches(1);
    } else {
        cudaMemsetAsync(ws.chunk_counts, 0, sizeof(unsigned long long) * ws.blocks, s);
    }
    compact::chunk_offsets_kernel<<<1, 1024, 0, s>>>(ws.chunk_counts, ws.blocks, ws.total,
                                              reinterpret_cast<unsigned long long*>(num_out_dev));
    count_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_densify_apply(const gs_params& p, const gs_params* m, const gs_params* v, const float* noise,
                                 const uint8_t* decision, const DensifyWorkspace& ws, int64_t n_out,
                                 const gs_param_grads& op, const gs_param_grads* om, const gs_param_grads* ov,
                                 double log_split, cudaStream_t s) {
    if (p.n == 0 || n_out == 0) return cudaSuccess;
    ApplyArgs a;
    a.p = group_of(p);
    a.op = out_group_of(op);
    a.moments = m != nullptr;
    if (a.moments) {
        a.m = group_of(*m);
        a.v = group_of(*v);
        a.om = out_group_of(*om);
        a.ov = out_group_of(*ov);
    }
    a.noise = noise;
    a.decision = decision;
    a.chunk_offsets = ws.chunk_counts;
    a.log_split = log_split;
    a.planes = sh_planes(p.sh_degree);
    a.n = p.n;
    a.n_out = n_out;
    a.chunk = ws.chunk;
    densify_apply_kernel<<<ws.blocks, kBlock, 0, s>>>(a);
    count_launches(1);
    return cudaGetLastError();
}

}  // namespace gsk
