// AdamW update of the flat parameter vector (the optimizer paragraph of the
// nanochat announcement, vpshk.cn, names Muon + AdamW and, as a plan, Adam with
// a learning rate per module; Muon is not defined there, AdamW is textbook):
// Adam's moment estimates (Kingma & Ba, "Adam", ICLR 2015) with the weight
// decay decoupled from the gradient (Loshchilov & Hutter, "Decoupled Weight
// Decay Regularization", ICLR 2019), per parameter group:
//   m <- b1 m + (1 - b1) g,  v <- b2 v + (1 - b2) g^2,
//   theta <- theta - lr (wd theta + (m / (1 - b1^t)) / (sqrt(v / (1 - b2^t)) + eps)).
// One memory-bound pass: fp32 master weights, moments and gradients in, the
// updated master weights and moments out, plus the compute copy of the weights
// in the step's type (bf16, rounded to nearest even, or fp32).
#include "nanochat_b200.h"
#include "common.cuh"
#include "kernels.h"

#include <cmath>

namespace nc {
namespace {

constexpr int kMaxGroups = NC_ADAMW_MAX_GROUPS;
constexpr int kThreads = 256;
constexpr int kPerThread = 8;                      // elements per thread (two 16-byte vectors)
constexpr int kChunk = kThreads * kPerThread;      // elements per block

struct GroupArg {
    int64_t offset, count;
    float lr, b1, b2, eps, wd, ibc1, ibc2;  // ibc* = 1 / (1 - b*^t)
};
struct AdamArgs {
    GroupArg g[kMaxGroups];
    int64_t block_start[kMaxGroups + 1];
    int n;
};

__device__ __forceinline__ uint32_t pack2(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ void adamw_one(const GroupArg& a, float& th, float& m, float& v, float g) {
    m = fmaf(a.b1, m, (1.f - a.b1) * g);
    v = fmaf(a.b2, v, (1.f - a.b2) * g * g);
    const float upd = (m * a.ibc1) / (sqrtf(v * a.ibc2) + a.eps);
    th = th - a.lr * fmaf(a.wd, th, upd);
}

template <typename W>
__global__ void __launch_bounds__(kThreads) adamw_kernel(const AdamArgs args, float* __restrict__ master,
                                                         W* __restrict__ weights, const float* __restrict__ grads,
                                                         float* __restrict__ mom1, float* __restrict__ mom2) {
    int gi = 0;
    while (gi + 1 < args.n && (int64_t)blockIdx.x >= args.block_start[gi + 1]) ++gi;
    const GroupArg& a = args.g[gi];
    const int64_t first = a.offset + ((int64_t)blockIdx.x - args.block_start[gi]) * kChunk;
    const int64_t end = a.offset + a.count;
    const int64_t i0 = first + (int64_t)threadIdx.x * kPerThread;
    if (i0 >= end) return;
    if (i0 + kPerThread <= end && (i0 & 7) == 0) {
        // two 16-byte vectors of every fp32 array (8-element aligned run)
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int64_t i = i0 + 4 * h;
            float4 th = *reinterpret_cast<const float4*>(master + i);
            float4 m = *reinterpret_cast<const float4*>(mom1 + i);
            float4 v = *reinterpret_cast<const float4*>(mom2 + i);
            const float4 g = *reinterpret_cast<const float4*>(grads + i);
            adamw_one(a, th.x, m.x, v.x, g.x);
            adamw_one(a, th.y, m.y, v.y, g.y);
            adamw_one(a, th.z, m.z, v.z, g.z);
            adamw_one(a, th.w, m.w, v.w, g.w);
            *reinterpret_cast<float4*>(master + i) = th;
            *reinterpret_cast<float4*>(mom1 + i) = m;
            *reinterpret_cast<float4*>(mom2 + i) = v;
            if constexpr (sizeof(W) == 4)
                *reinterpret_cast<float4*>(reinterpret_cast<float*>(weights) + i) = th;
            else
                *reinterpret_cast<uint2*>(weights + i) = make_uint2(pack2(th.x, th.y), pack2(th.z, th.w));
        }
    } else {
        for (int64_t i = i0; i < end && i < i0 + kPerThread; ++i) {
            float th = master[i], m = mom1[i], v = mom2[i];
            adamw_one(a, th, m, v, grads[i]);
            master[i] = th;
            mom1[i] = m;
            mom2[i] = v;
            weights[i] = fromf<W>(th);
        }
    }
}

}  // namespace
}  // namespace nc

extern "C" int nc_adamw_step(const nc_adamw_group* groups, int n_groups, int64_t n_params, int step,
                             float* master, void* weights, int weights_bf16, const float* grads, float* m, float* v,
                             void* stream) {
    using namespace nc;
    if (!groups || n_groups <= 0 || n_groups > kMaxGroups || step < 1 || n_params <= 0 || !master || !weights ||
        !grads || !m || !v)
        return NC_ERR_INVALID_ARG;
    auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
    if (!al16(master) || !al16(weights) || !al16(grads) || !al16(m) || !al16(v)) return NC_ERR_INVALID_ARG;
    AdamArgs args{};
    args.n = n_groups;
    int64_t blocks = 0;
    for (int i = 0; i < n_groups; ++i) {
        const nc_adamw_group& g = groups[i];
        if (g.offset < 0 || g.count < 0 || g.offset + g.count > n_params || !(g.beta1 >= 0.f && g.beta1 < 1.f) ||
            !(g.beta2 >= 0.f && g.beta2 < 1.f) || !(g.eps > 0.f) || !(g.lr >= 0.f) || !(g.weight_decay >= 0.f))
            return NC_ERR_INVALID_ARG;
        GroupArg& a = args.g[i];
        a.offset = g.offset;
        a.count = g.count;
        a.lr = g.lr; a.b1 = g.beta1; a.b2 = g.beta2; a.eps = g.eps; a.wd = g.weight_decay;
        a.ibc1 = (float)(1.0 / (1.0 - std::pow((double)g.beta1, (double)step)));
        a.ibc2 = (float)(1.0 / (1.0 - std::pow((double)g.beta2, (double)step)));
        args.block_start[i] = blocks;
        blocks += (g.count + kChunk - 1) / kChunk;
    }
    args.block_start[n_groups] = blocks;
    if (blocks == 0) return NC_OK;
    if (blocks > 0x7fffffff) return NC_ERR_UNSUPPORTED_SHAPE;
    cudaStream_t s = (cudaStream_t)stream;
    if (weights_bf16)
        adamw_kernel<bf16><<<(unsigned)blocks, kThreads, 0, s>>>(args, master, reinterpret_cast<bf16*>(weights), grads,
                                                                 m, v);
    else
        adamw_kernel<float><<<(unsigned)blocks, kThreads, 0, s>>>(args, master, reinterpret_cast<float*>(weights),
                                                                  grads, m, v);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}
