// Causal multi-query attention, forward and backward, as plain fp32-FMA
// kernels (the fp32 debug precision, and any shape the tensor-core kernels
// do not take).  Model item: multi-query attention with causal masking
// (nanochat announcement, vpshk.cn, architecture list).
//
// Layout: qkv rows [B*T, (H+2nkv)*hd] hold q heads, then k heads, then v
// heads.  Query head h reads kv head h / (H/nkv).  Scores are scaled by
// 1/sqrt(hd); key j is visible to query i iff j <= i (same row of the batch).
//
// Forward and dQ: one warp per (query position, head); key tiles of 32 are
// staged in shared memory, each lane scores one key, and the output dims are
// spread over the lanes.  dK/dV: one warp per key position and kv head,
// looping over tiles of 32 (query position, head) rows in a fixed order, so
// results are deterministic.
#include "common.cuh"
#include "kernels.h"
#include <math.h>

namespace nc {
namespace {

constexpr int KT = 32;  // keys (or query rows) per tile
constexpr int WPB = 8;  // warps per block

template <typename A, int HD>
__global__ void __launch_bounds__(256) attn_fwd_kernel(const A* __restrict__ qkv, A* __restrict__ o,
                                                       float* __restrict__ lse, int T, int H, int nkv) {
    constexpr int NI = (HD + 31) / 32;
    __shared__ float Ks[KT][HD + 1];
    __shared__ float Vs[KT][HD];
    __shared__ float Qs[WPB][HD];
    const int ld = (H + 2 * nkv) * HD;
    int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int b = blockIdx.z, h = blockIdx.y, g = h / (H / nkv);
    int p = blockIdx.x * WPB + w;
    const A* base = qkv + (size_t)b * T * ld;
    bool live = p < T;
    for (int c = lane; c < HD; c += 32) Qs[w][c] = live ? tof(base[(size_t)p * ld + h * HD + c]) : 0.f;
    float m = -INFINITY, l = 0.f, acc[NI];
#pragma unroll
    for (int i = 0; i < NI; ++i) acc[i] = 0.f;
    const float scale = rsqrtf((float)HD);
    int last = min(T - 1, blockIdx.x * WPB + WPB - 1);
    for (int k0 = 0; k0 <= last; k0 += KT) {
        __syncthreads();
        for (int e = threadIdx.x; e < KT * HD; e += 256) {
            int r = e / HD, c = e % HD, j = k0 + r;
            bool ok = j < T;
            Ks[r][c] = ok ? tof(base[(size_t)j * ld + (H + g) * HD + c]) : 0.f;
            Vs[r][c] = ok ? tof(base[(size_t)j * ld + (H + nkv + g) * HD + c]) : 0.f;
        }
        __syncthreads();
        if (!live) continue;
        int j = k0 + lane;
        float s = -INFINITY;
        if (j <= p) {
            float dot = 0.f;
#pragma unroll 8
            for (int c = 0; c < HD; ++c) dot = fmaf(Qs[w][c], Ks[lane][c], dot);
            s = dot * scale;
        }
        float mt = warp_max(s);
        float mn = fmaxf(m, mt);
        float alpha = (m == -INFINITY) ? 0.f : expf(m - mn);
        float pj = (j <= p) ? expf(s - mn) : 0.f;
        l = l * alpha + warp_sum(pj);
#pragma unroll
        for (int i = 0; i < NI; ++i) acc[i] *= alpha;
        for (int jj = 0; jj < KT; ++jj) {
            float pb = __shfl_sync(0xffffffffu, pj, jj);
#pragma unroll
            for (int i = 0; i < NI; ++i) {
                int c = lane + 32 * i;
                if (c < HD) acc[i] = fmaf(pb, Vs[jj][c], acc[i]);
            }
        }
        m = mn;
    }
    if (!live) return;
    size_t row = (size_t)b * T + p;
    float inv = 1.f / l;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
        int c = lane + 32 * i;
        if (c < HD) o[row * (size_t)(H * HD) + h * HD + c] = fromf<A>(acc[i] * inv);
    }
    if (lane == 0) lse[((size_t)b * H + h) * attn_tpad(T) + p] = m + logf(l);
}

// D[b, h, t] = sum_c dO[row, h, c] * o[row, h, c]; one warp per (row, head).
template <typename A>
__global__ void attn_bwd_dot_kernel(const A* __restrict__ o, const A* __restrict__ dO, float* __restrict__ D,
                                    int MH, int T, int H, int hd) {
    int wid = blockIdx.x * WPB + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (wid >= MH) return;
    const A* a = o + (size_t)wid * hd;
    const A* b = dO + (size_t)wid * hd;
    float s = 0.f;
    for (int c = lane; c < hd; c += 32) s += tof(a[c]) * tof(b[c]);
    s = warp_sum(s);
    int row = wid / H, h = wid % H;
    if (lane == 0) D[((size_t)(row / T) * H + h) * attn_tpad(T) + row % T] = s;
}

template <typename A, int HD>
__global__ void __launch_bounds__(256) attn_bwd_dq_kernel(const A* __restrict__ qkv, const A* __restrict__ dO,
                                                          const float* __restrict__ lse,
                                                          const float* __restrict__ D, A* __restrict__ dqkv,
                                                          int T, int H, int nkv) {
    constexpr int NI = (HD + 31) / 32;
    __shared__ float Ks[KT][HD + 1];
    __shared__ float Vs[KT][HD + 1];
    __shared__ float Qs[WPB][HD];
    __shared__ float Gs[WPB][HD];
    const int ld = (H + 2 * nkv) * HD;
    int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int b = blockIdx.z, h = blockIdx.y, g = h / (H / nkv);
    int p = blockIdx.x * WPB + w;
    const A* base = qkv + (size_t)b * T * ld;
    bool live = p < T;
    size_t row = (size_t)b * T + (live ? p : 0);
    for (int c = lane; c < HD; c += 32) {
        Qs[w][c] = live ? tof(base[(size_t)p * ld + h * HD + c]) : 0.f;
        Gs[w][c] = live ? tof(dO[row * (size_t)(H * HD) + h * HD + c]) : 0.f;
    }
    const size_t si = ((size_t)b * H + h) * attn_tpad(T) + (live ? p : 0);
    float L = live ? lse[si] : 0.f;
    float Dr = live ? D[si] : 0.f;
    float acc[NI];
#pragma unroll
    for (int i = 0; i < NI; ++i) acc[i] = 0.f;
    const float scale = rsqrtf((float)HD);
    int last = min(T - 1, blockIdx.x * WPB + WPB - 1);
    for (int k0 = 0; k0 <= last; k0 += KT) {
        __syncthreads();
        for (int e = threadIdx.x; e < KT * HD; e += 256) {
            int r = e / HD, c = e % HD, j = k0 + r;
            bool ok = j < T;
            Ks[r][c] = ok ? tof(base[(size_t)j * ld + (H + g) * HD + c]) : 0.f;
            Vs[r][c] = ok ? tof(base[(size_t)j * ld + (H + nkv + g) * HD + c]) : 0.f;
        }
        __syncthreads();
        if (!live) continue;
        int j = k0 + lane;
        float ds = 0.f;
        if (j <= p) {
            float s = 0.f, dp = 0.f;
#pragma unroll 8
            for (int c = 0; c < HD; ++c) {
                s = fmaf(Qs[w][c], Ks[lane][c], s);
                dp = fmaf(Gs[w][c], Vs[lane][c], dp);
            }
            float P = expf(s * scale - L);
            ds = P * (dp - Dr);
        }
        for (int jj = 0; jj < KT; ++jj) {
            float db = __shfl_sync(0xffffffffu, ds, jj);
#pragma unroll
            for (int i = 0; i < NI; ++i) {
                int c = lane + 32 * i;
                if (c < HD) acc[i] = fmaf(db, Ks[jj][c], acc[i]);
            }
        }
    }
    if (!live) return;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
        int c = lane + 32 * i;
        if (c < HD) dqkv[row * ld + h * HD + c] = fromf<A>(acc[i] * scale);
    }
}

template <typename A, int HD>
__global__ void __launch_bounds__(256) attn_bwd_dkv_kernel(const A* __restrict__ qkv, const A* __restrict__ dO,
                                                           const float* __restrict__ lse,
                                                           const float* __restrict__ D, A* __restrict__ dqkv,
                                                           int T, int H, int nkv) {
    constexpr int NI = (HD + 31) / 32;
    __shared__ float Qs[KT][HD + 1];
    __shared__ float Gs[KT][HD + 1];
    __shared__ float Ls[KT], Ds[KT];
    __shared__ float Kw[WPB][HD], Vw[WPB][HD];
    const int ld = (H + 2 * nkv) * HD;
    const int Hg = H / nkv;
    int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    int b = blockIdx.z, g = blockIdx.y;
    int i0 = blockIdx.x * WPB;
    int j = i0 + w;
    const A* base = qkv + (size_t)b * T * ld;
    bool live = j < T;
    for (int c = lane; c < HD; c += 32) {
        Kw[w][c] = live ? tof(base[(size_t)j * ld + (H + g) * HD + c]) : 0.f;
        Vw[w][c] = live ? tof(base[(size_t)j * ld + (H + nkv + g) * HD + c]) : 0.f;
    }
    float dk[NI], dv[NI];
#pragma unroll
    for (int i = 0; i < NI; ++i) { dk[i] = 0.f; dv[i] = 0.f; }
    const float scale = rsqrtf((float)HD);
    int NR = (T - i0) * Hg;
    for (int r0 = 0; r0 < NR; r0 += KT) {
        __syncthreads();
        for (int e = threadIdx.x; e < KT * HD; e += 256) {
            int r = e / HD, c = e % HD, rr = r0 + r;
            bool ok = rr < NR;
            int qi = i0 + rr / Hg, hh = g * Hg + rr % Hg;
            size_t qrow = (size_t)b * T + qi;
            Qs[r][c] = ok ? tof(base[(size_t)qi * ld + hh * HD + c]) : 0.f;
            Gs[r][c] = ok ? tof(dO[qrow * (size_t)(H * HD) + hh * HD + c]) : 0.f;
        }
        if (threadIdx.x < KT) {
            int rr = r0 + threadIdx.x;
            bool ok = rr < NR;
            int qi = i0 + rr / Hg, hh = g * Hg + rr % Hg;
            size_t si = ((size_t)b * H + hh) * attn_tpad(T) + qi;
            Ls[threadIdx.x] = ok ? lse[si] : 0.f;
            Ds[threadIdx.x] = ok ? D[si] : 0.f;
        }
        __syncthreads();
        if (!live) continue;
        int rr = r0 + lane;
        int qi = i0 + rr / Hg;
        float P = 0.f, ds = 0.f;
        if (rr < NR && qi >= j) {
            float s = 0.f, dp = 0.f;
#pragma unroll 8
            for (int c = 0; c < HD; ++c) {
                s = fmaf(Qs[lane][c], Kw[w][c], s);
                dp = fmaf(Gs[lane][c], Vw[w][c], dp);
            }
            P = expf(s * scale - Ls[lane]);
            ds = P * (dp - Ds[lane]);
        }
        for (int t = 0; t < KT; ++t) {
            float pb = __shfl_sync(0xffffffffu, P, t);
            float db = __shfl_sync(0xffffffffu, ds, t);
#pragma unroll
            for (int i = 0; i < NI; ++i) {
                int c = lane + 32 * i;
                if (c < HD) {
                    dv[i] = fmaf(pb, Gs[t][c], dv[i]);
                    dk[i] = fmaf(db, Qs[t][c], dk[i]);
                }
            }
        }
    }
    if (!live) return;
    size_t row = (size_t)b * T + j;
#pragma unroll
    for (int i = 0; i < NI; ++i) {
        int c = lane + 32 * i;
        if (c < HD) {
            dqkv[row * ld + (H + g) * HD + c] = fromf<A>(dk[i] * scale);
            dqkv[row * ld + (H + nkv + g) * HD + c] = fromf<A>(dv[i]);
        }
    }
}

template <typename A, int HD>
cudaError_t fwd_t(const void* qkv, void* o, float* lse, int B, int T, int H, int nkv, cudaStream_t s) {
    dim3 grid((T + WPB - 1) / WPB, H, B);
    attn_fwd_kernel<A, HD><<<grid, 256, 0, s>>>((const A*)qkv, (A*)o, lse, T, H, nkv);
    count_launch();
    return cudaGetLastError();
}

template <typename A, int HD>
cudaError_t bwd_t(const void* qkv, const void* o, const void* dO, const float* lse, float* Dbuf, void* dqkv,
                  int B, int T, int H, int nkv, cudaStream_t s) {
    int MH = B * T * H;
    attn_bwd_dot_kernel<A><<<(MH + WPB - 1) / WPB, 256, 0, s>>>((const A*)o, (const A*)dO, Dbuf, MH, T, H, HD);
    dim3 gq((T + WPB - 1) / WPB, H, B);
    attn_bwd_dq_kernel<A, HD><<<gq, 256, 0, s>>>((const A*)qkv, (const A*)dO, lse, Dbuf, (A*)dqkv, T, H, nkv);
    dim3 gk((T + WPB - 1) / WPB, nkv, B);
    attn_bwd_dkv_kernel<A, HD><<<gk, 256, 0, s>>>((const A*)qkv, (const A*)dO, lse, Dbuf, (A*)dqkv, T, H, nkv);
    count_launch(3);
    return cudaGetLastError();
}

template <typename A>
cudaError_t fwd_d(const void* qkv, void* o, float* lse, int B, int T, int H, int nkv, int hd, cudaStream_t s) {
    switch (hd) {
        case 16: return fwd_t<A, 16>(qkv, o, lse, B, T, H, nkv, s);
        case 32: return fwd_t<A, 32>(qkv, o, lse, B, T, H, nkv, s);
        case 64: return fwd_t<A, 64>(qkv, o, lse, B, T, H, nkv, s);
        case 128: return fwd_t<A, 128>(qkv, o, lse, B, T, H, nkv, s);
    }
    return cudaErrorInvalidValue;
}

template <typename A>
cudaError_t bwd_d(const void* qkv, const void* o, const void* dO, const float* lse, float* Dbuf, void* dqkv,
                  int B, int T, int H, int nkv, int hd, cudaStream_t s) {
    switch (hd) {
        case 16: return bwd_t<A, 16>(qkv, o, dO, lse, Dbuf, dqkv, B, T, H, nkv, s);
        case 32: return bwd_t<A, 32>(qkv, o, dO, lse, Dbuf, dqkv, B, T, H, nkv, s);
        case 64: return bwd_t<A, 64>(qkv, o, dO, lse, Dbuf, dqkv, B, T, H, nkv, s);
        case 128: return bwd_t<A, 128>(qkv, o, dO, lse, Dbuf, dqkv, B, T, H, nkv, s);
    }
    return cudaErrorInvalidValue;
}

}  // namespace

cudaError_t launch_attention_fwd_simt(DType at, const void* qkv, void* o, float* lse, int B, int T, int H,
                                      int nkv, int hd, cudaStream_t s) {
    return at == DT_BF16 ? fwd_d<bf16>(qkv, o, lse, B, T, H, nkv, hd, s)
                         : fwd_d<float>(qkv, o, lse, B, T, H, nkv, hd, s);
}

cudaError_t launch_attention_bwd_dot(DType at, const void* o, const void* dO, float* D, int B, int T, int H, int hd,
                                     cudaStream_t s) {
    const int MH = B * T * H;
    if (at == DT_BF16)
        attn_bwd_dot_kernel<bf16><<<(MH + WPB - 1) / WPB, 256, 0, s>>>((const bf16*)o, (const bf16*)dO, D, MH, T, H,
                                                                       hd);
    else
        attn_bwd_dot_kernel<float><<<(MH + WPB - 1) / WPB, 256, 0, s>>>((const float*)o, (const float*)dO, D, MH, T,
                                                                        H, hd);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_attention_bwd_simt(DType at, const void* qkv, const void* o, const void* dO,
                                      const float* lse, float* Dbuf, void* dqkv, int B, int T, int H, int nkv,
                                      int hd, cudaStream_t s) {
    return at == DT_BF16 ? bwd_d<bf16>(qkv, o, dO, lse, Dbuf, dqkv, B, T, H, nkv, hd, s)
                         : bwd_d<float>(qkv, o, dO, lse, Dbuf, dqkv, B, T, H, nkv, hd, s);
}

}  // namespace nc
