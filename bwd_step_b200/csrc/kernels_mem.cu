// Memory-bound kernels of the step: token-embedding gather + norm, the
// parameter-free RMSNorm forward/backward, QK-norm fused with RoPE (forward
// and backward), the LM-head cross-entropy over a chunk of rows, the loss
// mean, the deterministic embedding-gradient scatter and the split-K reduce.
//
// Model items (nanochat announcement, vpshk.cn, architecture list): RMSNorm
// without learnable parameters, normalised token embedding, rotary embedding,
// QK-norm, logit softcap.  One warp owns one row (d % 64 == 0), every lane
// moves 8 elements per step with 16-byte accesses, and row statistics are
// reduced with warp shuffles.
#include "common.cuh"
#include "kernels.h"
#include <math.h>

namespace nc {

namespace {

__device__ __forceinline__ void load8(const float* p, float* o) { load_vec(p, o); load_vec(p + 4, o + 4); }
__device__ __forceinline__ void load8(const bf16* p, float* o) { load_vec(p, o); }
__device__ __forceinline__ void store8(float* p, const float* v) { store_vec(p, v); store_vec(p + 4, v + 4); }
__device__ __forceinline__ void store8(bf16* p, const float* v) { store_vec(p, v); }

constexpr int kRowWarps = 8;  // rows per 256-thread block

inline int row_blocks(int M) { return (M + kRowWarps - 1) / kRowWarps; }

// ---------------------------------------------------------------- RoPE table
__global__ void rope_table_kernel(float* c, float* s, int T, int hd, double base, int pos0) {
    int half = hd / 2;
    int i = blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= T * half) return;
    int pos = pos0 + i / half, j = i % half;
    double theta = pow(base, -2.0 * (double)j / (double)hd);
    double ang = (double)pos * theta;
    c[i] = (float)cos(ang);
    s[i] = (float)sin(ang);
}

// ---------------------------------------------------------------- embedding
template <typename W>
__global__ void embed_norm_fwd_kernel(const int32_t* __restrict__ idx, const W* __restrict__ wte, int M,
                                      int V, int d, float* __restrict__ x, float* __restrict__ r0,
                                      int* status) {
    int row = blockIdx.x * kRowWarps + (threadIdx.x >> 5);
    int lane = threadIdx.x & 31;
    if (row >= M) return;
    int id = idx[row];
    bool bad = id < 0 || id >= V;
    if (bad && lane == 0) set_status(status, ST_BAD_TOKEN);
    const W* src = wte + (size_t)(bad ? 0 : id) * d;
    float ss = 0.f;
    for (int c = lane * 8; c < d; c += 256) {
        float v[8];
        load8(src + c, v);
#pragma unroll
        for (int k = 0; k < 8; ++k) ss += v[k] * v[k];
    }
    ss = warp_sum(ss);
    float r = bad ? 0.f : rsqrtf(ss / (float)d + kRmsEps);
    float* dst = x + (size_t)row * d;
    for (int c = lane * 8; c < d; c += 256) {
        float v[8];
        load8(src + c, v);
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] *= r;
        store8(dst + c, v);
    }
    if (lane == 0) r0[row] = r;
}

template <typename W>
__global__ void embed_norm_bwd_kernel(const float* __restrict__ dx, const int32_t* __restrict__ idx,
                                      const W* __restrict__ wte, const float* __restrict__ r0,
                                      float* __restrict__ de, int M, int V, int d) {
    int row = blockIdx.x * kRowWarps + (threadIdx.x >> 5);
    int lane = threadIdx.x & 31;
    if (row >= M) return;
    int id = idx[row];
    bool bad = id < 0 || id >= V;
    const W* src = wte + (size_t)(bad ? 0 : id) * d;
    const float* g = dx + (size_t)row * d;
    float r = r0[row];
    float dot = 0.f;
    for (int c = lane * 8; c < d; c += 256) {
        float e[8], gg[8];
        load8(src + c, e);
        load8(g + c, gg);
#pragma unroll
        for (int k = 0; k < 8; ++k) dot += gg[k] * e[k] * r;
    }
    dot = warp_sum(dot) / (float)d;
    float* dst = de + (size_t)row * d;
    for (int c = lane * 8; c < d; c += 256) {
        float e[8], gg[8], o[8];
        load8(src + c, e);
        load8(g + c, gg);
#pragma unroll
        for (int k = 0; k < 8; ++k) o[k] = r * (gg[k] - e[k] * r * dot);
        store8(dst + c, o);
    }
}

// ---------------------------------------------------------------- RMSNorm
// One warp per row, lane l owns the 8-element chunks l*8 + 256*i.  With NCH > 0
// (d <= 256*NCH) the row stays in registers between the reduction and the
// output pass, so every input is read from memory once; NCH = 0 is the plain
// two-pass loop for wider rows.
template <typename A, int NCH>
__global__ void rmsnorm_fwd_kernel(const float* __restrict__ x, A* __restrict__ y, float* __restrict__ r,
                                   int M, int d) {
    int row = blockIdx.x * kRowWarps + (threadIdx.x >> 5);
    int lane = threadIdx.x & 31;
    if (row >= M) return;
    const float* src = x + (size_t)row * d;
    A* dst = y + (size_t)row * d;
    float ss = 0.f;
    if constexpr (NCH > 0) {
        float v[NCH][8];
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
            const int c = lane * 8 + 256 * i;
            if (c < d) load8(src + c, v[i]);
        }
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
            if (lane * 8 + 256 * i < d) {
#pragma unroll
                for (int k = 0; k < 8; ++k) ss += v[i][k] * v[i][k];
            }
        }
        ss = warp_sum(ss);
        const float rr = rsqrtf(ss / (float)d + kRmsEps);
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
            const int c = lane * 8 + 256 * i;
            if (c < d) {
#pragma unroll
                for (int k = 0; k < 8; ++k) v[i][k] *= rr;
                store8(dst + c, v[i]);
            }
        }
        if (lane == 0) r[row] = rr;
    } else {
        for (int c = lane * 8; c < d; c += 256) {
            float v[8];
            load8(src + c, v);
#pragma unroll
            for (int k = 0; k < 8; ++k) ss += v[k] * v[k];
        }
        ss = warp_sum(ss);
        const float rr = rsqrtf(ss / (float)d + kRmsEps);
        for (int c = lane * 8; c < d; c += 256) {
            float v[8];
            load8(src + c, v);
#pragma unroll
            for (int k = 0; k < 8; ++k) v[k] *= rr;
            store8(dst + c, v);
        }
        if (lane == 0) r[row] = rr;
    }
}

template <typename A, typename DY, int NCH>
__global__ void rmsnorm_bwd_kernel(const DY* __restrict__ dy, const A* __restrict__ y,
                                   const float* __restrict__ r, float* dx, bool accumulate, A* dxb,
                                   int M, int d) {
    int row = blockIdx.x * kRowWarps + (threadIdx.x >> 5);
    int lane = threadIdx.x & 31;
    if (row >= M) return;
    const DY* g = dy + (size_t)row * d;
    const A* yy = y + (size_t)row * d;
    float* out = dx + (size_t)row * d;
    const float rr = r[row];
    float dot = 0.f;
    if constexpr (NCH > 0) {
        float a[NCH][8], b[NCH][8];
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
            const int c = lane * 8 + 256 * i;
            if (c < d) {
                load8(g + c, a[i]);
                load8(yy + c, b[i]);
            }
        }
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
            if (lane * 8 + 256 * i < d) {
#pragma unroll
                for (int k = 0; k < 8; ++k) dot += a[i][k] * b[i][k];
            }
        }
        dot = warp_sum(dot) / (float)d;
        // the row's contribution into a (b is dead afterwards), then every chunk of the
        // accumulated gradient loaded at once into b's registers (the loads in flight
        // together), added and stored
#pragma unroll
        for (int i = 0; i < NCH; ++i)
#pragma unroll
            for (int k = 0; k < 8; ++k) a[i][k] = rr * (a[i][k] - b[i][k] * dot);
        if (accumulate) {
#pragma unroll
            for (int i = 0; i < NCH; ++i) {
                const int c = lane * 8 + 256 * i;
                if (c < d) load8(out + c, b[i]);
            }
#pragma unroll
            for (int i = 0; i < NCH; ++i)
#pragma unroll
                for (int k = 0; k < 8; ++k) a[i][k] += b[i][k];
        }
#pragma unroll
        for (int i = 0; i < NCH; ++i) {
            const int c = lane * 8 + 256 * i;
            if (c < d) {
                store8(out + c, a[i]);
                if (dxb) store8(dxb + (size_t)row * d + c, a[i]);
            }
        }
    } else {
        for (int c = lane * 8; c < d; c += 256) {
            float a[8], b[8];
            load8(g + c, a);
            load8(yy + c, b);
#pragma unroll
            for (int k = 0; k < 8; ++k) dot += a[k] * b[k];
        }
        dot = warp_sum(dot) / (float)d;
        for (int c = lane * 8; c < d; c += 256) {
            float a[8], b[8], o[8];
            load8(g + c, a);
            load8(yy + c, b);
            if (accumulate) load8(out + c, o);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                float v = rr * (a[k] - b[k] * dot);
                o[k] = accumulate ? o[k] + v : v;
            }
            store8(out + c, o);
            if (dxb) store8(dxb + (size_t)row * d + c, o);
        }
    }
}

// ---------------------------------------------------------------- QK-norm + RoPE
// A warp handles a head vector of HD elements at a time (the forward one per
// warp, the backward all heads of a position).  Lane l holds EPL = HD/32
// consecutive elements (HD = 16: lanes 0..15 one each); the pair partner of
// element j < HD/2 is element j + HD/2, held by lane l ^ (HD/2/EPL).  Every
// access is a contiguous EPL-element vector, so a warp reads and writes each
// head vector in one coalesced request.
template <int HD> struct QkShape {
    static constexpr int EPL = HD >= 32 ? HD / 32 : 1;       // elements per lane
    static constexpr int LANES = HD / EPL;                    // active lanes
    static constexpr int XOR = (HD / 2) / EPL;                // partner lane offset
};

// N-element vector access (N*sizeof(A) bytes, naturally aligned here).
template <typename A, int N>
__device__ __forceinline__ void ldN(const A* p, float* v) {
    if constexpr (sizeof(A) == 2 && N == 4) {
        uint2 u = *reinterpret_cast<const uint2*>(p);
        float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u.x));
        float2 b = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162*>(&u.y));
        v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
    } else if constexpr (sizeof(A) == 2 && N == 2) {
        float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(p));
        v[0] = a.x; v[1] = a.y;
    } else if constexpr (sizeof(A) == 4 && N == 4) {
        float4 a = *reinterpret_cast<const float4*>(p);
        v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    } else if constexpr (sizeof(A) == 4 && N == 2) {
        float2 a = *reinterpret_cast<const float2*>(p);
        v[0] = a.x; v[1] = a.y;
    } else {
#pragma unroll
        for (int i = 0; i < N; ++i) v[i] = tof(p[i]);
    }
}
template <typename A, int N>
__device__ __forceinline__ void stN(A* p, const float* v) {
    if constexpr (sizeof(A) == 2 && N == 4) {
        __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), b = __floats2bfloat162_rn(v[2], v[3]);
        uint2 u;
        u.x = *reinterpret_cast<uint32_t*>(&a);
        u.y = *reinterpret_cast<uint32_t*>(&b);
        *reinterpret_cast<uint2*>(p) = u;
    } else if constexpr (sizeof(A) == 2 && N == 2) {
        *reinterpret_cast<__nv_bfloat162*>(p) = __floats2bfloat162_rn(v[0], v[1]);
    } else if constexpr (sizeof(A) == 4 && N == 4) {
        *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    } else if constexpr (sizeof(A) == 4 && N == 2) {
        *reinterpret_cast<float2*>(p) = make_float2(v[0], v[1]);
    } else {
#pragma unroll
        for (int i = 0; i < N; ++i) p[i] = fromf<A>(v[i]);
    }
}

template <typename A, int HD>
__global__ void __launch_bounds__(256) qknorm_rope_fwd_kernel(A* qkv, float* __restrict__ rqk,
                                                              const float* __restrict__ cos_t,
                                                              const float* __restrict__ sin_t, int M, int T, int H,
                                                              int nkv) {
    using S = QkShape<HD>;
    const int nh = H + nkv;
    const int vi = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (vi >= M * nh) return;
    const int m = vi / nh, head = vi % nh, pos = m % T;
    const bool act = lane < S::LANES;
    const int l = act ? lane : 0;
    A* v = qkv + (size_t)m * (size_t)(H + 2 * nkv) * HD + (size_t)head * HD + l * S::EPL;
    float x[S::EPL];
    ldN<A, S::EPL>(v, x);
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < S::EPL; ++i) ss += act ? x[i] * x[i] : 0.f;
    ss = warp_sum(ss);
    const float r = rsqrtf(ss / (float)HD + kRmsEps);
    const bool first = l * S::EPL < HD / 2;                   // holds x1 of its pairs
    const int j0 = first ? l * S::EPL : l * S::EPL - HD / 2;   // pair index of element 0
    float y[S::EPL];
#pragma unroll
    for (int i = 0; i < S::EPL; ++i) {
        const float other = __shfl_xor_sync(0xffffffffu, x[i], S::XOR);
        const float c = cos_t[pos * (HD / 2) + j0 + i], s = sin_t[pos * (HD / 2) + j0 + i];
        const float a = (first ? x[i] : other) * r, b = (first ? other : x[i]) * r;
        y[i] = first ? a * c - b * s : a * s + b * c;
    }
    if (!act) return;
    stN<A, S::EPL>(v, y);
    if (lane == 0) rqk[(size_t)m * nh + head] = r;
}

// One warp per position: the RoPE factors are loaded once, and the head
// vectors of the position are processed G at a time with all their loads
// issued before any of them is used.
template <typename A, int HD>
__global__ void __launch_bounds__(256, 4) qknorm_rope_bwd_kernel(A* dqkv, const A* __restrict__ qkv,
                                                              const float* __restrict__ rqk,
                                                              const float* __restrict__ cos_t,
                                                              const float* __restrict__ sin_t, int M, int T, int H,
                                                              int nkv) {
    using S = QkShape<HD>;
    constexpr int G = 4;
    const int nh = H + nkv;
    const int m = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
    if (m >= M) return;
    const int pos = m % T;
    const bool act = lane < S::LANES;
    const int l = act ? lane : 0;
    const bool first = l * S::EPL < HD / 2;
    const int j0 = first ? l * S::EPL : l * S::EPL - HD / 2;  // pair index of element 0
    float cs[S::EPL], sn[S::EPL];
    ldN<float, S::EPL>(cos_t + (size_t)pos * (HD / 2) + j0, cs);
    ldN<float, S::EPL>(sin_t + (size_t)pos * (HD / 2) + j0, sn);
    const size_t rowoff = (size_t)m * (size_t)(H + 2 * nkv) * HD + l * S::EPL;
    for (int h0 = 0; h0 < nh; h0 += G) {
        float g[G][S::EPL], y[G][S::EPL], r[G];
#pragma unroll
        for (int k = 0; k < G; ++k) {
            if (h0 + k < nh) {
                ldN<A, S::EPL>(dqkv + rowoff + (size_t)(h0 + k) * HD, g[k]);
                ldN<A, S::EPL>(qkv + rowoff + (size_t)(h0 + k) * HD, y[k]);
                r[k] = rqk[(size_t)m * nh + h0 + k];
            }
        }
#pragma unroll
        for (int k = 0; k < G; ++k) {
            if (h0 + k >= nh) break;
            float gu[S::EPL], yu[S::EPL], dot = 0.f;
#pragma unroll
            for (int i = 0; i < S::EPL; ++i) {
                const float go = __shfl_xor_sync(0xffffffffu, g[k][i], S::XOR);
                const float yo = __shfl_xor_sync(0xffffffffu, y[k][i], S::XOR);
                // inverse rotation of (x1, x2): (x1 c + x2 s, -x1 s + x2 c)
                const float g1 = first ? g[k][i] : go, g2 = first ? go : g[k][i];
                const float y1 = first ? y[k][i] : yo, y2 = first ? yo : y[k][i];
                gu[i] = first ? g1 * cs[i] + g2 * sn[i] : -g1 * sn[i] + g2 * cs[i];
                yu[i] = first ? y1 * cs[i] + y2 * sn[i] : -y1 * sn[i] + y2 * cs[i];
                dot += act ? gu[i] * yu[i] : 0.f;
            }
            dot = warp_sum(dot) / (float)HD;
#pragma unroll
            for (int i = 0; i < S::EPL; ++i) gu[i] = r[k] * (gu[i] - yu[i] * dot);
            if (act) stN<A, S::EPL>(dqkv + rowoff + (size_t)(h0 + k) * HD, gu);
        }
    }
}

// ---------------------------------------------------------------- cross-entropy
struct MaxSum { float m, s; };

__device__ __forceinline__ MaxSum ms_combine(MaxSum a, MaxSum b) {
    if (b.s == 0.f) return a;
    if (a.s == 0.f) return b;
    float m = fmaxf(a.m, b.m);
    return {m, a.s * __expf(a.m - m) + b.s * __expf(b.m - m)};
}

__device__ __forceinline__ void store4(float* p, const float* v) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void store4(bf16* p, const float* v) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), b = __floats2bfloat162_rn(v[2], v[3]);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t*>(&a);
    u.y = *reinterpret_cast<uint32_t*>(&b);
    *reinterpret_cast<uint2*>(p) = u;
}

// four logits (fp32 or bf16) as floats
__device__ __forceinline__ void load4z(const float* p, float* v) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
}
__device__ __forceinline__ void load4z(const bf16* p, float* v) {
    const uint2 u = *reinterpret_cast<const uint2*>(p);
    const float2 a = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.x));
    const float2 b = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&u.y));
    v[0] = a.x; v[1] = a.y; v[2] = b.x; v[3] = b.y;
}

// Loss and dl of one chunk of rows, one 1024-thread block per row (V % 4 == 0).
// Pass 1: running (max, sum of exp) over the row's softcapped logits z, two
// vectors of 4 logits in flight per thread (two blocks per SM); the block combines the partials
// into the LSE.  Pass 2 reads the row again (from L2: about 300 rows are in
// flight) and writes dl = (softmax - onehot) / M * (1 - (z/cap)^2).
template <typename Z, typename D>
__global__ void __launch_bounds__(1024, 2) ce_chunk_kernel(const Z* __restrict__ z, const int32_t* __restrict__ tgt,
                                                        int R, int V, float cap, float inv_M,
                                                        float* __restrict__ loss_rows, D* __restrict__ dl,
                                                        int* status) {
    constexpr float kL2e = 1.44269504088896340736f;
    constexpr int U = 2;
    __shared__ MaxSum red[32];
    __shared__ float s_lse;
    const int row = blockIdx.x;
    const Z* zr = z + (size_t)row * V;
    const int stride = blockDim.x * 4;
    MaxSum acc = {-INFINITY, 0.f};
    for (int c0 = threadIdx.x * 4; c0 < V; c0 += U * stride) {
        float v[U][4];
        float m = acc.m;
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = c0 + u * stride;
            if (c < V) {
                load4z(zr + c, v[u]);
            } else {
                v[u][0] = v[u][1] = v[u][2] = v[u][3] = -INFINITY;
            }
            m = fmaxf(m, fmaxf(fmaxf(v[u][0], v[u][1]), fmaxf(v[u][2], v[u][3])));
        }
        const float m2 = m * kL2e;
        float sacc = acc.s == 0.f ? 0.f : acc.s * exp2f(fmaf(acc.m, kL2e, -m2));
#pragma unroll
        for (int u = 0; u < U; ++u)
#pragma unroll
            for (int k = 0; k < 4; ++k) sacc += exp2f(fmaf(v[u][k], kL2e, -m2));
        acc = {m, sacc};
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        MaxSum other = {__shfl_xor_sync(0xffffffffu, acc.m, o), __shfl_xor_sync(0xffffffffu, acc.s, o)};
        acc = ms_combine(acc, other);
    }
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (lane == 0) red[w] = acc;
    __syncthreads();
    if (w == 0) {
        const int nw = blockDim.x >> 5;
        acc = lane < nw ? red[lane] : MaxSum{-INFINITY, 0.f};
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            MaxSum other = {__shfl_xor_sync(0xffffffffu, acc.m, o), __shfl_xor_sync(0xffffffffu, acc.s, o)};
            acc = ms_combine(acc, other);
        }
        if (lane == 0) s_lse = acc.m + logf(acc.s);
    }
    __syncthreads();
    const float lse = s_lse;
    const int t = tgt[row];
    const bool bad = t < 0 || t >= V;
    if (threadIdx.x == 0) {
        if (bad) set_status(status, ST_BAD_TOKEN);
        loss_rows[row] = bad ? 0.f : lse - tof(zr[t]);
    }
    const float inv_cap = 1.f / cap, lse2 = lse * kL2e;
    D* out = dl + (size_t)row * V;
    for (int c0 = threadIdx.x * 4; c0 < V; c0 += U * stride) {
        float v[U][4];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = c0 + u * stride;
            if (c < V) load4z(zr + c, v[u]);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int c = c0 + u * stride;
            if (c >= V) break;
            float g[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float pk = exp2f(fmaf(v[u][k], kL2e, -lse2)) - ((c + k) == t ? 1.f : 0.f);
                const float q = v[u][k] * inv_cap;
                g[k] = bad ? 0.f : pk * inv_M * (1.f - q * q);
            }
            store4(out + c, g);
        }
    }
}

// Loss and dl of one chunk of rows with bf16 logits, the whole row resident in
// registers as packed bf16 (one 512-thread block per row, CER_K 16-byte vectors
// per thread issued at once): the logits are read from HBM once and dl written
// once, with two block reductions (max, then sum of 2^((z - max)*log2 e)) in
// between.  For V a multiple of CER_NT * 8 up to CER_NT * CER_K * 8.
constexpr int CER_NT = 512, CER_K = 16;

// 2^x on the special-function unit (PTX ex2.approx, flush-to-zero)
__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void store8f(float* p, const float* g) {
    *reinterpret_cast<float4*>(p) = make_float4(g[0], g[1], g[2], g[3]);
    *reinterpret_cast<float4*>(p + 4) = make_float4(g[4], g[5], g[6], g[7]);
}

// block-wide reduction of one float (max or sum) over CER_NT threads
template <bool MAX>
__device__ __forceinline__ float ce_block_reduce(float v, float* red) {
    const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
    v = MAX ? warp_max(v) : warp_sum(v);
    if (lane == 0) red[w] = v;
    __syncthreads();
    float r = red[0];
#pragma unroll
    for (int i = 1; i < CER_NT / 32; ++i) r = MAX ? fmaxf(r, red[i]) : r + red[i];
    __syncthreads();  // red is reused by the next reduction
    return r;
}

template <typename D>
__global__ void __launch_bounds__(CER_NT, 1) ce_chunk_resident_kernel(const bf16* __restrict__ z,
                                                                       const int32_t* __restrict__ tgt, int V,
                                                                       float cap, float inv_M,
                                                                       float* __restrict__ loss_rows,
                                                                       D* __restrict__ dl, int* status) {
    constexpr float kL2e = 1.44269504088896340736f;
    constexpr int STEP = CER_NT * 8;  // logits per vector slot of the block
    __shared__ float red[CER_NT / 32];
    const int row = blockIdx.x;
    const int nk = V / STEP;  // V % STEP == 0: every slot is full or unused for all threads
    const bf16* zr = z + (size_t)row * V;
    const bf16* zt = zr + threadIdx.x * 8;
    uint4 v[CER_K];
#pragma unroll
    for (int k = 0; k < CER_K; ++k)
        if (k < nk) v[k] = *reinterpret_cast<const uint4*>(zt + k * STEP);
    float mx = -INFINITY;
#pragma unroll
    for (int k = 0; k < CER_K; ++k) {
        if (k < nk) {
            const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v[k]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(h[i]);
                mx = fmaxf(mx, fmaxf(f.x, f.y));
            }
        }
    }
    mx = ce_block_reduce<true>(mx, red);
    const float m2 = mx * kL2e;
    float sum = 0.f;
#pragma unroll
    for (int k = 0; k < CER_K; ++k) {
        if (k < nk) {
            const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v[k]);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(h[i]);
                sum += ex2_approx(fmaf(f.x, kL2e, -m2)) + ex2_approx(fmaf(f.y, kL2e, -m2));
            }
        }
    }
    sum = ce_block_reduce<false>(sum, red);
    const float lse = mx + logf(sum);
    const int t = tgt[row];
    const bool bad = t < 0 || t >= V;
    if (threadIdx.x == 0) {
        if (bad) set_status(status, ST_BAD_TOKEN);
        loss_rows[row] = bad ? 0.f : lse - __bfloat162float(zr[t]);
    }
    const float inv_cap = 1.f / cap, lse2 = lse * kL2e;
    const float gs = bad ? 0.f : inv_M;
    const int tl = t - (int)threadIdx.x * 8;  // target relative to this thread's first logit
    D* out = dl + (size_t)row * V + threadIdx.x * 8;
#pragma unroll
    for (int k = 0; k < CER_K; ++k) {
        if (k < nk) {
            const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v[k]);
            const int tk = tl - k * STEP;  // in 0..7 when the target is in this vector
            uint32_t w[4];
            float g[8];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = __bfloat1622float2(h[i]);
                const float q0 = f.x * inv_cap, q1 = f.y * inv_cap;
                const float p0 = ex2_approx(fmaf(f.x, kL2e, -lse2)) - (tk == 2 * i ? 1.f : 0.f);
                const float p1 = ex2_approx(fmaf(f.y, kL2e, -lse2)) - (tk == 2 * i + 1 ? 1.f : 0.f);
                g[2 * i] = p0 * gs * (1.f - q0 * q0);
                g[2 * i + 1] = p1 * gs * (1.f - q1 * q1);
                if constexpr (sizeof(D) == 2) {
                    __nv_bfloat162 b2 = __floats2bfloat162_rn(g[2 * i], g[2 * i + 1]);
                    w[i] = *reinterpret_cast<uint32_t*>(&b2);
                }
            }
            if constexpr (sizeof(D) == 2)
                *reinterpret_cast<uint4*>(out + k * STEP) = make_uint4(w[0], w[1], w[2], w[3]);
            else
                store8f(reinterpret_cast<float*>(out) + k * STEP, g);
        }
    }
}

// One warp per row of the fused LM head's chunk (see launch_lm_rowstats).
template <typename A>
__global__ void __launch_bounds__(256) lm_rowstats_kernel(const float* __restrict__ stats, int ntiles,
                                                         const float* __restrict__ zt, const float* __restrict__ ut,
                                                         const int32_t* __restrict__ tgt, int R, int V, int d,
                                                         float cap, float inv_M, A* __restrict__ u,
                                                         const A* __restrict__ xf, A* __restrict__ xfs,
                                                         float* __restrict__ rs, float* __restrict__ loss_rows,
                                                         int* status) {
    const int row = (int)((blockIdx.x * (size_t)blockDim.x + threadIdx.x) >> 5);
    const int lane = threadIdx.x & 31;
    if (row >= R) return;
    // S = sum over the row's tiles of sum exp(z - cap): lane-strided partial sums,
    // then a fixed butterfly (the same order on every run)
    const float* st = stats + (size_t)row * ntiles;
    float S = 0.f;
    for (int t = lane; t < ntiles; t += 32) S += st[t];
    S = warp_sum(S);
    const int t = tgt[row];
    const bool bad = t < 0 || t >= V;
    const float scale = bad ? 0.f : inv_M / S;
    if (lane == 0) {
        if (bad) set_status(status, ST_BAD_TOKEN);
        const float z = bad ? 0.f : zt[row];
        loss_rows[row] = bad ? 0.f : cap + logf(S) - z;
        rs[row] = scale;
        if (!bad) {
            // dl at the target is (e/S - 1)(1 - (z/cap)^2) / M = (ut - g S) * scale: fold the
            // one-hot term into u in fp32, so the target entry is rounded once
            const float q = z / cap;
            u[(size_t)row * V + t] = fromf<A>(ut[row] - (1.f - q * q) * S);
        }
    }
    // xfs = xf * scale (the dW product's operand: dW = u^T xfs)
    const A* x = xf + (size_t)row * d;
    A* y = xfs + (size_t)row * d;
    constexpr int VEC = Vec<A>::N;
    for (int c = lane * VEC; c < d; c += 32 * VEC) {
        float v[VEC];
        load_vec(x + c, v);
#pragma unroll
        for (int i = 0; i < VEC; ++i) v[i] *= scale;
        store_vec(y + c, v);
    }
}

__global__ void loss_reduce_kernel(const float* __restrict__ rows, int M, float* loss) {
    __shared__ float sh[1024];
    float s = 0.f;
    for (int i = threadIdx.x; i < M; i += blockDim.x) s += rows[i];
    sh[threadIdx.x] = s;
    __syncthreads();
    for (int o = blockDim.x >> 1; o > 0; o >>= 1) {
        if ((int)threadIdx.x < o) sh[threadIdx.x] += sh[threadIdx.x + o];
        __syncthreads();
    }
    if (threadIdx.x == 0) *loss = sh[0] / (float)M;
}

// ---------------------------------------------------------------- KV cache (inference)
// Copies the k and v heads of `rows` fused qkv rows (row r = batch row
// r / rows_per_b, position pos0 + r % rows_per_b) into the cache, one 16-byte
// vector per thread.  Cache: K and V each [B, T_max, nkv, hd].
template <typename A>
__global__ void kv_append_kernel(const A* __restrict__ qkv, int H, int nkv, int hd, int rows, int rows_per_b,
                                 int pos0, A* __restrict__ kc, A* __restrict__ vc, int T_max) {
    constexpr int VEC = Vec<A>::N;
    const int per_row = 2 * nkv * hd / VEC;  // vectors of k then v
    const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (long long)rows * per_row) return;
    const int r = (int)(i / per_row), e = (int)(i % per_row) * VEC;
    const int b = r / rows_per_b, t = pos0 + r % rows_per_b;
    const size_t Nqkv = (size_t)(H + 2 * nkv) * hd;
    const A* src = qkv + (size_t)r * Nqkv + (size_t)H * hd + e;
    const int kvn = nkv * hd;
    A* dst = (e < kvn ? kc : vc) + ((size_t)b * T_max + t) * kvn + (e < kvn ? e : e - kvn);
    *reinterpret_cast<uint4*>(dst) = *reinterpret_cast<const uint4*>(src);
}

// One query per (batch row, head) against the cached positions 0..len-1 (all
// visible: the query is the newest position).  Four warps split the
// positions; each keeps an online softmax in the log2 domain (running max,
// sum, and its share of the output, HD/32 dims per lane), and the four are
// combined at the end.  Scores scaled by 1/sqrt(hd).
template <typename A, int HD>
__global__ void __launch_bounds__(128) decode_attention_kernel(const A* __restrict__ qkv, const A* __restrict__ kc,
                                                               const A* __restrict__ vc, int T_max, int len, int H,
                                                               int nkv, float scale_log2, A* __restrict__ o) {
    constexpr int EPL = HD >= 32 ? HD / 32 : 1;  // dims per lane
    constexpr int LANES = HD / EPL;              // lanes holding dims
    __shared__ float sm[4], sl[4], so[4][HD];
    const int b = blockIdx.x, h = blockIdx.y;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = h / (H / nkv);
    const bool act = lane < LANES;
    const int c0 = (act ? lane : 0) * EPL;
    const size_t Nqkv = (size_t)(H + 2 * nkv) * HD;
    float q[EPL], acc[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
        q[i] = act ? tof(qkv[(size_t)b * Nqkv + (size_t)h * HD + c0 + i]) * scale_log2 : 0.f;
        acc[i] = 0.f;
    }
    float m = -INFINITY, l = 0.f;
    const A* kb = kc + ((size_t)b * T_max * nkv + g) * HD;
    const A* vb = vc + ((size_t)b * T_max * nkv + g) * HD;
    for (int j = warp; j < len; j += 4) {
        const A* kr = kb + (size_t)j * nkv * HD + c0;
        const A* vr = vb + (size_t)j * nkv * HD + c0;
        float sdot = 0.f, vv[EPL];
#pragma unroll
        for (int i = 0; i < EPL; ++i) {
            sdot += act ? q[i] * tof(kr[i]) : 0.f;
            vv[i] = act ? tof(vr[i]) : 0.f;
        }
        const float sc = warp_sum(sdot);
        const float mn = fmaxf(m, sc);
        const float alpha = exp2f(m - mn), pj = exp2f(sc - mn);
        l = l * alpha + pj;
#pragma unroll
        for (int i = 0; i < EPL; ++i) acc[i] = acc[i] * alpha + pj * vv[i];
        m = mn;
    }
    if (lane == 0) { sm[warp] = m; sl[warp] = l; }
    if (act) {
#pragma unroll
        for (int i = 0; i < EPL; ++i) so[warp][c0 + i] = acc[i];
    }
    __syncthreads();
    const float M = fmaxf(fmaxf(sm[0], sm[1]), fmaxf(sm[2], sm[3]));
    float wsc[4], L = 0.f;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        wsc[w] = sm[w] == -INFINITY ? 0.f : exp2f(sm[w] - M);  // a warp without positions adds nothing
        L += sl[w] * wsc[w];
    }
    for (int c = threadIdx.x; c < HD; c += blockDim.x) {
        float r = 0.f;
#pragma unroll
        for (int w = 0; w < 4; ++w) r += so[w][c] * wsc[w];
        o[(size_t)b * H * HD + (size_t)h * HD + c] = fromf<A>(r / L);
    }
}

// ---------------------------------------------------------------- embedding scatter
// dWte[v] = sum of de[m] over the positions m with idx[m] == v, in increasing m.
// Positions are bucketed by id (counting sort, then a canonical in-bucket
// order), each bucket's slot range is cut into pieces of kPiece slots, every
// piece is summed by its own CTA (hot ids under a Zipf law span many pieces),
// and buckets with several pieces add their piece sums in piece order.  All
// orders are fixed, so the result is bitwise reproducible.
constexpr int kPiece = 64;

__global__ void emb_hist_kernel(const int32_t* __restrict__ idx, int M, int V, int* count) {
    int m = blockIdx.x * blockDim.x + threadIdx.x;
    if (m >= M) return;
    int id = idx[m];
    if (id >= 0 && id < V) atomicAdd(&count[id], 1);
}

// Exclusive scans over the V buckets of (count, used?, pieces, partial pieces),
// and the list of used ids in increasing order, in three parallel passes:
// (1) every 1024-id block scans its own ids and records its totals, (2) one
// block scans the block totals, (3) every id adds its block's prefix.
struct Scan4 { int c, f, p, q; };

__device__ __forceinline__ Scan4 emb_vals(int k) {
    const int np = (k + kPiece - 1) / kPiece;
    return {k, k > 0 ? 1 : 0, np, np > 1 ? np : 0};
}

// Exclusive block-wide scan of four ints over 1024 threads; *total gets the block sums.
__device__ __forceinline__ Scan4 block_scan4(Scan4 v, Scan4* total) {
    __shared__ Scan4 warp_sums[32];
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    Scan4 inc = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int c = __shfl_up_sync(0xffffffffu, inc.c, o), f = __shfl_up_sync(0xffffffffu, inc.f, o);
        const int p = __shfl_up_sync(0xffffffffu, inc.p, o), q = __shfl_up_sync(0xffffffffu, inc.q, o);
        if (lane >= o) { inc.c += c; inc.f += f; inc.p += p; inc.q += q; }
    }
    if (lane == 31) warp_sums[w] = inc;
    __syncthreads();
    if (w == 0) {
        Scan4 t = warp_sums[lane];
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int c = __shfl_up_sync(0xffffffffu, t.c, o), f = __shfl_up_sync(0xffffffffu, t.f, o);
            const int p = __shfl_up_sync(0xffffffffu, t.p, o), q = __shfl_up_sync(0xffffffffu, t.q, o);
            if (lane >= o) { t.c += c; t.f += f; t.p += p; t.q += q; }
        }
        warp_sums[lane] = t;  // inclusive over warps
    }
    __syncthreads();
    const Scan4 before = w > 0 ? warp_sums[w - 1] : Scan4{0, 0, 0, 0};
    *total = warp_sums[31];
    return {before.c + inc.c - v.c, before.f + inc.f - v.f, before.p + inc.p - v.p, before.q + inc.q - v.q};
}

__global__ void __launch_bounds__(1024) emb_scan_local_kernel(const int* __restrict__ count, int V, int* offset,
                                                              int* fpre, int* piece_base, int* part_base, Scan4* blk) {
    const int i = blockIdx.x * 1024 + threadIdx.x;
    const Scan4 v = i < V ? emb_vals(count[i]) : Scan4{0, 0, 0, 0};
    Scan4 tot;
    const Scan4 ex = block_scan4(v, &tot);
    if (i < V) {
        offset[i] = ex.c;
        fpre[i] = ex.f;
        piece_base[i] = ex.p;
        part_base[i] = ex.q;
    }
    if (threadIdx.x == 0) blk[blockIdx.x] = tot;
}

// One block: exclusive scan of the nb block totals in place, and the grand totals.
__global__ void __launch_bounds__(1024) emb_scan_blocks_kernel(Scan4* blk, int nb, int V, int* offset, int* n_active,
                                                               int* totals) {
    const int per = (nb + 1023) / 1024;
    const int lo = min(nb, (int)threadIdx.x * per), hi = min(nb, lo + per);
    Scan4 sum{0, 0, 0, 0};
    for (int j = lo; j < hi; ++j) { const Scan4 b = blk[j]; sum.c += b.c; sum.f += b.f; sum.p += b.p; sum.q += b.q; }
    Scan4 tot;
    Scan4 run = block_scan4(sum, &tot);
    for (int j = lo; j < hi; ++j) {
        const Scan4 b = blk[j];
        blk[j] = run;
        run.c += b.c; run.f += b.f; run.p += b.p; run.q += b.q;
    }
    if (threadIdx.x == 0) {
        offset[V] = tot.c;
        *n_active = tot.f;
        totals[0] = tot.p;  // pieces
        totals[1] = tot.q;  // partial slots
    }
}

__global__ void __launch_bounds__(1024) emb_scan_add_kernel(const int* __restrict__ count, int V, const Scan4* blk,
                                                            int* offset, const int* __restrict__ fpre, int* piece_base,
                                                            int* part_base, int* active) {
    const int i = blockIdx.x * 1024 + threadIdx.x;
    if (i >= V) return;
    const Scan4 b = blk[blockIdx.x];
    offset[i] += b.c;
    piece_base[i] += b.p;
    part_base[i] += b.q;
    if (count[i] > 0) active[fpre[i] + b.f] = i;
}

__global__ void emb_fill_kernel(const int32_t* __restrict__ idx, int M, int V, const int* __restrict__ offset,
                                int* cursor, int* perm) {
    int m = blockIdx.x * blockDim.x + threadIdx.x;
    if (m >= M) return;
    int id = idx[m];
    if (id < 0 || id >= V) return;
    perm[offset[id] + atomicAdd(&cursor[id], 1)] = m;
}

// Puts the positions of every id in increasing order (the fill order above
// depends on atomic timing; this makes the final order unique).
__global__ void emb_canon_kernel(const int32_t* __restrict__ idx, int V, const int* __restrict__ offset,
                                 const int* __restrict__ perm, int* perm2) {
    int s = blockIdx.x * blockDim.x + threadIdx.x;
    if (s >= offset[V]) return;
    int p = perm[s];
    int v = idx[p];
    int lo = offset[v], hi = offset[v + 1], rank = 0;
    for (int u = lo; u < hi; ++u) rank += perm[u] < p;
    perm2[lo + rank] = p;
}

// piece -> bucket map, one thread per used bucket.
__global__ void emb_pieces_kernel(const int* __restrict__ count, const int* __restrict__ active,
                                  const int* __restrict__ n_active, const int* __restrict__ piece_base,
                                  int* piece_bucket) {
    int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= *n_active) return;
    int v = active[k];
    int np = (count[v] + kPiece - 1) / kPiece;
    for (int j = 0; j < np; ++j) piece_bucket[piece_base[v] + j] = v;
}

// One CTA per piece: sums its <= kPiece rows of de in slot order.
__global__ void emb_piece_sum_kernel(const float* __restrict__ de, int d, const int* __restrict__ count,
                                     const int* __restrict__ offset, const int* __restrict__ perm2,
                                     const int* __restrict__ piece_base, const int* __restrict__ part_base,
                                     const int* __restrict__ piece_bucket, const int* __restrict__ totals,
                                     float* __restrict__ dwte, float* __restrict__ partial) {
    __shared__ int rows[kPiece];
    int pc = blockIdx.x;
    if (pc >= totals[0]) return;
    int v = piece_bucket[pc];
    int k = pc - piece_base[v];
    int lo = offset[v] + k * kPiece, hi = min(offset[v + 1], lo + kPiece);
    int n = hi - lo;
    if ((int)threadIdx.x < n) rows[threadIdx.x] = perm2[lo + threadIdx.x];
    __syncthreads();
    int np = (count[v] + kPiece - 1) / kPiece;
    float* dst = np == 1 ? dwte + (size_t)v * d : partial + (size_t)(part_base[v] + k) * d;
    for (int c = threadIdx.x * 4; c < d; c += blockDim.x * 4) {
        float4 a0 = make_float4(0.f, 0.f, 0.f, 0.f), a1 = a0;
        int s = 0;
        for (; s + 1 < n; s += 2) {
            float4 g0 = *reinterpret_cast<const float4*>(de + (size_t)rows[s] * d + c);
            float4 g1 = *reinterpret_cast<const float4*>(de + (size_t)rows[s + 1] * d + c);
            a0.x += g0.x; a0.y += g0.y; a0.z += g0.z; a0.w += g0.w;
            a1.x += g1.x; a1.y += g1.y; a1.z += g1.z; a1.w += g1.w;
        }
        a0.x += a1.x; a0.y += a1.y; a0.z += a1.z; a0.w += a1.w;
        if (s < n) {
            float4 g = *reinterpret_cast<const float4*>(de + (size_t)rows[s] * d + c);
            a0.x += g.x; a0.y += g.y; a0.z += g.z; a0.w += g.w;
        }
        *reinterpret_cast<float4*>(dst + c) = a0;
    }
}

// Buckets with several pieces: add the piece sums in piece order.
__global__ void emb_combine_kernel(int d, const int* __restrict__ count, const int* __restrict__ active,
                                   const int* __restrict__ n_active, const int* __restrict__ part_base,
                                   const float* __restrict__ partial, float* __restrict__ dwte) {
    int k = blockIdx.x;
    if (k >= *n_active) return;
    int v = active[k];
    int np = (count[v] + kPiece - 1) / kPiece;
    if (np < 2) return;
    const float* src = partial + (size_t)part_base[v] * d;
    for (int c = threadIdx.x * 4; c < d; c += blockDim.x * 4) {
        float4 acc = *reinterpret_cast<const float4*>(src + c);
        for (int j = 1; j < np; ++j) {
            float4 g = *reinterpret_cast<const float4*>(src + (size_t)j * d + c);
            acc.x += g.x; acc.y += g.y; acc.z += g.z; acc.w += g.w;
        }
        *reinterpret_cast<float4*>(dwte + (size_t)v * d + c) = acc;
    }
}

// Rows of ids that never occur get exact zeros (every dWte row is written once).
__global__ void emb_zero_unused_kernel(const int* __restrict__ count, int V, int d4, float* __restrict__ dwte) {
    size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= (size_t)V * d4) return;
    if (count[i / d4] == 0) reinterpret_cast<float4*>(dwte)[i] = make_float4(0.f, 0.f, 0.f, 0.f);
}

// out[i] = ((accumulate ? out[i] : 0) + sum_s part[s][i]) * (rs ? rs[i / N] : 1),
// partials added in split order; up to eight of them loaded at once.
__global__ void splitk_reduce_kernel(const float* __restrict__ part, int splits, size_t n4,
                                     float* __restrict__ out, bool accumulate, const float* __restrict__ rs,
                                     int N4) {
    size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n4) return;
    const float4* p = reinterpret_cast<const float4*>(part) + i;
    float4 acc = accumulate ? reinterpret_cast<float4*>(out)[i] : make_float4(0.f, 0.f, 0.f, 0.f);
    constexpr int KMAX = 8;
    float4 g[KMAX];
#pragma unroll
    for (int k = 0; k < KMAX; ++k)
        if (k < splits) g[k] = p[(size_t)k * n4];
#pragma unroll
    for (int k = 0; k < KMAX; ++k)
        if (k < splits) { acc.x += g[k].x; acc.y += g[k].y; acc.z += g[k].z; acc.w += g[k].w; }
    for (int k = KMAX; k < splits; ++k) {
        const float4 h = p[(size_t)k * n4];
        acc.x += h.x; acc.y += h.y; acc.z += h.z; acc.w += h.w;
    }
    if (rs) {
        const float f = rs[i / N4];
        acc.x *= f; acc.y *= f; acc.z *= f; acc.w *= f;
    }
    reinterpret_cast<float4*>(out)[i] = acc;
}

// ---------------------------------------------------------------- bounded wait
// Waits on an mbarrier that nobody arrives at; each try_wait is bounded by
// the hardware's time limit and the loop by max_iters.  On expiry it records
// ST_TIMEOUT and returns.
__global__ void expired_wait_kernel(int* status, int max_iters) {
    __shared__ __align__(8) uint64_t bar;
    uint32_t addr = (uint32_t)__cvta_generic_to_shared(&bar);
    if (threadIdx.x == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(addr));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    __syncthreads();
    if (threadIdx.x != 0) return;
    uint32_t done = 0;
    for (int it = 0; it < max_iters && !done; ++it) {
        asm volatile(
            "{\n .reg .pred p;\n"
            " mbarrier.try_wait.parity.shared::cta.b64 p, [%1], 0;\n"
            " selp.u32 %0, 1, 0, p;\n}\n"
            : "=r"(done)
            : "r"(addr)
            : "memory");
    }
    if (!done) set_status(status, ST_TIMEOUT);
}

}  // namespace

std::atomic<long long> g_launches{0};

// ============================================================================ launchers
cudaError_t launch_rope_table(float* c, float* s, int T, int hd, float base, cudaStream_t st, int pos0) {
    int n = T * (hd / 2);
    rope_table_kernel<<<(n + 255) / 256, 256, 0, st>>>(c, s, T, hd, (double)base, pos0);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_embed_norm_fwd(DType wt, const int32_t* idx, const void* wte, int M, int V, int d,
                                  float* x, float* r0, int* status, cudaStream_t s) {
    if (wt == DT_BF16)
        embed_norm_fwd_kernel<bf16><<<row_blocks(M), 256, 0, s>>>(idx, (const bf16*)wte, M, V, d, x, r0, status);
    else
        embed_norm_fwd_kernel<float><<<row_blocks(M), 256, 0, s>>>(idx, (const float*)wte, M, V, d, x, r0, status);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_rmsnorm_fwd(DType at, const float* x, void* y, float* r, int M, int d, cudaStream_t s) {
    const int nch = (d + 255) / 256;
#define NC_RMS_FWD(A, N) rmsnorm_fwd_kernel<A, N><<<row_blocks(M), 256, 0, s>>>(x, (A*)y, r, M, d)
    if (at == DT_BF16) {
        switch (nch) {
            case 1: NC_RMS_FWD(bf16, 1); break;
            case 2: NC_RMS_FWD(bf16, 2); break;
            case 3: NC_RMS_FWD(bf16, 3); break;
            case 4: NC_RMS_FWD(bf16, 4); break;
            case 5: NC_RMS_FWD(bf16, 5); break;
            case 6: NC_RMS_FWD(bf16, 6); break;
            case 7: NC_RMS_FWD(bf16, 7); break;
            case 8: NC_RMS_FWD(bf16, 8); break;
            default: NC_RMS_FWD(bf16, 0); break;
        }
    } else {
        switch (nch) {
            case 1: NC_RMS_FWD(float, 1); break;
            case 2: NC_RMS_FWD(float, 2); break;
            case 3: NC_RMS_FWD(float, 3); break;
            case 4: NC_RMS_FWD(float, 4); break;
            case 5: NC_RMS_FWD(float, 5); break;
            case 6: NC_RMS_FWD(float, 6); break;
            case 7: NC_RMS_FWD(float, 7); break;
            case 8: NC_RMS_FWD(float, 8); break;
            default: NC_RMS_FWD(float, 0); break;
        }
    }
#undef NC_RMS_FWD
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_rmsnorm_bwd(DType at, const void* dy, bool dy_act, const void* y, const float* r, float* dx,
                               bool accumulate, void* dxb, int M, int d, cudaStream_t s) {
    const int nch = (d + 255) / 256;
#define NC_RMS_BWD(A, DY, N)                                                                                  \
    rmsnorm_bwd_kernel<A, DY, N><<<row_blocks(M), 256, 0, s>>>((const DY*)dy, (const A*)y, r, dx, accumulate, \
                                                             (A*)dxb, M, d)
#define NC_RMS_BWD_N(A, DY)                     \
    switch (nch) {                              \
        case 1: NC_RMS_BWD(A, DY, 1); break;    \
        case 2: NC_RMS_BWD(A, DY, 2); break;    \
        case 3: NC_RMS_BWD(A, DY, 3); break;    \
        case 4: NC_RMS_BWD(A, DY, 4); break;    \
        case 5: NC_RMS_BWD(A, DY, 5); break;    \
        case 6: NC_RMS_BWD(A, DY, 6); break;    \
        case 7: NC_RMS_BWD(A, DY, 7); break;    \
        case 8: NC_RMS_BWD(A, DY, 8); break;    \
        default: NC_RMS_BWD(A, DY, 0); break;   \
    }
    if (at == DT_BF16) {
        if (dy_act) {
            NC_RMS_BWD_N(bf16, bf16)
        } else {
            NC_RMS_BWD_N(bf16, float)
        }
    } else {
        NC_RMS_BWD_N(float, float)
    }
#undef NC_RMS_BWD_N
#undef NC_RMS_BWD
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_embed_norm_bwd(DType wt, const float* dx, const int32_t* idx, const void* wte,
                                  const float* r0, float* de, int M, int V, int d, cudaStream_t s) {
    if (wt == DT_BF16)
        embed_norm_bwd_kernel<bf16><<<row_blocks(M), 256, 0, s>>>(dx, idx, (const bf16*)wte, r0, de, M, V, d);
    else
        embed_norm_bwd_kernel<float><<<row_blocks(M), 256, 0, s>>>(dx, idx, (const float*)wte, r0, de, M, V, d);
    count_launch();
    return cudaGetLastError();
}

template <typename A, int HD>
static void qk_fwd_t(void* qkv, float* rqk, const float* c, const float* sn, int M, int T, int H, int nkv,
                     cudaStream_t s) {
    const long long vecs = (long long)M * (H + nkv);
    qknorm_rope_fwd_kernel<A, HD><<<(unsigned)((vecs + 7) / 8), 256, 0, s>>>((A*)qkv, rqk, c, sn, M, T, H, nkv);
}
template <typename A, int HD>
static void qk_bwd_t(void* dqkv, const void* qkv, const float* rqk, const float* c, const float* sn, int M, int T,
                     int H, int nkv, cudaStream_t s) {
    const long long vecs = M;  // one warp per position
    qknorm_rope_bwd_kernel<A, HD><<<(unsigned)((vecs + 7) / 8), 256, 0, s>>>((A*)dqkv, (const A*)qkv, rqk, c, sn, M,
                                                                              T, H, nkv);
}

template <typename A>
static cudaError_t qk_fwd_d(void* qkv, float* rqk, const float* c, const float* sn, int M, int T, int H, int nkv,
                            int hd, cudaStream_t s) {
    switch (hd) {
        case 16: qk_fwd_t<A, 16>(qkv, rqk, c, sn, M, T, H, nkv, s); break;
        case 32: qk_fwd_t<A, 32>(qkv, rqk, c, sn, M, T, H, nkv, s); break;
        case 64: qk_fwd_t<A, 64>(qkv, rqk, c, sn, M, T, H, nkv, s); break;
        case 128: qk_fwd_t<A, 128>(qkv, rqk, c, sn, M, T, H, nkv, s); break;
        default: return cudaErrorInvalidValue;
    }
    count_launch();
    return cudaGetLastError();
}
template <typename A>
static cudaError_t qk_bwd_d(void* dqkv, const void* qkv, const float* rqk, const float* c, const float* sn, int M,
                            int T, int H, int nkv, int hd, cudaStream_t s) {
    switch (hd) {
        case 16: qk_bwd_t<A, 16>(dqkv, qkv, rqk, c, sn, M, T, H, nkv, s); break;
        case 32: qk_bwd_t<A, 32>(dqkv, qkv, rqk, c, sn, M, T, H, nkv, s); break;
        case 64: qk_bwd_t<A, 64>(dqkv, qkv, rqk, c, sn, M, T, H, nkv, s); break;
        case 128: qk_bwd_t<A, 128>(dqkv, qkv, rqk, c, sn, M, T, H, nkv, s); break;
        default: return cudaErrorInvalidValue;
    }
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_qknorm_rope_fwd(DType at, void* qkv, float* rqk, const float* c, const float* sn, int M,
                                   int T, int H, int nkv, int hd, cudaStream_t s) {
    return at == DT_BF16 ? qk_fwd_d<bf16>(qkv, rqk, c, sn, M, T, H, nkv, hd, s)
                         : qk_fwd_d<float>(qkv, rqk, c, sn, M, T, H, nkv, hd, s);
}

cudaError_t launch_qknorm_rope_bwd(DType at, void* dqkv, const void* qkv, const float* rqk, const float* c,
                                   const float* sn, int M, int T, int H, int nkv, int hd, cudaStream_t s) {
    return at == DT_BF16 ? qk_bwd_d<bf16>(dqkv, qkv, rqk, c, sn, M, T, H, nkv, hd, s)
                         : qk_bwd_d<float>(dqkv, qkv, rqk, c, sn, M, T, H, nkv, hd, s);
}

cudaError_t launch_ce_chunk(DType zt, DType dlt, const void* z, const int32_t* tgt, int R, int V, float cap,
                            float inv_M, float* loss_rows, void* dl, int* status, cudaStream_t s) {
    if (R <= 0) return cudaSuccess;
    if (V % 4 != 0) return cudaErrorInvalidValue;
    if (zt == DT_BF16 && V % (CER_NT * 8) == 0 && V <= CER_NT * CER_K * 8) {
        if (dlt == DT_BF16)
            ce_chunk_resident_kernel<bf16><<<R, CER_NT, 0, s>>>((const bf16*)z, tgt, V, cap, inv_M, loss_rows,
                                                                (bf16*)dl, status);
        else
            ce_chunk_resident_kernel<float><<<R, CER_NT, 0, s>>>((const bf16*)z, tgt, V, cap, inv_M, loss_rows,
                                                                 (float*)dl, status);
        count_launch();
        return cudaGetLastError();
    }
#define NC_CE(ZT, DT) \
    ce_chunk_kernel<ZT, DT><<<R, 1024, 0, s>>>((const ZT*)z, tgt, R, V, cap, inv_M, loss_rows, (DT*)dl, status)
    if (zt == DT_BF16) {
        if (dlt == DT_BF16) NC_CE(bf16, bf16); else NC_CE(bf16, float);
    } else {
        if (dlt == DT_BF16) NC_CE(float, bf16); else NC_CE(float, float);
    }
#undef NC_CE
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_kv_append(DType at, const void* qkv, int H, int nkv, int hd, int rows, int rows_per_b,
                             int pos0, void* kc, void* vc, int T_max, cudaStream_t s) {
    const int vec = at == DT_BF16 ? 8 : 4;
    const long long n = (long long)rows * (2 * nkv * hd / vec);
    const unsigned blocks = (unsigned)((n + 255) / 256);
    if (at == DT_BF16)
        kv_append_kernel<bf16><<<blocks, 256, 0, s>>>(reinterpret_cast<const bf16*>(qkv), H, nkv, hd, rows, rows_per_b,
                                                      pos0, reinterpret_cast<bf16*>(kc), reinterpret_cast<bf16*>(vc),
                                                      T_max);
    else
        kv_append_kernel<float><<<blocks, 256, 0, s>>>(reinterpret_cast<const float*>(qkv), H, nkv, hd, rows,
                                                       rows_per_b, pos0, reinterpret_cast<float*>(kc),
                                                       reinterpret_cast<float*>(vc), T_max);
    count_launch();
    return cudaGetLastError();
}

template <typename A>
static cudaError_t decode_attention_t(const void* qkv, const void* kc, const void* vc, int T_max, int len, int B,
                                      int H, int nkv, int hd, void* o, cudaStream_t s) {
    const float sl = 1.44269504088896340736f / sqrtf((float)hd);
    const dim3 grid(B, H);
    const A* q = reinterpret_cast<const A*>(qkv);
    const A* k = reinterpret_cast<const A*>(kc);
    const A* v = reinterpret_cast<const A*>(vc);
    A* out = reinterpret_cast<A*>(o);
    switch (hd) {
        case 16: decode_attention_kernel<A, 16><<<grid, 128, 0, s>>>(q, k, v, T_max, len, H, nkv, sl, out); break;
        case 32: decode_attention_kernel<A, 32><<<grid, 128, 0, s>>>(q, k, v, T_max, len, H, nkv, sl, out); break;
        case 64: decode_attention_kernel<A, 64><<<grid, 128, 0, s>>>(q, k, v, T_max, len, H, nkv, sl, out); break;
        case 128: decode_attention_kernel<A, 128><<<grid, 128, 0, s>>>(q, k, v, T_max, len, H, nkv, sl, out); break;
        default: return cudaErrorInvalidValue;
    }
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_decode_attention(DType at, const void* qkv, const void* kc, const void* vc, int T_max, int len,
                                    int B, int H, int nkv, int hd, void* o, cudaStream_t s) {
    return at == DT_BF16 ? decode_attention_t<bf16>(qkv, kc, vc, T_max, len, B, H, nkv, hd, o, s)
                         : decode_attention_t<float>(qkv, kc, vc, T_max, len, B, H, nkv, hd, o, s);
}

cudaError_t launch_lm_rowstats(const float* stats, int ntiles, const float* zt, const float* ut,
                               const int32_t* tgt, int R, int V, int d, float cap, float inv_M, void* u,
                               const void* xf, void* xfs, float* rs, float* loss_rows, int* status, cudaStream_t s) {
    const unsigned blocks = (unsigned)(((size_t)R * 32 + 255) / 256);
    lm_rowstats_kernel<bf16><<<blocks, 256, 0, s>>>(stats, ntiles, zt, ut, tgt, R, V, d, cap, inv_M,
                                                    reinterpret_cast<bf16*>(u), reinterpret_cast<const bf16*>(xf),
                                                    reinterpret_cast<bf16*>(xfs), rs, loss_rows, status);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_loss_reduce(const float* rows, int M, float* loss, cudaStream_t s) {
    loss_reduce_kernel<<<1, 1024, 0, s>>>(rows, M, loss);
    count_launch();
    return cudaGetLastError();
}

static inline size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

static inline int emb_max_pieces(int M, int V) { return M / kPiece + (M < V ? M : V) + 1; }
static inline int emb_max_partials(int M) { return 2 * (M / kPiece) + 2; }
static inline int emb_scan_blocks(int V) { return (V + 1023) / 1024; }

size_t embed_scratch_bytes(int M, int V, int d) {
    return al256(4ull * V) * 2 + al256(4ull * (V + 1)) + al256(4ull * M) * 2 + al256(4ull * V) + 256 +
           al256(4ull * V) * 2 + al256(4ull * emb_max_pieces(M, V)) + 256 + al256(4ull * V) +
           al256(16ull * emb_scan_blocks(V)) + al256(4ull * emb_max_partials(M) * d);
}

EmbedScratch embed_scratch_carve(void* base, int M, int V, int d) {
    char* p = (char*)base;
    EmbedScratch s;
    s.count = (int*)p;        p += al256(4ull * V);
    s.cursor = (int*)p;       p += al256(4ull * V);   // count and cursor adjacent: one memset
    s.offset = (int*)p;       p += al256(4ull * (V + 1));
    s.perm = (int*)p;         p += al256(4ull * M);
    s.perm2 = (int*)p;        p += al256(4ull * M);
    s.active = (int*)p;       p += al256(4ull * V);
    s.n_active = (int*)p;     p += 256;
    s.piece_base = (int*)p;   p += al256(4ull * V);
    s.part_base = (int*)p;    p += al256(4ull * V);
    s.piece_bucket = (int*)p; p += al256(4ull * emb_max_pieces(M, V));
    s.totals = (int*)p;       p += 256;
    s.fpre = (int*)p;         p += al256(4ull * V);
    s.blk = p;                p += al256(16ull * emb_scan_blocks(V));
    s.partial = (float*)p;
    (void)d;
    return s;
}

cudaError_t launch_embed_scatter(const int32_t* idx, const float* de, int M, int V, int d, float* dwte,
                                 EmbedScratch sc, cudaStream_t s) {
    cudaError_t e = cudaMemsetAsync(sc.count, 0, 2 * al256(4ull * V), s);  // count + cursor
    if (e != cudaSuccess) return e;
    int mb = (M + 255) / 256;
    emb_hist_kernel<<<mb, 256, 0, s>>>(idx, M, V, sc.count);
    const int nb = emb_scan_blocks(V);
    Scan4* blk = reinterpret_cast<Scan4*>(sc.blk);
    emb_scan_local_kernel<<<nb, 1024, 0, s>>>(sc.count, V, sc.offset, sc.fpre, sc.piece_base, sc.part_base, blk);
    emb_scan_blocks_kernel<<<1, 1024, 0, s>>>(blk, nb, V, sc.offset, sc.n_active, sc.totals);
    emb_scan_add_kernel<<<nb, 1024, 0, s>>>(sc.count, V, blk, sc.offset, sc.fpre, sc.piece_base, sc.part_base,
                                            sc.active);
    emb_fill_kernel<<<mb, 256, 0, s>>>(idx, M, V, sc.offset, sc.cursor, sc.perm);
    emb_canon_kernel<<<mb, 256, 0, s>>>(idx, V, sc.offset, sc.perm, sc.perm2);
    int na = M < V ? M : V;
    emb_pieces_kernel<<<(na + 255) / 256, 256, 0, s>>>(sc.count, sc.active, sc.n_active, sc.piece_base,
                                                      sc.piece_bucket);
    emb_piece_sum_kernel<<<emb_max_pieces(M, V), 128, 0, s>>>(de, d, sc.count, sc.offset, sc.perm2, sc.piece_base,
                                                             sc.part_base, sc.piece_bucket, sc.totals, dwte,
                                                             sc.partial);
    emb_combine_kernel<<<na, 128, 0, s>>>(d, sc.count, sc.active, sc.n_active, sc.part_base, sc.partial, dwte);
    size_t n4 = (size_t)V * (d / 4);
    emb_zero_unused_kernel<<<(unsigned)((n4 + 255) / 256), 256, 0, s>>>(sc.count, V, d / 4, dwte);
    count_launch(11);
    return cudaGetLastError();
}

cudaError_t launch_splitk_reduce(const float* part, int splits, size_t n, float* out, bool accumulate,
                                 const float* rs, int N, cudaStream_t s) {
    size_t n4 = n / 4;
    splitk_reduce_kernel<<<(unsigned)((n4 + 255) / 256), 256, 0, s>>>(part, splits, n4, out, accumulate, rs, N / 4);
    count_launch();
    return cudaGetLastError();
}

cudaError_t launch_expired_wait(int* status, int max_iters, cudaStream_t s) {
    expired_wait_kernel<<<1, 32, 0, s>>>(status, max_iters);
    count_launch();
    return cudaGetLastError();
}

}  // namespace nc
