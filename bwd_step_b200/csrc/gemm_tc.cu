// tcgen05 GEMM for the step's linears: C = A B^T with bf16 operands and fp32
// accumulation in tensor memory (TMEM).  It serves every dense contraction of
// the bias-free linears (nanochat announcement, vpshk.cn, architecture list:
// "no biases in linear layers") in the forward and in both backward products
// (dX = dY W, dW = dY^T X), and the untied LM head.
//
// Design (one CTA per SM, persistent over output tiles):
//   warp 0     TMA producer: 128x64 A and 256x64 B bf16 tiles, 128-byte
//              swizzle, into a 4-stage shared-memory ring;
//   warp 1     allocates 512 TMEM columns and issues tcgen05.mma
//              (M=128, N=256, K=16) from one thread; commits release ring
//              slots and hand finished accumulators to the epilogue;
//   warps 2-9  epilogue: two warps per 32-lane TMEM quarter, one per 128-column
//              half of the tile; tcgen05.ld of their lanes (one output row per
//              thread), fused elementwise work, staged TMA stores.  Two warps per
//              SM sub-partition hide each other's latencies.
// Two 256-column accumulators let the epilogue of one tile overlap the main
// loop of the next.  Operands may be K-major or M/N-major (the backward
// products read activations and weights transposed without a copy).
// Split-K (fixed order, deterministic reduction) is used when there are too
// few output tiles to fill the SMs.  Every mbarrier wait is bounded.
#include "gemm_tc.h"
#include "tc_common.cuh"
#include <cudaTypedefs.h>
#include <algorithm>
#include <cstring>

namespace nc {
namespace {
using namespace tc;

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
static_assert(BN == 2 * kGemmStatCols, "each epilogue warp covers one 128-column half of a tile");
constexpr int A_BYTES = BM * BK * 2, B_BYTES = BN * BK * 2, STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int TMEM_COLS = 2 * BN;
constexpr int NTHREADS = 320;
constexpr int MAX_SPLITS = 8;
constexpr int STAGING_BYTES = 8 * 4096;  // epilogue staging: 4 KB per epilogue warp
constexpr size_t SMEM_BYTES = 1024 + (size_t)STAGES * STAGE_BYTES + STAGING_BYTES + 256;
static_assert(SMEM_BYTES <= 232448, "GEMM shared memory exceeds the per-block limit");

struct TcParams {
    int M, N, K;
    int tiles_m, tiles_n, splits, kb_per_split, num_kb, num_units, tn_fast;
    int a_mn, b_mn;
    int epi, c_bf16, vec_ok;
    void* C; int64_t ldc;
    void* C2; int64_t ldc2;
    const bf16* aux; int64_t ldaux;
    float cap;
    float* part;  // split-K partial sums [splits][M][N], or null
    int* status;
    int hd, T, qk_heads;
    float* rqk;
    const float* cos_t;
    const float* sin_t;
    int tma_out;  // epilogue stages 32x32 sub-tiles in shared memory and writes them by TMA
    const int32_t* tgt;  // EPI_LMHEAD
    float* stats;
    int stats_ld;
    float* zt;
    float* ut;
    const float* rs;  // EPI_ROWSCALE
    float* attn_d;    // EPI_ATTN_DO
    float* attn_lse2;
    const float* attn_lse;
    int attn_H;
};

// Per-row state of the epilogue across the 32-column chunks of one tile.
struct RowCtx {
    int tgt;    // EPI_LMHEAD: the row's target column (-1 for rows past M)
    float rs;   // EPI_ROWSCALE: the row's factor
    float sum;  // EPI_LMHEAD: sum of e over the tile's columns so far; EPI_ATTN_DO: dO . o of the head so far
};

// Attention-backward statistics in the epilogue of the GEMM that forms dO
// (softmax backward: dS = P (dP - D) with D = rowsum(dO * o)): the 32-column
// chunk n0.. of this row is rounded to the stored bf16 dO (so D uses the same
// values as the dP product), multiplied with o and summed; at the last chunk
// of a head, -D and -lse * log2(e) are written for (batch row, head, position).
__device__ __forceinline__ void attn_do_chunk(const TcParams& p, int row, int n0, float* v, RowCtx& rc) {
    constexpr float kL2e = 1.44269504088896340736f;
    const bf16* o = p.aux + (int64_t)row * p.ldaux + n0;
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        float ov[8];
        load_vec(o + 8 * e, ov);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            v[8 * e + i] = __bfloat162float(__float2bfloat16_rn(v[8 * e + i]));
            s = fmaf(v[8 * e + i], ov[i], s);
        }
    }
    rc.sum += s;
    if ((n0 + 32) % p.hd == 0) {  // last chunk of head h
        const int h = n0 / p.hd, b = row / p.T, t = row % p.T;
        const size_t i = ((size_t)b * p.attn_H + h) * (size_t)attn_tpad(p.T) + t;
        p.attn_d[i] = -rc.sum;  // both negated: the attention backward adds them
        p.attn_lse2[i] = -p.attn_lse[i] * kL2e;
        rc.sum = 0.f;
    }
}

__device__ __forceinline__ RowCtx row_ctx(const TcParams& p, int row) {
    RowCtx c;
    const bool live = row < p.M;
    c.tgt = (p.epi == EPI_LMHEAD && live) ? p.tgt[row] : -1;
    c.rs = (p.epi == EPI_ROWSCALE && live) ? p.rs[row] : 0.f;
    c.sum = 0.f;
    return c;
}

// LM-head epilogue of one 32-column chunk n0.. of a row (untied LM head and
// tanh logit softcap of the nanochat announcement, vpshk.cn, architecture
// list, followed by the cross-entropy's softmax): the softcapped logit
// z = cap tanh(l/cap) is bounded by cap, so e = exp(z - cap) lies in
// [exp(-2 cap), 1] and needs no running maximum; v becomes
// u = e (1 - (z/cap)^2), the product of the unnormalised softmax and the
// softcap's derivative.  The logits themselves are never stored.
// tanh on the special-function unit (PTX tanh.approx.f32: one instruction,
// relative error about 2^-11, i.e. |dz| <= 0.01 at cap 15 -- below the bf16
// rounding of a stored logit).  Used by the fused LM head only.
__device__ __forceinline__ float tanh_sfu(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ void lmhead_chunk(const TcParams& p, int row, int n0, float* v, RowCtx& rc) {
    constexpr float kL2e = 1.44269504088896340736f;
    const float ic = 1.f / p.cap, cl2 = p.cap * kL2e;
    if ((unsigned)(rc.tgt - n0) < 32u) {  // the target column is in this chunk: its z and u in fp32
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if (n0 + i == rc.tgt) {
                const float t = tanh_sfu(v[i] * ic);
                p.zt[row] = p.cap * t;
                p.ut[row] = ex2((t - 1.f) * cl2) * (1.f - t * t);
            }
    }
    const int nv = min(32, p.N - n0);
    // the scaling, the exponent and the sum as packed f32x2 operations on column pairs
    const uint64_t ic2 = f2_pack(ic, ic), cl2x = f2_pack(cl2, cl2), ncl2 = f2_pack(-cl2, -cl2);
    uint64_t s2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
        float a0, a1, x0, x1;
        f2_unpack(f2_mul(f2_pack(v[i], v[i + 1]), ic2), a0, a1);
        const float t0 = tanh_sfu(a0), t1 = tanh_sfu(a1);
        f2_unpack(f2_fma(f2_pack(t0, t1), cl2x, ncl2), x0, x1);  // (t - 1) cap log2(e)
        const float e0 = ex2(x0), e1 = ex2(x1);
        s2[(i >> 1) & 1] = f2_add(s2[(i >> 1) & 1], f2_pack(i < nv ? e0 : 0.f, i + 1 < nv ? e1 : 0.f));
        v[i] = e0 * (1.f - t0 * t0);
        v[i + 1] = e1 * (1.f - t1 * t1);
    }
    float a, b, c, d;
    f2_unpack(s2[0], a, b);
    f2_unpack(s2[1], c, d);
    rc.sum += (a + b) + (c + d);
}

__device__ __forceinline__ void decode(const TcParams& p, int u, int& tm, int& tn, int& ks) {
    int tile = u % (p.tiles_m * p.tiles_n);
    ks = u / (p.tiles_m * p.tiles_n);
    if (p.tn_fast) { tm = tile / p.tiles_n; tn = tile % p.tiles_n; }
    else { tn = tile / p.tiles_m; tm = tile % p.tiles_m; }
}

__device__ __forceinline__ void store_row_f32(float* dst, const float* v, int nv, bool vec) {
    if (vec && nv == 32) {
#pragma unroll
        for (int i = 0; i < 8; ++i)
            reinterpret_cast<float4*>(dst)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if (i < nv) dst[i] = v[i];
    }
}
__device__ __forceinline__ void store_row_bf16(bf16* dst, const float* v, int nv, bool vec) {
    if (vec && nv == 32) {
#pragma unroll
        for (int i = 0; i < 4; ++i) store_vec(dst + 8 * i, v + 8 * i);
    } else {
#pragma unroll
        for (int i = 0; i < 32; ++i)
            if (i < nv) dst[i] = __float2bfloat16_rn(v[i]);
    }
}
__device__ __forceinline__ void store_row(void* C, bool bf, int64_t off, const float* v, int nv, bool vec) {
    if (bf) store_row_bf16(reinterpret_cast<bf16*>(C) + off, v, nv, vec);
    else store_row_f32(reinterpret_cast<float*>(C) + off, v, nv, vec);
}

// Epilogue of 32 consecutive columns n0.. of one output row.
__device__ __forceinline__ void epilogue(const TcParams& p, int ks, int row, int n0, float* v, RowCtx& rc) {
    const int nv = min(32, p.N - n0);
    const bool vec = p.vec_ok != 0;
    if (p.part) {
        store_row_f32(p.part + ((size_t)ks * p.M + row) * p.N + n0, v, nv, vec);
        return;
    }
    const int64_t off = (int64_t)row * p.ldc + n0;
    switch (p.epi) {
        case EPI_STORE: store_row(p.C, p.c_bf16, off, v, nv, vec); break;
        case EPI_ACCUM: {
            float* c = reinterpret_cast<float*>(p.C) + off;
            if (vec && nv == 32) {
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    float4 o = reinterpret_cast<float4*>(c)[i];
                    v[4 * i] += o.x; v[4 * i + 1] += o.y; v[4 * i + 2] += o.z; v[4 * i + 3] += o.w;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (i < nv) v[i] += c[i];
            }
            store_row_f32(c, v, nv, vec);
        } break;
        case EPI_RELU2: {
            float r[32];
#pragma unroll
            for (int i = 0; i < 32; ++i) { r[i] = fmaxf(v[i], 0.f); v[i] = r[i] * r[i]; }
            store_row_bf16(reinterpret_cast<bf16*>(p.C) + off, v, nv, vec);
            store_row_bf16(reinterpret_cast<bf16*>(p.C2) + (int64_t)row * p.ldc2 + n0, r, nv, vec);
        } break;
        case EPI_RELU2_BWD: {
            const bf16* a = p.aux + (int64_t)row * p.ldaux + n0;
            if (vec && nv == 32) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float u[8];
                    load_vec(a + 8 * i, u);
#pragma unroll
                    for (int j = 0; j < 8; ++j) v[8 * i + j] *= 2.f * u[j];
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (i < nv) v[i] *= 2.f * __bfloat162float(a[i]);
            }
            store_row_bf16(reinterpret_cast<bf16*>(p.C) + off, v, nv, vec);
        } break;
        case EPI_SOFTCAP: {
            const float ic = 1.f / p.cap;
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = p.cap * tanhf(v[i] * ic);
            store_row(p.C, p.c_bf16, off, v, nv, vec);
        } break;
        case EPI_LMHEAD:
            lmhead_chunk(p, row, n0, v, rc);
            store_row_bf16(reinterpret_cast<bf16*>(p.C) + off, v, nv, vec);
            break;
        case EPI_ROWSCALE:
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= rc.rs;
            store_row_f32(reinterpret_cast<float*>(p.C) + off, v, nv, vec);
            break;
        case EPI_ATTN_DO:
            attn_do_chunk(p, row, n0, v, rc);
            store_row_bf16(reinterpret_cast<bf16*>(p.C) + off, v, nv, vec);
            break;
    }
}

// ------------------------------------------------------------------ staged epilogue
// Each epilogue warp owns a 4 KB staging buffer.  A 32-row x 32-column
// sub-tile is written into it in the layout of the output tensor map's
// swizzle (fp32: 128-byte rows, 128B swizzle; bf16: 64-byte rows, 64B
// swizzle; conflict-free for the row-per-thread writes), then one lane issues
// a TMA store -- or, for the residual-add epilogue, a TMA reduce-add, so C is
// never read into the SM.  The buffer is rewritten only after the previous
// chunk's store has finished reading it (the next chunk is already computed
// in registers by then).

__device__ __forceinline__ void stage_f32(uint8_t* buf, int lane, const float* v) {
#pragma unroll
    for (int k = 0; k < 8; ++k)
        *reinterpret_cast<float4*>(buf + lane * 128 + ((k ^ (lane & 7)) << 4)) =
            make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
}
__device__ __forceinline__ void stage_bf16(uint8_t* buf, int lane, const float* v) {
#pragma unroll
    for (int k = 0; k < 4; ++k) store_vec(reinterpret_cast<bf16*>(buf + lane * 64 + ((k ^ ((lane >> 1) & 3)) << 4)), v + 8 * k);
}

// One 32-column chunk through the staging buffers; called by all lanes of the warp.
__device__ __forceinline__ void epilogue_chunk_tma(const TcParams& p, const CUtensorMap* tmC, const CUtensorMap* tmC2,
                                                   uint8_t* stg, int lane, int ks, int row, int row0w, int n0, float* v,
                                                   int cnt, RowCtx& rc) {
    uint8_t* buf = stg;
    if (cnt >= 1) {
        if (lane == 0) bulk_wait_read_0();
        __syncwarp();
    }
    const int mode = p.part ? EPI_STORE : p.epi;
    const bool bf = p.part ? false : p.c_bf16 != 0;
    if (mode == EPI_RELU2) {
        float r[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) { r[i] = fmaxf(v[i], 0.f); v[i] = r[i] * r[i]; }
        stage_bf16(buf, lane, v);
        stage_bf16(buf + 2048, lane, r);
    } else {
        if (mode == EPI_RELU2_BWD && row < p.M) {
            const bf16* a = p.aux + (int64_t)row * p.ldaux + n0;
            const int nv = min(32, p.N - n0);
            if (nv == 32) {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    float u[8];
                    load_vec(a + 8 * i, u);
#pragma unroll
                    for (int j = 0; j < 8; ++j) v[8 * i + j] *= 2.f * u[j];
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i)
                    if (i < nv) v[i] *= 2.f * __bfloat162float(a[i]);
            }
        } else if (mode == EPI_SOFTCAP) {
            const float ic = 1.f / p.cap;
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = p.cap * tanhf(v[i] * ic);
        } else if (mode == EPI_LMHEAD) {
            if (row < p.M) lmhead_chunk(p, row, n0, v, rc);
        } else if (mode == EPI_ROWSCALE) {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= rc.rs;
        } else if (mode == EPI_ATTN_DO) {
            if (row < p.M) attn_do_chunk(p, row, n0, v, rc);
        }
        if (bf) stage_bf16(buf, lane, v);
        else stage_f32(buf, lane, v);
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
        if (p.part) tma_store_3d(tmC, n0, row0w, ks, smem_u32(buf));  // [splits, M, N]: clipped at M per split
        else if (mode == EPI_ACCUM) tma_reduce_add_2d(tmC, n0, row0w, smem_u32(buf));
        else tma_store_2d(tmC, n0, row0w, smem_u32(buf));
        if (mode == EPI_RELU2) tma_store_2d(tmC2, n0, row0w, smem_u32(buf + 2048));
        bulk_commit();
    }
}

// The epilogue of one accumulator row over the 32-column chunks of one
// 128-column half of the tile.  tb addresses the tile's first column.
__device__ __forceinline__ void epilogue_tile(const TcParams& p, const CUtensorMap* tmC, const CUtensorMap* tmC2,
                                              uint8_t* stg, int lane, int ks, int row, int row0w, int tn, int half,
                                              uint32_t tb, int& cnt) {
    const int col0 = tn * BN + half * kGemmStatCols;
    if (col0 >= p.N) return;
    RowCtx rc = row_ctx(p, row);
    const int nch = min(kGemmStatCols / 32, (p.N - col0 + 31) / 32);
    for (int c = 0; c < nch; ++c) {
        float v[32];
        tmem_ld32(tb + half * kGemmStatCols + c * 32, v);
        const int n0 = col0 + c * 32;
        if (p.tma_out) epilogue_chunk_tma(p, tmC, tmC2, stg, lane, ks, row, row0w, n0, v, cnt++, rc);
        else if (row < p.M) epilogue(p, ks, row, n0, v, rc);
    }
    if (p.epi == EPI_LMHEAD && row < p.M) p.stats[(size_t)row * p.stats_ld + tn * 2 + half] = rc.sum;
}

// Fused QK-norm + RoPE epilogue over one 256-column tile of the qkv
// projection (nanochat announcement, vpshk.cn, architecture list: rotary
// embeddings, QK norm): every head of HD columns is loaded whole from TMEM,
// normalised by its RMS (no parameters), rotated pair-wise (j, j + HD/2) by the
// row's position, and stored as bf16; value heads are stored unchanged.
template <int HD>
__device__ __forceinline__ void epilogue_qkrope(const TcParams& p, int row, int n_tile, uint32_t tb, int half) {
    constexpr int NC = HD / 32, HALF = HD / 2;
    const bool live = row < p.M;
    const int pos = live ? row % p.T : 0;
    const float* cs = p.cos_t + (size_t)pos * HALF;
    const float* sn = p.sin_t + (size_t)pos * HALF;
    bf16* crow = reinterpret_cast<bf16*>(p.C) + (int64_t)row * p.ldc;
    for (int h0 = half * kGemmStatCols; h0 < (half + 1) * kGemmStatCols; h0 += HD) {
        const int col = n_tile + h0;
        if (col >= p.N) break;
        const int head = col / HD;
        if (head >= p.qk_heads) {  // value head: plain store
#pragma unroll 1
            for (int c = 0; c < NC; ++c) {
                float v[32];
                tmem_ld32(tb + h0 + c * 32, v);
                if (live) store_row_bf16(crow + col + c * 32, v, 32, true);
            }
            continue;
        }
        // pass 1: sum of squares of the head vector
        float ss = 0.f;
#pragma unroll 1
        for (int c = 0; c < NC; ++c) {
            float v[32];
            tmem_ld32(tb + h0 + c * 32, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) ss += v[i] * v[i];
        }
        const float r = rsqrtf(ss / (float)HD + kRmsEps);
        if (live) p.rqk[(size_t)row * p.qk_heads + head] = r;
        // pass 2: rotate the pairs (j, j + HD/2), chunk c with chunk c + NC/2
#pragma unroll 1
        for (int c = 0; c < NC / 2; ++c) {
            float x1[32], x2[32];
            tmem_ld32(tb + h0 + c * 32, x1);
            tmem_ld32(tb + h0 + (c + NC / 2) * 32, x2);
            if (!live) continue;
#pragma unroll
            for (int i = 0; i < 32; i += 4) {
                const float4 c4 = *reinterpret_cast<const float4*>(cs + c * 32 + i);
                const float4 s4 = *reinterpret_cast<const float4*>(sn + c * 32 + i);
                const float cc[4] = {c4.x, c4.y, c4.z, c4.w}, ssn[4] = {s4.x, s4.y, s4.z, s4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float a = x1[i + e] * r, b = x2[i + e] * r;
                    x1[i + e] = a * cc[e] - b * ssn[e];
                    x2[i + e] = a * ssn[e] + b * cc[e];
                }
            }
            store_row_bf16(crow + col + c * 32, x1, 32, true);
            store_row_bf16(crow + col + (c + NC / 2) * 32, x2, 32, true);
        }
    }
}

__global__ void __launch_bounds__(NTHREADS, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmC2, const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t* staging = smem + (size_t)STAGES * STAGE_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(staging + STAGING_BYTES);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 4);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t tiles_base = smem_u32(smem);
    const uint32_t bar_full = smem_u32(bars), bar_empty = bar_full + 8 * STAGES;
    const uint32_t bar_tfull = bar_empty + 8 * STAGES, bar_tempty = bar_tfull + 16;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) { mbar_init(bar_full + 8 * s, 1); mbar_init(bar_empty + 8 * s, 1); }
        for (int b = 0; b < 2; ++b) { mbar_init(bar_tfull + 8 * b, 1); mbar_init(bar_tempty + 8 * b, 8); }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
    if (warp == 0 && lane == 0) { tma_prefetch(&tmA); tma_prefetch(&tmB); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer
            int stage = 0;
            uint32_t phase = 0, issued = 0, issued_phase = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < p.num_units; u += gridDim.x) {
                int tm, tn, ks;
                decode(p, u, tm, tn, ks);
                const int kb0 = ks * p.kb_per_split, kb1 = min(p.num_kb, kb0 + p.kb_per_split);
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1, abort_flag, p.status)) { ok = false; break; }
                    const uint32_t fb = bar_full + 8 * stage;
                    const uint32_t sa = tiles_base + stage * STAGE_BYTES, sb = sa + A_BYTES;
                    mbar_expect_tx(fb, STAGE_BYTES);
                    if (!p.a_mn) {
                        tma_load_2d(sa, &tmA, kb * BK, tm * BM, fb);
                    } else {
                        tma_load_2d(sa, &tmA, tm * BM, kb * BK, fb);
                        tma_load_2d(sa + 8192, &tmA, tm * BM + 64, kb * BK, fb);
                    }
                    if (!p.b_mn) {
                        tma_load_2d(sb, &tmB, kb * BK, tn * BN, fb);
                    } else {
#pragma unroll
                        for (int j = 0; j < 4; ++j) tma_load_2d(sb + j * 8192, &tmB, tn * BN + 64 * j, kb * BK, fb);
                    }
                    issued |= 1u << stage;
                    issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok) {
                // Let the copies already in flight land before the block exits.
                for (int s = 0; s < STAGES; ++s) {
                    if (!(issued >> s & 1)) continue;
                    uint64_t t0 = globaltimer();
                    while (!mbar_try(bar_full + 8 * s, (issued_phase >> s) & 1) && globaltimer() - t0 < 1000000ull) {}
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer
            const uint32_t idesc = idesc_bf16(BM, BN, p.a_mn != 0, p.b_mn != 0);
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < p.num_units; u += gridDim.x) {
                int tm, tn, ks;
                decode(p, u, tm, tn, ks);
                const int kb0 = ks * p.kb_per_split, kb1 = min(p.num_kb, kb0 + p.kb_per_split);
                if (!mbar_wait(bar_tempty + 8 * acc, acc_phase ^ 1, abort_flag, p.status)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + acc * BN;
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(bar_full + 8 * stage, phase, abort_flag, p.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = tiles_base + stage * STAGE_BYTES, sb = sa + A_BYTES;
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k) {
                        const uint64_t ad = p.a_mn ? smem_desc(sa + k * 2048, 8192, 1024) : smem_desc(sa + k * 32, 16, 1024);
                        const uint64_t bd = p.b_mn ? smem_desc(sb + k * 2048, 8192, 1024) : smem_desc(sb + k * 32, 16, 1024);
                        mma_bf16(d, ad, bd, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
                    }
                    mma_commit(bar_empty + 8 * stage);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                mma_commit(bar_tfull + 8 * acc);
                if (++acc == 2) { acc = 0; acc_phase ^= 1; }
            }
        }
    } else {
        // ---------------- epilogue warps 2..9; warp w reads TMEM lanes 32*(w%4)..,
        // the columns of half (w - 2) / 4 of each tile
        const int q = warp & 3, half = (warp - 2) >> 2;
        uint8_t* stg = staging + (warp - 2) * 4096;
        int cnt = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int u = blockIdx.x; u < p.num_units; u += gridDim.x) {
            int tm, tn, ks;
            decode(p, u, tm, tn, ks);
            if (!warp_wait(bar_tfull + 8 * acc, acc_phase, abort_flag, p.status)) break;
            tc_fence_after();
            const int row0w = tm * BM + q * 32;
            const int row = row0w + lane;
            const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN;
            if (p.epi == EPI_QKROPE) {
                if (p.hd == 128) epilogue_qkrope<128>(p, row, tn * BN, tb, half);
                else epilogue_qkrope<64>(p, row, tn * BN, tb, half);
            } else {
                epilogue_tile(p, &tmC, &tmC2, stg, lane, ks, row, row0w, tn, half, tb, cnt);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(bar_tempty + 8 * acc);
            if (++acc == 2) { acc = 0; acc_phase ^= 1; }
        }
        if (lane == 0) bulk_wait_all();  // staged stores finished before the block exits
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, TMEM_COLS);
    }
}


// ------------------------------------------------------------------ CTA-pair kernel
// Same roles, but a cluster of two CTAs computes a 256x256 output tile with
// tcgen05.mma.cta_group::2 (M = 256): each CTA loads its own 128 rows of A and
// 128 of the 256 B rows per 64-deep K slice (32 KB per stage instead of 48 KB
// for the same work per SM), the even CTA issues the MMAs, which read both
// CTAs' shared memory and write 128 rows into each CTA's TMEM.  Commits arrive
// on the matching barriers of both CTAs; each epilogue reads its own TMEM and
// signals the even CTA that the accumulator may be reused.
constexpr int STAGES2 = 6;
constexpr int STAGE2_BYTES = 2 * 128 * BK * 2;  // A 128x64 + B 128x64, bf16
constexpr size_t SMEM2_BYTES = 1024 + (size_t)STAGES2 * STAGE2_BYTES + STAGING_BYTES + 256;
static_assert(SMEM2_BYTES <= 232448, "paired GEMM shared memory exceeds the per-block limit");

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NTHREADS, 1)
gemm_tc2_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const __grid_constant__ CUtensorMap tmC, const __grid_constant__ CUtensorMap tmC2, const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    uint8_t* staging = smem + (size_t)STAGES2 * STAGE2_BYTES;
    uint64_t* bars = reinterpret_cast<uint64_t*>(staging + STAGING_BYTES);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES2 + 4);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_rank();
    const int cluster = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
    const uint32_t tiles_base = smem_u32(smem);
    const uint32_t bar_full = smem_u32(bars), bar_empty = bar_full + 8 * STAGES2;
    const uint32_t bar_tfull = bar_empty + 8 * STAGES2, bar_tempty = bar_tfull + 16;

    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES2; ++s) { mbar_init(bar_full + 8 * s, 1); mbar_init(bar_empty + 8 * s, 1); }
        for (int b = 0; b < 2; ++b) { mbar_init(bar_tfull + 8 * b, 1); mbar_init(bar_tempty + 8 * b, 16); }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc_pair(smem_u32(tmem_slot), TMEM_COLS);
    if (warp == 0 && lane == 0) { tma_prefetch(&tmA); tma_prefetch(&tmB); }
    tc_fence_before();
    cluster_sync();  // barriers of both CTAs initialised before any remote arrive
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer (both CTAs); bytes counted on the even CTA's barrier
            int stage = 0;
            uint32_t phase = 0, issued = 0, issued_phase = 0;
            bool ok = true;
            for (int u = cluster; ok && u < p.num_units; u += nclusters) {
                int tm, tn, ks;
                decode(p, u, tm, tn, ks);
                const int kb0 = ks * p.kb_per_split, kb1 = min(p.num_kb, kb0 + p.kb_per_split);
                const int arow = tm * 256 + (int)rank * 128, brow = tn * BN + (int)rank * 128;
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(bar_empty + 8 * stage, phase ^ 1, abort_flag, p.status)) { ok = false; break; }
                    const uint32_t fb = leader_addr(bar_full + 8 * stage);
                    const uint32_t sa = tiles_base + stage * STAGE2_BYTES, sb = sa + 16384;
                    if (rank == 0) mbar_expect_tx(bar_full + 8 * stage, 2 * STAGE2_BYTES);
                    if (!p.a_mn) {
                        tma_load_2d_pair(sa, &tmA, kb * BK, arow, fb);
                    } else {
                        tma_load_2d_pair(sa, &tmA, arow, kb * BK, fb);
                        tma_load_2d_pair(sa + 8192, &tmA, arow + 64, kb * BK, fb);
                    }
                    if (!p.b_mn) {
                        tma_load_2d_pair(sb, &tmB, kb * BK, brow, fb);
                    } else {
                        tma_load_2d_pair(sb, &tmB, brow, kb * BK, fb);
                        tma_load_2d_pair(sb + 8192, &tmB, brow + 64, kb * BK, fb);
                    }
                    issued |= 1u << stage;
                    issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES2) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok && rank == 0) {
                for (int s = 0; s < STAGES2; ++s) {
                    if (!(issued >> s & 1)) continue;
                    uint64_t t0 = globaltimer();
                    while (!mbar_try(bar_full + 8 * s, (issued_phase >> s) & 1) && globaltimer() - t0 < 1000000ull) {}
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ---------------- MMA issuer (even CTA only)
            const uint32_t idesc = idesc_bf16(256, BN, p.a_mn != 0, p.b_mn != 0);
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int u = cluster; ok && u < p.num_units; u += nclusters) {
                int tm, tn, ks;
                decode(p, u, tm, tn, ks);
                const int kb0 = ks * p.kb_per_split, kb1 = min(p.num_kb, kb0 + p.kb_per_split);
                if (!mbar_wait(bar_tempty + 8 * acc, acc_phase ^ 1, abort_flag, p.status)) break;
                tc_fence_after();
                const uint32_t d = tmem_base + acc * BN;
                for (int kb = kb0; kb < kb1; ++kb) {
                    if (!mbar_wait(bar_full + 8 * stage, phase, abort_flag, p.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = tiles_base + stage * STAGE2_BYTES, sb = sa + 16384;
#pragma unroll
                    for (int k = 0; k < BK / 16; ++k) {
                        const uint64_t ad = p.a_mn ? smem_desc(sa + k * 2048, 8192, 1024) : smem_desc(sa + k * 32, 16, 1024);
                        const uint64_t bd = p.b_mn ? smem_desc(sb + k * 2048, 8192, 1024) : smem_desc(sb + k * 32, 16, 1024);
                        mma_bf16_pair(d, ad, bd, idesc, (kb > kb0 || k > 0) ? 1u : 0u);
                    }
                    mma_commit_pair(bar_empty + 8 * stage);
                    if (++stage == STAGES2) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                mma_commit_pair(bar_tfull + 8 * acc);
                if (++acc == 2) { acc = 0; acc_phase ^= 1; }
            }
        }
    } else {
        // ---------------- epilogue warps 2..9 of both CTAs (lane quarter w%4, column half (w-2)/4)
        const int q = warp & 3, half = (warp - 2) >> 2;
        uint8_t* stg = staging + (warp - 2) * 4096;
        int cnt = 0;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int u = cluster; u < p.num_units; u += nclusters) {
            int tm, tn, ks;
            decode(p, u, tm, tn, ks);
            if (!warp_wait(bar_tfull + 8 * acc, acc_phase, abort_flag, p.status)) break;
            tc_fence_after();
            const int row0w = tm * 256 + (int)rank * 128 + q * 32;
            const int row = row0w + lane;
            const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + acc * BN;
            if (p.epi == EPI_QKROPE) {
                if (p.hd == 128) epilogue_qkrope<128>(p, row, tn * BN, tb, half);
                else epilogue_qkrope<64>(p, row, tn * BN, tb, half);
            } else {
                epilogue_tile(p, &tmC, &tmC2, stg, lane, ks, row, row0w, tn, half, tb, cnt);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(leader_addr(bar_tempty + 8 * acc));
            if (++acc == 2) { acc = 0; acc_phase ^= 1; }
        }
        if (lane == 0) bulk_wait_all();  // staged stores finished before the block exits
    }
    tc_fence_before();
    cluster_sync();  // no CTA leaves while its pair may still signal or read it
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc_pair(tmem_base, TMEM_COLS);
    }
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (!fn) {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
    }
    return fn;
}

// Tensor map for the staged epilogue's 32x32 output boxes (fp32: 128B
// swizzle, bf16: 64B swizzle) over a row-major [rows, cols] array.
bool make_out_map(CUtensorMap* map, void* base, bool bf16, uint64_t cols, uint64_t rows, uint64_t ld) {
    auto fn = encode_fn();
    if (!fn) return false;
    const uint64_t es = bf16 ? 2 : 4;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {ld * es};
    cuuint32_t box[2] = {32, 32};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, base, dims, strides,
              box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, bf16 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Same for the split-K partial sums, fp32 [splits, rows, cols] contiguous.
bool make_partial_map(CUtensorMap* map, void* base, uint64_t cols, uint64_t rows, uint64_t splits) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[3] = {cols, rows, splits};
    cuuint64_t strides[2] = {cols * 4, cols * rows * 4};
    cuuint32_t box[3] = {32, 32, 1};
    cuuint32_t estr[3] = {1, 1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, base, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D bf16 tensor map over a row-major [outer, inner] array with row stride ld
// elements; box [box_outer, box_inner], 128-byte swizzle, zero fill out of range.
bool make_map(CUtensorMap* map, const void* base, uint64_t inner, uint64_t outer, uint64_t ld, uint32_t box_inner,
              uint32_t box_outer) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {inner, outer};
    cuuint64_t strides[1] = {ld * 2};
    cuuint32_t box[2] = {box_inner, box_outer};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                    CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS;
}

int num_sms() { return device_sm_count(); }

}  // namespace

size_t gemm_tc_splitk_bytes(size_t max_out_elems) { return (size_t)MAX_SPLITS * max_out_elems * sizeof(float); }

int gemm_tc(const GemmDesc& g, void* splitk, size_t splitk_bytes, cudaStream_t s) {
    if (g.in_t != DT_BF16) return 1;
    if (g.epi == EPI_QKROPE &&
        ((g.hd != 64 && g.hd != 128) || g.c_t != DT_BF16 || g.T <= 0 || !g.rqk || !g.cos_t || !g.sin_t ||
         (reinterpret_cast<uintptr_t>(g.C) & 15) || (g.ldc % 8) || (g.N % g.hd)))
        return 1;
    if (g.epi == EPI_LMHEAD &&
        (g.c_t != DT_BF16 || !g.tgt || !g.stats || !g.zt || !g.ut || g.stats_ld < gemm_stat_groups(g.N) || !(g.cap > 0.f)))
        return 1;
    if (g.epi == EPI_ROWSCALE && (g.c_t != DT_F32 || !g.rs)) return 1;
    if (g.epi == EPI_ATTN_DO &&
        (g.c_t != DT_BF16 || !g.aux || !g.attn_d || !g.attn_lse2 || !g.attn_lse || g.T <= 0 || g.attn_H <= 0 ||
         (g.hd != 32 && g.hd != 64 && g.hd != 128) || g.N != g.attn_H * g.hd || g.ldaux % 8 ||
         (reinterpret_cast<uintptr_t>(g.aux) & 15)))
        return 1;
    if (g.M <= 0 || g.N <= 0 || g.K <= 0) return 1;
    auto al16 = [](const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15) == 0; };
    if (!al16(g.A) || !al16(g.B) || (g.lda * 2) % 16 || (g.ldb * 2) % 16) return 1;
    if (ensure_smem_limit((const void*)gemm_tc_kernel, (int)SMEM_BYTES) != cudaSuccess ||
        ensure_smem_limit((const void*)gemm_tc2_kernel, (int)SMEM2_BYTES) != cudaSuccess)
        return -1;

    // CTA pairs (256x256 tiles) when there are at least 256 rows
    const bool pair = g.M >= 256;
    TcParams p{};
    p.M = g.M; p.N = g.N; p.K = g.K;
    p.tiles_m = pair ? (g.M + 255) / 256 : (g.M + BM - 1) / BM;
    p.tiles_n = (g.N + BN - 1) / BN;
    p.num_kb = (g.K + BK - 1) / BK;
    p.tn_fast = p.tiles_n <= p.tiles_m ? 1 : 0;
    p.a_mn = g.a_kmajor ? 0 : 1;
    p.b_mn = g.b_kmajor ? 0 : 1;
    p.epi = g.epi;
    p.c_bf16 = g.c_t == DT_BF16 ? 1 : 0;
    p.C = g.C; p.ldc = g.ldc; p.C2 = g.C2; p.ldc2 = g.ldc2;
    p.aux = reinterpret_cast<const bf16*>(g.aux); p.ldaux = g.ldaux;
    p.cap = g.cap;
    p.status = g.status;
    p.hd = g.hd; p.T = g.T; p.qk_heads = g.qk_heads;
    p.rqk = g.rqk; p.cos_t = g.cos_t; p.sin_t = g.sin_t;
    p.tgt = g.tgt; p.stats = g.stats; p.stats_ld = g.stats_ld; p.zt = g.zt; p.ut = g.ut;
    p.rs = g.rs;
    p.attn_d = g.attn_d; p.attn_lse2 = g.attn_lse2; p.attn_lse = g.attn_lse; p.attn_H = g.attn_H;
    const int esz = p.c_bf16 ? 2 : 4;
    bool vec = al16(g.C) && (g.ldc * esz) % 16 == 0;
    if (g.epi == EPI_RELU2) vec = vec && al16(g.C2) && (g.ldc2 * 2) % 16 == 0;
    if (g.epi == EPI_RELU2_BWD) vec = vec && al16(g.aux) && (g.ldaux * 2) % 16 == 0;

    CUtensorMap ta, tb;
    const uint32_t brows = pair ? 128 : BN;  // B rows per CTA per K slice
    bool ok = g.a_kmajor ? make_map(&ta, g.A, g.K, g.M, g.lda, 64, BM) : make_map(&ta, g.A, g.M, g.K, g.lda, 64, 64);
    ok = ok && (g.b_kmajor ? make_map(&tb, g.B, g.K, g.N, g.ldb, 64, brows)
                           : make_map(&tb, g.B, g.N, g.K, g.ldb, 64, 64));
    if (!ok) return 1;

    // split-K when the output tiles cannot fill the SMs (a pair counts as one unit of two SMs)
    const int sms = pair ? num_sms() / 2 : num_sms();
    const int tiles = p.tiles_m * p.tiles_n;
    int splits = 1;
    // the split-K completion reads and writes C as float4: C must be 16-byte aligned
    const bool can_split = (g.epi == EPI_STORE || g.epi == EPI_ACCUM || g.epi == EPI_ROWSCALE) && !p.c_bf16 &&
                           g.ldc == g.N && splitk && g.N % 4 == 0 && al16(g.C);
    if (can_split && tiles < 2 * sms) {
        // Modelled time of each split count: per CTA pair, its waves of units (each 1/sp of
        // a tile's K loop plus about 5 us of pipeline fill and drain), then the fp32
        // partials written and read back and the output written.  Rates measured on the
        // weight-gradient and LM-head shapes of the d20, d30, 124M and long-context steps:
        // a CTA pair runs a 256x256 tile at about 23 TFLOP/s; partials that fit in half of
        // the L2 move at about 20 TB/s, larger ones at the HBM rate of about 6 TB/s.
        // Without the traffic term a 5120x1280 output (26 MB per partial) took 8 splits
        // and ran 5-12% slower than with 2.
        const double unit_flops = pair ? 23e12 : 11.5e12, fill = 5e-6;
        const double t_tile = 2.0 * (pair ? 256 : BM) * BN * (double)g.K / unit_flops;
        const double out_bytes = 4.0 * (double)g.M * g.N;
        double best = (double)((tiles + sms - 1) / sms) * (t_tile + fill) + out_bytes / 6e12;
        for (int sp = 2; sp <= MAX_SPLITS; ++sp) {
            if (p.num_kb / sp < 8) break;
            if ((size_t)sp * g.M * g.N * sizeof(float) > splitk_bytes) break;
            const double bw = sp * out_bytes <= 64e6 ? 20e12 : 6e12;
            const double cost =
                (double)((tiles * sp + sms - 1) / sms) * (t_tile / sp + fill) + (2.0 * sp + 1.0) * out_bytes / bw;
            if (cost < best * (1.0 - 1e-9)) { best = cost; splits = sp; }
        }
    }
    p.kb_per_split = (p.num_kb + splits - 1) / splits;
    p.splits = (p.num_kb + p.kb_per_split - 1) / p.kb_per_split;
    p.part = p.splits > 1 ? reinterpret_cast<float*>(splitk) : nullptr;
    p.vec_ok = (p.part ? (g.N % 4 == 0) : vec) ? 1 : 0;
    p.num_units = tiles * p.splits;
    // staged (TMA) epilogue for the plain, residual-add, relu^2 (both outputs),
    // relu^2-backward and softcap epilogues, and for split-K partials
    CUtensorMap tc_out, tc_out2;
    memset(&tc_out, 0, sizeof(tc_out));
    memset(&tc_out2, 0, sizeof(tc_out2));
    p.tma_out = 0;
    if (p.part) {
        if (make_partial_map(&tc_out, p.part, g.N, g.M, p.splits)) p.tma_out = 1;
    } else if (vec && g.epi != EPI_QKROPE) {
        const bool bf = p.c_bf16 != 0;
        if (g.epi == EPI_ACCUM && bf) {
            // reduce-add is fp32 only
        } else if (make_out_map(&tc_out, g.C, bf, g.N, g.M, g.ldc) &&
                   (g.epi != EPI_RELU2 || make_out_map(&tc_out2, g.C2, true, g.N, g.M, g.ldc2))) {
            p.tma_out = 1;
        }
    }
    const int grid = std::min(p.num_units, sms);
    if (pair) gemm_tc2_kernel<<<2 * grid, NTHREADS, SMEM2_BYTES, s>>>(ta, tb, tc_out, tc_out2, p);
    else gemm_tc_kernel<<<grid, NTHREADS, SMEM_BYTES, s>>>(ta, tb, tc_out, tc_out2, p);
    count_launch();
    if (cudaGetLastError() != cudaSuccess) return -1;
    if (p.part) {
        // the partials in split order (deterministic), then the row scale of EPI_ROWSCALE
        if (launch_splitk_reduce(p.part, p.splits, (size_t)g.M * g.N, reinterpret_cast<float*>(g.C),
                                 g.epi == EPI_ACCUM, g.epi == EPI_ROWSCALE ? g.rs : nullptr, g.N, s) != cudaSuccess)
            return -1;
    }
    return 0;
}

}  // namespace nc
