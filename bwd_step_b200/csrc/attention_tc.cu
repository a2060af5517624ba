// Causal multi-query attention on the tcgen05 tensor cores (bf16 operands,
// fp32 accumulation in TMEM, fp32 softmax).  Model item: multi-query
// attention, every query head reading the one shared K/V head (nanochat
// announcement, vpshk.cn, architecture list), causal within a row, scores
// scaled by 1/sqrt(hd).
//
// Forward, one CTA per (query block of 128 positions, head, batch row):
//   warp 0     TMA: the Q tile once, then K_j and V_j together in a 3-stage
//              ring for key blocks j = 0..qb (causal: blocks past the
//              diagonal are never loaded);
//   warp 1     tcgen05.mma: S_j = Q K_j^T into one of two 128-column TMEM
//              buffers, two blocks ahead; O += P_j V_j with P_j read from
//              TMEM (A operand) and V_j as an MN-major operand;
//   warps 2-9  softmax, two warps per TMEM lane quarter (one query row per
//              thread, 64 keys each): scores from TMEM, causal mask on the
//              diagonal block, running row max in the log2 domain shared by
//              the two warps of a row through shared memory, lazy rescaling
//              of O (only when the max grows by more than 2^8), and P stored
//              as packed bf16 over the first half of the warp's own score
//              columns.
// The K/V head is shared by all query heads; its tiles are re-read by the
// H CTAs of a query block from L2.
#include "attention_tc.h"
#include "tc_common.cuh"
#include <cudaTypedefs.h>

namespace nc {
namespace {
using namespace tc;

constexpr int NT = 320;  // forward: producer, MMA, 8 softmax warps (two per TMEM lane quarter)
constexpr int FSTG = 3;  // K/V ring stages
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;

struct AttnParams {
    int B, T, H, nkv, nqb;
    float scale_log2;  // log2(e) / sqrt(hd)
    bf16* o;
    float* lse;
    int* status;
};

template <int HD>
struct FwdLayout {
    static constexpr int KB = HD / 64;       // 64-column blocks of the head dim
    static constexpr int TILE = KB * 16384;  // [128 x HD] bf16, 128B-swizzled
    static constexpr int Q = 0;
    static constexpr int K = Q + TILE;
    static constexpr int V = K + FSTG * TILE;
    static constexpr int MX = V + FSTG * TILE;  // [2][2][128] fp32 partial row maxima (then row sums)
    static constexpr int BAR = MX + 2048;
    static constexpr int BYTES = BAR + 256;  // the dynamic shared memory base is 1024-aligned (checked)
    static_assert(BYTES <= 232448, "attention forward shared memory exceeds the per-block limit");
};

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

// the two softmax warps of TMEM lane quarter q (64 threads)
__device__ __forceinline__ void pair_sync(int q) {
    asm volatile("bar.sync %0, 64;" ::"r"(1 + q) : "memory");
}

// Store 32 consecutive 32-bit columns of this thread's TMEM lane, then wait.
__device__ __forceinline__ void tmem_st32u(uint32_t taddr, const uint32_t* v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
        ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
        "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]),
        "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

template <int HD>
__global__ void __launch_bounds__(NT, 1) attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm, const AttnParams p) {
    using Lay = FwdLayout<HD>;
    constexpr int KB = Lay::KB;
    constexpr int TILE = Lay::TILE;
    extern __shared__ __align__(1024) uint8_t smem_dyn[];
    if ((smem_u32(smem_dyn) & 1023u) != 0) {
        if (threadIdx.x == 0) set_status(p.status, ST_BAD_LAYOUT);
        return;
    }
    uint8_t* smem = smem_dyn;
    const uint32_t base = smem_u32(smem);
    const uint32_t sQ = base + Lay::Q, sK = base + Lay::K, sV = base + Lay::V;
    float* mxs = reinterpret_cast<float*>(smem + Lay::MX);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::BAR);
    const uint32_t b0 = smem_u32(bars);
    const uint32_t q_full = b0;
    const uint32_t kv_full = b0 + 8, kv_empty = b0 + 32;  // [FSTG]: K_j and V_j share a stage
    const uint32_t s_full = b0 + 56, p_full = b0 + 72;    // [2]: per TMEM score buffer
    const uint32_t o_last = b0 + 88;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 12);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qb = p.nqb - 1 - (int)blockIdx.z;  // grid z slowest: the longest blocks launch first
    const int h = blockIdx.x, b = blockIdx.y, g = h / (p.H / p.nkv);
    const int nblk = qb + 1;
    const int row0 = b * p.T;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < FSTG; ++s) { mbar_init(kv_full + 8 * s, 1); mbar_init(kv_empty + 8 * s, 1); }
        for (int s = 0; s < 2; ++s) { mbar_init(s_full + 8 * s, 1); mbar_init(p_full + 8 * s, 8); }
        mbar_init(o_last, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), 512);
    if (warp == 0 && lane == 0) tma_prefetch(&tm);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem, tO = tmem + 256;  // S[2] of 128 columns, O (HD columns)

    if (warp == 0) {
        // one thread loads Q, then K_j and V_j together into a 3-stage ring (a stage
        // frees after O += P_j V_j): one wait per key block for the MMA thread
        if (lane == 0) {
            const int xq = h * HD, xk = (p.H + g) * HD, xv = (p.H + p.nkv + g) * HD;
            mbar_expect_tx(q_full, TILE);
#pragma unroll
            for (int kb = 0; kb < KB; ++kb) tma_load_2d(sQ + kb * 16384, &tm, xq + kb * 64, row0 + qb * 128, q_full);
            int issued = 0;
            for (int j = 0; j < nblk; ++j) {
                const int st = j % FSTG;
                if (!mbar_wait(kv_empty + 8 * st, ((j / FSTG) & 1) ^ 1, abort_flag, p.status)) break;
                mbar_expect_tx(kv_full + 8 * st, 2 * TILE);
#pragma unroll
                for (int kb = 0; kb < KB; ++kb) {
                    tma_load_2d(sK + st * TILE + kb * 16384, &tm, xk + kb * 64, row0 + j * 128, kv_full + 8 * st);
                    tma_load_2d(sV + st * TILE + kb * 16384, &tm, xv + kb * 64, row0 + j * 128, kv_full + 8 * st);
                }
                issued = j + 1;
            }
            if (*abort_flag) {
                // let copies in flight land before the block exits
                uint64_t t0 = globaltimer();
                while (!mbar_try(q_full, 0) && globaltimer() - t0 < 1000000ull) {}
                for (int j = (issued > FSTG ? issued - FSTG : 0); j < issued; ++j) {
                    t0 = globaltimer();
                    while (!mbar_try(kv_full + 8 * (j % FSTG), (j / FSTG) & 1) && globaltimer() - t0 < 1000000ull) {}
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id_s = idesc_bf16(128, 128, false, false);
            const uint32_t id_o = idesc_bf16(128, HD, false, true);
            // S_j = Q K_j^T into buffer j & 1
            auto scores = [&](int j) -> bool {
                const int st = j % FSTG, sb = j & 1;
                if (!mbar_wait(kv_full + 8 * st, (j / FSTG) & 1, abort_flag, p.status)) return false;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < HD / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                    mma_bf16(tS + sb * 128, smem_desc(sQ + off, 16, 1024), smem_desc(sK + st * TILE + off, 16, 1024),
                             id_s, ks > 0 ? 1u : 0u);
                }
                mma_commit(s_full + 8 * sb);
                return true;
            };
            bool ok = mbar_wait(q_full, 0, abort_flag, p.status) && scores(0) && (nblk < 2 || scores(1));
            for (int j = 0; ok && j < nblk; ++j) {
                const int st = j % FSTG, sb = j & 1;
                // O += P_j V_j: keys 16kk..16kk+15 sit in the packed columns
                // 64*(kk/4) + 8*(kk%4) of score buffer j & 1 (written by column group kk/4)
                // (V_j landed with K_j, waited for before S_j)
                if (!mbar_wait(p_full + 8 * sb, (j >> 1) & 1, abort_flag, p.status)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16_ts(tO, tS + sb * 128 + 64 * (kk >> 2) + 8 * (kk & 3),
                                smem_desc(sV + st * TILE + kk * 2048, 16384, 1024), id_o, (j > 0 || kk > 0) ? 1u : 0u);
                mma_commit(kv_empty + 8 * st);
                // S_{j+2} overwrites P_j only after these MMAs (issue order)
                if (j + 2 < nblk && !scores(j + 2)) break;
            }
            mma_commit(o_last);
        }
    } else {
        // ---------------- softmax warps: warp w reads TMEM lanes 32*(w%4).., keys 64*cg..
        const int q = warp & 3, cg = (warp - 2) >> 2;
        const int r = q * 32 + lane;  // row of the tile
        const int qpos = qb * 128 + r;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        float m = -INFINITY, l = 0.f;
        // After a failed (timed-out or aborted) wait a warp skips its TMEM and
        // barrier work but still meets its partner at every pair_sync, so the
        // pair never waits on a warp that has left the loop.
        bool ok = true;
        for (int j = 0; j < nblk; ++j) {
            const int sb = j & 1;
            ok = ok && warp_wait(s_full + 8 * sb, (j >> 1) & 1, abort_flag, p.status);
            float s[64];
            float mx = -INFINITY;
            if (ok) {
                tc_fence_after();
                {
                    uint32_t rr[64];
                    tmem_ld32_issue(tS + lane_off + sb * 128 + cg * 64, rr);
                    tmem_ld32_issue(tS + lane_off + sb * 128 + cg * 64 + 32, rr + 32);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 64; ++i) s[i] = __uint_as_float(rr[i]);
                }
                if (j == qb) {
                    const int lim = r - cg * 64;  // keys cg*64 + c with c <= lim are visible
#pragma unroll
                    for (int c = 0; c < 64; ++c) {
                        s[c] = (c <= lim) ? s[c] * p.scale_log2 : -INFINITY;
                        mx = fmaxf(mx, s[c]);
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 64; ++c) {
                        s[c] *= p.scale_log2;
                        mx = fmaxf(mx, s[c]);
                    }
                }
            }
            // the row max over both halves of the block
            mxs[(sb * 2 + cg) * 128 + r] = mx;
            pair_sync(q);
            if (!ok) continue;
            mx = fmaxf(mx, mxs[(sb * 2 + (cg ^ 1)) * 128 + r]);
            const bool rescale = mx > m + 8.f;
            const float mu = rescale ? mx : m;
            const float alpha = rescale ? ex2(m - mx) : 1.f;
            float sum = 0.f;
            uint32_t pk[32];
#pragma unroll
            for (int c = 0; c < 64; c += 2) {
                const float e0 = ex2(s[c] - mu), e1 = ex2(s[c + 1] - mu);
                sum += e0 + e1;
                pk[c >> 1] = pack_bf16(e0, e1);
            }
            if (j > 0 && __any_sync(0xffffffffu, rescale)) {
                // O += P_{j-1} V_{j-1} has finished (its K/V stage was released); O(j) cannot
                // have started, so this phase of the barrier is the latest one
                const int jj = j - 1;
                ok = warp_wait(kv_empty + 8 * (jj % FSTG), (jj / FSTG) & 1, abort_flag, p.status);
                if (!ok) continue;
                tc_fence_after();
                // this warp rescales its half of the O columns
#pragma unroll 1
                for (int c = 0; c < HD / 32; ++c) {
                    float o[16];
                    tmem_ld16(tO + lane_off + cg * (HD / 2) + c * 16, o);
                    uint32_t u[16];
#pragma unroll
                    for (int i = 0; i < 16; ++i) u[i] = __float_as_uint(o[i] * alpha);
                    tmem_st16(tO + lane_off + cg * (HD / 2) + c * 16, u);
                }
            }
            l = l * alpha + sum;
            m = mu;
            tmem_st32u(tS + lane_off + sb * 128 + cg * 64, pk);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full + 8 * sb);
        }
        ok = ok && warp_wait(o_last, 0, abort_flag, p.status);
        // row sums of both halves (buffer 0 of the maxima is free: the partner read
        // this warp's last maximum before its P was handed over, which O needed)
        mxs[cg * 128 + r] = l;
        pair_sync(q);
        if (ok) {
            tc_fence_after();
            const float lt = l + mxs[(cg ^ 1) * 128 + r];
            const float inv = 1.f / lt;
            const bool live = qpos < p.T;
            bf16* orow = p.o + ((size_t)row0 + qpos) * (size_t)(p.H * HD) + h * HD + cg * (HD / 2);
#pragma unroll
            for (int c = 0; c < HD / 64; ++c) {
                float o[32];
                tmem_ld32(tO + lane_off + cg * (HD / 2) + c * 32, o);
                if (live) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        uint4 u = make_uint4(pack_bf16(o[8 * i] * inv, o[8 * i + 1] * inv),
                                             pack_bf16(o[8 * i + 2] * inv, o[8 * i + 3] * inv),
                                             pack_bf16(o[8 * i + 4] * inv, o[8 * i + 5] * inv),
                                             pack_bf16(o[8 * i + 6] * inv, o[8 * i + 7] * inv));
                        *reinterpret_cast<uint4*>(orow + c * 32 + 8 * i) = u;
                    }
                }
            }
            if (live && cg == 0) p.lse[((size_t)b * p.H + h) * attn_tpad(p.T) + qpos] = (m + __log2f(lt)) * kLn2;
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}


// ============================================================================ backward
// Both backward kernels keep every MMA at N = 128 (a 128 x 64 tile runs the
// tensor core at well under half rate on sm_100a) and feed one operand of the
// second product from TMEM: the softmax warps write their bf16 result back
// over fp32 columns they have just read (S in dQ, dP^T in dK/dV), and the MMA
// reads it there as the A operand.  Sixteen softmax warps (four per TMEM lane quarter, 32
// columns each) keep the special-function unit busy.
//
// dQ, one CTA per (query block of 128, head, batch row), key blocks j = 0..qb:
//   warp 0      TMA: Q and dO once; K_j into a 3-stage ring (freed by the dQ
//               MMA), V_j into a 2-stage ring (freed by the dP MMA), both on
//               one barrier per key block;
//   warp 1      tcgen05.mma: S_j = Q K_j^T into one of two TMEM buffers and
//               dP_j = dO V_j^T into one buffer as one group of 16 MMAs
//               (every wait or commit between 128-wide MMAs idles the tensor
//               core), then dQ += dS_{j-1} K_{j-1} with dS read from TMEM and
//               K as an MN-major operand;
//   warps 2-17  per key block: load the warp's S and dP columns, release dP,
//               form P = 2^(S*scale*log2e - lse*log2e) with the causal mask on
//               the diagonal block and dS = P (dP - D), and store dS as packed
//               bf16 over the first half of the warp's own S columns.
// dq = dQ / sqrt(hd).
constexpr int NTB = 576;  // backward: producer, MMA, 16 softmax warps
constexpr int NSM = 16;   // softmax warps

template <int HD>
struct DqLayout {
    static constexpr int KB = HD / 64;
    static constexpr int TILE = KB * 16384;  // [128 x HD] bf16, 128B-swizzled: Q, dO, a K or V block
    static constexpr int KSTG = 3, VSTG = 2;
    static constexpr int Q = 0;
    static constexpr int DO = Q + TILE;
    static constexpr int K = DO + TILE;
    static constexpr int V = K + KSTG * TILE;
    static constexpr int BAR = V + VSTG * TILE;
    static constexpr int BYTES = BAR + 256;  // the dynamic shared memory base is 1024-aligned (checked)
    static_assert(BYTES <= 232448, "dQ shared memory exceeds the per-block limit");
};

struct BwdParams {
    int B, T, H, nkv, nqb;
    float scale_log2, scale;
    const float* D;     // [B, H, Tp] rowsum(dO * o)
    const float* lse2;  // [B, H, Tp] lse * log2(e) (both zero past the sequence end)
    bf16* dqkv;
    int* status;
};

__device__ __forceinline__ void drain(uint32_t bar, uint32_t parity) {
    uint64_t t0 = globaltimer();
    while (!mbar_try(bar, parity) && globaltimer() - t0 < 1000000ull) {}
}

// sum of the products of two vectors of eight bf16
__device__ __forceinline__ float dot8(const uint4& a, const uint4& b) {
    const __nv_bfloat162* x = reinterpret_cast<const __nv_bfloat162*>(&a);
    const __nv_bfloat162* y = reinterpret_cast<const __nv_bfloat162*>(&b);
    float s = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const float2 u = __bfloat1622float2(x[i]), v = __bfloat1622float2(y[i]);
        s = fmaf(u.x, v.x, s);
        s = fmaf(u.y, v.y, s);
    }
    return s;
}

// D = rowsum(dO * o) and lse * log2(e) for every (batch row b, head h, position t
// < Tp), head-major [B, H, Tp], zero past the end of the sequence: HD/8 threads
// per entry, each with one 16-byte vector of o and dO.
template <int HD>
__global__ void __launch_bounds__(256) attn_bwd_stats_kernel(const bf16* __restrict__ o, const bf16* __restrict__ dO,
                                                             const float* __restrict__ lse, float* __restrict__ D,
                                                             float* __restrict__ lse2, int B, int T, int H) {
    constexpr int G = HD / 8;
    const int Tp = attn_tpad(T);
    const long long n = (long long)B * H * Tp;
    const long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) / G;
    const int k = threadIdx.x % G;
    const int t = (int)(w % Tp);
    const long long bh = w / Tp;
    const bool live = w < n && t < T;
    float s = 0.f;
    if (live) {
        const long long row = (bh / H) * T + t;
        const size_t off = ((size_t)row * H + (size_t)(bh % H)) * HD + 8 * k;
        s = dot8(*reinterpret_cast<const uint4*>(o + off), *reinterpret_cast<const uint4*>(dO + off));
    }
#pragma unroll
    for (int m = G / 2; m > 0; m >>= 1) s += __shfl_xor_sync(0xffffffffu, s, m);
    if (w < n && k == 0) {
        D[w] = s;
        lse2[w] = live ? lse[w] * kLog2e : 0.f;
    }
}

template <int HD>
__global__ void __launch_bounds__(NTB, 1) attn_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQKV,
                                                           const __grid_constant__ CUtensorMap tmDO,
                                                           const BwdParams p) {
    using Lay = DqLayout<HD>;
    constexpr int KB = Lay::KB, TILE = Lay::TILE, KSTG = Lay::KSTG, VSTG = Lay::VSTG;
    extern __shared__ __align__(1024) uint8_t smem_dyn[];
    if ((smem_u32(smem_dyn) & 1023u) != 0) {
        if (threadIdx.x == 0) set_status(p.status, ST_BAD_LAYOUT);
        return;
    }
    uint8_t* smem = smem_dyn;
    const uint32_t base = smem_u32(smem);
    const uint32_t sQ = base + Lay::Q, sDO = base + Lay::DO, sK = base + Lay::K, sV = base + Lay::V;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::BAR);
    const uint32_t b0 = smem_u32(bars);
    const uint32_t qd_full = b0;
    const uint32_t k_empty = b0 + 32;                    // [KSTG]
    const uint32_t v_full = b0 + 56, v_empty = b0 + 72;  // [VSTG]: v_full covers K_j and V_j
    const uint32_t dp_full = b0 + 104, dp_free = b0 + 112;
    const uint32_t ds_full = b0 + 120;                   // [2]: dS_j written over buffer j & 1
    const uint32_t dq_done = b0 + 136;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 18);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qb = p.nqb - 1 - (int)blockIdx.z;  // longest blocks launch first
    const int h = blockIdx.x, b = blockIdx.y, g = h / (p.H / p.nkv);
    const int nblk = qb + 1;
    const int row0 = b * p.T;
    const int Nqkv = (p.H + 2 * p.nkv) * HD;

    if (threadIdx.x == 0) {
        mbar_init(qd_full, 1);
        for (int s = 0; s < KSTG; ++s) mbar_init(k_empty + 8 * s, 1);
        for (int s = 0; s < VSTG; ++s) { mbar_init(v_full + 8 * s, 1); mbar_init(v_empty + 8 * s, 1); }
        for (int s = 0; s < 2; ++s) mbar_init(ds_full + 8 * s, NSM);
        mbar_init(dp_full, 1);
        mbar_init(dp_free, NSM);
        mbar_init(dq_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), 512);
    if (warp == 0 && lane == 0) { tma_prefetch(&tmQKV); tma_prefetch(&tmDO); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem, tdP = tmem + 256, tdQ = tmem + 384;  // S[2] of 128 columns, dP, dQ

    if (warp == 0) {
        // one thread loads Q and dO, then per key block K_j into the 3-stage K ring
        // (a slot frees after the dQ MMA) and V_j into the 2-stage V ring (after
        // the dP MMA); both land on the V stage's barrier, so the MMA thread waits
        // once per key block
        if (lane == 0) {
            const int xk = (p.H + g) * HD, xv = (p.H + p.nkv + g) * HD;
            mbar_expect_tx(qd_full, 2 * TILE);
#pragma unroll
            for (int kb = 0; kb < KB; ++kb) {
                tma_load_2d(sQ + kb * 16384, &tmQKV, h * HD + kb * 64, row0 + qb * 128, qd_full);
                tma_load_2d(sDO + kb * 16384, &tmDO, h * HD + kb * 64, row0 + qb * 128, qd_full);
            }
            int issued = 0;
            for (int j = 0; j < nblk; ++j) {
                const int kst = j % KSTG, vst = j % VSTG;
                if (!mbar_wait(k_empty + 8 * kst, ((j / KSTG) & 1) ^ 1, abort_flag, p.status)) break;
                if (!mbar_wait(v_empty + 8 * vst, ((j / VSTG) & 1) ^ 1, abort_flag, p.status)) break;
                mbar_expect_tx(v_full + 8 * vst, 2 * TILE);
#pragma unroll
                for (int kb = 0; kb < KB; ++kb) {
                    tma_load_2d(sK + kst * TILE + kb * 16384, &tmQKV, xk + kb * 64, row0 + j * 128, v_full + 8 * vst);
                    tma_load_2d(sV + vst * TILE + kb * 16384, &tmQKV, xv + kb * 64, row0 + j * 128, v_full + 8 * vst);
                }
                issued = j + 1;
            }
            if (*abort_flag) {
                drain(qd_full, 0);
                for (int j = (issued > VSTG ? issued - VSTG : 0); j < issued; ++j)
                    drain(v_full + 8 * (j % VSTG), (j / VSTG) & 1);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id_s = idesc_bf16(128, 128, false, false);
            const uint32_t id_q = idesc_bf16(128, HD, false, true);
            bool ok = mbar_wait(qd_full, 0, abort_flag, p.status);
            for (int j = 0; ok && j <= nblk; ++j) {
                if (j < nblk) {
                    // S_j and dP_j as one group: K_j, V_j landed, dP_{j-1} read out of TMEM
                    const int kst = j % KSTG, vst = j % VSTG, sb = j & 1;
                    if (!mbar_wait(v_full + 8 * vst, (j / VSTG) & 1, abort_flag, p.status)) break;
                    if (j > 0 && !mbar_wait(dp_free, (j - 1) & 1, abort_flag, p.status)) break;
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < HD / 16; ++ks) {
                        const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                        mma_bf16(tS + sb * 128, smem_desc(sQ + off, 16, 1024),
                                 smem_desc(sK + kst * TILE + off, 16, 1024), id_s, ks > 0 ? 1u : 0u);
                    }
#pragma unroll
                    for (int ks = 0; ks < HD / 16; ++ks) {
                        const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                        mma_bf16(tdP, smem_desc(sDO + off, 16, 1024), smem_desc(sV + vst * TILE + off, 16, 1024),
                                 id_s, ks > 0 ? 1u : 0u);
                    }
                    mma_commit(dp_full);
                    mma_commit(v_empty + 8 * vst);
                }
                if (j > 0) {
                    // dQ += dS_{j-1} K_{j-1}: keys 16kk..16kk+15 sit in the packed columns
                    // 32*(kk/2) + 8*(kk%2) of the S buffer (written by column group kk/2)
                    const int jj = j - 1, sb = jj & 1;
                    if (!mbar_wait(ds_full + 8 * sb, (jj >> 1) & 1, abort_flag, p.status)) break;
                    tc_fence_after();
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        mma_bf16_ts(tdQ, tS + sb * 128 + 32 * (kk >> 1) + 8 * (kk & 1),
                                    smem_desc(sK + (jj % KSTG) * TILE + kk * 2048, 16384, 1024), id_q,
                                    (jj > 0 || kk > 0) ? 1u : 0u);
                    mma_commit(k_empty + 8 * (jj % KSTG));
                }
            }
            mma_commit(dq_done);
        }
    } else {
        // warps 2..17: TMEM lane quarter q (query rows), key column group cg (32 keys)
        const int q = warp & 3, cg = (warp - 2) >> 2;
        const int r = q * 32 + lane;
        const int qpos = qb * 128 + r;
        const bool live = qpos < p.T;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        const size_t si = ((size_t)b * p.H + h) * attn_tpad(p.T) + qpos;
        const float Dr = p.D[si], lse2 = p.lse2[si];
        bool ok = true;
        for (int j = 0; j < nblk; ++j) {
            const int sb = j & 1;
            if (!warp_wait(dp_full, j & 1, abort_flag, p.status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t rs[32], rd[32];
            tmem_ld32_issue(tS + lane_off + sb * 128 + cg * 32, rs);
            tmem_ld32_issue(tdP + lane_off + cg * 32, rd);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(dp_free);
            // keys j*128 + cg*32 + e, e <= lim, are visible from this row
            const int lim = !live ? -1 : (j == qb ? r - cg * 32 : 31);
            uint32_t pk[16];
            if (__all_sync(0xffffffffu, lim >= 31)) {
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const float d0 = ex2(fmaf(__uint_as_float(rs[e]), p.scale_log2, -lse2)) *
                                     (__uint_as_float(rd[e]) - Dr);
                    const float d1 = ex2(fmaf(__uint_as_float(rs[e + 1]), p.scale_log2, -lse2)) *
                                     (__uint_as_float(rd[e + 1]) - Dr);
                    pk[e >> 1] = pack_bf16(d0, d1);
                }
            } else {
#pragma unroll
                for (int e = 0; e < 32; e += 2) {
                    const float d0 = e <= lim ? ex2(fmaf(__uint_as_float(rs[e]), p.scale_log2, -lse2)) *
                                                    (__uint_as_float(rd[e]) - Dr)
                                              : 0.f;
                    const float d1 = e + 1 <= lim ? ex2(fmaf(__uint_as_float(rs[e + 1]), p.scale_log2, -lse2)) *
                                                        (__uint_as_float(rd[e + 1]) - Dr)
                                                  : 0.f;
                    pk[e >> 1] = pack_bf16(d0, d1);
                }
            }
            tmem_st16(tS + lane_off + sb * 128 + cg * 32, pk);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(ds_full + 8 * sb);
        }
        if (ok && warp_wait(dq_done, 0, abort_flag, p.status)) {
            tc_fence_after();
            // column group cg writes dq columns 32*cg .. 32*cg+31 (hd 64: groups 0 and 1)
            if (cg * 32 < HD) {
                float v[32];
                tmem_ld32(tdQ + lane_off + cg * 32, v);
                if (live) {
                    bf16* out = p.dqkv + ((size_t)row0 + qpos) * Nqkv + h * HD + cg * 32;
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        *reinterpret_cast<uint4*>(out + 8 * e) =
                            make_uint4(pack_bf16(v[8 * e] * p.scale, v[8 * e + 1] * p.scale),
                                       pack_bf16(v[8 * e + 2] * p.scale, v[8 * e + 3] * p.scale),
                                       pack_bf16(v[8 * e + 4] * p.scale, v[8 * e + 5] * p.scale),
                                       pack_bf16(v[8 * e + 6] * p.scale, v[8 * e + 7] * p.scale));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

// dK / dV, one CTA per (key block of 128, K/V head, batch row).  Units are
// (query block i of 128, query head h of the group), the last query block
// first, so the CTAs of all key blocks of a batch row read the same Q / dO
// tiles at about the same time and find them in L2:
//   warp 0      TMA: K and V once; Q_i, dO_i with their lse2 / D rows into a
//               2-stage ring;
//   warp 1      tcgen05.mma: S^T = K Q_i^T and dP^T = V dO_i^T into TMEM,
//               dV += P^T dO_i with P^T read from TMEM, dK += dS^T Q_i with
//               dS^T from shared memory (Q_i, dO_i as MN-major operands),
//               in the order dV_u, S^T_{u+1}, dP^T_{u+1}, dK_u (the Q / dO
//               tiles of unit u+1 land while P^T_u is formed; those of the
//               unit after are prefetched into L2);
//   warps 2-17  per unit: load the warp's S^T columns (32 queries), release
//               S^T, form P^T = 2^(S^T*scale*log2e - lse2) with the causal
//               mask, load the dP^T columns and store P^T as packed bf16 over
//               the warp's own dP^T columns, then dS^T = P^T (dP^T - D) into
//               shared memory.
// dk = dK / sqrt(hd).
template <int HD>
struct DkvLayout {
    static constexpr int KB = HD / 64;
    static constexpr int TILE = KB * 16384;    // [128 x HD] bf16
    static constexpr int K = 0;
    static constexpr int V = K + TILE;
    static constexpr int Q = V + TILE;         // [2] stages
    static constexpr int DO = Q + 2 * TILE;    // [2] stages
    static constexpr int DST = DO + 2 * TILE;  // dS^T [128 keys x 128 queries] bf16, two 64-query boxes
    static constexpr int LSE = DST + 32768;    // [2][128] fp32 lse2 of the stage's queries
    static constexpr int DD = LSE + 1024;      // [2][128] fp32 D
    static constexpr int BAR = DD + 1024;
    static constexpr int BYTES = BAR + 256;  // the dynamic shared memory base is 1024-aligned (checked)
    static_assert(BYTES <= 232448, "dK/dV shared memory exceeds the per-block limit");
};

template <int HD>
__global__ void __launch_bounds__(NTB, 1) attn_dkv_tc_kernel(const __grid_constant__ CUtensorMap tmQKV,
                                                            const __grid_constant__ CUtensorMap tmDO,
                                                            const BwdParams p) {
    using Lay = DkvLayout<HD>;
    constexpr int KB = Lay::KB, TILE = Lay::TILE;
    extern __shared__ __align__(1024) uint8_t smem_dyn[];
    if ((smem_u32(smem_dyn) & 1023u) != 0) {
        if (threadIdx.x == 0) set_status(p.status, ST_BAD_LAYOUT);
        return;
    }
    uint8_t* smem = smem_dyn;
    const uint32_t base = smem_u32(smem);
    const uint32_t sK = base + Lay::K, sV = base + Lay::V, sQ = base + Lay::Q, sDO = base + Lay::DO;
    const uint32_t sDST = base + Lay::DST;
    const float* lse_s = reinterpret_cast<const float*>(smem + Lay::LSE);
    const float* d_s = reinterpret_cast<const float*>(smem + Lay::DD);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::BAR);
    const uint32_t b0 = smem_u32(bars);
    const uint32_t kv_full = b0, qo_full = b0 + 8, qo_empty = b0 + 24;  // qo_*[2]
    const uint32_t st_full = b0 + 40, dpt_full = b0 + 48, st_free = b0 + 56;
    const uint32_t p_full = b0 + 64, ds_full = b0 + 72, ds_free = b0 + 80, dkv_done = b0 + 88;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 12);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kvb = blockIdx.z;  // grid z slowest: key block 0 (the most units) launches first
    const int g = blockIdx.y, b = blockIdx.x;
    const int Hg = p.H / p.nkv;
    const int row0 = b * p.T;
    const int Nqkv = (p.H + 2 * p.nkv) * HD;
    const int nunits = (p.nqb - kvb) * Hg;

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        for (int s = 0; s < 2; ++s) { mbar_init(qo_full + 8 * s, 1); mbar_init(qo_empty + 8 * s, 1); }
        mbar_init(st_full, 1);
        mbar_init(dpt_full, 1);
        mbar_init(st_free, NSM);
        mbar_init(p_full, NSM);
        mbar_init(ds_full, NSM);
        mbar_init(ds_free, 1);
        mbar_init(dkv_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), 512);
    if (warp == 0 && lane == 0) { tma_prefetch(&tmQKV); tma_prefetch(&tmDO); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tSt = tmem, tdPt = tmem + 128, tdV = tmem + 256, tdK = tmem + 256 + HD;

    if (warp == 0) {
        if (lane == 0) {
            const int xk = (p.H + g) * HD, xv = (p.H + p.nkv + g) * HD;
            mbar_expect_tx(kv_full, 2 * TILE);
#pragma unroll
            for (int kb = 0; kb < KB; ++kb) {
                tma_load_2d(sK + kb * 16384, &tmQKV, xk + kb * 64, row0 + kvb * 128, kv_full);
                tma_load_2d(sV + kb * 16384, &tmQKV, xv + kb * 64, row0 + kvb * 128, kv_full);
            }
            int issued = 0;
            for (int u = 0; u < nunits; ++u) {
                const int st = u & 1;
                const int i = p.nqb - 1 - u / Hg, h = g * Hg + u % Hg;  // last query block first
                if (!mbar_wait(qo_empty + 8 * st, ((u >> 1) & 1) ^ 1, abort_flag, p.status)) break;
                mbar_expect_tx(qo_full + 8 * st, 2 * TILE + 1024);
                const size_t si = ((size_t)b * p.H + h) * attn_tpad(p.T) + (size_t)i * 128;
                bulk_load(base + Lay::LSE + st * 512, p.lse2 + si, 512, qo_full + 8 * st);
                bulk_load(base + Lay::DD + st * 512, p.D + si, 512, qo_full + 8 * st);
#pragma unroll
                for (int kb = 0; kb < KB; ++kb) {
                    tma_load_2d(sQ + st * TILE + kb * 16384, &tmQKV, h * HD + kb * 64, row0 + i * 128,
                                qo_full + 8 * st);
                    tma_load_2d(sDO + st * TILE + kb * 16384, &tmDO, h * HD + kb * 64, row0 + i * 128,
                                qo_full + 8 * st);
                }
                issued = u + 1;
                // the unit after next into L2, so its load finds it there once a stage frees
                if (u + 2 < nunits) {
                    const int i2 = p.nqb - 1 - (u + 2) / Hg, h2 = g * Hg + (u + 2) % Hg;
#pragma unroll
                    for (int kb = 0; kb < KB; ++kb) {
                        tma_prefetch_l2_2d(&tmQKV, h2 * HD + kb * 64, row0 + i2 * 128);
                        tma_prefetch_l2_2d(&tmDO, h2 * HD + kb * 64, row0 + i2 * 128);
                    }
                }
            }
            if (*abort_flag) {
                drain(kv_full, 0);
                for (int u = (issued > 2 ? issued - 2 : 0); u < issued; ++u) drain(qo_full + 8 * (u & 1), (u >> 1) & 1);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id_s = idesc_bf16(128, 128, false, false);
            const uint32_t id_kv = idesc_bf16(128, HD, false, true);
            // S^T_u = K Q_u^T
            auto scores = [&](int u) -> bool {
                const int st = u & 1;
                if (!mbar_wait(qo_full + 8 * st, (u >> 1) & 1, abort_flag, p.status)) return false;
                tc_fence_after();
#pragma unroll
                for (int ks = 0; ks < HD / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                    mma_bf16(tSt, smem_desc(sK + off, 16, 1024), smem_desc(sQ + st * TILE + off, 16, 1024), id_s,
                             ks > 0 ? 1u : 0u);
                }
                mma_commit(st_full);
                return true;
            };
            // dP^T_u = V dO_u^T (Q_u / dO_u already landed)
            auto dpt = [&](int u) {
                const int st = u & 1;
#pragma unroll
                for (int ks = 0; ks < HD / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                    mma_bf16(tdPt, smem_desc(sV + off, 16, 1024), smem_desc(sDO + st * TILE + off, 16, 1024), id_s,
                             ks > 0 ? 1u : 0u);
                }
                mma_commit(dpt_full);
            };
            bool ok = mbar_wait(kv_full, 0, abort_flag, p.status) && scores(0);
            if (ok) dpt(0);
            for (int u = 0; ok && u < nunits; ++u) {
                const int st = u & 1;
                // dV += P^T_u dO_u: queries 16kk..16kk+15 sit in the packed columns
                // 32*(kk/2) + 8*(kk%2) of dP^T (written by column group kk/2)
                if (!mbar_wait(p_full, u & 1, abort_flag, p.status)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16_ts(tdV, tdPt + 32 * (kk >> 1) + 8 * (kk & 1),
                                smem_desc(sDO + st * TILE + kk * 2048, 16384, 1024), id_kv,
                                (u > 0 || kk > 0) ? 1u : 0u);
                // the next unit's scores (its Q / dO tiles are loaded by now), then its
                // dP^T, which overwrites P^T only after the dV MMAs (issue order)
                if (u + 1 < nunits) {
                    if (!mbar_wait(st_free, u & 1, abort_flag, p.status) || !scores(u + 1)) break;
                    dpt(u + 1);
                }
                if (!mbar_wait(ds_full, u & 1, abort_flag, p.status)) break;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16(tdK, smem_desc(sDST + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                             smem_desc(sQ + st * TILE + kk * 2048, 16384, 1024), id_kv, (u > 0 || kk > 0) ? 1u : 0u);
                mma_commit(ds_free);
                mma_commit(qo_empty + 8 * st);
            }
            mma_commit(dkv_done);
        }
    } else {
        // warps 2..17: TMEM lane quarter q (key rows), query column group cg (32 queries)
        const int q = warp & 3, cg = (warp - 2) >> 2;
        const int r = q * 32 + lane;
        const int kpos = kvb * 128 + r;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        bool ok = true;
        for (int u = 0; u < nunits; ++u) {
            const int st = u & 1;
            const int i = p.nqb - 1 - u / Hg;
            if (!warp_wait(st_full, u & 1, abort_flag, p.status) ||
                !warp_wait(qo_full + 8 * st, (u >> 1) & 1, abort_flag, p.status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t rs[32];
            tmem_ld32_issue(tSt + lane_off + cg * 32, rs);
            tmem_wait_ld();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(st_free);
            // query q0 + e sees this key when lo <= e (causal) and e <= hi (inside the row)
            const int q0 = i * 128 + cg * 32;
            const int lo = kpos - q0, hi = p.T - 1 - q0;
            const float4* l4 = reinterpret_cast<const float4*>(lse_s + st * 128 + cg * 32);
            float pv[32];
            if (__all_sync(0xffffffffu, lo <= 0 && hi >= 31)) {
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const float4 l = l4[k];
                    pv[4 * k] = ex2(fmaf(__uint_as_float(rs[4 * k]), p.scale_log2, -l.x));
                    pv[4 * k + 1] = ex2(fmaf(__uint_as_float(rs[4 * k + 1]), p.scale_log2, -l.y));
                    pv[4 * k + 2] = ex2(fmaf(__uint_as_float(rs[4 * k + 2]), p.scale_log2, -l.z));
                    pv[4 * k + 3] = ex2(fmaf(__uint_as_float(rs[4 * k + 3]), p.scale_log2, -l.w));
                }
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const float4 l = l4[k];
                    const float lv[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const int e = 4 * k + t;
                        pv[e] = (e >= lo && e <= hi) ? ex2(fmaf(__uint_as_float(rs[e]), p.scale_log2, -lv[t])) : 0.f;
                    }
                }
            }
            if (!warp_wait(dpt_full, u & 1, abort_flag, p.status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t rd[32];
            tmem_ld32_issue(tdPt + lane_off + cg * 32, rd);
            tmem_wait_ld();
            // P^T over the first half of this warp's own dP^T columns (just read)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                uint32_t pk[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) pk[e] = pack_bf16(pv[16 * hf + 2 * e], pv[16 * hf + 2 * e + 1]);
                tmem_st8_nowait(tdPt + lane_off + cg * 32 + 8 * hf, pk);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
            // dS^T = P^T (dP^T - D); masked entries have P = 0 and D, dP finite
            const float4* d4 = reinterpret_cast<const float4*>(d_s + st * 128 + cg * 32);
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float4 dd = d4[k];
                pv[4 * k] *= __uint_as_float(rd[4 * k]) - dd.x;
                pv[4 * k + 1] *= __uint_as_float(rd[4 * k + 1]) - dd.y;
                pv[4 * k + 2] *= __uint_as_float(rd[4 * k + 2]) - dd.z;
                pv[4 * k + 3] *= __uint_as_float(rd[4 * k + 3]) - dd.w;
            }
            // the dK MMAs of the previous unit have read the dS^T tile
            if (u > 0 && !warp_wait(ds_free, (u - 1) & 1, abort_flag, p.status)) {
                ok = false;
                break;
            }
            uint8_t* drow = smem + Lay::DST + (cg >> 1) * 16384 + r * 128;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int c8 = (cg & 1) * 4 + k;
                const float* d = pv + 8 * k;
                *reinterpret_cast<uint4*>(drow + ((c8 ^ (r & 7)) << 4)) =
                    make_uint4(pack_bf16(d[0], d[1]), pack_bf16(d[2], d[3]), pack_bf16(d[4], d[5]),
                               pack_bf16(d[6], d[7]));
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(ds_full);
        }
        if (ok && warp_wait(dkv_done, 0, abort_flag, p.status)) {
            tc_fence_after();
            // column groups 0 and 1 write the two halves of dv, 2 and 3 those of dk
            const bool isk = cg >= 2;
            const int c0 = (cg & 1) * (HD / 2);
            const uint32_t tsrc = (isk ? tdK : tdV) + lane_off + c0;
            const float sc = isk ? p.scale : 1.f;
            const bool live = kpos < p.T;
            bf16* out = p.dqkv + ((size_t)row0 + (live ? kpos : 0)) * Nqkv + (isk ? p.H + g : p.H + p.nkv + g) * HD + c0;
#pragma unroll
            for (int c = 0; c < HD / 64; ++c) {
                float v[32];
                tmem_ld32(tsrc + c * 32, v);
                if (live) {
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        *reinterpret_cast<uint4*>(out + c * 32 + 8 * e) =
                            make_uint4(pack_bf16(v[8 * e] * sc, v[8 * e + 1] * sc),
                                       pack_bf16(v[8 * e + 2] * sc, v[8 * e + 3] * sc),
                                       pack_bf16(v[8 * e + 4] * sc, v[8 * e + 5] * sc),
                                       pack_bf16(v[8 * e + 6] * sc, v[8 * e + 7] * sc));
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 512);
    }
}

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

// Tensor map over a row-major bf16 [rows, cols] array, box [box_rows, 64],
// 128-byte swizzle, zero fill past the last row.
bool map_rows(CUtensorMap* map, const void* ptr, uint64_t cols, uint64_t rows, uint32_t box_rows) {
    auto fn = encode_fn();
    if (!fn) return false;
    cuuint64_t dims[2] = {cols, rows};
    cuuint64_t strides[1] = {cols * 2};
    cuuint32_t box[2] = {64, box_rows};
    cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

template <int HD>
int fwd_launch(const CUtensorMap& map, const AttnParams& p, cudaStream_t s) {
    if (ensure_smem_limit((const void*)attn_fwd_tc_kernel<HD>, FwdLayout<HD>::BYTES) != cudaSuccess) return -1;
    dim3 grid(p.H, p.B, p.nqb);
    attn_fwd_tc_kernel<HD><<<grid, NT, FwdLayout<HD>::BYTES, s>>>(map, p);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

template <int HD>
int dq_launch(const CUtensorMap& kv, const CUtensorMap& do128, const BwdParams& p, cudaStream_t s) {
    if (ensure_smem_limit((const void*)attn_dq_tc_kernel<HD>, DqLayout<HD>::BYTES) != cudaSuccess) return -1;
    attn_dq_tc_kernel<HD><<<dim3(p.H, p.B, p.nqb), NTB, DqLayout<HD>::BYTES, s>>>(kv, do128, p);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

template <int HD>
int dkv_launch(const CUtensorMap& kv, const CUtensorMap& do128, const BwdParams& p, cudaStream_t s) {
    if (ensure_smem_limit((const void*)attn_dkv_tc_kernel<HD>, DkvLayout<HD>::BYTES) != cudaSuccess) return -1;
    attn_dkv_tc_kernel<HD><<<dim3(p.B, p.nkv, p.nqb), NTB, DkvLayout<HD>::BYTES, s>>>(kv, do128, p);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

// Parameters and the two tensor maps (qkv and dO, 128-row boxes) of both kernels.
bool bwd_setup(const void* qkv, const void* o, const void* dO, const float* lse, float* Dbuf, void* dqkv, int B,
               int T, int H, int nkv, int hd, int* status, BwdParams* p, CUtensorMap* kv, CUtensorMap* do128) {
    if (!attention_tc_bwd_supported(hd)) return false;
    if (!aligned16(qkv) || !aligned16(dO) || !aligned16(dqkv) || !aligned16(Dbuf) || (o && !aligned16(o)))
        return false;
    if (B > 65535 || H > 65535 || nkv < 1 || H % nkv != 0) return false;
    const int Nqkv = (H + 2 * nkv) * hd;
    if (!map_rows(kv, qkv, Nqkv, (uint64_t)B * T, 128) || !map_rows(do128, dO, (uint64_t)H * hd, (uint64_t)B * T, 128))
        return false;
    *p = BwdParams{};
    p->B = B; p->T = T; p->H = H; p->nkv = nkv; p->nqb = (T + 127) / 128;
    p->scale = 1.f / sqrtf((float)hd);
    p->scale_log2 = kLog2e * p->scale;
    p->D = Dbuf;
    p->lse2 = Dbuf + attn_stat_elems(B, T, H);
    p->dqkv = reinterpret_cast<bf16*>(dqkv);
    p->status = status;
    return true;
}

}  // namespace

int attention_tc_fwd(const void* qkv, void* o, float* lse, int B, int T, int H, int nkv, int hd, void*, size_t,
                     int* status, cudaStream_t s) {
    if (hd != 64 && hd != 128) return 1;
    if (!aligned16(qkv) || !aligned16(o) || B > 65535 || H > 65535) return 1;
    const int Nqkv = (H + 2 * nkv) * hd;
    CUtensorMap map;
    if (!map_rows(&map, qkv, Nqkv, (uint64_t)B * T, 128)) return 1;
    AttnParams p;
    p.B = B; p.T = T; p.H = H; p.nkv = nkv; p.nqb = (T + 127) / 128;
    p.scale_log2 = kLog2e / sqrtf((float)hd);
    p.o = reinterpret_cast<bf16*>(o);
    p.lse = lse;
    p.status = status;
    return hd == 128 ? fwd_launch<128>(map, p, s) : fwd_launch<64>(map, p, s);
}

bool attention_tc_bwd_supported(int hd) { return hd == 64 || hd == 128; }

int attention_tc_bwd_dq(const void* qkv, const void* o, const void* dO, const float* lse, float* Dbuf, void* dqkv,
                        int B, int T, int H, int nkv, int hd, int* status, cudaStream_t s) {
    BwdParams p;
    CUtensorMap kv, do128;
    if (!o || !lse || !bwd_setup(qkv, o, dO, lse, Dbuf, dqkv, B, T, H, nkv, hd, status, &p, &kv, &do128)) return 1;
    {
        const long long threads = (long long)attn_stat_elems(B, T, H) * (hd / 8);
        const unsigned blocks = (unsigned)((threads + 255) / 256);
        const bf16* ob = reinterpret_cast<const bf16*>(o);
        const bf16* db = reinterpret_cast<const bf16*>(dO);
        float* D = Dbuf;
        float* l2 = Dbuf + attn_stat_elems(B, T, H);
        if (hd == 128) attn_bwd_stats_kernel<128><<<blocks, 256, 0, s>>>(ob, db, lse, D, l2, B, T, H);
        else attn_bwd_stats_kernel<64><<<blocks, 256, 0, s>>>(ob, db, lse, D, l2, B, T, H);
        count_launch();
        if (cudaGetLastError() != cudaSuccess) return -1;
    }
    return hd == 128 ? dq_launch<128>(kv, do128, p, s) : dq_launch<64>(kv, do128, p, s);
}

int attention_tc_bwd_dkv(const void* qkv, const void* dO, float* Dbuf, void* dqkv, int B, int T, int H, int nkv,
                         int hd, int* status, cudaStream_t s) {
    BwdParams p;
    CUtensorMap kv, do128;
    if (!bwd_setup(qkv, nullptr, dO, nullptr, Dbuf, dqkv, B, T, H, nkv, hd, status, &p, &kv, &do128)) return 1;
    return hd == 128 ? dkv_launch<128>(kv, do128, p, s) : dkv_launch<64>(kv, do128, p, s);
}

int attention_tc_bwd(const void* qkv, const void* o, const void* dO, const float* lse, float* Dbuf, void* dqkv,
                     int B, int T, int H, int nkv, int hd, void*, size_t, int* status, cudaStream_t s) {
    int r = attention_tc_bwd_dq(qkv, o, dO, lse, Dbuf, dqkv, B, T, H, nkv, hd, status, s);
    if (r != 0) return r;
    return attention_tc_bwd_dkv(qkv, dO, Dbuf, dqkv, B, T, H, nkv, hd, status, s);
}

size_t attention_tc_workspace_bytes(int, int, int, int, int) { return 0; }

}  // namespace nc
