// Causal multi-query attention on the tcgen05 tensor cores (bf16 operands,
// fp32 accumulation in TMEM, fp32 softmax).  Model item: multi-query
// attention, every query head reading the one shared K/V head (nanochat
// announcement, vpshk.cn, architecture list), causal within a row, scores
// scaled by 1/sqrt(hd).
//
// Forward, one CTA per (query block of 128 positions, head, batch row):
//   warp 0     TMA: the Q tile once, then K_j / V_j tiles (2-stage rings)
//              for key blocks j = 0..qb (causal: blocks past the diagonal
//              are never loaded);
//   warp 1     tcgen05.mma: S_j = Q K_j^T into one of two TMEM score
//              buffers, then O += P_{j-1} V_{j-1} (issued one block behind,
//              so the next score tile is computed while softmax runs);
//   warps 2-5  softmax, one query row per thread: scores from TMEM, causal
//              mask on the diagonal block, running max in the log2 domain
//              with lazy rescaling of O (only when the max grows by more
//              than 2^8), P as bf16 into shared memory in the 128-byte
//              swizzled K-major layout the next MMA reads.
// The K/V head is shared by all query heads; its tiles are re-read by the
// H CTAs of a query block from L2.
#include "attention_tc.h"
#include "tc_common.cuh"
#include <cudaTypedefs.h>

namespace nc {
namespace {
using namespace tc;

constexpr int NT = 192;   // forward: producer, MMA, 4 softmax warps
constexpr int NTB = 320;  // backward: producer, MMA, 8 softmax warps (two per TMEM lane quarter)
constexpr int STG = 2;
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
    static constexpr int KB = HD / 64;          // 64-column blocks of the head dim
    static constexpr int TILE = KB * 16384;     // [128 x HD] bf16, 128B-swizzled
    static constexpr int Q = 0;
    static constexpr int K = Q + TILE;
    static constexpr int V = K + STG * TILE;
    static constexpr int P = V + STG * TILE;    // [128 x 128] bf16
    static constexpr int BAR = P + 32768;
    static constexpr int BYTES = BAR + 256 + 1024;  // + barriers, + alignment slack
};

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

template <int HD>
__global__ void __launch_bounds__(NT, 1) attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm, const AttnParams p) {
    using Lay = FwdLayout<HD>;
    constexpr int KB = Lay::KB;
    constexpr int TILE = Lay::TILE;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t base = smem_u32(smem);
    const uint32_t sQ = base + Lay::Q, sK = base + Lay::K, sV = base + Lay::V, sP = base + Lay::P;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::BAR);
    const uint32_t b0 = smem_u32(bars);
    const uint32_t q_full = b0, k_full = b0 + 8, k_empty = b0 + 24, v_full = b0 + 40, v_empty = b0 + 56;
    const uint32_t s_full = b0 + 72, s_empty = b0 + 88, p_full = b0 + 104, o_done = b0 + 112;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qb = p.nqb - 1 - (int)blockIdx.z;  // grid z slowest: the longest blocks launch first
    const int h = blockIdx.x, b = blockIdx.y, g = h / (p.H / p.nkv);
    const int nblk = qb + 1;
    const int row0 = b * p.T;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        for (int s = 0; s < STG; ++s) {
            mbar_init(k_full + 8 * s, 1); mbar_init(k_empty + 8 * s, 1);
            mbar_init(v_full + 8 * s, 1); mbar_init(v_empty + 8 * s, 1);
        }
        for (int s = 0; s < 2; ++s) { mbar_init(s_full + 8 * s, 1); mbar_init(s_empty + 8 * s, 4); }
        mbar_init(p_full, 4);
        mbar_init(o_done, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), 512);
    if (warp == 0 && lane == 0) tma_prefetch(&tm);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem, tO = tmem + 256;

    if (warp == 0) {
        // lane 0 loads Q and the K ring, lane 1 the V ring: each waits only on
        // its own ring, so K tiles run ahead of the V slots that P*V frees late
        if (lane < 2) {
            const bool kl = lane == 0;
            const int xq = h * HD, xkv = kl ? (p.H + g) * HD : (p.H + p.nkv + g) * HD;
            const uint32_t full = kl ? k_full : v_full, empty = kl ? k_empty : v_empty;
            const uint32_t dst = kl ? sK : sV;
            if (kl) {
                mbar_expect_tx(q_full, TILE);
#pragma unroll
                for (int kb = 0; kb < KB; ++kb)
                    tma_load_2d(sQ + kb * 16384, &tm, xq + kb * 64, row0 + qb * 128, q_full);
            }
            int issued = 0;
            for (int j = 0; j < nblk; ++j) {
                const int st = j % STG;
                const uint32_t ph = (j / STG) & 1;
                if (!mbar_wait(empty + 8 * st, ph ^ 1, abort_flag, p.status)) break;
                mbar_expect_tx(full + 8 * st, TILE);
#pragma unroll
                for (int kb = 0; kb < KB; ++kb)
                    tma_load_2d(dst + st * TILE + kb * 16384, &tm, xkv + kb * 64, row0 + j * 128, full + 8 * st);
                issued = j + 1;
            }
            if (*abort_flag) {
                // let copies in flight land before the block exits
                uint64_t t0 = globaltimer();
                if (kl) while (!mbar_try(q_full, 0) && globaltimer() - t0 < 1000000ull) {}
                for (int j = (issued > STG ? issued - STG : 0); j < issued; ++j) {
                    t0 = globaltimer();
                    while (!mbar_try(full + 8 * (j % STG), (j / STG) & 1) && globaltimer() - t0 < 1000000ull) {}
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id_s = idesc_bf16(128, 128, false, false);
            const uint32_t id_o = idesc_bf16(128, HD, false, true);
            bool ok = mbar_wait(q_full, 0, abort_flag, p.status);
            for (int j = 0; ok && j <= nblk; ++j) {
                if (j < nblk) {
                    const int st = j % STG, sb = j & 1;
                    if (!mbar_wait(k_full + 8 * st, (j / STG) & 1, abort_flag, p.status)) break;
                    if (!mbar_wait(s_empty + 8 * sb, ((j >> 1) & 1) ^ 1, abort_flag, p.status)) break;
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < HD / 16; ++ks) {
                        const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                        mma_bf16(tS + sb * 128, smem_desc(sQ + off, 16, 1024), smem_desc(sK + st * TILE + off, 16, 1024),
                                 id_s, ks > 0 ? 1u : 0u);
                    }
                    mma_commit(s_full + 8 * sb);
                    mma_commit(k_empty + 8 * st);
                }
                if (j > 0) {
                    const int jj = j - 1, st = jj % STG;
                    if (!mbar_wait(p_full, jj & 1, abort_flag, p.status)) break;
                    if (!mbar_wait(v_full + 8 * st, (jj / STG) & 1, abort_flag, p.status)) break;
                    tc_fence_after();
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks) {
                        const uint32_t offp = (ks >> 2) * 16384 + (ks & 3) * 32;
                        mma_bf16(tO, smem_desc(sP + offp, 16, 1024), smem_desc(sV + st * TILE + ks * 2048, 16384, 1024),
                                 id_o, (jj > 0 || ks > 0) ? 1u : 0u);
                    }
                    mma_commit(o_done);
                    mma_commit(v_empty + 8 * st);
                }
            }
        }
    } else {
        // ---------------- softmax warps: warp w reads TMEM lanes 32*(w%4)..
        const int q = warp & 3;
        const int r = q * 32 + lane;  // row of the tile
        const int qpos = qb * 128 + r;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        float m = -INFINITY, l = 0.f;
        bool ok = true;
        for (int j = 0; j < nblk; ++j) {
            const int sb = j & 1;
            if (!warp_wait(s_full + 8 * sb, (j >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
            tc_fence_after();
            float s[128];
            {
                uint32_t rr[128];
#pragma unroll
                for (int c = 0; c < 4; ++c) tmem_ld32_issue(tS + lane_off + sb * 128 + c * 32, rr + 32 * c);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 128; ++i) s[i] = __uint_as_float(rr[i]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(s_empty + 8 * sb);
            float mx = -INFINITY;
            if (j == qb) {
#pragma unroll
                for (int c = 0; c < 128; ++c) {
                    s[c] = (c <= r) ? s[c] * p.scale_log2 : -INFINITY;
                    mx = fmaxf(mx, s[c]);
                }
            } else {
#pragma unroll
                for (int c = 0; c < 128; ++c) {
                    s[c] *= p.scale_log2;
                    mx = fmaxf(mx, s[c]);
                }
            }
            const bool rescale = mx > m + 8.f;
            const float mu = rescale ? mx : m;
            const float alpha = rescale ? ex2(m - mx) : 1.f;
            float sum = 0.f;
#pragma unroll
            for (int c = 0; c < 128; ++c) {
                s[c] = ex2(s[c] - mu);
                sum += s[c];
            }
            if (j > 0) {
                if (!warp_wait(o_done, (j - 1) & 1, abort_flag, p.status)) { ok = false; break; }
                tc_fence_after();
                if (__any_sync(0xffffffffu, rescale)) {
#pragma unroll
                    for (int c = 0; c < HD / 32; ++c) {
                        float o[32];
                        tmem_ld32(tO + lane_off + c * 32, o);
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] *= alpha;
                        tmem_st32(tO + lane_off + c * 32, o);
                    }
                }
            }
            l = l * alpha + sum;
            m = mu;
            uint8_t* prow = smem + Lay::P + r * 128;
#pragma unroll
            for (int kb = 0; kb < 2; ++kb) {
#pragma unroll
                for (int c8 = 0; c8 < 8; ++c8) {
                    const float* v = s + kb * 64 + c8 * 8;
                    uint4 u = make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                                         pack_bf16(v[6], v[7]));
                    *reinterpret_cast<uint4*>(prow + kb * 16384 + ((c8 ^ (r & 7)) << 4)) = u;
                }
            }
            fence_proxy_async_smem();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
        }
        if (ok && warp_wait(o_done, (nblk - 1) & 1, abort_flag, p.status)) {
            tc_fence_after();
            const float inv = 1.f / l;
            const bool live = qpos < p.T;
            bf16* orow = p.o + ((size_t)row0 + qpos) * (size_t)(p.H * HD) + h * HD;
#pragma unroll
            for (int c = 0; c < HD / 32; ++c) {
                float o[32];
                tmem_ld32(tO + lane_off + c * 32, o);
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
            if (live) p.lse[((size_t)b * p.H + h) * attn_tpad(p.T) + qpos] = (m + __log2f(l)) * kLn2;
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
// dQ, one CTA per (query block of 128, head, batch row).  Key blocks j = 0..qb
// are processed as 64-key sub-blocks t: S_t = Q K_t^T and dP_t = dO V_t^T into
// one of three TMEM buffers; per query row (one per thread)
// P = 2^(S*scale*log2e - lse*log2e) with the causal mask and dS = P (dP - D),
// as bf16 into one of two shared-memory tiles; dQ += dS_{t-2} K_{t-2} is issued
// two sub-blocks behind (the score MMAs of two sub-blocks cover the softmax
// round trip), with the K tile read again as an MN-major operand.
// dq = dQ / sqrt(hd).
template <int HD>
struct DqLayout {
    static constexpr int KB = HD / 64;
    static constexpr int TILE = KB * 16384;   // [128 x HD]: Q, dO
    static constexpr int HTILE = KB * 8192;   // [64 x HD]: a K or V sub-block
    static constexpr int RING = 4;            // K and V sub-block stages
    static constexpr int Q = 0;
    static constexpr int DO = Q + TILE;
    static constexpr int K = DO + TILE;
    static constexpr int V = K + RING * HTILE;
    static constexpr int DS = V + RING * HTILE;  // [2][128 x 64] bf16
    static constexpr int BAR = DS + 32768;
    static constexpr int BYTES = BAR + 256 + 1024;
    static_assert(BYTES <= 232448, "dQ shared memory exceeds the per-block limit");
};

struct BwdParams {
    int B, T, H, nkv, nqb;
    float scale_log2, scale;
    const float* lse;
    const float* D;
    bf16* dqkv;
    int* status;
    // When rqk is set, dq and dk are written as gradients of the pre-norm
    // projections (QK-norm and RoPE backward fused): qkv holds the saved
    // post-RoPE vectors, rqk their inverse RMS [B*T, H+nkv], cos/sin [T, hd/2].
    const bf16* qkv;
    const float* rqk;
    const float* cos_t;
    const float* sin_t;
};

// Writes the gradient of the pre-norm projection for one head row: g = scale *
// (the TMEM row at tsrc) is the gradient of y = rope(rmsnorm(x)); with the
// saved y, u = R^T g and w = R^T y (inverse rotation of the pairs (j, j+HD/2))
// give dx = r * (u - w * mean(u * w)).  Two passes over TMEM keep registers low.
template <int HD>
__device__ __forceinline__ void store_grad_through_qknorm(uint32_t tsrc, float scale, const bf16* y, float r,
                                                          const float* cs, const float* sn, bf16* out, bool live) {
    constexpr int NC = HD / 32, HALF = HD / 2;
    float dot = 0.f;
#pragma unroll 1
    for (int pass = 0; pass < 2; ++pass) {
        const float mdot = dot / (float)HD;
#pragma unroll 1
        for (int c = 0; c < NC / 2; ++c) {
            float g1[32], g2[32];
            tmem_ld32(tsrc + c * 32, g1);
            tmem_ld32(tsrc + (c + NC / 2) * 32, g2);
            if (!live) continue;
#pragma unroll
            for (int i = 0; i < 32; i += 8) {
                float y1[8], y2[8];
                load_vec(y + c * 32 + i, y1);
                load_vec(y + HALF + c * 32 + i, y2);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int j = c * 32 + i + e;
                    const float co = cs[j], si = sn[j];
                    const float a = g1[i + e] * scale, b = g2[i + e] * scale;
                    const float u1 = a * co + b * si, u2 = b * co - a * si;
                    const float w1 = y1[e] * co + y2[e] * si, w2 = y2[e] * co - y1[e] * si;
                    if (pass == 0) {
                        dot += u1 * w1 + u2 * w2;
                    } else {
                        g1[i + e] = r * (u1 - w1 * mdot);
                        g2[i + e] = r * (u2 - w2 * mdot);
                    }
                }
            }
            if (pass == 1) {
#pragma unroll
                for (int t4 = 0; t4 < 4; ++t4) {
                    store_vec(out + c * 32 + 8 * t4, g1 + 8 * t4);
                    store_vec(out + HALF + c * 32 + 8 * t4, g2 + 8 * t4);
                }
            }
        }
    }
}

__device__ __forceinline__ void drain(uint32_t bar, uint32_t parity) {
    uint64_t t0 = globaltimer();
    while (!mbar_try(bar, parity) && globaltimer() - t0 < 1000000ull) {}
}

template <int HD>
__global__ void __launch_bounds__(NTB, 1) attn_dq_tc_kernel(const __grid_constant__ CUtensorMap tmQKV,
                                                           const __grid_constant__ CUtensorMap tmKV64,
                                                           const __grid_constant__ CUtensorMap tmDO,
                                                           const BwdParams p) {
    using Lay = DqLayout<HD>;
    constexpr int KB = Lay::KB, TILE = Lay::TILE, HTILE = Lay::HTILE, RING = Lay::RING;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t base = smem_u32(smem);
    const uint32_t sQ = base + Lay::Q, sDO = base + Lay::DO, sK = base + Lay::K, sV = base + Lay::V;
    const uint32_t sDS = base + Lay::DS;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::BAR);
    const uint32_t b0 = smem_u32(bars);
    const uint32_t qd_full = b0;
    const uint32_t k_full = b0 + 8, k_empty = b0 + 40, v_full = b0 + 72, v_empty = b0 + 104;  // [RING]
    const uint32_t s_full = b0 + 136, s_empty = b0 + 160;  // [3]: S/dP TMEM buffers
    const uint32_t ds_full = b0 + 184, ds_done = b0 + 200; // [2]: dS smem tiles
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 28);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int qb = p.nqb - 1 - (int)blockIdx.z;  // longest blocks launch first
    const int h = blockIdx.x, b = blockIdx.y, g = h / (p.H / p.nkv);
    const int nblk = qb + 1, nsub = 2 * nblk;
    const int row0 = b * p.T;
    const int Nqkv = (p.H + 2 * p.nkv) * HD;

    if (threadIdx.x == 0) {
        mbar_init(qd_full, 1);
        for (int s = 0; s < RING; ++s) {
            mbar_init(k_full + 8 * s, 1); mbar_init(k_empty + 8 * s, 1);
            mbar_init(v_full + 8 * s, 1); mbar_init(v_empty + 8 * s, 1);
        }
        for (int s = 0; s < 2; ++s) { mbar_init(ds_full + 8 * s, 8); mbar_init(ds_done + 8 * s, 1); }
        for (int s = 0; s < 3; ++s) { mbar_init(s_full + 8 * s, 1); mbar_init(s_empty + 8 * s, 8); }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), 512);
    if (warp == 0 && lane == 0) { tma_prefetch(&tmQKV); tma_prefetch(&tmKV64); tma_prefetch(&tmDO); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tS = tmem, tdP = tmem + 192, tdQ = tmem + 384;  // S[3] and dP[3] of 64 columns

    if (warp == 0) {
        // lane 0 loads Q, dO and the K ring, lane 1 the V ring, one 64-key
        // sub-block per stage (V slots free after dP, K slots after dQ)
        if (lane < 2) {
            const bool kl = lane == 0;
            const int xkv = kl ? (p.H + g) * HD : (p.H + p.nkv + g) * HD;
            const uint32_t full = kl ? k_full : v_full, empty = kl ? k_empty : v_empty;
            const uint32_t dst = kl ? sK : sV;
            if (kl) {
                mbar_expect_tx(qd_full, 2 * TILE);
#pragma unroll
                for (int kb = 0; kb < KB; ++kb) {
                    tma_load_2d(sQ + kb * 16384, &tmQKV, h * HD + kb * 64, row0 + qb * 128, qd_full);
                    tma_load_2d(sDO + kb * 16384, &tmDO, h * HD + kb * 64, row0 + qb * 128, qd_full);
                }
            }
            int issued = 0;
            for (int t = 0; t < nsub; ++t) {
                const int st = t % RING;
                const uint32_t ph = (t / RING) & 1;
                if (!mbar_wait(empty + 8 * st, ph ^ 1, abort_flag, p.status)) break;
                mbar_expect_tx(full + 8 * st, HTILE);
#pragma unroll
                for (int kb = 0; kb < KB; ++kb)
                    tma_load_2d(dst + st * HTILE + kb * 8192, &tmKV64, xkv + kb * 64, row0 + t * 64, full + 8 * st);
                issued = t + 1;
            }
            if (*abort_flag) {
                if (kl) drain(qd_full, 0);
                for (int t = (issued > RING ? issued - RING : 0); t < issued; ++t)
                    drain(full + 8 * (t % RING), (t / RING) & 1);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id_s = idesc_bf16(128, 64, false, false);
            const uint32_t id_q = idesc_bf16(128, HD, false, true);
            if (mbar_wait(qd_full, 0, abort_flag, p.status)) {
                for (int t = 0; t <= nsub + 1; ++t) {
                    if (t < nsub) {
                        const int st = t % RING, sb = t % 3;
                        const uint32_t ph = (t / RING) & 1;
                        if (!mbar_wait(k_full + 8 * st, ph, abort_flag, p.status)) break;
                        if (!mbar_wait(v_full + 8 * st, ph, abort_flag, p.status)) break;
                        if (!mbar_wait(s_empty + 8 * sb, ((t / 3) & 1) ^ 1, abort_flag, p.status)) break;
                        tc_fence_after();
#pragma unroll
                        for (int ks = 0; ks < HD / 16; ++ks) {
                            const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                            const uint32_t offk = st * HTILE + (ks >> 2) * 8192 + (ks & 3) * 32;
                            mma_bf16(tS + sb * 64, smem_desc(sQ + off, 16, 1024), smem_desc(sK + offk, 16, 1024), id_s,
                                     ks > 0 ? 1u : 0u);
                            mma_bf16(tdP + sb * 64, smem_desc(sDO + off, 16, 1024), smem_desc(sV + offk, 16, 1024),
                                     id_s, ks > 0 ? 1u : 0u);
                        }
                        mma_commit(s_full + 8 * sb);
                        mma_commit(v_empty + 8 * st);
                    }
                    if (t > 1) {
                        const int tt = t - 2, st = tt % RING, db = tt & 1;
                        if (!mbar_wait(ds_full + 8 * db, (tt >> 1) & 1, abort_flag, p.status)) break;
                        tc_fence_after();
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks)
                            mma_bf16(tdQ, smem_desc(sDS + db * 16384 + ks * 32, 16, 1024),
                                     smem_desc(sK + st * HTILE + ks * 2048, 8192, 1024), id_q,
                                     (tt > 0 || ks > 0) ? 1u : 0u);
                        mma_commit(ds_done + 8 * db);
                        mma_commit(k_empty + 8 * st);
                    }
                }
            }
        }
    } else {
        // warps 2..9: TMEM lane quarter q = warp % 4 (query rows), key half ch of each sub-block
        const int q = warp & 3, ch = (warp - 2) >> 2;
        const int r = q * 32 + lane;
        const int qpos = qb * 128 + r;
        const bool live = qpos < p.T;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        const size_t si = ((size_t)b * p.H + h) * attn_tpad(p.T) + (live ? qpos : 0);
        const float lse2 = live ? p.lse[si] * kLog2e : 0.f;
        const float Dr = live ? p.D[si] : 0.f;
        bool ok = true;
        for (int t = 0; t < nsub; ++t) {
            const int j = t >> 1, hf = t & 1, sb = t % 3, db = t & 1;
            if (!warp_wait(s_full + 8 * sb, (t / 3) & 1, abort_flag, p.status)) { ok = false; break; }
            tc_fence_after();
            float d0[32];
            {
                float sv[32];
                {
                    uint32_t rs[32], rd[32];
                    tmem_ld32_issue(tS + lane_off + sb * 64 + ch * 32, rs);
                    tmem_ld32_issue(tdP + lane_off + sb * 64 + ch * 32, rd);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) { sv[i] = __uint_as_float(rs[i]); d0[i] = __uint_as_float(rd[i]); }
                }
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const bool valid = live && (j < qb || hf * 64 + ch * 32 + i <= r);
                    d0[i] = valid ? ex2(sv[i] * p.scale_log2 - lse2) * (d0[i] - Dr) : 0.f;
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(s_empty + 8 * sb);
            // dS buffer db was last read by the dQ MMAs of sub-block t-2
            if (t > 1 && !warp_wait(ds_done + 8 * db, ((t >> 1) - 1) & 1, abort_flag, p.status)) { ok = false; break; }
            uint8_t* drow = smem + Lay::DS + db * 16384 + r * 128;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float* v = d0 + 8 * k;
                const int c8 = ch * 4 + k;
                *reinterpret_cast<uint4*>(drow + ((c8 ^ (r & 7)) << 4)) =
                    make_uint4(pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]),
                               pack_bf16(v[6], v[7]));
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(ds_full + 8 * db);
        }
        if (ok && warp_wait(ds_done + 8 * ((nsub - 1) & 1), ((nsub - 1) >> 1) & 1, abort_flag, p.status)) {
            tc_fence_after();
            bf16* out = p.dqkv + ((size_t)row0 + qpos) * Nqkv + h * HD;
            if (p.rqk) {
                // the first four softmax warps write whole rows through the QK-norm backward
                if (ch == 0) {
                    const size_t rowi = (size_t)row0 + (live ? qpos : 0);
                    const int pos = live ? qpos : 0;
                    store_grad_through_qknorm<HD>(tdQ + lane_off, p.scale, p.qkv + rowi * Nqkv + h * HD,
                                                  live ? p.rqk[rowi * (p.H + p.nkv) + h] : 0.f,
                                                  p.cos_t + (size_t)pos * (HD / 2), p.sin_t + (size_t)pos * (HD / 2),
                                                  out, live);
                }
            } else
#pragma unroll
            for (int cc = 0; cc < HD / 64; ++cc) {
                const int c = ch * (HD / 64) + cc;
                float o[32];
                tmem_ld32(tdQ + lane_off + c * 32, o);
                if (live) {
#pragma unroll
                    for (int t4 = 0; t4 < 4; ++t4)
                        *reinterpret_cast<uint4*>(out + c * 32 + 8 * t4) = make_uint4(
                            pack_bf16(o[8 * t4] * p.scale, o[8 * t4 + 1] * p.scale),
                            pack_bf16(o[8 * t4 + 2] * p.scale, o[8 * t4 + 3] * p.scale),
                            pack_bf16(o[8 * t4 + 4] * p.scale, o[8 * t4 + 5] * p.scale),
                            pack_bf16(o[8 * t4 + 6] * p.scale, o[8 * t4 + 7] * p.scale));
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

// dK / dV, one CTA per (key block of 128, kv head, batch row): loops over the
// units (query block of 64, query head of this kv group) that can see the
// key block, in a fixed order (deterministic, no atomics): query blocks from
// the last one down, so the CTAs of all key blocks of a batch row read the
// same Q / dO tiles at about the same time and hit them in L2.  Per unit, with
// the key row as the MMA M dimension: S^T = K Q^T and dP^T = V dO^T into
// double-buffered TMEM; per key row (one per thread) P^T with the causal
// mask and dS^T = P^T (dP^T - D) as bf16 into shared memory; dV += P^T dO and
// dK += dS^T Q accumulate in TMEM over all units.  dk = dK / sqrt(hd).
constexpr int DKV_STG = 3;  // Q/dO/lse/D stages of the dK/dV kernel

template <int HD>
struct DkvLayout {
    static constexpr int KB = HD / 64;
    static constexpr int TILE = KB * 16384;   // [128 x HD]
    static constexpr int HTILE = KB * 8192;   // [64 x HD]
    static constexpr int K = 0;
    static constexpr int V = K + TILE;
    static constexpr int Q = V + TILE;
    static constexpr int DO = Q + DKV_STG * HTILE;
    static constexpr int PT = DO + DKV_STG * HTILE;  // [2][128 x 64] bf16, by unit parity
    static constexpr int DST = PT + 2 * 16384;       // [2][128 x 64] bf16, by unit parity
    static constexpr int LSE = DST + 2 * 16384;      // [DKV_STG][64] floats: lse of the unit's queries
    static constexpr int DD = LSE + DKV_STG * 256;   // [DKV_STG][64] floats: D of the unit's queries
    static constexpr int BAR = DD + DKV_STG * 256;
    static constexpr int BYTES = BAR + 256 + 1024;
    static_assert(BYTES <= 232448, "dK/dV shared memory exceeds the per-block limit");
};

template <int HD>
__global__ void __launch_bounds__(NTB, 1) attn_dkv_tc_kernel(const __grid_constant__ CUtensorMap tmKV,
                                                            const __grid_constant__ CUtensorMap tmQ64,
                                                            const __grid_constant__ CUtensorMap tmDO64,
                                                            const BwdParams p) {
    using Lay = DkvLayout<HD>;
    constexpr int KB = Lay::KB, TILE = Lay::TILE, HTILE = Lay::HTILE;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~(uintptr_t)1023);
    const uint32_t base = smem_u32(smem);
    const uint32_t sK = base + Lay::K, sV = base + Lay::V, sQ = base + Lay::Q, sDO = base + Lay::DO;
    const uint32_t sPT = base + Lay::PT, sDST = base + Lay::DST;
    float* lse_s = reinterpret_cast<float*>(smem + Lay::LSE);
    float* d_s = reinterpret_cast<float*>(smem + Lay::DD);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::BAR);
    const uint32_t b0 = smem_u32(bars);
    const uint32_t kv_full = b0, qo_full = b0 + 8, qo_empty = b0 + 32;  // qo_*[DKV_STG]
    const uint32_t st_full = b0 + 56, st_empty = b0 + 72;              // [2]
    // pd_full[b] / pd_done[b]: P^T and dS^T of the units with parity b written /
    // consumed (once per two units each).  Per-parity barriers keep every wait
    // from being lapped: the softmax warps may run two units ahead of the MMA
    // thread's wait on pd_full.
    const uint32_t pd_full = b0 + 88, pd_done = b0 + 104;              // [2] each
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int kvb = blockIdx.z;  // grid z slowest: key block 0 (the most units) launches first
    const int g = blockIdx.y, b = blockIdx.x;
    const int Hg = p.H / p.nkv;
    const int row0 = b * p.T;
    const int Nqkv = (p.H + 2 * p.nkv) * HD;
    const int nq64 = (p.T + 63) / 64;
    const int i0 = 2 * kvb;
    const int nunits = (nq64 - i0) * Hg;

    if (threadIdx.x == 0) {
        mbar_init(kv_full, 1);
        for (int s = 0; s < DKV_STG; ++s) { mbar_init(qo_full + 8 * s, 1); mbar_init(qo_empty + 8 * s, 1); }
        for (int s = 0; s < 2; ++s) { mbar_init(st_full + 8 * s, 1); mbar_init(st_empty + 8 * s, 8); }
        mbar_init(pd_full, 8);
        mbar_init(pd_full + 8, 8);
        mbar_init(pd_done, 1);
        mbar_init(pd_done + 8, 1);
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), 512);
    if (warp == 0 && lane == 0) { tma_prefetch(&tmKV); tma_prefetch(&tmQ64); tma_prefetch(&tmDO64); }
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
                tma_load_2d(sK + kb * 16384, &tmKV, xk + kb * 64, row0 + kvb * 128, kv_full);
                tma_load_2d(sV + kb * 16384, &tmKV, xv + kb * 64, row0 + kvb * 128, kv_full);
            }
            int issued = 0;
            for (int u = 0; u < nunits; ++u) {
                const int st = u % DKV_STG;
                const int i = nq64 - 1 - u / Hg, h = g * Hg + u % Hg;  // last query block first
                if (!mbar_wait(qo_empty + 8 * st, ((u / DKV_STG) & 1) ^ 1, abort_flag, p.status)) break;
                mbar_expect_tx(qo_full + 8 * st, 2 * HTILE + 512);
                const size_t si = ((size_t)b * p.H + h) * attn_tpad(p.T) + (size_t)i * 64;
                bulk_load(base + Lay::LSE + st * 256, p.lse + si, 256, qo_full + 8 * st);
                bulk_load(base + Lay::DD + st * 256, p.D + si, 256, qo_full + 8 * st);
#pragma unroll
                for (int kb = 0; kb < KB; ++kb) {
                    tma_load_2d(sQ + st * HTILE + kb * 8192, &tmQ64, h * HD + kb * 64, row0 + i * 64, qo_full + 8 * st);
                    tma_load_2d(sDO + st * HTILE + kb * 8192, &tmDO64, h * HD + kb * 64, row0 + i * 64,
                                qo_full + 8 * st);
                }
                issued = u + 1;
            }
            if (*abort_flag) {
                drain(kv_full, 0);
                for (int u = (issued > DKV_STG ? issued - DKV_STG : 0); u < issued; ++u)
                    drain(qo_full + 8 * (u % DKV_STG), (u / DKV_STG) & 1);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id_st = idesc_bf16(128, 64, false, false);
            const uint32_t id_kv = idesc_bf16(128, HD, false, true);
            if (mbar_wait(kv_full, 0, abort_flag, p.status)) {
                for (int u = 0; u <= nunits; ++u) {
                    if (u < nunits) {
                        const int st = u % DKV_STG, sb = u & 1;
                        if (!mbar_wait(qo_full + 8 * st, (u / DKV_STG) & 1, abort_flag, p.status)) break;
                        if (!mbar_wait(st_empty + 8 * sb, ((u >> 1) & 1) ^ 1, abort_flag, p.status)) break;
                        tc_fence_after();
#pragma unroll
                        for (int ks = 0; ks < HD / 16; ++ks) {
                            const uint32_t ok_ = (ks >> 2) * 16384 + (ks & 3) * 32;
                            const uint32_t oq = (ks >> 2) * 8192 + (ks & 3) * 32;
                            mma_bf16(tSt + sb * 64, smem_desc(sK + ok_, 16, 1024),
                                     smem_desc(sQ + st * HTILE + oq, 16, 1024), id_st, ks > 0 ? 1u : 0u);
                            mma_bf16(tdPt + sb * 64, smem_desc(sV + ok_, 16, 1024),
                                     smem_desc(sDO + st * HTILE + oq, 16, 1024), id_st, ks > 0 ? 1u : 0u);
                        }
                        mma_commit(st_full + 8 * sb);
                    }
                    if (u > 0) {
                        const int uu = u - 1, st = uu % DKV_STG;
                        if (!mbar_wait(pd_full + 8 * (uu & 1), (uu >> 1) & 1, abort_flag, p.status)) break;
                        tc_fence_after();
#pragma unroll
                        for (int ks = 0; ks < 4; ++ks) {
                            const uint32_t pb = (uu & 1) * 16384 + ks * 32;
                            mma_bf16(tdV, smem_desc(sPT + pb, 16, 1024),
                                     smem_desc(sDO + st * HTILE + ks * 2048, 8192, 1024), id_kv,
                                     (uu > 0 || ks > 0) ? 1u : 0u);
                            mma_bf16(tdK, smem_desc(sDST + pb, 16, 1024),
                                     smem_desc(sQ + st * HTILE + ks * 2048, 8192, 1024), id_kv,
                                     (uu > 0 || ks > 0) ? 1u : 0u);
                        }
                        mma_commit(pd_done + 8 * (uu & 1));
                        mma_commit(qo_empty + 8 * st);
                    }
                }
            }
        }
    } else {
        // warps 2..9: TMEM lane quarter q = warp % 4 (key rows), query half ch of each unit
        const int q = warp & 3, ch = (warp - 2) >> 2;
        const int r = q * 32 + lane;
        const int kpos = kvb * 128 + r;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        bool ok = true;
        for (int u = 0; u < nunits; ++u) {
            const int sb = u & 1, st = u % DKV_STG;
            const int i = nq64 - 1 - u / Hg;
            if (!warp_wait(st_full + 8 * sb, (u >> 1) & 1, abort_flag, p.status)) { ok = false; break; }
            // this unit's Q/dO/lse/D stage has landed (the phase cannot move on
            // before this warp finishes the unit, which frees the stage)
            if (!warp_wait(qo_full + 8 * st, (u / DKV_STG) & 1, abort_flag, p.status)) { ok = false; break; }
            tc_fence_after();
            // this warp's 32 query columns of the unit: lse (to log2 units) and D
            float l2[32], dd[32];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float4 a = reinterpret_cast<const float4*>(lse_s + st * 64 + ch * 32)[k];
                const float4 b = reinterpret_cast<const float4*>(d_s + st * 64 + ch * 32)[k];
                l2[4 * k] = a.x * kLog2e; l2[4 * k + 1] = a.y * kLog2e; l2[4 * k + 2] = a.z * kLog2e;
                l2[4 * k + 3] = a.w * kLog2e;
                dd[4 * k] = b.x; dd[4 * k + 1] = b.y; dd[4 * k + 2] = b.z; dd[4 * k + 3] = b.w;
            }
            // units whose queries all see every key of the block need no mask
            const bool full = i * 64 + ch * 32 >= kvb * 128 + 127 && i * 64 + ch * 32 + 31 < p.T;
            float sv[32], dp[32];
            {
                uint32_t rs[32], rd[32];
                tmem_ld32_issue(tSt + lane_off + sb * 64 + ch * 32, rs);
                tmem_ld32_issue(tdPt + lane_off + sb * 64 + ch * 32, rd);
                tmem_wait_ld();
#pragma unroll
                for (int i = 0; i < 32; ++i) { sv[i] = __uint_as_float(rs[i]); dp[i] = __uint_as_float(rd[i]); }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(st_empty + 8 * sb);
            if (full) {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const float P = ex2(sv[e] * p.scale_log2 - l2[e]);
                    dp[e] = P * (dp[e] - dd[e]);
                    sv[e] = P;
                }
            } else {
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int qpos = i * 64 + ch * 32 + e;
                    const bool valid = qpos >= kpos && qpos < p.T;
                    const float P = valid ? ex2(sv[e] * p.scale_log2 - l2[e]) : 0.f;
                    dp[e] = valid ? P * (dp[e] - dd[e]) : 0.f;
                    sv[e] = P;
                }
            }
            // P^T / dS^T buffer (u & 1) was last read by the dV/dK MMAs of unit u-2
            if (u > 1 && !warp_wait(pd_done + 8 * (u & 1), ((u >> 1) - 1) & 1, abort_flag, p.status)) {
                ok = false;
                break;
            }
            uint8_t* prow = smem + Lay::PT + (u & 1) * 16384 + r * 128;
            uint8_t* drow = smem + Lay::DST + (u & 1) * 16384 + r * 128;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int idx = ch * 4 + k;
                const uint32_t sw = (uint32_t)((idx ^ (r & 7)) << 4);
                const float* a = sv + 8 * k;
                const float* d = dp + 8 * k;
                *reinterpret_cast<uint4*>(prow + sw) = make_uint4(pack_bf16(a[0], a[1]), pack_bf16(a[2], a[3]),
                                                                  pack_bf16(a[4], a[5]), pack_bf16(a[6], a[7]));
                *reinterpret_cast<uint4*>(drow + sw) = make_uint4(pack_bf16(d[0], d[1]), pack_bf16(d[2], d[3]),
                                                                  pack_bf16(d[4], d[5]), pack_bf16(d[6], d[7]));
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(pd_full + 8 * (u & 1));
        }
        if (ok && warp_wait(pd_done + 8 * ((nunits - 1) & 1), ((nunits - 1) >> 1) & 1, abort_flag, p.status)) {
            tc_fence_after();
            const bool live = kpos < p.T;
            if (p.rqk && ch == 1) {
                // dK through the QK-norm backward (the other four warps write dV below)
                const size_t rowi = (size_t)row0 + (live ? kpos : 0);
                const int pos = live ? kpos : 0;
                bf16* outk = p.dqkv + rowi * Nqkv + (p.H + g) * HD;
                store_grad_through_qknorm<HD>(tdK + lane_off, p.scale, p.qkv + rowi * Nqkv + (p.H + g) * HD,
                                              live ? p.rqk[rowi * (p.H + p.nkv) + p.H + g] : 0.f,
                                              p.cos_t + (size_t)pos * (HD / 2), p.sin_t + (size_t)pos * (HD / 2),
                                              outk, live);
            } else {
            // the first four softmax warps write dV, the other four dK
            bf16* out = p.dqkv + ((size_t)row0 + kpos) * Nqkv + (ch == 0 ? (p.H + p.nkv + g) : (p.H + g)) * HD;
            const uint32_t tsrc = ch == 0 ? tdV : tdK;
            const float sc = ch == 0 ? 1.f : p.scale;
#pragma unroll
            for (int c = 0; c < HD / 32; ++c) {
                float v[32];
                tmem_ld32(tsrc + lane_off + c * 32, v);
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
    static bool attr = false;
    if (!attr) {
        if (cudaFuncSetAttribute(attn_fwd_tc_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 FwdLayout<HD>::BYTES) != cudaSuccess)
            return -1;
        attr = true;
    }
    dim3 grid(p.H, p.B, p.nqb);
    attn_fwd_tc_kernel<HD><<<grid, NT, FwdLayout<HD>::BYTES, s>>>(map, p);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

template <int HD>
int dq_launch(const CUtensorMap& kv, const CUtensorMap& kv64, const CUtensorMap& do128, const BwdParams& p,
              cudaStream_t s) {
    static bool attr = false;
    if (!attr) {
        if (cudaFuncSetAttribute(attn_dq_tc_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 DqLayout<HD>::BYTES) != cudaSuccess)
            return -1;
        attr = true;
    }
    attn_dq_tc_kernel<HD><<<dim3(p.H, p.B, p.nqb), NTB, DqLayout<HD>::BYTES, s>>>(kv, kv64, do128, p);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

template <int HD>
int dkv_launch(const CUtensorMap& kv, const CUtensorMap& q64, const CUtensorMap& do64, const BwdParams& p,
               cudaStream_t s) {
    static bool attr = false;
    if (!attr) {
        if (cudaFuncSetAttribute(attn_dkv_tc_kernel<HD>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 DkvLayout<HD>::BYTES) != cudaSuccess)
            return -1;
        attr = true;
    }
    attn_dkv_tc_kernel<HD><<<dim3(p.B, p.nkv, p.nqb), NTB, DkvLayout<HD>::BYTES, s>>>(kv, q64, do64, p);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

BwdParams bwd_params(const float* lse, const float* Dbuf, void* dqkv, int B, int T, int H, int nkv, int hd,
                     int* status) {
    BwdParams p{};
    p.B = B; p.T = T; p.H = H; p.nkv = nkv; p.nqb = (T + 127) / 128;
    p.scale = 1.f / sqrtf((float)hd);
    p.scale_log2 = kLog2e * p.scale;
    p.lse = lse; p.D = Dbuf;
    p.dqkv = reinterpret_cast<bf16*>(dqkv);
    p.status = status;
    return p;
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
                        int B, int T, int H, int nkv, int hd, int* status, cudaStream_t s, const QkNormFuse* fuse) {
    if (!attention_tc_bwd_supported(hd)) return 1;
    if (!aligned16(qkv) || !aligned16(o) || !aligned16(dO) || !aligned16(dqkv) || B > 65535 || H > 65535) return 1;
    const int Nqkv = (H + 2 * nkv) * hd;
    CUtensorMap kv, kv64, do128;
    if (!map_rows(&kv, qkv, Nqkv, (uint64_t)B * T, 128) || !map_rows(&kv64, qkv, Nqkv, (uint64_t)B * T, 64) ||
        !map_rows(&do128, dO, (uint64_t)H * hd, (uint64_t)B * T, 128))
        return 1;
    if (launch_attention_bwd_dot(DT_BF16, o, dO, Dbuf, B, T, H, hd, s) != cudaSuccess) return -1;
    BwdParams p = bwd_params(lse, Dbuf, dqkv, B, T, H, nkv, hd, status);
    if (fuse) {
        p.qkv = reinterpret_cast<const bf16*>(qkv);
        p.rqk = fuse->rqk; p.cos_t = fuse->cos_t; p.sin_t = fuse->sin_t;
    }
    return hd == 128 ? dq_launch<128>(kv, kv64, do128, p, s) : dq_launch<64>(kv, kv64, do128, p, s);
}

int attention_tc_bwd_dkv(const void* qkv, const void* dO, const float* lse, const float* Dbuf, void* dqkv, int B,
                         int T, int H, int nkv, int hd, int* status, cudaStream_t s, const QkNormFuse* fuse) {
    if (!attention_tc_bwd_supported(hd)) return 1;
    if (!aligned16(qkv) || !aligned16(dO) || !aligned16(dqkv) || B > 65535 || nkv > 65535) return 1;
    const int Nqkv = (H + 2 * nkv) * hd;
    CUtensorMap kv, q64, do64;
    if (!map_rows(&kv, qkv, Nqkv, (uint64_t)B * T, 128) || !map_rows(&q64, qkv, Nqkv, (uint64_t)B * T, 64) ||
        !map_rows(&do64, dO, (uint64_t)H * hd, (uint64_t)B * T, 64))
        return 1;
    BwdParams p = bwd_params(lse, Dbuf, dqkv, B, T, H, nkv, hd, status);
    if (fuse) {
        p.qkv = reinterpret_cast<const bf16*>(qkv);
        p.rqk = fuse->rqk; p.cos_t = fuse->cos_t; p.sin_t = fuse->sin_t;
    }
    return hd == 128 ? dkv_launch<128>(kv, q64, do64, p, s) : dkv_launch<64>(kv, q64, do64, p, s);
}

int attention_tc_bwd(const void* qkv, const void* o, const void* dO, const float* lse, float* Dbuf, void* dqkv,
                     int B, int T, int H, int nkv, int hd, void*, size_t, int* status, cudaStream_t s) {
    int r = attention_tc_bwd_dq(qkv, o, dO, lse, Dbuf, dqkv, B, T, H, nkv, hd, status, s, nullptr);
    if (r != 0) return r;
    return attention_tc_bwd_dkv(qkv, dO, lse, Dbuf, dqkv, B, T, H, nkv, hd, status, s, nullptr);
}

size_t attention_tc_workspace_bytes(int, int, int, int, int) { return 0; }

}  // namespace nc
