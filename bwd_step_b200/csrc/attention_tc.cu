// Causal multi-query attention on the tcgen05 tensor cores (bf16 operands,
// fp32 accumulation in TMEM, fp32 softmax).  Model item: multi-query
// attention, every query head reading the one shared K/V head (nanochat
// announcement, vpshk.cn, architecture list), causal within a row, scores
// scaled by 1/sqrt(hd).
//
// Forward, persistent: one CTA per SM walks the units (query block of 128
// positions, pair of query heads of one K/V group, batch row), longest first.
// Both heads of a pair read the same K_j / V_j tiles from shared memory (the
// K/V head is shared), and their work is interleaved so that one head's
// softmax runs while the tensor core computes the other head's products:
//   warp 0     TMA: Q of both heads per unit, then K_j and V_j into two rings
//              for key blocks j = 0..qb (causal: blocks past the diagonal are
//              never loaded), K running one block ahead of V;
//   warp 1     tcgen05.mma in the order ... O_a += P_a(j) V_j, S_a(j+1),
//              O_b += P_b(j) V_j, S_b(j+1) ...: S = Q K^T into the head's
//              128 TMEM score columns, O += P V with P read from TMEM (A
//              operand) over the first half of those columns and V as an
//              MN-major operand;
//   warps 2-5  softmax of head a, warps 6-9 of head b: one query row per
//              thread, all 128 keys of the block from TMEM, causal mask on
//              the diagonal block, running max in the log2 domain, lazy
//              rescaling of O (only when the max grows by more than 2^8),
//              P stored as packed bf16; then the normalised output and the
//              log-sum-exp of the unit.
// 2^x is taken from the special-function unit (ex2), except for one score in
// kPolyEvery of the full blocks, which takes a cubic on the FMA pipe, so that
// the two units share the work of the exponentials.
#include "attention_tc.h"
#include "tc_common.cuh"
#include <cudaTypedefs.h>
#include <algorithm>
#include <type_traits>

namespace nc {
namespace {
using namespace tc;

constexpr int NT = 320;  // forward: producer, MMA, 2 x 4 softmax warps
// One score in kPolyEvery (even, or 0 for none) of the forward's full blocks takes
// 2^x from the FMA pipe (exp2_fma) instead of the special-function unit.
constexpr int kPolyEvery = 8;
constexpr float kLn2 = 0.69314718055994530942f;
constexpr float kLog2e = 1.44269504088896340736f;

struct AttnParams {
    int B, T, H, nkv, nqb;
    int pairs_per_group, npair, num_units;  // head pairs within each K/V group; units = B * npair * nqb
    float scale_log2;                       // log2(e) / sqrt(hd)
    bf16* o;
    float* lse;
    int* status;
};

template <int HD>
struct FwdLayout {
    static constexpr int KB = HD / 64;       // 64-column blocks of the head dim
    static constexpr int TILE = KB * 16384;  // [128 x HD] bf16, 128B-swizzled
    static constexpr int KVSTG = HD == 128 ? 2 : 3;
    static constexpr int QA = 0;             // Q of head a, then Q of head b
    static constexpr int K = 2 * TILE;
    static constexpr int V = K + KVSTG * TILE;
    static constexpr int BAR = V + KVSTG * TILE;
    static constexpr int BYTES = BAR + 256;  // the dynamic shared memory base is 1024-aligned (checked)
    static_assert(BYTES <= 232448, "attention forward shared memory exceeds the per-block limit");
};

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
}

// The three-input maximum.
__device__ __forceinline__ float max3f(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// Store 32 consecutive 32-bit columns of this thread's TMEM lane (no wait).
__device__ __forceinline__ void tmem_st32u_nowait(uint32_t taddr, const uint32_t* v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
        "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
        ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15]),
        "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]), "r"(v[21]), "r"(v[22]), "r"(v[23]),
        "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]), "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])
        : "memory");
}

// Waits (at most 1 ms) for a barrier phase: used on the abort path to let
// copies in flight land before the block exits.
__device__ __forceinline__ void drain(uint32_t bar, uint32_t parity) {
    uint64_t t0 = globaltimer();
    while (!mbar_try(bar, parity) && globaltimer() - t0 < 1000000ull) {}
}

// Store 16 consecutive 32-bit columns of this thread's TMEM lane (no wait).
__device__ __forceinline__ void tmem_st16_nowait(uint32_t taddr, const uint32_t* v) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
        ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), "r"(v[7]),
        "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]), "r"(v[14]), "r"(v[15])
        : "memory");
}

// 2^x on the FMA pipe, for x >= -126 (smaller x give a value below 2^-125):
// x = n + f with n = round(x) and |f| <= 1/2; 2^f by a cubic fitted here to
// 2^f on [-1/2, 1/2] with the Remez exchange on the relative error (maximum
// relative error 7.5e-5, below the bf16 rounding of P); n is added to the
// exponent field.  The rounding uses the 1.5 * 2^23 shift, after which the
// low mantissa bits of t hold n in two's complement.
__device__ __forceinline__ float exp2_fma(float x) {
    x = fmaxf(x, -126.f);
    const float t = x + 12582912.f;
    const float f = x - (t - 12582912.f);
    float p = fmaf(0.0551716685f, f, 0.2426111251f);
    p = fmaf(p, f, 0.6932609677f);
    p = fmaf(p, f, 0.9999280572f);
    return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// Unit u -> batch row, query block (longest first), first head of the pair and
// whether the pair has a second head (a K/V group of odd size ends with a
// single head).
__device__ __forceinline__ void fwd_unit(const AttnParams& p, int u, int& b, int& qb, int& h0, bool& two) {
    const int per = p.B * p.npair;
    qb = p.nqb - 1 - u / per;
    const int rem = u % per;
    b = rem / p.npair;
    const int pi = rem % p.npair;
    const int Hg = p.H / p.nkv;
    const int g = pi / p.pairs_per_group, k = pi % p.pairs_per_group;
    h0 = g * Hg + 2 * k;
    two = 2 * k + 1 < Hg;
}

template <int HD>
__global__ void __launch_bounds__(NT, 1) attn_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm, const AttnParams p) {
    using Lay = FwdLayout<HD>;
    constexpr int KB = Lay::KB, TILE = Lay::TILE, KVSTG = Lay::KVSTG;
    extern __shared__ __align__(1024) uint8_t smem_dyn[];
    if ((smem_u32(smem_dyn) & 1023u) != 0) {
        if (threadIdx.x == 0) set_status(p.status, ST_BAD_LAYOUT);
        return;
    }
    const uint32_t base = smem_u32(smem_dyn);
    const uint32_t sQ = base + Lay::QA, sK = base + Lay::K, sV = base + Lay::V;
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem_dyn + Lay::BAR);
    const uint32_t b0 = smem_u32(bars);
    const uint32_t q_full = b0, q_empty = b0 + 8;
    const uint32_t k_full = b0 + 16, k_empty = k_full + 8 * KVSTG;    // [KVSTG] K ring
    const uint32_t v_full = k_empty + 8 * KVSTG, v_empty = v_full + 8 * KVSTG;  // [KVSTG] V ring
    const uint32_t s_full = v_empty + 8 * KVSTG;                        // [2] per head of the pair
    const uint32_t p_full = s_full + 16;                                // [2]
    const uint32_t o_full = p_full + 16;                                // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 8 + 4 * KVSTG);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        mbar_init(q_full, 1);
        mbar_init(q_empty, 1);
        for (int st = 0; st < KVSTG; ++st) {
            mbar_init(k_full + 8 * st, 1); mbar_init(k_empty + 8 * st, 1);
            mbar_init(v_full + 8 * st, 1); mbar_init(v_empty + 8 * st, 1);
        }
        for (int x = 0; x < 2; ++x) {
            mbar_init(s_full + 8 * x, 1);
            mbar_init(p_full + 8 * x, 4);
            mbar_init(o_full + 8 * x, 1);
        }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), 512);
    if (warp == 0 && lane == 0) tma_prefetch(&tm);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // TMEM: scores (then P) of heads a and b in columns [0,128) and [128,256),
    // their outputs O in [256, 256 + HD) and [256 + HD, 256 + 2 HD)

    if (warp == 0) {
        if (lane == 0) {
            // Q of the pair, then K and V in two rings: K_{j+1} is loaded before V_j,
            // because K_j is free as soon as both heads' scores S(j) have been formed,
            // long before O += P(j) V_j releases V_j
            int k = 0, ki = 0, vi = 0, inflight_q = 0;
            uint32_t q_par = 0, issued = 0, phase_bits = 0;  // bit st: K stage st, bit 8 + st: V stage st
            bool ok = true;
            auto load = [&](bool isv, int i, int xsrc, int row) -> bool {
                const int st = i % KVSTG;
                const uint32_t ph = (i / KVSTG) & 1;
                const uint32_t full = (isv ? v_full : k_full) + 8 * st, empty = (isv ? v_empty : k_empty) + 8 * st;
                if (!mbar_wait(empty, ph ^ 1, abort_flag, p.status)) return false;
                mbar_expect_tx(full, TILE);
                const uint32_t dst = (isv ? sV : sK) + st * TILE;
#pragma unroll
                for (int c = 0; c < KB; ++c) tma_load_2d(dst + c * 16384, &tm, xsrc + 64 * c, row, full);
                const int bit = (isv ? 8 : 0) + st;
                issued |= 1u << bit;
                phase_bits = (phase_bits & ~(1u << bit)) | (ph << bit);
                return true;
            };
            for (int u = blockIdx.x; ok && u < p.num_units; u += gridDim.x, ++k) {
                int b, qb, h0;
                bool two;
                fwd_unit(p, u, b, qb, h0, two);
                const int g = h0 / (p.H / p.nkv);
                const int xk = (p.H + g) * HD, xv = (p.H + p.nkv + g) * HD;
                const int row0 = b * p.T;
                if (!mbar_wait(q_empty, (k & 1) ^ 1, abort_flag, p.status)) { ok = false; break; }
                mbar_expect_tx(q_full, two ? 2 * TILE : TILE);
#pragma unroll
                for (int c = 0; c < KB; ++c) {
                    tma_load_2d(sQ + c * 16384, &tm, h0 * HD + 64 * c, row0 + qb * 128, q_full);
                    if (two) tma_load_2d(sQ + TILE + c * 16384, &tm, (h0 + 1) * HD + 64 * c, row0 + qb * 128, q_full);
                }
                inflight_q = 1;
                q_par = k & 1;
                if (!load(false, ki++, xk, row0)) { ok = false; break; }
                for (int j = 0; j <= qb; ++j) {
                    if (j < qb && !load(false, ki++, xk, row0 + (j + 1) * 128)) { ok = false; break; }
                    if (!load(true, vi++, xv, row0 + j * 128)) { ok = false; break; }
                }
            }
            if (!ok) {
                // let the copies in flight land before the block exits
                if (inflight_q) drain(q_full, q_par);
                for (int st = 0; st < KVSTG; ++st) {
                    if (issued >> st & 1) drain(k_full + 8 * st, (phase_bits >> st) & 1);
                    if (issued >> (8 + st) & 1) drain(v_full + 8 * st, (phase_bits >> (8 + st)) & 1);
                }
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t id_s = idesc_bf16(128, 128, false, false);
            const uint32_t id_o = idesc_bf16(128, HD, false, true);
            int k = 0, ki = 0, vi = 0;
            uint32_t pcnt0 = 0, pcnt1 = 0;  // P hand-overs waited for, per head
            bool ok = true;
            auto ready = [&](bool isv, int i) -> bool {
                return mbar_wait((isv ? v_full : k_full) + 8 * (i % KVSTG), (i / KVSTG) & 1, abort_flag, p.status);
            };
            // S_x = Q_x K^T for head x of the pair, from K stage st
            auto scores = [&](int x, int st) {
#pragma unroll
                for (int ks = 0; ks < HD / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                    mma_bf16(tmem + 128 * x, smem_desc(sQ + x * TILE + off, 16, 1024),
                             smem_desc(sK + st * TILE + off, 16, 1024), id_s, ks > 0 ? 1u : 0u);
                }
                mma_commit(s_full + 8 * x);
            };
            // both heads' scores of the next K tile, then K's stage is released
            auto scores_both = [&](bool two) -> bool {
                if (!ready(false, ki)) return false;
                tc_fence_after();
                const int st = ki % KVSTG;
                scores(0, st);
                if (two) scores(1, st);
                mma_commit(k_empty + 8 * st);
                ++ki;
                return true;
            };
            // O_x += P_x V: keys 16kk..16kk+15 sit in the packed columns 8kk..8kk+7
            auto pv = [&](int x, int st, bool acc) -> bool {
                if (!mbar_wait(p_full + 8 * x, (x ? pcnt1 : pcnt0) & 1, abort_flag, p.status)) return false;
                if (x) ++pcnt1;
                else ++pcnt0;
                tc_fence_after();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16_ts(tmem + 256 + x * HD, tmem + 128 * x + 8 * kk,
                                smem_desc(sV + st * TILE + kk * 2048, 16384, 1024), id_o, (acc || kk > 0) ? 1u : 0u);
                return true;
            };
            for (int u = blockIdx.x; ok && u < p.num_units; u += gridDim.x, ++k) {
                int b, qb, h0;
                bool two;
                fwd_unit(p, u, b, qb, h0, two);
                const int nblk = qb + 1;
                if (!mbar_wait(q_full, k & 1, abort_flag, p.status) || !scores_both(two)) { ok = false; break; }
                if (nblk == 1) mma_commit(q_empty);  // the unit's last products that read Q
                for (int j = 0; j < nblk; ++j) {
                    const bool more = j + 1 < nblk;
                    const int vst = vi % KVSTG;
                    if (!ready(true, vi)) { ok = false; break; }
                    // head a: O += P(j) V_j, then S(j+1) (which overwrites P(j) after it, in issue order)
                    if (!pv(0, vst, j > 0)) { ok = false; break; }
                    if (more) {
                        if (!ready(false, ki)) { ok = false; break; }
                        tc_fence_after();
                        scores(0, ki % KVSTG);
                    } else {
                        mma_commit(o_full);
                    }
                    // head b likewise; V_j and (after both heads' scores) K_{j+1} are then released
                    if (two && !pv(1, vst, j > 0)) { ok = false; break; }
                    mma_commit(v_empty + 8 * vst);
                    ++vi;
                    if (more) {
                        if (two) scores(1, ki % KVSTG);
                        mma_commit(k_empty + 8 * (ki % KVSTG));
                        ++ki;
                    } else if (two) {
                        mma_commit(o_full + 8);
                    }
                    if (j + 2 == nblk) mma_commit(q_empty);
                }
            }
        }
    } else {
        // ---------------- softmax: head x of the pair, TMEM lane quarter q, one query row per thread
        const int x = (warp - 2) >> 2, q = warp & 3;
        const int r = q * 32 + lane;
        const uint32_t lane_off = (uint32_t)(q * 32) << 16;
        const uint32_t tS = tmem + lane_off + 128 * x, tO = tmem + lane_off + 256 + x * HD;
        uint32_t scnt = 0, ocnt = 0;
        for (int u = blockIdx.x; u < p.num_units; u += gridDim.x) {
            int b, qb, h0;
            bool two;
            fwd_unit(p, u, b, qb, h0, two);
            if (x == 1 && !two) continue;
            const int h = h0 + x;
            float m = -INFINITY, l = 0.f;
            bool ok = true;
            for (int j = 0; j <= qb; ++j) {
                if (!warp_wait(s_full + 8 * x, scnt & 1, abort_flag, p.status)) { ok = false; break; }
                ++scnt;
                tc_fence_after();
                const bool diag = j == qb;  // key c of the diagonal block is visible from row r iff c <= r
                // the whole score row in registers: four loads in flight, one wait
                uint32_t sr[128];
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) tmem_ld32_issue(tS + 32 * q4, sr + 32 * q4);
                tmem_wait_ld();
                // the row maximum as four independent partial maxima (no 128-long
                // dependency chain)
                float mx4[4];
#pragma unroll
                for (int k = 0; k < 4; ++k) mx4[k] = -INFINITY;
                if (diag) {
#pragma unroll
                    for (int c = 0; c < 128; c += 2)
                        mx4[(c >> 1) & 3] = max3f(mx4[(c >> 1) & 3], c > r ? -INFINITY : __uint_as_float(sr[c]),
                                                  c + 1 > r ? -INFINITY : __uint_as_float(sr[c + 1]));
                } else {
#pragma unroll
                    for (int c = 0; c < 128; c += 2)
                        mx4[(c >> 1) & 3] = max3f(mx4[(c >> 1) & 3], __uint_as_float(sr[c]), __uint_as_float(sr[c + 1]));
                }
                float mx = fmaxf(fmaxf(mx4[0], mx4[1]), fmaxf(mx4[2], mx4[3]));
                mx *= p.scale_log2;
                const bool rescale = mx > m + 8.f;
                const float mu = rescale ? mx : m;
                const float alpha = rescale ? ex2(m - mx) : 1.f;
                // P = 2^(s*scale - mu) as packed bf16 over the first 64 score columns (the
                // scaling as packed f32x2 FMAs), the row sum as two partial sums of pairs;
                // with kPoly one score in kPolyEvery comes from the FMA pipe (full blocks
                // only: exp2_fma does not take the masked -inf scores of the diagonal block)
                const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2), nmu2 = f2_pack(-mu, -mu);
                uint64_t sum2[2] = {f2_pack(0.f, 0.f), f2_pack(0.f, 0.f)};
                auto exp_pack = [&](auto poly) {
                    constexpr bool kPoly = decltype(poly)::value;
                    constexpr int kPE = kPolyEvery > 0 ? kPolyEvery : 2;
#pragma unroll
                    for (int q8 = 0; q8 < 8; ++q8) {
                        uint32_t pk[8];
#pragma unroll
                        for (int c = 0; c < 16; c += 2) {
                            const int cc = 16 * q8 + c;
                            float x0, x1;
                            f2_unpack(f2_fma(f2_pack(__uint_as_float(sr[cc]), __uint_as_float(sr[cc + 1])), sc2, nmu2),
                                      x0, x1);
                            if (!kPoly && diag) {
                                if (cc > r) x0 = -INFINITY;
                                if (cc + 1 > r) x1 = -INFINITY;
                            }
                            const float e0 = ex2(x0);
                            const float e1 = (kPoly && (c / 2) % (kPE / 2) == kPE / 2 - 1) ? exp2_fma(x1) : ex2(x1);
                            sum2[(c >> 1) & 1] = f2_add(sum2[(c >> 1) & 1], f2_pack(e0, e1));
                            pk[c >> 1] = pack_bf16(e0, e1);
                        }
                        tmem_st8_nowait(tS + 8 * q8, pk);
                    }
                };
                if (!diag && kPolyEvery > 0) exp_pack(std::true_type{});
                else exp_pack(std::false_type{});
                tmem_wait_st();
                float s00, s01, s10, s11;
                f2_unpack(sum2[0], s00, s01);
                f2_unpack(sum2[1], s10, s11);
                const float sum = (s00 + s01) + (s10 + s11);
                if (j > 0 && __any_sync(0xffffffffu, rescale)) {
                    // O_x += P(j-1) V has completed (S(j) was issued after it and has landed);
                    // O_x += P(j) V waits for this warp's hand-over below
#pragma unroll 1
                    for (int c = 0; c < HD / 32; ++c) {
                        uint32_t o[32];
                        tmem_ld32_issue(tO + c * 32, o);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                        tmem_st32u_nowait(tO + c * 32, o);
                        tmem_wait_st();
                    }
                }
                l = l * alpha + sum;
                m = mu;
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(p_full + 8 * x);
            }
            if (!ok || !warp_wait(o_full + 8 * x, ocnt & 1, abort_flag, p.status)) break;
            ++ocnt;
            tc_fence_after();
            const int qpos = qb * 128 + r;
            const bool live = qpos < p.T;
            const float inv = 1.f / l;
            bf16* orow = p.o + ((size_t)b * p.T + (live ? qpos : 0)) * (size_t)(p.H * HD) + (size_t)h * HD;
#pragma unroll 1
            for (int c = 0; c < HD / 32; ++c) {
                float o[32];
                tmem_ld32(tO + c * 32, o);
                if (live) {
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        *reinterpret_cast<uint4*>(orow + c * 32 + 8 * i) =
                            make_uint4(pack_bf16(o[8 * i] * inv, o[8 * i + 1] * inv),
                                       pack_bf16(o[8 * i + 2] * inv, o[8 * i + 3] * inv),
                                       pack_bf16(o[8 * i + 4] * inv, o[8 * i + 5] * inv),
                                       pack_bf16(o[8 * i + 6] * inv, o[8 * i + 7] * inv));
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
// Three launches: (1) -D = -rowsum(dO * o) and -lse * log2(e) per (row, head)
// (or the same statistics from the epilogue of the GEMM that forms dO);
// (2) the dK/dV kernel, which recomputes S^T and dP^T per (key block, query
// block, query head), forms P^T and dS^T, accumulates dV and dK, and stores
// every dS^T tile; (3) dq = dS K / sqrt(hd) as a plain tensor-core product
// over the stored tiles.  S and dP are formed once (in (2)), so the backward
// issues the minimal five 128-wide products per tile pair (S^T, dP^T, dV,
// dK, dQ), deterministically: every sum runs in a fixed order, no atomics.
//
// The dK/dV kernel keeps every MMA at N = 128 (a 128 x 64 tile runs the
// tensor core at well under half rate on sm_100a) and feeds one operand of the
// second product from TMEM: the softmax warps write P^T as bf16 back over
// dP^T columns they have just read, and the dV MMA reads it there as the A
// operand.  Sixteen softmax warps (four per TMEM lane quarter, 32 columns
// each) keep the special-function unit busy.
constexpr int NTB = 608;  // dK/dV: producer, MMA, 16 softmax warps, dS store
constexpr int NSM = 16;   // softmax warps

struct BwdParams {
    int B, T, H, nkv, nqb, ntri;
    float scale_log2, scale;
    const float* D;     // [B, H, Tp] -rowsum(dO * o)
    const float* lse2;  // [B, H, Tp] -lse * log2(e) (both zero past the sequence end; negated so the
                        // softmax warps add them with packed f32x2 FMAs)
    bf16* dqkv;
    bf16* ds;           // dS^T tiles (see ds_tile), written by the dK/dV kernel
    int* status;
};

// The dK/dV kernel stores every causal 128 x 128 tile of dS = P (dP - D) it
// forms, transposed ([128 keys][128 queries] bf16, row-major), for the dQ
// product.  Tiles of one (batch row, query head) are packed by query block,
// then key block: tile (qb, kb), kb <= qb, is number qb (qb + 1) / 2 + kb of
// its head, so the key blocks of one query block are adjacent.
__host__ __device__ inline size_t ds_tile(int b, int h, int H, int ntri, int qb, int kb) {
    return ((size_t)b * H + h) * (size_t)ntri + (size_t)qb * (qb + 1) / 2 + kb;
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
        D[w] = -s;
        lse2[w] = live ? -lse[w] * kLog2e : 0.f;
    }
}

// dq = dS K / sqrt(hd) from the stored dS^T tiles.  Persistent: one CTA per
// SM walks the units (query block, head, batch row), longest first.
//   warp 0      TMA: per key block kb <= qb, the dS^T tile (two boxes of
//               [128 keys][64 queries]) and the K_kb tile into a ring;
//   warp 1      tcgen05.mma: D[q, c] += sum_k dS^T[k, q] K[k, c] with both
//               operands MN-major in shared memory, into one of two TMEM
//               accumulators, so the epilogue of one unit overlaps the next;
//   warps 2-5   epilogue: one query row per thread, scaled, bf16, into the
//               q columns of dqkv.
template <int HD>
struct DqdsLayout {
    static constexpr int KB = HD / 64;
    static constexpr int A_BYTES = 32768;       // dS^T tile, bf16, two 64-query boxes
    static constexpr int B_BYTES = KB * 16384;  // K tile [128 keys x HD] bf16
    static constexpr int STAGE = A_BYTES + B_BYTES;
    static constexpr int STAGES = HD == 128 ? 3 : 4;
    static constexpr int BAR = STAGES * STAGE;
    static constexpr int BYTES = BAR + 256;  // the dynamic shared memory base is 1024-aligned (checked)
    static_assert(BYTES <= 232448, "dQ shared memory exceeds the per-block limit");
};
constexpr int NTQ = 192;  // dQ product: producer, MMA, four epilogue warps

struct DqdsParams {
    int B, T, H, nkv, nqb, ntri, num_units;
    float scale;
    bf16* dqkv;
    int* status;
};

__device__ __forceinline__ void dq_unit(const DqdsParams& p, int u, int& b, int& h, int& qb) {
    const int bh = u % (p.B * p.H);
    qb = p.nqb - 1 - u / (p.B * p.H);  // the longest units first
    b = bh / p.H;
    h = bh % p.H;
}

template <int HD>
__global__ void __launch_bounds__(NTQ, 1) attn_dq_ds_kernel(const __grid_constant__ CUtensorMap tmDS,
                                                           const __grid_constant__ CUtensorMap tmQKV,
                                                           const DqdsParams p) {
    using Lay = DqdsLayout<HD>;
    constexpr int KB = Lay::KB, STAGES = Lay::STAGES;
    extern __shared__ __align__(1024) uint8_t smem_dyn[];
    if ((smem_u32(smem_dyn) & 1023u) != 0) {
        if (threadIdx.x == 0) set_status(p.status, ST_BAD_LAYOUT);
        return;
    }
    const uint32_t base = smem_u32(smem_dyn);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem_dyn + Lay::BAR);
    const uint32_t b0 = smem_u32(bars);
    const uint32_t full = b0, empty = b0 + 8 * STAGES;              // [STAGES]
    const uint32_t acc_full = b0 + 16 * STAGES, acc_empty = acc_full + 16;  // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 4);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr uint32_t kCols = 2 * HD;  // two accumulators (128 or 256 columns)

    if (threadIdx.x == 0) {
        for (int st = 0; st < STAGES; ++st) { mbar_init(full + 8 * st, 1); mbar_init(empty + 8 * st, 1); }
        for (int a = 0; a < 2; ++a) { mbar_init(acc_full + 8 * a, 1); mbar_init(acc_empty + 8 * a, 4); }
        *abort_flag = 0;
        fence_barrier_init();
    }
    if (warp == 1) tmem_alloc(smem_u32(tmem_slot), kCols);
    if (warp == 0 && lane == 0) { tma_prefetch(&tmDS); tma_prefetch(&tmQKV); }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            int stage = 0;
            uint32_t phase = 0, issued = 0, issued_phase = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < p.num_units; u += gridDim.x) {
                int b, h, qb;
                dq_unit(p, u, b, h, qb);
                const int g = h / (p.H / p.nkv);
                const int xk = (p.H + g) * HD;
                const int trow = (int)(ds_tile(b, h, p.H, p.ntri, qb, 0) * 128);
                for (int kb = 0; kb <= qb; ++kb) {
                    if (!mbar_wait(empty + 8 * stage, phase ^ 1, abort_flag, p.status)) { ok = false; break; }
                    const uint32_t fb = full + 8 * stage;
                    const uint32_t sa = base + stage * Lay::STAGE, sb = sa + Lay::A_BYTES;
                    mbar_expect_tx(fb, Lay::STAGE);
                    tma_load_2d(sa, &tmDS, 0, trow + kb * 128, fb);
                    tma_load_2d(sa + 16384, &tmDS, 64, trow + kb * 128, fb);
#pragma unroll
                    for (int c = 0; c < KB; ++c) tma_load_2d(sb + c * 16384, &tmQKV, xk + 64 * c, b * p.T + kb * 128, fb);
                    issued |= 1u << stage;
                    issued_phase = (issued_phase & ~(1u << stage)) | (phase << stage);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
            }
            if (!ok) {
                for (int st = 0; st < STAGES; ++st)
                    if (issued >> st & 1) drain(full + 8 * st, (issued_phase >> st) & 1);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idesc = idesc_bf16(128, HD, true, true);
            int stage = 0, acc = 0;
            uint32_t phase = 0, acc_phase = 0;
            bool ok = true;
            for (int u = blockIdx.x; ok && u < p.num_units; u += gridDim.x) {
                int b, h, qb;
                dq_unit(p, u, b, h, qb);
                if (!mbar_wait(acc_empty + 8 * acc, acc_phase ^ 1, abort_flag, p.status)) break;
                tc_fence_after();
                const uint32_t d = tmem + acc * HD;
                for (int kb = 0; kb <= qb; ++kb) {
                    if (!mbar_wait(full + 8 * stage, phase, abort_flag, p.status)) { ok = false; break; }
                    tc_fence_after();
                    const uint32_t sa = base + stage * Lay::STAGE, sb = sa + Lay::A_BYTES;
#pragma unroll
                    for (int ks = 0; ks < 8; ++ks)
                        mma_bf16(d, smem_desc(sa + ks * 2048, 16384, 1024), smem_desc(sb + ks * 2048, 16384, 1024),
                                 idesc, (kb > 0 || ks > 0) ? 1u : 0u);
                    mma_commit(empty + 8 * stage);
                    if (++stage == STAGES) { stage = 0; phase ^= 1; }
                }
                if (!ok) break;
                mma_commit(acc_full + 8 * acc);
                if (++acc == 2) { acc = 0; acc_phase ^= 1; }
            }
        }
    } else {
        // epilogue warps 2..5: warp w reads TMEM lanes 32*(w%4).. (query rows)
        const int q = warp & 3;
        const int Nqkv = (p.H + 2 * p.nkv) * HD;
        int acc = 0;
        uint32_t acc_phase = 0;
        for (int u = blockIdx.x; u < p.num_units; u += gridDim.x) {
            int b, h, qb;
            dq_unit(p, u, b, h, qb);
            if (!warp_wait(acc_full + 8 * acc, acc_phase, abort_flag, p.status)) break;
            tc_fence_after();
            const int qpos = qb * 128 + q * 32 + lane;
            const bool live = qpos < p.T;
            const size_t rowi = (size_t)b * p.T + (live ? qpos : 0);
            bf16* out = p.dqkv + rowi * Nqkv + (size_t)h * HD;
            const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16) + acc * HD;
#pragma unroll 1
            for (int c = 0; c < HD / 32; ++c) {
                float v[32];
                tmem_ld32(tb + c * 32, v);
                if (live) {
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        *reinterpret_cast<uint4*>(out + c * 32 + 8 * e) =
                            make_uint4(pack_bf16(v[8 * e] * p.scale, v[8 * e + 1] * p.scale),
                                       pack_bf16(v[8 * e + 2] * p.scale, v[8 * e + 3] * p.scale),
                                       pack_bf16(v[8 * e + 4] * p.scale, v[8 * e + 5] * p.scale),
                                       pack_bf16(v[8 * e + 6] * p.scale, v[8 * e + 7] * p.scale));
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acc_empty + 8 * acc);
            if (++acc == 2) { acc = 0; acc_phase ^= 1; }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, kCols);
    }
}

// dK / dV, one CTA per (key block of 128, K/V head, batch row).  Units are
// (query block i of 128, query head h of the group), the last query block
// first, so the CTAs of all key blocks of a batch row read the same Q / dO
// tiles at about the same time and find them in L2:
//   warp 0      TMA: K and V once; Q_i, dO_i with their lse2 / D rows into a
//               2-stage ring;
//   warp 1      tcgen05.mma: S^T = K Q_i^T and dP^T = V dO_i^T into TMEM,
//               dV += P^T dO_i with P^T read from TMEM (the A operand, written
//               over the dP^T columns) and dK += dS^T Q_i with dS^T from one
//               shared-memory tile X (Q_i, dO_i as MN-major operands).  Each
//               product is issued as soon as its inputs are ready (the thread
//               polls its barriers): the next unit's S^T once the softmax warps
//               have read this unit's, its dP^T after this unit's dV (which
//               reads P^T from those columns), dK once dS^T is in X;
//   warps 2-17  per unit: load the warp's S^T columns (32 queries), form
//               P^T = 2^(S^T*scale*log2e - lse2) with the causal mask, load the
//               dP^T columns and write P^T (bf16) over them, form
//               dS^T = P^T (dP^T - D) and write it to X once the previous unit's
//               dK and dS^T store have read X;
//   warp 18     TMA-stores each finished dS^T tile to global memory (for the dQ
//               product) and reports when X may be reused.
// dk = dK / sqrt(hd).
template <int HD>
struct DkvLayout {
    static constexpr int KB = HD / 64;
    static constexpr int TILE = KB * 16384;    // [128 x HD] bf16
    static constexpr int K = 0;
    static constexpr int V = K + TILE;
    static constexpr int Q = V + TILE;         // [2] stages
    static constexpr int DO = Q + 2 * TILE;    // [2] stages
    static constexpr int X = DO + 2 * TILE;    // dS^T [128 keys x 128 queries] bf16, two 64-query boxes
    static constexpr int LSE = X + 32768;      // [2][128] fp32 lse2 of the stage's queries
    static constexpr int DD = LSE + 1024;      // [2][128] fp32 D
    static constexpr int BAR = DD + 1024;
    static constexpr int BYTES = BAR + 256;  // the dynamic shared memory base is 1024-aligned (checked)
    static_assert(BYTES <= 232448, "dK/dV shared memory exceeds the per-block limit");
};

template <int HD>
__global__ void __launch_bounds__(NTB, 1) attn_dkv_tc_kernel(const __grid_constant__ CUtensorMap tmQKV,
                                                            const __grid_constant__ CUtensorMap tmDO,
                                                            const __grid_constant__ CUtensorMap tmDS,
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
    const uint32_t sX = base + Lay::X;
    const float* lse_s = reinterpret_cast<const float*>(smem + Lay::LSE);
    const float* d_s = reinterpret_cast<const float*>(smem + Lay::DD);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + Lay::BAR);
    const uint32_t b0 = smem_u32(bars);
    const uint32_t kv_full = b0, qo_full = b0 + 8, qo_empty = b0 + 24;  // qo_*[2]
    const uint32_t s_full = b0 + 40, dp_full = b0 + 48;    // S^T / dP^T of the unit in TMEM
    const uint32_t s_free = b0 + 56;                       // S^T read by the softmax warps
    const uint32_t p_full = b0 + 72;                       // P^T written over the dP^T columns
    const uint32_t ds_full = b0 + 88, dk_done = b0 + 96;   // dS^T in X / read by the dK MMAs
    const uint32_t dst_read = b0 + 104;                    // dS^T read out of X by its store
    const uint32_t dkv_done = b0 + 112;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 16);
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
        mbar_init(s_full, 1);
        mbar_init(dp_full, 1);
        mbar_init(s_free, NSM);
        mbar_init(p_full, NSM);
        mbar_init(ds_full, NSM);
        mbar_init(dk_done, 1);
        mbar_init(dst_read, 1);
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
            auto scores = [&](int u) {
                const int st = u & 1;
#pragma unroll
                for (int ks = 0; ks < HD / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                    mma_bf16(tSt, smem_desc(sK + off, 16, 1024), smem_desc(sQ + st * TILE + off, 16, 1024), id_s,
                             ks > 0 ? 1u : 0u);
                }
                mma_commit(s_full);
            };
            // dP^T_u = V dO_u^T
            auto dpt = [&](int u) {
                const int st = u & 1;
#pragma unroll
                for (int ks = 0; ks < HD / 16; ++ks) {
                    const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
                    mma_bf16(tdPt, smem_desc(sV + off, 16, 1024), smem_desc(sDO + st * TILE + off, 16, 1024), id_s,
                             ks > 0 ? 1u : 0u);
                }
                mma_commit(dp_full);
            };
            // acc (+)= X Bop^T over the 128 queries of the unit: X = P^T or dS^T [keys x queries]
            // (K-major, two 64-query boxes), Bop = dO_u or Q_u as an MN-major operand
            // dV += P^T dO_u with P^T as the TMEM A operand: queries 16kk..16kk+15 sit in the
            // packed columns 32*(kk/2) + 8*(kk%2) of dP^T (written by column group kk/2)
            auto pv_product = [&](int u) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16_ts(tdV, tdPt + 32 * (kk >> 1) + 8 * (kk & 1),
                                smem_desc(sDO + (u & 1) * TILE + kk * 2048, 16384, 1024), id_kv,
                                (u > 0 || kk > 0) ? 1u : 0u);
            };
            auto x_product = [&](uint32_t acc, uint32_t bop, int u) {
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16(acc, smem_desc(sX + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                             smem_desc(bop + kk * 2048, 16384, 1024), id_kv, (u > 0 || kk > 0) ? 1u : 0u);
            };
            // The four products are issued as their inputs become ready (polled, so a
            // Q / dO load still in flight for the next unit does not hold back this
            // unit's dV and dK): dV_u once P^T_u is in X, dK_u once dS^T_u is, S^T_{u+1}
            // once the softmax warps have read S^T_u and Q_{u+1} has landed, dP^T_{u+1}
            // once they have read dP^T_u.  Each barrier is polled for its next phase
            // only, which it cannot pass before the product waiting on it is issued.
            bool ok = mbar_wait(kv_full, 0, abort_flag, p.status) && mbar_wait(qo_full, 0, abort_flag, p.status);
            if (ok) {
                tc_fence_after();
                scores(0);
                dpt(0);
            }
            int nv = 0, nk = 0, ns = 1, np = 1;  // next dV, dK, S^T, dP^T unit
            uint64_t t0 = globaltimer();
            uint32_t idle = 0;
            while (ok && nk < nunits) {
                bool prog = false;
                if (nv < np && mbar_test(p_full, nv & 1)) {  // P^T_nv written over dP^T
                    tc_fence_after();
                    pv_product(nv);
                    ++nv;
                    prog = true;
                }
                if (nk < nv && mbar_test(ds_full, nk & 1)) {
                    tc_fence_after();
                    x_product(tdK, sQ + (nk & 1) * TILE, nk);
                    mma_commit(dk_done);
                    mma_commit(qo_empty + 8 * (nk & 1));
                    ++nk;
                    prog = true;
                }
                if (ns < nunits && mbar_test(s_free, (ns - 1) & 1) && mbar_test(qo_full + 8 * (ns & 1), (ns >> 1) & 1)) {
                    tc_fence_after();
                    scores(ns);
                    ++ns;
                    prog = true;
                }
                if (np < ns && np == nv) {  // after dV_{np-1}, which reads P^T from these columns
                    dpt(np);
                    ++np;
                    prog = true;
                }
                if (prog) {
                    t0 = globaltimer();
                    idle = 0;
                } else if ((++idle & 63) == 0) {
                    if (*abort_flag) {
                        ok = false;
                    } else if (globaltimer() - t0 > kWaitLimitNs) {
                        set_status(p.status, ST_TIMEOUT);
                        *abort_flag = 1;
                        ok = false;
                    }
                }
            }
            mma_commit(dkv_done);
        }
    } else if (warp == 2 + NSM) {
        // one thread writes every finished dS^T tile to global memory (two TMA stores
        // of [128 keys][64 queries]) and reports when shared memory may be reused
        if (lane == 0) {
            for (int u = 0; u < nunits; ++u) {
                const int i = p.nqb - 1 - u / Hg, h = g * Hg + u % Hg;
                if (!mbar_wait(ds_full, u & 1, abort_flag, p.status)) break;
                const int trow = (int)(ds_tile(b, h, p.H, p.ntri, i, kvb) * 128);
                tma_store_2d(&tmDS, 0, trow, sX);
                tma_store_2d(&tmDS, 64, trow, sX + 16384);
                bulk_commit();
                bulk_wait_read_0();
                mbar_arrive(dst_read);
            }
            bulk_wait_all();  // the tiles are in global memory before the block exits
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
            if (!warp_wait(s_full, u & 1, abort_flag, p.status) ||
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
            if (lane == 0) mbar_arrive(s_free);
            // query q0 + e sees this key when lo <= e (causal) and e <= hi (inside the row)
            const int q0 = i * 128 + cg * 32;
            const int lo = kpos - q0, hi = p.T - 1 - q0;
            const float4* l4 = reinterpret_cast<const float4*>(lse_s + st * 128 + cg * 32);
            float pv[32];
            if (__all_sync(0xffffffffu, lo <= 0 && hi >= 31)) {
                // one exponential in four on the FMA pipe (exp2_fma), the others on the
                // special-function unit
                const uint64_t sc2 = f2_pack(p.scale_log2, p.scale_log2);
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const float4 l = l4[k];  // -lse2
                    float x0, x1, x2, x3;
                    f2_unpack(f2_fma(f2_pack(__uint_as_float(rs[4 * k]), __uint_as_float(rs[4 * k + 1])), sc2,
                                     f2_pack(l.x, l.y)), x0, x1);
                    f2_unpack(f2_fma(f2_pack(__uint_as_float(rs[4 * k + 2]), __uint_as_float(rs[4 * k + 3])), sc2,
                                     f2_pack(l.z, l.w)), x2, x3);
                    pv[4 * k] = ex2(x0);
                    pv[4 * k + 1] = ex2(x1);
                    pv[4 * k + 2] = ex2(x2);
                    pv[4 * k + 3] = exp2_fma(x3);
                }
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k) {
                    const float4 l = l4[k];
                    const float lv[4] = {l.x, l.y, l.z, l.w};
#pragma unroll
                    for (int t = 0; t < 4; ++t) {
                        const int e = 4 * k + t;
                        pv[e] = (e >= lo && e <= hi) ? ex2(fmaf(__uint_as_float(rs[e]), p.scale_log2, lv[t])) : 0.f;
                    }
                }
            }
            // this warp's 32 queries of row r in the swizzled [128 keys x 64 queries] boxes of X
            uint8_t* xrow = smem + Lay::X + (cg >> 1) * 16384 + r * 128;
            // P^T rounded to bf16 (the values dV uses; dS^T is formed from them as well)
            uint32_t pk[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) pk[e] = pack_bf16(pv[2 * e], pv[2 * e + 1]);
            if (!warp_wait(dp_full, u & 1, abort_flag, p.status)) {
                ok = false;
                break;
            }
            tc_fence_after();
            uint32_t rd[32];
            tmem_ld32_issue(tdPt + lane_off + cg * 32, rd);
            tmem_wait_ld();
            // P^T over the first 16 of the warp's own (just read) dP^T columns
            tmem_st16_nowait(tdPt + lane_off + cg * 32, pk);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(p_full);
            // dS^T = P^T (dP^T - D) (d_s holds -D); masked entries have P = 0 and D, dP finite
            const float4* d4 = reinterpret_cast<const float4*>(d_s + st * 128 + cg * 32);
            uint32_t dk[16];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const float4 dd = d4[k];
                const float2 p01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pk[2 * k]));
                const float2 p23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pk[2 * k + 1]));
                float d0, d1, d2, d3;
                f2_unpack(f2_mul(f2_pack(p01.x, p01.y),
                                 f2_add(f2_pack(__uint_as_float(rd[4 * k]), __uint_as_float(rd[4 * k + 1])),
                                        f2_pack(dd.x, dd.y))),
                          d0, d1);
                f2_unpack(f2_mul(f2_pack(p23.x, p23.y),
                                 f2_add(f2_pack(__uint_as_float(rd[4 * k + 2]), __uint_as_float(rd[4 * k + 3])),
                                        f2_pack(dd.z, dd.w))),
                          d2, d3);
                dk[2 * k] = pack_bf16(d0, d1);
                dk[2 * k + 1] = pack_bf16(d2, d3);
            }
            // X is free once the dK MMAs of the previous unit and the store of its dS^T tile
            // to global memory (for the dQ product) have read it
            if (u > 0 && (!warp_wait(dk_done, (u - 1) & 1, abort_flag, p.status) ||
                          !warp_wait(dst_read, (u - 1) & 1, abort_flag, p.status))) {
                ok = false;
                break;
            }
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int c8 = (cg & 1) * 4 + k;
                *reinterpret_cast<uint4*>(xrow + ((c8 ^ (r & 7)) << 4)) =
                    make_uint4(dk[4 * k], dk[4 * k + 1], dk[4 * k + 2], dk[4 * k + 3]);
            }
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(ds_full);
        }
        if (ok && warp_wait(dkv_done, 0, abort_flag, p.status)) {
            tc_fence_after();
            const bool live = kpos < p.T;
            const size_t rowi = (size_t)row0 + (live ? kpos : 0);
            // column groups 0 and 1 write the two halves of dv, 2 and 3 those of dk
            const bool isk = cg >= 2;
            const int c0 = (cg & 1) * (HD / 2);
            const uint32_t tsrc = (isk ? tdK : tdV) + lane_off + c0;
            const float sc = isk ? p.scale : 1.f;
            bf16* out = p.dqkv + rowi * Nqkv + (size_t)(isk ? p.H + g : p.H + p.nkv + g) * HD + c0;
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
    const int grid = std::min(p.num_units, device_sm_count());
    attn_fwd_tc_kernel<HD><<<grid, NT, FwdLayout<HD>::BYTES, s>>>(map, p);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

template <int HD>
int dq_ds_launch(const CUtensorMap& ds, const CUtensorMap& kv, const DqdsParams& p, cudaStream_t s) {
    if (ensure_smem_limit((const void*)attn_dq_ds_kernel<HD>, DqdsLayout<HD>::BYTES) != cudaSuccess) return -1;
    const int grid = std::min(p.num_units, device_sm_count());
    attn_dq_ds_kernel<HD><<<grid, NTQ, DqdsLayout<HD>::BYTES, s>>>(ds, kv, p);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

template <int HD>
int dkv_launch(const CUtensorMap& kv, const CUtensorMap& do128, const CUtensorMap& ds, const BwdParams& p,
               cudaStream_t s) {
    if (ensure_smem_limit((const void*)attn_dkv_tc_kernel<HD>, DkvLayout<HD>::BYTES) != cudaSuccess) return -1;
    attn_dkv_tc_kernel<HD><<<dim3(p.B, p.nkv, p.nqb), NTB, DkvLayout<HD>::BYTES, s>>>(kv, do128, ds, p);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

// Parameters and the two tensor maps (qkv and dO, 128-row boxes) of both kernels.
int ntri_of(int T) {
    const int nqb = (T + 127) / 128;
    return nqb * (nqb + 1) / 2;
}

// Parameters and the two tensor maps (qkv and dO, 128-row boxes) of the dK/dV kernel.
bool bwd_setup(const void* qkv, const void* dO, float* Dbuf, void* dqkv, void* ds, int B, int T, int H, int nkv,
               int hd, int* status, BwdParams* p, CUtensorMap* kv, CUtensorMap* do128) {
    if (!attention_tc_bwd_supported(hd)) return false;
    if (!aligned16(qkv) || !aligned16(dO) || !aligned16(dqkv) || !aligned16(Dbuf) || !aligned16(ds)) return false;
    if (B > 65535 || H > 65535 || nkv < 1 || H % nkv != 0) return false;
    const int Nqkv = (H + 2 * nkv) * hd;
    if (!map_rows(kv, qkv, Nqkv, (uint64_t)B * T, 128) || !map_rows(do128, dO, (uint64_t)H * hd, (uint64_t)B * T, 128))
        return false;
    *p = BwdParams{};
    p->B = B; p->T = T; p->H = H; p->nkv = nkv; p->nqb = (T + 127) / 128; p->ntri = ntri_of(T);
    p->scale = 1.f / sqrtf((float)hd);
    p->scale_log2 = kLog2e * p->scale;
    p->D = Dbuf;
    p->lse2 = Dbuf + attn_stat_elems(B, T, H);
    p->dqkv = reinterpret_cast<bf16*>(dqkv);
    p->ds = reinterpret_cast<bf16*>(ds);
    p->status = status;
    return true;
}

}  // namespace

int attention_tc_fwd(const void* qkv, void* o, float* lse, int B, int T, int H, int nkv, int hd, void*, size_t,
                     int* status, cudaStream_t s) {
    if (hd != 64 && hd != 128) return 1;
    if (!aligned16(qkv) || !aligned16(o) || nkv < 1 || H % nkv) return 1;
    const int Nqkv = (H + 2 * nkv) * hd;
    CUtensorMap map;
    if (!map_rows(&map, qkv, Nqkv, (uint64_t)B * T, 128)) return 1;
    AttnParams p{};
    p.B = B; p.T = T; p.H = H; p.nkv = nkv; p.nqb = (T + 127) / 128;
    p.pairs_per_group = (H / nkv + 1) / 2;
    p.npair = nkv * p.pairs_per_group;
    const long long units = (long long)B * p.npair * p.nqb;
    if (units > (1ll << 30)) return 1;
    p.num_units = (int)units;
    p.scale_log2 = kLog2e / sqrtf((float)hd);
    p.o = reinterpret_cast<bf16*>(o);
    p.lse = lse;
    p.status = status;
    return hd == 128 ? fwd_launch<128>(map, p, s) : fwd_launch<64>(map, p, s);
}

bool attention_tc_bwd_supported(int hd) { return hd == 64 || hd == 128; }

size_t attention_tc_workspace_bytes(int B, int T, int H, int, int hd) {
    if (!attention_tc_bwd_supported(hd)) return 0;
    return (size_t)B * H * ntri_of(T) * 128 * 128 * sizeof(bf16);
}

int attention_tc_bwd_stats(const void* o, const void* dO, const float* lse, float* Dbuf, int B, int T, int H, int hd,
                           cudaStream_t s) {
    if (!attention_tc_bwd_supported(hd) || !aligned16(o) || !aligned16(dO) || !lse || !Dbuf) return 1;
    const long long threads = (long long)attn_stat_elems(B, T, H) * (hd / 8);
    const unsigned blocks = (unsigned)((threads + 255) / 256);
    const bf16* ob = reinterpret_cast<const bf16*>(o);
    const bf16* db = reinterpret_cast<const bf16*>(dO);
    float* l2 = Dbuf + attn_stat_elems(B, T, H);
    if (hd == 128) attn_bwd_stats_kernel<128><<<blocks, 256, 0, s>>>(ob, db, lse, Dbuf, l2, B, T, H);
    else attn_bwd_stats_kernel<64><<<blocks, 256, 0, s>>>(ob, db, lse, Dbuf, l2, B, T, H);
    count_launch();
    return cudaGetLastError() == cudaSuccess ? 0 : -1;
}

int attention_tc_bwd_dkv(const void* qkv, const void* dO, float* Dbuf, void* dqkv, void* ws, size_t ws_bytes, int B,
                         int T, int H, int nkv, int hd, int* status, cudaStream_t s) {
    BwdParams p;
    CUtensorMap kv, do128;
    if (!ws || ws_bytes < attention_tc_workspace_bytes(B, T, H, nkv, hd)) return 1;
    if (!bwd_setup(qkv, dO, Dbuf, dqkv, ws, B, T, H, nkv, hd, status, &p, &kv, &do128)) return 1;
    CUtensorMap mds;
    if (!map_rows(&mds, ws, 128, (uint64_t)B * H * ntri_of(T) * 128, 128)) return 1;
    return hd == 128 ? dkv_launch<128>(kv, do128, mds, p, s) : dkv_launch<64>(kv, do128, mds, p, s);
}

int attention_tc_bwd_dq(const void* qkv, const void* ws, size_t ws_bytes, void* dqkv, int B, int T, int H, int nkv,
                        int hd, int* status, cudaStream_t s) {
    if (!attention_tc_bwd_supported(hd) || !ws || ws_bytes < attention_tc_workspace_bytes(B, T, H, nkv, hd)) return 1;
    if (!aligned16(qkv) || !aligned16(ws) || !aligned16(dqkv) || B > 65535 || nkv < 1 || H % nkv) return 1;
    const int Nqkv = (H + 2 * nkv) * hd;
    CUtensorMap mds, mkv;
    const uint64_t ds_rows = (uint64_t)B * H * ntri_of(T) * 128;
    if (!map_rows(&mds, ws, 128, ds_rows, 128) || !map_rows(&mkv, qkv, Nqkv, (uint64_t)B * T, 128)) return 1;
    DqdsParams p{};
    p.B = B; p.T = T; p.H = H; p.nkv = nkv; p.nqb = (T + 127) / 128; p.ntri = ntri_of(T);
    p.num_units = B * H * p.nqb;
    p.scale = 1.f / sqrtf((float)hd);
    p.dqkv = reinterpret_cast<bf16*>(dqkv);
    p.status = status;
    return hd == 128 ? dq_ds_launch<128>(mds, mkv, p, s) : dq_ds_launch<64>(mds, mkv, p, s);
}

int attention_tc_bwd(const void* qkv, const void* o, const void* dO, const float* lse, float* Dbuf, void* dqkv,
                     int B, int T, int H, int nkv, int hd, void* ws, size_t ws_bytes, int* status, cudaStream_t s) {
    int r = attention_tc_bwd_stats(o, dO, lse, Dbuf, B, T, H, hd, s);
    if (r == 0) r = attention_tc_bwd_dkv(qkv, dO, Dbuf, dqkv, ws, ws_bytes, B, T, H, nkv, hd, status, s);
    if (r == 0) r = attention_tc_bwd_dq(qkv, ws, ws_bytes, dqkv, B, T, H, nkv, hd, status, s);
    return r;
}

}  // namespace nc
