// C ABI of the step (nanochat_b200.h) and the host-side orchestration: config
// validation, the flat parameter layout, the workspace plan, and the launch
// sequence of the forward+backward pass on one stream.
//
// Model (nanochat announcement, vpshk.cn, architecture list): normalised
// token embedding -> n_layer pre-norm blocks [x += Wo attn(rope(norm(q)),
// rope(norm(k)), v); x += Wproj relu(Wfc norm(x))^2] -> final norm -> untied
// LM head -> tanh softcap -> mean next-token cross-entropy.
#include "nanochat_b200.h"
#include "common.cuh"
#include "kernels.h"
#include "gemm_tc.h"
#include "attention_tc.h"

#include <string>
#include <vector>
#include <algorithm>

using namespace nc;

struct ParamEntry { std::string name; int64_t offset; int rows, cols; };

struct nc_model {
    nc_config cfg;
    nc_precision prec;
    int device = 0;
    int* status = nullptr;  // device int[64]: [0] = status flags, [1] = loss scratch for the host variant
    std::vector<ParamEntry> layout;
    int64_t nparams = 0;
    int V, d, L, H, nkv, hd, F, Nqkv;
    DType at;  // weight / activation type
    bool tc = false;  // tcgen05 path available (bf16 on sm_100)
    // LM head: fused (logits never stored; tensor-core path only) or materialised
    // logit chunks with a separate cross-entropy pass; rows per chunk (0 = default)
    int lm_mode = NC_LM_HEAD_FUSED;
    int lm_rows = 0;
    // activations recomputed in the backward instead of saved (NC_RECOMPUTE_*)
    int recompute = NC_RECOMPUTE_NONE;
    // caller-owned events recorded when each gradient bucket is final (may be empty)
    std::vector<cudaEvent_t> grad_events;
    // the backward's weight-gradient GEMMs run on this second stream, overlapping the
    // input-gradient chain on the caller's stream; kSideEvents order the two (null: off)
    static constexpr int kSideEvents = 6;
    cudaStream_t side = nullptr;
    cudaEvent_t sev[kSideEvents] = {};
    // profiler: CUDA events around every launch while enabled
    struct Rec { int cls; cudaEvent_t a, b; double flops, bytes; long long launches; };
    bool prof_on = false;
    std::vector<cudaEvent_t> ev_pool;
    size_t ev_next = 0;
    std::vector<Rec> recs;
    cudaEvent_t event() {
        if (ev_next == ev_pool.size()) {
            cudaEvent_t e = nullptr;
            if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
            ev_pool.push_back(e);
        }
        return ev_pool[ev_next++];
    }
};

namespace {

#define CK(x) do { cudaError_t e_ = (x); if (e_ != cudaSuccess) return NC_ERR_CUDA; } while (0)

inline size_t al256(size_t x) { return (x + 255) & ~(size_t)255; }

struct Plan {
    int B = 0, T = 0, M = 0, R = 0;
    size_t total = 0;
    size_t tok, tgt, cosb, sinb, x, dx, g, dxb, xf, r0, rf;
    size_t layers, lay_stride;
    size_t l_a, l_r1, l_qkv, l_rqk, l_o, l_lse, l_m, l_r2, l_ru, l_h;
    bool mlp_shared = false;  // relu(u), relu(u)^2 in one slot for all layers (recomputed in the backward)
    size_t mlp_ru, mlp_h;
    size_t du, dO, dqkv, Dbuf, zc, dlc, loss_rows, emb, splitk, splitk_bytes, attn_ws, attn_ws_bytes;
    size_t lm_stats, lm_zt, lm_ut, lm_rs, lm_xfs;
    int lm_tiles = 0;
};

bool lm_fused(const nc_model* m) { return m->tc && m->lm_mode == NC_LM_HEAD_FUSED; }

// Rows of the LM head processed at once, so that the full [B*T, V] tensor is
// never materialised.  Fused: the [R, V] bf16 chunk of u = e (1 - (z/cap)^2)
// (no logits) is kept near 512 MiB; materialised: the [R, V] logit chunk and
// its gradient near 1 GiB together.  A caller-chosen row count overrides.
int lm_chunk_rows(const nc_model* m, int M) {
    size_t R;
    if (m->lm_rows > 0) {
        R = (size_t)m->lm_rows;
    } else {
        const size_t per_row = (size_t)m->V * dt_size(m->at) * (lm_fused(m) ? 1 : 2);
        const size_t budget = lm_fused(m) ? ((size_t)512 << 20) : ((size_t)1024 << 20);
        R = std::max<size_t>(128, budget / per_row / 128 * 128);
    }
    return (int)std::min<size_t>(R, (size_t)M);
}

// Workspace layout for (B, T).  fwd_only: the forward alone (logits, inference
// prefill): one reused layer slot and none of the backward's buffers.
Plan make_plan(const nc_model* m, int B, int T, bool fwd_only = false) {
    Plan p;
    p.B = B; p.T = T; p.M = B * T;
    const size_t M = p.M, d = m->d, A = dt_size(m->at);
    const bool bwd = !fwd_only;
    size_t off = 0;
    auto take = [&](size_t bytes) { size_t o = off; off += al256(bytes); return o; };
    p.tok = take(4 * M);
    p.tgt = take(bwd ? 4 * M : 0);
    p.cosb = take(4ull * T * (m->hd / 2));
    p.sinb = take(4ull * T * (m->hd / 2));
    p.x = take(4 * M * d);
    p.dx = take(bwd ? 4 * M * d : 0);
    p.g = take(bwd ? 4 * M * d : 0);
    p.dxb = take(bwd ? A * M * d : 0);
    p.xf = take(A * M * d);
    p.r0 = take(4 * M);
    p.rf = take(4 * M);
    // per-layer saved activations
    size_t lo = 0;
    auto ltake = [&](size_t bytes) { size_t o = lo; lo += al256(bytes); return o; };
    p.l_a = ltake(A * M * d);
    p.l_r1 = ltake(4 * M);
    p.l_qkv = ltake(A * M * m->Nqkv);
    p.l_rqk = ltake(4 * M * (m->H + m->nkv));
    p.l_o = ltake(A * M * m->H * m->hd);
    p.l_lse = ltake(4 * attn_stat_elems(B, T, m->H));
    p.l_m = ltake(A * M * d);
    p.l_r2 = ltake(4 * M);
    p.mlp_shared = bwd && (m->recompute & NC_RECOMPUTE_MLP);
    p.l_ru = ltake(p.mlp_shared ? 0 : A * M * m->F);
    p.l_h = ltake(p.mlp_shared ? 0 : A * M * m->F);
    p.lay_stride = lo;
    p.layers = take(lo * (bwd ? m->L : 1));
    p.mlp_ru = take(p.mlp_shared ? A * M * m->F : 0);
    p.mlp_h = take(p.mlp_shared ? A * M * m->F : 0);
    p.du = take(bwd ? A * M * m->F : 0);
    p.dO = take(bwd ? A * M * m->H * m->hd : 0);
    p.dqkv = take(bwd ? A * M * m->Nqkv : 0);
    p.Dbuf = take(bwd ? 4 * attn_dbuf_elems(B, T, m->H) : 0);
    p.R = lm_chunk_rows(m, p.M);
    const bool fz = bwd && lm_fused(m);
    p.zc = take(bwd ? A * (size_t)p.R * m->V : 0);                     // logits, or u on the fused path
    p.dlc = take(bwd && !lm_fused(m) ? A * (size_t)p.R * m->V : 0);   // their gradient (materialised path)
    p.lm_tiles = gemm_stat_groups(m->V);
    p.lm_stats = take(fz ? 4ull * p.R * p.lm_tiles : 0);
    p.lm_zt = take(fz ? 4ull * p.R : 0);
    p.lm_ut = take(fz ? 4ull * p.R : 0);
    p.lm_rs = take(fz ? 4ull * p.R : 0);
    p.lm_xfs = take(fz ? A * (size_t)p.R * d : 0);
    p.loss_rows = take(bwd ? 4 * M : 0);
    p.emb = take(bwd ? embed_scratch_bytes(p.M, m->V, m->d) : 0);
    size_t max_out = std::max({(size_t)m->F * d, (size_t)m->H * m->hd * d, (size_t)m->Nqkv * d});
    max_out = std::max(max_out, bwd ? (size_t)p.R * d : std::min(M * d, (size_t)1 << 22));
    p.splitk_bytes = m->tc ? gemm_tc_splitk_bytes(max_out) : 0;
    p.splitk = take(p.splitk_bytes);
    p.attn_ws_bytes = m->tc && bwd ? attention_tc_workspace_bytes(B, T, m->H, m->nkv, m->hd) : 0;
    p.attn_ws = take(p.attn_ws_bytes);
    p.total = off;
    return p;
}

struct Ctx {
    nc_model* m;
    Plan p;
    char* ws;
    cudaStream_t s;
    template <typename T = void> T* at(size_t off) const { return reinterpret_cast<T*>(ws + off); }
    char* layer(int l) const { return ws + p.layers + (size_t)l * p.lay_stride; }
    // relu(u) and relu(u)^2 of layer l's MLP (one shared slot when they are recomputed)
    void* mlp_ru(char* lb) const { return p.mlp_shared ? ws + p.mlp_ru : lb + p.l_ru; }
    void* mlp_h(char* lb) const { return p.mlp_shared ? ws + p.mlp_h : lb + p.l_h; }
};

enum ProfCls {
    P_GEMM_FWD = 0, P_GEMM_DGRAD, P_GEMM_WGRAD, P_GEMM_LM_Z, P_GEMM_LM_DX, P_GEMM_LM_DW, P_GEMM_FMA,
    P_ATTN_FWD, P_ATTN_BWD, P_ATTN_BWD_DQ, P_ATTN_BWD_DKV, P_NORM_FWD, P_NORM_BWD, P_QKROPE_FWD, P_QKROPE_BWD,
    P_EMBED_FWD, P_EMBED_BWD, P_CE, P_OTHER, P_GEMM_RECOMPUTE, P_COUNT
};
// tcgen05 GEMM launches are tagged by role: forward y = x W^T, input
// gradient dX = dY W, weight gradient dW = dY^T X, and the three LM-head products.
const char* const kProfNames[P_COUNT] = {
    "gemm_fwd", "gemm_dgrad", "gemm_wgrad", "gemm_lmhead_z", "gemm_lmhead_dx", "gemm_lmhead_dw", "gemm_fma",
    "attention_fwd", "attention_bwd", "attention_bwd_dq", "attention_bwd_dkv", "rmsnorm_fwd", "rmsnorm_bwd",
    "qknorm_rope_fwd", "qknorm_rope_bwd", "embed_fwd", "embed_bwd", "cross_entropy", "other",
    "gemm_recompute"};

// Records a CUDA event pair around the launches made in its lifetime (only
// while profiling is enabled), with the algorithmic FLOPs / HBM bytes of the work.
struct Prof {
    nc_model* m; cudaStream_t s; int cls; double flops, bytes; cudaEvent_t a = nullptr; long long l0 = 0;
    Prof(const Ctx& c, int cls_, double f, double b) : m(c.m), s(c.s), cls(cls_), flops(f), bytes(b) {
        if (m->prof_on && (a = m->event())) { cudaEventRecord(a, s); l0 = g_launches.load(); }
    }
    ~Prof() {
        if (!a) return;
        cudaEvent_t b = m->event();
        if (!b) return;
        cudaEventRecord(b, s);
        m->recs.push_back({cls, a, b, flops, bytes, g_launches.load() - l0});
    }
};

// C = A B^T with the tensor-core kernel where it applies, else the FMA kernel.
int run_gemm(const Ctx& c, const GemmDesc& g, int role) {
    const double es = g.in_t == DT_BF16 ? 2.0 : 4.0;
    Prof pr(c, role, 2.0 * g.M * g.N * (double)g.K,
            es * ((double)g.M * g.K + (double)g.N * g.K) + (g.c_t == DT_BF16 ? 2.0 : 4.0) * g.M * (double)g.N);
    pr.cls = (c.m->tc && g.in_t == DT_BF16) ? role : P_GEMM_FMA;
    if (c.m->tc && g.in_t == DT_BF16) {
        int r = gemm_tc(g, c.ws + c.p.splitk, c.p.splitk_bytes, c.s);
        if (r == 0) return NC_OK;
        if (r < 0) return NC_ERR_CUDA;
        // r > 0: shape not taken by the tensor-core kernel, fall through
        pr.cls = P_GEMM_FMA;
    }
    CK(gemm_simt(g, c.s));
    return NC_OK;
}

// A GEMM whose epilogue only the tensor-core kernel implements.
int run_gemm_tc(const Ctx& c, const GemmDesc& g, int role) {
    Prof pr(c, role, 2.0 * g.M * g.N * (double)g.K,
            2.0 * ((double)g.M * g.K + (double)g.N * g.K) + (g.c_t == DT_BF16 ? 2.0 : 4.0) * g.M * (double)g.N);
    const int r = gemm_tc(g, c.ws + c.p.splitk, c.p.splitk_bytes, c.s);
    if (r > 0) return NC_ERR_UNSUPPORTED_SHAPE;
    return r == 0 ? NC_OK : NC_ERR_CUDA;
}

GemmDesc mk(const nc_model* m, int M, int N, int K, const void* A, int64_t lda, bool ak, const void* B,
            int64_t ldb, bool bk, Epi epi, void* C, int64_t ldc, DType ct) {
    GemmDesc g;
    g.M = M; g.N = N; g.K = K; g.in_t = m->at;
    g.A = A; g.lda = lda; g.a_kmajor = ak;
    g.B = B; g.ldb = ldb; g.b_kmajor = bk;
    g.epi = epi; g.C = C; g.ldc = ldc; g.c_t = ct;
    g.cap = m->cfg.softcap;
    g.status = m->status;
    return g;
}

#define RG(x) do { int r_ = (x); if (r_ != NC_OK) return r_; } while (0)

// Causal attention FLOPs of one pass over the batch: QK^T and PV over the
// T(T+1)/2 visible (query, key) pairs of every head.
double attn_flops(const Ctx& c) {
    return 4.0 * c.p.B * c.m->H * (double)c.m->hd * (double)c.p.T * (c.p.T + 1) / 2.0;
}

int attention_fwd(const Ctx& c, const void* qkv, void* o, float* lse) {
    const nc_model* m = c.m;
    Prof pr(c, P_ATTN_FWD, attn_flops(c), 0.0);
    if (m->tc) {
        int r = attention_tc_fwd(qkv, o, lse, c.p.B, c.p.T, m->H, m->nkv, m->hd, c.ws + c.p.attn_ws,
                                 c.p.attn_ws_bytes, m->status, c.s);
        if (r == 0) return NC_OK;
        if (r < 0) return NC_ERR_CUDA;
    }
    CK(launch_attention_fwd_simt(m->at, qkv, o, lse, c.p.B, c.p.T, m->H, m->nkv, m->hd, c.s));
    return NC_OK;
}

// Attention backward, then the QK-norm + RoPE backward into the pre-norm q, k
// gradients (one pass over all heads of each position).  Tensor cores:
// statistics (unless the dO GEMM's epilogue wrote them) and dk / dv (which also
// stores the dS tiles), then dq from those tiles; otherwise the plain-FMA kernels.
int attention_bwd(const Ctx& c, const void* qkv, const void* o, const void* dO, const float* lse, const float* rqk,
                  void* dqkv, bool stats_ready) {
    const nc_model* m = c.m;
    float* Dbuf = c.at<float>(c.p.Dbuf);
    const float* cs = c.at<float>(c.p.cosb);
    const float* sn = c.at<float>(c.p.sinb);
    bool done = false;
    if (m->tc && attention_tc_bwd_supported(m->hd)) {
        void* ws = c.ws + c.p.attn_ws;
        int r;
        {
            Prof pr(c, P_ATTN_BWD_DKV, 2.0 * attn_flops(c), 0.0);
            r = stats_ready ? 0 : attention_tc_bwd_stats(o, dO, lse, Dbuf, c.p.B, c.p.T, m->H, m->hd, c.s);
            if (r == 0)
                r = attention_tc_bwd_dkv(qkv, dO, Dbuf, dqkv, ws, c.p.attn_ws_bytes, c.p.B, c.p.T, m->H, m->nkv,
                                         m->hd, m->status, c.s);
        }
        if (r == 0) {
            Prof pr(c, P_ATTN_BWD_DQ, 0.5 * attn_flops(c), 0.0);
            r = attention_tc_bwd_dq(qkv, ws, c.p.attn_ws_bytes, dqkv, c.p.B, c.p.T, m->H, m->nkv, m->hd, m->status,
                                    c.s);
        }
        if (r < 0) return NC_ERR_CUDA;
        done = r == 0;
    }
    if (!done) {
        Prof pr(c, P_ATTN_BWD, 2.0 * attn_flops(c), 0.0);
        CK(launch_attention_bwd_simt(m->at, qkv, o, dO, lse, Dbuf, dqkv, c.p.B, c.p.T, m->H, m->nkv, m->hd, c.s));
    }
    const double A = (double)dt_size(m->at);
    Prof pr(c, P_QKROPE_BWD, 0.0, (double)c.p.M * (m->H + m->nkv) * (3.0 * A * m->hd + 4.0));
    CK(launch_qknorm_rope_bwd(m->at, dqkv, qkv, rqk, cs, sn, c.p.M, c.p.T, m->H, m->nkv, m->hd, c.s));
    return NC_OK;
}

struct W {  // weight pointers of one call
    const char* base; size_t es; const nc_model* m;
    const void* p(int idx) const { return base + (size_t)m->layout[idx].offset * es; }
    const void* wte() const { return p(0); }
    const void* wqkv(int l) const { return p(1 + 6 * l); }
    const void* wo(int l) const { return p(1 + 6 * l + 3); }
    const void* wfc(int l) const { return p(1 + 6 * l + 4); }
    const void* wproj(int l) const { return p(1 + 6 * l + 5); }
    const void* wlm() const { return p(1 + 6 * m->L); }
};

// Inference KV cache of one call: K and V [n_layer][B, T_max, nkv, hd] each
// (activation type).  Prefill writes positions 0..T-1; a decode step (one
// token per row, T = 1 in the plan) writes position pos and attends to 0..pos.
struct KvCache {
    char* base;
    int T_max, pos;
    bool decode;
    size_t layer_bytes;  // K + V of one layer
    void* k(int l) const { return base + (size_t)l * layer_bytes; }
    void* v(int l) const { return base + (size_t)l * layer_bytes + layer_bytes / 2; }
};

// Forward through the blocks; with `save` every layer keeps its own
// activations for the backward, otherwise layer slot 0 is reused.  With `kv`
// the k, v heads of every layer go to the inference cache, and in a decode
// step the attention reads the cache instead of the call's own positions.
int forward_blocks(const Ctx& c, const W& w, const int32_t* tok, bool save, const KvCache* kv = nullptr) {
    nc_model* m = c.m;
    const int M = c.p.M, d = m->d;
    float* x = c.at<float>(c.p.x);
    const float* cs = c.at<float>(c.p.cosb);
    const float* sn = c.at<float>(c.p.sinb);
    const bool decode = kv && kv->decode;
    {
        Prof pr(c, P_OTHER, 0.0, 8.0 * c.p.T * (m->hd / 2));
        CK(launch_rope_table(c.at<float>(c.p.cosb), c.at<float>(c.p.sinb), c.p.T, m->hd, m->cfg.rope_base, c.s,
                             decode ? kv->pos : 0));
    }
    const double A = (double)dt_size(m->at);
    { Prof pr(c, P_EMBED_FWD, 0.0, (double)M * (A * d + 4.0 * d + 8.0)); CK(launch_embed_norm_fwd(m->at, tok, w.wte(), M, m->V, d, x, c.at<float>(c.p.r0), m->status, c.s)); }
    const size_t Hhd = (size_t)m->H * m->hd;
    for (int l = 0; l < m->L; ++l) {
        char* lb = c.layer(save ? l : 0);
        void* a = lb + c.p.l_a;
        void* qkv = lb + c.p.l_qkv;
        void* o = lb + c.p.l_o;
        void* mm = lb + c.p.l_m;
        void* ru = c.mlp_ru(lb);
        void* h = c.mlp_h(lb);
        { Prof pr(c, P_NORM_FWD, 0.0, (double)M * (4.0 * d + A * d + 4.0)); CK(launch_rmsnorm_fwd(m->at, x, a, (float*)(lb + c.p.l_r1), M, d, c.s)); }
        // q, k, v = a Wq^T, a Wk^T, a Wv^T; then q, k <- rope(rmsnorm(q, k)) per head, fused into
        // the GEMM epilogue on the tensor-core path
        bool qk_fused = false;
        float* rqk = (float*)(lb + c.p.l_rqk);
        if (m->tc && (m->hd == 64 || m->hd == 128)) {
            GemmDesc gq = mk(m, M, m->Nqkv, d, a, d, true, w.wqkv(l), d, true, EPI_QKROPE, qkv, m->Nqkv, m->at);
            gq.hd = m->hd; gq.T = c.p.T; gq.qk_heads = m->H + m->nkv;
            gq.rqk = rqk; gq.cos_t = cs; gq.sin_t = sn;
            Prof pr(c, P_GEMM_FWD, 2.0 * M * m->Nqkv * (double)d,
                    A * ((double)M * d + (double)m->Nqkv * d + (double)M * m->Nqkv));
            int r = gemm_tc(gq, c.ws + c.p.splitk, c.p.splitk_bytes, c.s);
            if (r < 0) return NC_ERR_CUDA;
            qk_fused = r == 0;
        }
        if (!qk_fused) {
            RG(run_gemm(c, mk(m, M, m->Nqkv, d, a, d, true, w.wqkv(l), d, true, EPI_STORE, qkv, m->Nqkv, m->at),
                        P_GEMM_FWD));
            Prof pr(c, P_QKROPE_FWD, 0.0, (double)M * (m->H + m->nkv) * (2.0 * A * m->hd + 4.0));
            CK(launch_qknorm_rope_fwd(m->at, qkv, rqk, cs, sn, M, c.p.T, m->H, m->nkv, m->hd, c.s));
        }
        if (kv) {
            Prof pr(c, P_OTHER, 0.0, 4.0 * A * M * m->nkv * m->hd);
            CK(launch_kv_append(m->at, qkv, m->H, m->nkv, m->hd, M, c.p.T, decode ? kv->pos : 0, kv->k(l), kv->v(l),
                                kv->T_max, c.s));
        }
        if (decode) {
            Prof pr(c, P_ATTN_FWD, 4.0 * M * m->H * (double)m->hd * (kv->pos + 1), 0.0);
            CK(launch_decode_attention(m->at, qkv, kv->k(l), kv->v(l), kv->T_max, kv->pos + 1, c.p.B, m->H, m->nkv,
                                       m->hd, o, c.s));
        } else {
            RG(attention_fwd(c, qkv, o, (float*)(lb + c.p.l_lse)));
        }
        RG(run_gemm(c, mk(m, M, d, (int)Hhd, o, Hhd, true, w.wo(l), Hhd, true, EPI_ACCUM, x, d, DT_F32), P_GEMM_FWD));
        { Prof pr(c, P_NORM_FWD, 0.0, (double)M * (4.0 * d + A * d + 4.0)); CK(launch_rmsnorm_fwd(m->at, x, mm, (float*)(lb + c.p.l_r2), M, d, c.s)); }
        GemmDesc fc = mk(m, M, m->F, d, mm, d, true, w.wfc(l), d, true, EPI_RELU2, h, m->F, m->at);
        fc.C2 = ru; fc.ldc2 = m->F;
        RG(run_gemm(c, fc, P_GEMM_FWD));
        RG(run_gemm(c, mk(m, M, d, m->F, h, m->F, true, w.wproj(l), m->F, true, EPI_ACCUM, x, d, DT_F32), P_GEMM_FWD));
    }
    { Prof pr(c, P_NORM_FWD, 0.0, (double)M * (4.0 * d + A * d + 4.0)); CK(launch_rmsnorm_fwd(m->at, x, c.at(c.p.xf), c.at<float>(c.p.rf), M, d, c.s)); }
    return NC_OK;
}

int step(nc_model* m, const int32_t* tok, const int32_t* tgt, int B, int T, const void* weights, float* grads,
         float* loss, void* workspace, cudaStream_t s) {
    Ctx c{m, make_plan(m, B, T), (char*)workspace, s};
    W w{(const char*)weights, dt_size(m->at), m};
    const int M = c.p.M, d = m->d, V = m->V, F = m->F, Nqkv = m->Nqkv;
    const int Hhd = m->H * m->hd;
    auto G = [&](int idx) { return grads + m->layout[idx].offset; };
    RG(forward_blocks(c, w, tok, true));

    // ---- LM head + softcap + cross-entropy, then its backward, R rows at a time
    void* xf = c.at(c.p.xf);
    float* gbuf = c.at<float>(c.p.g);
    float* loss_rows = c.at<float>(c.p.loss_rows);
    const size_t A = dt_size(m->at);
    float* dwlm = G(1 + 6 * m->L);
    if (lm_fused(m)) {
        // fused: the GEMM epilogue turns each logit tile into u = e (1 - (z/cap)^2),
        // e = exp(z - cap), with per-tile sums of e; a row pass gives the loss and the
        // row factors 1 / (S M); then dX = diag(1/(S M)) u Wlm and dWlm += u^T (xf / (S M))
        void* uc = c.at(c.p.zc);
        float* stats = c.at<float>(c.p.lm_stats);
        float* zt = c.at<float>(c.p.lm_zt);
        float* ut = c.at<float>(c.p.lm_ut);
        float* rs = c.at<float>(c.p.lm_rs);
        void* xfs = c.at(c.p.lm_xfs);
        for (int r0 = 0; r0 < M; r0 += c.p.R) {
            const int rc = std::min(c.p.R, M - r0);
            const char* xfc = (const char*)xf + (size_t)r0 * d * A;
            GemmDesc gz = mk(m, rc, V, d, xfc, d, true, w.wlm(), d, true, EPI_LMHEAD, uc, V, DT_BF16);
            gz.tgt = tgt + r0; gz.stats = stats; gz.stats_ld = c.p.lm_tiles; gz.zt = zt; gz.ut = ut;
            RG(run_gemm_tc(c, gz, P_GEMM_LM_Z));
            {
                Prof pr(c, P_CE, 0.0, (double)rc * (4.0 * c.p.lm_tiles + 2.0 * A * d + 16.0));
                CK(launch_lm_rowstats(stats, c.p.lm_tiles, zt, ut, tgt + r0, rc, V, d, m->cfg.softcap,
                                      1.0f / (float)M, uc, xfc, xfs, rs, loss_rows + r0, m->status, s));
            }
            GemmDesc gx = mk(m, rc, d, V, uc, V, true, w.wlm(), d, false, EPI_ROWSCALE, gbuf + (size_t)r0 * d, d,
                             DT_F32);
            gx.rs = rs;
            RG(run_gemm_tc(c, gx, P_GEMM_LM_DX));
            RG(run_gemm(c, mk(m, V, d, rc, uc, V, false, xfs, d, false, r0 == 0 ? EPI_STORE : EPI_ACCUM, dwlm, d,
                              DT_F32), P_GEMM_LM_DW));
        }
    } else {
        // materialised: softcapped logits in the activation type (bf16 on the
        // mixed-precision path, fp32 on the debug path), then a cross-entropy pass
        // writing dl, then dX = dl Wlm and dWlm += dl^T xf
        void* zc = c.at(c.p.zc);
        void* dlc = c.at(c.p.dlc);
        for (int r0 = 0; r0 < M; r0 += c.p.R) {
            int rc = std::min(c.p.R, M - r0);
            const char* xfc = (const char*)xf + (size_t)r0 * d * A;
            RG(run_gemm(c, mk(m, rc, V, d, xfc, d, true, w.wlm(), d, true, EPI_SOFTCAP, zc, V, m->at), P_GEMM_LM_Z));
            {
                Prof pr(c, P_CE, 0.0, (double)rc * V * (2.0 * A));
                CK(launch_ce_chunk(m->at, m->at, zc, tgt + r0, rc, V, m->cfg.softcap, 1.0f / (float)M,
                                   loss_rows + r0, dlc, m->status, s));
            }
            RG(run_gemm(c, mk(m, rc, d, V, dlc, V, true, w.wlm(), d, false, EPI_STORE, gbuf + (size_t)r0 * d, d,
                              DT_F32), P_GEMM_LM_DX));
            RG(run_gemm(c, mk(m, V, d, rc, dlc, V, false, xfc, d, false, r0 == 0 ? EPI_STORE : EPI_ACCUM, dwlm, d,
                              DT_F32), P_GEMM_LM_DW));
        }
    }
    { Prof pr(c, P_OTHER, 0.0, 4.0 * M); CK(launch_loss_reduce(loss_rows, M, loss, s)); }
    // bucket i of the gradients is final: record the caller's event, if any
    auto bucket_done = [&](int i) -> int {
        if (!m->grad_events.empty() && cudaEventRecord(m->grad_events[i], s) != cudaSuccess) return NC_ERR_CUDA;
        return NC_OK;
    };
    RG(bucket_done(0));  // dWlm

    // ---- backward through the blocks
    float* dx = c.at<float>(c.p.dx);
    void* dxb = c.at(c.p.dxb);
    { Prof pr(c, P_NORM_BWD, 0.0, (double)M * (8.0 * d + 2.0 * A * d + 4.0)); CK(launch_rmsnorm_bwd(m->at, gbuf, false, xf, c.at<float>(c.p.rf), dx, false, dxb, M, d, s)); }
    void* du = c.at(c.p.du);
    void* dO = c.at(c.p.dO);
    void* dqkv = c.at(c.p.dqkv);
    float* Dbuf = c.at<float>(c.p.Dbuf);
    // the attention statistics come from the dO GEMM's epilogue (rows t < T only): the
    // padding of the last query block past T stays zero for the whole backward
    const bool fuse_stats = m->tc && attention_tc_bwd_supported(m->hd);
    if (fuse_stats && T % 128 != 0) CK(cudaMemsetAsync(Dbuf, 0, 4 * attn_dbuf_elems(B, T, m->H), s));
    // Weight-gradient GEMMs on the second stream (when there is one): each starts once the
    // caller's stream has produced its inputs, and the caller's stream waits for it only
    // before overwriting an input it reads (dxb by the next norm backward, du by the next
    // layer's first GEMM, dqkv by the next layer's attention backward).  They are the only
    // users of the split-K scratch during the loop and run in order on their stream.
    // While the per-launch profiler is on everything stays on the caller's stream, so
    // that each event pair times one kernel running alone.
    const cudaStream_t side = m->prof_on ? nullptr : m->side;
    Ctx c2 = c;
    if (side) c2.s = side;
    enum { EV_FORK = 0, EV_PROJ, EV_FC, EV_OPROJ, EV_QKV, EV_END };
    auto fork = [&]() -> bool {  // the side stream continues after the caller's stream's work so far
        return !side || (cudaEventRecord(m->sev[EV_FORK], s) == cudaSuccess &&
                       cudaStreamWaitEvent(side, m->sev[EV_FORK], 0) == cudaSuccess);
    };
    auto mark = [&](int e) -> bool { return !side || cudaEventRecord(m->sev[e], side) == cudaSuccess; };
    auto after = [&](int e) -> bool { return !side || cudaStreamWaitEvent(s, m->sev[e], 0) == cudaSuccess; };
    auto layer_done = [&](int i) -> int {  // this layer's weight gradients are the side stream's work so far
        if (m->grad_events.empty()) return NC_OK;
        return cudaEventRecord(m->grad_events[i], side ? side : s) == cudaSuccess ? NC_OK : NC_ERR_CUDA;
    };
    for (int l = m->L - 1; l >= 0; --l) {
        char* lb = c.layer(l);
        int base = 1 + 6 * l;
        // MLP: x_out = x_mid + h Wproj^T, h = relu(u)^2, u = m Wfc^T
        if (c.p.mlp_shared && l != m->L - 1) {
            // recompute relu(u) and relu(u)^2 from the saved m (the last layer's are still in the slot)
            GemmDesc fc = mk(m, M, F, d, lb + c.p.l_m, d, true, w.wfc(l), d, true, EPI_RELU2, c.mlp_h(lb), F, m->at);
            fc.C2 = c.mlp_ru(lb); fc.ldc2 = F;
            RG(run_gemm(c, fc, P_GEMM_RECOMPUTE));
        }
        if (!after(EV_FC)) return NC_ERR_CUDA;  // the previous layer's dWfc has read du
        GemmDesc g1 = mk(m, M, F, d, dxb, d, true, w.wproj(l), F, false, EPI_RELU2_BWD, du, F, m->at);
        g1.aux = c.mlp_ru(lb); g1.ldaux = F;
        RG(run_gemm(c, g1, P_GEMM_DGRAD));
        if (!fork()) return NC_ERR_CUDA;
        RG(run_gemm(c2, mk(m, d, F, M, dxb, d, false, c.mlp_h(lb), F, false, EPI_STORE, G(base + 5), F, DT_F32),
                    P_GEMM_WGRAD));
        if (!mark(EV_PROJ)) return NC_ERR_CUDA;
        RG(run_gemm(c2, mk(m, F, d, M, du, F, false, lb + c.p.l_m, d, false, EPI_STORE, G(base + 4), d, DT_F32),
                    P_GEMM_WGRAD));
        if (!mark(EV_FC)) return NC_ERR_CUDA;
        RG(run_gemm(c, mk(m, M, d, F, du, F, true, w.wfc(l), d, false, EPI_STORE, gbuf, d, m->at), P_GEMM_DGRAD));
        if (!after(EV_PROJ)) return NC_ERR_CUDA;  // dWproj has read dxb
        { Prof pr(c, P_NORM_BWD, 0.0, (double)M * (8.0 * d + 3.0 * A * d + 4.0)); CK(launch_rmsnorm_bwd(m->at, gbuf, true, lb + c.p.l_m, (float*)(lb + c.p.l_r2), dx, true, dxb, M, d, s)); }
        // attention: x_mid = x_in + o Wo^T; dO = dx Wo, with the softmax-backward statistics
        // D = rowsum(dO * o) and lse*log2(e) formed in the same GEMM's epilogue (tensor-core path)
        bool stats_ready = false;
        if (fuse_stats) {
            GemmDesc gd = mk(m, M, Hhd, d, dxb, d, true, w.wo(l), Hhd, false, EPI_ATTN_DO, dO, Hhd, m->at);
            gd.aux = lb + c.p.l_o; gd.ldaux = Hhd;
            gd.hd = m->hd; gd.T = T; gd.attn_H = m->H;
            gd.attn_d = Dbuf; gd.attn_lse2 = Dbuf + attn_stat_elems(B, T, m->H);
            gd.attn_lse = (const float*)(lb + c.p.l_lse);
            RG(run_gemm_tc(c, gd, P_GEMM_DGRAD));
            stats_ready = true;
        } else {
            RG(run_gemm(c, mk(m, M, Hhd, d, dxb, d, true, w.wo(l), Hhd, false, EPI_STORE, dO, Hhd, m->at),
                        P_GEMM_DGRAD));
        }
        if (!fork()) return NC_ERR_CUDA;
        RG(run_gemm(c2, mk(m, d, Hhd, M, dxb, d, false, lb + c.p.l_o, Hhd, false, EPI_STORE, G(base + 3), Hhd,
                           DT_F32), P_GEMM_WGRAD));
        if (!mark(EV_OPROJ)) return NC_ERR_CUDA;
        if (!after(EV_QKV)) return NC_ERR_CUDA;  // the previous layer's dWqkv has read dqkv
        RG(attention_bwd(c, lb + c.p.l_qkv, lb + c.p.l_o, dO, (float*)(lb + c.p.l_lse), (float*)(lb + c.p.l_rqk),
                         dqkv, stats_ready));
        RG(run_gemm(c, mk(m, M, d, Nqkv, dqkv, Nqkv, true, w.wqkv(l), d, false, EPI_STORE, gbuf, d, m->at),
                    P_GEMM_DGRAD));
        if (!fork()) return NC_ERR_CUDA;
        RG(run_gemm(c2, mk(m, Nqkv, d, M, dqkv, Nqkv, false, lb + c.p.l_a, d, false, EPI_STORE, G(base), d,
                           DT_F32), P_GEMM_WGRAD));
        if (!mark(EV_QKV)) return NC_ERR_CUDA;
        RG(layer_done(m->L - l));  // this layer's six weight gradients
        if (!after(EV_OPROJ)) return NC_ERR_CUDA;  // dWo has read dxb
        {
            Prof pr(c, P_NORM_BWD, 0.0, (double)M * (8.0 * d + (l > 0 ? 3.0 : 2.0) * A * d + 4.0));
            CK(launch_rmsnorm_bwd(m->at, gbuf, true, lb + c.p.l_a, (float*)(lb + c.p.l_r1), dx, true,
                                  l > 0 ? dxb : nullptr, M, d, s));
        }
    }
    // the caller's stream ends after every weight gradient
    if (!mark(EV_END) || !after(EV_END)) return NC_ERR_CUDA;
    // ---- token embedding: norm backward, then the deterministic scatter-add
    {
        // norm backward (dx, Wte row, r0 -> de), then de read once and dWte written once
        Prof pr(c, P_EMBED_BWD, 0.0, (double)M * (8.0 * d + A * d + 8.0) + 4.0 * M * d + 4.0 * (double)V * d);
        CK(launch_embed_norm_bwd(m->at, dx, tok, w.wte(), c.at<float>(c.p.r0), gbuf, M, V, d, s));
        CK(launch_embed_scatter(tok, gbuf, M, V, d, G(0), embed_scratch_carve(c.ws + c.p.emb, M, V, d), s));
    }
    RG(bucket_done(m->L + 1));  // dWte
    return NC_OK;
}

// The model's device must be current: its buffers are that device's memory,
// and kernels launched on another device would reach them as peer memory.
bool on_model_device(const nc_model* m) {
    int dev = -1;
    return cudaGetDevice(&dev) == cudaSuccess && dev == m->device;
}

int validate_call(nc_model* m, int B, int T, size_t ws_bytes, const void* const* ptrs, int nptr,
                  bool fwd_only = false) {
    if (!m || B <= 0 || T <= 0) return NC_ERR_INVALID_ARG;
    if (!on_model_device(m)) return NC_ERR_INVALID_ARG;
    if ((long long)B * T > (1 << 24)) return NC_ERR_UNSUPPORTED_SHAPE;
    for (int i = 0; i < nptr; ++i)
        if (!ptrs[i]) return NC_ERR_INVALID_ARG;
    if (ws_bytes < make_plan(m, B, T, fwd_only).total) return NC_ERR_WORKSPACE_TOO_SMALL;
    return NC_OK;
}

}  // namespace

// ============================================================================ C ABI
extern "C" {

int nc_model_create(const nc_config* cfg, nc_precision prec, nc_model** out) {
    if (!out) return NC_ERR_INVALID_ARG;
    *out = nullptr;
    if (!cfg) return NC_ERR_INVALID_ARG;
    if (prec != NC_PREC_BF16 && prec != NC_PREC_FP32_DEBUG) return NC_ERR_INVALID_ARG;
    const nc_config& c = *cfg;
    if (c.vocab <= 0 || c.d_model <= 0 || c.n_layer <= 0 || c.n_head <= 0 || c.n_kv_head <= 0 ||
        c.head_dim <= 0 || c.mlp_mult <= 0 || !(c.softcap > 0.f) || !(c.rope_base > 1.f))
        return NC_ERR_INVALID_ARG;
    if (c.vocab % 64 || c.d_model % 64 || c.n_head % c.n_kv_head) return NC_ERR_UNSUPPORTED_SHAPE;
    if (c.head_dim != 16 && c.head_dim != 32 && c.head_dim != 64 && c.head_dim != 128)
        return NC_ERR_UNSUPPORTED_SHAPE;
    if ((long long)c.vocab * c.d_model > (1ll << 31) || (long long)c.mlp_mult * c.d_model > (1 << 20))
        return NC_ERR_UNSUPPORTED_SHAPE;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NC_ERR_NO_DEVICE;
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess || major != 10)
        return NC_ERR_NO_DEVICE;
    nc_model* m = new nc_model();
    m->cfg = c;
    m->prec = prec;
    m->device = dev;
    m->V = c.vocab; m->d = c.d_model; m->L = c.n_layer; m->H = c.n_head; m->nkv = c.n_kv_head;
    m->hd = c.head_dim; m->F = c.mlp_mult * c.d_model; m->Nqkv = (c.n_head + 2 * c.n_kv_head) * c.head_dim;
    m->at = prec == NC_PREC_BF16 ? DT_BF16 : DT_F32;
    m->tc = prec == NC_PREC_BF16;
    m->lm_mode = m->tc ? NC_LM_HEAD_FUSED : NC_LM_HEAD_MATERIALISED;
    int64_t off = 0;
    auto add = [&](const std::string& n, int r, int cc) { m->layout.push_back({n, off, r, cc}); off += (int64_t)r * cc; };
    add("wte", m->V, m->d);
    for (int l = 0; l < m->L; ++l) {
        std::string p = "h." + std::to_string(l) + ".";
        add(p + "wq", m->H * m->hd, m->d);
        add(p + "wk", m->nkv * m->hd, m->d);
        add(p + "wv", m->nkv * m->hd, m->d);
        add(p + "wo", m->d, m->H * m->hd);
        add(p + "wfc", m->F, m->d);
        add(p + "wproj", m->d, m->F);
    }
    add("wlm", m->V, m->d);
    m->nparams = off;
    if (cudaMalloc(&m->status, 64 * sizeof(int)) != cudaSuccess ||
        cudaMemset(m->status, 0, 64 * sizeof(int)) != cudaSuccess) {
        cudaFree(m->status);
        delete m;
        return NC_ERR_CUDA;
    }
    // second stream for the weight-gradient GEMMs (the step runs without it if it cannot be made)
    bool side_ok = cudaStreamCreateWithFlags(&m->side, cudaStreamNonBlocking) == cudaSuccess;
    for (int i = 0; side_ok && i < nc_model::kSideEvents; ++i)
        side_ok = cudaEventCreateWithFlags(&m->sev[i], cudaEventDisableTiming) == cudaSuccess;
    if (!side_ok) {
        for (int i = 0; i < nc_model::kSideEvents; ++i)
            if (m->sev[i]) cudaEventDestroy(m->sev[i]), m->sev[i] = nullptr;
        if (m->side) cudaStreamDestroy(m->side);
        m->side = nullptr;
        cudaGetLastError();
    }
    *out = m;
    return NC_OK;
}

void nc_model_destroy(nc_model* m) {
    if (!m) return;
    for (cudaEvent_t e : m->ev_pool) cudaEventDestroy(e);
    for (cudaEvent_t e : m->sev)
        if (e) cudaEventDestroy(e);
    if (m->side) cudaStreamDestroy(m->side);
    cudaFree(m->status);
    delete m;
}

int64_t nc_num_params(const nc_model* m) { return m ? m->nparams : 0; }

int nc_param_layout(const nc_model* m, int i, const char** name, int64_t* offset, int* rows, int* cols) {
    if (!m || i < 0 || i >= (int)m->layout.size()) return NC_ERR_INVALID_ARG;
    const ParamEntry& e = m->layout[i];
    if (name) *name = e.name.c_str();
    if (offset) *offset = e.offset;
    if (rows) *rows = e.rows;
    if (cols) *cols = e.cols;
    return NC_OK;
}

size_t nc_workspace_bytes(const nc_model* m, int B, int T) {
    if (!m || B <= 0 || T <= 0 || (long long)B * T > (1 << 24)) return 0;
    return make_plan(m, B, T).total;
}

int nc_forward_backward(nc_model* m, const int32_t* tokens, const int32_t* targets, int B, int T,
                        const void* weights, float* grads, float* loss, void* workspace, size_t ws_bytes,
                        void* stream) {
    const void* ptrs[] = {tokens, targets, weights, grads, loss, workspace};
    int v = validate_call(m, B, T, ws_bytes, ptrs, 6);
    if (v != NC_OK) return v;
    int r = step(m, tokens, targets, B, T, weights, grads, loss, workspace, (cudaStream_t)stream);
    if (r != NC_OK) return r;
    return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

int nc_forward_backward_host(nc_model* m, const int32_t* h_tokens, const int32_t* h_targets, int B, int T,
                             const void* weights, float* grads, float* h_loss, void* workspace, size_t ws_bytes,
                             void* stream) {
    const void* ptrs[] = {h_tokens, h_targets, weights, grads, h_loss, workspace};
    int v = validate_call(m, B, T, ws_bytes, ptrs, 6);
    if (v != NC_OK) return v;
    cudaStream_t s = (cudaStream_t)stream;
    Plan p = make_plan(m, B, T);
    char* ws = (char*)workspace;
    int32_t* dtok = (int32_t*)(ws + p.tok);
    int32_t* dtgt = (int32_t*)(ws + p.tgt);
    size_t bytes = sizeof(int32_t) * (size_t)B * T;
    CK(cudaMemcpyAsync(dtok, h_tokens, bytes, cudaMemcpyHostToDevice, s));
    CK(cudaMemcpyAsync(dtgt, h_targets, bytes, cudaMemcpyHostToDevice, s));
    float* dloss = (float*)(m->status + 1);
    int r = step(m, dtok, dtgt, B, T, weights, grads, dloss, workspace, s);
    if (r != NC_OK) return r;
    CK(cudaMemcpyAsync(h_loss, dloss, sizeof(float), cudaMemcpyDeviceToHost, s));
    CK(cudaStreamSynchronize(s));
    return NC_OK;
}

int nc_forward_logits(nc_model* m, const int32_t* tokens, int B, int T, const void* weights, void* logits,
                      void* workspace, size_t ws_bytes, void* stream) {
    const void* ptrs[] = {tokens, weights, logits, workspace};
    int v = validate_call(m, B, T, ws_bytes, ptrs, 4, true);
    if (v != NC_OK) return v;
    Ctx c{m, make_plan(m, B, T, true), (char*)workspace, (cudaStream_t)stream};
    W w{(const char*)weights, dt_size(m->at), m};
    RG(forward_blocks(c, w, tokens, false));
    RG(run_gemm(c, mk(m, c.p.M, m->V, m->d, c.at(c.p.xf), m->d, true, w.wlm(), m->d, true, EPI_SOFTCAP, logits,
                      m->V, m->at), P_GEMM_LM_Z));
    return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

size_t nc_kv_cache_bytes(const nc_model* m, int B, int T_max) {
    if (!m || B <= 0 || T_max <= 0) return 0;
    return (size_t)m->L * 2 * B * (size_t)T_max * m->nkv * m->hd * dt_size(m->at);
}

size_t nc_inference_workspace_bytes(const nc_model* m, int B, int T_max) {
    if (!m || B <= 0 || T_max <= 0 || (long long)B * T_max > (1 << 24)) return 0;
    return std::max(make_plan(m, B, T_max, true).total, make_plan(m, B, 1, true).total);
}

int nc_prefill(nc_model* m, const int32_t* tokens, int B, int T, const void* weights, void* kv_cache, int T_max,
               void* logits, void* workspace, size_t ws_bytes, void* stream) {
    const void* ptrs[] = {tokens, weights, kv_cache, logits, workspace};
    if (T_max < T) return NC_ERR_INVALID_ARG;
    int v = validate_call(m, B, T, ws_bytes, ptrs, 5, true);
    if (v != NC_OK) return v;
    Ctx c{m, make_plan(m, B, T, true), (char*)workspace, (cudaStream_t)stream};
    W w{(const char*)weights, dt_size(m->at), m};
    const KvCache kv{(char*)kv_cache, T_max, 0, false, nc_kv_cache_bytes(m, B, T_max) / m->L};
    RG(forward_blocks(c, w, tokens, false, &kv));
    // logits of the last position of every row: rows b*T + T-1 of xf (row stride T*d)
    const char* last = (const char*)c.at(c.p.xf) + (size_t)(T - 1) * m->d * dt_size(m->at);
    RG(run_gemm(c, mk(m, B, m->V, m->d, last, (int64_t)T * m->d, true, w.wlm(), m->d, true, EPI_SOFTCAP, logits,
                      m->V, m->at), P_GEMM_LM_Z));
    return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

int nc_decode_step(nc_model* m, const int32_t* tokens, int B, int pos, const void* weights, void* kv_cache,
                   int T_max, void* logits, void* workspace, size_t ws_bytes, void* stream) {
    const void* ptrs[] = {tokens, weights, kv_cache, logits, workspace};
    if (pos < 0 || pos >= T_max) return NC_ERR_INVALID_ARG;
    int v = validate_call(m, B, 1, ws_bytes, ptrs, 5, true);
    if (v != NC_OK) return v;
    Ctx c{m, make_plan(m, B, 1, true), (char*)workspace, (cudaStream_t)stream};
    W w{(const char*)weights, dt_size(m->at), m};
    const KvCache kv{(char*)kv_cache, T_max, pos, true, nc_kv_cache_bytes(m, B, T_max) / m->L};
    RG(forward_blocks(c, w, tokens, false, &kv));
    RG(run_gemm(c, mk(m, B, m->V, m->d, c.at(c.p.xf), m->d, true, w.wlm(), m->d, true, EPI_SOFTCAP, logits, m->V,
                      m->at), P_GEMM_LM_Z));
    return cudaGetLastError() == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

int nc_check(nc_model* m, void* stream) {
    if (!m) return NC_ERR_INVALID_ARG;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaStreamSynchronize(s) != cudaSuccess) return NC_ERR_CUDA;
    int st = 0;
    if (cudaMemcpy(&st, m->status, sizeof(int), cudaMemcpyDeviceToHost) != cudaSuccess) return NC_ERR_CUDA;
    if (cudaMemset(m->status, 0, sizeof(int)) != cudaSuccess) return NC_ERR_CUDA;
    if (st & ST_TIMEOUT) return NC_ERR_DEVICE_TIMEOUT;
    if (st & ST_BAD_LAYOUT) return NC_ERR_CUDA;
    if (st & ST_BAD_TOKEN) return NC_ERR_BAD_TOKEN;
    return NC_OK;
}

const char* nc_status_string(int code) {
    switch (code) {
        case NC_OK: return "ok";
        case NC_ERR_INVALID_ARG: return "invalid argument";
        case NC_ERR_UNSUPPORTED_SHAPE: return "unsupported shape";
        case NC_ERR_WORKSPACE_TOO_SMALL: return "workspace too small";
        case NC_ERR_CUDA: return "CUDA error";
        case NC_ERR_BAD_TOKEN: return "token or target id out of range";
        case NC_ERR_DEVICE_TIMEOUT: return "bounded device wait expired";
        case NC_ERR_NO_DEVICE: return "no sm_100 CUDA device";
    }
    return "unknown status";
}

int nc_profile_enable(nc_model* m, int enable) {
    if (!m) return NC_ERR_INVALID_ARG;
    if (enable) { m->recs.clear(); m->ev_next = 0; }
    m->prof_on = enable != 0;
    return NC_OK;
}

int nc_profile_read(nc_model* m, void* stream, nc_profile_row* rows, int max_rows) {
    if (!m || (!rows && max_rows > 0)) return NC_ERR_INVALID_ARG;
    if (cudaStreamSynchronize((cudaStream_t)stream) != cudaSuccess) return NC_ERR_CUDA;
    nc_profile_row agg[P_COUNT] = {};
    bool seen[P_COUNT] = {};
    for (const auto& r : m->recs) {
        float ms = 0.f;
        if (cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) return NC_ERR_CUDA;
        nc_profile_row& a = agg[r.cls];
        a.kernel = kProfNames[r.cls];
        a.launches += r.launches;
        a.ms += ms;
        a.flops += r.flops;
        a.bytes += r.bytes;
        seen[r.cls] = true;
    }
    int n = 0;
    for (int k = 0; k < P_COUNT; ++k)
        if (seen[k] && n < max_rows) rows[n++] = agg[k];
    return n;
}

int64_t nc_launch_count(void) { return g_launches.load(); }

int nc_debug_expired_wait(nc_model* m, int max_iters, void* stream) {
    if (!m || max_iters <= 0 || !on_model_device(m)) return NC_ERR_INVALID_ARG;
    CK(launch_expired_wait(m->status, max_iters, (cudaStream_t)stream));
    return NC_OK;
}

int nc_set_lm_head(nc_model* m, int mode, int chunk_rows) {
    if (!m || chunk_rows < 0) return NC_ERR_INVALID_ARG;
    if (mode != NC_LM_HEAD_FUSED && mode != NC_LM_HEAD_MATERIALISED) return NC_ERR_INVALID_ARG;
    if (mode == NC_LM_HEAD_FUSED && !m->tc) return NC_ERR_INVALID_ARG;
    m->lm_mode = mode;
    m->lm_rows = chunk_rows;
    return NC_OK;
}

int nc_set_recompute(nc_model* m, int flags) {
    if (!m || (flags & ~NC_RECOMPUTE_MLP)) return NC_ERR_INVALID_ARG;
    m->recompute = flags;
    return NC_OK;
}

int nc_grad_bucket_count(const nc_model* m) { return m ? m->L + 2 : NC_ERR_INVALID_ARG; }

int nc_grad_bucket(const nc_model* m, int i, int64_t* offset, int64_t* count) {
    if (!m || !offset || !count || i < 0 || i > m->L + 1) return NC_ERR_INVALID_ARG;
    auto size = [&](int idx) { return (int64_t)m->layout[idx].rows * m->layout[idx].cols; };
    int first, last;  // layout entries of the bucket (adjacent in the flat layout)
    if (i == 0) {
        first = last = 1 + 6 * m->L;  // wlm
    } else if (i == m->L + 1) {
        first = last = 0;  // wte
    } else {
        const int l = m->L - i;  // layers in backward order
        first = 1 + 6 * l;
        last = first + 5;
    }
    *offset = m->layout[first].offset;
    *count = m->layout[last].offset + size(last) - m->layout[first].offset;
    return NC_OK;
}

int nc_set_grad_events(nc_model* m, void* const* events, int n) {
    if (!m) return NC_ERR_INVALID_ARG;
    if (n == 0) {
        m->grad_events.clear();
        return NC_OK;
    }
    if (!events || n != m->L + 2) return NC_ERR_INVALID_ARG;
    std::vector<cudaEvent_t> ev((size_t)n);
    for (int i = 0; i < n; ++i) {
        if (!events[i]) return NC_ERR_INVALID_ARG;
        ev[i] = static_cast<cudaEvent_t>(events[i]);
    }
    m->grad_events.swap(ev);
    return NC_OK;
}

}  // extern "C"

// ============================================================================ testing ABI
#include "nanochat_b200_testing.h"

extern "C" int nc_test_gemm(int M, int N, int K, int in_bf16, const void* A, int64_t lda, int a_kmajor,
                            const void* B, int64_t ldb, int b_kmajor, int epi, void* C, int64_t ldc, int c_bf16,
                            void* C2, int64_t ldc2, const void* aux, int64_t ldaux, float cap, int use_tc,
                            void* scratch, size_t scratch_bytes, int* status, void* stream) {
    if (M <= 0 || N <= 0 || K <= 0 || !A || !B || !C || epi < 0 || epi > 4) return NC_ERR_INVALID_ARG;
    if ((epi == EPI_RELU2 && !C2) || (epi == EPI_RELU2_BWD && !aux)) return NC_ERR_INVALID_ARG;
    GemmDesc g;
    g.M = M; g.N = N; g.K = K; g.in_t = in_bf16 ? DT_BF16 : DT_F32;
    g.A = A; g.lda = lda; g.a_kmajor = a_kmajor != 0;
    g.B = B; g.ldb = ldb; g.b_kmajor = b_kmajor != 0;
    g.epi = (Epi)epi; g.C = C; g.ldc = ldc; g.c_t = c_bf16 ? DT_BF16 : DT_F32;
    g.C2 = C2; g.ldc2 = ldc2; g.aux = aux; g.ldaux = ldaux; g.cap = cap; g.status = status;
    cudaStream_t s = (cudaStream_t)stream;
    if (use_tc) {
        int r = gemm_tc(g, scratch, scratch_bytes, s);
        if (r > 0) return NC_ERR_UNSUPPORTED_SHAPE;
        return r == 0 ? NC_OK : NC_ERR_CUDA;
    }
    return gemm_simt(g, s) == cudaSuccess ? NC_OK : NC_ERR_CUDA;
}

extern "C" size_t nc_test_attention_workspace_bytes(int B, int T, int H, int nkv, int hd) {
    if (B <= 0 || T <= 0 || H <= 0 || nkv <= 0) return 0;
    return attention_tc_workspace_bytes(B, T, H, nkv, hd);
}

extern "C" int nc_test_attention(int B, int T, int H, int nkv, int hd, const void* qkv, void* o, float* lse,
                                 const void* dO, void* dqkv, float* Dbuf, void* ws, size_t ws_bytes, int use_tc,
                                 int* status, void* stream) {
    if (B <= 0 || T <= 0 || H <= 0 || nkv <= 0 || H % nkv || !qkv || !o || !lse) return NC_ERR_INVALID_ARG;
    if (hd != 16 && hd != 32 && hd != 64 && hd != 128) return NC_ERR_UNSUPPORTED_SHAPE;
    cudaStream_t s = (cudaStream_t)stream;
    if (use_tc) {
        int r = attention_tc_fwd(qkv, o, lse, B, T, H, nkv, hd, nullptr, 0, status, s);
        if (r != 0) return r > 0 ? NC_ERR_UNSUPPORTED_SHAPE : NC_ERR_CUDA;
        if (dO) {
            if (!dqkv || !Dbuf) return NC_ERR_INVALID_ARG;
            r = attention_tc_bwd(qkv, o, dO, lse, Dbuf, dqkv, B, T, H, nkv, hd, ws, ws_bytes, status, s);
            if (r != 0) return r > 0 ? NC_ERR_UNSUPPORTED_SHAPE : NC_ERR_CUDA;
        }
        return NC_OK;
    }
    if (launch_attention_fwd_simt(DT_BF16, qkv, o, lse, B, T, H, nkv, hd, s) != cudaSuccess) return NC_ERR_CUDA;
    if (dO) {
        if (!dqkv || !Dbuf) return NC_ERR_INVALID_ARG;
        if (launch_attention_bwd_simt(DT_BF16, qkv, o, dO, lse, Dbuf, dqkv, B, T, H, nkv, hd, s) != cudaSuccess)
            return NC_ERR_CUDA;
    }
    return NC_OK;
}
