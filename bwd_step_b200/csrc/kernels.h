// Host-side launchers of the step's kernels (internal to the library).
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>
#include <stddef.h>

#include <atomic>

namespace nc {

// Kernels launched by this library so far (process-wide), for launch accounting.
extern std::atomic<long long> g_launches;
inline void count_launch(int n = 1) { g_launches.fetch_add(n, std::memory_order_relaxed); }

enum DType : int { DT_F32 = 0, DT_BF16 = 1 };
inline size_t dt_size(DType t) { return t == DT_BF16 ? 2 : 4; }

// ---------------------------------------------------------------- memory-bound
// cos/sin [T, hd/2] of pos * base^(-2j/hd) for pos = pos0 .. pos0 + T - 1, evaluated in double.
cudaError_t launch_rope_table(float* cos_t, float* sin_t, int T, int hd, float base, cudaStream_t s, int pos0 = 0);

// x[m] = rmsnorm(wte[idx[m]]) (fp32 residual stream), r0[m] = its inverse RMS.
cudaError_t launch_embed_norm_fwd(DType wt, const int32_t* idx, const void* wte, int M, int V, int d,
                                  float* x, float* r0, int* status, cudaStream_t s);
// y = x * r, r = (mean(x^2)+eps)^-1/2 per row; y in activation type.
cudaError_t launch_rmsnorm_fwd(DType at, const float* x, void* y, float* r, int M, int d, cudaStream_t s);
// dx = (accumulate ? dx : 0) + r*(dy - y*mean(dy*y)); optional dxb = dx in activation type.
// dy is fp32, or in the activation type when dy_act.
cudaError_t launch_rmsnorm_bwd(DType at, const void* dy, bool dy_act, const void* y, const float* r, float* dx,
                               bool accumulate, void* dxb, int M, int d, cudaStream_t s);
// de = gradient through the token-embedding norm, recomputing y = wte[idx]*r0.
cudaError_t launch_embed_norm_bwd(DType wt, const float* dx, const int32_t* idx, const void* wte,
                                  const float* r0, float* de, int M, int V, int d, cudaStream_t s);
// In place on the fused qkv rows [M, (H+2nkv)*hd]: q,k <- rope(rmsnorm_hd(q,k)); rqk [M, H+nkv].
cudaError_t launch_qknorm_rope_fwd(DType at, void* qkv, float* rqk, const float* cos_t, const float* sin_t,
                                   int M, int T, int H, int nkv, int hd, cudaStream_t s);
// In place on the q,k parts of dqkv: inverse rotation then RMSNorm backward.
cudaError_t launch_qknorm_rope_bwd(DType at, void* dqkv, const void* qkv, const float* rqk,
                                   const float* cos_t, const float* sin_t, int M, int T, int H, int nkv,
                                   int hd, cudaStream_t s);
// Cross-entropy over R rows of softcapped logits z [R, V] (fp32 or bf16, V % 4 == 0):
// loss_rows[r] = lse - z[tgt]; dl = inv_M*(softmax - onehot)*(1-(z/cap)^2).
cudaError_t launch_ce_chunk(DType zt, DType dlt, const void* z, const int32_t* tgt, int R, int V, float cap,
                            float inv_M, float* loss_rows, void* dl, int* status, cudaStream_t s);
// After the EPI_LMHEAD GEMM of R rows (u [R, V] bf16, stats [R, ntiles]): per row
// S = sum of the tile sums (fixed order), loss_rows[r] = cap + log S - zt[r];
// rs[r] = inv_M / S; u[r, tgt] = ut[r] - (1 - (zt/cap)^2) S (folds the one-hot
// term into u, in fp32, before the single rounding); xfs[r] = xf[r] * rs[r].
// A target outside [0, V) sets ST_BAD_TOKEN and zeroes the row's loss, rs and xfs.
cudaError_t launch_lm_rowstats(const float* stats, int ntiles, const float* zt, const float* ut,
                               const int32_t* tgt, int R, int V, int d, float cap, float inv_M, void* u,
                               const void* xf, void* xfs, float* rs, float* loss_rows, int* status, cudaStream_t s);
// Inference KV cache, K and V each [B, T_max, nkv, hd] in the activation type:
// copies the k, v heads of `rows` qkv rows (batch row r / rows_per_b, position
// pos0 + r % rows_per_b) into it.
cudaError_t launch_kv_append(DType at, const void* qkv, int H, int nkv, int hd, int rows, int rows_per_b,
                             int pos0, void* kc, void* vc, int T_max, cudaStream_t s);
// o[b, h] = softmax(q_bh . K[b, 0..len)^T / sqrt(hd)) V[b, 0..len) for the one
// query per row in qkv rows [B, (H+2nkv) hd] (kv head h / (H / nkv)).
cudaError_t launch_decode_attention(DType at, const void* qkv, const void* kc, const void* vc, int T_max, int len,
                                    int B, int H, int nkv, int hd, void* o, cudaStream_t s);
// loss = mean(loss_rows[0..M)), fixed summation order.
cudaError_t launch_loss_reduce(const float* loss_rows, int M, float* loss, cudaStream_t s);

struct EmbedScratch {
    int* count;        // [V] positions per id
    int* offset;       // [V+1] first slot of each id
    int* cursor;       // [V]
    int* perm;         // [M] positions bucketed by id
    int* perm2;        // [M] same, increasing position within a bucket
    int* active;       // [V] ids that occur
    int* n_active;     // [1]
    int* piece_base;   // [V] first piece of each id
    int* part_base;    // [V] first partial-sum slot of each multi-piece id
    int* piece_bucket; // [pieces] id of each piece
    int* totals;       // [2] pieces, partial slots
    int* fpre;         // [V] used ids before each id within its block of 1024
    void* blk;         // [ceil(V/1024)] per-block scan totals, then prefixes
    float* partial;    // [partial slots, d] piece sums of multi-piece ids
};
size_t embed_scratch_bytes(int M, int V, int d);
EmbedScratch embed_scratch_carve(void* base, int M, int V, int d);
// dwte[v] = sum over positions m with idx[m] == v of de[m], in increasing m;
// rows of unused ids are zero.  Deterministic.
cudaError_t launch_embed_scatter(const int32_t* idx, const float* de, int M, int V, int d, float* dwte,
                                 EmbedScratch sc, cudaStream_t s);
// out[i] = ((accumulate ? out[i] : 0) + sum_{s < splits} part[s*n + i]) * (rs ? rs[i / N] : 1),
// in increasing s (N = row length, a multiple of 4).
cudaError_t launch_splitk_reduce(const float* part, int splits, size_t n, float* out, bool accumulate,
                                 const float* rs, int N, cudaStream_t s);

// ---------------------------------------------------------------- GEMM
// C[m,n] = sum_k A(m,k) * B(n,k).
//   A(m,k) = a_kmajor ? A[m*lda + k] : A[k*lda + m]
//   B(n,k) = b_kmajor ? B[n*ldb + k] : B[k*ldb + n]
enum Epi : int {
    EPI_STORE = 0,      // C = acc                         (C fp32 or activation type)
    EPI_ACCUM = 1,      // C += acc                        (C fp32)
    EPI_RELU2 = 2,      // C = relu(acc)^2, C2 = relu(acc) (activation type)
    EPI_RELU2_BWD = 3,  // C = acc * 2 * aux               (aux = relu(u), activation type)
    EPI_SOFTCAP = 4,    // C = cap * tanh(acc / cap)       (C fp32 or activation type)
    EPI_QKROPE = 5,     // fused qkv rows: per head of the first qk_heads heads,
                        // C = rope(rmsnorm_hd(acc)) and rqk = its inverse RMS; other
                        // columns (v) C = acc.  bf16 C, head_dim 64 or 128 (tcgen05 only)
    EPI_LMHEAD = 6,     // LM head, logits never stored: z = cap*tanh(acc/cap), e = exp(z - cap),
                        // C = e * (1 - (z/cap)^2) (bf16); per (row, 128-column group) the sum of e
                        // into stats[row * stats_ld + group]; at the column tgt[row], z and C in
                        // fp32 into zt[row], ut[row] (tcgen05 only)
    EPI_ROWSCALE = 7,   // C = acc * rs[row]                 (C fp32; tcgen05 only)
    EPI_ATTN_DO = 8,    // attention output gradient dO: C = acc (bf16), and per (row, head of hd
                        // columns) -D = -(sum of C * aux) (aux = o, the attention output) and
                        // -lse * log2(e), into the [B, H, Tp] statistics of the tensor-core
                        // backward (row = b T + t; tcgen05 only)
};

struct GemmDesc {
    int M = 0, N = 0, K = 0;
    DType in_t = DT_F32;  // type of A and B
    const void* A = nullptr; int64_t lda = 0; bool a_kmajor = true;
    const void* B = nullptr; int64_t ldb = 0; bool b_kmajor = true;
    Epi epi = EPI_STORE;
    void* C = nullptr; int64_t ldc = 0; DType c_t = DT_F32;
    void* C2 = nullptr; int64_t ldc2 = 0;
    const void* aux = nullptr; int64_t ldaux = 0;
    float cap = 0.f;
    int* status = nullptr;  // device status word for bounded-wait timeouts
    // EPI_QKROPE: head_dim, sequence length (position = row % T), number of
    // normalised heads (H + n_kv), their inverse RMS [M, qk_heads], RoPE tables [T, hd/2]
    int hd = 0, T = 0, qk_heads = 0;
    float* rqk = nullptr;
    const float* cos_t = nullptr;
    const float* sin_t = nullptr;
    // EPI_LMHEAD: targets of the M rows, per-(row, tile) sums, target z / C values
    const int32_t* tgt = nullptr;
    float* stats = nullptr;
    int stats_ld = 0;
    float* zt = nullptr;
    float* ut = nullptr;
    // EPI_ROWSCALE: one factor per row
    const float* rs = nullptr;
    // EPI_ATTN_DO: statistics D and lse*log2(e) [B, H, attn_tpad(T)], the lse they come from,
    // the number of heads (hd and T as above)
    float* attn_d = nullptr;
    float* attn_lse2 = nullptr;
    const float* attn_lse = nullptr;
    int attn_H = 0;
};

// Column groups of the tensor-core GEMM's output (EPI_LMHEAD writes one sum per group).
constexpr int kGemmStatCols = 128;
inline int gemm_stat_groups(int N) { return (N + kGemmStatCols - 1) / kGemmStatCols; }

// Plain fp32-FMA tiled GEMM (any strides, any sizes).
cudaError_t gemm_simt(const GemmDesc& g, cudaStream_t s);

// ---------------------------------------------------------------- attention
// qkv rows [B*T, (H+2nkv)*hd] hold q (post norm+rope), k (same), v.
// o [B*T, H*hd].  Per-(row, head) softmax statistics (lse, natural log, and
// the backward's D) are stored head-major with the sequence padded to a
// multiple of 128 (one query block): index (b*H + h)*attn_tpad(T) + t.
__host__ __device__ inline int attn_tpad(int T) { return (T + 127) / 128 * 128; }
inline size_t attn_stat_elems(int B, int T, int H) { return (size_t)B * H * attn_tpad(T); }
// The backward's buffer: D (tensor-core path: -D), then (tensor-core path) -lse * log2(e),
// each attn_stat_elems.
inline size_t attn_dbuf_elems(int B, int T, int H) { return 2 * attn_stat_elems(B, T, H); }
cudaError_t launch_attention_fwd_simt(DType at, const void* qkv, void* o, float* lse, int B, int T, int H,
                                      int nkv, int hd, cudaStream_t s);
// Writes dq (into the q columns), dk, dv of dqkv.  Dbuf [B*T, H] scratch.
cudaError_t launch_attention_bwd_simt(DType at, const void* qkv, const void* o, const void* dO,
                                      const float* lse, float* Dbuf, void* dqkv, int B, int T, int H,
                                      int nkv, int hd, cudaStream_t s);

// D[b, h, t] = sum_c dO[b*T+t, h, c] * o[b*T+t, h, c] (softmax backward row term).
cudaError_t launch_attention_bwd_dot(DType at, const void* o, const void* dO, float* D, int B, int T, int H, int hd,
                                     cudaStream_t s);

// ---------------------------------------------------------------- launch helpers
// Raises the dynamic shared-memory limit of kernel `func` to `bytes` on the
// current device, once per (kernel, device): the attribute is per device.
// Thread-safe.
cudaError_t ensure_smem_limit(const void* func, int bytes);
// Streaming multiprocessors of the current device.
int device_sm_count();

// ---------------------------------------------------------------- bounded wait
cudaError_t launch_expired_wait(int* status, int max_iters, cudaStream_t s);

}  // namespace nc
