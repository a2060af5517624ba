/*
 * nanochat_b200_testing.h -- kernel-level entry points used by the unit tests
 * of the step's building blocks.  Same conventions as nanochat_b200.h: device
 * pointers owned by the caller, work enqueued on `stream`, NC_* return codes.
 * Not needed to run the step.
 */
#ifndef NANOCHAT_B200_TESTING_H
#define NANOCHAT_B200_TESTING_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* One GEMM C = A B^T of a bias-free linear layer (nanochat announcement,
 * vpshk.cn, architecture list: linear layers without biases), with the
 * step's fused epilogues.
 *   A(m,k) = a_kmajor ? A[m*lda + k] : A[k*lda + m]      (m < M, k < K)
 *   B(n,k) = b_kmajor ? B[n*ldb + k] : B[k*ldb + n]      (n < N, k < K)
 *   in_bf16: A and B are bf16 (else fp32).  use_tc: 1 = tcgen05 tensor-core
 *   kernel (bf16 only; NC_ERR_UNSUPPORTED_SHAPE if it cannot take the
 *   layout), 0 = plain FMA kernel.
 *   epi: 0 store C=acc; 1 C+=acc (C fp32); 2 C=relu(acc)^2 and C2=relu(acc);
 *        3 C=acc*2*aux; 4 C=cap*tanh(acc/cap).  c_bf16 selects C's type for
 *        0, 2, 3, 4 (2 and 3 need the operand type).
 *   scratch / scratch_bytes: split-K partial sums (may be NULL / 0). */
int nc_test_gemm(int M, int N, int K, int in_bf16, const void* A, int64_t lda, int a_kmajor, const void* B,
                 int64_t ldb, int b_kmajor, int epi, void* C, int64_t ldc, int c_bf16, void* C2, int64_t ldc2,
                 const void* aux, int64_t ldaux, float cap, int use_tc, void* scratch, size_t scratch_bytes,
                 int* status, void* stream);

/* Causal multi-query attention (nanochat announcement, vpshk.cn,
 * architecture list: multi-query attention), bf16, on the fused qkv rows
 * [B*T, (H+2*nkv)*hd] (q heads, k heads, v heads per row).  Writes
 * o [B*T, H*hd] and lse (natural log).  When dO != NULL also runs
 * the backward: dq, dk, dv into the matching columns of dqkv (same layout as
 * qkv), with Dbuf fp32 scratch.  lse is laid out [B, H, Tp] with Tp = T
 * rounded up to a multiple of 128; Dbuf holds 2 * B * H * Tp floats.  ws /
 * ws_bytes: device scratch of the tensor-core backward (the dS tiles),
 * nc_test_attention_workspace_bytes(B, T, H, nkv, hd) bytes (0 when the
 * kernels need none).  use_tc: 1 = tcgen05 kernels (head_dim 64 or 128), 0 =
 * plain FMA kernels. */
size_t nc_test_attention_workspace_bytes(int B, int T, int H, int nkv, int hd);
int nc_test_attention(int B, int T, int H, int nkv, int hd, const void* qkv, void* o, float* lse,
                      const void* dO, void* dqkv, float* Dbuf, void* ws, size_t ws_bytes, int use_tc, int* status,
                      void* stream);

#ifdef __cplusplus
}
#endif
#endif /* NANOCHAT_B200_TESTING_H */
