// Tensor-core causal multi-query attention (bf16 operands, fp32 softmax).
#pragma once
#include "kernels.h"

namespace nc {
// Return 0 when done, > 0 when the shape is not taken (caller falls back),
// < 0 on a CUDA error.
int attention_tc_fwd(const void* qkv, void* o, float* lse, int B, int T, int H, int nkv, int hd, void* ws,
                     size_t ws_bytes, int* status, cudaStream_t s);
bool attention_tc_bwd_supported(int hd);
// Scratch of the backward: the stored dS^T tiles (bf16), one 128 x 128 tile
// per causal (query block, key block) pair of every (batch row, query head).
size_t attention_tc_workspace_bytes(int B, int T, int H, int nkv, int hd);
// The whole backward: stats, then dk/dv (storing dS), then dq.  Dbuf holds
// attn_dbuf_elems(B, T, H) floats: -D = -rowsum(dO * o) and -lse * log2(e), both
// [B, H, attn_tpad(T)] (negated: the dK/dV softmax adds them).
int attention_tc_bwd(const void* qkv, const void* o, const void* dO, const float* lse, float* Dbuf, void* dqkv,
                     int B, int T, int H, int nkv, int hd, void* ws, size_t ws_bytes, int* status, cudaStream_t s);
// Its three launches, in order.
int attention_tc_bwd_stats(const void* o, const void* dO, const float* lse, float* Dbuf, int B, int T, int H, int hd,
                           cudaStream_t s);
int attention_tc_bwd_dkv(const void* qkv, const void* dO, float* Dbuf, void* dqkv, void* ws, size_t ws_bytes, int B,
                         int T, int H, int nkv, int hd, int* status, cudaStream_t s);
int attention_tc_bwd_dq(const void* qkv, const void* ws, size_t ws_bytes, void* dqkv, int B, int T, int H, int nkv,
                        int hd, int* status, cudaStream_t s);
}  // namespace nc
