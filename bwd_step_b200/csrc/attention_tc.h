// Tensor-core causal multi-query attention (bf16 operands, fp32 softmax).
#pragma once
#include "kernels.h"

namespace nc {
// Return 0 when done, > 0 when the shape is not taken (caller falls back),
// < 0 on a CUDA error.
int attention_tc_fwd(const void* qkv, void* o, float* lse, int B, int T, int H, int nkv, int hd, void* ws,
                     size_t ws_bytes, int* status, cudaStream_t s);
// Dbuf holds attn_dbuf_elems(B, T, H) floats: D = rowsum(dO * o) and lse * log2(e),
// both [B, H, attn_tpad(T)], written by the dq kernel and read by the dk/dv kernel.
int attention_tc_bwd(const void* qkv, const void* o, const void* dO, const float* lse, float* Dbuf, void* dqkv,
                     int B, int T, int H, int nkv, int hd, void* ws, size_t ws_bytes, int* status, cudaStream_t s);
// The two halves of attention_tc_bwd: dq (with D and the log2-domain lse), then dk/dv.
bool attention_tc_bwd_supported(int hd);
int attention_tc_bwd_dq(const void* qkv, const void* o, const void* dO, const float* lse, float* Dbuf, void* dqkv,
                        int B, int T, int H, int nkv, int hd, int* status, cudaStream_t s);
int attention_tc_bwd_dkv(const void* qkv, const void* dO, float* Dbuf, void* dqkv, int B, int T, int H, int nkv,
                         int hd, int* status, cudaStream_t s);
size_t attention_tc_workspace_bytes(int B, int T, int H, int nkv, int hd);
}  // namespace nc
