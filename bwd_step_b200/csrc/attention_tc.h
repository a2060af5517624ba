// Tensor-core causal multi-query attention (bf16 operands, fp32 softmax).
#pragma once
#include "kernels.h"

namespace nc {
// Return 0 when done, > 0 when the shape is not taken (caller falls back),
// < 0 on a CUDA error.
int attention_tc_fwd(const void* qkv, void* o, float* lse, int B, int T, int H, int nkv, int hd, void* ws,
                     size_t ws_bytes, int* status, cudaStream_t s);
int attention_tc_bwd(const void* qkv, const void* o, const void* dO, const float* lse, float* Dbuf, void* dqkv,
                     int B, int T, int H, int nkv, int hd, void* ws, size_t ws_bytes, int* status, cudaStream_t s);
// The two halves of attention_tc_bwd: D = rowsum(dO*o) and dq, then dk/dv.
// With `fuse`, dq and dk are written through the QK-norm + RoPE backward
// (gradients of the projections before the norm), using the saved post-RoPE
// q/k in qkv, their inverse RMS rqk [B*T, H+nkv] and the RoPE tables [T, hd/2].
struct QkNormFuse {
    const float* rqk;
    const float* cos_t;
    const float* sin_t;
};
bool attention_tc_bwd_supported(int hd);
int attention_tc_bwd_dq(const void* qkv, const void* o, const void* dO, const float* lse, float* Dbuf, void* dqkv,
                        int B, int T, int H, int nkv, int hd, int* status, cudaStream_t s, const QkNormFuse* fuse);
int attention_tc_bwd_dkv(const void* qkv, const void* dO, const float* lse, const float* Dbuf, void* dqkv, int B,
                         int T, int H, int nkv, int hd, int* status, cudaStream_t s, const QkNormFuse* fuse);
size_t attention_tc_workspace_bytes(int B, int T, int H, int nkv, int hd);
}  // namespace nc
