// tcgen05 (5th-generation tensor core) GEMM for bf16 operands, fp32
// accumulation in tensor memory, operands staged by TMA.
#pragma once
#include "kernels.h"

namespace nc {
// Runs g on the tensor cores.  Returns 0 when done, > 0 when the shape or
// layout is not taken (the caller falls back), < 0 on a CUDA error.
// `splitk` is scratch for split-K partial sums (gemm_tc_splitk_bytes bytes).
int gemm_tc(const GemmDesc& g, void* splitk, size_t splitk_bytes, cudaStream_t s);
// Split-K scratch for outputs of at most max_out_elems fp32 elements.
size_t gemm_tc_splitk_bytes(size_t max_out_elems);
}  // namespace nc
