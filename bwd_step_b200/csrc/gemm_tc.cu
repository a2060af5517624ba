#include "gemm_tc.h"
namespace nc {
int gemm_tc(const GemmDesc&, void*, size_t, cudaStream_t) { return 1; }
size_t gemm_tc_splitk_bytes(int, int, int, int, int) { return 0; }
}  // namespace nc
