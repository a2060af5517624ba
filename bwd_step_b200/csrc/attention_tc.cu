#include "attention_tc.h"
namespace nc {
int attention_tc_fwd(const void*, void*, float*, int, int, int, int, int, void*, size_t, cudaStream_t) { return 1; }
int attention_tc_bwd(const void*, const void*, const void*, const float*, float*, void*, int, int, int, int, int,
                     void*, size_t, cudaStream_t) { return 1; }
size_t attention_tc_workspace_bytes(int, int, int, int, int) { return 0; }
}  // namespace nc
