// Weight-gradient GEMM that allocates nothing: its split-K partial sums live
// in a file-scope static device array instead of caller- or library-allocated
// workspace.  For callers that cannot call cudaMalloc (see nanochat_b200.h,
// nc_gemm_wgrad_noalloc).
#include "nanochat_b200.h"
#include "kernels.h"
#include "gemm_tc.h"

#include <mutex>

namespace {

// Split-K scratch shared by every call on a device.  Every GPU that loads this
// library holds these bytes until the process exits.
constexpr size_t kWgradScratchBytes = (size_t)NC_WGRAD_NOALLOC_SCRATCH_BYTES;
__device__ __align__(256) unsigned char g_wgrad_scratch[kWgradScratchBytes];

// Device address of g_wgrad_scratch per device ordinal, looked up once with
// that device current (host code may not use the symbol itself as a pointer).
constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

int scratch_for_current_device(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return NC_ERR_NO_DEVICE;
    if (dev < 0 || dev >= kMaxDevices) return NC_ERR_NO_DEVICE;
    std::lock_guard<std::mutex> lock(g_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        if (cudaGetSymbolAddress(&p, g_wgrad_scratch) != cudaSuccess || !p) return NC_ERR_CUDA;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return NC_OK;
}

}  // namespace

extern "C" int nc_gemm_wgrad_noalloc(int rows, int n_out, int n_in, const void* dy, int64_t ld_dy, const void* x,
                                     int64_t ld_x, float* dw, int accumulate, int* status, void* stream) {
    if (rows <= 0 || n_out <= 0 || n_in <= 0 || !dy || !x || !dw) return NC_ERR_INVALID_ARG;
    if (ld_dy < n_out || ld_x < n_in) return NC_ERR_INVALID_ARG;
    // TMA reads dy and x in 16-byte units and the split-K reduction writes dw as
    // float4: every base address and row pitch must be 16-byte aligned
    auto al16 = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; };
    if (!al16(dy) || !al16(x) || !al16(dw) || ld_dy % 8 || ld_x % 8) return NC_ERR_INVALID_ARG;
    // the array must hold at least two K-split partials of the [n_out, n_in] result
    if ((size_t)n_out * (size_t)n_in * sizeof(float) * 2 > kWgradScratchBytes) return NC_ERR_UNSUPPORTED_SHAPE;
    void* scratch = nullptr;
    int r = scratch_for_current_device(&scratch);
    if (r != NC_OK) return r;
    nc::GemmDesc g;
    g.M = n_out; g.N = n_in; g.K = rows; g.in_t = nc::DT_BF16;
    g.A = dy; g.lda = ld_dy; g.a_kmajor = false;  // A(o, t) = dy[t*ld_dy + o]
    g.B = x; g.ldb = ld_x; g.b_kmajor = false;    // B(i, t) = x[t*ld_x + i]
    g.epi = accumulate ? nc::EPI_ACCUM : nc::EPI_STORE;
    g.C = dw; g.ldc = n_in; g.c_t = nc::DT_F32;
    g.status = status;
    r = nc::gemm_tc(g, scratch, kWgradScratchBytes, (cudaStream_t)stream);
    if (r > 0) return NC_ERR_UNSUPPORTED_SHAPE;
    return r == 0 ? NC_OK : NC_ERR_CUDA;
}
