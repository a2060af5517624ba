// Host-side launch helpers shared by the kernels' launchers: per-device
// function attributes and device properties.
#include "kernels.h"

#include <mutex>
#include <set>
#include <utility>

namespace nc {

namespace {
std::mutex g_attr_mu;
std::set<std::pair<const void*, int>> g_attr_done;  // (kernel, device) pairs already raised
}  // namespace

cudaError_t ensure_smem_limit(const void* func, int bytes) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    std::lock_guard<std::mutex> lock(g_attr_mu);
    if (g_attr_done.count({func, dev})) return cudaSuccess;
    e = cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) g_attr_done.insert({func, dev});
    return e;
}

int device_sm_count() {
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0)
        return 148;
    return n;
}

}  // namespace nc
