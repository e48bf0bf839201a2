// Facts and one-time set-up that belong to a device, not to the process: a
// process may drive several GPUs, and both a kernel's shared-memory opt-in
// (cudaFuncSetAttribute) and the SM count are properties of one device.
#include <map>
#include <mutex>
#include <utility>

#include "common.cuh"

namespace la {
namespace {

constexpr int kMaxDevices = 64;
std::mutex g_dev_mu;
int g_sm_count[kMaxDevices] = {};
// Largest dynamic shared memory each (device, kernel) has been opted in to.
std::map<std::pair<int, const void*>, int> g_smem_set;

}  // namespace

int current_device() {
    int dev = -1;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return -1;
    }
    return (dev >= 0 && dev < kMaxDevices) ? dev : -1;
}

int device_sm_count() {
    const int dev = current_device();
    if (dev < 0) return kDefaultSmCount;
    std::lock_guard<std::mutex> lock(g_dev_mu);
    if (g_sm_count[dev] <= 0) {
        int n = 0;
        if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            n <= 0) {
            cudaGetLastError();
            return kDefaultSmCount;
        }
        g_sm_count[dev] = n;
    }
    return g_sm_count[dev];
}

cudaError_t ensure_dyn_smem(const void* kernel, int bytes) {
    const int dev = current_device();
    if (dev < 0) return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_dev_mu);
    const std::pair<int, const void*> key(dev, kernel);
    auto it = g_smem_set.find(key);
    if (it != g_smem_set.end() && it->second >= bytes) return cudaSuccess;
    // A kernel whose shared memory depends on the call's shape (D) may ask
    // for more than an earlier call did: raise the limit, never lower it.
    const cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return e;
    }
    g_smem_set[key] = bytes;
    return cudaSuccess;
}

}  // namespace la
