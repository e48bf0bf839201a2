// Facts and one-time set-up that belong to a device, not to the process: a
// process may drive several GPUs, and both a kernel's shared-memory opt-in
// (cudaFuncSetAttribute) and the SM count are properties of one device.
#include <mutex>
#include <set>
#include <utility>

#include "common.cuh"

namespace la {
namespace {

constexpr int kMaxDevices = 64;
std::mutex g_dev_mu;
int g_sm_count[kMaxDevices] = {};
std::set<std::pair<int, const void*>> g_smem_done;   // (device, kernel) pairs set up

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
    if (g_smem_done.count(key)) return cudaSuccess;
    const cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e != cudaSuccess) {
        cudaGetLastError();
        return e;
    }
    g_smem_done.insert(key);
    return cudaSuccess;
}

}  // namespace la
