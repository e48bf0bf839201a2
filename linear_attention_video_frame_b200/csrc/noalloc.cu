// la_scan_gdn_noalloc: the frame-wise GDN scan for callers that cannot
// allocate device memory.
//
// Some callers have no way to hand the library a workspace: code that runs
// under a host framework which owns every device allocation and exposes no
// scratch API to its plug-ins, or latency-critical loops whose rules forbid
// cudaMalloc/cudaFree (they synchronise the device and can fail at run time).
// For them this entry point uses a fixed scratch area that is part of the
// library image itself: a file-scope __device__ array, created by the CUDA
// driver when the library's device code is loaded on a GPU and kept there
// until the process exits.
//
// The host cannot use the array's name as a device address (in host code it
// names a host-side stand-in), so the address is fetched once per device with
// cudaGetSymbolAddress while that device is current, cached, and passed to
// the regular GDN entry point as its workspace.  Nothing here allocates.
#include <mutex>

#include "common.cuh"

namespace {

static __device__ __align__(256) unsigned char g_scan_scratch[LA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {};

// Device address of the scratch array on the current device (set up on the
// first call made with that device current).
la_status scratch_of_current_device(void** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) {
        cudaGetLastError();
        return LA_ERR_CUDA;
    }
    if (dev < 0 || dev >= kMaxDevices) return LA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
        void* p = nullptr;
        const cudaError_t e = cudaGetSymbolAddress(&p, g_scan_scratch);
        if (e != cudaSuccess || p == nullptr) {
            cudaGetLastError();
            return LA_ERR_CUDA;
        }
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return LA_OK;
}

}  // namespace

extern "C" la_status la_scan_gdn_noalloc(const void* q, const void* k, const void* v, void* o,
                                         la_dtype dt, const float* alpha, const float* beta,
                                         float k_scale, const float* state_in, float* state_out,
                                         int B, int H, int F, int S, int D, cudaStream_t stream) {
    const size_t need = la_workspace_size(LA_MODE_GDN, B, H, F, S, D);
    if (need > (size_t)LA_NOALLOC_SCRATCH_BYTES) return LA_ERR_UNSUPPORTED;
    void* scratch = nullptr;
    // A shape la_workspace_size rejects (need == 0) still goes to la_scan_gdn,
    // which reports the precise argument error without enqueuing anything.
    const la_status s = scratch_of_current_device(&scratch);
    if (s != LA_OK) return s;
    return la_scan_gdn(q, k, v, o, dt, alpha, beta, k_scale, state_in, state_out, B, H, F, S, D,
                       scratch, (size_t)LA_NOALLOC_SCRATCH_BYTES, stream);
}

// The status word lives in the first bytes of the scratch array, exactly as
// it does in a caller's workspace, so the workspace query reads it once the
// array's device address is known.
extern "C" la_status la_query_noalloc_status(cudaStream_t stream) {
    void* scratch = nullptr;
    const la_status s = scratch_of_current_device(&scratch);
    if (s != LA_OK) return s;
    return la_query_device_status(scratch, stream);
}
