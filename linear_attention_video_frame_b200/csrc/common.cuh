// Shared definitions of the scan library (host and device).
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "la_scan.h"

namespace la {

// Workspace header: the first 256 bytes of every workspace.
struct WsHeader {
    unsigned int status;        // 0 = ok, LA_ERR_TIMEOUT when a bounded wait gave up
    unsigned int where;         // which wait gave up (diagnostic)
    unsigned int ticket;        // dynamic work counter of persistent kernels
    unsigned int done;          // blocks finished (persistent kernels)
    unsigned int pad[60];
};
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

constexpr size_t kWsHeaderBytes = 256;

__host__ __device__ inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Arguments shared by every scan launcher.
struct ScanArgs {
    const void* q;
    const void* k;
    const void* v;
    void* o;                 // NULL for a state step
    const float* alpha;      // GDN only
    const float* beta;       // GDN only (per frame)
    const float* beta_tok;   // GDN with a per-token update gate [B, H, F, S], else NULL
    const float* state_in;   // may be NULL
    const float* z_in;       // ReLU only, may be NULL
    float* state_out;        // may be NULL
    float* z_out;            // ReLU only, may be NULL
    float k_scale;
    float eps;
    int B, H, F, S, D;
    int mode;                // LA_MODE_RELU / LA_MODE_GDN
    int bf16;                // 1 if q,k,v,o are bf16
    int rev_chunk;           // > 0: reversed GDN scan reset every rev_chunk frames
    float* trans_out;        // GDN interval composite: the transition A_F ... A_1 of the
                             // interval goes here (and the input composite to state_out)
    void* ws;
    size_t ws_bytes;
};

// Frame processed at step s of a scan over F frames: s itself for the
// forward scan (C == 0); for the reversed scan reset at chunk boundaries
// (C > 0), chunk [c C, min((c + 1) C, F)) is taken from its last frame back
// to its first.  A step starts a new chunk (zero state) when s % C == 0.
__host__ __device__ inline int step_frame(int s, int F, int C) {
    if (C <= 0) return s;
    const int c0 = (s / C) * C;
    const int end = c0 + C < F ? c0 + C : F;
    return end - 1 - (s - c0);
}
__host__ __device__ inline bool step_resets(int s, int C) { return C > 0 && s % C == 0; }

// Element access for the two storage types.
__device__ __forceinline__ float load_elem(const void* p, size_t i, int bf16) {
    if (bf16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
    return reinterpret_cast<const float*>(p)[i];
}
__device__ __forceinline__ void store_elem(void* p, size_t i, float x, int bf16) {
    if (bf16) reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(x);
    else reinterpret_cast<float*>(p)[i] = x;
}

// Per-device facts (devinfo.cu).  A process may drive several GPUs, so
// everything that belongs to a device is cached per device.
constexpr int kDefaultSmCount = 148;   // B200; used only when no device is visible
int current_device();                   // current device, or -1
int device_sm_count();                  // SMs of the current device (cached per device)
// Opt `kernel` in to `bytes` of dynamic shared memory on the current device
// (once per device and kernel); returns the CUDA error of the first failure.
cudaError_t ensure_dyn_smem(const void* kernel, int bytes);

// Launchers (host side), each returns cudaGetLastError() of its launches.
cudaError_t launch_simt(const ScanArgs& a, cudaStream_t st);
int simt_kernel_count(const ScanArgs& a);
size_t simt_workspace_bytes(const ScanArgs& a);

// Tensor-core path: bf16 inputs, 64 <= D <= 128, F > 0.
bool tc_eligible(const ScanArgs& a);
size_t tc_workspace_bytes(const ScanArgs& a);
int tc_kernel_count(const ScanArgs& a);
cudaError_t launch_tc(const ScanArgs& a, cudaStream_t st);

// Wide-head tensor-core path: bf16 inputs, 128 < D <= 256, F > 0.
bool wide_eligible(const ScanArgs& a);
size_t wide_workspace_bytes(const ScanArgs& a);
int wide_kernel_count(const ScanArgs& a);
cudaError_t launch_wide(const ScanArgs& a, cudaStream_t st);

// Exclusive prefix over GDN interval composites (composite.cu).
// T and U of interval r start at T + r * stride and U + r * stride (floats).
cudaError_t launch_compose_prefix(const float* T, const float* U, size_t stride, const float* m0,
                                  float* starts, float* mout, int n, int B, int H, int D,
                                  cudaStream_t st);

// Fused persistent tensor-core path (one cooperative launch).
bool fused_eligible(const ScanArgs& a);
size_t fused_workspace_bytes(const ScanArgs& a);
cudaError_t launch_fused(const ScanArgs& a, cudaStream_t st);

}  // namespace la
