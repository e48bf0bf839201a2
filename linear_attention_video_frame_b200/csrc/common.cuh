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
    int has_prep;            // 1: RMSNorm, ReLU and (prep.rope) 3D RoPE of q and k in the scan
    la_prep prep;
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

// 3D RoPE (fused input preparation).  Pairs of a head of D channels: the
// first rope_nt(D) are temporal, then rope_nhw(D) height, then rope_nhw(D)
// width pairs; pair i of a group of n pairs turns by pos * base^(-i / n).
__host__ __device__ inline int rope_nhw(int D) { return (D / 2) / 3; }
__host__ __device__ inline int rope_nt(int D) { return D / 2 - 2 * rope_nhw(D); }

// cos and sin of pos * base^(-i / n).  The angle is formed and reduced
// modulo 2 pi in double, so that positions up to 2^24 keep float accuracy.
__device__ inline void rope_cos_sin(int pos, int i, int n, double log2_base, float& c, float& s) {
    const double th = exp2(-(double)i / (double)n * log2_base);
    double ang = (double)pos * th;
    const double two_pi = 6.283185307179586476925286766559;
    ang -= two_pi * rint(ang / two_pi);
    sincosf((float)ang, &s, &c);
}

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
// Opt `kernel` in to at least `bytes` of dynamic shared memory on the
// current device (the limit is raised when a call asks for more than any
// earlier one, never lowered); returns the CUDA error of a failure.
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
// The fused kernel prepares q and k itself (GDN) when its RoPE tables fit.
bool fused_prep_fits(const ScanArgs& a);
size_t fused_workspace_bytes(const ScanArgs& a);
cudaError_t launch_fused(const ScanArgs& a, cudaStream_t st);

}  // namespace la
