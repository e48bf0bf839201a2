// Host side of the C ABI: argument validation, workspace sizing, dispatch.
#include <cmath>
#include <cstdlib>
#include <cstring>

#include "common.cuh"

namespace la {
namespace {

bool shape_supported(int D) { return D >= 16 && D <= 256 && D % 16 == 0; }

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// A pointer the kernels may dereference: device or managed memory of the
// current device.  NULL is accepted here (callers decide whether NULL is legal).
la_status check_ptr(const void* p, int dev) {
    if (!p) return LA_OK;
    if (!aligned16(p)) return LA_ERR_INVALID_ARG;
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return LA_ERR_INVALID_ARG;
    }
    if (at.type == cudaMemoryTypeManaged) return LA_OK;
    if (at.type != cudaMemoryTypeDevice || at.device != dev) return LA_ERR_INVALID_ARG;
    return LA_OK;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    if (!a || !b) return false;
    uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

// sm_100 (B200 family) is required: kernels are built for sm_100a only.
la_status check_device(int* dev_out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return LA_ERR_CUDA; }
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cudaGetLastError();
        return LA_ERR_CUDA;
    }
    if (major != 10 || minor != 0) return LA_ERR_UNSUPPORTED;
    *dev_out = dev;
    return LA_OK;
}

// LA_SCAN_FORCE_SIMT=1 in the environment routes every call to the float32
// SIMT kernel (used by tests to compare the two kernel paths).
bool force_simt() {
    const char* e = std::getenv("LA_SCAN_FORCE_SIMT");
    return e && e[0] == '1';
}

// Calls with a fused input preparation take the single-kernel path (GDN) or
// the SIMT kernel, never the three-kernel or wide paths.
bool use_tc(const ScanArgs& a) { return !force_simt() && tc_eligible(a) && !a.has_prep; }

// The reversed scan and the per-token gate run on the three-kernel tensor-core
// path or the SIMT kernel.
// So do the interval composites (one chunk, chain on 2 BH blocks).
bool special(const ScanArgs& a) {
    return a.rev_chunk != 0 || a.beta_tok != nullptr || a.trans_out != nullptr || a.has_prep;
}

// The wide path also takes the reversed scan (its chunk resets are a zero decay
// at each chunk's first step, so its pipeline chunks need not align) and the
// per-token gate (sqrt(beta) row scaling in the gram kernel), GDN only.
bool use_wide(const ScanArgs& a) {
    if (force_simt() || !wide_eligible(a)) return false;
    if (a.rev_chunk || a.beta_tok)     // reversed scan, per-token gate (GDN)
        return a.mode == LA_MODE_GDN && !(a.rev_chunk && a.beta_tok) && !a.trans_out && !a.has_prep;
    return !special(a);
}

// LA_SCAN_NO_FUSE=1 keeps tensor-core calls on the three-kernel path (tests
// compare the two).
bool use_fused(const ScanArgs& a) {
    const char* e = std::getenv("LA_SCAN_NO_FUSE");
    if (e && e[0] == '1') return false;
    if (a.has_prep)
        return !force_simt() && tc_eligible(a) && a.mode == LA_MODE_GDN && a.rev_chunk == 0 &&
               !a.beta_tok && !a.trans_out && fused_eligible(a) && fused_prep_fits(a);
    // the reversed scan and the per-token gate (GDN) run in the fused kernel too
    if (a.rev_chunk || a.beta_tok)
        return use_tc(a) && a.mode == LA_MODE_GDN && !a.trans_out && fused_eligible(a);
    return use_tc(a) && !special(a) && fused_eligible(a);
}

size_t workspace_needed(const ScanArgs& a) {
    if (use_fused(a)) return fused_workspace_bytes(a);
    if (use_tc(a)) return tc_workspace_bytes(a);
    return use_wide(a) ? wide_workspace_bytes(a) : simt_workspace_bytes(a);
}

// The fused input preparation's own arguments (no CUDA call).
la_status validate_prep(const ScanArgs& a) {
    const la_prep& p = a.prep;
    if (!(std::isfinite(p.norm_eps) && p.norm_eps >= 0.f)) return LA_ERR_INVALID_ARG;
    if (p.frame_offset < 0 || (double)p.frame_offset + a.F > 16777216.0) return LA_ERR_INVALID_ARG;
    if (p.rope) {
        if (!(std::isfinite(p.rope_base) && p.rope_base > 1.f)) return LA_ERR_INVALID_ARG;
        if (p.grid_h < 1 || p.grid_w < 1 || (long long)p.grid_h * p.grid_w != a.S)
            return LA_ERR_INVALID_ARG;
    }
    return LA_OK;
}

// Validation common to every entry point.  `need_q` is false for a state step.
la_status validate(const ScanArgs& a, bool need_q) {
    if (a.B < 1 || a.H < 1 || a.F < 0 || a.S < 1) return LA_ERR_INVALID_ARG;
    if (a.B > 65535 || a.H > 65535) return LA_ERR_INVALID_ARG;
    if (!shape_supported(a.D)) return LA_ERR_UNSUPPORTED;
    const double elems = (double)a.B * a.H * a.F * a.S * a.D;
    if (elems > 9.0e15) return LA_ERR_INVALID_ARG;
    if (a.mode == LA_MODE_RELU && !(std::isfinite(a.eps) && a.eps >= 0.f)) return LA_ERR_INVALID_ARG;
    if (a.mode == LA_MODE_GDN && !std::isfinite(a.k_scale)) return LA_ERR_INVALID_ARG;
    if (a.has_prep) {
        const la_status ps = validate_prep(a);
        if (ps != LA_OK) return ps;
    }
    if (!a.ws) return LA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(a.ws) & 255u) != 0) return LA_ERR_INVALID_ARG;
    if (a.ws_bytes < workspace_needed(a)) return LA_ERR_INVALID_ARG;
    if (a.F > 0) {
        if (!a.k || !a.v) return LA_ERR_INVALID_ARG;
        if (need_q && (!a.q || !a.o)) return LA_ERR_INVALID_ARG;
        if (a.mode == LA_MODE_GDN && (!a.alpha || (!a.beta && !a.beta_tok)))
            return LA_ERR_INVALID_ARG;
    }
    int dev = 0;
    la_status s = check_device(&dev);
    if (s != LA_OK) return s;
    const void* ptrs[] = {a.q, a.k, a.v, a.o, a.alpha, a.beta, a.beta_tok, a.state_in, a.z_in,
                          a.state_out, a.z_out, a.trans_out, a.ws,
                          a.has_prep ? a.prep.q_weight : nullptr,
                          a.has_prep ? a.prep.k_weight : nullptr};
    for (const void* p : ptrs)
        if ((s = check_ptr(p, dev)) != LA_OK) return s;
    if (a.o) {
        const size_t n = (size_t)a.B * a.H * a.F * a.S * a.D * (a.bf16 ? 2 : 4);
        if (overlaps(a.o, n, a.q, n) || overlaps(a.o, n, a.k, n) || overlaps(a.o, n, a.v, n))
            return LA_ERR_INVALID_ARG;
    }
    return LA_OK;
}

la_status run(const ScanArgs& a, cudaStream_t st) {
    // Reset the device status word recorded in the workspace header.
    if (cudaMemsetAsync(a.ws, 0, kWsHeaderBytes, st) != cudaSuccess) {
        cudaGetLastError();
        return LA_ERR_CUDA;
    }
    cudaError_t e = use_fused(a) ? launch_fused(a, st)
                    : use_tc(a)  ? launch_tc(a, st)
                    : use_wide(a) ? launch_wide(a, st)
                                  : launch_simt(a, st);
    if (e != cudaSuccess) { cudaGetLastError(); return LA_ERR_CUDA; }
    return LA_OK;
}

// Arguments of a size or plan query for `mode`: the variants are marked by
// non-NULL placeholders that are never dereferenced.
void mark_mode(ScanArgs& a, la_mode mode) {
    a.mode = (mode == LA_MODE_RELU || mode == LA_MODE_RELU_PREP) ? LA_MODE_RELU : LA_MODE_GDN;
    if (mode == LA_MODE_GDN_PREP || mode == LA_MODE_RELU_PREP) {
        // sizes and plans assume a grid whose RoPE tables fit the fused kernel
        a.has_prep = 1;
        a.prep.rope = 1;
        a.prep.grid_h = 1;
        a.prep.grid_w = 1;
        a.prep.rope_base = 10000.f;
    }
    a.rev_chunk = mode == LA_MODE_GDN_REVERSE ? 1 : 0;
    if (mode == LA_MODE_GDN_TOKEN_BETA) a.beta_tok = reinterpret_cast<const float*>(uintptr_t(16));
    if (mode == LA_MODE_GDN_COMPOSITE) a.trans_out = reinterpret_cast<float*>(uintptr_t(16));
}

ScanArgs base_args(const void* k, const void* v, la_dtype dt, int B, int H, int F, int S, int D,
                   void* ws, size_t wsb) {
    ScanArgs a;
    std::memset(&a, 0, sizeof(a));
    a.k = k; a.v = v;
    a.bf16 = (dt == LA_BF16);
    a.B = B; a.H = H; a.F = F; a.S = S; a.D = D;
    a.ws = ws; a.ws_bytes = wsb;
    a.k_scale = 1.f;
    return a;
}

}  // namespace
}  // namespace la

using namespace la;

extern "C" la_status la_scan_relu(const void* q, const void* k, const void* v, void* o, la_dtype dt,
                                  const float* state_in, const float* z_in,
                                  float* state_out, float* z_out,
                                  int B, int H, int F, int S, int D, float eps,
                                  void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    if (dt != LA_F32 && dt != LA_BF16) return LA_ERR_INVALID_ARG;
    ScanArgs a = base_args(k, v, dt, B, H, F, S, D, workspace, workspace_bytes);
    a.q = q; a.o = o; a.mode = LA_MODE_RELU; a.eps = eps;
    a.state_in = state_in; a.z_in = z_in; a.state_out = state_out; a.z_out = z_out;
    la_status s = validate(a, true);
    if (s != LA_OK) return s;
    return run(a, stream);
}

extern "C" la_status la_scan_gdn(const void* q, const void* k, const void* v, void* o, la_dtype dt,
                                 const float* alpha, const float* beta, float k_scale,
                                 const float* state_in, float* state_out,
                                 int B, int H, int F, int S, int D,
                                 void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    if (dt != LA_F32 && dt != LA_BF16) return LA_ERR_INVALID_ARG;
    ScanArgs a = base_args(k, v, dt, B, H, F, S, D, workspace, workspace_bytes);
    a.q = q; a.o = o; a.mode = LA_MODE_GDN; a.k_scale = k_scale;
    a.alpha = alpha; a.beta = beta; a.state_in = state_in; a.state_out = state_out;
    la_status s = validate(a, true);
    if (s != LA_OK) return s;
    return run(a, stream);
}

extern "C" la_status la_scan_gdn_prep(const void* q, const void* k, const void* v, void* o,
                                      la_dtype dt, const float* alpha, const float* beta,
                                      float k_scale, const la_prep* prep,
                                      const float* state_in, float* state_out,
                                      int B, int H, int F, int S, int D,
                                      void* workspace, size_t workspace_bytes,
                                      cudaStream_t stream) {
    if (dt != LA_F32 && dt != LA_BF16) return LA_ERR_INVALID_ARG;
    if (!prep) return LA_ERR_INVALID_ARG;
    ScanArgs a = base_args(k, v, dt, B, H, F, S, D, workspace, workspace_bytes);
    a.q = q; a.o = o; a.mode = LA_MODE_GDN; a.k_scale = k_scale;
    a.alpha = alpha; a.beta = beta; a.state_in = state_in; a.state_out = state_out;
    a.has_prep = 1;
    a.prep = *prep;
    la_status s = validate(a, true);
    if (s != LA_OK) return s;
    return run(a, stream);
}

extern "C" la_status la_scan_relu_prep(const void* q, const void* k, const void* v, void* o,
                                       la_dtype dt, const la_prep* prep,
                                       const float* state_in, const float* z_in,
                                       float* state_out, float* z_out,
                                       int B, int H, int F, int S, int D, float eps,
                                       void* workspace, size_t workspace_bytes,
                                       cudaStream_t stream) {
    if (dt != LA_F32 && dt != LA_BF16) return LA_ERR_INVALID_ARG;
    if (!prep) return LA_ERR_INVALID_ARG;
    ScanArgs a = base_args(k, v, dt, B, H, F, S, D, workspace, workspace_bytes);
    a.q = q; a.o = o; a.mode = LA_MODE_RELU; a.eps = eps;
    a.state_in = state_in; a.z_in = z_in; a.state_out = state_out; a.z_out = z_out;
    a.has_prep = 1;
    a.prep = *prep;
    la_status s = validate(a, true);
    if (s != LA_OK) return s;
    return run(a, stream);
}

extern "C" la_status la_scan_gdn_reverse(const void* q, const void* k, const void* v, void* o,
                                         la_dtype dt, const float* alpha, const float* beta,
                                         float k_scale, int chunk_frames,
                                         int B, int H, int F, int S, int D,
                                         void* workspace, size_t workspace_bytes,
                                         cudaStream_t stream) {
    if (dt != LA_F32 && dt != LA_BF16) return LA_ERR_INVALID_ARG;
    if (chunk_frames < 1) return LA_ERR_INVALID_ARG;
    ScanArgs a = base_args(k, v, dt, B, H, F, S, D, workspace, workspace_bytes);
    a.q = q; a.o = o; a.mode = LA_MODE_GDN; a.k_scale = k_scale;
    a.alpha = alpha; a.beta = beta;
    a.rev_chunk = chunk_frames;
    la_status s = validate(a, true);
    if (s != LA_OK) return s;
    return run(a, stream);
}

extern "C" la_status la_scan_gdn_token_beta(const void* q, const void* k, const void* v, void* o,
                                            la_dtype dt, const float* alpha,
                                            const float* beta_token, float k_scale,
                                            const float* state_in, float* state_out,
                                            int B, int H, int F, int S, int D,
                                            void* workspace, size_t workspace_bytes,
                                            cudaStream_t stream) {
    if (dt != LA_F32 && dt != LA_BF16) return LA_ERR_INVALID_ARG;
    if (F > 0 && !beta_token) return LA_ERR_INVALID_ARG;
    ScanArgs a = base_args(k, v, dt, B, H, F, S, D, workspace, workspace_bytes);
    a.q = q; a.o = o; a.mode = LA_MODE_GDN; a.k_scale = k_scale;
    a.alpha = alpha; a.beta_tok = beta_token;
    a.state_in = state_in; a.state_out = state_out;
    la_status s = validate(a, true);
    if (s != LA_OK) return s;
    return run(a, stream);
}

extern "C" la_status la_state_step(la_mode mode, const void* k, const void* v, la_dtype dt,
                                   const float* alpha, const float* beta, float k_scale,
                                   const float* state_in, const float* z_in,
                                   float* state_out, float* z_out,
                                   int B, int H, int F, int S, int D,
                                   void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    if (dt != LA_F32 && dt != LA_BF16) return LA_ERR_INVALID_ARG;
    if (mode != LA_MODE_RELU && mode != LA_MODE_GDN) return LA_ERR_INVALID_ARG;
    ScanArgs a = base_args(k, v, dt, B, H, F, S, D, workspace, workspace_bytes);
    a.mode = mode;
    a.state_in = state_in; a.state_out = state_out;
    if (mode == LA_MODE_GDN) {
        a.alpha = alpha; a.beta = beta; a.k_scale = k_scale;
    } else {
        a.z_in = z_in; a.z_out = z_out;
    }
    la_status s = validate(a, false);
    if (s != LA_OK) return s;
    return run(a, stream);
}

extern "C" la_status la_gdn_interval_composite(const void* k, const void* v, la_dtype dt,
                                               const float* alpha, const float* beta,
                                               float k_scale, float* transition_out,
                                               float* input_out, int B, int H, int F, int S,
                                               int D, void* workspace, size_t workspace_bytes,
                                               cudaStream_t stream) {
    if (dt != LA_F32 && dt != LA_BF16) return LA_ERR_INVALID_ARG;
    if (!transition_out || !input_out) return LA_ERR_INVALID_ARG;
    ScanArgs a = base_args(k, v, dt, B, H, F, S, D, workspace, workspace_bytes);
    a.mode = LA_MODE_GDN;
    a.alpha = alpha; a.beta = beta; a.k_scale = k_scale;
    a.state_out = input_out;
    a.trans_out = transition_out;
    if (B > 0 && H > 0 && D > 0) {
        const size_t n = (size_t)B * H * D * D * sizeof(float);
        if (overlaps(transition_out, n, input_out, n)) return LA_ERR_INVALID_ARG;
    }
    const la_status s = validate(a, false);
    if (s != LA_OK) return s;
    return run(a, stream);
}

extern "C" la_status la_gdn_compose_prefix(const float* transitions, const float* inputs,
                                           size_t interval_stride, const float* state_in,
                                           float* starts_out, float* state_out, int n, int B,
                                           int H, int D, cudaStream_t stream) {
    if (n < 1 || B < 1 || H < 1 || B > 65535 || H > 65535) return LA_ERR_INVALID_ARG;
    if ((double)B * H > 65535.0) return LA_ERR_INVALID_ARG;
    if (!shape_supported(D)) return LA_ERR_UNSUPPORTED;
    if (!transitions || !inputs || !starts_out) return LA_ERR_INVALID_ARG;
    const size_t one_n = (size_t)B * H * D * D;              // floats of one [B, H, D, D]
    if (interval_stride < one_n) return LA_ERR_INVALID_ARG;
    int dev = 0;
    la_status s = check_device(&dev);
    if (s != LA_OK) return s;
    const void* ptrs[] = {transitions, inputs, state_in, starts_out, state_out};
    for (const void* p : ptrs)
        if ((s = check_ptr(p, dev)) != LA_OK) return s;
    const size_t one = one_n * sizeof(float);
    const size_t span = ((size_t)(n - 1) * interval_stride + one_n) * sizeof(float);
    const size_t all = one * n;
    const void* ins[] = {transitions, inputs, state_in};
    const size_t in_n[] = {span, span, one};
    for (int i = 0; i < 3; ++i)
        if (overlaps(starts_out, all, ins[i], in_n[i]) || overlaps(state_out, one, ins[i], in_n[i]))
            return LA_ERR_INVALID_ARG;
    if (overlaps(starts_out, all, state_out, one)) return LA_ERR_INVALID_ARG;
    if (launch_compose_prefix(transitions, inputs, interval_stride, state_in, starts_out,
                              state_out, n, B, H, D, stream) != cudaSuccess) {
        cudaGetLastError();
        return LA_ERR_CUDA;
    }
    return LA_OK;
}

extern "C" size_t la_workspace_size(la_mode mode, int B, int H, int F, int S, int D) {
    if (B < 1 || H < 1 || F < 0 || S < 1 || !shape_supported(D)) return 0;
    if (mode < LA_MODE_RELU || mode > LA_MODE_RELU_PREP) return 0;
    ScanArgs a = base_args(nullptr, nullptr, LA_BF16, B, H, F, S, D, nullptr, 0);
    mark_mode(a, mode);
    size_t n = workspace_needed(a);
    a.bf16 = 0;
    size_t n32 = workspace_needed(a);
    return n > n32 ? n : n32;
}

extern "C" la_status la_query_device_status(void* workspace, cudaStream_t stream) {
    if (!workspace) return LA_ERR_INVALID_ARG;
    if (cudaStreamSynchronize(stream) != cudaSuccess) { cudaGetLastError(); return LA_ERR_CUDA; }
    unsigned int status = 0;
    if (cudaMemcpy(&status, workspace, sizeof(status), cudaMemcpyDeviceToHost) != cudaSuccess) {
        cudaGetLastError();
        return LA_ERR_CUDA;
    }
    return status == 0 ? LA_OK : (la_status)status;
}

extern "C" const char* la_plan(la_mode mode, la_dtype dt, int B, int H, int F, int S, int D,
                               int* kernels) {
    if (B < 1 || H < 1 || F < 0 || S < 1 || !shape_supported(D)) return nullptr;
    if (mode < LA_MODE_RELU || mode > LA_MODE_RELU_PREP || (dt != LA_F32 && dt != LA_BF16))
        return nullptr;
    ScanArgs a = base_args(nullptr, nullptr, dt, B, H, F, S, D, nullptr, 0);
    mark_mode(a, mode);
    if (mode != LA_MODE_GDN_COMPOSITE)
        a.o = reinterpret_cast<void*>(uintptr_t(1));    // a scan (with outputs)
    if (use_fused(a)) {
        if (kernels) *kernels = 1;
        return "tcgen05_fused";
    }
    if (use_tc(a)) {
        if (kernels) *kernels = tc_kernel_count(a);
        return "tcgen05";
    }
    if (use_wide(a)) {
        if (kernels) *kernels = wide_kernel_count(a);
        return "tcgen05_wide";
    }
    if (kernels) *kernels = simt_kernel_count(a);
    return "simt_f32";
}

extern "C" const char* la_status_string(la_status s) {
    switch (s) {
        case LA_OK: return "LA_OK";
        case LA_ERR_INVALID_ARG: return "LA_ERR_INVALID_ARG";
        case LA_ERR_UNSUPPORTED: return "LA_ERR_UNSUPPORTED";
        case LA_ERR_CUDA: return "LA_ERR_CUDA";
        case LA_ERR_TIMEOUT: return "LA_ERR_TIMEOUT";
    }
    return "LA_ERR_UNKNOWN";
}
