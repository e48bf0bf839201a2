// la_scan_host: the frame-wise scan over q, k, v, o held in HOST memory.
//
// A video clip is scanned frame chunk by frame chunk.  The recurrent state is
// what carries the causal dependency from one chunk to the next (the
// chunk-causal rollout of the SANA-WM paper summary, section 3, and the
// block KV cache of the SANA-Video talk), so the clip never has to be
// resident on the GPU as a whole.  Three streams form a pipeline over a ring
// of device slots:
//
//   copy-in stream   H2D of chunk c+1 (q, k, v and the gates)
//   caller's stream  the scan of chunk c, state carried in place
//   copy-out stream  D2H of chunk c-1's output
//
// PCIe is full duplex and the scan of a chunk takes a small fraction of its
// transfer time, so a call costs about the larger of the two transfers plus
// one chunk of fill and drain, instead of their sum.
//
// Every input row of a chunk is one (b, h) pair: n frames of S*D elements,
// contiguous in the host array with a pitch of F*S*D elements.  A chunk moves
// as one 2-D copy of B*H rows into a dense [B, H, n, S, D] device slot, which
// is the layout la_scan_relu / la_scan_gdn take.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>

#include "common.cuh"

namespace la {
namespace {

constexpr int kSlots = 3;
constexpr int kMaxDevices = 64;
constexpr int kAutoChunks = 16;     // chunk count aimed at when chunk_frames <= 0

// Streams and events of one device, made on first use and kept until exit.
struct HostCtx {
    bool ready = false;
    cudaStream_t h2d = nullptr, d2h = nullptr;
    cudaEvent_t start = nullptr, end = nullptr;
    cudaEvent_t in[kSlots] = {}, comp[kSlots] = {}, out[kSlots] = {};
    size_t max_pitch = 0;
};

std::mutex g_mu[kMaxDevices];
HostCtx g_ctx[kMaxDevices];

cudaError_t init_ctx(HostCtx& c, int dev) {
    if (c.ready) return cudaSuccess;
    cudaError_t e = cudaStreamCreateWithFlags(&c.h2d, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&c.d2h, cudaStreamNonBlocking);
    cudaEvent_t* evs[] = {&c.start, &c.end};
    for (cudaEvent_t* p : evs)
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(p, cudaEventDisableTiming);
    for (int i = 0; i < kSlots && e == cudaSuccess; ++i) {
        e = cudaEventCreateWithFlags(&c.in[i], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c.comp[i], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c.out[i], cudaEventDisableTiming);
    }
    int mp = 0;
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&mp, cudaDevAttrMaxPitch, dev);
    if (e != cudaSuccess) return e;     // partial objects stay until exit; the next call retries
    c.max_pitch = (size_t)mp;
    c.ready = true;
    return cudaSuccess;
}

// Host memory: page-locked (registered) or ordinary pageable memory.
bool is_host_ptr(const void* p) {
    if (!p) return true;
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
        cudaGetLastError();
        return false;
    }
    return at.type == cudaMemoryTypeHost || at.type == cudaMemoryTypeUnregistered;
}

bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
    if (!a || !b) return false;
    uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
    return x < y + nb && y < x + na;
}

int chunk_of(int F, int chunk_frames) {
    if (chunk_frames > 0) return std::min(chunk_frames, std::max(F, 1));
    return std::max(1, (F + kAutoChunks - 1) / kAutoChunks);
}

// Byte layout of the device workspace.  The scan workspace comes first so
// that la_query_device_status works on the host-call workspace unchanged.
struct HostLayout {
    size_t scan, state, z, slot_q, slot_a, slot, total;
    size_t off_state, off_z, off_slots;
    int n;                      // frames per chunk
};

bool host_layout(la_mode mode, la_dtype dt, int B, int H, int F, int S, int D, int chunk_frames,
                 HostLayout* L) {
    const int n = chunk_of(F, chunk_frames);
    const size_t scan = la_workspace_size(mode, B, H, n, S, D);
    if (scan == 0) return false;
    const size_t esz = dt == LA_BF16 ? 2 : 4;
    const size_t bh = (size_t)B * H;
    L->n = n;
    L->scan = align_up(scan, 256);
    L->state = align_up(bh * D * D * 4, 256);
    L->z = mode == LA_MODE_RELU ? align_up(bh * D * 4, 256) : 0;
    L->slot_q = align_up(bh * n * S * D * esz, 256);
    L->slot_a = mode == LA_MODE_GDN ? align_up(bh * n * 4, 256) : 0;
    L->slot = 4 * L->slot_q + 2 * L->slot_a;          // q, k, v, o, alpha, beta
    L->off_state = L->scan;
    L->off_z = L->off_state + L->state;
    L->off_slots = L->off_z + L->z;
    L->total = L->off_slots + (size_t)kSlots * L->slot;
    return true;
}

// B*H rows of `width` bytes: one 2-D copy when the pitches allow it, else
// one copy per row.
cudaError_t copy_rows(void* dst, size_t dpitch, const void* src, size_t spitch, size_t width,
                      size_t rows, size_t max_pitch, cudaStream_t s) {
    if (width == 0 || rows == 0) return cudaSuccess;
    if (dpitch == width && spitch == width)
        return cudaMemcpyAsync(dst, src, width * rows, cudaMemcpyDefault, s);
    if (dpitch <= max_pitch && spitch <= max_pitch)
        return cudaMemcpy2DAsync(dst, dpitch, src, spitch, width, rows, cudaMemcpyDefault, s);
    for (size_t r = 0; r < rows; ++r) {
        cudaError_t e = cudaMemcpyAsync(static_cast<char*>(dst) + r * dpitch,
                                        static_cast<const char*>(src) + r * spitch, width,
                                        cudaMemcpyDefault, s);
        if (e != cudaSuccess) return e;
    }
    return cudaSuccess;
}

struct HostArgs {
    la_mode mode;
    la_dtype dt;
    const void *q, *k, *v;
    void* o;
    const float *alpha, *beta;
    float k_scale, eps;
    const float *state_in, *z_in;
    float *state_out, *z_out;
    int B, H, F, S, D, chunk_frames;
    void* ws;
    size_t ws_bytes;
};

la_status validate_host(const HostArgs& a, HostLayout* L, int* dev_out) {
    if (a.dt != LA_F32 && a.dt != LA_BF16) return LA_ERR_INVALID_ARG;
    if (a.mode != LA_MODE_RELU && a.mode != LA_MODE_GDN) return LA_ERR_INVALID_ARG;
    if (a.B < 1 || a.H < 1 || a.F < 0 || a.S < 1) return LA_ERR_INVALID_ARG;
    if (!(a.D >= 16 && a.D <= 256 && a.D % 16 == 0)) return LA_ERR_UNSUPPORTED;
    if (!host_layout(a.mode, a.dt, a.B, a.H, a.F, a.S, a.D, a.chunk_frames, L))
        return LA_ERR_INVALID_ARG;
    if (a.mode == LA_MODE_RELU && !(std::isfinite(a.eps) && a.eps >= 0.f)) return LA_ERR_INVALID_ARG;
    if (a.mode == LA_MODE_GDN && !std::isfinite(a.k_scale)) return LA_ERR_INVALID_ARG;
    if (!a.ws || (reinterpret_cast<uintptr_t>(a.ws) & 255u) != 0) return LA_ERR_INVALID_ARG;
    if (a.ws_bytes < L->total) return LA_ERR_INVALID_ARG;
    if (a.F > 0) {
        if (!a.q || !a.k || !a.v || !a.o) return LA_ERR_INVALID_ARG;
        if (a.mode == LA_MODE_GDN && (!a.alpha || !a.beta)) return LA_ERR_INVALID_ARG;
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return LA_ERR_CUDA; }
    if (dev < 0 || dev >= kMaxDevices) return LA_ERR_UNSUPPORTED;
    int major = 0, minor = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess) {
        cudaGetLastError();
        return LA_ERR_CUDA;
    }
    if (major != 10 || minor != 0) return LA_ERR_UNSUPPORTED;   // kernels are built for sm_100a
    const void* host_ptrs[] = {a.q, a.k, a.v, a.o, a.alpha, a.beta,
                               a.state_in, a.z_in, a.state_out, a.z_out};
    for (const void* p : host_ptrs)
        if (!is_host_ptr(p)) return LA_ERR_INVALID_ARG;
    cudaPointerAttributes at;
    if (cudaPointerGetAttributes(&at, a.ws) != cudaSuccess) { cudaGetLastError(); return LA_ERR_INVALID_ARG; }
    if (at.type != cudaMemoryTypeDevice || at.device != dev) return LA_ERR_INVALID_ARG;
    const size_t n = (size_t)a.B * a.H * a.F * a.S * a.D * (a.dt == LA_BF16 ? 2 : 4);
    if (overlaps(a.o, n, a.q, n) || overlaps(a.o, n, a.k, n) || overlaps(a.o, n, a.v, n))
        return LA_ERR_INVALID_ARG;
    *dev_out = dev;
    return LA_OK;
}

// Enqueue the whole pipeline.  Returns the first failure; the caller's
// stream is joined with both copy streams in every case.
la_status enqueue(const HostArgs& a, const HostLayout& L, HostCtx& c, cudaStream_t st) {
    char* ws = static_cast<char*>(a.ws);
    float* state = reinterpret_cast<float*>(ws + L.off_state);
    float* z = a.mode == LA_MODE_RELU ? reinterpret_cast<float*>(ws + L.off_z) : nullptr;
    const size_t esz = a.dt == LA_BF16 ? 2 : 4;
    const size_t bh = (size_t)a.B * a.H;
    const size_t frame_bytes = (size_t)a.S * a.D * esz;
    const size_t state_bytes = bh * a.D * a.D * 4, z_bytes = bh * a.D * 4;

    la_status res = LA_OK;
    cudaError_t e = cudaSuccess;
    auto ok = [&](cudaError_t x) {
        if (x != cudaSuccess && e == cudaSuccess) e = x;
        return e == cudaSuccess;
    };

    // Nothing starts before the work already queued on the caller's stream
    // (it may still be producing the host inputs or using the workspace).
    ok(cudaEventRecord(c.start, st));
    ok(cudaStreamWaitEvent(c.h2d, c.start, 0));
    ok(cudaStreamWaitEvent(c.d2h, c.start, 0));
    const bool have_state = a.state_in != nullptr;
    const bool have_z = a.z_in != nullptr;
    if (have_state) ok(cudaMemcpyAsync(state, a.state_in, state_bytes, cudaMemcpyDefault, c.h2d));
    if (have_z) ok(cudaMemcpyAsync(z, a.z_in, z_bytes, cudaMemcpyDefault, c.h2d));

    const int nchunks = a.F == 0 ? 1 : (a.F + L.n - 1) / L.n;
    for (int ci = 0; ci < nchunks && e == cudaSuccess && res == LA_OK; ++ci) {
        const int slot = ci % kSlots;
        const int f0 = ci * L.n;
        const int nf = std::min(L.n, a.F - f0);          // 0 only when F == 0
        char* sb = ws + L.off_slots + (size_t)slot * L.slot;
        void* dq = sb;
        void* dk = sb + L.slot_q;
        void* dv = sb + 2 * L.slot_q;
        void* dout = sb + 3 * L.slot_q;
        float* dal = reinterpret_cast<float*>(sb + 4 * L.slot_q);
        float* dbe = reinterpret_cast<float*>(sb + 4 * L.slot_q + L.slot_a);

        // copy-in: the slot's inputs are free once chunk ci - kSlots was scanned
        if (ci >= kSlots) ok(cudaStreamWaitEvent(c.h2d, c.comp[slot], 0));
        const size_t w = (size_t)nf * frame_bytes, sp = (size_t)a.F * frame_bytes;
        const size_t off = (size_t)f0 * frame_bytes;
        ok(copy_rows(dq, w, static_cast<const char*>(a.q) + off, sp, w, bh, c.max_pitch, c.h2d));
        ok(copy_rows(dk, w, static_cast<const char*>(a.k) + off, sp, w, bh, c.max_pitch, c.h2d));
        ok(copy_rows(dv, w, static_cast<const char*>(a.v) + off, sp, w, bh, c.max_pitch, c.h2d));
        if (a.mode == LA_MODE_GDN) {
            const size_t gw = (size_t)nf * 4, gp = (size_t)a.F * 4;
            ok(copy_rows(dal, gw, a.alpha + f0, gp, gw, bh, c.max_pitch, c.h2d));
            ok(copy_rows(dbe, gw, a.beta + f0, gp, gw, bh, c.max_pitch, c.h2d));
        }
        ok(cudaEventRecord(c.in[slot], c.h2d));

        // scan: needs the slot's inputs, and its output buffer drained
        ok(cudaStreamWaitEvent(st, c.in[slot], 0));
        if (ci >= kSlots) ok(cudaStreamWaitEvent(st, c.out[slot], 0));
        if (e != cudaSuccess) break;
        const bool carry = ci > 0 || have_state;
        if (a.mode == LA_MODE_GDN) {
            res = la_scan_gdn(dq, dk, dv, dout, a.dt, dal, dbe, a.k_scale,
                              carry ? state : nullptr, state, a.B, a.H, nf, a.S, a.D,
                              a.ws, L.scan, st);
        } else {
            const bool carry_z = ci > 0 || have_z;
            res = la_scan_relu(dq, dk, dv, dout, a.dt, carry ? state : nullptr,
                               carry_z ? z : nullptr, state, z, a.B, a.H, nf, a.S, a.D, a.eps,
                               a.ws, L.scan, st);
        }
        ok(cudaEventRecord(c.comp[slot], st));

        // copy-out of this chunk's output
        ok(cudaStreamWaitEvent(c.d2h, c.comp[slot], 0));
        ok(copy_rows(static_cast<char*>(a.o) + off, sp, dout, w, w, bh, c.max_pitch, c.d2h));
        ok(cudaEventRecord(c.out[slot], c.d2h));
    }
    // Final state after the last chunk (ordered behind it on the copy-out stream).
    if (e == cudaSuccess && res == LA_OK) {
        if (a.state_out) ok(cudaMemcpyAsync(a.state_out, state, state_bytes, cudaMemcpyDefault, c.d2h));
        if (a.z_out) ok(cudaMemcpyAsync(a.z_out, z, z_bytes, cudaMemcpyDefault, c.d2h));
    }
    // Join: the caller's stream continues after every copy of this call.
    cudaError_t j = cudaEventRecord(c.end, c.h2d);
    if (j == cudaSuccess) j = cudaStreamWaitEvent(st, c.end, 0);
    if (j == cudaSuccess) j = cudaEventRecord(c.end, c.d2h);
    if (j == cudaSuccess) j = cudaStreamWaitEvent(st, c.end, 0);
    if (res != LA_OK) return res;
    if (e != cudaSuccess || j != cudaSuccess) {
        cudaGetLastError();
        return LA_ERR_CUDA;
    }
    return LA_OK;
}

}  // namespace
}  // namespace la

using namespace la;

extern "C" size_t la_host_workspace_size(la_mode mode, la_dtype dt, int B, int H, int F, int S,
                                         int D, int chunk_frames) {
    if ((mode != LA_MODE_RELU && mode != LA_MODE_GDN) || (dt != LA_F32 && dt != LA_BF16)) return 0;
    if (B < 1 || H < 1 || F < 0 || S < 1) return 0;
    HostLayout L;
    if (!host_layout(mode, dt, B, H, F, S, D, chunk_frames, &L)) return 0;
    return L.total;
}

extern "C" int la_host_chunk_frames(int F, int chunk_frames) {
    if (F < 0) return 0;
    return chunk_of(F, chunk_frames);
}

extern "C" la_status la_scan_host(la_mode mode, const void* q, const void* k, const void* v,
                                  void* o, la_dtype dt, const float* alpha, const float* beta,
                                  float k_scale, float eps, const float* state_in,
                                  const float* z_in, float* state_out, float* z_out,
                                  int B, int H, int F, int S, int D, int chunk_frames,
                                  void* workspace, size_t workspace_bytes, cudaStream_t stream) {
    HostArgs a;
    std::memset(&a, 0, sizeof(a));
    a.mode = mode; a.dt = dt;
    a.q = q; a.k = k; a.v = v; a.o = o;
    a.k_scale = k_scale; a.eps = eps;
    a.state_in = state_in; a.state_out = state_out;
    if (mode == LA_MODE_RELU) {
        a.z_in = z_in;
        a.z_out = z_out;
    } else {
        a.alpha = alpha;
        a.beta = beta;
    }
    a.B = B; a.H = H; a.F = F; a.S = S; a.D = D; a.chunk_frames = chunk_frames;
    a.ws = workspace; a.ws_bytes = workspace_bytes;
    HostLayout L;
    int dev = 0;
    la_status s = validate_host(a, &L, &dev);
    if (s != LA_OK) return s;
    std::lock_guard<std::mutex> lock(g_mu[dev]);
    if (init_ctx(g_ctx[dev], dev) != cudaSuccess) {
        cudaGetLastError();
        return LA_ERR_CUDA;
    }
    return enqueue(a, L, g_ctx[dev], stream);
}
