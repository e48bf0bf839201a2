// Generic float32 SIMT scan: both modes, both storage types, every legal D.
//
// This is the path for float32 inputs (fp32 FMA keeps the 1e-4 parity bar
// that bf16 or tf32 tensor-core operands cannot meet) and for shapes the
// tensor-core path does not cover.  One block owns one (b, h) pair and a
// slice of kDJ state columns (the last slice may be partial): the value columns of the state are
// independent in both modes, so slices never talk to each other.
//
// GDN uses the residual form of the frame update, algebraically equal to
// the frame-wise Gated DeltaNet of the SANA-WM paper summary (section 3,
// "Hybrid GDN/Softmax Attention"):
//     M_f = alpha M_{f-1} + beta Kh^T (V - alpha Kh M_{f-1})
// which needs only the block's own columns of M, V and O.
// ReLU mode accumulates the additive block state and normaliser of the
// SANA-Video block KV cache (talk, block KV cache segment).  With
// rev_chunk > 0 the GDN frames are taken in the reversed, chunk-reset order
// of the SANA-WM paper summary (section 3, "Chunk-causal deployment").  With
// trans_out set (the interval composites of that summary's context-parallel
// training, appendix C.1) a second set of blocks runs the same GDN
// recurrence from the identity with V = 0, which leaves the transition
// composite A_F ... A_1; the first set, from a zero state, leaves the input
// composite.
#include "common.cuh"

namespace la {
namespace {

constexpr int kDJ = 32;        // state columns per block
constexpr int kT = 32;         // tokens per tile
constexpr int kThreads = 256;  // 8 warps
constexpr int kRowsPerPass = kThreads / kDJ;   // 8

struct SimtSmem {
    // offsets in floats
    int M, K, V, U, z, den;
    int total;
};

__host__ __device__ inline SimtSmem simt_smem(int D) {
    SimtSmem s;
    s.M = 0;                    // [D][kDJ]
    s.K = s.M + D * kDJ;        // [kT][D]   keys (GDN: scaled) or queries
    s.V = s.K + kT * D;         // [kT][kDJ]
    s.U = s.V + kT * kDJ;       // [kT][kDJ] residual (GDN)
    s.z = s.U + kT * kDJ;       // [D]       normaliser (ReLU)
    s.den = s.z + D;            // [kT]
    s.total = s.den + kT;
    return s;
}

__global__ void __launch_bounds__(kThreads)
simt_scan_kernel(ScanArgs a) {
    extern __shared__ float smem[];
    const int D = a.D, S = a.S, F = a.F;
    const SimtSmem L = simt_smem(D);
    float* sM = smem + L.M;
    float* sK = smem + L.K;
    float* sV = smem + L.V;
    float* sU = smem + L.U;
    float* sz = smem + L.z;
    float* sden = smem + L.den;

    const int j0 = blockIdx.x * kDJ;
    // With trans_out set, blocks z >= B compute the interval's transition
    // composite A_F ... A_1: the same recurrence from the identity with V = 0.
    const bool trans = a.trans_out && (int)blockIdx.z >= a.B;
    const int h = blockIdx.y, b = trans ? (int)blockIdx.z - a.B : (int)blockIdx.z;
    const int tid = threadIdx.x;
    const int jj = tid % kDJ;          // this thread's state column within the slice
    const int rr = tid / kDJ;          // row phase 0..7
    const bool relu = (a.mode == LA_MODE_RELU);
    const size_t bh = (size_t)b * a.H + h;

    // ---- initial state slice (and normaliser) ----
    for (int i = tid; i < D * kDJ; i += kThreads) {
        int d = i / kDJ, j = i % kDJ;
        if (trans) sM[i] = (d == j0 + j) ? 1.f : 0.f;
        else sM[i] = (a.state_in && j0 + j < D) ? a.state_in[(bh * D + d) * D + j0 + j] : 0.f;
    }
    if (relu)
        for (int d = tid; d < D; d += kThreads) sz[d] = a.z_in ? a.z_in[bh * D + d] : 0.f;
    __syncthreads();

    const int nacc = D / kRowsPerPass;      // <= 32 accumulators (D <= 256)
    for (int st = 0; st < F; ++st) {
        const int f = step_frame(st, F, a.rev_chunk);
        if (step_resets(st, a.rev_chunk)) {            // a new chunk of the reversed scan
            __syncthreads();
            for (int i = tid; i < D * kDJ; i += kThreads) sM[i] = 0.f;
            __syncthreads();
        }
        const size_t frame = (bh * F + f) * (size_t)S;   // first token row of the frame
        float al = 1.f, bt = 1.f;
        if (!relu) {
            al = a.alpha[bh * F + f];
            bt = a.beta_tok ? 1.f : a.beta[bh * F + f];   // per-token gates weigh U below
        }
        const float* btok = a.beta_tok ? a.beta_tok + (bh * F + f) * (size_t)S : nullptr;

        float acc[32];
#pragma unroll
        for (int r = 0; r < 32; ++r) acc[r] = 0.f;
        float dz = 0.f;

        // ---------------- state update over token tiles ----------------
        for (int t0 = 0; t0 < S; t0 += kT) {
            const int nt = min(kT, S - t0);
            for (int i = tid; i < kT * D; i += kThreads) {
                int t = i / D;
                float x = 0.f;
                if (t < nt) x = load_elem(a.k, (frame + t0) * D + i, a.bf16);
                sK[i] = relu ? fmaxf(x, 0.f) : x * a.k_scale;
            }
            for (int i = tid; i < kT * kDJ; i += kThreads) {
                int t = i / kDJ, j = i % kDJ;
                sV[i] = (!trans && t < nt && j0 + j < D)
                            ? load_elem(a.v, (frame + t0 + t) * D + j0 + j, a.bf16) : 0.f;
            }
            __syncthreads();
            const float* src = sV;
            if (!relu) {
                // U = V - alpha Kh M_{f-1}  (old state for the whole frame)
                for (int t = rr; t < kT; t += kRowsPerPass) {
                    float s = 0.f;
                    for (int d = 0; d < D; ++d) s = fmaf(sK[t * D + d], sM[d * kDJ + jj], s);
                    const float w = (btok && t < nt) ? btok[t0 + t] : 1.f;
                    sU[t * kDJ + jj] = w * (sV[t * kDJ + jj] - al * s);
                }
                __syncthreads();
                src = sU;
            }
            // acc[d, j] += sum_t K~[t, d] src[t, j]
#pragma unroll
            for (int r = 0; r < 32; ++r) {
                if (r < nacc) {
                    const int d = rr + r * kRowsPerPass;
                    float s = acc[r];
                    for (int t = 0; t < kT; ++t) s = fmaf(sK[t * D + d], src[t * kDJ + jj], s);
                    acc[r] = s;
                }
            }
            if (relu && tid < D) {
                float s = dz;
                for (int t = 0; t < kT; ++t) s += sK[t * D + tid];
                dz = s;
            }
            __syncthreads();
        }
        // ---------------- commit the frame's state ----------------
#pragma unroll
        for (int r = 0; r < 32; ++r) {
            if (r < nacc) {
                const int d = rr + r * kRowsPerPass;
                float& m = sM[d * kDJ + jj];
                m = relu ? (m + acc[r]) : fmaf(al, m, bt * acc[r]);
            }
        }
        if (relu && tid < D) sz[tid] += dz;
        __syncthreads();

        // ---------------- outputs: O_f = Q~_f M_f (ReLU: / (phi(Q) z + eps)) ----------------
        if (a.o) {
            for (int t0 = 0; t0 < S; t0 += kT) {
                const int nt = min(kT, S - t0);
                for (int i = tid; i < kT * D; i += kThreads) {
                    int t = i / D;
                    float x = 0.f;
                    if (t < nt) x = load_elem(a.q, (frame + t0) * D + i, a.bf16);
                    sK[i] = relu ? fmaxf(x, 0.f) : x;
                }
                __syncthreads();
                if (relu && tid < kT) {
                    float s = 0.f;
                    for (int d = 0; d < D; ++d) s = fmaf(sK[tid * D + d], sz[d], s);
                    sden[tid] = s + a.eps;
                }
                __syncthreads();
                for (int t = rr; t < nt; t += kRowsPerPass) {
                    float s = 0.f;
                    for (int d = 0; d < D; ++d) s = fmaf(sK[t * D + d], sM[d * kDJ + jj], s);
                    if (relu) s = s / sden[t];
                    if (j0 + jj < D) store_elem(a.o, (frame + t0 + t) * D + j0 + jj, s, a.bf16);
                }
                __syncthreads();
            }
        }
    }

    // ---- final state (or transition composite) ----
    float* out = trans ? a.trans_out : a.state_out;
    if (out)
        for (int i = tid; i < D * kDJ; i += kThreads) {
            int d = i / kDJ, j = i % kDJ;
            if (j0 + j < D) out[(bh * D + d) * D + j0 + j] = sM[i];
        }
    if (relu && a.z_out && blockIdx.x == 0)
        for (int d = tid; d < D; d += kThreads) a.z_out[bh * D + d] = sz[d];
}

}  // namespace

size_t simt_workspace_bytes(const ScanArgs&) { return kWsHeaderBytes; }

int simt_kernel_count(const ScanArgs&) { return 1; }

cudaError_t launch_simt(const ScanArgs& a, cudaStream_t st) {
    const size_t smem = (size_t)simt_smem(a.D).total * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(simt_scan_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((a.D + kDJ - 1) / kDJ, a.H, a.B * (a.trans_out ? 2 : 1));
    simt_scan_kernel<<<grid, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace la
