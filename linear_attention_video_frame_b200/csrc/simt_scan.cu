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
    int M, K, Kn, V, U, z, den;
    int total;
};

// Kn holds the unrotated features of a tile (ReLU with RoPE: the normaliser
// reads them, the numerator the rotated ones in K).
__host__ __device__ inline SimtSmem simt_smem(int D, bool kn) {
    SimtSmem s;
    s.M = 0;                    // [D][kDJ]
    s.K = s.M + D * kDJ;        // [kT][D]   keys (GDN: scaled) or queries
    s.Kn = s.K + kT * D;        // [kT][D]   unrotated features (ReLU with RoPE)
    s.V = s.Kn + (kn ? kT * D : 0);   // [kT][kDJ]
    s.U = s.V + kT * kDJ;       // [kT][kDJ] residual (GDN)
    s.z = s.U + kT * kDJ;       // [D]       normaliser (ReLU)
    s.den = s.z + D;            // [kT]
    s.total = s.den + kT;
    return s;
}

__host__ __device__ inline bool simt_needs_kn(const ScanArgs& a) {
    return a.has_prep && a.prep.rope && a.mode == LA_MODE_RELU;
}

// Fused input preparation of a tile of raw rows x[t][D] (t < nt, tokens
// t0 .. t0 + nt - 1 of frame f): RMSNorm with weight w (NULL = ones), ReLU,
// then (prep.rope) 3D RoPE, and finally a factor `post` (the GDN key scale).
// x receives the prepared rows; xn (if not NULL) the unrotated ones.  Eight
// threads share a row (D / 8 consecutive channels each, an even count).
__device__ void simt_prep_rows(const ScanArgs& a, float* x, float* xn, int nt, int t0, int f,
                               const float* w, float post) {
    const int D = a.D, tid = threadIdx.x;
    const int row = tid >> 3, part = tid & 7, span = D / 8, c0 = part * span;
    const bool live = row < nt;
    float ss = 0.f;
    if (live)
        for (int c = c0; c < c0 + span; ++c) ss = fmaf(x[row * D + c], x[row * D + c], ss);
    ss += __shfl_xor_sync(0xffffffffu, ss, 1);
    ss += __shfl_xor_sync(0xffffffffu, ss, 2);
    ss += __shfl_xor_sync(0xffffffffu, ss, 4);
    if (!live) {               // rows past the frame's last token stay zero in both copies
        if (xn)
            for (int c = c0; c < c0 + span; ++c) xn[row * D + c] = 0.f;
        return;
    }
    const float r = rsqrtf(ss / (float)D + a.prep.norm_eps);
    const int nt_p = rope_nt(D), nhw = rope_nhw(D);
    const int s = t0 + row;
    const double l2b = log2((double)a.prep.rope_base);
    for (int c = c0; c < c0 + span; c += 2) {
        float y0 = x[row * D + c] * r * (w ? w[c] : 1.f);
        float y1 = x[row * D + c + 1] * r * (w ? w[c + 1] : 1.f);
        y0 = fmaxf(y0, 0.f);
        y1 = fmaxf(y1, 0.f);
        if (xn) {
            xn[row * D + c] = y0;
            xn[row * D + c + 1] = y1;
        }
        if (a.prep.rope) {
            const int i = c / 2;
            int pos, ig, n;
            if (i < nt_p) { pos = a.prep.frame_offset + f; ig = i; n = nt_p; }
            else if (i < nt_p + nhw) { pos = s / a.prep.grid_w; ig = i - nt_p; n = nhw; }
            else { pos = s % a.prep.grid_w; ig = i - nt_p - nhw; n = nhw; }
            float cs, sn;
            rope_cos_sin(pos, ig, n, l2b, cs, sn);
            const float r0 = y0 * cs - y1 * sn, r1 = y0 * sn + y1 * cs;
            y0 = r0;
            y1 = r1;
        }
        x[row * D + c] = y0 * post;
        x[row * D + c + 1] = y1 * post;
    }
}

__global__ void __launch_bounds__(kThreads)
simt_scan_kernel(ScanArgs a) {
    extern __shared__ float smem[];
    const int D = a.D, S = a.S, F = a.F;
    const bool kn = simt_needs_kn(a);
    const SimtSmem L = simt_smem(D, kn);
    float* sM = smem + L.M;
    float* sK = smem + L.K;
    float* sKn = kn ? smem + L.Kn : sK;     // features the normaliser reads (ReLU)
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
                sK[i] = a.has_prep ? x : (relu ? fmaxf(x, 0.f) : x * a.k_scale);
            }
            if (a.has_prep) {
                __syncthreads();
                simt_prep_rows(a, sK, kn ? sKn : nullptr, nt, t0, f,
                               a.prep.k_weight ? a.prep.k_weight + (size_t)h * D : nullptr,
                               relu ? 1.f : a.k_scale);
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
                for (int t = 0; t < kT; ++t) s += sKn[t * D + tid];
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
                    sK[i] = (relu && !a.has_prep) ? fmaxf(x, 0.f) : x;
                }
                __syncthreads();
                if (a.has_prep) {
                    simt_prep_rows(a, sK, kn ? sKn : nullptr, nt, t0, f,
                                   a.prep.q_weight ? a.prep.q_weight + (size_t)h * D : nullptr,
                                   1.f);
                    __syncthreads();
                }
                if (relu && tid < kT) {
                    float s = 0.f;
                    for (int d = 0; d < D; ++d) s = fmaf(sKn[tid * D + d], sz[d], s);
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
    const size_t smem = (size_t)simt_smem(a.D, simt_needs_kn(a)).total * sizeof(float);
    cudaError_t e = cudaFuncSetAttribute(simt_scan_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid((a.D + kDJ - 1) / kDJ, a.H, a.B * (a.trans_out ? 2 : 1));
    simt_scan_kernel<<<grid, kThreads, smem, st>>>(a);
    return cudaGetLastError();
}

}  // namespace la
