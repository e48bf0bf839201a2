// Exclusive prefix over GDN interval composites.
//
// SANA-WM paper summary (paperlayer), appendix C.1, context-parallel
// training: each rank summarises its frame interval r by a transition
// composite T_r and an input composite U_r; the gathered summaries are
// composed as an exclusive prefix, which gives every interval its exact
// initial state:
//     start_0 = M_0,   start_{r+1} = T_r start_r + U_r.
// The columns of the state never mix (T acts on the key dimension, the
// rows), so one block owns one (b, h) pair and a slice of kCJ value columns
// and carries that slice through the intervals in shared memory.  T_r is
// staged in 32-row tiles; a warp's 32 lanes share a row of T (broadcast)
// and own 32 consecutive columns of the state (conflict-free).  float32
// FMA throughout: this is D^3 work per interval and head, far off the hot
// path, and float32 keeps the exactness the prefix is for.
#include <utility>

#include "common.cuh"

namespace la {
namespace {

constexpr int kCJ = 32;                 // state columns per block
constexpr int kCThreads = 256;          // 8 warps
constexpr int kCRows = kCThreads / kCJ; // row phases (8)
constexpr int kTRows = 32;              // rows of T staged per tile

__host__ __device__ inline size_t compose_smem_floats(int D) {
    return 2 * (size_t)D * kCJ + (size_t)kTRows * D;
}

__global__ void __launch_bounds__(kCThreads)
compose_prefix_kernel(const float* __restrict__ T, const float* __restrict__ U, size_t stride,
                      const float* __restrict__ m0, float* __restrict__ starts,
                      float* __restrict__ mout, int n, int BH, int D) {
    extern __shared__ float sm[];
    float* cur = sm;                          // [D][kCJ] state slice before interval r
    float* nxt = cur + D * kCJ;               // [D][kCJ] after it
    float* sT = nxt + D * kCJ;                // [kTRows][D] rows of T_r
    const int j0 = blockIdx.x * kCJ;
    const size_t bh = blockIdx.y;
    const int tid = threadIdx.x, jj = tid % kCJ, rr = tid / kCJ;
    const size_t mat = (size_t)D * D;
    const bool col_live = j0 + jj < D;

    for (int i = tid; i < D * kCJ; i += kCThreads) {
        const int d = i / kCJ, j = i % kCJ;
        cur[i] = (m0 && j0 + j < D) ? m0[bh * mat + (size_t)d * D + j0 + j] : 0.f;
    }
    __syncthreads();
    for (int r = 0; r < n; ++r) {
        const size_t base = (size_t)r * stride + bh * mat;      // interval r in T and U
        const size_t sbase = ((size_t)r * BH + bh) * mat;       // interval r in starts
        for (int i = tid; i < D * kCJ; i += kCThreads) {
            const int d = i / kCJ, j = i % kCJ;
            if (j0 + j < D) starts[sbase + (size_t)d * D + j0 + j] = cur[i];
        }
        for (int d0 = 0; d0 < D; d0 += kTRows) {
            const int nrows = min(kTRows, D - d0);           // 16 or 32 (D % 16 == 0)
            for (int i = tid; i < nrows * D; i += kCThreads)
                sT[i] = T[base + (size_t)d0 * D + i];       // rows d0 .. d0 + nrows - 1
            __syncthreads();
#pragma unroll
            for (int q = 0; q < kTRows / kCRows; ++q) {
                const int dl = rr + q * kCRows;              // row within the tile
                if (dl >= nrows) break;
                const float* trow = sT + dl * D;
                float s = 0.f;
                for (int e = 0; e < D; ++e) s = fmaf(trow[e], cur[e * kCJ + jj], s);
                const size_t idx = base + (size_t)(d0 + dl) * D + j0 + jj;
                nxt[(d0 + dl) * kCJ + jj] = col_live ? s + U[idx] : 0.f;
            }
            __syncthreads();
        }
        float* t = cur;
        cur = nxt;
        nxt = t;
    }
    if (mout)
        for (int i = tid; i < D * kCJ; i += kCThreads) {
            const int d = i / kCJ, j = i % kCJ;
            if (j0 + j < D) mout[bh * mat + (size_t)d * D + j0 + j] = cur[i];
        }
}

}  // namespace

cudaError_t launch_compose_prefix(const float* T, const float* U, size_t stride, const float* m0,
                                  float* starts, float* mout, int n, int B, int H, int D,
                                  cudaStream_t st) {
    const int bytes = (int)(compose_smem_floats(D) * sizeof(float));
    cudaError_t e = ensure_dyn_smem(reinterpret_cast<const void*>(compose_prefix_kernel), bytes);
    if (e != cudaSuccess) return e;
    dim3 grid((D + kCJ - 1) / kCJ, B * H);
    compose_prefix_kernel<<<grid, kCThreads, bytes, st>>>(T, U, stride, m0, starts, mout, n, B * H,
                                                          D);
    return cudaGetLastError();
}

}  // namespace la
