// Tensor-core (tcgen05) scan for wide heads: bf16 inputs, 128 < D <= 256.
//
// A D x D state of up to 256 x 256 fp32 is as large as a whole SM's tensor
// memory, so the work is cut into 128-row / 128-column blocks (dimensions
// beyond D are zero padding that the TMA fills and the math keeps at zero):
//
//   gram   (frame-parallel) one CTA per (b, h, f, key-row block r):
//            GDN : G''_f[r] = -alpha_f beta_f kappa^2 K[:, r]^T K   (bf16 image)
//                  B~_f[r]  =  beta_f kappa     K[:, r]^T V         (bf16 tiles)
//            ReLU: dM_f[r] = phi(K)[:, r]^T V (fp32), dz_f[r] = phi(K)[:, r]^T 1
//   chain  (sequential per (b, h)); column blocks of the state evolve
//          independently, so each column half c has its own CTA:
//            GDN : M_f[:, c] = alpha_f M_{f-1}[:, c] + G''_f bf16(M_{f-1})[:, c]
//                              + B~_f[:, c]   (fp32 state in tensor memory)
//            ReLU: M_f = M_{f-1} + dM_f, z_f = z_{f-1} + dz_f (a plain prefix
//                  sum, held in registers, one CTA per 32 state columns)
//          and writes bf16(M_f)[:, c] as an MMA operand image.
//   output (frame-parallel) one CTA per (b, h, f, value-column half c):
//            O_f[:, c] = Q~_f bf16(M_f)[:, c]  (ReLU: / (phi(Q_f) z_f + eps))
//
// Equations: the frame-wise Gated DeltaNet of the SANA-WM paper summary
// (section 3, "Hybrid GDN/Softmax Attention") in its affine form, and the
// block-causal ReLU linear attention of the SANA-Video talk (block KV cache
// segment).  The split of the state into independent column blocks is plain
// linear algebra: M_f[:, c] depends only on M_{f-1}[:, c].
//
// Operand images (128-byte swizzle, 16-byte chunk j of row r at j ^ (r % 8)):
//   G''[r] image : 128 rows (key i in block r) x 256 columns (key j), K-major,
//                  four 64-column blocks of 16 KB.
//   M[:, c] image: 256 rows (key i) x 128 columns (value j in half c),
//                  MN-major, two 64-column blocks of 32 KB.
// dM blocks (ReLU) are fp32 [128 x 256] "quad-interleaved": element (i, j) at
// ((j / 4) * 128 + i) * 4 + j % 4; B~ tiles (GDN) are bf16 [128 x 128] per
// (frame, r, c), 16-byte chunk jc (columns 8 jc .. 8 jc + 7) of row i at
// (jc * 128 + i) * 16 bytes.  Either way a warp's 32 rows touch 512
// contiguous bytes.  B~ is kept in bf16 like the state image; the state
// itself and all accumulation stay fp32.
#include <algorithm>
#include <cstdlib>
#include <mutex>

#include "tc_common.cuh"
#include "tmap.cuh"

namespace la {
namespace {

using namespace tc;

constexpr int kDW = 256;                      // padded head dimension
constexpr int kTokG = 64;                     // tokens per gram tile
constexpr int kTokO = 128;                    // tokens per output tile
constexpr uint32_t kBoxG = 64 * kTokG * 2;    // 8 KB: 64 columns x 64 tokens
constexpr uint32_t kBoxO = 64 * kTokO * 2;    // 16 KB: 64 columns x 128 tokens
constexpr uint32_t kGTile = 4 * kBoxG;        // 32 KB: one 256-wide gram tile of K or V
constexpr uint32_t kOTile = 4 * kBoxO;        // 64 KB: one 256-wide output tile of Q
constexpr uint32_t kGImg = 65536;             // G''[r] image
constexpr uint32_t kMImg = 65536;             // M[:, c] image
constexpr uint32_t kQuad = 128 * 256;         // floats of one fp32 [128 x 256] block
constexpr uint32_t kBTile = 16 * 128;         // 16-byte chunks of one bf16 [128 x 128] B~ tile
constexpr int kOAcc = 4;                      // output accumulator slots (128 columns each)

struct WideParams {
    const float* alpha;
    const float* beta;
    const float* state_in;
    const float* z_in;
    float* state_out;
    float* z_out;
    unsigned int* status;   // workspace header (status, where)
    uint8_t* gimg;          // [BHF][2] x kGImg                 (GDN)
    uint4* btil;            // [BHF][2][2] x kBTile bf16 B~     (GDN)
    float* bmat;            // [BHF][2] x kQuad fp32 dM          (ReLU)
    float* dz;              // [BHF][2] x 128                   (ReLU)
    uint8_t* mimg;          // [BHF][2] x kMImg
    float* zf;              // [BHF] x 256                      (ReLU)
    float k_scale;
    float eps;
    int BH, F, S, D;        // F: frames of the clip (global frame index = bh F + f)
    int f0, Fc;             // this launch covers scan steps [f0, f0 + Fc) of every head
    int want_output;
    int rev_chunk;          // > 0: reversed GDN scan reset every rev_chunk frames
    const float* beta_tok;  // per-token update gate [BH][F][S] (TOKB gram), or NULL
};

// Global frame index (into q, k, v, o, alpha, beta) of chunk-local scan step
// `loc` = bh * Fc + fl (step f0 + fl covers frame step_frame(f0 + fl)); per-step
// workspace buffers are indexed by `loc`.
__device__ __forceinline__ int global_frame(const WideParams& p, int loc) {
    const int bh = loc / p.Fc;
    return bh * p.F + step_frame(p.f0 + (loc - bh * p.Fc), p.F, p.rev_chunk);
}

// Decay of chunk-local step `loc`: zero where the reversed scan starts a chunk,
// which makes G'' zero and restarts the carried state.
__device__ __forceinline__ float step_alpha(const WideParams& p, int loc) {
    const int bh = loc / p.Fc;
    return step_resets(p.f0 + (loc - bh * p.Fc), p.rev_chunk) ? 0.f : p.alpha[global_frame(p, loc)];
}

// Write 16 consecutive columns [c0, c0 + 16) of row `row` of a swizzled bf16
// image whose 64-column blocks are `blk_bytes` apart.
__device__ __forceinline__ void store_row16(uint8_t* img, uint32_t blk_bytes, int row, int c0,
                                            const float (&v)[16]) {
    const int blk = c0 >> 6, ch = (c0 & 63) >> 3;
    uint4 a = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                         pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
    uint4 b = make_uint4(pack_bf16x2(v[8], v[9]), pack_bf16x2(v[10], v[11]),
                         pack_bf16x2(v[12], v[13]), pack_bf16x2(v[14], v[15]));
    *reinterpret_cast<uint4*>(img + blk * blk_bytes + sw128_off(row, ch)) = a;
    *reinterpret_cast<uint4*>(img + blk * blk_bytes + sw128_off(row, ch + 1)) = b;
}

// Offset (in floats) of element (row, col) of a quad-interleaved fp32 block.
__device__ __forceinline__ uint32_t quad_off(int row, int col) {
    return ((uint32_t)(col >> 2) * 128u + (uint32_t)row) * 4u + (uint32_t)(col & 3);
}

// Read-out of one gram item (workspace item `item` = 2 loc + r: key-row block
// r of chunk-local step loc) by one epilogue group g (half of the 512
// accumulator columns; thread <-> accumulator row `row`, TMEM lane base in tl).
template <bool RELU, bool TOKB>
__device__ __forceinline__ void gram_readout(const WideParams& p, uint32_t tl, int item, int g,
                                             int row) {
    // four 16-column TMEM loads in flight per wait
    float v[4][16];
    auto load64 = [&](uint32_t col) {
#pragma unroll
        for (int u = 0; u < 4; ++u) tmem_ld16(tl + col + 16 * u, v[u]);
        tmem_wait_ld();
    };
    if (!RELU) {
        const int frame = global_frame(p, item >> 1);
        const float al = step_alpha(p, item >> 1), bt = TOKB ? 1.f : p.beta[frame];
        const float sg = -al * bt * p.k_scale * p.k_scale, sw = bt * p.k_scale;
        if (g == 0) {
            // the G''[r] image goes straight from registers to its workspace slot
            uint8_t* gi = p.gimg + (size_t)item * kGImg;
            for (int c0 = 0; c0 < kDW; c0 += 64) {
                load64(c0);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) v[u][e] *= sg;
                    store_row16(gi, 16384, row, c0 + 16 * u, v[u]);
                }
            }
        } else {
            for (int c0 = 0; c0 < kDW; c0 += 64) {
                load64(256 + c0);
                uint4* bt4 = p.btil + ((size_t)item * 2 + (c0 >> 7)) * kBTile;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int jc = ((c0 + 16 * u) & 127) >> 3;
#pragma unroll
                    for (int h = 0; h < 2; ++h)
                        bt4[(jc + h) * 128 + row] = make_uint4(
                            pack_bf16x2(v[u][8 * h] * sw, v[u][8 * h + 1] * sw),
                            pack_bf16x2(v[u][8 * h + 2] * sw, v[u][8 * h + 3] * sw),
                            pack_bf16x2(v[u][8 * h + 4] * sw, v[u][8 * h + 5] * sw),
                            pack_bf16x2(v[u][8 * h + 6] * sw, v[u][8 * h + 7] * sw));
                }
            }
        }
    } else {
        float* bq = p.bmat + (size_t)item * kQuad;
        for (int c0 = 128 * g; c0 < 128 * g + 128; c0 += 64) {
            load64(c0);
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int w = 0; w < 4; ++w)
                    *reinterpret_cast<float4*>(bq + quad_off(row, c0 + 16 * u + 4 * w)) =
                        make_float4(v[u][4 * w], v[u][4 * w + 1], v[u][4 * w + 2], v[u][4 * w + 3]);
        }
        if (g == 0) {
            tmem_ld16(tl + 256, v[0]);
            tmem_wait_ld();
            p.dz[(size_t)item * 128 + row] = v[0][0];
        }
    }
}

// ============================================================================
// gram: per-frame contractions over tokens, one key-row block per CTA
// ============================================================================
// warp 0: TMA producer; warp 1: TMEM owner + MMA issuer; warps 6-9 (ReLU):
// phi(K) in place before the MMA; two epilogue groups of four warps (2-5, and
// 6-9 or, with ReLU, 10-13) read out the two halves of the 512 accumulator
// columns side by side (GDN: G'' and B~; ReLU: value columns 0-127 with dz,
// and 128-255), so the next item's MMAs wait half as long for the TMEM.
// With the per-token update gate (TOKB, GDN), warps 6-9 scale every K and V
// token row of a tile by sqrt(beta_t) in shared memory (packed bf16) before
// the unchanged MMAs, which then give Kh^T diag(beta) Kh and Kh^T diag(beta) V.
constexpr int wide_gram_threads(bool xf) { return xf ? 448 : 320; }

template <bool RELU, bool TOKB = false>
__global__ void __launch_bounds__(wide_gram_threads(RELU || TOKB), 1)
wide_gram_kernel(const WideParams p, const __grid_constant__ CUtensorMap mapK,
                 const __grid_constant__ CUtensorMap mapV) {
    constexpr int kStages = 3;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* ring = smem;                                  // kStages x (K 32 KB | V 32 KB)
    uint8_t* ones = ring + kStages * 2 * kGTile;           // 2 KB of bf16 1.0 (ReLU)
    uint64_t* full = reinterpret_cast<uint64_t*>(ones + 2048);
    uint64_t* empty = full + kStages;
    uint64_t* xform = empty + kStages;
    uint64_t* accfull = xform + kStages;
    uint64_t* accempty = accfull + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accempty + 1);
    uint32_t* abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int D = p.D;
    const int nbx = (D + 63) / 64;                         // column boxes that hold data
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&xform[s], 4);
        }
        mbar_init(accfull, 1);
        mbar_init(accempty, 8);                            // both epilogue groups
        *abort_flag = 0;
        fence_mbar_init();
    }
    // Column boxes past D are never loaded: zero them once.
    for (int s = 0; s < kStages; ++s)
        for (int t = 0; t < 2; ++t)
            for (int b = nbx; b < 4; ++b) {
                uint4* z = reinterpret_cast<uint4*>(ring + s * 2 * kGTile + t * kGTile + b * kBoxG);
                for (int i = threadIdx.x; i < (int)(kBoxG / 16); i += blockDim.x)
                    z[i] = make_uint4(0, 0, 0, 0);
            }
    if (RELU)
        for (int i = threadIdx.x; i < 2048 / 4; i += blockDim.x)
            reinterpret_cast<uint32_t*>(ones)[i] = 0x3F803F80u;
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const Abort ab{abort_flag, p.status};
    const int nitems = p.BH * p.Fc * 2;
    const int nt = (p.S + kTokG - 1) / kTokG;

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&mapK);
            tma_prefetch_desc(&mapV);
            const uint64_t pol = policy_evict_first();
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            PhaseLog armed;     // loads in flight are waited for after an abort
            for (int item = blockIdx.x; item < nitems && ok; item += gridDim.x) {
                const int frame = global_frame(p, item >> 1);
                for (int t = 0; t < nt; ++t) {
                    if (!(ok = mbar_wait(&empty[s], ph ^ 1, ab, 0x601))) break;
                    uint8_t* st = ring + s * 2 * kGTile;
                    mbar_expect_tx(&full[s], 2 * nbx * kBoxG);
                    for (int b = 0; b < nbx; ++b) {
                        tma_load_3d(st + b * kBoxG, &mapK, &full[s], 64 * b, t * kTokG, frame, pol);
                        tma_load_3d(st + kGTile + b * kBoxG, &mapV, &full[s], 64 * b, t * kTokG,
                                    frame, pol);
                    }
                    armed.note(s, ph);
                    if (++s == kStages) { s = 0; ph ^= 1; }
                }
            }
            armed.drain_if_aborted(full, kStages, ab);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idW = idesc_bf16(128, kDW, true, true);
            const uint32_t idZ = idesc_bf16(128, 16, true, false);
            const uint64_t ones_d = sdesc_sw128(smem_u32(ones), 16, 1024);
            // GDN: G at columns [0, 256), B~ at [256, 512); ReLU: dM at [0, 256), dz at 256.
            const uint32_t dA = tbase, dB = tbase + 256;
            int s = 0, li = 0;
            uint32_t ph = 0;
            bool ok = true;
            PhaseLog armed;     // MMAs in flight are waited for after an abort
            for (int item = blockIdx.x; item < nitems && ok; item += gridDim.x, ++li) {
                const int r = item & 1;
                if (!(ok = mbar_wait(accempty, (li & 1) ^ 1, ab, 0x602))) break;
                tc_fence_after();
                for (int t = 0; t < nt; ++t) {
                    if (!(ok = mbar_wait((RELU || TOKB) ? &xform[s] : &full[s], ph, ab, 0x603))) break;
                    tc_fence_after();
                    const uint32_t sk = smem_u32(ring + s * 2 * kGTile), sv = sk + kGTile;
#pragma unroll
                    for (int k = 0; k < kTokG / 16; ++k) {
                        // A = K[:, block r]^T (MN-major), B = K or V (MN-major, N = 256)
                        const uint64_t ad = sdesc_sw128(sk + 2 * r * kBoxG + k * 2048, kBoxG, 1024);
                        const uint64_t bk = sdesc_sw128(sk + k * 2048, kBoxG, 1024);
                        const uint64_t bv = sdesc_sw128(sv + k * 2048, kBoxG, 1024);
                        const uint32_t acc = (t | k) ? 1u : 0u;
                        if (RELU) {
                            mma_bf16(dA, ad, bv, idW, acc);
                            mma_bf16(dB, ad, ones_d, idZ, acc);
                        } else {
                            mma_bf16(dA, ad, bk, idW, acc);
                            mma_bf16(dB, ad, bv, idW, acc);
                        }
                    }
                    mma_commit(&empty[s]);
                    armed.note(s, ph);
                    if (++s == kStages) { s = 0; ph ^= 1; }
                }
                if (ok) mma_commit(accfull);
            }
            armed.drain_if_aborted(empty, kStages, ab);
        }
    } else if (TOKB && warp >= 6 && warp < 10) {
        // ---------------- per-token gate: sqrt(beta_t) on the K and V rows ----------------
        const int tl = threadIdx.x - 192;          // 0..127: row tl % 64 of K (tl < 64) or V
        const int row = tl & 63;
        const int nch = (D + 7) / 8;
        int s = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < nitems && ok; item += gridDim.x) {
            const float* bsrc = p.beta_tok + (size_t)global_frame(p, item >> 1) * p.S;
            float bv_next = row < p.S ? __ldg(bsrc + row) : 0.f;    // gates one tile ahead
            for (int t = 0; t < nt; ++t) {
                const float bv = bv_next;
                const int tok_n = (t + 1) * kTokG + row;
                bv_next = (t + 1 < nt && tok_n < p.S) ? __ldg(bsrc + tok_n) : 0.f;
                if (!(ok = mbar_wait(&full[s], ph, ab, 0x606))) break;
                const float sb = sqrtf(fmaxf(bv, 0.f));
                const __nv_bfloat162 g = __floats2bfloat162_rn(sb, sb);
                uint8_t* const base = ring + s * 2 * kGTile + (tl >> 6) * kGTile;
                for (int c = 0; c < nch; ++c) {
                    uint4* pc = reinterpret_cast<uint4*>(base + (c >> 3) * kBoxG + sw128_off(row, c & 7));
                    uint4 x = *pc;
                    __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&x);
                    h[0] = __hmul2(h[0], g); h[1] = __hmul2(h[1], g);
                    h[2] = __hmul2(h[2], g); h[3] = __hmul2(h[3], g);
                    *pc = x;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&xform[s]);
                if (++s == kStages) { s = 0; ph ^= 1; }
            }
        }
    } else if (RELU && warp >= 6 && warp < 10) {
        // ---------------- ReLU transform: phi(K) in place ----------------
        const int tl = threadIdx.x - 192;          // 0..127
        int s = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < nitems && ok; item += gridDim.x) {
            for (int t = 0; t < nt; ++t) {
                if (!(ok = mbar_wait(&full[s], ph, ab, 0x605))) break;
                uint4* kt = reinterpret_cast<uint4*>(ring + s * 2 * kGTile);
                for (int i = tl; i < nbx * (int)kBoxG / 16; i += 128) {
                    uint4 x = kt[i];
                    x.x = relu_bf16x2(x.x); x.y = relu_bf16x2(x.y);
                    x.z = relu_bf16x2(x.z); x.w = relu_bf16x2(x.w);
                    kt[i] = x;
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&xform[s]);
                if (++s == kStages) { s = 0; ph ^= 1; }
            }
        }
    } else {
        // ---------------- epilogue: TMEM -> workspace, two groups ----------------
        const int q = warp & 3, row = q * 32 + lane;
        const int g = warp < 6 ? 0 : 1;                 // half of the accumulator columns
        int li = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < nitems && ok; item += gridDim.x, ++li) {
            if (!(ok = mbar_wait(accfull, li & 1, ab, 0x604))) break;
            tc_fence_after();
            gram_readout<RELU, TOKB>(p, tbase + (uint32_t(q * 32) << 16), item, g, row);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(accempty);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tbase, 512);
}

// ============================================================================
// gram on a CTA pair (cta_group::2): one cluster of two CTAs per (b, h, f)
// ============================================================================
// The pair computes the item's 256 x 512 accumulator [K^T K | K^T V] (ReLU:
// [phi(K)^T V | phi(K)^T 1]) with M = 256 MMAs that the even CTA issues.
// CTA c holds key columns 128 c .. 128 c + 127 of every K and V tile: they
// are at once its 128 rows of A = K^T and its 128 columns of B = K or V.  Its
// tensor memory receives accumulator rows 128 c .. 128 c + 127, i.e. key-row
// block r = c of the single-CTA kernel, which the same read-out handles.  So
// every K and V byte is fetched once per frame and each CTA's shared memory
// serves half the operand bytes of the single-CTA kernel.
//
// Barriers (every wait bounded):
//   full[s]   (each CTA)  this CTA's TMA bytes of stage s have landed
//   ready[s]  (even CTA)  stage s usable by the pair's MMAs: with no transform
//                         the odd CTA's warp 1 forwards its full[s] (the even
//                         CTA's MMA issuer waits on its own full[s] too); with
//                         a transform, the four transform warps of both CTAs
//                         arrive when their pass is done
//   empty[s]  (each CTA)  the pair's MMAs have read stage s (commit to each CTA)
//   accfull   (each CTA)  the item's accumulator is complete (commit to each CTA)
//   accempty  (even CTA)  all 16 epilogue warps of the pair have read the TMEM
// Warps: 0 TMA producer; 1 TMEM (both CTAs), MMA issuer (even CTA) or
// forwarder (odd CTA); 2-5 and 6-9 (10-13 with a transform) the two epilogue
// groups; 6-9 with a transform: phi(K) (ReLU) or sqrt(beta_t) row scaling.
constexpr int kPairStages = 6;
constexpr uint32_t kPairTile = 2 * kBoxG;                  // 16 KB: 128 columns x 64 tokens
constexpr uint32_t kPairStage = 2 * kPairTile;             // K | V
constexpr size_t kSmemWidePair = 1024 + kPairStages * kPairStage + 2048 + 512;

template <bool RELU, bool TOKB = false>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(wide_gram_threads(RELU || TOKB), 1)
wide_gram_pair_kernel(const WideParams p, const __grid_constant__ CUtensorMap mapK,
                      const __grid_constant__ CUtensorMap mapV) {
    constexpr bool XF = RELU || TOKB;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* ring = smem;                                  // kPairStages x (K 16 KB | V 16 KB)
    uint8_t* ones = ring + kPairStages * kPairStage;       // 2 KB of bf16 1.0 (ReLU)
    uint64_t* full = reinterpret_cast<uint64_t*>(ones + 2048);
    uint64_t* empty = full + kPairStages;
    uint64_t* ready = empty + kPairStages;
    uint64_t* accfull = ready + kPairStages;
    uint64_t* accempty = accfull + 1;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accempty + 1);
    uint32_t* abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t rank = cluster_ctarank();
    const int cid = (int)cluster_id_x(), ncl = (int)ncluster_x();
    const int D = p.D;
    // 64-column boxes of this CTA's half that hold data (the rest stay zero)
    const int nbl = max(0, min(2, (D + 63) / 64 - 2 * (int)rank));
    if (threadIdx.x == 0) {
        for (int s = 0; s < kPairStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&ready[s], XF ? 8 : 1);
        }
        mbar_init(accfull, 1);
        mbar_init(accempty, 16);
        *abort_flag = 0;
        fence_mbar_init();
    }
    for (int s = 0; s < kPairStages; ++s)
        for (int t = 0; t < 2; ++t)
            for (int b = nbl; b < 2; ++b) {
                uint4* z = reinterpret_cast<uint4*>(ring + s * kPairStage + t * kPairTile + b * kBoxG);
                for (int i = threadIdx.x; i < (int)(kBoxG / 16); i += blockDim.x)
                    z[i] = make_uint4(0, 0, 0, 0);
            }
    if (RELU)
        for (int i = threadIdx.x; i < 2048 / 4; i += blockDim.x)
            reinterpret_cast<uint32_t*>(ones)[i] = 0x3F803F80u;
    if (warp == 1) {
        tmem_alloc_pair(tmem_slot, 512);
        tmem_relinquish_pair();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    cluster_sync();            // both CTAs' barriers, zero boxes and TMEM ready
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const Abort ab{abort_flag, p.status};
    const int nitems = p.BH * p.Fc;
    const int nt = (p.S + kTokG - 1) / kTokG;

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&mapK);
            tma_prefetch_desc(&mapV);
            const uint64_t pol = policy_evict_first();
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            PhaseLog armed;     // loads in flight are waited for after an abort
            for (int item = cid; item < nitems && ok; item += ncl) {
                const int frame = global_frame(p, item);
                for (int t = 0; t < nt; ++t) {
                    if (!(ok = mbar_wait(&empty[s], ph ^ 1, ab, 0x611))) break;
                    uint8_t* st = ring + s * kPairStage;
                    mbar_expect_tx(&full[s], 2 * nbl * kBoxG);
                    for (int b = 0; b < nbl; ++b) {
                        const int x = 128 * (int)rank + 64 * b;
                        tma_load_3d(st + b * kBoxG, &mapK, &full[s], x, t * kTokG, frame, pol);
                        tma_load_3d(st + kPairTile + b * kBoxG, &mapV, &full[s], x, t * kTokG,
                                    frame, pol);
                    }
                    armed.note(s, ph);
                    if (++s == kPairStages) { s = 0; ph ^= 1; }
                }
            }
            armed.drain_if_aborted(full, kPairStages, ab);
        }
    } else if (warp == 1) {
        if (lane == 0 && rank == 0) {
            // ---------------- MMA issuer of the pair ----------------
            const uint32_t idW = idesc_bf16(256, kDW, true, true);
            const uint32_t idZ = idesc_bf16(256, 16, true, false);
            const uint64_t ones_d = sdesc_sw128(smem_u32(ones), 16, 1024);
            // GDN: G at columns [0, 256), B~ at [256, 512); ReLU: dM at [0, 256), dz at 256.
            const uint32_t dA = tbase, dB = tbase + 256;
            int s = 0, li = 0;
            uint32_t ph = 0;
            bool ok = true;
            PhaseLog armed;     // MMAs in flight are waited for after an abort
            for (int item = cid; item < nitems && ok; item += ncl, ++li) {
                if (!(ok = mbar_wait(accempty, (li & 1) ^ 1, ab, 0x612, true))) break;
                tc_fence_after();
                for (int t = 0; t < nt; ++t) {
                    if (!XF && !(ok = mbar_wait(&full[s], ph, ab, 0x613))) break;
                    if (!(ok = mbar_wait(&ready[s], ph, ab, 0x614, true))) break;
                    tc_fence_after();
                    const uint32_t sk = smem_u32(ring + s * kPairStage), sv = sk + kPairTile;
#pragma unroll
                    for (int k = 0; k < kTokG / 16; ++k) {
                        // A = this CTA's K columns ^T (MN-major, 2 boxes), B = K or V
                        // (MN-major, this CTA's 128 of the N = 256 columns)
                        const uint64_t ak = sdesc_sw128(sk + k * 2048, kBoxG, 1024);
                        const uint64_t bv = sdesc_sw128(sv + k * 2048, kBoxG, 1024);
                        const uint32_t acc = (t | k) ? 1u : 0u;
                        if (RELU) {
                            mma_bf16_pair(dA, ak, bv, idW, acc);
                            mma_bf16_pair(dB, ak, ones_d, idZ, acc);
                        } else {
                            mma_bf16_pair(dA, ak, ak, idW, acc);
                            mma_bf16_pair(dB, ak, bv, idW, acc);
                        }
                    }
                    mma_commit_pair(&empty[s], 0);
                    mma_commit_pair(&empty[s], 1);
                    armed.note(s, ph);
                    if (++s == kPairStages) { s = 0; ph ^= 1; }
                }
                if (ok) {
                    mma_commit_pair(accfull, 0);
                    mma_commit_pair(accfull, 1);
                }
            }
            armed.drain_if_aborted(empty, kPairStages, ab);
        } else if (lane == 0 && !XF) {
            // ---------------- odd CTA: forward each landed stage ----------------
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int item = cid; item < nitems && ok; item += ncl)
                for (int t = 0; t < nt; ++t) {
                    if (!(ok = mbar_wait(&full[s], ph, ab, 0x615))) break;
                    mbar_arrive_cluster(&ready[s], 0);
                    if (++s == kPairStages) { s = 0; ph ^= 1; }
                }
        }
    } else if (XF && warp >= 6 && warp < 10) {
        // ---------------- transform of this CTA's K (and V) columns ----------------
        const int tl = threadIdx.x - 192;          // 0..127
        const int row = tl & 63;
        int s = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int item = cid; item < nitems && ok; item += ncl) {
            const float* bsrc = TOKB ? p.beta_tok + (size_t)global_frame(p, item) * p.S : nullptr;
            float bv_next = (TOKB && row < p.S) ? __ldg(bsrc + row) : 0.f;   // gates one tile ahead
            for (int t = 0; t < nt; ++t) {
                const float bv = bv_next;
                if (TOKB) {
                    const int tok_n = (t + 1) * kTokG + row;
                    bv_next = (t + 1 < nt && tok_n < p.S) ? __ldg(bsrc + tok_n) : 0.f;
                }
                if (!(ok = mbar_wait(&full[s], ph, ab, 0x616))) break;
                uint8_t* st = ring + s * kPairStage;
                if (TOKB) {
                    // thread -> token row `row` of K (tl < 64) or V: 8 columns per chunk
                    const float sb = sqrtf(fmaxf(bv, 0.f));
                    const __nv_bfloat162 gsc = __floats2bfloat162_rn(sb, sb);
                    uint8_t* const base = st + (tl >> 6) * kPairTile;
                    for (int c = 0; c < 8 * nbl; ++c) {
                        uint4* pc = reinterpret_cast<uint4*>(base + (c >> 3) * kBoxG + sw128_off(row, c & 7));
                        uint4 x = *pc;
                        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&x);
                        h[0] = __hmul2(h[0], gsc); h[1] = __hmul2(h[1], gsc);
                        h[2] = __hmul2(h[2], gsc); h[3] = __hmul2(h[3], gsc);
                        *pc = x;
                    }
                } else {
                    uint4* kt = reinterpret_cast<uint4*>(st);
                    for (int i = tl; i < nbl * (int)kBoxG / 16; i += 128) {
                        uint4 x = kt[i];
                        x.x = relu_bf16x2(x.x); x.y = relu_bf16x2(x.y);
                        x.z = relu_bf16x2(x.z); x.w = relu_bf16x2(x.w);
                        kt[i] = x;
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive_cluster(&ready[s], 0);
                if (++s == kPairStages) { s = 0; ph ^= 1; }
            }
        }
    } else if (warp >= 2) {
        // ---------------- epilogue: key-row block r = rank ----------------
        const int q = warp & 3, row = q * 32 + lane;
        const int g = warp < 6 ? 0 : 1;                 // half of the accumulator columns
        int li = 0;
        bool ok = true;
        for (int item = cid; item < nitems && ok; item += ncl, ++li) {
            if (!(ok = mbar_wait(accfull, li & 1, ab, 0x617))) break;
            tc_fence_after();
            gram_readout<RELU, TOKB>(p, tbase + (uint32_t(q * 32) << 16), 2 * item + (int)rank, g, row);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_cluster(accempty, 0);
        }
    }
    tc_fence_before();
    __syncthreads();
    cluster_sync();            // no CTA leaves while its pair may still reach its memory
    tc_fence_after();
    if (warp == 1) tmem_dealloc_pair(tbase, 512);
}

// ============================================================================
// chain (GDN): one CTA per (b, h, value-column half c), state in TMEM
// ============================================================================
// warp 0: bulk loader of the two G''[r] row blocks of each frame;
// warp 1: TMEM owner + MMA issuer; warps 2-9: epilogue, warp w handles key-row
// block r = (w - 2) / 4 and TMEM lanes 32 (w % 4) .. 32 (w % 4) + 31;
// warp 10: publisher of the M[:, c] image of each frame.
__global__ void __launch_bounds__(352, 1)
wide_chain_gdn_kernel(const WideParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* stage = smem;                                 // 2 x 64 KB: G''[0], G''[1]
    uint8_t* img = stage + 2 * kGImg;                      // M[:, c] image (64 KB)
    uint64_t* gfull = reinterpret_cast<uint64_t*>(img + kMImg);
    uint64_t* gempty = gfull + 2;
    uint64_t* mdone = gempty + 2;      // both row-block MMAs of the frame finished
    uint64_t* mready = mdone + 1;      // TMEM holds alpha M, image of M written (both groups)
    uint64_t* idone = mready + 1;      // image of the frame written (both groups)
    uint64_t* ipub = idone + 1;        // publisher has read the image out
    int* bc_ok = reinterpret_cast<int*>(ipub + 1);          // [2] per row group
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bc_ok + 2);
    uint32_t* abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.x >> 1, c = blockIdx.x & 1;
    const int F = p.Fc, D = p.D;          // frames of this launch; buffers are chunk-local
    if (threadIdx.x == 0) {
        for (int r = 0; r < 2; ++r) {
            mbar_init(&gfull[r], 1);
            mbar_init(&gempty[r], 1);
        }
        mbar_init(mdone, 1);
        mbar_init(mready, 2);
        mbar_init(idone, 2);
        mbar_init(ipub, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tM = *tmem_slot;
    const Abort ab{abort_flag, p.status};

    if (warp == 0) {
        if (lane == 0) {
            PhaseLog armed;     // loads in flight are waited for after an abort
            for (int f = 0; f < F; ++f) {
                bool ok = true;
                for (int r = 0; r < 2 && ok; ++r) {
                    if (!(ok = mbar_wait(&gempty[r], (f & 1) ^ 1, ab, 0x701))) break;
                    mbar_expect_tx(&gfull[r], kGImg);
                    bulk_load(stage + r * kGImg, p.gimg + ((size_t)bh * F + f) * 2 * kGImg + r * kGImg,
                              kGImg, &gfull[r]);
                    armed.note(r, f & 1);
                }
                if (!ok) break;
            }
            armed.drain_if_aborted(gfull, 2, ab);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idC = idesc_bf16(128, 128, false, true);
            const uint32_t ib = smem_u32(img);
            PhaseLog armed;     // MMAs in flight are waited for after an abort
            for (int f = 0; f < F; ++f) {
                if (!mbar_wait(mready, f & 1, ab, 0x702)) break;
                bool ok = true;
                for (int r = 0; r < 2 && ok; ++r) {
                    if (!(ok = mbar_wait(&gfull[r], f & 1, ab, 0x703))) break;
                    tc_fence_after();
                    const uint32_t sa = smem_u32(stage + r * kGImg);
                    for (int kk = 0; kk < kDW / 16; ++kk) {
                        const uint64_t ad = sdesc_sw128(sa + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                        const uint64_t bd = sdesc_sw128(ib + kk * 2048, 32768, 1024);
                        mma_bf16(tM + r * 128, ad, bd, idC, 1u);
                    }
                    mma_commit(&gempty[r]);
                    armed.note(r, f & 1);
                }
                if (!ok) break;
                mma_commit(mdone);
            }
            armed.drain_if_aborted(gempty, 2, ab);
        }
    } else if (warp < 10) {
        // ---------------- epilogue ----------------
        const int r = (warp - 2) >> 2, q = warp & 3, row = q * 32 + lane;
        const int i = 128 * r + row;                      // key row of the state
        const bool live = i < D;
        const bool leader = ((threadIdx.x - 64) & 127) == 0;
        const int bar_id = 1 + r;
        const uint32_t tl = tM + (uint32_t(q * 32) << 16) + r * 128;
        // decay of this head's chunk-local step f (the chunk has F = Fc steps)
        auto alpha_at = [&](int f) { return step_alpha(p, bh * F + f); };
        // initial state: image of M_0 and alpha_0 M_0 in TMEM
        {
            const float a0 = alpha_at(0);
            for (int j0 = 0; j0 < 128; j0 += 16) {
                float v[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int col = 128 * c + j0 + e;
                    v[e] = (p.state_in && live && col < D) ? p.state_in[((size_t)bh * D + i) * D + col]
                                                           : 0.f;
                }
                store_row16(img, 32768, i, j0, v);
#pragma unroll
                for (int e = 0; e < 16; ++e) v[e] *= a0;
                tmem_st16(tl + j0, v);
            }
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(bar_id, 128);
            if (leader) mbar_arrive(mready);
        }
        // B~ row of the coming frame: 128 bf16 columns in 16 registers of 16 bytes,
        // fetched one frame ahead so the loads never wait on the critical path.
        uint4 bb[16];
        auto fetch_b = [&](int f) {
            const uint4* bt = p.btil + ((((size_t)bh * F + f) * 2 + r) * 2 + c) * kBTile;
#pragma unroll
            for (int jc = 0; jc < 16; ++jc) bb[jc] = __ldg(bt + jc * 128 + row);
        };
        fetch_b(0);
        bool ok = true;
        for (int f = 0; f < F; ++f) {
            const bool more = f + 1 < F;
            const float an = more ? alpha_at(f + 1) : 1.f;
            if (leader) {
                ok = ok && mbar_wait(mdone, f & 1, ab, 0x704);
                if (f >= 1) ok = ok && mbar_wait(ipub, (f - 1) & 1, ab, 0x705);
                bc_ok[r] = ok;
            }
            named_bar_sync(bar_id, 128);
            const bool go = bc_ok[r];
            tc_fence_after();
            if (go) {
#pragma unroll
                for (int j0 = 0; j0 < 128; j0 += 16) {
                    float v[16];
                    tmem_ld16(tl + j0, v);
                    tmem_wait_ld();
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const uint4 w = bb[j0 / 8 + h];
                        v[8 * h + 0] += bf16_lo(w.x); v[8 * h + 1] += bf16_hi(w.x);
                        v[8 * h + 2] += bf16_lo(w.y); v[8 * h + 3] += bf16_hi(w.y);
                        v[8 * h + 4] += bf16_lo(w.z); v[8 * h + 5] += bf16_hi(w.z);
                        v[8 * h + 6] += bf16_lo(w.w); v[8 * h + 7] += bf16_hi(w.w);
                    }
                    store_row16(img, 32768, i, j0, v);
                    if (!more) {
                        if (p.state_out && live) {
#pragma unroll
                            for (int e = 0; e < 16; ++e) {
                                const int col = 128 * c + j0 + e;
                                if (col < D) p.state_out[((size_t)bh * D + i) * D + col] = v[e];
                            }
                        }
                    } else {
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] *= an;
                        tmem_st16(tl + j0, v);
                    }
                }
                if (more) fetch_b(f + 1);
            }
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(bar_id, 128);
            if (leader) {
                mbar_arrive(mready);
                mbar_arrive(idone);
            }
        }
    } else {
        // ---------------- publisher ----------------
        if (lane == 0) {
            for (int f = 0; f < F; ++f) {
                if (!mbar_wait(idone, f & 1, ab, 0x706)) break;
                if (p.want_output) {
                    bulk_store(p.mimg + (((size_t)bh * F + f) * 2 + c) * kMImg, img, kMImg);
                    bulk_commit();
                    bulk_wait_read<0>();
                }
                mbar_arrive(ipub);
            }
            bulk_wait_all<0>();
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tM, 256);
}

// ============================================================================
// chain (ReLU): prefix sums of dM and dz, one CTA per (b, h, 32 state columns)
// ============================================================================
// Thread i owns key row i and 32 columns of the state in registers; the
// next frame's increments are fetched while the current frame is written.
__global__ void __launch_bounds__(256)
wide_chain_relu_kernel(const WideParams p) {
    const int bh = blockIdx.x >> 3, cc = blockIdx.x & 7;
    const int i = threadIdx.x, r = i >> 7, row = i & 127;
    const int F = p.Fc, D = p.D;          // frames of this launch; buffers are chunk-local
    const int c = cc >> 2, jl0 = (cc & 3) * 32;        // column half and first local column
    const int j0 = 32 * cc;                           // first global column
    const bool live = i < D;
    float s[32];
#pragma unroll
    for (int e = 0; e < 32; ++e)
        s[e] = (p.state_in && live && j0 + e < D) ? p.state_in[((size_t)bh * D + i) * D + j0 + e] : 0.f;
    float z = (cc == 0 && p.z_in && live) ? p.z_in[(size_t)bh * D + i] : 0.f;

    float4 nx[8];
    float dzn = 0.f;
    auto fetch = [&](int f) {
        const float* bq = p.bmat + (((size_t)bh * F + f) * 2 + r) * kQuad;
#pragma unroll
        for (int u = 0; u < 8; ++u) nx[u] = __ldg(reinterpret_cast<const float4*>(bq + quad_off(row, j0 + 4 * u)));
        if (cc == 0) dzn = __ldg(p.dz + (((size_t)bh * F + f) * 2 + r) * 128 + row);
    };
    if (F > 0) fetch(0);
    for (int f = 0; f < F; ++f) {
#pragma unroll
        for (int u = 0; u < 8; ++u) {
            s[4 * u] += nx[u].x; s[4 * u + 1] += nx[u].y;
            s[4 * u + 2] += nx[u].z; s[4 * u + 3] += nx[u].w;
        }
        z += dzn;
        if (f + 1 < F) fetch(f + 1);
        if (p.want_output) {
            uint8_t* im = p.mimg + (((size_t)bh * F + f) * 2 + c) * kMImg;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const int jl = jl0 + 8 * w;
                const uint4 x = make_uint4(pack_bf16x2(s[8 * w], s[8 * w + 1]),
                                           pack_bf16x2(s[8 * w + 2], s[8 * w + 3]),
                                           pack_bf16x2(s[8 * w + 4], s[8 * w + 5]),
                                           pack_bf16x2(s[8 * w + 6], s[8 * w + 7]));
                *reinterpret_cast<uint4*>(im + (jl >> 6) * 32768 + sw128_off(i, (jl & 63) >> 3)) = x;
            }
            if (cc == 0) p.zf[((size_t)bh * F + f) * 256 + i] = z;
        }
    }
    if (p.state_out && live) {
#pragma unroll
        for (int e = 0; e < 32; ++e)
            if (j0 + e < D) p.state_out[((size_t)bh * D + i) * D + j0 + e] = s[e];
    }
    if (cc == 0 && p.z_out && live) p.z_out[(size_t)bh * D + i] = z;
}

// ============================================================================
// output: O_f = Q~_f bf16(M_f)   (ReLU: / (phi(Q_f) z_f + eps))
// ============================================================================
// One CTA item per (b, h, f) computes all 256 value columns: the whole
// bf16(M_f) image (128 KB, both value halves) sits in shared memory, Q is
// streamed in 64-column boxes of 128-token tiles (kQS-stage ring), and each
// box feeds four N = 256 MMAs into one of two 256-column TMEM accumulators.
// Q is read once per frame, and the ReLU feature map and denominators are
// formed once per token.
// warp 0: producer (the first Q boxes of an item, then its M image (+ z) by
// bulk copy once the previous item's MMAs are done, then the other boxes);
// warp 1: TMEM owner + MMA issuer; warps 2-5: epilogue (TMEM -> bf16 ->
// TMA store, one 64-column box at a time); warps 6-9 (ReLU): phi(Q) in place
// and the per-token denominators.
constexpr int kQS = 3;                        // Q box ring stages (16 KB each)
constexpr int kOutStg = 2;                    // epilogue staging boxes (16 KB each)

template <bool RELU>
__global__ void __launch_bounds__(RELU ? 320 : 192, 1)
wide_output_kernel(const WideParams p, const __grid_constant__ CUtensorMap mapQ,
                   const __grid_constant__ CUtensorMap mapO) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* mbuf = smem;                                  // bf16(M_f) image, 2 x kMImg
    uint8_t* qring = mbuf + 2 * kMImg;                     // kQS x 16 KB Q boxes
    uint8_t* ostage = qring + kQS * kBoxO;                 // kOutStg x 16 KB output boxes
    float* zbuf = reinterpret_cast<float*>(ostage + kOutStg * kBoxO);   // 256 (ReLU)
    float* denbuf = zbuf + 256;                            // 2 x 128 (ReLU)
    uint64_t* qfull = reinterpret_cast<uint64_t*>(denbuf + 256);
    uint64_t* qempty = qfull + kQS;
    uint64_t* xform = qempty + kQS;
    uint64_t* mfull = xform + kQS;
    uint64_t* mempty = mfull + 1;
    uint64_t* accfull = mempty + 1;                        // [2]
    uint64_t* accempty = accfull + 2;                      // [2]
    uint64_t* denready = accempty + 2;                     // [2]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(denready + 2);
    uint32_t* abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int D = p.D;
    const int nbx = (D + 63) / 64;                         // Q boxes per tile (3 or 4)
    if (threadIdx.x == 0) {
        for (int s = 0; s < kQS; ++s) {
            mbar_init(&qfull[s], 1);
            mbar_init(&qempty[s], 1);
            mbar_init(&xform[s], 4);
        }
        mbar_init(mfull, 1);
        mbar_init(mempty, 1);
        for (int a = 0; a < 2; ++a) {
            mbar_init(&accfull[a], 1);
            mbar_init(&accempty[a], 4);
            mbar_init(&denready[a], 4);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 512);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = *tmem_slot;
    const Abort ab{abort_flag, p.status};
    const int nitems = p.BH * p.Fc;
    const int nt = (p.S + kTokO - 1) / kTokO;

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&mapQ);
            tma_prefetch_desc(&mapO);
            const uint64_t pol = policy_evict_first();
            int s = 0, li = 0;
            uint32_t ph = 0;
            bool ok = true;
            PhaseLog armed_q, armed_m;     // loads in flight are waited for after an abort
            for (int item = blockIdx.x; item < nitems && ok; item += gridDim.x, ++li) {
                const int frame = global_frame(p, item);
                const int nq = nt * nbx;                   // Q boxes of the item
                auto load_q = [&](int g) {                 // box g = tile g / nbx, column box g % nbx
                    if (!(ok = ok && mbar_wait(&qempty[s], ph ^ 1, ab, 0x802))) return;
                    mbar_expect_tx(&qfull[s], kBoxO);
                    tma_load_3d(qring + s * kBoxO, &mapQ, &qfull[s], 64 * (g % nbx),
                                (g / nbx) * kTokO, frame, pol);
                    armed_q.note(s, ph);
                    if (++s == kQS) { s = 0; ph ^= 1; }
                };
                const int early = min(nq, kQS);
                for (int g = 0; g < early; ++g) load_q(g);
                // the image buffer is free once the previous item's MMAs are done
                ok = ok && mbar_wait(mempty, (li & 1) ^ 1, ab, 0x801);
                if (!ok) break;
                mbar_expect_tx(mfull, 2 * kMImg + (RELU ? 1024 : 0));
                bulk_load(mbuf, p.mimg + (size_t)item * 2 * kMImg, 2 * kMImg, mfull);
                if (RELU) bulk_load(zbuf, p.zf + (size_t)item * 256, 1024, mfull);
                armed_m.note(0, li & 1);
                for (int g = early; g < nq; ++g) load_q(g);
            }
            armed_q.drain_if_aborted(qfull, kQS, ab);
            armed_m.drain_if_aborted(mfull, 1, ab);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idO = idesc_bf16(128, kDW, false, true);
            const uint32_t mb = smem_u32(mbuf);
            int s = 0, li = 0, gt = 0;
            uint32_t ph = 0;
            bool ok = true;
            PhaseLog armed;     // MMAs in flight are waited for after an abort
            for (int item = blockIdx.x; item < nitems && ok; item += gridDim.x, ++li) {
                if (!(ok = mbar_wait(mfull, li & 1, ab, 0x803))) break;
                tc_fence_after();
                for (int t = 0; t < nt && ok; ++t, ++gt) {
                    const int a = gt & 1;
                    if (!(ok = mbar_wait(&accempty[a], ((gt >> 1) & 1) ^ 1, ab, 0x804))) break;
                    tc_fence_after();
                    for (int b = 0; b < nbx; ++b) {
                        if (!(ok = mbar_wait(RELU ? &xform[s] : &qfull[s], ph, ab, 0x805))) break;
                        tc_fence_after();
                        const uint32_t qa = smem_u32(qring + s * kBoxO);
#pragma unroll
                        for (int kk = 0; kk < 4; ++kk) {
                            const uint64_t ad = sdesc_sw128(qa + kk * 32, 16, 1024);
                            const uint64_t bd = sdesc_sw128(mb + (4 * b + kk) * 2048, 32768, 1024);
                            mma_bf16(tbase + a * 256, ad, bd, idO, (b | kk) ? 1u : 0u);
                        }
                        mma_commit(&qempty[s]);
                        armed.note(s, ph);
                        if (++s == kQS) { s = 0; ph ^= 1; }
                    }
                    if (ok) mma_commit(&accfull[a]);
                }
                if (ok) mma_commit(mempty);
            }
            armed.drain_if_aborted(qempty, kQS, ab);
        }
    } else if (warp < 6) {
        // ---------------- epilogue: TMEM -> bf16 -> TMA store ----------------
        const int q = warp & 3, row = q * 32 + lane;
        const bool issuer = (threadIdx.x == 64);
        int gt = 0, gb = 0;
        bool ok = true;     // every epilogue warp runs every named barrier, even after an abort
        for (int item = blockIdx.x; item < nitems; item += gridDim.x) {
            const int frame = global_frame(p, item);
            for (int t = 0; t < nt; ++t, ++gt) {
                const int a = gt & 1;
                ok = ok && mbar_wait(&accfull[a], (gt >> 1) & 1, ab, 0x806);
                if (RELU) ok = ok && mbar_wait(&denready[a], (gt >> 1) & 1, ab, 0x807);
                tc_fence_after();
                const float inv = (RELU && ok) ? 1.f / denbuf[a * 128 + row] : 1.f;
                const uint32_t tl = tbase + (uint32_t(q * 32) << 16) + a * 256;
                for (int b = 0; b < nbx; ++b, ++gb) {
                    uint8_t* os = ostage + (gb % kOutStg) * kBoxO;
                    if (issuer) bulk_wait_read<kOutStg - 1>();   // this staging box is free
                    named_bar_sync(1, 128);
                    for (int c0 = 0; c0 < 64 && ok; c0 += 16) {
                        float v[16];
                        tmem_ld16(tl + 64 * b + c0, v);
                        tmem_wait_ld();
                        if (RELU) {
#pragma unroll
                            for (int e = 0; e < 16; ++e) v[e] *= inv;
                        }
                        store_row16(os, 16384, row, c0, v);
                    }
                    if (b == nbx - 1) {                   // the accumulator is read out
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(&accempty[a]);
                    }
                    fence_proxy_async_smem();
                    named_bar_sync(1, 128);
                    if (issuer && ok) {
                        tma_store_3d(&mapO, os, 64 * b, t * kTokO, frame);
                        bulk_commit();
                    }
                }
            }
        }
        if (issuer) bulk_wait_all<0>();
    } else {
        // ---------------- ReLU: phi(Q) in place, denominators ----------------
        const int row = threadIdx.x - 192;                // token row in the tile
        int s = 0, li = 0, gt = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < nitems && ok; item += gridDim.x, ++li) {
            if (!(ok = mbar_wait(mfull, li & 1, ab, 0x808))) break;
            for (int t = 0; t < nt && ok; ++t, ++gt) {
                const int a = gt & 1;
                // denbuf[a] is free once the epilogue has read this accumulator's last use
                if (!(ok = mbar_wait(&accempty[a], ((gt >> 1) & 1) ^ 1, ab, 0x80a))) break;
                float den = 0.f;
                for (int b = 0; b < nbx; ++b) {
                    if (!(ok = mbar_wait(&qfull[s], ph, ab, 0x809))) break;
                    uint8_t* st = qring + s * kBoxO;
                    for (int ch = 0; ch < 8; ++ch) {
                        uint4* pch = reinterpret_cast<uint4*>(st + sw128_off(row, ch));
                        uint4 x = *pch;
                        x.x = relu_bf16x2(x.x); x.y = relu_bf16x2(x.y);
                        x.z = relu_bf16x2(x.z); x.w = relu_bf16x2(x.w);
                        *pch = x;
                        const float* zz = zbuf + b * 64 + ch * 8;
                        den = fmaf(bf16_lo(x.x), zz[0], den);
                        den = fmaf(bf16_hi(x.x), zz[1], den);
                        den = fmaf(bf16_lo(x.y), zz[2], den);
                        den = fmaf(bf16_hi(x.y), zz[3], den);
                        den = fmaf(bf16_lo(x.z), zz[4], den);
                        den = fmaf(bf16_hi(x.z), zz[5], den);
                        den = fmaf(bf16_lo(x.w), zz[6], den);
                        den = fmaf(bf16_hi(x.w), zz[7], den);
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&xform[s]);
                    if (++s == kQS) { s = 0; ph ^= 1; }
                }
                if (!ok) break;
                denbuf[a * 128 + row] = den + p.eps;
                __syncwarp();
                if (lane == 0) mbar_arrive(&denready[a]);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tbase, 512);
}

// ----------------------------------------------------------------------------
// Host side
// ----------------------------------------------------------------------------
// Frames per pipeline chunk: about 8 chunks, at least 4 frames (LA_WIDE_CHUNK
// in the environment overrides it, for tuning).
int wide_chunk(int F) {
    const char* e = std::getenv("LA_WIDE_CHUNK");
    int c = e ? std::atoi(e) : 0;
    if (c <= 0) c = std::max(4, (F + 7) / 8);
    return std::max(1, std::min(c, F));
}

// Workspace: header | state, z carried between chunks | two chunk buffer sets
// of the gram outputs | two chunk buffer sets of the chain outputs.
struct WideLayout {
    size_t state, z;
    size_t gimg[2], btil[2], bmat[2], dz[2], mimg[2], zf[2];
    size_t total;
    int Fc;
};

WideLayout wide_layout(const ScanArgs& a) {
    WideLayout L;
    const size_t bh = (size_t)a.B * a.H;
    L.Fc = wide_chunk(a.F);
    const size_t bhf = bh * L.Fc;
    const bool gdn = a.mode == LA_MODE_GDN;
    const int nsets = a.F > L.Fc ? 2 : 1;        // a second buffer set only if chunks overlap
    size_t off = kWsHeaderBytes;
    L.state = off;
    off = align_up(off + bh * a.D * a.D * 4, 256);
    L.z = off;
    off = align_up(off + bh * a.D * 4, 256);
    for (int b = 0; b < 2; ++b) {
        if (b == nsets) {                        // a single chunk: both names, one set
            L.gimg[1] = L.gimg[0]; L.btil[1] = L.btil[0]; L.bmat[1] = L.bmat[0]; L.dz[1] = L.dz[0];
            break;
        }
        L.gimg[b] = off;
        if (gdn) off += bhf * 2 * kGImg;
        L.btil[b] = off;
        if (gdn) off += bhf * 4 * kBTile * 16;
        L.bmat[b] = off;
        if (!gdn) off += bhf * 2 * kQuad * 4;
        L.dz[b] = off;
        if (!gdn) off += bhf * 2 * 512;
        off = align_up(off, 256);
    }
    for (int b = 0; b < 2; ++b) {
        if (b == nsets) {
            L.mimg[1] = L.mimg[0]; L.zf[1] = L.zf[0];
            break;
        }
        L.mimg[b] = off;
        off += bhf * 2 * kMImg;
        L.zf[b] = off;
        if (!gdn) off += bhf * 1024;
        off = align_up(off, 256);
    }
    L.total = off;
    return L;
}

constexpr size_t kSmemWideGram = 1024 + 3 * 2 * kGTile + 2048 + 256;
static_assert(kSmemWidePair <= 232448, "pair gram smem");

// LA_WIDE_PAIR=1 runs the gram on CTA pairs (cta_group::2) instead of one CTA
// per key-row block.  The pair halves the operand bytes each SM loads and
// reads, but the gram is not bound by them: the item's accumulator fills all
// 512 TMEM columns, so the read-out and the next item's MMAs take turns, and
// the pair adds a cross-CTA hand-off to every stage.  Measured slower (full
// 512-frame D = 256 calls, GDN / ReLU: 4.65 / 5.72 ms on pairs, 4.49 / 5.03
// ms one CTA per block), so the one-CTA kernel is the default.
bool wide_pair_gram() {
    const char* e = std::getenv("LA_WIDE_PAIR");
    return e && e[0] == '1';
}
constexpr size_t kSmemWideChain = 1024 + 2 * kGImg + kMImg + 256;
template <bool RELU>
constexpr size_t smem_wide_out() {
    return 1024 + 2 * kMImg + kQS * kBoxO + kOutStg * kBoxO + 1024 + 1024 + 256;
}
static_assert(kSmemWideGram <= 232448, "gram smem");
static_assert(kSmemWideChain <= 232448, "chain smem");
static_assert(smem_wide_out<false>() <= 232448 && smem_wide_out<true>() <= 232448, "output smem");

// Streams and events of one device for the chunk pipeline: the gram kernels
// run on the caller's stream, the chain and output kernels on two streams of
// the library's own, forked from and joined back to the caller's stream.
constexpr int kMaxDevices = 64;
struct WideCtx {
    bool ready = false;
    cudaStream_t s_chain = nullptr, s_out = nullptr;
    cudaEvent_t start = nullptr, gram[2] = {}, chain[2] = {}, out[2] = {};
};
std::mutex g_wide_mu[kMaxDevices];
WideCtx g_wide_ctx[kMaxDevices];

cudaError_t wide_ctx_init(WideCtx& c) {
    if (c.ready) return cudaSuccess;
    cudaError_t e = cudaStreamCreateWithFlags(&c.s_chain, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&c.s_out, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c.start, cudaEventDisableTiming);
    for (int b = 0; b < 2 && e == cudaSuccess; ++b) {
        e = cudaEventCreateWithFlags(&c.gram[b], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c.chain[b], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c.out[b], cudaEventDisableTiming);
    }
    if (e == cudaSuccess) c.ready = true;
    return e;
}

template <bool RELU>
cudaError_t launch_wide_mode(const ScanArgs& a, cudaStream_t st) {
    const WideLayout L = wide_layout(a);
    uint8_t* ws = reinterpret_cast<uint8_t*>(a.ws);
    WideParams p;
    p.alpha = a.alpha;
    p.rev_chunk = a.rev_chunk;
    p.beta_tok = a.beta_tok;
    p.beta = a.beta;
    p.status = reinterpret_cast<unsigned int*>(ws);
    p.k_scale = a.k_scale;
    p.eps = a.eps;
    p.BH = a.B * a.H;
    p.F = a.F;
    p.S = a.S;
    p.D = a.D;
    p.want_output = a.o != nullptr;
    if ((uint64_t)p.BH * p.F * 2 >= (1ull << 31)) return cudaErrorInvalidValue;

    const uint64_t bhf = (uint64_t)p.BH * p.F;
    CUtensorMap mK, mV, mQ, mO;
    if (!make_tmap_bf16_3d(&mK, a.k, a.D, a.S, bhf, 64, kTokG) ||
        !make_tmap_bf16_3d(&mV, a.v, a.D, a.S, bhf, 64, kTokG))
        return cudaErrorInvalidValue;
    if (p.want_output && (!make_tmap_bf16_3d(&mQ, a.q, a.D, a.S, bhf, 64, kTokO) ||
                          !make_tmap_bf16_3d(&mO, a.o, a.D, a.S, bhf, 64, kTokO)))
        return cudaErrorInvalidValue;

    const bool pair = wide_pair_gram();
    {
        const void* gk = pair ? (a.beta_tok ? reinterpret_cast<const void*>(wide_gram_pair_kernel<false, true>)
                                            : reinterpret_cast<const void*>(wide_gram_pair_kernel<RELU>))
                              : (a.beta_tok ? reinterpret_cast<const void*>(wide_gram_kernel<false, true>)
                                            : reinterpret_cast<const void*>(wide_gram_kernel<RELU>));
        const void* kernels[] = {gk, reinterpret_cast<const void*>(wide_chain_gdn_kernel),
                                 reinterpret_cast<const void*>(wide_output_kernel<RELU>)};
        const int bytes[] = {(int)(pair ? kSmemWidePair : kSmemWideGram), (int)kSmemWideChain,
                             (int)smem_wide_out<RELU>()};
        for (int i = 0; i < 3; ++i) {
            const cudaError_t e = ensure_dyn_smem(kernels[i], bytes[i]);
            if (e != cudaSuccess) return e;
        }
    }
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices)
        return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_wide_mu[dev]);
    WideCtx& cx = g_wide_ctx[dev];
    cudaError_t e = wide_ctx_init(cx);
    if (e != cudaSuccess) return e;

    const int nsm = device_sm_count();
    const int nchunks = (p.F + L.Fc - 1) / L.Fc;
    // GDN: with more than one chunk, chain(c) (about 3.5 us per frame on its
    // own SMs) runs beside gram(c + 1) and output(c - 1), which share the
    // other SMs.  ReLU: the chain is a short prefix sum, so the three kernels
    // of a chunk simply run in order on the caller's stream (measured faster
    // than overlapping them).
    const int chain_sms = RELU ? 0 : std::min(2 * p.BH, nsm / 2);
    const int share = nchunks > 1 ? nsm - chain_sms : nsm;
    cudaStream_t s_chain = RELU ? st : cx.s_chain, s_out = RELU ? st : cx.s_out;
    const int thr = RELU ? 320 : 192;
    float* st_ws = reinterpret_cast<float*>(ws + L.state);
    float* z_ws = reinterpret_cast<float*>(ws + L.z);

    auto ok = [&](cudaError_t x) {
        if (x != cudaSuccess && e == cudaSuccess) e = x;
        return e == cudaSuccess;
    };
    ok(cudaEventRecord(cx.start, st));
    ok(cudaStreamWaitEvent(s_chain, cx.start, 0));
    ok(cudaStreamWaitEvent(s_out, cx.start, 0));
    int last_b = 0;
    for (int ci = 0; ci < nchunks && e == cudaSuccess; ++ci) {
        const int b = ci & 1;
        const bool first = ci == 0, last = ci == nchunks - 1;
        p.f0 = ci * L.Fc;
        p.Fc = std::min(L.Fc, p.F - p.f0);
        p.gimg = ws + L.gimg[b];
        p.btil = reinterpret_cast<uint4*>(ws + L.btil[b]);
        p.bmat = reinterpret_cast<float*>(ws + L.bmat[b]);
        p.dz = reinterpret_cast<float*>(ws + L.dz[b]);
        p.mimg = ws + L.mimg[b];
        p.zf = reinterpret_cast<float*>(ws + L.zf[b]);
        p.state_in = first ? a.state_in : st_ws;
        p.z_in = first ? a.z_in : z_ws;
        p.state_out = last ? a.state_out : st_ws;
        p.z_out = last ? a.z_out : z_ws;
        const int items = p.BH * p.Fc * 2;
        const int grid = std::min(items, share);
        // gram(c) overwrites the buffers chain(c - 2) read
        if (ci >= 2) ok(cudaStreamWaitEvent(st, cx.chain[b], 0));
        if (pair) {
            // one CTA pair per (b, h, f); the grid is a whole number of pairs
            const int grid2 = 2 * std::max(1, std::min(p.BH * p.Fc, share / 2));
            if (!RELU && p.beta_tok)
                wide_gram_pair_kernel<false, true>
                    <<<grid2, wide_gram_threads(true), kSmemWidePair, st>>>(p, mK, mV);
            else
                wide_gram_pair_kernel<RELU>
                    <<<grid2, wide_gram_threads(RELU), kSmemWidePair, st>>>(p, mK, mV);
        } else if (!RELU && p.beta_tok) {
            wide_gram_kernel<false, true><<<grid, wide_gram_threads(true), kSmemWideGram, st>>>(p, mK, mV);
        } else {
            wide_gram_kernel<RELU><<<grid, wide_gram_threads(RELU), kSmemWideGram, st>>>(p, mK, mV);
        }
        ok(cudaGetLastError());
        ok(cudaEventRecord(cx.gram[b], st));
        // chain(c) needs gram(c), and overwrites the images output(c - 2) read
        ok(cudaStreamWaitEvent(s_chain, cx.gram[b], 0));
        if (ci >= 2 && p.want_output) ok(cudaStreamWaitEvent(s_chain, cx.out[b], 0));
        if (RELU)
            wide_chain_relu_kernel<<<p.BH * 8, 256, 0, s_chain>>>(p);
        else
            wide_chain_gdn_kernel<<<p.BH * 2, 352, kSmemWideChain, s_chain>>>(p);
        ok(cudaGetLastError());
        ok(cudaEventRecord(cx.chain[b], s_chain));
        if (p.want_output) {
            ok(cudaStreamWaitEvent(s_out, cx.chain[b], 0));
            const int grid_o = std::min(p.BH * p.Fc, share);     // one item per frame
            wide_output_kernel<RELU><<<grid_o, thr, smem_wide_out<RELU>(), s_out>>>(p, mQ, mO);
            ok(cudaGetLastError());
            ok(cudaEventRecord(cx.out[b], s_out));
        }
        last_b = b;
    }
    // join: the caller's stream continues after the last chain and output
    cudaError_t j = cudaStreamWaitEvent(st, cx.chain[last_b], 0);
    if (j == cudaSuccess && p.want_output) j = cudaStreamWaitEvent(st, cx.out[last_b], 0);
    if (e == cudaSuccess) e = j;
    return e;
}

}  // namespace

bool wide_eligible(const ScanArgs& a) {
    return a.bf16 && a.D > 128 && a.D <= 256 && a.F > 0;
}

size_t wide_workspace_bytes(const ScanArgs& a) { return wide_layout(a).total; }

int wide_kernel_count(const ScanArgs& a) {
    const int n = (a.F + wide_chunk(a.F) - 1) / wide_chunk(a.F);
    return (a.o ? 3 : 2) * n;
}

cudaError_t launch_wide(const ScanArgs& a, cudaStream_t st) {
    return a.mode == LA_MODE_RELU ? launch_wide_mode<true>(a, st) : launch_wide_mode<false>(a, st);
}

}  // namespace la
