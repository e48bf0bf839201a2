// Tensor-core (tcgen05) scan for bf16 inputs and 64 <= D <= 128.
//
// The scan is split along what depends on what:
//
//   gram   (frame-parallel)  per (b, h, f): stream K_f, V_f through TMA and
//          contract over the frame's tokens on the tensor core.
//            GDN : G'_f = beta kappa^2 K^T K  (bf16 operand image)
//                  B_f  = beta kappa   K^T V  (fp32)
//            ReLU: dM_f = phi(K)^T V (fp32), dz_f = phi(K)^T 1 (fp32)
//   chain  (sequential per (b, h)): the fp32 state lives in tensor memory.
//            GDN : M_f = alpha_f (M_{f-1} - G'_f bf16(M_{f-1})) + B_f
//                  (one D x D x D MMA per frame, negated A accumulated onto M)
//            ReLU: M_f = M_{f-1} + dM_f,  z_f = z_{f-1} + dz_f
//          and publishes bf16(M_f) as an MMA operand image for the outputs.
//   output (frame-parallel)  per (b, h, f): O_f = Q~_f bf16(M_f), with the
//          ReLU feature map and the normaliser phi(Q) z_f + eps fused.
//
// This is the frame-wise Gated DeltaNet of the SANA-WM paper summary
// (section 3, "Hybrid GDN/Softmax Attention"), written in its affine form
// M_f = A_f M_{f-1} + B_f with A_f = alpha_f (I - beta_f Kh^T Kh) -- the same
// per-frame affine map whose composites the paper's context-parallel training
// exchanges (appendix C.1) -- and the block-causal ReLU linear attention of
// the SANA-Video talk (block KV cache segment).
//
// Variants.  Interval composites (SANA-WM paper summary, appendix C.1,
// context-parallel training) run the gram once and the chain on 2 BH
// blocks: from a zero state (input composite) and, without the input term,
// from the identity (transition composite).
// The reversed GDN scan reset at chunk boundaries (SANA-WM paper
// summary, section 3, "Chunk-causal deployment") changes only the chain:
// its frame order and a zero state at each chunk start.  The per-token
// update gate (section 3, "Hybrid GDN/Softmax Attention") changes only the
// gram: each token row of K and V is scaled by sqrt(beta_t) before the
// contractions, which then give Kh^T diag(beta) Kh and Kh^T diag(beta) V.
//
// Pipeline.  Clips of 32+ frames with few enough heads run as chunks of
// frames: chain(c) on its own SMs beside gram(c + 1) and output(c - 1), on
// streams forked from and joined to the caller's, with the fp32 state
// carried between the chunk launches.
//
// Layouts.  q, k, v, o are viewed by TMA as [B*H*F][S][D] bf16 with a 64-wide
// (128-byte) swizzled box; out-of-range tokens and columns read as zero.
// Operand images in the workspace are byte-exact shared-memory images
// (128 B rows, 128-byte swizzle, two 64-column blocks of 16 KB):
//   G' image: K-major, row i = key dim, columns = key dim (symmetric).
//   M  image: MN-major, row i = key dim, columns = value dim.
// The fp32 per-frame matrices B_f / dM_f are stored "quad-interleaved":
// element (i, j) at ((j / 4) * 128 + i) * 4 + j % 4, so that the 32 lanes of
// a warp, which own 32 consecutive rows, touch 512 contiguous bytes.
#include <algorithm>
#include <cstdlib>
#include <mutex>

#include "tc_common.cuh"
#include "tmap.cuh"

namespace la {
namespace {

using namespace tc;

constexpr int kTokG = 64;                   // tokens per gram tile
constexpr int kTokO = 128;                  // tokens per output tile
constexpr int kGStages = 4;                 // gram TMA ring depth
constexpr int kCStages = 2;                 // chain operand ring depth
constexpr int kOStages = 2;                 // output Q ring depth
constexpr int kOAcc = 4;                    // output accumulator slots (128 cols each)
constexpr uint32_t kBoxG = 64 * kTokG * 2;  // 8 KB: one 64-column box of a gram tile
constexpr uint32_t kBoxO = 64 * kTokO * 2;  // 16 KB: one 64-column box of an output tile
constexpr uint32_t kImg = 2 * 16384;        // 32 KB: 128 rows x 128 columns bf16 image
constexpr uint32_t kQuadMat = 128 * 128 * 4;// 64 KB: fp32 128 x 128 quad-interleaved
constexpr int kEpiThreads = 128;            // 4 epilogue warps

struct TcParams {
    const float* alpha;
    const float* beta;
    const float* state_in;
    const float* z_in;
    float* state_out;
    float* z_out;
    unsigned int* status;   // workspace header (status, where)
    uint8_t* gimg;          // [BHF] x kImg          (GDN)
    float* bmat;            // [BHF] x 128 x 128 fp32 quad-interleaved
    uint8_t* mimg;          // [BHF] x kImg
    float* dz;              // [BHF] x 128           (ReLU)
    float* zf;              // [BHF] x 128           (ReLU)
    float k_scale;
    float eps;
    int BH, F, S, D;
    int want_output;
    int rev_chunk;          // > 0: reversed GDN scan reset every rev_chunk frames
    const float* beta_tok;  // per-token update gate [BHF][S] (GDN), or NULL
    int f0, Fc;             // this launch covers frames [f0, f0 + Fc) of every head
    int bh0;                // ... of heads bh0 .. bh0 + BH - 1 (BH: heads of this launch)
    float* trans_out;       // GDN interval composite: chain blocks BH .. 2 BH - 1 leave
                            // the transition A_F ... A_1 here, or NULL
};

// Global frame index (into q, k, v, o, the gates and the per-frame workspace
// buffers, all sized for the whole clip and every head) of launch-local item
// `it` = bh Fc + fl.
__device__ __forceinline__ int global_item(const TcParams& p, int it) {
    const int bh = it / p.Fc;
    return (p.bh0 + bh) * p.F + p.f0 + (it - bh * p.Fc);
}

// ============================================================================
// gram: per-frame contractions over tokens
// ============================================================================
// warp 0: TMA producer; warp 1: TMEM owner + MMA issuer; warps 2-5: epilogue;
// warps 6-9 (ReLU): apply phi to each K tile in shared memory before the MMA;
// (GDN with a per-token update gate, TOKB): scale every token row of the K and
// V tiles by sqrt(beta_t), so that the unchanged MMAs produce
// Kh^T diag(beta) Kh and Kh^T diag(beta) V.
template <bool RELU, bool TOKB = false>
__global__ void __launch_bounds__((RELU || TOKB) ? 320 : 192, 1)
tc_gram_kernel(const TcParams p, const __grid_constant__ CUtensorMap mapK,
               const __grid_constant__ CUtensorMap mapV) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* ring = smem;                              // kGStages x (K 16 KB | V 16 KB)
    uint8_t* stage_img = ring + kGStages * 32768;      // G' image staging (GDN)
    uint8_t* ones = stage_img + kImg;                  // 2 KB of bf16 1.0 (ReLU)
    uint64_t* full = reinterpret_cast<uint64_t*>(ones + 2048);
    uint64_t* empty = full + kGStages;
    uint64_t* xform = empty + kGStages;
    uint64_t* accfull = xform + kGStages;
    uint64_t* accempty = accfull + 2;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accempty + 2);
    uint32_t* abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kGStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&xform[s], 4);
        }
        for (int a = 0; a < 2; ++a) {
            mbar_init(&accfull[a], 1);
            mbar_init(&accempty[a], 4);
        }
        *abort_flag = 0;
        fence_mbar_init();
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
    const int nitems = p.BH * p.Fc;
    const int nt = (p.S + kTokG - 1) / kTokG;
    const int D = p.D;

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&mapK);
            tma_prefetch_desc(&mapV);
            const uint64_t pol = policy_evict_first();
            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            PhaseLog armed;     // loads in flight are waited for after an abort
            for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
            const int item = global_item(p, it);
                for (int t = 0; t < nt; ++t) {
                    if (!(ok = mbar_wait(&empty[s], ph ^ 1, ab, 0x101))) break;
                    uint8_t* st = ring + s * 32768;
                    mbar_expect_tx(&full[s], 4 * kBoxG);
                    tma_load_3d(st, &mapK, &full[s], 0, t * kTokG, item, pol);
                    tma_load_3d(st + kBoxG, &mapK, &full[s], 64, t * kTokG, item, pol);
                    tma_load_3d(st + 16384, &mapV, &full[s], 0, t * kTokG, item, pol);
                    tma_load_3d(st + 16384 + kBoxG, &mapV, &full[s], 64, t * kTokG, item, pol);
                    armed.note(s, ph);
                    if (++s == kGStages) { s = 0; ph ^= 1; }
                }
            }
            armed.drain_if_aborted(full, kGStages, ab);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idKK = idesc_bf16(128, D, true, true);
            const uint32_t idZ = idesc_bf16(128, 16, true, false);
            const uint64_t ones_d = sdesc_sw128(smem_u32(ones), 16, 1024);
            int s = 0, li = 0;
            uint32_t ph = 0;
            bool ok = true;
            PhaseLog armed;
            for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x, ++li) {
            const int item = global_item(p, it);
                const int slot = li & 1;
                if (!(ok = mbar_wait(&accempty[slot], ((li >> 1) & 1) ^ 1, ab, 0x102))) break;
                tc_fence_after();
                const uint32_t dG = tbase + slot * 256, dW = dG + 128;
                for (int t = 0; t < nt; ++t) {
                    if (!(ok = mbar_wait((RELU || TOKB) ? &xform[s] : &full[s], ph, ab, 0x103)))
                        break;
                    tc_fence_after();
                    const uint32_t sk = smem_u32(ring + s * 32768), sv = sk + 16384;
#pragma unroll
                    for (int k = 0; k < kTokG / 16; ++k) {
                        const uint64_t ad = sdesc_sw128(sk + k * 2048, kBoxG, 1024);
                        const uint64_t bv = sdesc_sw128(sv + k * 2048, kBoxG, 1024);
                        const uint32_t acc = (t | k) ? 1u : 0u;
                        if (RELU) {
                            mma_bf16(dW, ad, bv, idKK, acc);
                            mma_bf16(dG, ad, ones_d, idZ, acc);
                        } else {
                            mma_bf16(dG, ad, ad, idKK, acc);
                            mma_bf16(dW, ad, bv, idKK, acc);
                        }
                    }
                    mma_commit(&empty[s]);
                    armed.note(s, ph);
                    if (++s == kGStages) { s = 0; ph ^= 1; }
                }
                if (ok) mma_commit(&accfull[slot]);
            }
            armed.drain_if_aborted(empty, kGStages, ab);    // MMAs in flight
        }
    } else if (warp < 6) {
        // ---------------- epilogue: TMEM -> workspace ----------------
        const int q = warp & 3, row = q * 32 + lane;
        const bool issuer = (threadIdx.x == 64);
        int li = 0;
        bool ok = true;     // every epilogue warp runs every named barrier, even after an abort
        for (int it = blockIdx.x; it < nitems; it += gridDim.x, ++li) {
            const int item = global_item(p, it);
            const int slot = li & 1;
            ok = ok && mbar_wait(&accfull[slot], (li >> 1) & 1, ab, 0x104);
            tc_fence_after();
            const uint32_t tl = tbase + (uint32_t(q * 32) << 16) + slot * 256;
            float* bq = p.bmat + (size_t)item * (kQuadMat / 4);
            if (!RELU) {
                const float bt = TOKB ? 1.f : p.beta[item];   // TOKB: beta is in the operands
                const float sg = bt * p.k_scale * p.k_scale, sw = bt * p.k_scale;
                if (issuer) bulk_wait_read<0>();       // staging free again
                named_bar_sync(1, kEpiThreads);
                for (int c0 = 0; c0 < D && ok; c0 += 64) {
                    float v[4][16];
                    const int nu = min(4, (D - c0) / 16);
                    tmem_ld64(tl + c0, nu, v);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (u < nu) {
#pragma unroll
                            for (int e = 0; e < 16; ++e) v[u][e] *= sg;
                            store_row16_bf16(stage_img, row, c0 + 16 * u, v[u]);
                        }
                }
                for (int c0 = 0; c0 < D && ok; c0 += 64) {
                    float v[4][16];
                    const int nu = min(4, (D - c0) / 16);
                    tmem_ld64(tl + 128 + c0, nu, v);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (u < nu)
#pragma unroll
                            for (int w = 0; w < 4; ++w)
                                *reinterpret_cast<float4*>(bq + (((c0 + 16 * u) / 4 + w) * 128 + row) * 4) =
                                    make_float4(v[u][4 * w] * sw, v[u][4 * w + 1] * sw,
                                                v[u][4 * w + 2] * sw, v[u][4 * w + 3] * sw);
                }
            } else if (ok) {
                for (int c0 = 0; c0 < D; c0 += 64) {
                    float v[4][16];
                    const int nu = min(4, (D - c0) / 16);
                    tmem_ld64(tl + 128 + c0, nu, v);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (u < nu)
#pragma unroll
                            for (int w = 0; w < 4; ++w)
                                *reinterpret_cast<float4*>(bq + (((c0 + 16 * u) / 4 + w) * 128 + row) * 4) =
                                    make_float4(v[u][4 * w], v[u][4 * w + 1], v[u][4 * w + 2],
                                                v[u][4 * w + 3]);
                }
                float v[16];
                tmem_ld16(tl, v);
                tmem_wait_ld();
                p.dz[(size_t)item * 128 + row] = v[0];
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&accempty[slot]);
            if (!RELU) {
                fence_proxy_async_smem();
                named_bar_sync(1, kEpiThreads);
                if (issuer && ok) {
                    bulk_store(p.gimg + (size_t)item * kImg, stage_img, kImg);
                    bulk_commit();
                }
            }
        }
        if (issuer) bulk_wait_all<0>();
    } else {
        // ---------------- transform: phi(K) (ReLU) or sqrt(beta_t) rows (TOKB) ----------------
        const int tl = threadIdx.x - 192;          // 0..127
        int s = 0;
        uint32_t ph = 0;
        bool ok = true;
        // TOKB: chunk i = tl + 128 m of a stage lies in token row (tl / 8 + 16 m) % 64,
        // so a thread needs the gates of 4 rows per tile; they are fetched one
        // tile ahead.
        auto gates4 = [&](int item, int t, float (&w)[4]) {
            const float* bq = p.beta_tok + (size_t)item * p.S;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int tok = t * kTokG + (tl >> 3) + 16 * u;
                w[u] = tok < p.S ? __ldg(bq + tok) : 0.f;
            }
        };
        float wn[4] = {0.f, 0.f, 0.f, 0.f};
        if (TOKB && (int)blockIdx.x < nitems) gates4(global_item(p, blockIdx.x), 0, wn);
        for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x) {
            const int item = global_item(p, it);
            for (int t = 0; t < nt; ++t) {
                float w[4];
#pragma unroll
                for (int u = 0; u < 4; ++u) w[u] = sqrtf(wn[u]);
                if (TOKB) {                                   // the next tile's gates
                    if (t + 1 < nt) gates4(item, t + 1, wn);
                    else if (it + (int)gridDim.x < nitems)
                        gates4(global_item(p, it + gridDim.x), 0, wn);
                }
                if (!(ok = mbar_wait(&full[s], ph, ab, 0x105))) break;
                uint4* kt = reinterpret_cast<uint4*>(ring + s * 32768);
                if (TOKB) {
                    // all 32 KB of the stage (K and V, both 64-column boxes): 64 token
                    // rows of 128 bytes per box; a row's 16-byte chunks are permuted
                    // by the swizzle but stay in the row, so row scaling ignores it
#pragma unroll 4
                    for (int m = 0; m < 16; ++m) {
                        const int i = tl + 128 * m;
                        const float ww = w[m & 3];
                        uint4 x = kt[i];
                        x.x = pack_bf16x2(bf16_lo(x.x) * ww, bf16_hi(x.x) * ww);
                        x.y = pack_bf16x2(bf16_lo(x.y) * ww, bf16_hi(x.y) * ww);
                        x.z = pack_bf16x2(bf16_lo(x.z) * ww, bf16_hi(x.z) * ww);
                        x.w = pack_bf16x2(bf16_lo(x.w) * ww, bf16_hi(x.w) * ww);
                        kt[i] = x;
                    }
                } else {
                    for (int i = tl; i < 2 * (int)kBoxG / 16; i += 128) {
                        uint4 x = kt[i];
                        x.x = relu_bf16x2(x.x); x.y = relu_bf16x2(x.y);
                        x.z = relu_bf16x2(x.z); x.w = relu_bf16x2(x.w);
                        kt[i] = x;
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&xform[s]);
                if (++s == kGStages) { s = 0; ph ^= 1; }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tbase, 512);
}

// ============================================================================
// chain: the per-(b, h) recurrence, state resident in tensor memory
// ============================================================================
// warp 0: bulk loader of the per-frame operands; warp 1: TMEM owner + MMA
// issuer (GDN); warps 2-9: epilogue (thread <-> state row and column half).
constexpr int kChainEpi = 256;
constexpr int kChainThreads = 64 + kChainEpi;
template <bool RELU>
__global__ void __launch_bounds__(kChainThreads, 1)
tc_chain_kernel(const TcParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    // stage s: [G' image 32 KB (GDN)] [B / dM 64 KB] [dz 512 B (ReLU)]
    constexpr uint32_t kStage = (RELU ? 0 : kImg) + kQuadMat + (RELU ? 512 : 0);
    uint8_t* ring = smem;
    uint8_t* mimg = ring + kCStages * kStage;          // bf16(M) operand image
    mimg = align1024(mimg);
    uint64_t* full = reinterpret_cast<uint64_t*>(mimg + kImg);
    uint64_t* empty = full + kCStages;
    uint64_t* mdone = empty + kCStages;    // MMA of the frame finished
    uint64_t* mready = mdone + 1;          // image of the current state written
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(mready + 1);
    uint32_t* abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    // Interval composites (trans_out set): blocks BH .. 2 BH - 1 run the same
    // recurrence from the identity without the input term, which leaves the
    // transition composite A_F ... A_1; blocks 0 .. BH - 1 leave the input
    // composite (the state from zero).
    const bool trans = p.trans_out && (int)blockIdx.x >= p.BH;
    const int bh = p.bh0 + (trans ? (int)blockIdx.x - p.BH : (int)blockIdx.x);
    const int F = p.F, D = p.D;
    const int nsteps = p.Fc;                // steps of this launch: clip steps f0 .. f0 + Fc - 1
    if (threadIdx.x == 0) {
        for (int s = 0; s < kCStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], RELU ? 8 : 9);     // epilogue warps (+ the MMA for GDN)
        }
        mbar_init(mdone, 1);
        mbar_init(mready, 8);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, 128);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tM = *tmem_slot;
    const Abort ab{abort_flag, p.status};

    if (warp == 0) {
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            PhaseLog armed;     // loads in flight are waited for after an abort
            for (int f = 0; f < nsteps; ++f) {
                if (!mbar_wait(&empty[s], ph ^ 1, ab, 0x201)) break;
                const size_t frame = (size_t)bh * F + step_frame(p.f0 + f, F, p.rev_chunk);
                uint8_t* st = ring + s * kStage;
                if (!RELU) {
                    mbar_expect_tx(&full[s], trans ? kImg : kStage);
                    bulk_load(st, p.gimg + frame * kImg, kImg, &full[s]);
                    if (!trans)
                        bulk_load(st + kImg, p.bmat + frame * (kQuadMat / 4), kQuadMat, &full[s]);
                } else {
                    mbar_expect_tx(&full[s], kStage);
                    bulk_load(st, p.bmat + frame * (kQuadMat / 4), kQuadMat, &full[s]);
                    bulk_load(st + kQuadMat, p.dz + frame * 128, 512, &full[s]);
                }
                armed.note(s, ph);
                if (++s == kCStages) { s = 0; ph ^= 1; }
            }
            armed.drain_if_aborted(full, kCStages, ab);
        }
    } else if (warp == 1) {
        if (!RELU && lane == 0) {
            const uint32_t idC = idesc_bf16(128, D, false, true, /*negate_a=*/true);
            int s = 0;
            uint32_t ph = 0;
            PhaseLog armed;     // MMAs in flight are waited for after an abort
            for (int f = 0; f < nsteps; ++f) {
                if (!mbar_wait(&full[s], ph, ab, 0x202)) break;
                if (!mbar_wait(mready, f & 1, ab, 0x203)) break;
                tc_fence_after();
                const uint32_t ga = smem_u32(ring + s * kStage), mb = smem_u32(mimg);
                for (int kk = 0; kk < D / 16; ++kk) {
                    const uint64_t ad = sdesc_sw128(ga + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                    const uint64_t bd = sdesc_sw128(mb + kk * 2048, 16384, 1024);
                    mma_bf16(tM, ad, bd, idC, 1u);
                }
                mma_commit(mdone);
                mma_commit(&empty[s]);
                armed.note(s, ph);
                if (++s == kCStages) { s = 0; ph ^= 1; }
            }
            armed.drain_if_aborted(empty, kCStages, ab);
        }
    } else {
        // ------------- epilogue: thread <-> (state row, column half) -------------
        // warps 2-9: TMEM lane quadrant q = warp % 4 (the rows it may access),
        // column half h; two 16-column TMEM loads in flight per wait
        const int q = warp & 3, row = q * 32 + lane;
        const int h = (warp - 2) >> 2;
        const int c_mid = ((D / 16 + 1) / 2) * 16;
        const int c_lo = h ? c_mid : 0, c_hi = h ? D : c_mid;
        const bool issuer = (threadIdx.x == 64);
        const uint32_t tl = tM + (uint32_t(q * 32) << 16);
        const bool live = row < D;
        // initial state: TMEM (fp32) and operand image (bf16); the row's
        // columns c_lo .. c_hi - 1 (at most 64) arrive as float4 loads, all
        // in flight at once
        {
            const float* src = (!trans && p.state_in && live)
                                   ? p.state_in + ((size_t)bh * D + row) * D : nullptr;
            float4 r[16];
#pragma unroll
            for (int u = 0; u < 16; ++u)
                r[u] = (src && c_lo + 4 * u < c_hi)
                           ? __ldg(reinterpret_cast<const float4*>(src + c_lo + 4 * u))
                           : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const int c0 = c_lo + 16 * k;
                if (c0 < c_hi) {
                    float v[16];
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        v[4 * u] = r[4 * k + u].x;
                        v[4 * u + 1] = r[4 * k + u].y;
                        v[4 * u + 2] = r[4 * k + u].z;
                        v[4 * u + 3] = r[4 * k + u].w;
                    }
                    if (trans)
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] = (row == c0 + e) ? 1.f : 0.f;
                    tmem_st16(tl + c0, v);
                    store_row16_bf16(mimg, row, c0, v);
                }
            }
        }
        float z = 0.f;
        if (RELU && h == 0 && p.z_in && live) z = p.z_in[(size_t)bh * D + row];
        tmem_wait_st();
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(mready);

        // the decay of step f + 1 is read during step f
        auto alpha_of = [&](int f) -> float {
            if (RELU || f >= nsteps) return 1.f;
            return __ldg(p.alpha + (size_t)bh * F + step_frame(p.f0 + f, F, p.rev_chunk));
        };
        float al_next = alpha_of(0);
        int s = 0;
        uint32_t ph = 0;
        bool ok = true;     // every epilogue warp runs every named barrier, even after an abort
        for (int f = 0; f < nsteps; ++f) {
            const size_t frame = (size_t)bh * F + step_frame(p.f0 + f, F, p.rev_chunk);
            // first frame of a chunk of the reversed scan: the state restarts
            // from zero, so whatever the MMA left in TMEM is not used
            const bool reset = step_resets(p.f0 + f, p.rev_chunk);
            ok = ok && mbar_wait(&full[s], ph, ab, 0x204);
            if (!RELU) ok = ok && mbar_wait(mdone, f & 1, ab, 0x205);
            tc_fence_after();
            const float al = al_next;
            al_next = alpha_of(f + 1);
            const uint8_t* st = ring + s * kStage;
            const float* bq = reinterpret_cast<const float*>(st + (RELU ? 0 : kImg));
            if (issuer && p.want_output) bulk_wait_read<0>();   // image free for rewriting
            named_bar_sync(1, kChainEpi);
            const bool last = (f == nsteps - 1);
            float* sout = trans ? p.trans_out : p.state_out;
            for (int c0 = c_lo; c0 < c_hi && ok; c0 += 32) {
                const bool two = c0 + 16 < c_hi;
                float v0[16], v1[16];
                tmem_ld16(tl + c0, v0);
                if (two) tmem_ld16(tl + c0 + 16, v1);
                float4 b[8];
#pragma unroll
                for (int u = 0; u < 8; ++u)
                    b[u] = (trans || (u >= 4 && !two))
                               ? make_float4(0.f, 0.f, 0.f, 0.f)
                               : *reinterpret_cast<const float4*>(bq + ((c0 / 4 + u) * 128 + row) * 4);
                tmem_wait_ld();
                // reset: the state restarts from B (the TMEM value is not read,
                // so a non-finite leftover cannot leak in)
                auto upd = [&](float& x, float bv) { x = reset ? bv : fmaf(al, x, bv); };
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    upd(v0[4 * u], b[u].x);
                    upd(v0[4 * u + 1], b[u].y);
                    upd(v0[4 * u + 2], b[u].z);
                    upd(v0[4 * u + 3], b[u].w);
                    upd(v1[4 * u], b[4 + u].x);
                    upd(v1[4 * u + 1], b[4 + u].y);
                    upd(v1[4 * u + 2], b[4 + u].z);
                    upd(v1[4 * u + 3], b[4 + u].w);
                }
                tmem_st16(tl + c0, v0);
                store_row16_bf16(mimg, row, c0, v0);
                if (two) {
                    tmem_st16(tl + c0 + 16, v1);
                    store_row16_bf16(mimg, row, c0 + 16, v1);
                }
                if (last && sout && live) {
                    float* so = sout + ((size_t)bh * D + row) * D + c0;
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        *reinterpret_cast<float4*>(so + 4 * u) =
                            make_float4(v0[4 * u], v0[4 * u + 1], v0[4 * u + 2], v0[4 * u + 3]);
                    if (two)
#pragma unroll
                        for (int u = 0; u < 4; ++u)
                            *reinterpret_cast<float4*>(so + 16 + 4 * u) =
                                make_float4(v1[4 * u], v1[4 * u + 1], v1[4 * u + 2], v1[4 * u + 3]);
                }
            }
            if (RELU && h == 0 && ok) {
                z += reinterpret_cast<const float*>(st + kQuadMat)[row];
                if (p.want_output) p.zf[frame * 128 + row] = z;
                if (last && p.z_out && live) p.z_out[(size_t)bh * D + row] = z;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);     // this warp is done with stage s
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(1, kChainEpi);
            if (issuer && p.want_output && ok) {
                bulk_store(p.mimg + frame * kImg, mimg, kImg);
                bulk_commit();
            }
            if (lane == 0) mbar_arrive(mready);
            if (++s == kCStages) { s = 0; ph ^= 1; }
        }
        if (issuer) bulk_wait_all<0>();
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tM, 128);
}

// ============================================================================
// output: O_f = Q~_f bf16(M_f)   (ReLU: / (phi(Q_f) z_f + eps))
// ============================================================================
// warp 0: producer (M image + z by bulk copy, Q tiles by TMA); warp 1: TMEM
// owner + MMA issuer; warps 2-5: epilogue (TMEM -> bf16 -> TMA store);
// warps 6-9 (ReLU): phi(Q) in place and the per-token denominators.
template <bool RELU>
__global__ void __launch_bounds__(RELU ? 320 : 192, 1)
tc_output_kernel(const TcParams p, const __grid_constant__ CUtensorMap mapQ,
                 const __grid_constant__ CUtensorMap mapO) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    uint8_t* qring = smem;                             // kOStages x 32 KB
    uint8_t* mbuf = qring + kOStages * 32768;          // 2 x 32 KB M images
    uint8_t* ostage = mbuf + 2 * kImg;                 // 2 x 32 KB output staging
    float* zbuf = reinterpret_cast<float*>(ostage + 2 * 32768);   // 2 x 128
    float* denbuf = zbuf + 2 * 128;                                // kOAcc x 128
    uint64_t* qfull = reinterpret_cast<uint64_t*>(denbuf + kOAcc * 128);
    uint64_t* qempty = qfull + kOStages;
    uint64_t* xform = qempty + kOStages;
    uint64_t* mfull = xform + kOStages;
    uint64_t* mempty = mfull + 2;
    uint64_t* accfull = mempty + 2;
    uint64_t* accempty = accfull + kOAcc;
    uint64_t* denready = accempty + kOAcc;     // ReLU denominators of a slot written
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(denready + kOAcc);
    uint32_t* abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kOStages; ++s) {
            mbar_init(&qfull[s], 1);
            mbar_init(&qempty[s], 1);
            mbar_init(&xform[s], 4);
        }
        for (int m = 0; m < 2; ++m) {
            mbar_init(&mfull[m], 1);
            mbar_init(&mempty[m], RELU ? 5 : 1);
        }
        for (int a = 0; a < kOAcc; ++a) {
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
    const int D = p.D;

    if (warp == 0) {
        if (lane == 0) {
            tma_prefetch_desc(&mapQ);
            tma_prefetch_desc(&mapO);
            const uint64_t pol = policy_evict_first();
            int s = 0, li = 0;
            uint32_t ph = 0;
            bool ok = true;
            PhaseLog armed_q, armed_m;     // loads in flight are waited for after an abort
            for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x, ++li) {
            const int item = global_item(p, it);
                const int mb = li & 1;
                if (!(ok = mbar_wait(&mempty[mb], ((li >> 1) & 1) ^ 1, ab, 0x301))) break;
                mbar_expect_tx(&mfull[mb], kImg + (RELU ? 512 : 0));
                bulk_load(mbuf + mb * kImg, p.mimg + (size_t)item * kImg, kImg, &mfull[mb]);
                if (RELU) bulk_load(zbuf + mb * 128, p.zf + (size_t)item * 128, 512, &mfull[mb]);
                armed_m.note(mb, (li >> 1) & 1);
                for (int t = 0; t < nt; ++t) {
                    if (!(ok = mbar_wait(&qempty[s], ph ^ 1, ab, 0x302))) break;
                    uint8_t* st = qring + s * 32768;
                    mbar_expect_tx(&qfull[s], 2 * kBoxO);
                    tma_load_3d(st, &mapQ, &qfull[s], 0, t * kTokO, item, pol);
                    tma_load_3d(st + kBoxO, &mapQ, &qfull[s], 64, t * kTokO, item, pol);
                    armed_q.note(s, ph);
                    if (++s == kOStages) { s = 0; ph ^= 1; }
                }
            }
            armed_q.drain_if_aborted(qfull, kOStages, ab);
            armed_m.drain_if_aborted(mfull, 2, ab);
        }
    } else if (warp == 1) {
        if (lane == 0) {
            const uint32_t idO = idesc_bf16(128, D, false, true);
            int s = 0, li = 0, gt = 0;
            uint32_t ph = 0;
            bool ok = true;
            PhaseLog armed;     // MMAs in flight are waited for after an abort
            for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x, ++li) {
            const int item = global_item(p, it);
                const int mb = li & 1;
                if (!(ok = mbar_wait(&mfull[mb], (li >> 1) & 1, ab, 0x303))) break;
                const uint32_t mimg_a = smem_u32(mbuf + mb * kImg);
                for (int t = 0; t < nt; ++t, ++gt) {
                    const int a = gt % kOAcc;
                    if (!(ok = mbar_wait(&accempty[a], ((gt / kOAcc) & 1) ^ 1, ab, 0x304))) break;
                    if (!(ok = mbar_wait(RELU ? &xform[s] : &qfull[s], ph, ab, 0x305))) break;
                    tc_fence_after();
                    const uint32_t qa = smem_u32(qring + s * 32768);
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t ad = sdesc_sw128(qa + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                        const uint64_t bd = sdesc_sw128(mimg_a + kk * 2048, 16384, 1024);
                        mma_bf16(tbase + a * 128, ad, bd, idO, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&qempty[s]);
                    mma_commit(&accfull[a]);
                    armed.note(s, ph);
                    if (++s == kOStages) { s = 0; ph ^= 1; }
                }
                if (ok) mma_commit(&mempty[mb]);
            }
            armed.drain_if_aborted(qempty, kOStages, ab);
        }
    } else if (warp < 6) {
        // ---------------- epilogue: TMEM -> bf16 -> TMA store ----------------
        const int q = warp & 3, row = q * 32 + lane;
        const bool issuer = (threadIdx.x == 64);
        int gt = 0;
        bool ok = true;     // every epilogue warp runs every named barrier, even after an abort
        for (int it = blockIdx.x; it < nitems; it += gridDim.x) {
            const int item = global_item(p, it);
            for (int t = 0; t < nt; ++t, ++gt) {
                const int a = gt % kOAcc, ob = gt & 1;
                ok = ok && mbar_wait(&accfull[a], (gt / kOAcc) & 1, ab, 0x306);
                if (RELU) ok = ok && mbar_wait(&denready[a], (gt / kOAcc) & 1, ab, 0x30a);
                tc_fence_after();
                if (issuer) bulk_wait_read<1>();     // staging ob no longer read by its store
                named_bar_sync(1, kEpiThreads);
                uint8_t* os = ostage + ob * 32768;
                const float inv = (RELU && ok) ? 1.f / denbuf[a * 128 + row] : 1.f;
                const uint32_t tl = tbase + (uint32_t(q * 32) << 16) + a * 128;
                for (int c0 = 0; c0 < D && ok; c0 += 64) {
                    float v[4][16];
                    const int nu = min(4, (D - c0) / 16);
                    tmem_ld64(tl + c0, nu, v);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        if (u < nu) {
                            if (RELU) {
#pragma unroll
                                for (int e = 0; e < 16; ++e) v[u][e] *= inv;
                            }
                            store_row16_bf16(os, row, c0 + 16 * u, v[u]);
                        }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&accempty[a]);
                fence_proxy_async_smem();
                named_bar_sync(1, kEpiThreads);
                if (issuer && ok) {
                    tma_store_3d(&mapO, os, 0, t * kTokO, item);
                    if (D > 64) tma_store_3d(&mapO, os + kBoxO, 64, t * kTokO, item);
                    bulk_commit();
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
        for (int it = blockIdx.x; it < nitems && ok; it += gridDim.x, ++li) {
            const int item = global_item(p, it);
            const int mb = li & 1;
            if (!(ok = mbar_wait(&mfull[mb], (li >> 1) & 1, ab, 0x307))) break;
            const float* z = zbuf + mb * 128;
            for (int t = 0; t < nt; ++t, ++gt) {
                const int a = gt % kOAcc;
                if (!(ok = mbar_wait(&qfull[s], ph, ab, 0x308))) break;
                if (!(ok = mbar_wait(&accempty[a], ((gt / kOAcc) & 1) ^ 1, ab, 0x309))) break;
                uint8_t* st = qring + s * 32768;
                float den = 0.f;
                for (int blk = 0; blk < 2; ++blk) {
                    if (blk * 64 >= D) break;
                    for (int c = 0; c < 8; ++c) {
                        uint4* pch = reinterpret_cast<uint4*>(st + blk * 16384 + sw128_off(row, c));
                        uint4 x = *pch;
                        x.x = relu_bf16x2(x.x); x.y = relu_bf16x2(x.y);
                        x.z = relu_bf16x2(x.z); x.w = relu_bf16x2(x.w);
                        *pch = x;
                        const float* zz = z + blk * 64 + c * 8;
                        den = fmaf(bf16_lo(x.x), zz[0], den);
                        den = fmaf(bf16_hi(x.x), zz[1], den);
                        den = fmaf(bf16_lo(x.y), zz[2], den);
                        den = fmaf(bf16_hi(x.y), zz[3], den);
                        den = fmaf(bf16_lo(x.z), zz[4], den);
                        den = fmaf(bf16_hi(x.z), zz[5], den);
                        den = fmaf(bf16_lo(x.w), zz[6], den);
                        den = fmaf(bf16_hi(x.w), zz[7], den);
                    }
                }
                denbuf[a * 128 + row] = den + p.eps;
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&xform[s]);
                    mbar_arrive(&denready[a]);
                }
                if (++s == kOStages) { s = 0; ph ^= 1; }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&mempty[mb]);
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tbase, 512);
}

// ----------------------------------------------------------------------------
// Host side
// ----------------------------------------------------------------------------
struct WsLayout {
    size_t gimg, bmat, mimg, dz, zf, state, z, total;
};

WsLayout ws_layout(const ScanArgs& a) {
    const size_t bhf = (size_t)a.B * a.H * a.F;
    WsLayout L;
    size_t off = kWsHeaderBytes;
    L.gimg = off;
    if (a.mode == LA_MODE_GDN) off += bhf * kImg;
    L.bmat = off;
    off += bhf * kQuadMat;
    L.mimg = off;
    off += bhf * kImg;
    L.dz = off;
    L.zf = off;
    if (a.mode == LA_MODE_RELU) {
        off += bhf * 512;
        L.zf = off;
        off += bhf * 512;
    }
    // state (and z) carried between the chunk launches of the pipeline
    const size_t bh = (size_t)a.B * a.H;
    off = align_up(off, 256);
    L.state = off;
    off += bh * a.D * a.D * 4;
    L.z = off;
    off += bh * a.D * 4;
    L.total = align_up(off, 256);
    return L;
}

constexpr size_t smem_gram = 1024 + kGStages * 32768 + kImg + 2048 + 256;
constexpr size_t smem_chain_gdn = 1024 + kCStages * (kImg + kQuadMat) + 1024 + kImg + 256;
constexpr size_t smem_chain_relu = 1024 + kCStages * (kQuadMat + 512) + 1024 + kImg + 256;
constexpr size_t smem_out = 1024 + kOStages * 32768 + 2 * kImg + 2 * 32768 +
                            (2 + kOAcc) * 512 + 256;
static_assert(smem_chain_gdn <= 232448, "chain smem");
static_assert(smem_out <= 232448, "output smem");

// Frames per pipeline chunk of the three-kernel path: about 8 chunks of at
// least 16 frames, and whole chunks of the reversed scan; one chunk (no
// pipeline) for short clips or when the per-head chain CTAs would take more
// than half of the SMs.
int tc_chunk(const ScanArgs& a, int nsm) {
    int c = a.F;
    if (a.trans_out) return std::max(1, a.F);     // interval composites: one chunk
    if (a.F >= 32 && 2 * a.B * a.H <= nsm) c = std::max(16, (a.F + 7) / 8);
    if (a.rev_chunk > 0) c = (c + a.rev_chunk - 1) / a.rev_chunk * a.rev_chunk;
    if (const char* e = std::getenv("LA_TC_CHUNK")) {
        const int v = std::atoi(e);
        if (v > 0) c = a.rev_chunk > 0 ? (v + a.rev_chunk - 1) / a.rev_chunk * a.rev_chunk : v;
    }
    return std::max(1, std::min(c, std::max(a.F, 1)));
}

constexpr int kMaxHeadGroups = 8;

// Head groups of a one-chunk call.  With a single frame chunk the chain of
// every head waits for the whole gram and holds up the whole output; heads
// are independent, so with two groups the chain of the first half of the
// heads runs beside the gram of the second half.  More groups lose: every
// group's chain still takes its F latency-bound steps and its gram and output
// their fill and drain (LA_TC_HEAD_GROUPS overrides, 1 .. min(B H, 8)).
int tc_head_groups(const ScanArgs& a, int nsm, int Fc) {
    const int BH = a.B * a.H;
    if (a.trans_out || Fc < a.F || a.F < 1) return 1;
    int g = ((long)BH * a.F >= 2L * nsm && BH >= 8) ? 2 : 1;
    if (const char* e = std::getenv("LA_TC_HEAD_GROUPS")) {
        const int v = std::atoi(e);
        if (v > 0) g = std::min(v, std::min(BH, kMaxHeadGroups));
    }
    return g;
}

// Streams and events of one device for the chunk pipeline (gram kernels on
// the caller's stream, chain and output kernels on two streams of the
// library's own, forked from and joined back to the caller's stream).
constexpr int kMaxDevicesTc = 64;
struct TcCtx {
    bool ready = false;
    cudaStream_t s_chain = nullptr, s_out = nullptr;
    cudaEvent_t start = nullptr, gram = nullptr, chain = nullptr, out = nullptr;
    // head groups: chain and output of group g on s_grp[g] (high priority),
    // after its gram (grp_in[g]); the caller's stream joins every grp_done[g]
    bool grp_ready = false;
    cudaStream_t s_grp[kMaxHeadGroups] = {};
    cudaEvent_t grp_in[kMaxHeadGroups] = {}, grp_done[kMaxHeadGroups] = {};
};
std::mutex g_tc_mu[kMaxDevicesTc];
TcCtx g_tc_ctx[kMaxDevicesTc];

cudaError_t tc_ctx_init(TcCtx& c) {
    if (c.ready) return cudaSuccess;
    cudaError_t e = cudaStreamCreateWithFlags(&c.s_chain, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&c.s_out, cudaStreamNonBlocking);
    cudaEvent_t* evs[] = {&c.start, &c.gram, &c.chain, &c.out};
    for (cudaEvent_t* p : evs)
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(p, cudaEventDisableTiming);
    if (e == cudaSuccess) c.ready = true;
    return e;
}

cudaError_t tc_ctx_init_groups(TcCtx& c) {
    if (c.grp_ready) return cudaSuccess;
    int lo = 0, hi = 0;
    cudaError_t e = cudaDeviceGetStreamPriorityRange(&lo, &hi);
    for (int g = 0; g < kMaxHeadGroups && e == cudaSuccess; ++g) {
        e = cudaStreamCreateWithPriority(&c.s_grp[g], cudaStreamNonBlocking, hi);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c.grp_in[g], cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&c.grp_done[g], cudaEventDisableTiming);
    }
    if (e == cudaSuccess) c.grp_ready = true;
    return e;
}

template <bool RELU>
cudaError_t launch_tc_mode(const ScanArgs& a, cudaStream_t st) {
    const WsLayout L = ws_layout(a);
    uint8_t* ws = reinterpret_cast<uint8_t*>(a.ws);
    TcParams p;
    p.alpha = a.alpha;
    p.beta = a.beta;
    p.status = reinterpret_cast<unsigned int*>(ws);
    p.gimg = ws + L.gimg;
    p.bmat = reinterpret_cast<float*>(ws + L.bmat);
    p.mimg = ws + L.mimg;
    p.dz = reinterpret_cast<float*>(ws + L.dz);
    p.zf = reinterpret_cast<float*>(ws + L.zf);
    p.k_scale = a.k_scale;
    p.eps = a.eps;
    p.BH = a.B * a.H;
    p.F = a.F;
    p.S = a.S;
    p.D = a.D;
    p.want_output = a.o != nullptr;
    p.rev_chunk = a.rev_chunk;
    p.beta_tok = a.beta_tok;
    p.trans_out = a.trans_out;
    p.bh0 = 0;

    const uint64_t bhf = (uint64_t)p.BH * p.F;
    CUtensorMap mK, mV, mQ, mO;
    if (!make_tmap_bf16_3d(&mK, a.k, a.D, a.S, bhf, 64, kTokG) ||
        !make_tmap_bf16_3d(&mV, a.v, a.D, a.S, bhf, 64, kTokG))
        return cudaErrorInvalidValue;
    if (p.want_output && (!make_tmap_bf16_3d(&mQ, a.q, a.D, a.S, bhf, 64, kTokO) ||
                          !make_tmap_bf16_3d(&mO, a.o, a.D, a.S, bhf, 64, kTokO)))
        return cudaErrorInvalidValue;

    {
        const void* kernels[] = {reinterpret_cast<const void*>(tc_gram_kernel<RELU>),
                                 reinterpret_cast<const void*>(tc_chain_kernel<RELU>),
                                 reinterpret_cast<const void*>(tc_output_kernel<RELU>),
                                 reinterpret_cast<const void*>(tc_gram_kernel<false, true>)};
        const int bytes[] = {(int)smem_gram, (int)(RELU ? smem_chain_relu : smem_chain_gdn),
                             (int)smem_out, (int)smem_gram};
        for (int i = 0; i < (RELU ? 3 : 4); ++i) {
            const cudaError_t e = ensure_dyn_smem(kernels[i], bytes[i]);
            if (e != cudaSuccess) return e;
        }
    }
    const int nsm = device_sm_count();
    const int Fc = tc_chunk(a, nsm);
    const int nchunks = (p.F + Fc - 1) / Fc;
    const int thr = RELU ? 320 : 192;
    float* st_ws = reinterpret_cast<float*>(ws + L.state);
    float* z_ws = reinterpret_cast<float*>(ws + L.z);
    auto set_chunk = [&](int ci) {
        p.f0 = ci * Fc;
        p.Fc = std::min(Fc, p.F - p.f0);
        p.state_in = ci == 0 ? a.state_in : st_ws;
        p.z_in = ci == 0 ? a.z_in : z_ws;
        p.state_out = ci == nchunks - 1 ? a.state_out : st_ws;
        p.z_out = ci == nchunks - 1 ? a.z_out : z_ws;
    };
    auto gram = [&](int grid, cudaStream_t s) {
        if (!RELU && p.beta_tok)
            tc_gram_kernel<false, true><<<grid, 320, smem_gram, s>>>(p, mK, mV);
        else
            tc_gram_kernel<RELU><<<grid, thr, smem_gram, s>>>(p, mK, mV);
    };
    const int ngroups = nchunks == 1 ? tc_head_groups(a, nsm, Fc) : 1;
    if (nchunks == 1 && ngroups == 1) {
        set_chunk(0);
        const int grid_f = (int)std::min<uint64_t>(bhf, (uint64_t)nsm);
        gram(grid_f, st);
        tc_chain_kernel<RELU><<<p.BH * (p.trans_out ? 2 : 1), kChainThreads,
                                RELU ? smem_chain_relu : smem_chain_gdn, st>>>(p);
        if (p.want_output) tc_output_kernel<RELU><<<grid_f, thr, smem_out, st>>>(p, mQ, mO);
        return cudaGetLastError();
    }
    // Pipeline: chain(c) (one CTA per head, on its own SMs) runs beside
    // gram(c + 1) and output(c - 1), which share the other SMs.  Every chunk
    // writes its own frames of the clip-sized buffers, so only gram -> chain
    // -> output of the same chunk (and chain -> chain through the carried
    // state, in stream order) must be ordered.  A one-chunk call pipelines
    // over head groups instead: a group's launches cover heads
    // [bh0, bh0 + BH) of the same buffers, so again only its own gram ->
    // chain -> output are ordered.
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevicesTc)
        return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_tc_mu[dev]);
    TcCtx& cx = g_tc_ctx[dev];
    cudaError_t e = tc_ctx_init(cx);
    if (e != cudaSuccess) return e;
    auto ok = [&](cudaError_t x) {
        if (x != cudaSuccess && e == cudaSuccess) e = x;
        return e == cudaSuccess;
    };
    if (ngroups > 1) {
        // Head groups: the grams in order on the caller's stream; the chain
        // and output of group g on stream g, so that the chains of several
        // groups (each a few microseconds per frame whatever its head count)
        // overlap one another and the grams and outputs of other groups.
        ok(tc_ctx_init_groups(cx));
        const int BH = p.BH;
        int recorded = 0;
        set_chunk(0);
        for (int g = 0; g < ngroups && e == cudaSuccess; ++g) {
            p.bh0 = (int)((long)g * BH / ngroups);
            p.BH = (int)((long)(g + 1) * BH / ngroups) - p.bh0;
            const int grid = std::min(p.BH * p.Fc, std::max(8, nsm - p.BH));
            cudaStream_t sg = cx.s_grp[g];
            gram(grid, st);
            ok(cudaGetLastError());
            ok(cudaEventRecord(cx.grp_in[g], st));
            ok(cudaStreamWaitEvent(sg, cx.grp_in[g], 0));
            tc_chain_kernel<RELU><<<p.BH, kChainThreads, RELU ? smem_chain_relu : smem_chain_gdn, sg>>>(p);
            ok(cudaGetLastError());
            if (p.want_output) {
                tc_output_kernel<RELU><<<grid, thr, smem_out, sg>>>(p, mQ, mO);
                ok(cudaGetLastError());
            }
            if (ok(cudaEventRecord(cx.grp_done[g], sg))) recorded = g + 1;
        }
        // join: the caller's stream continues after every group's output
        for (int g = 0; g < recorded; ++g) {
            const cudaError_t j = cudaStreamWaitEvent(st, cx.grp_done[g], 0);
            if (j != cudaSuccess && e == cudaSuccess) e = j;
        }
        return e;
    }
    const int share = std::max(8, nsm - p.BH);
    ok(cudaEventRecord(cx.start, st));
    ok(cudaStreamWaitEvent(cx.s_chain, cx.start, 0));
    ok(cudaStreamWaitEvent(cx.s_out, cx.start, 0));
    for (int ci = 0; ci < nchunks && e == cudaSuccess; ++ci) {
        set_chunk(ci);
        const int grid = std::min(p.BH * p.Fc, share);
        gram(grid, st);
        ok(cudaGetLastError());
        ok(cudaEventRecord(cx.gram, st));
        ok(cudaStreamWaitEvent(cx.s_chain, cx.gram, 0));
        tc_chain_kernel<RELU><<<p.BH, kChainThreads, RELU ? smem_chain_relu : smem_chain_gdn, cx.s_chain>>>(p);
        ok(cudaGetLastError());
        ok(cudaEventRecord(cx.chain, cx.s_chain));
        if (p.want_output) {
            ok(cudaStreamWaitEvent(cx.s_out, cx.chain, 0));
            tc_output_kernel<RELU><<<grid, thr, smem_out, cx.s_out>>>(p, mQ, mO);
            ok(cudaGetLastError());
        }
    }
    // join: the caller's stream continues after the last chain and output
    cudaError_t j = cudaEventRecord(cx.out, cx.s_out);
    if (j == cudaSuccess) j = cudaStreamWaitEvent(st, cx.chain, 0);
    if (j == cudaSuccess) j = cudaStreamWaitEvent(st, cx.out, 0);
    if (e == cudaSuccess) e = j;
    return e;
}

}  // namespace

bool tc_eligible(const ScanArgs& a) {
    return a.bf16 && a.D >= 64 && a.D <= 128 && a.F > 0;
}

size_t tc_workspace_bytes(const ScanArgs& a) { return ws_layout(a).total; }

int tc_kernel_count(const ScanArgs& a) {
    const int nsm = device_sm_count();
    const int Fc = tc_chunk(a, nsm);
    const int nchunks = (a.F + Fc - 1) / Fc;
    return (a.o ? 3 : 2) * nchunks * (nchunks == 1 ? tc_head_groups(a, nsm, Fc) : 1);
}

cudaError_t launch_tc(const ScanArgs& a, cudaStream_t st) {
    return a.mode == LA_MODE_RELU ? launch_tc_mode<true>(a, st) : launch_tc_mode<false>(a, st);
}

}  // namespace la
