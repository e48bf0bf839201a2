// Fused persistent tensor-core scan (bf16, 64 <= D <= 128): one cooperative
// launch in which the sequential per-head recurrence runs concurrently with
// the frame-parallel streaming work, handing per-frame operands through small
// L2-resident rings instead of HBM round trips.
//
// Roles (one block per SM, all blocks co-resident):
//   chain blocks  (blockIdx < n_chain): one per head; advances its head frame
//     by frame.  The fp32 state lives in tensor memory; per frame
//        GDN : M_f = alpha_f M_{f-1} + G''_f bf16(M_{f-1}) + B~_f
//              (G''_f = -alpha_f beta_f kappa^2 K_f^T K_f, B~_f = beta_f kappa K_f^T V_f)
//        ReLU: M_f = M_{f-1} + B~_f,  z_f = z_{f-1} + dz_f
//              (B~_f = phi(K_f)^T V_f, dz_f = column sums of phi(K_f))
//     and publishes bf16(M_f) as an MMA operand image.
//   worker blocks (the rest): take items in ticket order from a global
//     counter.  A gram item (b,h,f) streams K_f, V_f and produces the bf16
//     images of G''_f and B~_f (ReLU: B~_f and dz_f); an output item (b,h,f)
//     streams Q_f and produces O_f = Q~_f bf16(M_f) (ReLU: / (phi(Q_f) z_f + eps)).
//
// Ordering and progress.  Tickets list, for frame step j, the gram items of
// frame j of every head and then the output items of frame j - lag.  A gram
// item waits only for its ring slot to be consumed by the chain; an output
// item waits only for the chain to publish its frame.  Every wait is on an
// item with a smaller ticket or on a chain block, and chain blocks are always
// resident, so the smallest unfinished ticket can always proceed.
//
// Hand-off protocol (per head, ring of kRG / kRM slots):
//   gram  -> chain : G'' and B~ images (bulk stores), then
//                    gram_ready[slot] = f + 1 (release)
//   chain -> output: M image (bulk store), then chain_done[head][f & 1] = f + 1
//                    (even and odd frames are published by two threads, each
//                    in frame order, so frame f is out once the flag of its
//                    parity reaches f + 1)
//   output -> chain: mimg_consumed[slot] = f + 1 once the image is in smem
//                    (with output items split in token halves: each half adds 1
//                    and the slot of frame f is free once it counts 2 (f / kRM))
//   chain -> gram  : chain_done[head][g & 1] >= g + 1, g = f - kRG, frees gram
//                    slot f (frame g was consumed before it was published)
// Every spin is bounded; a block that gives up records LA_ERR_TIMEOUT in the
// status word, which makes every other block give up too.
//
// This is the frame-wise Gated DeltaNet of the SANA-WM paper summary
// (section 3, "Hybrid GDN/Softmax Attention") in its affine form, and the
// block-causal ReLU linear attention of the SANA-Video talk (block KV cache
// segment); the cross-block hand-off of per-frame affine summaries mirrors
// the composite exchange of the paper's context-parallel training (appendix
// C.1), applied between blocks of one GPU.
#include <algorithm>
#include <cstdlib>

#include "tc_common.cuh"
#include "tmap.cuh"

namespace la {
namespace {

using namespace tc;

// Tuning knobs (compile-time; the defaults are the measured best).
#ifndef LA_FUSED_WSTAGES
#define LA_FUSED_WSTAGES 4
#endif
#ifndef LA_FUSED_WSTG
#define LA_FUSED_WSTG 2
#endif
#ifndef LA_FUSED_EARLY_Q
#define LA_FUSED_EARLY_Q 1
#endif
#ifndef LA_FUSED_LAG
#define LA_FUSED_LAG 14
#endif
#ifndef LA_FUSED_L2_HINTS
#define LA_FUSED_L2_HINTS 1
#endif
#if LA_FUSED_L2_HINTS
#define LA_POL_KEEP policy_evict_last
#define LA_POL_STREAM policy_evict_first
#else
#define LA_POL_KEEP policy_evict_normal
#define LA_POL_STREAM policy_evict_normal
#endif
#ifndef LA_FUSED_PUB_EVICT_LAST
#define LA_FUSED_PUB_EVICT_LAST 1
#endif
#ifndef LA_FUSED_PUBLAG
#define LA_FUSED_PUBLAG 1
#endif

constexpr int kRG = 16;                 // per-head ring slots: gram -> chain
constexpr int kRM = 16;                 // per-head ring slots: chain -> output
constexpr int kWStages = LA_FUSED_WSTAGES;   // worker TMA ring (32 KB stages)
constexpr int kWStg = LA_FUSED_WSTG;         // worker epilogue staging buffers (16 KB)
constexpr int kCStages = 2;             // chain operand ring depth
constexpr int kIQ = 4;                  // worker item queue depth
constexpr int kThreads = 384;           // 12 warps
constexpr int kTokG = 64, kTokO = 128;
constexpr uint32_t kBoxG = 64 * kTokG * 2;   // 8 KB
constexpr uint32_t kBoxO = 64 * kTokO * 2;   // 16 KB
constexpr uint32_t kImg = 32768;             // bf16 128 x 128 operand image

enum : int { kItemStop = 0, kItemGram = 1, kItemOut = 2 };

// Optional event trace (built only with -DLA_TRACE, for tuning).  Each
// writer (block, role) owns a region of kTraceCap records of two 64-bit
// words {kind << 56 | block << 40 | aux, %globaltimer}; plain stores only.
#ifdef LA_TRACE
constexpr uint32_t kTraceCap = 4096;
constexpr uint32_t kTraceWriters = 6;
__device__ unsigned long long* g_trace = nullptr;
__device__ __forceinline__ void trace_event(uint32_t& n, uint32_t writer, uint32_t kind, uint64_t aux) {
    unsigned long long* t = g_trace;
    if (!t || n >= kTraceCap) return;
    unsigned long long* r = t + 2 * ((size_t)(blockIdx.x * kTraceWriters + writer) * kTraceCap + n++);
    r[0] = ((uint64_t)kind << 56) | ((uint64_t)blockIdx.x << 40) | (aux & 0xFFFFFFFFFFull);
    r[1] = global_timer_ns();
}
#define LA_TRACE_EVENT(kind, aux) trace_event(trace_n, trace_w, (kind), (aux))
#define LA_TRACE_WRITER(w) uint32_t trace_n = 0; const uint32_t trace_w = (w)
#else
#define LA_TRACE_EVENT(kind, aux) ((void)0)
#define LA_TRACE_WRITER(w) ((void)0)
#endif
struct Item {
    int type, bh, f, pad;
};

struct FusedParams {
    const float* alpha;
    const float* beta;
    const float* state_in;
    const float* z_in;
    float* state_out;
    float* z_out;
    unsigned int* status;      // header: [0] status, [1] where, [2] ticket
    uint32_t* chain_done;      // [BH][2]: frames published, per frame parity
    uint32_t* gram_ready;      // [BH][kRG]
    uint32_t* mimg_consumed;   // [BH][kRM]
    uint8_t* gimg;             // [BH][kRG] x kImg  -alpha beta kappa^2 K^T K   (GDN)
    uint8_t* bimg;             // [BH][kRG] x kImg  beta kappa K^T V  /  phi(K)^T V
    float* dz;                 // [BH][kRG] x 128   phi(K)^T 1                    (ReLU)
    uint8_t* mimg;             // [BH][kRM] x kImg
    float* zf;                 // [BH][kRM] x 128             (ReLU)
    float k_scale;
    float eps;
    int BH, F, S, D;
    int want_output;
    int n_chain;
    int heads_per_chain;
    int lag;
    int rev_chunk;             // > 0: reversed GDN scan reset every rev_chunk frames (steps
                               // are processed in scan order; step j is frame step_frame(j))
    const float* beta_tok;     // per-token update gate [BH][F][S] (TOKB instantiation)
    int den_col;               // ReLU, D <= 112: z_f rides in column D (hi) and D + 1 (lo) of
                               // the state image, so one MMA gives numerator and denominator
    int skip_publish;          // test hook: frame of head 0 whose gram_ready is never set
    int out_split;             // output items cover one token half of a frame each (Item.pad)
    // fused input preparation (GDN, PREP instantiation): RMSNorm, ReLU, 3D RoPE of K and Q
    int H;
    const float* q_weight;     // [H, D] or NULL
    const float* k_weight;     // [H, D] or NULL
    float norm_eps;
    int rope, grid_w, grid_max, frame_offset;
    float rope_base;
};

// What the worker's transform warps do to the tiles between TMA and the MMA
// (besides phi in ReLU mode): nothing, the fused input preparation, or the
// per-token update gate's sqrt(beta) row scaling of the gram tiles.
constexpr int kXfNone = 0, kXfPrep = 1, kXfTokB = 2;

// Shared memory of the input preparation, after the worker's own layout:
// the RMSNorm weight row of the current item (D floats), the temporal
// cos/sin of its frame, and the height/width cos/sin table (the two groups
// have the same pair count and frequencies, so one table indexed by
// position serves both).
constexpr uint32_t kPrepSmem = 24576;
constexpr uint32_t kPrepTabEntries = (kPrepSmem - 512 - 512 - 1536) / 8;   // float2 entries

constexpr size_t kWorkerSmem = kWStages * 32768 + kImg + kWStg * 16384 + 2048 + 512 + 2048 + 512 +
                               (kIQ + 2) * sizeof(Item) + 16 +
                               (3 * kWStages + 2 + 12 + 2 * kIQ) * 8 + 8;
constexpr size_t kChainSmem = kCStages * 2 * kImg + 2 * kImg + 1024 + 8 + 12 * 8 + 8 + 8;
constexpr size_t kFusedSmem = 1024 + (kWorkerSmem > kChainSmem ? kWorkerSmem : kChainSmem);
static_assert(kFusedSmem <= 232448, "fused kernel shared memory");
// the preparation region starts at align_up(kWorkerSmem, 16) after the 1024-byte alignment slack
constexpr size_t kFusedSmemPrep =
    1024 + ((kWorkerSmem > kChainSmem ? kWorkerSmem : kChainSmem) + 15) / 16 * 16 + kPrepSmem;
static_assert(kFusedSmemPrep <= 232448, "fused kernel shared memory with the input preparation");

__device__ __forceinline__ Item decode_ticket(const FusedParams& p, uint32_t t) {
    const uint32_t BH = p.BH, F = p.F;
    Item it{kItemStop, 0, 0, 0};
    if (!p.want_output) {
        if (t < BH * F) it = Item{kItemGram, (int)(t % BH), (int)(t / BH), 0};
        return it;
    }
    // output items per (head, frame): the frame, or its two token halves
    // (part in Item.pad; all heads' first halves, then all second halves)
    const uint32_t no = p.out_split ? 2 : 1, per = (1 + no) * BH;
    const uint32_t L = p.lag;
    const uint32_t g0 = min(L, F) * BH;
    if (t < g0) return Item{kItemGram, (int)(t % BH), (int)(t / BH), 0};
    uint32_t u = t - g0;
    const uint32_t nm = F > L ? F - L : 0;
    if (u < nm * per) {
        const uint32_t j = L + u / per, r = u % per;
        if (r < BH) return Item{kItemGram, (int)r, (int)j, 0};
        const uint32_t o = r - BH;
        return Item{kItemOut, (int)(o % BH), (int)(j - L), (int)(o / BH)};
    }
    u -= nm * per;
    const uint32_t f0 = F > L ? F - L : 0;
    if (u < (F - f0) * no * BH) {
        const uint32_t o = u % (no * BH);
        return Item{kItemOut, (int)(o % BH), (int)(f0 + u / (no * BH)), (int)(o / BH)};
    }
    return it;
}

// Output tiles [lo, hi) of an output item: the whole frame, or one of its two
// token halves (split only when a frame has at least two output tiles).
__device__ __forceinline__ void out_range(const FusedParams& p, const Item& it, int nto, int& lo,
                                          int& hi) {
    const int h = (nto + 1) >> 1;
    lo = (p.out_split && it.pad) ? h : 0;
    hi = (p.out_split && !it.pad) ? h : nto;
}

// ============================================================================
// worker blocks
// ============================================================================
template <bool RELU, int XF>
__device__ __forceinline__ void worker_role(const FusedParams& p, uint8_t* smem,
                                            const CUtensorMap* mK, const CUtensorMap* mV,
                                            const CUtensorMap* mQ, const CUtensorMap* mO) {
    constexpr bool PREP = XF == kXfPrep, TOKB = XF == kXfTokB;
    uint8_t* ring = smem;                                  // kWStages x 32 KB
    uint8_t* mbuf = ring + kWStages * 32768;               // M image of the current output item
    uint8_t* stg = mbuf + kImg;                            // kWStg x 16 KB epilogue staging
    uint8_t* ones = stg + kWStg * 16384;                   // 2 KB bf16 1.0 (ReLU)
    float* zbuf = reinterpret_cast<float*>(ones + 2048);   // 128 (ReLU)
    float* denbuf = zbuf + 128;                            // 4 x 128 (ReLU)
    float* dzst = denbuf + 4 * 128;                        // 128: dz_f staging (ReLU)
    Item* items = reinterpret_cast<Item*>(dzst + 128);
    Item* bc_item = items + kIQ;                           // broadcast slots
    int* bc_ok = reinterpret_cast<int*>(bc_item + 2);
    uint64_t* full = reinterpret_cast<uint64_t*>(bc_ok + 4);
    uint64_t* empty = full + kWStages;
    uint64_t* xform = empty + kWStages;
    uint64_t* mfull = xform + kWStages;
    uint64_t* mempty = mfull + 1;
    uint64_t* qfull = mempty + 1;
    uint64_t* qempty = qfull + 4;
    uint64_t* denready = qempty + 4;
    uint64_t* iqfull = denready + 4;
    uint64_t* iqempty = iqfull + kIQ;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(iqempty + kIQ);
    uint32_t* abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kWStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
            mbar_init(&xform[s], (PREP || TOKB) ? 6 : 4);      // transform warps
        }
        mbar_init(mfull, 1);
        mbar_init(mempty, RELU ? 5 : 1);
        for (int q = 0; q < 4; ++q) {
            mbar_init(&qfull[q], 1);
            mbar_init(&qempty[q], 4);
            mbar_init(&denready[q], 4);
        }
        for (int i = 0; i < kIQ; ++i) {
            mbar_init(&iqfull[i], 1);
            mbar_init(&iqempty[i], (RELU || PREP || TOKB) ? 3 : 2);
        }
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (RELU)
        for (int i = threadIdx.x; i < 2048 / 4; i += blockDim.x)
            reinterpret_cast<uint32_t*>(ones)[i] = 0x3F803F80u;
    // input preparation: weight row, temporal cos/sin, height/width table
    // [weights 128 floats][temporal 64 float2][row partial sums 2 x 3 x 64 floats][h/w table]
    float* prep_w = reinterpret_cast<float*>(smem + align_up(kWorkerSmem, 16));
    float2* prep_t = reinterpret_cast<float2*>(prep_w + 128);
    float2* prep_hw = prep_t + 64;
    const int nhw = rope_nhw(p.D), ntp = rope_nt(p.D);
    const double l2b = PREP ? log2((double)p.rope_base) : 0.0;
    if (PREP && p.rope)
        for (int i = threadIdx.x; i < p.grid_max * nhw; i += blockDim.x) {
            float c, sn;
            rope_cos_sin(i / nhw, i % nhw, nhw, l2b, c, sn);
            prep_hw[192 + i] = make_float2(c, sn);            // past the row partial sums
        }
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
    const int F = p.F, D = p.D;
    const int ntg = (p.S + kTokG - 1) / kTokG, nto = (p.S + kTokO - 1) / kTokO;

    if (warp == 0) {
        // ---------------- producer: tickets, dependencies, loads ----------------
        if (lane == 0) {
            tma_prefetch_desc(mK);
            tma_prefetch_desc(mV);
            if (p.want_output) {
                tma_prefetch_desc(mQ);
                tma_prefetch_desc(mO);
            }
            const uint64_t pol = LA_POL_STREAM();
            uint32_t iq = 0, nout = 0, ph = 0;
            int s = 0;
            bool ok = true;
            PhaseLog armed, armed_m;     // loads in flight are waited for after an abort
            LA_TRACE_WRITER(0);
            while (true) {
                Item it{kItemStop, 0, 0, 0};
                if (ok) it = decode_ticket(p, atomicAdd(&p.status[2], 1u));
                const int qi = iq % kIQ;
                ok = ok && mbar_wait(&iqempty[qi], ((iq / kIQ) & 1) ^ 1, ab, 0x401);
                if (!ok) it.type = kItemStop;
                items[qi] = it;
                mbar_arrive(&iqfull[qi]);
                ++iq;
                if (it.type == kItemStop) break;
                const int frame = it.bh * F + step_frame(it.f, F, p.rev_chunk);
                LA_TRACE_EVENT(it.type == kItemGram ? 1 : 2, frame);
                if (it.type == kItemGram) {
                    if (it.f >= kRG)
                        ok = ok && wait_flag_ge(&p.chain_done[2 * it.bh + ((it.f - kRG) & 1)],
                                                it.f - kRG + 1, ab, 0x402);
                    LA_TRACE_EVENT(3, frame);
                    for (int t = 0; t < ntg; ++t) {
                        ok = ok && mbar_wait(&empty[s], ph ^ 1, ab, 0x403);
                        if (ok) {
                            uint8_t* st = ring + s * 32768;
                            mbar_expect_tx(&full[s], 4 * kBoxG);
                            tma_load_3d(st, mK, &full[s], 0, t * kTokG, frame, pol);
                            tma_load_3d(st + kBoxG, mK, &full[s], 64, t * kTokG, frame, pol);
                            tma_load_3d(st + 16384, mV, &full[s], 0, t * kTokG, frame, pol);
                            tma_load_3d(st + 16384 + kBoxG, mV, &full[s], 64, t * kTokG, frame, pol);
                            armed.note(s, ph);
                        }
                        if (++s == kWStages) { s = 0; ph ^= 1; }
                    }
                } else {
                    // Q does not depend on the chain: fill the ring with Q tiles first,
                    // then wait for the state image of the frame and fetch it.
                    auto fetch_state = [&]() {
                        ok = ok && wait_flag_ge(&p.chain_done[2 * it.bh + (it.f & 1)], it.f + 1, ab,
                                                0x404);
                        LA_TRACE_EVENT(4, frame);
                        fence_proxy_async_global();
                        ok = ok && mbar_wait(mempty, (nout & 1) ^ 1, ab, 0x405);
                        ++nout;
                        if (ok) {
                            const size_t ms = (size_t)it.bh * kRM + it.f % kRM;
                            mbar_expect_tx(mfull, kImg + (RELU ? 512 : 0));
                            bulk_load_hint(mbuf, p.mimg + ms * kImg, kImg, mfull, pol);
                            if (RELU) bulk_load_hint(zbuf, p.zf + ms * 128, 512, mfull, pol);
                            armed_m.note(0, (nout - 1) & 1);
                        }
                    };
                    int t_lo, t_hi;
                    out_range(p, it, nto, t_lo, t_hi);
                    const int early = LA_FUSED_EARLY_Q ? min(t_hi - t_lo, kWStages) : 0;
                    for (int t = t_lo; t < t_hi; ++t) {
                        if (t - t_lo == early) fetch_state();
                        ok = ok && mbar_wait(&empty[s], ph ^ 1, ab, 0x406);
                        if (ok) {
                            uint8_t* st = ring + s * 32768;
                            mbar_expect_tx(&full[s], 2 * kBoxO);
                            tma_load_3d(st, mQ, &full[s], 0, t * kTokO, frame, pol);
                            tma_load_3d(st + kBoxO, mQ, &full[s], 64, t * kTokO, frame, pol);
                            armed.note(s, ph);
                        }
                        if (++s == kWStages) { s = 0; ph ^= 1; }
                    }
                    if (early == t_hi - t_lo) fetch_state();
                }
            }
            armed.drain_if_aborted(full, kWStages, ab);
            armed_m.drain_if_aborted(mfull, 1, ab);
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer ----------------
        if (lane == 0) {
            const uint32_t idKK = idesc_bf16(128, D, true, true);
            const uint32_t idZ = idesc_bf16(128, 16, true, false);
            const uint32_t idO = idesc_bf16(128, p.den_col ? D + 16 : D, false, true);
            const uint64_t ones_d = sdesc_sw128(smem_u32(ones), 16, 1024);
            uint32_t iq = 0, ph = 0, qctr = 0, nout = 0;
            int s = 0;
            bool ok = true;
            PhaseLog armed;     // MMAs in flight are waited for after an abort
            while (ok) {
                const int qi = iq % kIQ;
                if (!(ok = mbar_wait(&iqfull[qi], (iq / kIQ) & 1, ab, 0x411))) break;
                const Item it = items[qi];
                mbar_arrive(&iqempty[qi]);
                ++iq;
                if (it.type == kItemStop) break;
                if (it.type == kItemGram) {
                    const uint32_t qa = qctr & 3, qb = (qctr + 1) & 3;
                    ok = mbar_wait(&qempty[qa], ((qctr >> 2) & 1) ^ 1, ab, 0x412) &&
                         mbar_wait(&qempty[qb], (((qctr + 1) >> 2) & 1) ^ 1, ab, 0x413);
                    qctr += 2;
                    if (!ok) break;
                    tc_fence_after();
                    const uint32_t dG = tbase + qa * 128, dW = tbase + qb * 128;
                    for (int t = 0; t < ntg && ok; ++t) {
                        if (!(ok = mbar_wait((RELU || PREP || TOKB) ? &xform[s] : &full[s], ph, ab,
                                             0x414)))
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
                        if (++s == kWStages) { s = 0; ph ^= 1; }
                    }
                    if (!ok) break;
                    mma_commit(&qfull[qa]);
                    mma_commit(&qfull[qb]);
                } else {
                    if (!(ok = mbar_wait(mfull, nout & 1, ab, 0x415))) break;
                    ++nout;
                    // The image is in shared memory: its ring slot may be rewritten.
                    uint32_t* mc = &p.mimg_consumed[(size_t)it.bh * kRM + it.f % kRM];
                    if (p.out_split) add_release_gpu(mc, 1u);
                    else st_release_gpu(mc, it.f + 1);
                    const uint32_t mb = smem_u32(mbuf);
                    int t_lo, t_hi;
                    out_range(p, it, nto, t_lo, t_hi);
                    for (int t = t_lo; t < t_hi && ok; ++t) {
                        const uint32_t qa = qctr & 3;
                        ok = mbar_wait(&qempty[qa], ((qctr >> 2) & 1) ^ 1, ab, 0x416) &&
                             mbar_wait((RELU || PREP) ? &xform[s] : &full[s], ph, ab, 0x417);
                        ++qctr;
                        if (!ok) break;
                        tc_fence_after();
                        const uint32_t qs = smem_u32(ring + s * 32768);
                        for (int kk = 0; kk < D / 16; ++kk) {
                            const uint64_t ad = sdesc_sw128(qs + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                            const uint64_t bd = sdesc_sw128(mb + kk * 2048, 16384, 1024);
                            mma_bf16(tbase + qa * 128, ad, bd, idO, kk > 0 ? 1u : 0u);
                        }
                        mma_commit(&empty[s]);
                        mma_commit(&qfull[qa]);
                        armed.note(s, ph);
                        if (++s == kWStages) { s = 0; ph ^= 1; }
                    }
                    if (!ok) break;
                    mma_commit(mempty);
                }
            }
            armed.drain_if_aborted(empty, kWStages, ab);
        }
    } else if (warp < 6) {
        // ---------------- epilogue (4 warps; the leader waits, all follow) ----------------
        const int q = warp & 3, row = q * 32 + lane;
        const bool leader = (threadIdx.x == 64);
        const uint32_t lanebase = uint32_t(q * 32) << 16;
        uint32_t iq = 0, qctr = 0, sctr = 0;
        uint32_t dpar = 0;    // bit q: parity of quarter q's next output-tile use (denready)
        bool ok = true;
        const uint64_t pol_keep = LA_POL_KEEP();          // hand-off data: re-read soon
        const uint64_t pol_stream = LA_POL_STREAM();       // outputs: never re-read
        LA_TRACE_WRITER(1);
        while (true) {
            if (leader) {
                const int qi = iq % kIQ;
                Item it{kItemStop, 0, 0, 0};
                ok = ok && mbar_wait(&iqfull[qi], (iq / kIQ) & 1, ab, 0x421);
                if (ok) {
                    it = items[qi];
                    mbar_arrive(&iqempty[qi]);
                }
                bc_item[0] = it;
            }
            ++iq;
            named_bar_sync(1, 128);
            const Item it = bc_item[0];
            if (it.type == kItemStop) break;
            const int frame = it.bh * F + step_frame(it.f, F, p.rev_chunk);
            const int nblk = D > 64 ? 2 : 1;
            if (it.type == kItemGram) {
                const uint32_t qa = qctr & 3, qb = (qctr + 1) & 3;
                if (leader) {
                    ok = ok && mbar_wait(&qfull[qa], (qctr >> 2) & 1, ab, 0x422) &&
                         mbar_wait(&qfull[qb], ((qctr + 1) >> 2) & 1, ab, 0x423);
                    if (RELU) bulk_wait_read<0>();     // dz staging free again
                    *bc_ok = ok;
                }
                qctr += 2;
                named_bar_sync(1, 128);
                const bool go = *bc_ok;
                tc_fence_after();
                const size_t sidx = (size_t)it.bh * kRG + it.f % kRG;
                // GDN: G'' = -alpha beta kappa^2 K^T K (A operand of the chain's MMA),
                //      B~  = beta kappa K^T V (added by the chain through an identity MMA).
                // ReLU: B~ = phi(K)^T V, and dz = phi(K)^T 1 in fp32.
                // a step that starts a chunk of the reversed scan has a zero decay:
                // G'' = 0 and the chain's carried state is zero
                const float al = RELU ? 1.f : (step_resets(it.f, p.rev_chunk) ? 0.f : p.alpha[frame]);
                const float bt = (RELU || TOKB) ? 1.f : p.beta[frame];   // TOKB: in the rows
                const float sg = -al * bt * p.k_scale * p.k_scale;
                const float sw = RELU ? 1.f : bt * p.k_scale;
                for (int im = RELU ? 1 : 0; im < 2; ++im) {
                    const uint32_t qq = im == 0 ? qa : qb;
                    const float sc = im == 0 ? sg : sw;
                    uint8_t* dst = (im == 0 ? p.gimg : p.bimg) + sidx * kImg;
                    for (int blk = 0; blk < nblk; ++blk) {
                        if (leader) bulk_wait_read<kWStg - 1>();
                        named_bar_sync(1, 128);
                        uint8_t* sb = stg + (sctr % kWStg) * 16384;
                        ++sctr;
                        if (go)
                            for (int c0 = blk * 64; c0 < min(D, blk * 64 + 64); c0 += 16) {
                                float v[16];
                                tmem_ld16(tbase + lanebase + qq * 128 + c0, v);
                                tmem_wait_ld();
#pragma unroll
                                for (int e = 0; e < 16; ++e) v[e] *= sc;
                                store_row16_bf16(sb, row, c0 & 63, v);
                            }
                        fence_proxy_async_smem();
                        named_bar_sync(1, 128);
                        if (leader && go) {
                            bulk_store_hint(dst + blk * 16384, sb, 16384, pol_keep);
                            bulk_commit();
                        }
                    }
                }
                if (RELU) {
                    if (go) {
                        float v[16];
                        tmem_ld16(tbase + lanebase + qa * 128, v);
                        tmem_wait_ld();
                        dzst[row] = v[0];
                    }
                    fence_proxy_async_smem();
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) {
                    mbar_arrive(&qempty[qa]);
                    mbar_arrive(&qempty[qb]);
                }
                named_bar_sync(1, 128);
                if (leader && go) {
                    if (RELU) {
                        bulk_store_hint(p.dz + sidx * 128, dzst, 512, pol_keep);
                        bulk_commit();
                    }
                    bulk_wait_all<0>();
                    fence_proxy_async_global();
                    if (!(it.bh == 0 && it.f == p.skip_publish))
                        st_release_gpu(&p.gram_ready[sidx], it.f + 1);
                    LA_TRACE_EVENT(5, frame);
                }
            } else {
                int t_lo, t_hi;
                out_range(p, it, nto, t_lo, t_hi);
                for (int t = t_lo; t < t_hi; ++t) {
                    const uint32_t qa = qctr & 3;
                    if (leader) {
                        ok = ok && mbar_wait(&qfull[qa], (qctr >> 2) & 1, ab, 0x424);
                        if (RELU && !p.den_col)
                            ok = ok && mbar_wait(&denready[qa], (dpar >> qa) & 1, ab, 0x425);
                        *bc_ok = ok;
                    }
                    dpar ^= 1u << qa;
                    ++qctr;
                    named_bar_sync(1, 128);
                    const bool go = *bc_ok;
                    tc_fence_after();
                    float inv = 1.f;
                    if (RELU && go) {
                        if (p.den_col) {             // phi(Q) z_hi and phi(Q) z_lo from the MMA
                            float dv[16];
                            tmem_ld16(tbase + lanebase + qa * 128 + D, dv);
                            tmem_wait_ld();
                            inv = 1.f / (dv[0] + dv[1] + p.eps);
                        } else {
                            inv = 1.f / denbuf[qa * 128 + row];
                        }
                    }
                    // one 64-column block (16 KB) at a time through staging
                    for (int blk = 0; blk < nblk; ++blk) {
                        if (leader) bulk_wait_read<kWStg - 1>();
                        named_bar_sync(1, 128);
                        uint8_t* sb = stg + (sctr % kWStg) * 16384;
                        ++sctr;
                        if (go)
                            for (int c0 = blk * 64; c0 < min(D, blk * 64 + 64); c0 += 16) {
                                float v[16];
                                tmem_ld16(tbase + lanebase + qa * 128 + c0, v);
                                tmem_wait_ld();
                                if (RELU) {
#pragma unroll
                                    for (int e = 0; e < 16; ++e) v[e] *= inv;
                                }
                                store_row16_bf16(sb, row, c0 & 63, v);
                            }
                        if (blk == nblk - 1) {
                            tc_fence_before();
                            __syncwarp();
                            if (lane == 0) mbar_arrive(&qempty[qa]);
                        }
                        fence_proxy_async_smem();
                        named_bar_sync(1, 128);
                        if (leader && go) {
                            tma_store_3d_hint(mO, sb, blk * 64, t * kTokO, frame, pol_stream);
                            bulk_commit();
                            if (t == t_hi - 1 && blk == nblk - 1) LA_TRACE_EVENT(6, frame);
                        }
                    }
                }
            }
        }
        if (leader) bulk_wait_all<0>();
    } else if (PREP && warp >= 6) {
        // ---------------- input preparation of K (gram) and Q (output) tiles ----------------
        // RMSNorm with the head's weight, ReLU and 3D RoPE, in place on the
        // bf16 tile between its TMA load and the MMA (SANA-WM digest, method
        // details: RMSNorm + ReLU + key scaling + RoPE fused with the scan;
        // the key scale stays on the fp32 accumulators).  Six warps; in each
        // block of 64 rows, thread tl owns row tl % 64 and one third of its
        // 16-byte chunks (part tl / 64), so every warp works on the same
        // channels of 32 consecutive tokens: weights, pair groups and the
        // temporal cos/sin are broadcast reads, the width cos/sin of
        // consecutive tokens hit distinct banks.  The three partial sums of
        // squares of a row meet in shared memory.
        const int tl = threadIdx.x - 192;          // 0..191
        const bool leader = (tl == 0);
        const int prow = tl & 63, part = tl >> 6;
        const int nch = D / 8;
        const int c_lo = (part * nch + 2) / 3, c_hi = ((part + 1) * nch + 2) / 3;   // <= 6 chunks
        float* ssp = reinterpret_cast<float*>(prep_t + 64);   // [2][3][64] partial sums
        float2* prep_tab = prep_hw + 192;                     // height/width table (moved past ssp)
        uint32_t iq = 0, ph = 0, bcn = 0, blk_par = 0;
        int s = 0;
        bool ok = true;
        int* bc2 = bc_ok + 2;
        const float inv_d = 1.f / (float)D;
        while (true) {
            if (leader) {
                const int qi = iq % kIQ;
                Item it{kItemStop, 0, 0, 0};
                ok = ok && mbar_wait(&iqfull[qi], (iq / kIQ) & 1, ab, 0x441);
                if (ok) {
                    it = items[qi];
                    mbar_arrive(&iqempty[qi]);
                }
                bc_item[1] = it;
            }
            ++iq;
            named_bar_sync(2, 192);
            const Item it = bc_item[1];
            if (it.type == kItemStop) break;
            const bool gram = it.type == kItemGram;
            const float* wsrc = gram ? p.k_weight : p.q_weight;
            const size_t wrow = (size_t)(it.bh % p.H) * D;
            for (int i = tl; i < D; i += 192) prep_w[i] = wsrc ? __ldg(wsrc + wrow + i) : 1.f;
            if (p.rope)
                for (int i = tl; i < ntp; i += 192) {
                    float c, sn;
                    rope_cos_sin(p.frame_offset + it.f, i, ntp, l2b, c, sn);
                    prep_t[i] = make_float2(c, sn);
                }
            named_bar_sync(2, 192);
            int t_lo = 0, t_hi = ntg;
            if (!gram) out_range(p, it, nto, t_lo, t_hi);
            const int rows = gram ? kTokG : kTokO;
            const uint32_t box = gram ? kBoxG : kBoxO;
            for (int t = t_lo; t < t_hi; ++t) {
                if (leader) {
                    ok = ok && mbar_wait(&full[s], ph, ab, 0x442);
                    bc2[bcn & 1] = ok;
                }
                named_bar_sync(2, 192);
                if (bc2[(bcn++) & 1]) {
                    uint8_t* const tile = ring + s * 32768;
                    for (int r0 = 0; r0 < rows; r0 += 64, blk_par ^= 1) {
                        const int row = r0 + prow;
                        float* sp = ssp + blk_par * 192;
                        uint4 x[6];
                        float ss = 0.f;
#pragma unroll
                        for (int u = 0; u < 6; ++u) {
                            const int c = c_lo + u;
                            if (c < c_hi) {
                                x[u] = *reinterpret_cast<const uint4*>(tile + (c >> 3) * box +
                                                                       sw128_off(row, c & 7));
                                const uint32_t wv[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
#pragma unroll
                                for (int e2 = 0; e2 < 4; ++e2) {
                                    const float a0 = bf16_lo(wv[e2]), a1 = bf16_hi(wv[e2]);
                                    ss = fmaf(a0, a0, fmaf(a1, a1, ss));
                                }
                            }
                        }
                        sp[part * 64 + prow] = ss;
                        named_bar_sync(2, 192);
                        const float ms = fmaf(sp[prow] + sp[64 + prow] + sp[128 + prow], inv_d,
                                              p.norm_eps);
                        const float r = ms > 0.f ? rsqrtf(ms) : 0.f;   // a zero row stays zero
                        const int tok = t * rows + row;
                        const bool real = tok < p.S;
                        const int hp = real ? tok / p.grid_w : 0, wp = real ? tok - hp * p.grid_w : 0;
#pragma unroll
                        for (int u = 0; u < 6; ++u) {
                            const int c = c_lo + u;
                            if (c < c_hi) {
                                const uint32_t wv[4] = {x[u].x, x[u].y, x[u].z, x[u].w};
                                const float4 wa = *reinterpret_cast<const float4*>(prep_w + 8 * c);
                                const float4 wb = *reinterpret_cast<const float4*>(prep_w + 8 * c + 4);
                                const float wt[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
                                uint32_t out[4];
#pragma unroll
                                for (int e2 = 0; e2 < 4; ++e2) {
                                    const int i = 4 * c + e2;               // channel pair
                                    float2 cs = make_float2(1.f, 0.f);
                                    if (p.rope && real)
                                        cs = i < ntp ? prep_t[i]
                                           : i < ntp + nhw ? prep_tab[hp * nhw + (i - ntp)]
                                                           : prep_tab[wp * nhw + (i - ntp - nhw)];
                                    const float rc = r * cs.x, rs = r * cs.y;
                                    const float y0 = fmaxf(bf16_lo(wv[e2]) * wt[2 * e2], 0.f);
                                    const float y1 = fmaxf(bf16_hi(wv[e2]) * wt[2 * e2 + 1], 0.f);
                                    out[e2] = pack_bf16x2(fmaf(y0, rc, -y1 * rs), fmaf(y0, rs, y1 * rc));
                                }
                                *reinterpret_cast<uint4*>(tile + (c >> 3) * box + sw128_off(row, c & 7)) =
                                    make_uint4(out[0], out[1], out[2], out[3]);
                            }
                        }
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&xform[s]);
                if (++s == kWStages) { s = 0; ph ^= 1; }
            }
        }
    } else if (TOKB) {
        // ---------------- per-token update gate: sqrt(beta_t) on K and V rows ----------------
        // Every token row of a gram item's K and V tiles is scaled by
        // sqrt(beta_t) in shared memory (bf16), so the unchanged contractions
        // give Kh^T diag(beta) Kh and Kh^T diag(beta) V (SANA-WM paper
        // summary, section 3, "Hybrid GDN/Softmax Attention", per-token update
        // gate).  Six warps: unit u = tl + 192 i of a tile is 16-byte chunk
        // (u / 64) % nch of row u % 64 of K (u < 64 nch) or V, so a thread
        // always works on row tl % 64 and needs one gate per tile.  Every
        // thread waits for the stage itself (no barrier per tile); output
        // tiles pass untouched through the same wait / arrive protocol.
        const int tl = threadIdx.x - 192;          // 0..191
        const bool leader = (tl == 0);
        const int row = tl & 63;
        const int nch = D / 8, nunits = 2 * 64 * nch;
        uint32_t iq = 0, ph = 0;
        int s = 0;
        bool ok = true;
        while (true) {
            if (leader) {
                const int qi = iq % kIQ;
                Item it{kItemStop, 0, 0, 0};
                ok = ok && mbar_wait(&iqfull[qi], (iq / kIQ) & 1, ab, 0x451);
                if (ok) {
                    it = items[qi];
                    mbar_arrive(&iqempty[qi]);
                }
                bc_item[1] = it;
            }
            ++iq;
            named_bar_sync(2, 192);
            const Item it = bc_item[1];
            named_bar_sync(2, 192);                // bc_item read before the next write
            if (it.type == kItemStop) break;
            // Output tiles are not touched, but they pass through the same
            // wait / arrive protocol: every use of a ring stage completes one
            // phase of its xform barrier, whose parity the MMA tracks by stage use.
            const bool gram = it.type == kItemGram;
            const float* bsrc =
                p.beta_tok + ((size_t)it.bh * F + step_frame(it.f, F, p.rev_chunk)) * p.S;
            // the gates of a tile are fetched one tile ahead, off the critical path
            float bv_next = (gram && row < p.S) ? __ldg(bsrc + row) : 0.f;
            int t_lo = 0, t_hi = ntg;
            if (!gram) out_range(p, it, nto, t_lo, t_hi);
            for (int t = t_lo; t < t_hi; ++t) {
                const float bv = bv_next;
                const int tok_n = (t + 1) * kTokG + row;
                bv_next = (gram && t + 1 < ntg && tok_n < p.S) ? __ldg(bsrc + tok_n) : 0.f;
                ok = ok && mbar_wait(&full[s], ph, ab, 0x452);
                if (ok && gram) {
                    const float sb = sqrtf(fmaxf(bv, 0.f));
                    const __nv_bfloat162 g = __floats2bfloat162_rn(sb, sb);
                    uint8_t* const tile = ring + s * 32768;
#pragma unroll 4
                    for (int u = tl; u < nunits; u += 192) {
                        const int tv = u >= 64 * nch ? 1 : 0;                 // K or V
                        const int c = (u - tv * 64 * nch) >> 6;
                        uint4* pc = reinterpret_cast<uint4*>(tile + tv * 16384 + (c >> 3) * kBoxG +
                                                             sw128_off(row, c & 7));
                        uint4 x = *pc;
                        __nv_bfloat162* h = reinterpret_cast<__nv_bfloat162*>(&x);
                        h[0] = __hmul2(h[0], g); h[1] = __hmul2(h[1], g);
                        h[2] = __hmul2(h[2], g); h[3] = __hmul2(h[3], g);
                        *pc = x;
                    }
                }
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&xform[s]);
                if (++s == kWStages) { s = 0; ph ^= 1; }
            }
        }
    } else if (RELU && warp < 10) {
        // ---------------- ReLU transforms: phi(K), phi(Q) and denominators ----------------
        const int tl = threadIdx.x - 192;          // 0..127
        const bool leader = (tl == 0);
        uint32_t iq = 0, qctr = 0, nout = 0, ph = 0, bcn = 0;
        int s = 0;
        bool ok = true;
        // The leader's per-tile verdict alternates between two slots: with a
        // single barrier per tile, a slow warp may still be reading the
        // previous tile's slot when the leader writes the next one.
        int* bc2 = bc_ok + 2;
        while (true) {
            if (leader) {
                const int qi = iq % kIQ;
                Item it{kItemStop, 0, 0, 0};
                ok = ok && mbar_wait(&iqfull[qi], (iq / kIQ) & 1, ab, 0x431);
                if (ok) {
                    it = items[qi];
                    mbar_arrive(&iqempty[qi]);
                }
                bc_item[1] = it;
            }
            ++iq;
            named_bar_sync(2, 128);
            const Item it = bc_item[1];
            if (it.type == kItemStop) break;
            if (it.type == kItemGram) {
                qctr += 2;
                for (int t = 0; t < ntg; ++t) {
                    if (leader) {
                        ok = ok && mbar_wait(&full[s], ph, ab, 0x432);
                        bc2[bcn & 1] = ok;
                    }
                    named_bar_sync(2, 128);
                    if (bc2[(bcn++) & 1]) {
                        uint4* kt = reinterpret_cast<uint4*>(ring + s * 32768);
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
                    if (++s == kWStages) { s = 0; ph ^= 1; }
                }
            } else {
                if (leader) ok = ok && mbar_wait(mfull, nout & 1, ab, 0x433);
                ++nout;
                int t_lo, t_hi;
                out_range(p, it, nto, t_lo, t_hi);
                for (int t = t_lo; t < t_hi; ++t) {
                    const uint32_t qa = qctr & 3;
                    if (leader) {
                        if (!p.den_col)
                            ok = ok && mbar_wait(&qempty[qa], ((qctr >> 2) & 1) ^ 1, ab, 0x434);
                        ok = ok && mbar_wait(&full[s], ph, ab, 0x435);
                        bc2[bcn & 1] = ok;
                    }
                    ++qctr;
                    named_bar_sync(2, 128);
                    if (bc2[(bcn++) & 1] && p.den_col) {
                        // phi(Q) only: the MMA forms the denominator from z in the image
                        uint4* qt = reinterpret_cast<uint4*>(ring + s * 32768);
                        for (int i = tl; i < 2 * (int)kBoxO / 16; i += 128) {
                            uint4 x = qt[i];
                            x.x = relu_bf16x2(x.x); x.y = relu_bf16x2(x.y);
                            x.z = relu_bf16x2(x.z); x.w = relu_bf16x2(x.w);
                            qt[i] = x;
                        }
                    } else if (bc2[(bcn - 1) & 1]) {
                        uint8_t* st = ring + s * 32768;
                        float den = 0.f;
                        for (int blk = 0; blk < 2 && blk * 64 < D; ++blk) {
                            for (int c = 0; c < 8; ++c) {
                                uint4* pch = reinterpret_cast<uint4*>(st + blk * 16384 + sw128_off(tl, c));
                                uint4 x = *pch;
                                x.x = relu_bf16x2(x.x); x.y = relu_bf16x2(x.y);
                                x.z = relu_bf16x2(x.z); x.w = relu_bf16x2(x.w);
                                *pch = x;
                                const float* zz = zbuf + blk * 64 + c * 8;
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
                        denbuf[qa * 128 + tl] = den + p.eps;
                    }
                    fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        mbar_arrive(&xform[s]);
                        if (!p.den_col) mbar_arrive(&denready[qa]);
                    }
                    if (++s == kWStages) { s = 0; ph ^= 1; }
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(mempty);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tbase, 512);
}

// ============================================================================
// chain blocks (one head each)
// ============================================================================
// warp 0: loader -- waits for the gram item of each frame and bulk-copies its
//         G'' and B~ images (ReLU: dz_f and B~) into a 2-stage ring;
// warp 1: TMEM owner + MMA issuer (GDN);
// warps 2-9: epilogue -- thread <-> (state row, half of the columns);
// warps 10, 11: publishers of the even and the odd frames -- store bf16(M_f)
//         (and z_f) to the head's ring slot once the slot is free, then release
//         the progress flag of their parity.  Image buffer b holds the frames
//         of parity b, so each publisher owns one buffer; two of them keep the
//         per-frame store and flag latencies off the recurrence.
// The epilogue's critical path touches only shared and tensor memory.
template <bool RELU>
__device__ __forceinline__ void chain_role(const FusedParams& p, uint8_t* smem) {
    // stage s (64 KB): [0, 32 KB) G'' image (GDN) or dz_f (ReLU); [32 KB, 64 KB) B~ image
    uint8_t* stage = smem;                                  // kCStages x 64 KB
    uint8_t* imgs = stage + kCStages * 2 * kImg;            // 2 x 32 KB bf16 state images
    float* zst = reinterpret_cast<float*>(imgs + 2 * kImg); // [2][128] z_f staging (ReLU)
    float* abc = zst + 256;                                 // [2] alpha_{f+1} broadcast per half
    uint64_t* gfull = reinterpret_cast<uint64_t*>(abc + 2);
    uint64_t* gempty = gfull + kCStages;
    uint64_t* mdone = gempty + kCStages;   // [2] MMA of the frame finished (per column half)
    uint64_t* mready = mdone + 2;          // [2] TMEM holds alpha_f M_{f-1}, image written (per half)
    uint64_t* iready = mready + 2;         // [2] image buffer b holds a frame to publish
    uint64_t* iread = iready + 2;          // [2] publisher has read image buffer b out
    int* bc_ok = reinterpret_cast<int*>(iread + 2);        // [2] per half
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bc_ok + 2);
    uint32_t* abort_flag = tmem_slot + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int bh = blockIdx.x;
    const int F = p.F, D = p.D;
    const int nhalf = D > 64 ? 2 : 1;      // independent column halves of the state
    if (threadIdx.x == 0) {
        for (int s = 0; s < kCStages; ++s) {
            mbar_init(&gfull[s], 1);
            // the epilogue halves (and, for GDN, the MMA) are done with the stage
            mbar_init(&gempty[s], nhalf + (RELU ? 0 : 1));
        }
        for (int h = 0; h < 2; ++h) {
            mbar_init(&mdone[h], 1);
            mbar_init(&mready[h], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&iready[b], nhalf);
            mbar_init(&iread[b], 1);
        }
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
        // ---------------- loader ----------------
        if (lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            const uint64_t pol_last_use = LA_POL_STREAM();
            PhaseLog armed;     // loads in flight are waited for after an abort
            LA_TRACE_WRITER(0);
            for (int f = 0; f < F; ++f) {
                const size_t sidx = (size_t)bh * kRG + f % kRG;
                if (!wait_flag_ge(&p.gram_ready[sidx], f + 1, ab, 0x501)) break;
                LA_TRACE_EVENT(10, (uint64_t)bh * F + f);
                fence_proxy_async_global();
                if (!mbar_wait(&gempty[s], ph ^ 1, ab, 0x502)) break;
                LA_TRACE_EVENT(18, (uint64_t)bh * F + f);
                uint8_t* st = stage + s * 2 * kImg;
                if (!RELU) {
                    mbar_expect_tx(&gfull[s], 2 * kImg);
                    bulk_load_hint(st, p.gimg + sidx * kImg, kImg, &gfull[s], pol_last_use);
                } else {
                    mbar_expect_tx(&gfull[s], kImg + 512);
                    bulk_load_hint(st, p.dz + sidx * 128, 512, &gfull[s], pol_last_use);
                }
                bulk_load_hint(st + kImg, p.bimg + sidx * kImg, kImg, &gfull[s], pol_last_use);
                armed.note(s, ph);
                if (++s == kCStages) { s = 0; ph ^= 1; }
            }
            armed.drain_if_aborted(gfull, kCStages, ab);
        }
    } else if (warp == 1) {
        // ---------------- MMA (GDN): D[:, half] += G'' bf16(M_{f-1})[:, half] ----------------
        if (!RELU && lane == 0) {
            int s = 0;
            uint32_t ph = 0;
            PhaseLog armed, armed_h;     // MMAs in flight are waited for after an abort
            LA_TRACE_WRITER(3);
            for (int f = 0; f < F; ++f) {
                if (!mbar_wait(&gfull[s], ph, ab, 0x503)) break;
                LA_TRACE_EVENT(19, (uint64_t)bh * F + f);
                const uint32_t sa = smem_u32(stage + s * 2 * kImg);
                const uint32_t mb = smem_u32(imgs + ((f + 1) & 1) * kImg);   // image of M_{f-1}
                bool ok = true;
                for (int h = 0; h < nhalf; ++h) {
                    if (!(ok = mbar_wait(&mready[h], f & 1, ab, 0x504))) break;
                    LA_TRACE_EVENT(22 + h, (uint64_t)bh * F + f);
                    tc_fence_after();
                    const int nh = min(64, D - 64 * h);
                    const uint32_t idH = idesc_bf16(128, nh, false, true);
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint64_t ad = sdesc_sw128(sa + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                        const uint64_t bd = sdesc_sw128(mb + h * 16384 + kk * 2048, 16384, 1024);
                        mma_bf16(tM + 64 * h, ad, bd, idH, 1u);
                    }
                    mma_commit(&mdone[h]);
                    armed_h.note(h, f & 1);
                }
                if (!ok) break;
                mma_commit(&gempty[s]);
                armed.note(s, ph);
                if (++s == kCStages) { s = 0; ph ^= 1; }
            }
            armed.drain_if_aborted(gempty, kCStages, ab);
            armed_h.drain_if_aborted(mdone, nhalf, ab);
        }
    } else if (warp < 10) {
        // ---------------- epilogue: two independent column halves ----------------
        const int h = (warp - 2) >> 2;                  // column half of this warp
        const int q = warp & 3, row = q * 32 + lane;
        const int c_lo = 64 * h, c_hi = min(D, c_lo + 64);
        const bool active = h < nhalf;
        const bool leader = ((threadIdx.x & 127) == 0); // first thread of each half group
        const int bar_id = 1 + h;
        const uint32_t tl = tM + (uint32_t(q * 32) << 16);
        const bool live = row < D;
        LA_TRACE_WRITER(1 + h);
        if (active) {
            // alpha_{f+1} is read two frames ahead from the gate array (a read-only input)
            const float* ap = p.alpha + (size_t)bh * F;
            // decay of scan step j (frame step_frame(j)); zero where the reversed
            // scan starts a chunk, so that the carried state restarts from zero
            auto alpha_at = [&](int j) -> float {
                if (RELU || j >= F) return 1.f;
                return step_resets(j, p.rev_chunk) ? 0.f : __ldg(ap + step_frame(j, F, p.rev_chunk));
            };
            float a_cur = alpha_at(0);                               // step 0
            float a_nxt = alpha_at(1);                               // step 1
            // initial state: image of M_0 (buffer 1 = "frame -1") and TMEM alpha_0 M_0
            float z = 0.f;
            {
                // the row's columns c_lo .. c_hi - 1 (at most 64) as float4
                // loads, all in flight at once
                const float* src = (p.state_in && live) ? p.state_in + ((size_t)bh * D + row) * D
                                                        : nullptr;
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
                        store_row16_bf16(imgs + kImg, row, c0, v);
#pragma unroll
                        for (int e = 0; e < 16; ++e) v[e] *= a_cur;
                        tmem_st16(tl + c0, v);
                    }
                }
            }
            if (RELU && h == 0 && p.z_in && live) z = p.z_in[(size_t)bh * D + row];
            tmem_wait_st();
            fence_proxy_async_smem();
            tc_fence_before();
            named_bar_sync(bar_id, 128);
            if (leader) mbar_arrive(&mready[h]);

            int s = 0;
            uint32_t ph = 0;
            bool ok = true;
            for (int f = 0; f < F; ++f) {
                const int frame = bh * F + f;
                (void)frame;                       // used by the optional trace only
                const int ib = f & 1;
                const bool more = f + 1 < F;
                if (leader) {
                    ok = ok && mbar_wait(&gfull[s], ph, ab, 0x505);
                    if (!RELU) ok = ok && mbar_wait(&mdone[h], f & 1, ab, 0x506);
                    LA_TRACE_EVENT(16 + 20 * h, frame);
                    // image buffer ib was last used by frame f - 2: read out by the publisher
                    if (f >= 2) ok = ok && mbar_wait(&iread[ib], ((f >> 1) - 1) & 1, ab, 0x507);
                    bc_ok[h] = ok;
                    abc[h] = a_nxt;
                    LA_TRACE_EVENT(11 + 20 * h, frame);
                }
                named_bar_sync(bar_id, 128);
                const bool go = bc_ok[h];
                const float an = abc[h];
                tc_fence_after();
                if (leader) a_nxt = alpha_at(f + 2);
                if (go) {
                    const uint8_t* bimg = stage + s * 2 * kImg + kImg + h * 16384;
                    uint8_t* img = imgs + ib * kImg;
#pragma unroll
                    for (int cc = 0; cc < 2; ++cc) {
                        const int c0 = c_lo + 32 * cc;
                        if (c0 < c_hi) {
                            const bool two = c0 + 16 < c_hi;
                            float v0[16], v1[16];
                            tmem_ld16(tl + c0, v0);
                            if (two) tmem_ld16(tl + c0 + 16, v1);
                            // B~ (bf16) columns c0 .. c0+31 of this row
                            uint4 bw[4];
#pragma unroll
                            for (int u = 0; u < 4; ++u)
                                bw[u] = *reinterpret_cast<const uint4*>(
                                    bimg + sw128_off(row, ((c0 & 63) >> 3) + u));
                            tmem_wait_ld();
#pragma unroll
                            for (int u = 0; u < 2; ++u) {
                                v0[8 * u + 0] += bf16_lo(bw[u].x); v0[8 * u + 1] += bf16_hi(bw[u].x);
                                v0[8 * u + 2] += bf16_lo(bw[u].y); v0[8 * u + 3] += bf16_hi(bw[u].y);
                                v0[8 * u + 4] += bf16_lo(bw[u].z); v0[8 * u + 5] += bf16_hi(bw[u].z);
                                v0[8 * u + 6] += bf16_lo(bw[u].w); v0[8 * u + 7] += bf16_hi(bw[u].w);
                                v1[8 * u + 0] += bf16_lo(bw[u + 2].x); v1[8 * u + 1] += bf16_hi(bw[u + 2].x);
                                v1[8 * u + 2] += bf16_lo(bw[u + 2].y); v1[8 * u + 3] += bf16_hi(bw[u + 2].y);
                                v1[8 * u + 4] += bf16_lo(bw[u + 2].z); v1[8 * u + 5] += bf16_hi(bw[u + 2].z);
                                v1[8 * u + 6] += bf16_lo(bw[u + 2].w); v1[8 * u + 7] += bf16_hi(bw[u + 2].w);
                            }
                            store_row16_bf16(img, row, c0, v0);
                            if (two) store_row16_bf16(img, row, c0 + 16, v1);
                            if (!more && p.state_out && live) {
                                float* so = p.state_out + ((size_t)bh * D + row) * D + c0;
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
                            if (more) {
                                if (!RELU)
#pragma unroll
                                    for (int e = 0; e < 16; ++e) {
                                        v0[e] *= an;
                                        v1[e] *= an;
                                    }
                                tmem_st16(tl + c0, v0);
                                if (two) tmem_st16(tl + c0 + 16, v1);
                            }
                        }
                    }
                    if (RELU && h == 0) {
                        z += reinterpret_cast<const float*>(stage + s * 2 * kImg)[row];
                        zst[ib * 128 + row] = z;
                        if (p.den_col) {
                            float zv[16] = {};
                            zv[0] = z;                                          // rounds to z_hi
                            zv[1] = z - __bfloat162float(__float2bfloat16_rn(z));   // z_lo
                            store_row16_bf16(img, row, D, zv);
                        }
                        if (!more && p.z_out && live) p.z_out[(size_t)bh * D + row] = z;
                    }
                }
                tmem_wait_st();
                fence_proxy_async_smem();
                tc_fence_before();
                named_bar_sync(bar_id, 128);
                if (leader) {
                    mbar_arrive(&gempty[s]);
                    mbar_arrive(&mready[h]);
                    mbar_arrive(&iready[ib]);
                    LA_TRACE_EVENT(12 + 20 * h, frame);
                }
                if (++s == kCStages) { s = 0; ph ^= 1; }
            }
        }
    } else if (warp >= 10) {
        // ---------------- publishers (frames of parity par = warp - 10) ----------------
        // Frame f's stores are issued as soon as its image is written and its
        // ring slot is free.  Up to kPubLag store groups stay in flight; a
        // frame is published (flag = f + 1) once its stores have completed,
        // so store latency never holds back the image buffer.  The slot-free
        // flag of the publisher's next frame is read one frame ahead.
        const int par = warp - 10;
        if (lane == 0) {
            constexpr int kPubLag = LA_FUSED_PUBLAG;
            const uint64_t pol_keep = LA_POL_KEEP();
            uint32_t* flag = &p.chain_done[2 * bh + par];
            LA_TRACE_WRITER(4 + par);
            int published = 0;            // frames of this parity published so far
            uint32_t seen = 0;            // last value read from the next slot's flag
            int i = 0;                    // this frame is the i-th of its parity
            for (int f = par; f < F; f += 2, ++i) {
                const size_t msidx = (size_t)bh * kRM + f % kRM;
                // the slot's previous frame f - kRM has been read by its output item(s)
                const uint32_t need = p.out_split ? 2u * (uint32_t)(f / kRM) : (uint32_t)(f - kRM + 1);
                if (p.want_output && f >= kRM && seen < need &&
                    !wait_flag_ge(&p.mimg_consumed[msidx], need, ab, 0x509))
                    break;
                LA_TRACE_EVENT(24, (uint64_t)bh * F + f);
                if (!mbar_wait(&iready[par], i & 1, ab, 0x508)) break;
                LA_TRACE_EVENT(25, (uint64_t)bh * F + f);
                if (p.want_output) {
#if LA_FUSED_PUB_EVICT_LAST
                    bulk_store_hint(p.mimg + msidx * kImg, imgs + par * kImg, kImg, pol_keep);
#else
                    bulk_store(p.mimg + msidx * kImg, imgs + par * kImg, kImg);
#endif
                    if (RELU) bulk_store_hint(p.zf + msidx * 128, zst + par * 128, 512, pol_keep);
                    bulk_commit();
                    bulk_wait_read<0>();
                }
                LA_TRACE_EVENT(26, (uint64_t)bh * F + f);
                mbar_arrive(&iread[par]);
                // look at the next frame's slot while this frame's stores drain
                seen = (p.want_output && f + 2 < F && f + 2 >= kRM)
                           ? ld_acquire_gpu(&p.mimg_consumed[(size_t)bh * kRM + (f + 2) % kRM])
                           : 0u;
                if (p.want_output) {
                    if (i + 1 - published > kPubLag) {
                        bulk_wait_all<kPubLag>();
                        fence_proxy_async_global();
                        published = i + 1 - kPubLag;
                        const int g = par + 2 * (published - 1);     // newest completed frame
                        st_release_gpu(flag, g + 1);
                        LA_TRACE_EVENT(27, (uint64_t)bh * F + g);
                    }
                } else {
                    published = i + 1;
                    st_release_gpu(flag, f + 1);
                }
            }
            if (p.want_output && published < i && !ab.raised()) {
                bulk_wait_all<0>();
                fence_proxy_async_global();
                st_release_gpu(flag, par + 2 * (i - 1) + 1);
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) tmem_dealloc(tM, 128);
}

template <bool RELU, int XF>
__global__ void __launch_bounds__(kThreads, 1)
tc_fused_kernel(const FusedParams p, const __grid_constant__ CUtensorMap mK,
                const __grid_constant__ CUtensorMap mV, const __grid_constant__ CUtensorMap mQ,
                const __grid_constant__ CUtensorMap mO) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = align1024(smem_raw);
    if ((int)blockIdx.x < p.n_chain)
        chain_role<RELU>(p, smem);
    else
        worker_role<RELU, XF>(p, smem, &mK, &mV, &mQ, &mO);
}

// ----------------------------------------------------------------------------
// Host side
// ----------------------------------------------------------------------------
struct FusedLayout {
    size_t chain_done, gram_ready, mimg_consumed, flags_end;
    size_t gimg, bimg, dz, mimg, zf, total;
};

FusedLayout fused_layout(const ScanArgs& a) {
    const size_t bh = (size_t)a.B * a.H;
    FusedLayout L;
    size_t off = kWsHeaderBytes;
    L.chain_done = off;
    off += bh * 2 * 4;
    L.gram_ready = off;
    off += bh * kRG * 4;
    L.mimg_consumed = off;
    off += bh * kRM * 4;
    off = align_up(off, 256);
    L.flags_end = off;
    L.gimg = off;
    if (a.mode == LA_MODE_GDN) off += bh * kRG * kImg;
    L.bimg = off;
    off += bh * kRG * kImg;
    L.dz = off;
    if (a.mode == LA_MODE_RELU) off += bh * kRG * 512;
    L.mimg = off;
    off += bh * kRM * kImg;
    L.zf = off;
    if (a.mode == LA_MODE_RELU) off += bh * kRM * 512;
    L.total = align_up(off, 256);
    return L;
}



template <bool RELU, int XF>
cudaError_t launch_fused_mode(const ScanArgs& a, cudaStream_t st) {
    constexpr bool PREP = XF == kXfPrep;
    const FusedLayout L = fused_layout(a);
    uint8_t* ws = reinterpret_cast<uint8_t*>(a.ws);
    FusedParams p;
    p.alpha = a.alpha;
    p.beta = a.beta;
    p.state_in = a.state_in;
    p.z_in = a.z_in;
    p.state_out = a.state_out;
    p.z_out = a.z_out;
    p.status = reinterpret_cast<unsigned int*>(ws);
    p.chain_done = reinterpret_cast<uint32_t*>(ws + L.chain_done);
    p.gram_ready = reinterpret_cast<uint32_t*>(ws + L.gram_ready);
    p.mimg_consumed = reinterpret_cast<uint32_t*>(ws + L.mimg_consumed);
    p.gimg = ws + L.gimg;
    p.bimg = ws + L.bimg;
    p.dz = reinterpret_cast<float*>(ws + L.dz);
    p.mimg = ws + L.mimg;
    p.zf = reinterpret_cast<float*>(ws + L.zf);
    p.k_scale = a.k_scale;
    p.eps = a.eps;
    p.BH = a.B * a.H;
    p.F = a.F;
    p.S = a.S;
    p.D = a.D;
    p.want_output = a.o != nullptr;
    p.lag = LA_FUSED_LAG;
    p.den_col = (RELU && a.D <= 112) ? 1 : 0;
    p.rev_chunk = a.rev_chunk;
    p.beta_tok = a.beta_tok;
    if (const char* e = std::getenv("LA_SCAN_LAG")) p.lag = std::max(1, std::min(std::atoi(e), kRG + kRM - 1));
    p.H = a.H;
    p.q_weight = a.has_prep ? a.prep.q_weight : nullptr;
    p.k_weight = a.has_prep ? a.prep.k_weight : nullptr;
    p.norm_eps = a.prep.norm_eps;
    p.rope = a.has_prep && a.prep.rope;
    p.grid_w = p.rope ? a.prep.grid_w : 1;
    p.grid_max = p.rope ? std::max(a.prep.grid_h, a.prep.grid_w) : 0;
    p.frame_offset = a.prep.frame_offset;
    p.rope_base = p.rope ? a.prep.rope_base : 10000.f;
    p.skip_publish = -1;
    // Split output items into token halves when there are few per worker
    // (short clips: the last frames' outputs otherwise leave most workers
    // idle); LA_FUSED_OUT_SPLIT=0/1 overrides.
    {
        const int nto = (a.S + 127) / 128;
        const long workers = std::max(1, device_sm_count() - p.BH);
        p.out_split = (nto >= 2 && (long)p.BH * p.F < 4 * workers) ? 1 : 0;
        if (const char* e = std::getenv("LA_FUSED_OUT_SPLIT"))
            p.out_split = (e[0] == '1' && nto >= 2) ? 1 : 0;
    }
    if (const char* e = std::getenv("LA_SCAN_TEST_SKIP_PUBLISH")) p.skip_publish = std::atoi(e);
    const int nsm = device_sm_count();
    p.n_chain = p.BH;                 // one chain block per (b, h)
    p.heads_per_chain = 1;
    if (p.n_chain >= nsm || 2ull * p.BH * p.F >= (1ull << 31)) return cudaErrorInvalidValue;

    const uint64_t bhf = (uint64_t)p.BH * p.F;
    CUtensorMap mK, mV, mQ, mO;
    if (!make_tmap_bf16_3d(&mK, a.k, a.D, a.S, bhf, 64, kTokG) ||
        !make_tmap_bf16_3d(&mV, a.v, a.D, a.S, bhf, 64, kTokG))
        return cudaErrorInvalidValue;
    if (p.want_output) {
        if (!make_tmap_bf16_3d(&mQ, a.q, a.D, a.S, bhf, 64, kTokO) ||
            !make_tmap_bf16_3d(&mO, a.o, a.D, a.S, bhf, 64, kTokO))
            return cudaErrorInvalidValue;
    } else {
        mQ = mK;
        mO = mK;
    }
    // flags and counters start at zero
    cudaError_t e = cudaMemsetAsync(a.ws, 0, L.flags_end, st);
    if (e != cudaSuccess) return e;

    const size_t smem = PREP ? kFusedSmemPrep : kFusedSmem;
    e = ensure_dyn_smem(reinterpret_cast<const void*>(tc_fused_kernel<RELU, XF>), (int)smem);
    if (e != cudaSuccess) return e;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(nsm);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeCooperative;
    attr[0].val.cooperative = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, tc_fused_kernel<RELU, XF>, p, mK, mV, mQ, mO);
    if (e != cudaSuccess) return e;
    return cudaGetLastError();
}

}  // namespace

#ifdef LA_TRACE
extern "C" __attribute__((visibility("default"))) int la_trace_install(void* buf) {
    unsigned long long* p = reinterpret_cast<unsigned long long*>(buf);
    return (int)cudaMemcpyToSymbol(g_trace, &p, sizeof(p));
}
#endif

// One chain block per (b, h) pair, at most a third of the SMs, so that at
// least two thirds of them stream.
bool fused_eligible(const ScanArgs& a) {
    if (!tc_eligible(a)) return false;
    const int nsm = device_sm_count();
    return (long)a.B * a.H <= (long)(nsm / 3);
}

size_t fused_workspace_bytes(const ScanArgs& a) { return fused_layout(a).total; }

// The height/width cos/sin table holds max(grid_h, grid_w) x D/6 entries.
bool fused_prep_fits(const ScanArgs& a) {
    if (!a.prep.rope) return true;
    const long n = (long)std::max(a.prep.grid_h, a.prep.grid_w) * rope_nhw(a.D);
    return n <= (long)kPrepTabEntries && rope_nt(a.D) <= 64;
}

cudaError_t launch_fused(const ScanArgs& a, cudaStream_t st) {
    if (a.has_prep) return launch_fused_mode<false, kXfPrep>(a, st);      // GDN only
    if (a.beta_tok) return launch_fused_mode<false, kXfTokB>(a, st);      // GDN only
    return a.mode == LA_MODE_RELU ? launch_fused_mode<true, kXfNone>(a, st)
                                  : launch_fused_mode<false, kXfNone>(a, st);
}

}  // namespace la
