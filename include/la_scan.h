/*
 * la_scan.h -- C ABI of the block-causal, frame-wise linear-attention scan
 * (SANA-Video ReLU linear attention and SANA-WM frame-wise Gated DeltaNet)
 * for NVIDIA B200 (sm_100a).
 *
 * Equations (per batch item b and head h; frame f = 1..F holds the [S, D]
 * token matrices Q_f, K_f, V_f; the state is stored key-major, M[dk][dv]):
 *
 *   ReLU mode  (SANA-Video talk, ICLR 2026 oral, block KV cache segment;
 *               SANA-Video guide, lpnh.cn, section "核心机制"):
 *     M_f = M_{f-1} + phi(K_f)^T V_f,     z_f = z_{f-1} + sum_t phi(K_f[t,:])
 *     O_f[t,:] = phi(Q_f[t,:]) M_f / (phi(Q_f[t,:]) . z_f + eps),  phi = max(x,0)
 *
 *   GDN mode   (SANA-WM paper summary, paperlayer, section 3 "Hybrid
 *               GDN/Softmax Attention"; SANA-WM digest, method details,
 *               "Spatial Explosion" paragraph for the key scale):
 *     Kh_f = k_scale * K_f
 *     M_f  = alpha_f (I - beta_f Kh_f^T Kh_f) M_{f-1} + beta_f Kh_f^T V_f
 *     O_f  = Q_f M_f
 *
 * Causality is inclusive: frame f reads the state after its own update.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Layout.      q, k, v, o: [B, H, F, S, D] contiguous, D fastest.
 *              alpha, beta: [B, H, F] float32.
 *              state_in / state_out: [B, H, D, D] float32, key-major
 *              (element [b][h][dk][dv]).  z_in / z_out: [B, H, D] float32.
 * Dtype.       q, k, v, o share one dtype, LA_F32 or LA_BF16 (bf16 outputs
 *              are rounded to nearest even).  The state, the normaliser and
 *              all accumulation are float32.
 * Memory.      Every pointer is a device pointer of the current device (or
 *              managed memory), 16-byte aligned (la_scan_host takes host
 *              pointers instead; see there).  The caller owns all
 *              buffers, including the workspace; the library never
 *              allocates, frees or synchronises (except
 *              la_query_device_status, which synchronises on purpose).
 * Asynchrony.  Work is enqueued on `stream`; argument errors are returned
 *              before anything is enqueued; a failed launch returns
 *              LA_ERR_CUDA.  Device-side waits are bounded: a wait that
 *              gives up records LA_ERR_TIMEOUT in the workspace, which
 *              la_query_device_status reports.
 * Streams.     Wide heads (bf16, D > 128) and the three-kernel path on
 *              clips of 32 or more frames pipeline frame chunks over two
 *              streams of the library's own; one-chunk three-kernel calls
 *              with many heads run two head groups, each group's chain and
 *              output on a further stream of the library's own.  These
 *              streams are forked from `stream` (after the work already
 *              queued on it) and joined back to it, so the call is still
 *              ordered on `stream` as a whole (and can be captured into a
 *              CUDA graph).  The first such call on a device creates those
 *              streams and a few events and keeps them until the process
 *              exits; calls on one device serialise their enqueueing on a
 *              lock.
 * Aliasing.    state_in == state_out (and z_in == z_out) is allowed (in
 *              place).  o must not overlap q, k or v.
 * NULL state.  state_in == NULL (z_in == NULL) means a zero initial state;
 *              state_out == NULL (z_out == NULL) means "do not write".
 * Shapes.      B >= 1, H >= 1, F >= 0, S >= 1; D a multiple of 16 in
 *              [16, 256], else LA_ERR_UNSUPPORTED.  F == 0 writes state_in
 *              (or zeros) to state_out and touches nothing else.
 * Workspace.   At least la_workspace_size(mode, B, H, F, S, D) bytes of
 *              device memory, 256-byte aligned, private to the call while
 *              it runs (two calls in flight need two workspaces).
 * Threads.     Thread-safe when concurrent calls use distinct workspaces.
 */
#ifndef LA_SCAN_H
#define LA_SCAN_H

#include <stddef.h>
#include <cuda_runtime_api.h>

#if defined(__GNUC__)
#define LA_API __attribute__((visibility("default")))
#else
#define LA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum la_status {
    LA_OK = 0,
    LA_ERR_INVALID_ARG = 1,   /* NULL/misaligned/overlapping pointer, bad size, small workspace */
    LA_ERR_UNSUPPORTED = 2,   /* D not a multiple of 16 in [16, 256], or no sm_100 device      */
    LA_ERR_CUDA = 3,          /* a CUDA runtime call or kernel launch failed                   */
    LA_ERR_TIMEOUT = 4        /* a bounded device-side wait gave up (see la_query_device_status) */
} la_status;

typedef enum la_dtype { LA_F32 = 0, LA_BF16 = 1 } la_dtype;
typedef enum la_mode {
    LA_MODE_RELU = 0,
    LA_MODE_GDN = 1,
    LA_MODE_GDN_REVERSE = 2,     /* la_scan_gdn_reverse (for la_workspace_size, la_plan) */
    LA_MODE_GDN_TOKEN_BETA = 3,  /* la_scan_gdn_token_beta (for la_workspace_size, la_plan) */
    LA_MODE_GDN_COMPOSITE = 4,   /* la_gdn_interval_composite (for la_workspace_size, la_plan) */
    LA_MODE_GDN_PREP = 5,        /* la_scan_gdn_prep (for la_workspace_size, la_plan) */
    LA_MODE_RELU_PREP = 6        /* la_scan_relu_prep (for la_workspace_size, la_plan) */
} la_mode;

/*
 * Input preparation fused into the scan: RMSNorm, ReLU and 3D RoPE of q and
 * k.  Source: SANA-WM digest, method details, "Context-Parallel + Fused
 * Triton" paragraph -- RMSNorm, ReLU, key scaling, UCPE/RoPE and the GDN
 * scan run as one kernel; SANA-WM paper summary, appendix C.1 (the fused
 * kernel combines normalization, activation, scaling, positional
 * preparation and recurrent scanning); SANA-Video talk, 3D RoPE for the
 * linear attention.  The pages give the order, not the formulas; reading:
 *   y  = x / sqrt(mean_d x_d^2 + norm_eps) * weight[h]   (per token, per head)
 *   y  = max(y, 0)
 *   y~ = RoPE(y): channel pairs (2i, 2i+1); the first D/2 - 2 floor(D/6)
 *        pairs are temporal, the next floor(D/6) height, the last floor(D/6)
 *        width; pair i of a group of n pairs turns by pos * rope_base^(-i/n),
 *        pos = frame_offset + frame, s / grid_w or s % grid_w for token s.
 * The key scale k_scale is still applied inside the scan.
 */
typedef struct la_prep {
    const float* q_weight;  /* [H, D] f32 RMSNorm weight of q, or NULL (ones)              */
    const float* k_weight;  /* [H, D] f32 RMSNorm weight of k, or NULL (ones)              */
    float norm_eps;         /* RMSNorm epsilon, finite and >= 0 (1e-6 is usual)            */
    int rope;               /* non-zero: 3D RoPE after the ReLU                            */
    int grid_h, grid_w;     /* latent grid of a frame (rope only): S == grid_h * grid_w    */
    int frame_offset;       /* temporal position of frame 0 (a chunk of a longer clip), >= 0 */
    float rope_base;        /* RoPE base, finite and > 1 (10000 is usual)                   */
} la_prep;

/*
 * Block-causal ReLU linear attention with normaliser over latent frames.
 * Source: SANA-Video talk (ICLR 2026 oral), block KV cache segment -- the
 * D x D state is updated additively, block by block, and each block reads
 * the cached state of the earlier blocks plus its own contribution;
 * SANA-Video guide (lpnh.cn), section "核心机制".
 *
 * q, k, v     in : [B,H,F,S,D] of dtype dt.
 * o           out: [B,H,F,S,D] of dtype dt.
 * state_in    in : [B,H,D,D] f32 or NULL (zeros).   z_in  in : [B,H,D] f32 or NULL.
 * state_out   out: [B,H,D,D] f32 or NULL.           z_out out: [B,H,D] f32 or NULL.
 * eps         finite, >= 0; added to the denominator (1e-6 is the usual value).
 */
LA_API la_status la_scan_relu(const void* q, const void* k, const void* v, void* o, la_dtype dt,
                       const float* state_in, const float* z_in,
                       float* state_out, float* z_out,
                       int B, int H, int F, int S, int D, float eps,
                       void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Frame-wise Gated DeltaNet with key scaling.
 * Source: SANA-WM paper summary (paperlayer), section 3 "Hybrid GDN/Softmax
 * Attention" -- a D x D recurrent state is kept while each latent frame's
 * spatial tokens are processed together; a decay gate and an update gate
 * control forgetting; SANA-WM digest, method details, "Spatial Explosion"
 * paragraph -- keys are scaled by 1/sqrt(D*S) so that the transition's
 * spectral norm stays at most 1.
 *
 * alpha, beta in : [B,H,F] f32 (decay and update gate of each frame).
 * k_scale        : the key scale, usually 1/sqrt(D*S); applied inside the
 *                  scan in f32 (it is not folded into bf16 keys).
 * state_in/out   : [B,H,D,D] f32, key-major; NULL as described above.
 */
LA_API la_status la_scan_gdn(const void* q, const void* k, const void* v, void* o, la_dtype dt,
                      const float* alpha, const float* beta, float k_scale,
                      const float* state_in, float* state_out,
                      int B, int H, int F, int S, int D,
                      void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Reversed frame-wise GDN, reset at every chunk boundary.
 * Source: SANA-WM paper summary (paperlayer), section 3, "Chunk-causal
 * deployment" -- a reversed GDN scan that restarts at each chunk boundary
 * gives every frame the later frames of its own chunk as context without
 * leaking information across chunks.  Reading (the page gives no formula):
 * frames are split into chunks [c C, min((c+1) C, F)), C = chunk_frames;
 * inside a chunk the recurrence of la_scan_gdn runs from the chunk's last
 * frame back to its first, from a zero state:
 *   M_{e+1} = 0 (e = last frame of the chunk)
 *   M_f = alpha_f (I - beta_f Kh_f^T Kh_f) M_{f+1} + beta_f Kh_f^T V_f
 *   O_f = Q_f M_f
 *
 * Arguments and layouts are those of la_scan_gdn, without state in or out;
 * chunk_frames >= 1 (chunk_frames >= F reverses the whole clip).  The
 * workspace is la_workspace_size(LA_MODE_GDN_REVERSE, B, H, F, S, D) bytes.
 * bf16 inputs with 64 <= D <= 256 run on tensor cores (a chunk start is a
 * zero decay at that scan step); other shapes on the float32 SIMT kernel.
 */
LA_API la_status la_scan_gdn_reverse(const void* q, const void* k, const void* v, void* o,
                                     la_dtype dt, const float* alpha, const float* beta,
                                     float k_scale, int chunk_frames,
                                     int B, int H, int F, int S, int D,
                                     void* workspace, size_t workspace_bytes,
                                     cudaStream_t stream);

/*
 * Frame-wise GDN with a per-token update gate.
 * Source: SANA-WM paper summary (paperlayer), section 3, "Hybrid GDN/Softmax
 * Attention" -- a decay gate and a per-token update gate control how old
 * content is kept.  Reading: the update gate of frame f is one value per
 * spatial token, weighing that token's erase and write:
 *   M_f = alpha_f (M_{f-1} - Kh_f^T diag(beta_f) Kh_f M_{f-1}) + Kh_f^T diag(beta_f) V_f
 *   O_f = Q_f M_f
 *
 * beta_token  in : [B,H,F,S] f32, each value >= 0 (the gate of token s of
 *                  frame f); alpha [B,H,F] as for la_scan_gdn.
 * Everything else as for la_scan_gdn.  The workspace is
 * la_workspace_size(LA_MODE_GDN_TOKEN_BETA, B, H, F, S, D) bytes.  bf16
 * inputs with 64 <= D <= 256 run on tensor cores (each token row of K and V
 * is scaled by sqrt(beta) in shared memory, in bf16, before the unchanged
 * contractions); other shapes on the float32 SIMT kernel.
 */
LA_API la_status la_scan_gdn_token_beta(const void* q, const void* k, const void* v, void* o,
                                        la_dtype dt, const float* alpha,
                                        const float* beta_token, float k_scale,
                                        const float* state_in, float* state_out,
                                        int B, int H, int F, int S, int D,
                                        void* workspace, size_t workspace_bytes,
                                        cudaStream_t stream);

/*
 * Frame-wise GDN on raw q and k with the input preparation (la_prep) fused
 * into the scan: q~ = RoPE(ReLU(RMSNorm(q))), k~ = RoPE(ReLU(RMSNorm(k))), then
 * the recurrence of la_scan_gdn with Kh = k_scale k~ and O_f = Q~_f M_f.
 * Arguments as for la_scan_gdn plus `prep` (required).  Workspace:
 * la_workspace_size(LA_MODE_GDN_PREP, ...).  bf16 inputs with
 * 64 <= D <= 128 on the single-kernel path (B*H <= SMs/3), when the RoPE
 * tables of the grid fit in shared memory (about (grid_h + grid_w) * D / 6
 * entries of 8 bytes, at most 24 KiB), prepare the tiles in shared memory
 * between the TMA loads and the tensor core; other shapes run on the
 * float32 SIMT kernel.
 */
LA_API la_status la_scan_gdn_prep(const void* q, const void* k, const void* v, void* o,
                                  la_dtype dt, const float* alpha, const float* beta,
                                  float k_scale, const la_prep* prep,
                                  const float* state_in, float* state_out,
                                  int B, int H, int F, int S, int D,
                                  void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Block-causal ReLU linear attention on raw q and k with the input
 * preparation fused: phi_x = ReLU(RMSNorm(x)); RoPE (if prep->rope) enters
 * the numerator only, the normaliser keeps the unrotated features (reading:
 * rotated features can be negative, which would remove the positivity the
 * normaliser relies on):
 *   M_f = M_{f-1} + RoPE(phi_k)^T V_f,   z_f = z_{f-1} + sum_t phi_k[t]
 *   O_f[t] = RoPE(phi_q)[t] M_f / (phi_q[t] . z_f + eps)
 * Arguments as for la_scan_relu plus `prep` (required).  Workspace:
 * la_workspace_size(LA_MODE_RELU_PREP, ...).  Runs on the float32 SIMT
 * kernel.
 */
LA_API la_status la_scan_relu_prep(const void* q, const void* k, const void* v, void* o,
                                   la_dtype dt, const la_prep* prep,
                                   const float* state_in, const float* z_in,
                                   float* state_out, float* z_out,
                                   int B, int H, int F, int S, int D, float eps,
                                   void* workspace, size_t workspace_bytes,
                                   cudaStream_t stream);

/*
 * Advance the cached state over finished frames without producing outputs:
 * the scan above minus Q and O.  Source: SANA-Video talk, block KV cache
 * segment -- after a block is final its contribution is added to the cache
 * that the next block reads; SANA-WM paper summary, section 3,
 * "Chunk-causal deployment" -- autoregressive rollout carries the recurrent
 * state from chunk to chunk.
 *
 * mode LA_MODE_RELU uses (state, z) and ignores alpha, beta, k_scale;
 * mode LA_MODE_GDN uses (state) and ignores z_in / z_out.
 */
LA_API la_status la_state_step(la_mode mode, const void* k, const void* v, la_dtype dt,
                        const float* alpha, const float* beta, float k_scale,
                        const float* state_in, const float* z_in,
                        float* state_out, float* z_out,
                        int B, int H, int F, int S, int D,
                        void* workspace, size_t workspace_bytes, cudaStream_t stream);

/*
 * Transition and input composites of a frame interval (GDN).
 * Source: SANA-WM paper summary (paperlayer), appendix C.1, "Context-parallel
 * training" -- the 961-frame latent sequence is sharded over P GPUs along
 * time; each rank summarises its frame interval by a compact GDN transition
 * composite and input composite, the gathered summaries are combined by an
 * exclusive prefix, and every rank recovers its exact initial state.
 * Every frame is affine in the state, M_f = A_f M_{f-1} + B_f with
 * A_f = alpha_f (I - beta_f Kh_f^T Kh_f) and B_f = beta_f Kh_f^T V_f, so for
 * the F frames given here:
 *   transition_out = A_F ... A_1            [B,H,D,D] f32 (key x key)
 *   input_out      = sum_j A_F ... A_{j+1} B_j
 *                  = the state after the F frames from a zero state
 *                                           [B,H,D,D] f32, key-major
 * and the state after the interval from any start M is
 * transition_out . M + input_out.
 *
 * k, v, alpha, beta, k_scale as for la_scan_gdn (no q, no outputs); both
 * output pointers are required and must not overlap.  F == 0 gives the
 * identity and zeros.  Workspace: la_workspace_size(LA_MODE_GDN_COMPOSITE,
 * B, H, F, S, D) bytes.  bf16 inputs with 64 <= D <= 128 run on the
 * tensor-core path (the gram once, then 2 B H chain blocks: the input
 * composite from zero and the transition from the identity); other shapes
 * on the float32 SIMT kernel.
 */
LA_API la_status la_gdn_interval_composite(const void* k, const void* v, la_dtype dt,
                                           const float* alpha, const float* beta,
                                           float k_scale, float* transition_out,
                                           float* input_out, int B, int H, int F, int S, int D,
                                           void* workspace, size_t workspace_bytes,
                                           cudaStream_t stream);

/*
 * Exclusive prefix over interval composites: the initial state of every
 * interval.  Source: SANA-WM paper summary (paperlayer), appendix C.1 --
 * the all-gathered composite summaries are composed as an exclusive prefix,
 * which restores each rank's mathematically exact initial GDN state.
 *
 *   starts_out[0]   = state_in (zeros if NULL)
 *   starts_out[r+1] = T_r . starts_out[r] + U_r
 *
 * transitions, inputs in : the composites of n consecutive intervals in frame
 *                          order, each a [B, H, D, D] f32 block as
 *                          la_gdn_interval_composite writes it; T_r starts
 *                          at transitions + r * interval_stride and U_r at
 *                          inputs + r * interval_stride (in floats, at least
 *                          B*H*D*D).  Packed arrays use B*H*D*D; the
 *                          all-gathered [n][2][B, H, D, D] buffer of a
 *                          context-parallel exchange is read in place with
 *                          inputs = transitions + B*H*D*D and 2*B*H*D*D.
 * state_in            in : [B, H, D, D] f32 or NULL.
 * starts_out         out : [n, B, H, D, D] f32, the start state of each interval.
 * state_out          out : [B, H, D, D] f32 or NULL: the state after all n
 *                          intervals.
 * n >= 1; D a multiple of 16 in [16, 256].  No workspace: starts_out holds
 * the running state.  The outputs must not overlap the inputs.  float32
 * SIMT kernel, one launch.
 */
LA_API la_status la_gdn_compose_prefix(const float* transitions, const float* inputs,
                                       size_t interval_stride, const float* state_in,
                                       float* starts_out, float* state_out, int n, int B, int H,
                                       int D, cudaStream_t stream);

/*
 * Frame-wise GDN scan for callers that cannot allocate device memory.
 * No counterpart in the pages: it is the same computation as la_scan_gdn,
 * but its scratch is a fixed area built into the library instead of a
 * caller-provided workspace.  It exists for callers that cannot call
 * cudaMalloc: for example a plug-in running inside a host framework that
 * owns every device allocation and gives its plug-ins no scratch memory, or
 * a real-time loop whose rules forbid cudaMalloc/cudaFree because they
 * synchronise the device and can fail mid-run.
 *
 * Arguments, layouts and errors are those of la_scan_gdn; there is no
 * workspace argument.  The caller still owns and passes every input and
 * output.  This entry point calls no cudaMalloc, cudaFree or other
 * allocating routine.
 *
 * Scratch.  A __device__ array of LA_NOALLOC_SCRATCH_BYTES (64 MiB) that
 *   every GPU which loads the library holds until the process exits.  A call
 *   whose la_workspace_size(LA_MODE_GDN, B, H, F, S, D) exceeds it returns
 *   LA_ERR_UNSUPPORTED before enqueuing anything.  What fits (la_workspace_size
 *   is the exact test):
 *     - bf16 inputs, 64 <= D <= 128, B*H <= 49 (on a 148-SM B200: the
 *       single-kernel path): about 1.5 MiB per (b, h) pair whatever F is,
 *       so B*H <= 42;
 *     - bf16 inputs, 64 <= D <= 128, more pairs (the three-kernel path):
 *       per-frame buffers of 128 KiB per (b, h, frame) plus the state
 *       (64 KiB per pair at D = 128), so about B*H*F <= 480 at D = 128
 *       (for example B*H = 63 with F <= 7);
 *     - bf16 inputs, 128 < D <= 256: per-frame buffers of about 0.4 MiB per
 *       (b, h, frame of a pipeline chunk), so only short clips of few heads;
 *     - float32 inputs, or D < 64: a few hundred bytes.
 * Sharing.  All calls on a device share the one array, and it keeps the
 *   last call's contents; the library clears what must start at zero at the
 *   start of every call.  Calls whose GPU work overlaps (on different
 *   streams, or from different threads) race on the array and give wrong
 *   results: serialise them, for example on one stream.
 * Set-up.  The first call on each device looks up the array's device
 *   address (cudaGetSymbolAddress) with that device current; make that first
 *   call before any stream capture begins.
 * Status.  A bounded device-side wait that gives up records LA_ERR_TIMEOUT in
 *   the array, and the outputs of that call are then not valid;
 *   la_query_noalloc_status reads it back.
 */
#define LA_NOALLOC_SCRATCH_BYTES (64u * 1024u * 1024u)
LA_API la_status la_scan_gdn_noalloc(const void* q, const void* k, const void* v, void* o,
                                     la_dtype dt, const float* alpha, const float* beta,
                                     float k_scale, const float* state_in, float* state_out,
                                     int B, int H, int F, int S, int D, cudaStream_t stream);

/* Synchronise `stream`, then report the device-side status that the most
 * recent la_scan_gdn_noalloc call on the current device recorded in the
 * built-in scratch array: LA_OK, or LA_ERR_TIMEOUT when a bounded wait gave
 * up (that call's outputs are then not valid).  Returns LA_ERR_CUDA if the
 * synchronisation fails.  Like la_query_device_status, it synchronises on
 * purpose.  No counterpart in the pages. */
LA_API la_status la_query_noalloc_status(cudaStream_t stream);

/*
 * The scan of a clip held in HOST memory, streamed through the GPU in chunks
 * of frames.  Source: SANA-WM paper summary (paperlayer), section 3,
 * "Chunk-causal deployment", and the SANA-Video talk, block KV cache
 * segment -- the recurrent state carries everything a later chunk needs
 * from the earlier ones, so a clip can be processed chunk by chunk.
 * The computation is that of la_scan_relu (mode LA_MODE_RELU) or
 * la_scan_gdn (mode LA_MODE_GDN) on the whole clip; the chunking changes
 * only where the data is while it runs.
 *
 * Pipeline.  Chunk c+1 is copied in (host to device) while chunk c is
 *   scanned on `stream` and chunk c-1's output is copied out, on two copy
 *   streams of the library's own, over a ring of three chunk slots in the
 *   workspace.  The state stays on the device between chunks.
 * Memory.  q, k, v, o, alpha, beta, state_in, z_in, state_out and z_out
 *   are HOST pointers with the layouts of the shared conventions above
 *   (device or managed pointers are rejected with LA_ERR_INVALID_ARG).
 *   Page-locked (pinned) host memory lets the copies overlap the scan and
 *   each other; pageable memory is accepted, but the driver stages its
 *   copies and the call may return only after them.  `workspace` is device
 *   memory of the current device, 256-byte aligned, of at least
 *   la_host_workspace_size(mode, dt, B, H, F, S, D, chunk_frames) bytes;
 *   la_query_device_status accepts it.
 * Chunking.  chunk_frames > 0 sets the frames per chunk (the last chunk may
 *   be shorter); chunk_frames <= 0 picks about 16 chunks
 *   (la_host_chunk_frames reports the choice).
 * Mode.    LA_MODE_GDN uses alpha, beta, k_scale and ignores eps, z_in and
 *   z_out; LA_MODE_RELU uses eps, z_in and z_out and ignores the gates.
 * Asynchrony.  Nothing starts before the work already queued on `stream`,
 *   and work queued on `stream` after the call starts after every copy of
 *   the call (host buffers may be read or reused once `stream` reaches that
 *   point).  Argument errors return before anything is enqueued; a later
 *   failure returns LA_ERR_CUDA (or the chunk scan's status) with the chunks
 *   enqueued so far still ordered on `stream`.
 * Resources.  The first call on a device creates two non-blocking streams
 *   and a few events for it, kept until the process exits; calls on one
 *   device serialise their enqueueing on a lock and share the copy streams.
 */
LA_API la_status la_scan_host(la_mode mode, const void* q, const void* k, const void* v, void* o,
                              la_dtype dt, const float* alpha, const float* beta, float k_scale,
                              float eps, const float* state_in, const float* z_in,
                              float* state_out, float* z_out,
                              int B, int H, int F, int S, int D, int chunk_frames,
                              void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Device workspace bytes la_scan_host needs for this mode, dtype, shape and
 * chunking; 0 for an unsupported or invalid combination. */
LA_API size_t la_host_workspace_size(la_mode mode, la_dtype dt, int B, int H, int F, int S, int D,
                                     int chunk_frames);

/* Frames per chunk that la_scan_host uses for F frames and this
 * chunk_frames argument (0 when F < 0). */
LA_API int la_host_chunk_frames(int F, int chunk_frames);

/* Workspace bytes a call of this mode and shape needs (either dtype).
 * Returns 0 for an unsupported shape.  The library has no counterpart in
 * the pages; it exists because the library never allocates. */
LA_API size_t la_workspace_size(la_mode mode, int B, int H, int F, int S, int D);

/* Synchronise `stream`, then report the device-side status that the most
 * recent call using `workspace` recorded: LA_OK, or LA_ERR_TIMEOUT when a
 * bounded inter-block wait gave up (its outputs are then not valid).
 * Returns LA_ERR_CUDA if the synchronisation itself fails. */
LA_API la_status la_query_device_status(void* workspace, cudaStream_t stream);

/* How a call of this mode, dtype and shape runs: stores the number of
 * kernels one call launches in *kernels (if not NULL) and returns the name
 * of the kernel path: "tcgen05_fused" (bf16, 64 <= D <= 128, few heads: one
 * persistent kernel), "tcgen05" (bf16, 64 <= D <= 128, many heads: three
 * kernels per frame chunk or head group), "tcgen05_wide" (bf16,
 * 128 < D <= 256: three kernels per frame chunk) or "simt_f32" (float32
 * inputs, D < 64); NULL for an unsupported
 * shape.  No counterpart in the pages: it lets a caller check which
 * kernels its calls use. */
LA_API const char* la_plan(la_mode mode, la_dtype dt, int B, int H, int F, int S, int D,
                           int* kernels);

/* Static, human-readable name of a status code. */
LA_API const char* la_status_string(la_status s);

#ifdef __cplusplus
}
#endif
#endif /* LA_SCAN_H */
