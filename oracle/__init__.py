"""CPU oracle for the block-causal, frame-wise linear-attention scan.

TEST INFRASTRUCTURE ONLY.  This package is a plain, slow, obviously correct
float64 restatement of what the scan computes.  Only the test suite, the
smoke check in ``__graft_entry__`` and the CPU-baseline leg of ``bench.py``
may import it; the CUDA library and its Python binding never do, and share
no code with it.  The two meet only through the seeded generator in
``synth``.

Equations (frozen before any kernel was written).  Per batch b and head h,
frame f = 1..F holds Q_f, K_f, V_f of shape [S, D].  The state is stored
key-major, M in R^{D_k x D_v}, so that the output is always O_f = Q~_f M_f.

ReLU mode -- SANA-Video talk (ICLR 2026 oral), block KV cache segment: the
D x D state is updated additively block by block and each block reads the
cached state of all earlier blocks plus its own contribution; SANA-Video
guide (lpnh.cn), section "核心机制": each block attends to itself and to
every earlier block.  phi = max(x, 0):
    M_f = M_{f-1} + phi(K_f)^T V_f
    z_f = z_{f-1} + sum_t phi(K_f[t, :])
    O_f[t, :] = phi(Q_f[t, :]) M_f / (phi(Q_f[t, :]) . z_f + eps)

GDN mode -- SANA-WM digest, method details ("Periodic softmax" and "Spatial
Explosion" paragraphs) and SANA-WM paper summary (paperlayer), section 3,
"Hybrid GDN/Softmax Attention": a D x D state is scanned latent frame by
latent frame, all spatial tokens of a frame enter one update, a decay gate
and an update gate control forgetting, and keys are scaled by 1/sqrt(D*S):
    Kh_f = k_scale * K_f
    M_f  = alpha_f (I - beta_f Kh_f^T Kh_f) M_{f-1} + beta_f Kh_f^T V_f
    O_f  = Q_f M_f
Readings where the pages are silent: inclusive causality (frame f reads
M_f); alpha scales the decayed-and-erased old state but not the write;
beta scales both erase and write; gates are per (b, h, f); no feature map
or normaliser in GDN mode; eps = 1e-6 by default in ReLU mode.

Composite form (SANA-WM paper summary, appendix C.1, context-parallel
training): each frame is affine, M_f = A_f M_{f-1} + B_f with
A_f = alpha_f (I - beta_f G_f), G_f = Kh_f^T Kh_f, B_f = beta_f Kh_f^T V_f,
so a frame interval has a transition composite and an input composite, and
an exclusive prefix over intervals recovers each interval's exact initial
state.

Reversed GDN scan -- SANA-WM paper summary, section 3, "Chunk-causal
deployment": a reversed GDN scan that is reset at every chunk boundary gives
each frame the later frames of its own chunk as context without leaking
across chunks.  Reading (the pages give no formula): frames are split into
chunks [c C, min((c + 1) C, F)); inside a chunk the GDN recurrence above
runs from the chunk's last frame back to its first, from a zero state, and
frame f reads the state after its own update:
    M_{e+1} = 0 (e = last frame of the chunk)
    M_f = alpha_f (I - beta_f Kh_f^T Kh_f) M_{f+1} + beta_f Kh_f^T V_f
    O_f = Q_f M_f

Per-token update gate -- SANA-WM paper summary, section 3, "Hybrid
GDN/Softmax Attention": a decay and a per-token update gate control old
content.  Reading: the update gate of frame f is a vector beta_f in R^S (one
value per spatial token) that weighs each token's erase and write, i.e.
beta_f Kh^T Kh and beta_f Kh^T V become Kh^T diag(beta_f) Kh and
Kh^T diag(beta_f) V:
    M_f = alpha_f (M_{f-1} - Kh_f^T diag(beta_f) Kh_f M_{f-1}) + Kh_f^T diag(beta_f) V_f

Fused input preparation -- SANA-WM digest, method details, "Context-Parallel
+ Fused Triton" paragraph (RMSNorm + ReLU + key scaling + UCPE/RoPE + GDN
scan fused into one kernel); SANA-WM paper summary, appendix C.1 (the fused
kernel combines normalization, activation, scaling, positional preparation
and recurrent scanning); SANA-Video talk, 3D RoPE for the linear attention.
Readings (the pages give the order of the steps, no formulas):
  - RMSNorm over the head dimension of each token, with a per-head weight:
        y = x / sqrt(mean_d x_d^2 + eps_n) * w
  - then phi = ReLU, then 3D RoPE over (latent frame, row, column): the D/2
    adjacent channel pairs (2i, 2i+1) are split into a temporal group (the
    first D/2 - 2 floor(D/6) pairs), a height group and a width group
    (floor(D/6) pairs each); pair i of a group of n pairs turns by
    pos * base^(-i / n), pos being the token's frame (plus a frame offset),
    row or column on the latent grid (token s of a frame sits at row
    s // grid_w, column s % grid_w);
  - the key scale stays inside the scan (k_scale), as before;
  - GDN: q~ = RoPE(phi(RMSNorm(q))), k~ = RoPE(phi(RMSNorm(k))) enter the scan;
  - ReLU: the numerator uses the rotated features and the normaliser the
    unrotated ones (rotated ReLU features can be negative, which would
    remove the positivity the normaliser relies on):
        M_f = M_{f-1} + RoPE(phi_k)^T V_f,   z_f = z_{f-1} + sum_t phi_k[t]
        O_f[t] = RoPE(phi_q)[t] M_f / (phi_q[t] . z_f + eps),
    with phi_x = phi(RMSNorm(x)).

Array layout: q, k, v, o are [B, H, F, S, D]; alpha, beta are [B, H, F];
state is [B, H, D, D] (key-major); z is [B, H, D].  Every input is widened
to float64 first (bf16 and fp32 widen exactly).
"""
from __future__ import annotations

from typing import List, Optional, Sequence, Tuple

import numpy as np

__all__ = [
    "relu_scan", "gdn_scan", "relu_state_step", "gdn_state_step",
    "gdn_interval_composite", "compose_exclusive_prefix", "gdn_scan_reverse_chunked",
    "gdn_scan_token_beta", "rms_norm", "rope3d_groups", "rope3d_angles", "rope3d_apply",
    "prep_features", "gdn_scan_prep", "relu_scan_prep",
]


def _f64(x):
    return None if x is None else np.asarray(x, dtype=np.float64)


def _phi(x: np.ndarray) -> np.ndarray:
    """ReLU feature map of the SANA-Video linear attention."""
    return np.maximum(x, 0.0)


def _shape(k: np.ndarray) -> Tuple[int, int, int, int, int]:
    if k.ndim != 5:
        raise ValueError("expected [B, H, F, S, D]")
    return k.shape  # type: ignore[return-value]


# ----------------------------------------------------------------------------
# ReLU linear attention with normaliser
# ----------------------------------------------------------------------------
def relu_scan(q, k, v, eps: float = 1e-6, state_in=None, z_in=None,
              want_output: bool = True):
    """Block-causal ReLU linear attention over latent frames.

    SANA-Video talk, block KV cache segment (state S of fixed shape D x D,
    added to block by block, cached between blocks) and SANA-Video guide,
    "核心机制" (each block sees itself and all earlier blocks).

    Returns (o, M_F, z_F); o is None when want_output is False.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, H, F, S, D = _shape(k)
    o = np.zeros((B, H, F, S, D)) if want_output else None
    m_out = np.zeros((B, H, D, D))
    z_out = np.zeros((B, H, D))
    m0 = _f64(state_in)
    z0 = _f64(z_in)
    for b in range(B):
        for h in range(H):
            M = np.zeros((D, D)) if m0 is None else m0[b, h].copy()
            z = np.zeros(D) if z0 is None else z0[b, h].copy()
            for f in range(F):
                pk = _phi(k[b, h, f])                 # [S, D_k]
                M = M + pk.T @ v[b, h, f]             # additive state update
                z = z + pk.sum(axis=0)                # normaliser update
                if want_output:
                    pq = _phi(q[b, h, f])             # [S, D_k]
                    num = pq @ M                      # [S, D_v]
                    den = pq @ z                      # [S]
                    o[b, h, f] = num / (den + eps)[:, None]
            m_out[b, h] = M
            z_out[b, h] = z
    return o, m_out, z_out


def relu_state_step(k, v, state_in=None, z_in=None):
    """Advance the ReLU cache over finished frames without producing outputs."""
    _, m, z = relu_scan(k, k, v, 0.0, state_in, z_in, want_output=False)
    return m, z


# ----------------------------------------------------------------------------
# Frame-wise Gated DeltaNet
# ----------------------------------------------------------------------------
def gdn_scan(q, k, v, alpha, beta, k_scale: float, state_in=None,
             want_output: bool = True):
    """Frame-wise Gated DeltaNet with key scaling.

    SANA-WM digest, method details, and SANA-WM paper summary, section 3
    ("Hybrid GDN/Softmax Attention"): one D x D state per head, one update
    per latent frame that takes in all of the frame's spatial tokens; decay
    and update gates; keys scaled by 1/sqrt(D*S) (passed as k_scale).

    Each frame is computed in the direct order
        P = Kh M;  M <- alpha (M - beta Kh^T P) + beta Kh^T V;  O = Q M.
    Returns (o, M_F); o is None when want_output is False.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    alpha, beta = _f64(alpha), _f64(beta)
    B, H, F, S, D = _shape(k)
    o = np.zeros((B, H, F, S, D)) if want_output else None
    m_out = np.zeros((B, H, D, D))
    m0 = _f64(state_in)
    kappa = float(k_scale)
    for b in range(B):
        for h in range(H):
            M = np.zeros((D, D)) if m0 is None else m0[b, h].copy()
            for f in range(F):
                a = alpha[b, h, f]
                bt = beta[b, h, f]
                kh = kappa * k[b, h, f]               # [S, D_k]
                P = kh @ M                            # [S, D_v]  read old state
                M = a * (M - bt * (kh.T @ P)) + bt * (kh.T @ v[b, h, f])
                if want_output:
                    o[b, h, f] = q[b, h, f] @ M       # reads the updated state
            m_out[b, h] = M
    return o, m_out


def gdn_scan_reverse_chunked(q, k, v, alpha, beta, k_scale: float, chunk_frames: int):
    """Reversed frame-wise GDN, reset at every chunk boundary.

    SANA-WM paper summary, section 3, "Chunk-causal deployment".  For each
    chunk of chunk_frames frames (the last one may be shorter) the state
    starts at zero after the chunk's last frame and the frames are taken
    from last to first, each in the direct order of gdn_scan:
        P = Kh M;  M <- alpha (M - beta Kh^T P) + beta Kh^T V;  O = Q M.
    No state enters or leaves.  Returns o, [B, H, F, S, D].
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    alpha, beta = _f64(alpha), _f64(beta)
    B, H, F, S, D = _shape(k)
    C = int(chunk_frames)
    if C < 1:
        raise ValueError("chunk_frames must be >= 1")
    o = np.zeros((B, H, F, S, D))
    kappa = float(k_scale)
    for b in range(B):
        for h in range(H):
            for start in range(0, F, C):
                end = min(start + C, F)               # frames start .. end-1
                M = np.zeros((D, D))                  # reset at the chunk boundary
                for f in range(end - 1, start - 1, -1):
                    a = alpha[b, h, f]
                    bt = beta[b, h, f]
                    kh = kappa * k[b, h, f]
                    P = kh @ M
                    M = a * (M - bt * (kh.T @ P)) + bt * (kh.T @ v[b, h, f])
                    o[b, h, f] = q[b, h, f] @ M
    return o


def gdn_scan_token_beta(q, k, v, alpha, beta_token, k_scale: float, state_in=None):
    """Frame-wise GDN with a per-token update gate.

    SANA-WM paper summary, section 3 ("Hybrid GDN/Softmax Attention"): decay
    gate per frame, update gate per token.  beta_token: [B, H, F, S].  Each
    frame in the direct order
        P = Kh M;  M <- alpha (M - Kh^T (beta * P)) + Kh^T (beta * V);  O = Q M,
    where beta * X scales row t (token t) of X by beta_t.
    Returns (o, M_F).
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    alpha, bt = _f64(alpha), _f64(beta_token)
    B, H, F, S, D = _shape(k)
    o = np.zeros((B, H, F, S, D))
    m_out = np.zeros((B, H, D, D))
    m0 = _f64(state_in)
    kappa = float(k_scale)
    for b in range(B):
        for h in range(H):
            M = np.zeros((D, D)) if m0 is None else m0[b, h].copy()
            for f in range(F):
                a = alpha[b, h, f]
                w = bt[b, h, f][:, None]              # [S, 1] token weights
                kh = kappa * k[b, h, f]
                P = kh @ M
                M = a * (M - kh.T @ (w * P)) + kh.T @ (w * v[b, h, f])
                o[b, h, f] = q[b, h, f] @ M
            m_out[b, h] = M
    return o, m_out


def gdn_state_step(k, v, alpha, beta, k_scale: float, state_in=None):
    """Advance the GDN state over finished frames without producing outputs."""
    _, m = gdn_scan(k, k, v, alpha, beta, k_scale, state_in, want_output=False)
    return m


def gdn_interval_composite(k, v, alpha, beta, k_scale: float):
    """Transition and input composites of one frame interval for one head.

    SANA-WM paper summary, appendix C.1: a rank owning a frame interval
    summarises it by a compact transition composite and input composite.
    For frames j = 1..n of the interval, with A_j = alpha_j (I - beta_j G_j)
    and B_j = beta_j Kh_j^T V_j:
        T = A_n ... A_1,    U = sum_j A_n ... A_{j+1} B_j,
    so that M_end = T M_start + U.
    k, v: [n, S, D]; alpha, beta: [n].  Returns (T, U), each [D, D].
    """
    k, v = _f64(k), _f64(v)
    alpha, beta = _f64(alpha), _f64(beta)
    n, S, D = k.shape
    T = np.eye(D)
    U = np.zeros((D, D))
    for j in range(n):
        kh = float(k_scale) * k[j]
        A = alpha[j] * (np.eye(D) - beta[j] * (kh.T @ kh))
        Bj = beta[j] * (kh.T @ v[j])
        T = A @ T
        U = A @ U + Bj
    return T, U


def compose_exclusive_prefix(composites: Sequence[Tuple[np.ndarray, np.ndarray]],
                             m0: Optional[np.ndarray] = None) -> List[np.ndarray]:
    """Initial state of each interval from the interval composites.

    SANA-WM paper summary, appendix C.1: the gathered composite summaries are
    combined by an exclusive prefix, giving every interval its exact initial
    state.  Returns [M_start of interval 0, M_start of interval 1, ...].
    """
    D = composites[0][0].shape[0]
    M = np.zeros((D, D)) if m0 is None else _f64(m0).copy()
    starts = []
    for T, U in composites:
        starts.append(M.copy())
        M = T @ M + U
    return starts


# ----------------------------------------------------------------------------
# Fused input preparation: RMSNorm, ReLU, 3D RoPE
# ----------------------------------------------------------------------------
def rms_norm(x, weight=None, eps: float = 1e-6):
    """RMSNorm of every token over the head dimension (the last axis):
    x / sqrt(mean(x^2) + eps) * weight.  weight: [D] or None (ones)."""
    x = _f64(x)
    y = x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)
    return y if weight is None else y * _f64(weight)


def rope3d_groups(D: int) -> Tuple[int, int, int]:
    """Channel pairs of the temporal, height and width groups of 3D RoPE."""
    P = D // 2
    n_hw = P // 3
    return P - 2 * n_hw, n_hw, n_hw


def rope3d_angles(F: int, grid_h: int, grid_w: int, D: int, frame_offset: int = 0,
                  base: float = 10000.0) -> np.ndarray:
    """Rotation angle of every (frame, token, channel pair): [F, grid_h*grid_w, D/2].
    Pair i of a group of n pairs turns by pos * base^(-i/n)."""
    n_t, n_h, n_w = rope3d_groups(D)
    S = grid_h * grid_w
    shape = (F, S)
    f_pos = np.broadcast_to((np.arange(F) + frame_offset)[:, None].astype(np.float64), shape)
    r_pos = np.broadcast_to((np.arange(S) // grid_w)[None, :].astype(np.float64), shape)
    c_pos = np.broadcast_to((np.arange(S) % grid_w)[None, :].astype(np.float64), shape)
    ang = np.zeros((F, S, D // 2))
    col = 0
    for n, pos in ((n_t, f_pos), (n_h, r_pos), (n_w, c_pos)):
        for i in range(n):
            ang[:, :, col + i] = pos * base ** (-i / n)
        col += n
    return ang


def rope3d_apply(x, angles) -> np.ndarray:
    """Turn each channel pair (2i, 2i+1) of x [..., F, S, D] by angles [F, S, D/2]."""
    x = _f64(x)
    c, s = np.cos(angles), np.sin(angles)
    x0, x1 = x[..., 0::2], x[..., 1::2]
    y = np.empty_like(x)
    y[..., 0::2] = x0 * c - x1 * s
    y[..., 1::2] = x0 * s + x1 * c
    return y


def prep_features(x, weight, norm_eps: float, grid_h: int, grid_w: int,
                  frame_offset: int = 0, base: float = 10000.0, relu: bool = True,
                  rope: bool = True):
    """The prepared features of x [B, H, F, S, D]: RMSNorm (weight [H, D] or
    None), then ReLU, then 3D RoPE.  Returns (rotated, unrotated)."""
    x = _f64(x)
    B, H, F, S, D = x.shape
    if grid_h * grid_w != S:
        raise ValueError("S must equal grid_h * grid_w")
    y = np.empty_like(x)
    for h in range(H):
        y[:, h] = rms_norm(x[:, h], None if weight is None else _f64(weight)[h], norm_eps)
    if relu:
        y = _phi(y)
    if not rope:
        return y, y
    return rope3d_apply(y, rope3d_angles(F, grid_h, grid_w, D, frame_offset, base)), y


def gdn_scan_prep(q, k, v, alpha, beta, k_scale: float, q_weight, k_weight,
                  norm_eps: float, grid_h: int, grid_w: int, frame_offset: int = 0,
                  base: float = 10000.0, relu: bool = True, rope: bool = True,
                  state_in=None):
    """Frame-wise GDN on prepared queries and keys (the fused kernel of the
    SANA-WM digest: RMSNorm + ReLU + key scaling + RoPE + GDN scan).
    Returns (o, M_F)."""
    qt, _ = prep_features(q, q_weight, norm_eps, grid_h, grid_w, frame_offset, base, relu, rope)
    kt, _ = prep_features(k, k_weight, norm_eps, grid_h, grid_w, frame_offset, base, relu, rope)
    return gdn_scan(qt, kt, v, alpha, beta, k_scale, state_in)


def relu_scan_prep(q, k, v, eps: float, q_weight, k_weight, norm_eps: float, grid_h: int,
                   grid_w: int, frame_offset: int = 0, base: float = 10000.0,
                   rope: bool = True, state_in=None, z_in=None):
    """Block-causal ReLU linear attention on prepared features: RoPE on the
    numerator's features only, the normaliser on the unrotated ones.
    Returns (o, M_F, z_F)."""
    qr, qn = prep_features(q, q_weight, norm_eps, grid_h, grid_w, frame_offset, base, True, rope)
    kr, kn = prep_features(k, k_weight, norm_eps, grid_h, grid_w, frame_offset, base, True, rope)
    v = _f64(v)
    B, H, F, S, D = v.shape
    o = np.zeros((B, H, F, S, D))
    m_out = np.zeros((B, H, D, D))
    z_out = np.zeros((B, H, D))
    m0, z0 = _f64(state_in), _f64(z_in)
    for b in range(B):
        for h in range(H):
            M = np.zeros((D, D)) if m0 is None else m0[b, h].copy()
            z = np.zeros(D) if z0 is None else z0[b, h].copy()
            for f in range(F):
                M = M + kr[b, h, f].T @ v[b, h, f]        # rotated keys in the state
                z = z + kn[b, h, f].sum(axis=0)          # unrotated keys in the normaliser
                num = qr[b, h, f] @ M
                den = qn[b, h, f] @ z
                o[b, h, f] = num / (den + eps)[:, None]
            m_out[b, h] = M
            z_out[b, h] = z
    return o, m_out, z_out
