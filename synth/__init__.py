"""Seeded synthetic inputs for the frame-wise linear-attention scan.

This module only draws random tensors and rounds them to the storage
precision.  It holds none of the scan's arithmetic: no feature map, no
state update, no gate application.  Both the CPU oracle and the CUDA path
are fed from here, so that they see bit-identical inputs.

Layout conventions (shared by every consumer):
  q, k, v, o : [B, H, F, S, D]   D fastest; float32 or bfloat16 bits
  alpha, beta: [B, H, F]         float32
  state      : [B, H, D, D]      float32, key-major (row = key dim)
  z          : [B, H, D]         float32

Random streams: numpy PCG64 seeded by SeedSequence([seed, tensor_id, b, h])
so that any (b, h) slice can be regenerated on its own.  bf16 values are
made in float32 and rounded to nearest, ties to even.

The workload shapes mirror the pages' video latents: 480x832 video with a
[4, 8, 8] VAE stride and 2x2 patches gives a 30x52 token grid per latent
frame (SANA-Video guide, lpnh.cn, model config section); a 720p minute at
24 fps gives 181 latent frames of 22x40 tokens (SANA-WM digest, method
details).  No benchmark item of the pages is reproduced; the tensors are
random.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Tuple

import numpy as np

TENSOR_IDS = {"q": 0, "k": 1, "v": 2, "alpha": 10, "beta": 11, "beta_token": 12,
              "outlier": 20, "state": 30, "z": 31, "q_weight": 40, "k_weight": 41}


# ----------------------------------------------------------------------------
# bf16 storage helpers (round to nearest even; exact widening)
# ----------------------------------------------------------------------------
def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bfloat16 (nearest, ties to even); return uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Widen bfloat16 bits to float32 exactly."""
    b = np.ascontiguousarray(b, dtype=np.uint16)
    return (b.astype(np.uint32) << np.uint32(16)).view(np.float32)


# ----------------------------------------------------------------------------
# Workload description
# ----------------------------------------------------------------------------
@dataclasses.dataclass(frozen=True)
class Spec:
    name: str
    B: int
    H: int
    F: int
    S: int
    D: int
    dtype: str                      # "f32" or "bf16": storage of q, k, v, o
    seed: int
    modes: Tuple[str, ...] = ("relu", "gdn")
    keys_l2: bool = False           # L2-normalise each key token (fp32) before rounding
    outlier_frac: float = 0.0       # fraction of token positions scaled x outlier_scale
    outlier_scale: float = 20.0
    alpha: Tuple = ("uniform", 0.9, 1.0)
    beta: Tuple = ("uniform", 0.0, 1.0)
    eps: float = 1e-6               # ReLU-mode normaliser epsilon
    chunk_frames: int = 0           # >0: streamed in chunks of this many frames
    grid: Optional[Tuple[int, int]] = None   # latent grid (rows, columns) of a frame, S = rows * cols

    @property
    def k_scale(self) -> float:
        """1/sqrt(D*S), rounded to float32 (passed to the scan as an argument)."""
        return float(np.float32(1.0 / math.sqrt(self.D * self.S)))

    @property
    def elem_bytes(self) -> int:
        return 4 if self.dtype == "f32" else 2

    def with_(self, **kw) -> "Spec":
        return dataclasses.replace(self, **kw)


# The five workloads (seeds are the position in this table).
WORKLOADS = {
    "tiny_fp32": Spec("tiny_fp32_B1_H2_D32_F8_S64", B=1, H=2, F=8, S=64, D=32, dtype="f32",
            seed=0, modes=("relu", "gdn"), alpha=("uniform", 0.9, 1.0),
            beta=("uniform", 0.0, 1.0)),
    "relu_480p": Spec("relu_480p_B1_H20_D112_F21_S1560", B=1, H=20, F=21, S=1560, D=112,
            dtype="bf16", seed=1, modes=("relu",), grid=(30, 52)),
    "gdn_720p_60s": Spec("gdn_720p_60s_B1_H20_D128_F181_S880", B=1, H=20, F=181, S=880, D=128,
            dtype="bf16", seed=2, modes=("gdn",), keys_l2=True,
            alpha=("sigmoid_normal", 3.0, 1.0), beta=("sigmoid_normal", 0.0, 1.0),
            grid=(22, 40)),
    # the 720p clip with raw keys, for the scan with the input preparation
    # fused (RMSNorm replaces the harness's L2 normalisation of the keys)
    "gdn_720p_60s_raw": Spec("gdn_720p_60s_raw_B1_H20_D128_F181_S880", B=1, H=20, F=181, S=880,
            D=128, dtype="bf16", seed=2, modes=("gdn",), keys_l2=False,
            alpha=("sigmoid_normal", 3.0, 1.0), beta=("sigmoid_normal", 0.0, 1.0),
            grid=(22, 40)),
    "gdn_stream": Spec("gdn_stream_B4_H20_D128_8x8frames_S880", B=4, H=20, F=64, S=880, D=128,
            dtype="bf16", seed=3, modes=("gdn",), keys_l2=True,
            alpha=("sigmoid_normal", 3.0, 1.0), beta=("sigmoid_normal", 0.0, 1.0),
            chunk_frames=8, grid=(22, 40)),
    "stress_d256": Spec("stress_B1_H16_D256_F512_S1024", B=1, H=16, F=512, S=1024, D=256,
            dtype="bf16", seed=4, modes=("relu", "gdn"), outlier_frac=0.01,
            alpha=("uniform", 0.8, 1.0), beta=("uniform", 0.0, 1.0), grid=(32, 32)),
}


WORKLOAD_NAMES = tuple(WORKLOADS)


def workload(name: str) -> Spec:
    """The seeded synthetic workload of this name (see WORKLOADS)."""
    return WORKLOADS[name]


def _rng(*key: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence(list(key))))


def outlier_rows(spec: Spec, b: int) -> np.ndarray:
    """Token positions (flat index f*S+s) scaled as outliers in batch item b.

    Exactly round(frac*F*S) positions, uniform without replacement, shared by
    q, k and v and by every head (an outlier token).
    """
    n = int(round(spec.outlier_frac * spec.F * spec.S))
    if n == 0:
        return np.zeros(0, dtype=np.int64)
    rng = _rng(spec.seed, TENSOR_IDS["outlier"], b)
    return np.sort(rng.choice(spec.F * spec.S, size=n, replace=False))


def _raw_slice(spec: Spec, tensor: str, b: int, h: int) -> np.ndarray:
    rng = _rng(spec.seed, TENSOR_IDS[tensor], b, h)
    x = rng.standard_normal((spec.F, spec.S, spec.D), dtype=np.float32)
    rows = outlier_rows(spec, b)
    if rows.size:
        flat = x.reshape(spec.F * spec.S, spec.D)
        flat[rows] *= np.float32(spec.outlier_scale)
    if tensor == "k" and spec.keys_l2:
        nrm = np.sqrt(np.sum(x.astype(np.float64) ** 2, axis=-1, keepdims=True))
        x = (x / nrm.astype(np.float32)).astype(np.float32)
    return x


def slice_storage(spec: Spec, tensor: str, b: int, h: int) -> np.ndarray:
    """Storage array of one (b, h) slice, [F, S, D]: float32, or uint16 bf16 bits."""
    x = _raw_slice(spec, tensor, b, h)
    if spec.dtype == "bf16":
        return f32_to_bf16_bits(x)
    return x


def slice_values(spec: Spec, tensor: str, b: int, h: int) -> np.ndarray:
    """The exact values the scan sees for one (b, h) slice, as float32 [F, S, D]."""
    s = slice_storage(spec, tensor, b, h)
    if spec.dtype == "bf16":
        return bf16_bits_to_f32(s)
    return s


def for_each_slice(spec: Spec, tensor: str, sink, threads: Optional[int] = None) -> None:
    """Generate every (b, h) slice of `tensor` on a thread pool and hand each
    to sink(b, h, storage_array).  Slices are independent streams, so the
    result does not depend on the thread count or order."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    jobs = [(b, h) for b in range(spec.B) for h in range(spec.H)]
    n = threads or min(len(jobs), max(1, len(os.sched_getaffinity(0))))

    def one(bh):
        b, h = bh
        return b, h, slice_storage(spec, tensor, b, h)

    if n <= 1:
        for bh in jobs:
            sink(*one(bh))
        return
    with ThreadPoolExecutor(n) as ex:
        for b, h, arr in ex.map(one, jobs):
            sink(b, h, arr)


def full_storage(spec: Spec, tensor: str, threads: Optional[int] = None) -> np.ndarray:
    """Storage array [B, H, F, S, D] (float32 or uint16 bf16 bits)."""
    dt = np.float32 if spec.dtype == "f32" else np.uint16
    out = np.empty((spec.B, spec.H, spec.F, spec.S, spec.D), dtype=dt)

    def put(b, h, arr):
        out[b, h] = arr

    for_each_slice(spec, tensor, put, threads)
    return out


def full_values(spec: Spec, tensor: str) -> np.ndarray:
    st = full_storage(spec, tensor)
    return bf16_bits_to_f32(st) if spec.dtype == "bf16" else st


def _draw_gate(dist: Tuple, rng: np.random.Generator, shape) -> np.ndarray:
    kind = dist[0]
    if kind == "uniform":
        x = rng.uniform(dist[1], dist[2], size=shape)
    elif kind == "sigmoid_normal":
        n = rng.normal(dist[1], dist[2], size=shape)
        x = 1.0 / (1.0 + np.exp(-n))
    elif kind == "const":
        x = np.full(shape, float(dist[1]))
    else:
        raise ValueError(f"unknown gate distribution {dist!r}")
    return x.astype(np.float32)


def gates(spec: Spec) -> Tuple[np.ndarray, np.ndarray]:
    """Per-frame, per-head decay alpha and update gate beta, float32 [B, H, F]."""
    shape = (spec.B, spec.H, spec.F)
    a = _draw_gate(spec.alpha, _rng(spec.seed, TENSOR_IDS["alpha"]), shape)
    bt = _draw_gate(spec.beta, _rng(spec.seed, TENSOR_IDS["beta"]), shape)
    return a, bt


def token_gates(spec: Spec) -> np.ndarray:
    """Per-token update gate beta, float32 [B, H, F, S], drawn from the
    workload's beta distribution (one value per token instead of per frame)."""
    shape = (spec.B, spec.H, spec.F, spec.S)
    return _draw_gate(spec.beta, _rng(spec.seed, TENSOR_IDS["beta_token"]), shape)


def norm_weights(spec: Spec, tensor: str) -> np.ndarray:
    """Per-head RMSNorm weight of q or k for the fused input preparation,
    float32 [H, D] drawn from U(0.5, 1.5) (random-init stand-in for a
    trained weight)."""
    rng = _rng(spec.seed, TENSOR_IDS[tensor + "_weight"])
    return rng.uniform(0.5, 1.5, size=(spec.H, spec.D)).astype(np.float32)


def random_state(spec: Spec, scale: float = 1.0) -> Tuple[np.ndarray, np.ndarray]:
    """A float32 initial state [B,H,D,D] and non-negative normaliser [B,H,D]."""
    rng = _rng(spec.seed, TENSOR_IDS["state"])
    m = (scale * rng.standard_normal((spec.B, spec.H, spec.D, spec.D))).astype(np.float32)
    rz = _rng(spec.seed, TENSOR_IDS["z"])
    z = (scale * np.abs(rz.standard_normal((spec.B, spec.H, spec.D)))).astype(np.float32)
    return m, z


def small(B=1, H=2, F=4, S=48, D=32, dtype="bf16", seed=7, **kw) -> Spec:
    """A small ad-hoc workload (tests): same generator, any shape."""
    return Spec(f"small_B{B}_H{H}_F{F}_S{S}_D{D}_{dtype}", B=B, H=H, F=F, S=S, D=D,
                dtype=dtype, seed=seed, **kw)
