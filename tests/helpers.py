"""Shared helpers of the test suite: device upload of seeded inputs, error metric."""
from __future__ import annotations

import numpy as np
import torch

import synth

# Parity bars: max|gpu - ref| / max|ref| over the compared tensor.
TOL_F32 = 1e-4      # float32 inputs
TOL_BF16 = 2e-2     # bfloat16 inputs, float32 state


def tol_for(spec) -> float:
    return TOL_F32 if spec.dtype == "f32" else TOL_BF16


def to_device(arr: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    """Upload a storage array (float32, or uint16 bf16 bits) as a CUDA tensor."""
    t = torch.from_numpy(np.ascontiguousarray(arr))
    if dtype == "bf16":
        t = t.view(torch.bfloat16)
    return t.to(device)


def device_inputs(spec, device="cuda"):
    out = {}
    for name in ("q", "k", "v"):
        dt = torch.bfloat16 if spec.dtype == "bf16" else torch.float32
        t = torch.empty((spec.B, spec.H, spec.F, spec.S, spec.D), dtype=dt, device=device)

        def put(b, h, arr, t=t):
            t[b, h].copy_(to_device(arr, spec.dtype, device))

        synth.for_each_slice(spec, name, put)
        out[name] = t
    a, bt = synth.gates(spec)
    out["alpha"] = torch.from_numpy(a).to(device)
    out["beta"] = torch.from_numpy(bt).to(device)
    return out


def oracle_slice(spec, b: int, h: int):
    """float64 q, k, v of one (b, h) as [1, 1, F, S, D], and its gates [1, 1, F]."""
    q = synth.slice_values(spec, "q", b, h).astype(np.float64)[None, None]
    k = synth.slice_values(spec, "k", b, h).astype(np.float64)[None, None]
    v = synth.slice_values(spec, "v", b, h).astype(np.float64)[None, None]
    a, bt = synth.gates(spec)
    return q, k, v, a[b:b + 1, h:h + 1].astype(np.float64), bt[b:b + 1, h:h + 1].astype(np.float64)


def rel_err(got, ref) -> float:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.max(np.abs(ref))
    if den == 0:
        return float(np.max(np.abs(got)))
    return float(np.max(np.abs(got - ref)) / den)


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)
