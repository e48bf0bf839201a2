"""Python binding of the ``la_scan`` C ABI (include/la_scan.h).

Argument marshalling only: every step of the scan runs in the CUDA kernels of
``liblavf.so``.  PyTorch supplies device memory and streams.  There is no CPU
fallback: importing this package fails if the library is missing, and every
call raises ``LaScanError`` on a non-zero status.

The functions keep the C names.  Tensors follow the C layouts:
q, k, v, o ``[B, H, F, S, D]`` (bfloat16 or float32, contiguous); alpha, beta
``[B, H, F]`` float32; state ``[B, H, D, D]`` float32 key-major; z
``[B, H, D]`` float32.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import torch

__all__ = [
    "LA_OK", "LA_ERR_INVALID_ARG", "LA_ERR_UNSUPPORTED", "LA_ERR_CUDA", "LA_ERR_TIMEOUT",
    "LA_F32", "LA_BF16", "LA_MODE_RELU", "LA_MODE_GDN", "LA_MODE_GDN_REVERSE", "LaScanError",
    "lib", "LIB_PATH", "la_scan_gdn_reverse", "la_scan_gdn_token_beta",
    "LA_MODE_GDN_TOKEN_BETA",
    "la_scan_relu", "la_scan_gdn", "la_state_step", "la_workspace_size",
    "la_query_device_status", "la_status_string", "la_plan", "workspace_for",
    "la_scan_gdn_noalloc", "la_query_noalloc_status", "LA_NOALLOC_SCRATCH_BYTES", "la_scan_host",
    "la_host_workspace_size", "la_host_chunk_frames", "host_workspace_for",
    "LA_MODE_GDN_COMPOSITE", "la_gdn_interval_composite", "la_gdn_compose_prefix",
    "LA_MODE_GDN_PREP", "LA_MODE_RELU_PREP", "LaPrep", "make_prep", "la_scan_gdn_prep",
    "la_scan_relu_prep",
]

LA_OK, LA_ERR_INVALID_ARG, LA_ERR_UNSUPPORTED, LA_ERR_CUDA, LA_ERR_TIMEOUT = 0, 1, 2, 3, 4
LA_F32, LA_BF16 = 0, 1
LA_MODE_RELU, LA_MODE_GDN, LA_MODE_GDN_REVERSE, LA_MODE_GDN_TOKEN_BETA = 0, 1, 2, 3
LA_MODE_GDN_COMPOSITE, LA_MODE_GDN_PREP, LA_MODE_RELU_PREP = 4, 5, 6
LA_NOALLOC_SCRATCH_BYTES = 64 * 1024 * 1024

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "liblavf.so")


class LaPrep(ctypes.Structure):
    """The C struct la_prep (fused input preparation of q and k)."""
    _fields_ = [("q_weight", ctypes.c_void_p), ("k_weight", ctypes.c_void_p),
                ("norm_eps", ctypes.c_float), ("rope", ctypes.c_int),
                ("grid_h", ctypes.c_int), ("grid_w", ctypes.c_int),
                ("frame_offset", ctypes.c_int), ("rope_base", ctypes.c_float)]


class LaScanError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {la_status_string(status)} ({status})")


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing; build it with "
            "`python linear_attention_video_frame_b200/build.py` (there is no fallback)")
    L = ctypes.CDLL(LIB_PATH)
    P, I, F, Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
    L.la_scan_relu.argtypes = [P, P, P, P, I, P, P, P, P, I, I, I, I, I, F, P, Z, P]
    L.la_scan_relu.restype = I
    L.la_scan_gdn.argtypes = [P, P, P, P, I, P, P, F, P, P, I, I, I, I, I, P, Z, P]
    L.la_scan_gdn.restype = I
    L.la_state_step.argtypes = [I, P, P, I, P, P, F, P, P, P, P, I, I, I, I, I, P, Z, P]
    L.la_state_step.restype = I
    L.la_workspace_size.argtypes = [I, I, I, I, I, I]
    L.la_workspace_size.restype = Z
    L.la_query_device_status.argtypes = [P, P]
    L.la_query_device_status.restype = I
    L.la_scan_gdn_token_beta.argtypes = [P, P, P, P, I, P, P, F, P, P, I, I, I, I, I, P, Z, P]
    L.la_scan_gdn_token_beta.restype = I
    L.la_scan_gdn_reverse.argtypes = [P, P, P, P, I, P, P, F, I, I, I, I, I, I, P, Z, P]
    L.la_scan_gdn_reverse.restype = I
    L.la_scan_gdn_noalloc.argtypes = [P, P, P, P, I, P, P, F, P, P, I, I, I, I, I, P]
    L.la_scan_gdn_noalloc.restype = I
    L.la_query_noalloc_status.argtypes = [P]
    L.la_query_noalloc_status.restype = I
    L.la_plan.argtypes = [I, I, I, I, I, I, I, ctypes.POINTER(ctypes.c_int)]
    L.la_plan.restype = ctypes.c_char_p
    L.la_scan_host.argtypes = [I, P, P, P, P, I, P, P, F, F, P, P, P, P,
                               I, I, I, I, I, I, P, Z, P]
    L.la_scan_host.restype = I
    L.la_host_workspace_size.argtypes = [I, I, I, I, I, I, I, I]
    L.la_host_workspace_size.restype = Z
    L.la_host_chunk_frames.argtypes = [I, I]
    L.la_host_chunk_frames.restype = I
    L.la_gdn_interval_composite.argtypes = [P, P, I, P, P, F, P, P, I, I, I, I, I, P, Z, P]
    L.la_gdn_interval_composite.restype = I
    L.la_gdn_compose_prefix.argtypes = [P, P, Z, P, P, P, I, I, I, I, P]
    L.la_gdn_compose_prefix.restype = I
    L.la_scan_gdn_prep.argtypes = [P, P, P, P, I, P, P, F, ctypes.POINTER(LaPrep), P, P,
                                   I, I, I, I, I, P, Z, P]
    L.la_scan_gdn_prep.restype = I
    L.la_scan_relu_prep.argtypes = [P, P, P, P, I, ctypes.POINTER(LaPrep), P, P, P, P,
                                    I, I, I, I, I, F, P, Z, P]
    L.la_scan_relu_prep.restype = I
    L.la_status_string.argtypes = [I]
    L.la_status_string.restype = ctypes.c_char_p
    return L


lib = _load()


def la_status_string(s: int) -> str:
    return lib.la_status_string(int(s)).decode()


def la_plan(mode: int, dt: int, B: int, H: int, F: int, S: int, D: int):
    """(path name, kernels per call) of a call of this shape; (None, 0) if unsupported."""
    n = ctypes.c_int(0)
    name = lib.la_plan(mode, dt, B, H, F, S, D, ctypes.byref(n))
    return (name.decode() if name else None), int(n.value)


def la_workspace_size(mode: int, B: int, H: int, F: int, S: int, D: int) -> int:
    return int(lib.la_workspace_size(mode, B, H, F, S, D))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return LA_BF16
    if t.dtype == torch.float32:
        return LA_F32
    raise TypeError(f"q/k/v must be bfloat16 or float32, got {t.dtype}")


def _check(t: Optional[torch.Tensor], name: str, shape=None, dtype=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")


def workspace_for(mode: int, B: int, H: int, F: int, S: int, D: int, device=None) -> torch.Tensor:
    """A caller-owned workspace tensor of the size the library asks for."""
    n = la_workspace_size(mode, B, H, F, S, D)
    if n == 0:
        raise LaScanError(LA_ERR_UNSUPPORTED, "la_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def _raise(st: int, where: str):
    if st != LA_OK:
        raise LaScanError(st, where)


def la_scan_relu(q, k, v, o=None, state_in=None, z_in=None, state_out=None, z_out=None,
                 eps: float = 1e-6, workspace=None, stream=None):
    B, H, F, S, D = k.shape
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _check(t, n, (B, H, F, S, D), k.dtype)
    for t, n in ((state_in, "state_in"), (state_out, "state_out")):
        _check(t, n, (B, H, D, D), torch.float32)
    for t, n in ((z_in, "z_in"), (z_out, "z_out")):
        _check(t, n, (B, H, D), torch.float32)
    if o is None:
        o = torch.empty_like(q)
    if workspace is None:
        workspace = workspace_for(LA_MODE_RELU, B, H, F, S, D, q.device)
    st = lib.la_scan_relu(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _dtype_code(k), _ptr(state_in),
                          _ptr(z_in), _ptr(state_out), _ptr(z_out), B, H, F, S, D, float(eps),
                          _ptr(workspace), workspace.numel(), _stream(stream))
    _raise(st, "la_scan_relu")
    return o


def la_scan_gdn(q, k, v, alpha, beta, k_scale: float, o=None, state_in=None, state_out=None,
                workspace=None, stream=None):
    B, H, F, S, D = k.shape
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _check(t, n, (B, H, F, S, D), k.dtype)
    for t, n in ((alpha, "alpha"), (beta, "beta")):
        _check(t, n, (B, H, F), torch.float32)
    for t, n in ((state_in, "state_in"), (state_out, "state_out")):
        _check(t, n, (B, H, D, D), torch.float32)
    if o is None:
        o = torch.empty_like(q)
    if workspace is None:
        workspace = workspace_for(LA_MODE_GDN, B, H, F, S, D, q.device)
    st = lib.la_scan_gdn(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _dtype_code(k), _ptr(alpha),
                         _ptr(beta), float(k_scale), _ptr(state_in), _ptr(state_out),
                         B, H, F, S, D, _ptr(workspace), workspace.numel(), _stream(stream))
    _raise(st, "la_scan_gdn")
    return o


def la_scan_gdn_reverse(q, k, v, alpha, beta, k_scale: float, chunk_frames: int, o=None,
                        workspace=None, stream=None):
    """Reversed frame-wise GDN, reset every chunk_frames frames (no state in
    or out; see include/la_scan.h)."""
    B, H, F, S, D = k.shape
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _check(t, n, (B, H, F, S, D), k.dtype)
    for t, n in ((alpha, "alpha"), (beta, "beta")):
        _check(t, n, (B, H, F), torch.float32)
    if o is None:
        o = torch.empty_like(q)
    if workspace is None:
        workspace = workspace_for(LA_MODE_GDN_REVERSE, B, H, F, S, D, q.device)
    st = lib.la_scan_gdn_reverse(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _dtype_code(k), _ptr(alpha),
                                 _ptr(beta), float(k_scale), int(chunk_frames), B, H, F, S, D,
                                 _ptr(workspace), workspace.numel(), _stream(stream))
    _raise(st, "la_scan_gdn_reverse")
    return o


def la_scan_gdn_token_beta(q, k, v, alpha, beta_token, k_scale: float, o=None, state_in=None,
                           state_out=None, workspace=None, stream=None):
    """Frame-wise GDN with a per-token update gate beta_token [B, H, F, S]
    (see include/la_scan.h)."""
    B, H, F, S, D = k.shape
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _check(t, n, (B, H, F, S, D), k.dtype)
    _check(alpha, "alpha", (B, H, F), torch.float32)
    _check(beta_token, "beta_token", (B, H, F, S), torch.float32)
    for t, n in ((state_in, "state_in"), (state_out, "state_out")):
        _check(t, n, (B, H, D, D), torch.float32)
    if o is None:
        o = torch.empty_like(q)
    if workspace is None:
        workspace = workspace_for(LA_MODE_GDN_TOKEN_BETA, B, H, F, S, D, q.device)
    st = lib.la_scan_gdn_token_beta(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _dtype_code(k),
                                    _ptr(alpha), _ptr(beta_token), float(k_scale),
                                    _ptr(state_in), _ptr(state_out), B, H, F, S, D,
                                    _ptr(workspace), workspace.numel(), _stream(stream))
    _raise(st, "la_scan_gdn_token_beta")
    return o


def la_scan_gdn_noalloc(q, k, v, alpha, beta, k_scale: float, o=None, state_in=None,
                        state_out=None, stream=None):
    """la_scan_gdn without a workspace: the library's built-in scratch is used
    (for callers that cannot allocate; see include/la_scan.h)."""
    B, H, F, S, D = k.shape
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _check(t, n, (B, H, F, S, D), k.dtype)
    for t, n in ((alpha, "alpha"), (beta, "beta")):
        _check(t, n, (B, H, F), torch.float32)
    for t, n in ((state_in, "state_in"), (state_out, "state_out")):
        _check(t, n, (B, H, D, D), torch.float32)
    if o is None:
        o = torch.empty_like(q)
    st = lib.la_scan_gdn_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _dtype_code(k), _ptr(alpha),
                                 _ptr(beta), float(k_scale), _ptr(state_in), _ptr(state_out),
                                 B, H, F, S, D, _stream(stream))
    _raise(st, "la_scan_gdn_noalloc")
    return o


def la_gdn_interval_composite(k, v, alpha, beta, k_scale: float, out=None, workspace=None,
                              stream=None):
    """Transition and input composites of this frame interval, written to
    out[0] (A_F ... A_1) and out[1] (the state from zero): out is
    [2, B, H, D, D] float32 and is returned."""
    B, H, F, S, D = k.shape
    _check(k, "k", (B, H, F, S, D))
    _check(v, "v", (B, H, F, S, D), k.dtype)
    for t, n in ((alpha, "alpha"), (beta, "beta")):
        _check(t, n, (B, H, F), torch.float32)
    if out is None:
        out = torch.empty((2, B, H, D, D), dtype=torch.float32, device=k.device)
    _check(out, "out", (2, B, H, D, D), torch.float32)
    if workspace is None:
        workspace = workspace_for(LA_MODE_GDN_COMPOSITE, B, H, F, S, D, k.device)
    st = lib.la_gdn_interval_composite(_ptr(k), _ptr(v), _dtype_code(k), _ptr(alpha), _ptr(beta),
                                       float(k_scale), _ptr(out[0]), _ptr(out[1]), B, H, F, S, D,
                                       _ptr(workspace), workspace.numel(), _stream(stream))
    _raise(st, "la_gdn_interval_composite")
    return out


def la_gdn_compose_prefix(composites, state_in=None, starts=None, state_out=None, stream=None):
    """Exclusive prefix over interval composites.  composites: [n, 2, B, H, D, D]
    float32 (T_r, U_r of interval r, as la_gdn_interval_composite writes them
    and as an all-gather stacks them).  Returns starts [n, B, H, D, D], the
    initial state of every interval; state_out (if given) gets the state
    after all n intervals."""
    n, two, B, H, D, D2 = composites.shape
    if two != 2 or D2 != D:
        raise ValueError(f"composites must be [n, 2, B, H, D, D], got {tuple(composites.shape)}")
    _check(composites, "composites", None, torch.float32)
    _check(state_in, "state_in", (B, H, D, D), torch.float32)
    _check(state_out, "state_out", (B, H, D, D), torch.float32)
    if starts is None:
        starts = torch.empty((n, B, H, D, D), dtype=torch.float32, device=composites.device)
    _check(starts, "starts", (n, B, H, D, D), torch.float32)
    one = B * H * D * D
    st = lib.la_gdn_compose_prefix(_ptr(composites), _ptr(composites[0, 1]), 2 * one,
                                   _ptr(state_in), _ptr(starts), _ptr(state_out), n, B, H, D,
                                   _stream(stream))
    _raise(st, "la_gdn_compose_prefix")
    return starts


def make_prep(q_weight=None, k_weight=None, norm_eps: float = 1e-6, rope: bool = True,
              grid=(1, 1), frame_offset: int = 0, rope_base: float = 10000.0) -> LaPrep:
    """An la_prep struct; q_weight / k_weight are [H, D] float32 CUDA tensors or None.
    The struct holds raw pointers: keep the weight tensors alive while it is used."""
    for t, n in ((q_weight, "q_weight"), (k_weight, "k_weight")):
        _check(t, n, None, torch.float32)
    return LaPrep(_ptr(q_weight), _ptr(k_weight), float(norm_eps), int(bool(rope)),
                  int(grid[0]), int(grid[1]), int(frame_offset), float(rope_base))


def la_scan_gdn_prep(q, k, v, alpha, beta, k_scale: float, prep: LaPrep, o=None, state_in=None,
                     state_out=None, workspace=None, stream=None):
    """la_scan_gdn on raw q, k with RMSNorm, ReLU and 3D RoPE fused (see la_prep)."""
    B, H, F, S, D = k.shape
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _check(t, n, (B, H, F, S, D), k.dtype)
    for t, n in ((alpha, "alpha"), (beta, "beta")):
        _check(t, n, (B, H, F), torch.float32)
    for t, n in ((state_in, "state_in"), (state_out, "state_out")):
        _check(t, n, (B, H, D, D), torch.float32)
    if o is None:
        o = torch.empty_like(q)
    if workspace is None:
        workspace = workspace_for(LA_MODE_GDN_PREP, B, H, F, S, D, q.device)
    st = lib.la_scan_gdn_prep(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _dtype_code(k), _ptr(alpha),
                              _ptr(beta), float(k_scale), ctypes.byref(prep), _ptr(state_in),
                              _ptr(state_out), B, H, F, S, D, _ptr(workspace), workspace.numel(),
                              _stream(stream))
    _raise(st, "la_scan_gdn_prep")
    return o


def la_scan_relu_prep(q, k, v, prep: LaPrep, o=None, state_in=None, z_in=None, state_out=None,
                      z_out=None, eps: float = 1e-6, workspace=None, stream=None):
    """la_scan_relu on raw q, k with RMSNorm, ReLU and (numerator) 3D RoPE fused."""
    B, H, F, S, D = k.shape
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _check(t, n, (B, H, F, S, D), k.dtype)
    for t, n in ((state_in, "state_in"), (state_out, "state_out")):
        _check(t, n, (B, H, D, D), torch.float32)
    for t, n in ((z_in, "z_in"), (z_out, "z_out")):
        _check(t, n, (B, H, D), torch.float32)
    if o is None:
        o = torch.empty_like(q)
    if workspace is None:
        workspace = workspace_for(LA_MODE_RELU_PREP, B, H, F, S, D, q.device)
    st = lib.la_scan_relu_prep(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _dtype_code(k),
                               ctypes.byref(prep), _ptr(state_in), _ptr(z_in), _ptr(state_out),
                               _ptr(z_out), B, H, F, S, D, float(eps), _ptr(workspace),
                               workspace.numel(), _stream(stream))
    _raise(st, "la_scan_relu_prep")
    return o


def la_state_step(mode: int, k, v, alpha=None, beta=None, k_scale: float = 1.0,
                  state_in=None, z_in=None, state_out=None, z_out=None, workspace=None,
                  stream=None):
    B, H, F, S, D = k.shape
    _check(k, "k", (B, H, F, S, D))
    _check(v, "v", (B, H, F, S, D), k.dtype)
    for t, n in ((alpha, "alpha"), (beta, "beta")):
        _check(t, n, (B, H, F), torch.float32)
    for t, n in ((state_in, "state_in"), (state_out, "state_out")):
        _check(t, n, (B, H, D, D), torch.float32)
    for t, n in ((z_in, "z_in"), (z_out, "z_out")):
        _check(t, n, (B, H, D), torch.float32)
    if workspace is None:
        workspace = workspace_for(mode, B, H, F, S, D, k.device)
    st = lib.la_state_step(int(mode), _ptr(k), _ptr(v), _dtype_code(k), _ptr(alpha), _ptr(beta),
                           float(k_scale), _ptr(state_in), _ptr(z_in), _ptr(state_out),
                           _ptr(z_out), B, H, F, S, D, _ptr(workspace), workspace.numel(),
                           _stream(stream))
    _raise(st, "la_state_step")


def la_query_device_status(workspace, stream=None) -> int:
    return int(lib.la_query_device_status(_ptr(workspace), _stream(stream)))


def la_query_noalloc_status(stream=None) -> int:
    """Status the last la_scan_gdn_noalloc call on the current device recorded."""
    return int(lib.la_query_noalloc_status(_stream(stream)))


def la_host_workspace_size(mode: int, dt: int, B: int, H: int, F: int, S: int, D: int,
                           chunk_frames: int = 0) -> int:
    return int(lib.la_host_workspace_size(mode, dt, B, H, F, S, D, int(chunk_frames)))


def la_host_chunk_frames(F: int, chunk_frames: int = 0) -> int:
    return int(lib.la_host_chunk_frames(int(F), int(chunk_frames)))


def host_workspace_for(mode: int, dt: int, B: int, H: int, F: int, S: int, D: int,
                       chunk_frames: int = 0, device=None) -> torch.Tensor:
    """Device workspace of the size la_scan_host asks for."""
    n = la_host_workspace_size(mode, dt, B, H, F, S, D, chunk_frames)
    if n == 0:
        raise LaScanError(LA_ERR_UNSUPPORTED, "la_host_workspace_size")
    return torch.empty(n, dtype=torch.uint8, device=device or "cuda")


def _check_host(t: Optional[torch.Tensor], name: str, shape=None, dtype=None):
    if t is None:
        return
    if t.is_cuda:
        raise ValueError(f"{name} must be a host (CPU) tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} has dtype {t.dtype}, expected {dtype}")


def la_scan_host(mode: int, q, k, v, o=None, alpha=None, beta=None, k_scale: float = 1.0,
                 eps: float = 1e-6, state_in=None, z_in=None, state_out=None, z_out=None,
                 chunk_frames: int = 0, workspace=None, stream=None):
    """The scan of host-resident q, k, v into host o, streamed through the GPU
    chunk by chunk (pinned tensors let the copies overlap the scan).  The call
    is asynchronous on `stream`: synchronise it before reading o."""
    B, H, F, S, D = k.shape
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (o, "o")):
        _check_host(t, n, (B, H, F, S, D), k.dtype)
    for t, n in ((alpha, "alpha"), (beta, "beta")):
        _check_host(t, n, (B, H, F), torch.float32)
    for t, n in ((state_in, "state_in"), (state_out, "state_out")):
        _check_host(t, n, (B, H, D, D), torch.float32)
    for t, n in ((z_in, "z_in"), (z_out, "z_out")):
        _check_host(t, n, (B, H, D), torch.float32)
    if workspace is None:
        raise ValueError("la_scan_host needs a device workspace (see host_workspace_for)")
    if not workspace.is_cuda:
        raise ValueError("the workspace must be a CUDA tensor")
    if o is None:
        o = torch.empty_like(q, pin_memory=q.is_pinned())
    st = lib.la_scan_host(int(mode), _ptr(q), _ptr(k), _ptr(v), _ptr(o), _dtype_code(k),
                          _ptr(alpha), _ptr(beta), float(k_scale), float(eps), _ptr(state_in),
                          _ptr(z_in), _ptr(state_out), _ptr(z_out), B, H, F, S, D,
                          int(chunk_frames), _ptr(workspace), workspace.numel(), _stream(stream))
    _raise(st, "la_scan_host")
    return o
