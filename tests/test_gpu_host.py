"""GPU tests of la_scan_host: the scan of host-resident buffers, streamed
through the GPU chunk by chunk with copies overlapping the scan.

Two checks per case: the host call equals, bit for bit, the device entry
point run chunk by chunk with the state carried in place (the same kernel
launches on the same data, so any difference is a plumbing error: a wrong
offset, pitch, slot or ordering); and it matches the CPU oracle's scan of the
whole clip within the parity bar.
"""
import ctypes

import numpy as np
import pytest
import torch

import linear_attention_video_frame_b200 as la
import oracle
import synth
from helpers import TOL_BF16, oracle_slice, rel_err, to_np, tol_for

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.init()


def _host_inputs(spec, pinned=True):
    dt = torch.bfloat16 if spec.dtype == "bf16" else torch.float32
    out = {}
    for name in ("q", "k", "v"):
        arr = synth.full_storage(spec, name)
        t = torch.from_numpy(arr.view(np.int16) if arr.dtype == np.uint16 else arr)
        t = t.view(dt) if spec.dtype == "bf16" else t
        out[name] = t.pin_memory() if pinned else t.clone()
    a, bt = synth.gates(spec)
    out["alpha"] = torch.from_numpy(a)
    out["beta"] = torch.from_numpy(bt)
    if pinned:
        out["alpha"], out["beta"] = out["alpha"].pin_memory(), out["beta"].pin_memory()
    return out


def _host_scan(spec, mode, inp, chunk, m0=None, z0=None, pinned=True):
    B, H, F, S, D = spec.B, spec.H, spec.F, spec.S, spec.D
    m = la.LA_MODE_RELU if mode == "relu" else la.LA_MODE_GDN
    dtc = la.LA_BF16 if spec.dtype == "bf16" else la.LA_F32
    ws = la.host_workspace_for(m, dtc, B, H, F, S, D, chunk)
    so = torch.full((B, H, D, D), float("nan")).pin_memory()
    zo = torch.full((B, H, D), float("nan")).pin_memory() if mode == "relu" else None
    o = torch.full_like(inp["q"], float("nan"))
    o = o.pin_memory() if pinned else o
    la.la_scan_host(m, inp["q"], inp["k"], inp["v"], o=o,
                    alpha=inp["alpha"] if mode == "gdn" else None,
                    beta=inp["beta"] if mode == "gdn" else None,
                    k_scale=spec.k_scale, eps=spec.eps, state_in=m0, z_in=z0,
                    state_out=so, z_out=zo, chunk_frames=chunk, workspace=ws)
    torch.cuda.current_stream().synchronize()
    assert la.la_query_device_status(ws) == la.LA_OK
    return o, so, zo


def _device_chunk_loop(spec, mode, inp, chunk, m0=None, z0=None):
    """The device entry points, one call per chunk, state carried in place."""
    B, H, F, S, D = spec.B, spec.H, spec.F, spec.S, spec.D
    n = la.la_host_chunk_frames(F, chunk)
    state = torch.zeros((B, H, D, D), device="cuda")
    z = torch.zeros((B, H, D), device="cuda")
    if m0 is not None:
        state.copy_(m0)
    if z0 is not None:
        z.copy_(z0)
    outs = []
    for c, f0 in enumerate(range(0, F, n)):
        sl = slice(f0, min(F, f0 + n))
        part = {x: inp[x][:, :, sl].contiguous().cuda() for x in ("q", "k", "v", "alpha", "beta")}
        carry = c > 0 or m0 is not None
        if mode == "gdn":
            o = la.la_scan_gdn(part["q"], part["k"], part["v"], part["alpha"], part["beta"],
                               spec.k_scale, state_in=state if carry else None, state_out=state)
        else:
            o = la.la_scan_relu(part["q"], part["k"], part["v"],
                                state_in=state if carry else None,
                                z_in=z if (c > 0 or z0 is not None) else None,
                                state_out=state, z_out=z, eps=spec.eps)
        outs.append(o)
    torch.cuda.synchronize()
    return torch.cat(outs, dim=2).cpu(), state.cpu(), z.cpu()


def _oracle_check(spec, mode, o, so, zo, m0=None, z0=None, heads=None):
    pairs = heads or [(b, h) for b in range(spec.B) for h in range(spec.H)]
    worst = 0.0
    for b, h in pairs:
        q, k, v, a, bt = oracle_slice(spec, b, h)
        rm0 = None if m0 is None else m0[b:b + 1, h:h + 1].double().numpy()
        if mode == "gdn":
            ro, rm = oracle.gdn_scan(q, k, v, a, bt, spec.k_scale, rm0)
        else:
            rz0 = None if z0 is None else z0[b:b + 1, h:h + 1].double().numpy()
            ro, rm, rz = oracle.relu_scan(q, k, v, spec.eps, rm0, rz0)
            assert rel_err(to_np(zo[b, h]), rz[0, 0]) < 1e-5
        worst = max(worst, rel_err(to_np(o[b, h]), ro[0, 0]), rel_err(to_np(so[b, h]), rm[0, 0]))
    assert worst <= tol_for(spec), f"error {worst:.3e}"
    return worst


CASES = [
    # (mode, spec, chunk_frames)
    ("gdn", dict(B=1, H=3, F=21, S=200, D=128), 4),      # ragged last chunk (1 frame)
    ("gdn", dict(B=2, H=2, F=9, S=100, D=64), 1),        # one frame per chunk
    ("gdn", dict(B=1, H=2, F=7, S=130, D=128), 0),       # automatic chunking
    ("gdn", dict(B=1, H=2, F=6, S=64, D=128), 50),       # one chunk, longer than the clip
    ("relu", dict(B=1, H=3, F=21, S=200, D=112), 5),
    ("relu", dict(B=2, H=2, F=10, S=96, D=32, dtype="f32"), 3),   # float32, SIMT path
    ("gdn", dict(B=1, H=2, F=8, S=64, D=48, dtype="f32"), 3),
]


@pytest.mark.parametrize("mode,shape,chunk", CASES)
def test_host_scan_equals_device_chunk_loop_and_oracle(mode, shape, chunk):
    spec = synth.small(keys_l2=(mode == "gdn"), **shape)
    inp = _host_inputs(spec)
    o, so, zo = _host_scan(spec, mode, inp, chunk)
    ro, rs, rz = _device_chunk_loop(spec, mode, inp, chunk)
    assert torch.equal(o.view(torch.int16) if o.dtype == torch.bfloat16 else o,
                       ro.view(torch.int16) if ro.dtype == torch.bfloat16 else ro)
    assert torch.equal(so, rs)
    if mode == "relu":
        assert torch.equal(zo, rz)
    e = _oracle_check(spec, mode, o, so, zo)
    print(f"\n[host] {spec.name} {mode} chunk={chunk}: error {e:.3e}")


@pytest.mark.parametrize("mode", ["gdn", "relu"])
def test_host_scan_with_initial_state(mode):
    spec = synth.small(B=1, H=2, F=11, S=128, D=128, keys_l2=(mode == "gdn"))
    inp = _host_inputs(spec)
    m0n, z0n = synth.random_state(spec, scale=0.05)
    m0 = torch.from_numpy(m0n).pin_memory()
    z0 = torch.from_numpy(z0n).pin_memory() if mode == "relu" else None
    o, so, zo = _host_scan(spec, mode, inp, 4, m0, z0)
    ro, rs, rz = _device_chunk_loop(spec, mode, inp, 4, m0, z0)
    assert torch.equal(o.view(torch.int16), ro.view(torch.int16))
    assert torch.equal(so, rs)
    _oracle_check(spec, mode, o, so, zo, m0, z0)


def test_host_scan_pageable_memory():
    spec = synth.small(B=1, H=2, F=9, S=96, D=128, keys_l2=True)
    pinned = _host_inputs(spec, pinned=True)
    pageable = _host_inputs(spec, pinned=False)
    assert not pageable["q"].is_pinned()
    a, sa, _ = _host_scan(spec, "gdn", pinned, 2)
    b, sb, _ = _host_scan(spec, "gdn", pageable, 2, pinned=False)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(sa, sb)


def test_host_scan_full_720p_gdn_all_heads():
    """The 720p 60 s GDN workload (B1 H20 D128 F181 S880) through the host
    path with the automatic chunking the end-to-end benchmark uses."""
    spec = synth.workload("gdn_720p_60s")
    inp = _host_inputs(spec)
    o, so, _ = _host_scan(spec, "gdn", inp, 0)
    assert la.la_host_chunk_frames(spec.F, 0) == 12
    e = _oracle_check(spec, "gdn", o, so, None, heads=[(0, h) for h in range(spec.H)])
    print(f"\n[host] {spec.name}: error {e:.3e}")


@pytest.mark.parametrize("mode", ["gdn", "relu"])
def test_host_scan_zero_frames_passes_the_state_through(mode):
    spec = synth.small(B=1, H=2, F=0, S=16, D=64)
    m0n, z0n = synth.random_state(spec)
    m0, z0 = torch.from_numpy(m0n), torch.from_numpy(z0n)
    B, H, D = 1, 2, 64
    m = la.LA_MODE_RELU if mode == "relu" else la.LA_MODE_GDN
    ws = la.host_workspace_for(m, la.LA_BF16, B, H, 0, 16, D, 0)
    q = torch.zeros((B, H, 0, 16, D), dtype=torch.bfloat16)
    g = torch.zeros((B, H, 0))
    so = torch.full((B, H, D, D), float("nan"))
    zo = torch.full((B, H, D), float("nan"))
    la.la_scan_host(m, q, q, q, o=q.clone(), alpha=g, beta=g, k_scale=0.1, state_in=m0,
                    z_in=z0 if mode == "relu" else None, state_out=so,
                    z_out=zo if mode == "relu" else None, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(so, m0)
    if mode == "relu":
        assert torch.equal(zo, z0)
    # no initial state: zeros come out
    la.la_scan_host(m, q, q, q, o=q.clone(), alpha=g, beta=g, k_scale=0.1, state_out=so,
                    workspace=ws)
    torch.cuda.synchronize()
    assert torch.count_nonzero(so) == 0


def test_host_scan_rejects_device_buffers_and_small_workspace():
    B, H, F, S, D = 1, 1, 2, 16, 64
    ws = la.host_workspace_for(la.LA_MODE_GDN, la.LA_BF16, B, H, F, S, D, 0)
    hq = torch.zeros((B, H, F, S, D), dtype=torch.bfloat16).pin_memory()
    dq = hq.cuda()
    g = torch.ones((B, H, F)).pin_memory()
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    L = la.lib
    o = torch.empty_like(hq).pin_memory()
    args = lambda q, w, n: (la.LA_MODE_GDN, P(q), P(hq), P(hq), P(o), la.LA_BF16, P(g), P(g),
                            0.1, 1e-6, None, None, None, None, B, H, F, S, D, 0, P(w), n, None)
    assert L.la_scan_host(*args(hq, ws, ws.numel())) == la.LA_OK
    assert L.la_scan_host(*args(dq, ws, ws.numel())) == la.LA_ERR_INVALID_ARG
    assert L.la_scan_host(*args(hq, ws, ws.numel() - 256)) == la.LA_ERR_INVALID_ARG
    hw = torch.empty(ws.numel(), dtype=torch.uint8).pin_memory()
    assert L.la_scan_host(*args(hq, hw, hw.numel())) == la.LA_ERR_INVALID_ARG
    # output overlapping an input
    bad = (la.LA_MODE_GDN, P(hq), P(hq), P(hq), P(hq), la.LA_BF16, P(g), P(g), 0.1, 1e-6,
           None, None, None, None, B, H, F, S, D, 0, P(ws), ws.numel(), None)
    assert L.la_scan_host(*bad) == la.LA_ERR_INVALID_ARG
    torch.cuda.synchronize()


def test_host_scan_orders_after_and_before_the_callers_stream():
    """Work queued on the stream before the call (writing the host input) is
    seen by it; work queued after it sees the host output."""
    spec = synth.small(B=1, H=2, F=6, S=128, D=128, keys_l2=True)
    inp = _host_inputs(spec)
    ref, _, _ = _host_scan(spec, "gdn", inp, 2)
    B, H, F, S, D = spec.B, spec.H, spec.F, spec.S, spec.D
    s = torch.cuda.Stream()
    ws = la.host_workspace_for(la.LA_MODE_GDN, la.LA_BF16, B, H, F, S, D, 2)
    dq = inp["q"].cuda()
    hq = torch.zeros_like(inp["q"]).pin_memory()
    o = torch.zeros_like(inp["q"]).pin_memory()
    back = torch.empty_like(inp["q"], device="cuda")
    with torch.cuda.stream(s):
        torch.cuda._sleep(20_000_000)           # keep the stream busy before the copy
        hq.copy_(dq, non_blocking=True)         # the host input is produced on the stream
        la.la_scan_host(la.LA_MODE_GDN, hq, inp["k"], inp["v"], o=o, alpha=inp["alpha"],
                        beta=inp["beta"], k_scale=spec.k_scale, chunk_frames=2, workspace=ws,
                        stream=s)
        back.copy_(o, non_blocking=True)        # consumer of the host output
    s.synchronize()
    assert torch.equal(o.view(torch.int16), ref.view(torch.int16))
    assert torch.equal(back.cpu().view(torch.int16), ref.view(torch.int16))
