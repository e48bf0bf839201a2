"""GPU parity of the scans with the fused input preparation (RMSNorm, ReLU,
3D RoPE; SANA-WM digest, method details, "Context-Parallel + Fused Triton")
against the oracle, on raw q and k of the same seeded inputs.

Bars as for the plain scans: 1e-4 for float32 inputs, 2e-2 for bfloat16
inputs (the single-kernel path rounds the prepared tiles to bf16 operands).
"""
import ctypes

import numpy as np
import pytest
import torch

import linear_attention_video_frame_b200 as la
import oracle
import synth
from helpers import TOL_BF16, device_inputs, oracle_slice, rel_err, to_np, tol_for

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _weights(spec):
    wq, wk = synth.norm_weights(spec, "q"), synth.norm_weights(spec, "k")
    return wq, wk, torch.from_numpy(wq).cuda(), torch.from_numpy(wk).cuda()


def _compare(spec, mode, rope=True, frame_offset=0, with_state=False, heads=None, path=None):
    inp = device_inputs(spec)
    wq, wk, wqd, wkd = _weights(spec)
    gh, gw = spec.grid
    prep = la.make_prep(wqd, wkd, 1e-6, rope, (gh, gw), frame_offset)
    B, H, F, S, D = spec.B, spec.H, spec.F, spec.S, spec.D
    m_mode = la.LA_MODE_GDN_PREP if mode == "gdn" else la.LA_MODE_RELU_PREP
    dt = la.LA_BF16 if spec.dtype == "bf16" else la.LA_F32
    if path is not None:
        assert la.la_plan(m_mode, dt, B, H, F, S, D)[0] == path
    m0n, z0n = synth.random_state(spec, 0.05)
    m0 = torch.from_numpy(m0n).cuda() if with_state else None
    z0 = torch.from_numpy(z0n).cuda() if with_state else None
    so = torch.full((B, H, D, D), float("nan"), device="cuda")
    ws = la.workspace_for(m_mode, B, H, F, S, D)
    if mode == "gdn":
        o = la.la_scan_gdn_prep(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                                spec.k_scale, prep, state_in=m0, state_out=so, workspace=ws)
    else:
        zo = torch.full((B, H, D), float("nan"), device="cuda")
        o = la.la_scan_relu_prep(inp["q"], inp["k"], inp["v"], prep, state_in=m0, z_in=z0,
                                 state_out=so, z_out=zo, eps=spec.eps, workspace=ws)
    st = la.la_query_device_status(ws)
    assert st == la.LA_OK, la.la_status_string(st)
    tol = tol_for(spec)
    pairs = heads or [(b, h) for b in range(B) for h in range(H)]
    num_o = den_o = num_m = den_m = 0.0
    for b, h in pairs:
        q, k, v, a, bt = oracle_slice(spec, b, h)
        sm0 = m0n[b:b + 1, h:h + 1] if with_state else None
        if mode == "gdn":
            ro, rm = oracle.gdn_scan_prep(q, k, v, a, bt, spec.k_scale, wq[h:h + 1], wk[h:h + 1],
                                          1e-6, gh, gw, frame_offset, rope=rope, state_in=sm0)
        else:
            ro, rm, rz = oracle.relu_scan_prep(q, k, v, spec.eps, wq[h:h + 1], wk[h:h + 1], 1e-6,
                                               gh, gw, frame_offset, rope=rope, state_in=sm0,
                                               z_in=z0n[b:b + 1, h:h + 1] if with_state else None)
            assert rel_err(to_np(zo[b, h]), rz[0, 0]) < 1e-4
        go, gm = to_np(o[b, h]), to_np(so[b, h])
        num_o, den_o = max(num_o, np.abs(go - ro[0, 0]).max()), max(den_o, np.abs(ro).max())
        num_m, den_m = max(num_m, np.abs(gm - rm[0, 0]).max()), max(den_m, np.abs(rm).max())
    e_o, e_m = num_o / den_o, num_m / den_m
    print(f"\n[prep] {spec.name} {mode} rope={rope}: output {e_o:.3e} state {e_m:.3e}")
    assert e_o <= tol and e_m <= tol
    return o


@pytest.mark.parametrize("mode", ["gdn", "relu"])
@pytest.mark.parametrize("dtype,D,grid,F", [
    ("f32", 32, (3, 4), 5),          # SIMT path
    ("f32", 48, (1, 17), 3),         # ragged tiles, D / 2 not a multiple of 3
    ("bf16", 64, (8, 8), 3),
    ("bf16", 128, (10, 13), 4),      # ragged token tail
    ("bf16", 112, (6, 9), 3),
    ("bf16", 256, (5, 7), 2),        # wide heads: SIMT path
])
def test_prep_scan_matches_oracle(mode, dtype, D, grid, F):
    spec = synth.small(B=2, H=2, F=F, S=grid[0] * grid[1], D=D, dtype=dtype, seed=D + F,
                       grid=grid)
    _compare(spec, mode, with_state=True, frame_offset=5)


@pytest.mark.parametrize("mode", ["gdn", "relu"])
def test_prep_scan_without_rope(mode):
    spec = synth.small(B=1, H=3, F=4, S=96, D=128, dtype="bf16", seed=81, grid=(8, 12))
    _compare(spec, mode, rope=False)


@pytest.mark.parametrize("mode", ["gdn", "relu"])
def test_prep_outputs_ignore_a_global_frame_shift(mode):
    """Both q and k of every token turn by the same extra temporal angles,
    so the outputs do not change (up to rounding)."""
    spec = synth.small(B=1, H=2, F=4, S=60, D=64, dtype="f32", seed=83, grid=(6, 10))
    o0 = _compare(spec, mode, frame_offset=0)
    o1 = _compare(spec, mode, frame_offset=400)
    torch.cuda.synchronize()
    assert rel_err(to_np(o1), to_np(o0)) < 1e-4


def test_prep_argument_errors():
    spec = synth.small(B=1, H=1, F=2, S=12, D=32, dtype="bf16", grid=(3, 4))
    inp = device_inputs(spec)
    ws = la.workspace_for(la.LA_MODE_GDN_PREP, 1, 1, 2, 12, 32)
    P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    s = torch.cuda.current_stream().cuda_stream
    o = torch.empty_like(inp["q"])

    def call(prep):
        return la.lib.la_scan_gdn_prep(P(inp["q"]), P(inp["k"]), P(inp["v"]), P(o), la.LA_BF16,
                                       P(inp["alpha"]), P(inp["beta"]), 0.1,
                                       None if prep is None else ctypes.byref(prep), None, None,
                                       1, 1, 2, 12, 32, P(ws), ws.numel(), s)

    assert call(None) == la.LA_ERR_INVALID_ARG
    assert call(la.make_prep(grid=(3, 5))) == la.LA_ERR_INVALID_ARG          # 3 x 5 != 12
    assert call(la.make_prep(grid=(3, 4), rope_base=1.0)) == la.LA_ERR_INVALID_ARG
    assert call(la.make_prep(grid=(3, 4), norm_eps=-1.0)) == la.LA_ERR_INVALID_ARG
    assert call(la.make_prep(grid=(3, 4), frame_offset=-1)) == la.LA_ERR_INVALID_ARG
    host_w = torch.ones(1, 32)
    bad = la.LaPrep(ctypes.c_void_p(host_w.data_ptr()), None, 1e-6, 1, 3, 4, 0, 1e4)
    assert call(bad) == la.LA_ERR_INVALID_ARG                                 # host weight
    assert call(la.make_prep(grid=(3, 4))) == la.LA_OK
    torch.cuda.synchronize()


def test_prep_720p_gdn_all_heads():
    """The 720p 60 s GDN workload (B1 H20 D128 F181 S880 on a 22 x 40 grid)
    on raw q and k with the preparation fused."""
    spec = synth.workload("gdn_720p_60s").with_(keys_l2=False)
    _compare(spec, "gdn")
