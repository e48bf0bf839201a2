"""GPU parity of the frame-wise GDN with a per-token update gate
(la_scan_gdn_token_beta) against the CPU oracle.

Bars: 1e-4 for float32 inputs, 2e-2 for bfloat16 inputs.  bf16 heads with
64 <= D <= 128 run on the single-kernel tensor-core path (the three-kernel
path for many heads) and 128 < D <= 256 on the wide path, K and V token rows
scaled by sqrt(beta) in shared memory; the rest on the SIMT kernel.
"""
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
    torch.cuda.init()


def _run(spec, inp, btok, m0=None):
    B, H, F, S, D = spec.B, spec.H, spec.F, spec.S, spec.D
    ws = la.workspace_for(la.LA_MODE_GDN_TOKEN_BETA, B, H, F, S, D)
    so = torch.full((B, H, D, D), float("nan"), device="cuda")
    o = la.la_scan_gdn_token_beta(inp["q"], inp["k"], inp["v"], inp["alpha"], btok,
                                  spec.k_scale, state_in=m0, state_out=so, workspace=ws)
    assert la.la_query_device_status(ws) == la.LA_OK
    return o, so


def _compare(spec, heads=None, with_state=False):
    inp = device_inputs(spec)
    btn = synth.token_gates(spec)
    btok = torch.from_numpy(btn).cuda()
    m0n = m0 = None
    if with_state:
        m0n, _ = synth.random_state(spec, scale=0.05)
        m0 = torch.from_numpy(m0n).cuda()
    o, so = _run(spec, inp, btok, m0)
    torch.cuda.synchronize()
    pairs = heads or [(b, h) for b in range(spec.B) for h in range(spec.H)]
    go, ro, gm, rm = [], [], [], []
    for b, h in pairs:
        q, k, v, a, _ = oracle_slice(spec, b, h)
        r_o, r_m = oracle.gdn_scan_token_beta(
            q, k, v, a, btn[b:b + 1, h:h + 1].astype(np.float64), spec.k_scale,
            None if m0n is None else m0n[b:b + 1, h:h + 1])
        go.append(to_np(o[b, h])); ro.append(r_o[0, 0])
        gm.append(to_np(so[b, h])); rm.append(r_m[0, 0])
    e_o, e_m = rel_err(np.stack(go), np.stack(ro)), rel_err(np.stack(gm), np.stack(rm))
    print(f"\n[token-beta] {spec.name}: output {e_o:.3e} state {e_m:.3e} (bar {tol_for(spec)})")
    assert e_o <= tol_for(spec) and e_m <= tol_for(spec)


@pytest.mark.parametrize("dtype,D,S,F", [
    ("bf16", 128, 130, 5),         # tensor-core path, ragged token tail
    ("bf16", 64, 64, 3),
    ("bf16", 112, 200, 4),
    ("f32", 32, 40, 6),            # SIMT path
    ("bf16", 256, 70, 3),          # wide heads: wide tensor-core path
])
def test_token_gate_scan_matches_oracle(dtype, D, S, F):
    spec = synth.small(B=2, H=2, F=F, S=S, D=D, dtype=dtype, seed=D + S, keys_l2=True)
    _compare(spec, with_state=True)


def test_token_gate_scan_720p_gdn_all_heads():
    """The 720p 60 s GDN workload with one update gate per token."""
    spec = synth.workload("gdn_720p_60s")
    assert la.la_plan(la.LA_MODE_GDN_TOKEN_BETA, la.LA_BF16, 1, 20, 181, 880, 128) == \
        ("tcgen05_fused", 1)
    _compare(spec)


def test_token_gate_tensor_core_path_matches_simt_path(monkeypatch):
    spec = synth.small(B=1, H=3, F=6, S=333, D=128, dtype="bf16", seed=57, keys_l2=True)
    inp = device_inputs(spec)
    btok = torch.from_numpy(synth.token_gates(spec)).cuda()
    o_tc, m_tc = _run(spec, inp, btok)
    monkeypatch.setenv("LA_SCAN_FORCE_SIMT", "1")
    o_s, m_s = _run(spec, inp, btok)
    torch.cuda.synchronize()
    assert rel_err(to_np(o_tc), to_np(o_s)) <= TOL_BF16
    assert rel_err(to_np(m_tc), to_np(m_s)) <= TOL_BF16


def test_constant_token_gate_equals_frame_gate():
    spec = synth.small(B=1, H=2, F=5, S=150, D=128, dtype="bf16", seed=59, keys_l2=True)
    inp = device_inputs(spec)
    btok = inp["beta"][..., None].expand(-1, -1, -1, spec.S).contiguous()
    o_t, m_t = _run(spec, inp, btok)
    o_f = la.la_scan_gdn(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], spec.k_scale)
    torch.cuda.synchronize()
    assert rel_err(to_np(o_t), to_np(o_f)) <= TOL_BF16


def test_token_gate_fused_kernel_matches_three_kernel_path(monkeypatch):
    spec = synth.small(B=2, H=3, F=9, S=333, D=112, dtype="bf16", seed=67, keys_l2=True,
                       alpha=("sigmoid_normal", 3.0, 1.0), beta=("sigmoid_normal", 0.0, 1.0))
    assert la.la_plan(la.LA_MODE_GDN_TOKEN_BETA, la.LA_BF16, 2, 3, 9, 333, 112)[0] == \
        "tcgen05_fused"
    inp = device_inputs(spec)
    btok = torch.from_numpy(synth.token_gates(spec)).cuda()
    m0 = torch.from_numpy(synth.random_state(spec, 0.05)[0]).cuda()
    o_f, m_f = _run(spec, inp, btok, m0)
    o_f, m_f = o_f.clone(), m_f.clone()
    monkeypatch.setenv("LA_SCAN_NO_FUSE", "1")
    o_3, m_3 = _run(spec, inp, btok, m0)
    torch.cuda.synchronize()
    assert rel_err(to_np(o_f), to_np(o_3)) <= TOL_BF16
    assert rel_err(to_np(m_f), to_np(m_3)) <= TOL_BF16
    monkeypatch.delenv("LA_SCAN_NO_FUSE")
    _compare(spec, with_state=True)


def test_token_gate_wide_path_matches_oracle_across_pipeline_chunks(monkeypatch):
    """D = 256 on the wide tensor-core path, clip split into pipeline chunks."""
    spec = synth.small(B=1, H=2, F=11, S=140, D=256, dtype="bf16", seed=99, keys_l2=True)
    assert la.la_plan(la.LA_MODE_GDN_TOKEN_BETA, la.LA_BF16, 1, 2, 11, 140, 256)[0] == \
        "tcgen05_wide"
    monkeypatch.setenv("LA_WIDE_CHUNK", "4")
    _compare(spec, with_state=True)
