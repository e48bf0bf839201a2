"""GPU parity: the CUDA scan (through the C ABI) against the CPU oracle.

Bars (max|gpu - ref| / max|ref| over the compared tensor): 1e-4 for float32
inputs, 2e-2 for bfloat16 inputs with a float32 state.  Small cases are
compared element by element in full; the full-size workloads in the launch
configuration the benchmark times are compared on every head.
"""
import ctypes

import numpy as np
import pytest
import torch

import linear_attention_video_frame_b200 as la
import oracle
import synth
from helpers import (TOL_BF16, TOL_F32, device_inputs, oracle_slice, rel_err, to_device,
                     to_np, tol_for)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.init()


def _check_status(ws):
    st = la.la_query_device_status(ws)
    where = int(ws[4:8].view(torch.int32).item())
    assert st == la.LA_OK, f"device status {la.la_status_string(st)} at wait 0x{where:x}"


def _run(spec, mode, inp, state_in=None, z_in=None, want_state=True):
    B, H, F, S, D = spec.B, spec.H, spec.F, spec.S, spec.D
    so = torch.full((B, H, D, D), float("nan"), device="cuda") if want_state else None
    m = la.LA_MODE_RELU if mode == "relu" else la.LA_MODE_GDN
    ws = la.workspace_for(m, B, H, F, S, D)
    if mode == "relu":
        zo = torch.full((B, H, D), float("nan"), device="cuda") if want_state else None
        o = la.la_scan_relu(inp["q"], inp["k"], inp["v"], state_in=state_in, z_in=z_in,
                            state_out=so, z_out=zo, eps=spec.eps, workspace=ws)
        _check_status(ws)
        return o, so, zo
    o = la.la_scan_gdn(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], spec.k_scale,
                       state_in=state_in, state_out=so, workspace=ws)
    _check_status(ws)
    return o, so, None


def _oracle(spec, mode, b, h, m0=None, z0=None):
    q, k, v, a, bt = oracle_slice(spec, b, h)
    if mode == "relu":
        o, m, z = oracle.relu_scan(q, k, v, spec.eps, m0, z0)
        return o[0, 0], m[0, 0], z[0, 0]
    o, m = oracle.gdn_scan(q, k, v, a, bt, spec.k_scale, m0)
    return o[0, 0], m[0, 0], None


class _MaxRel:
    """max|got - ref| / max|ref| over several slices, accumulated slice by slice
    (a full-size head is about 1 GB in float64, so heads are not stacked)."""

    def __init__(self):
        self.num = 0.0
        self.den = 0.0

    def add(self, got, ref):
        got = np.asarray(got, dtype=np.float64)
        ref = np.asarray(ref, dtype=np.float64)
        self.num = max(self.num, float(np.max(np.abs(got - ref))))
        self.den = max(self.den, float(np.max(np.abs(ref))))

    @property
    def value(self) -> float:
        return self.num / self.den if self.den > 0 else self.num


def _compare(spec, mode, heads=None, with_state=False, inp=None, tol=None):
    inp = device_inputs(spec) if inp is None else inp
    m0 = z0 = None
    if with_state:
        m0n, z0n = synth.random_state(spec, scale=0.05)
        m0, z0 = torch.from_numpy(m0n).cuda(), torch.from_numpy(z0n).cuda()
    o, so, zo = _run(spec, mode, inp, m0, z0 if mode == "relu" else None)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all()
    tol = tol_for(spec) if tol is None else tol
    pairs = heads if heads is not None else [(b, h) for b in range(spec.B) for h in range(spec.H)]
    e_o, e_m = _MaxRel(), _MaxRel()
    for b, h in pairs:
        rm0 = None if m0 is None else m0n[b:b + 1, h:h + 1]
        rz0 = None if z0 is None else z0n[b:b + 1, h:h + 1]
        ro, rm, rz = _oracle(spec, mode, b, h, rm0, rz0)
        e_o.add(to_np(o[b, h]), ro)
        e_m.add(to_np(so[b, h]), rm)
        if rz is not None:
            assert rel_err(to_np(zo[b, h]), rz) < 1e-5
        del ro, rm
    print(f"\n[parity] {spec.name} {mode} ({len(pairs)} heads): output {e_o.value:.3e} "
          f"state {e_m.value:.3e} (bar {tol})")
    assert e_o.value <= tol, f"output error {e_o.value:.3e} > {tol}"
    assert e_m.value <= tol, f"state error {e_m.value:.3e} > {tol}"
    return e_o.value, e_m.value


# ----------------------------------------------------------------------------
# The five workloads
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("mode", ["relu", "gdn"])
def test_tiny_fp32_config(mode):
    _compare(synth.workload("tiny_fp32"), mode)


@pytest.mark.parametrize("mode", ["relu", "gdn"])
def test_tiny_fp32_config_with_state_in(mode):
    _compare(synth.workload("tiny_fp32"), mode, with_state=True)


def test_relu_480p_all_heads():
    _compare(synth.workload("relu_480p"), "relu")


def test_gdn_720p_60s_all_heads():
    _compare(synth.workload("gdn_720p_60s"), "gdn")


@pytest.mark.parametrize("mode", ["relu", "gdn"])
def test_stress_d256_all_heads(mode):
    # all 16 heads, element by element: the outlier tokens are shared by every head
    _compare(synth.workload("stress_d256"), mode)


def test_fused_relu_on_a_60s_clip():
    """The single-kernel path adds each frame's increment phi(K)^T V to the
    fp32 state as a bf16 operand; ReLU has no decay, so over 181 frames the
    rounding of the increments would compound if it were biased."""
    spec = synth.workload("gdn_720p_60s").with_(name="relu_720p_60s_B1_H20_D128_F181_S880",
                                                keys_l2=False, modes=("relu",))
    assert la.la_plan(la.LA_MODE_RELU, la.LA_BF16, 1, 20, 181, 880, 128) == ("tcgen05_fused", 1)
    _compare(spec, "relu")


def test_fused_gdn_near_additive_on_a_60s_clip():
    """alpha = 1 and small beta: the GDN state is nearly a plain sum of the
    bf16-rounded increments beta kappa K^T V over all 181 frames."""
    spec = synth.workload("gdn_720p_60s").with_(name="gdn_720p_60s_alpha1_beta0.05",
                                                alpha=("const", 1.0),
                                                beta=("uniform", 0.0, 0.05))
    assert la.la_plan(la.LA_MODE_GDN, la.LA_BF16, 1, 20, 181, 880, 128) == ("tcgen05_fused", 1)
    _compare(spec, "gdn")


def test_streaming_chunks_equal_single_scan():
    spec = synth.workload("gdn_stream")
    inp = device_inputs(spec)
    B, H, F, D, C = spec.B, spec.H, spec.F, spec.D, spec.chunk_frames
    whole, m_whole, _ = _run(spec, "gdn", inp)
    state = torch.empty((B, H, D, D), device="cuda")
    outs = []
    for c in range(F // C):
        sl = slice(c * C, (c + 1) * C)
        part = {n: inp[n][:, :, sl].contiguous() for n in ("q", "k", "v", "alpha", "beta")}
        o = la.la_scan_gdn(part["q"], part["k"], part["v"], part["alpha"], part["beta"],
                           spec.k_scale, state_in=state if c else None, state_out=state)
        outs.append(o)
    chunked = torch.cat(outs, dim=2)
    torch.cuda.synchronize()
    # chunked == single scan up to float32 summation order
    assert rel_err(to_np(chunked), to_np(whole)) < 1e-2
    assert rel_err(to_np(state), to_np(m_whole)) < 1e-3
    # and both match the oracle's single 64-frame scan on every (b, h)
    e_o, e_m = _MaxRel(), _MaxRel()
    for b in range(B):
        for h in range(H):
            ro, rm, _ = _oracle(spec, "gdn", b, h)
            e_o.add(to_np(chunked[b, h]), ro)
            e_m.add(to_np(state[b, h]), rm)
    print(f"\n[parity] {spec.name} chunked, {B * H} heads: output {e_o.value:.3e} "
          f"state {e_m.value:.3e}")
    assert e_o.value <= TOL_BF16 and e_m.value <= TOL_BF16


# ----------------------------------------------------------------------------
# Edge cases: ragged token tails, odd head dims, one token, in-place state
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("mode", ["relu", "gdn"])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("D,S,F", [(16, 1, 3), (48, 17, 2), (64, 130, 3), (80, 64, 2),
                                   (96, 300, 2), (112, 200, 2), (128, 129, 3), (128, 1, 4),
                                   (144, 100, 3), (192, 257, 2), (240, 1, 2), (256, 70, 2)])
def test_small_shapes(mode, dtype, D, S, F):
    spec = synth.small(B=2, H=2, F=F, S=S, D=D, dtype=dtype, seed=D + S)
    _compare(spec, mode, with_state=True)


@pytest.mark.parametrize("mode", ["relu", "gdn"])
def test_zero_frames_copies_state(mode):
    spec = synth.small(B=1, H=3, F=0, S=8, D=32, dtype="bf16")
    m0n, z0n = synth.random_state(spec)
    m0, z0 = torch.from_numpy(m0n).cuda(), torch.from_numpy(z0n).cuda()
    inp = device_inputs(spec)
    o, so, zo = _run(spec, mode, inp, m0, z0 if mode == "relu" else None)
    torch.cuda.synchronize()
    assert torch.equal(so, m0)
    if mode == "relu":
        assert torch.equal(zo, z0)
    # NULL state_in: zeros
    o, so, zo = _run(spec, mode, inp)
    torch.cuda.synchronize()
    assert torch.count_nonzero(so) == 0


@pytest.mark.parametrize("mode", ["relu", "gdn"])
@pytest.mark.parametrize("D", [64, 192])
def test_in_place_state(mode, D):
    spec = synth.small(B=1, H=2, F=3, S=40, D=D, dtype="bf16", seed=9)
    inp = device_inputs(spec)
    m0n, z0n = synth.random_state(spec, 0.1)
    m, z = torch.from_numpy(m0n).cuda(), torch.from_numpy(z0n).cuda()
    if mode == "relu":
        la.la_scan_relu(inp["q"], inp["k"], inp["v"], state_in=m, z_in=z, state_out=m, z_out=z)
    else:
        la.la_scan_gdn(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], spec.k_scale,
                       state_in=m, state_out=m)
    torch.cuda.synchronize()
    for h in range(2):
        _, rm, rz = _oracle(spec, mode, 0, h, m0n[:, h:h + 1], z0n[:, h:h + 1])
        assert rel_err(to_np(m[0, h]), rm) <= TOL_BF16
        if mode == "relu":
            assert rel_err(to_np(z[0, h]), rz) <= 1e-5


@pytest.mark.parametrize("mode", ["relu", "gdn"])
@pytest.mark.parametrize("D", [128, 256])
def test_state_step_matches_oracle(mode, D):
    spec = synth.small(B=2, H=2, F=4, S=100, D=D, dtype="bf16", seed=21, keys_l2=True)
    inp = device_inputs(spec)
    m0n, z0n = synth.random_state(spec, 0.05)
    m0, z0 = torch.from_numpy(m0n).cuda(), torch.from_numpy(z0n).cuda()
    so = torch.empty_like(m0)
    zo = torch.empty_like(z0)
    mode_c = la.LA_MODE_RELU if mode == "relu" else la.LA_MODE_GDN
    la.la_state_step(mode_c, inp["k"], inp["v"], inp["alpha"], inp["beta"], spec.k_scale,
                     state_in=m0, z_in=z0, state_out=so, z_out=zo)
    torch.cuda.synchronize()
    for b in range(2):
        for h in range(2):
            _, k, v, a, bt = oracle_slice(spec, b, h)
            if mode == "relu":
                rm, rz = oracle.relu_state_step(k, v, m0n[b:b + 1, h:h + 1], z0n[b:b + 1, h:h + 1])
                assert rel_err(to_np(zo[b, h]), rz[0, 0]) < 1e-5
            else:
                rm = oracle.gdn_state_step(k, v, a, bt, spec.k_scale, m0n[b:b + 1, h:h + 1])
            assert rel_err(to_np(so[b, h]), rm[0, 0]) <= TOL_BF16


@pytest.mark.parametrize("D", [48, 144])
def test_outputs_do_not_write_outside_their_buffers(D):
    spec = synth.small(B=1, H=2, F=2, S=77, D=D, dtype="bf16", seed=5)
    inp = device_inputs(spec)
    n = spec.B * spec.H * spec.F * spec.S * spec.D
    guard = 4096
    buf = torch.full((n + 2 * guard,), 7.0, dtype=torch.bfloat16, device="cuda")
    o = buf[guard:guard + n].view(spec.B, spec.H, spec.F, spec.S, spec.D)
    sbuf = torch.full((spec.H * spec.D * spec.D + 2 * guard,), 3.0, device="cuda")
    so = sbuf[guard:guard + spec.H * spec.D * spec.D].view(1, spec.H, spec.D, spec.D)
    la.la_scan_gdn(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], spec.k_scale,
                   o=o, state_out=so)
    la.la_scan_relu(inp["q"], inp["k"], inp["v"], o=o, state_out=so)
    torch.cuda.synchronize()
    assert torch.all(buf[:guard] == 7.0) and torch.all(buf[guard + n:] == 7.0)
    assert torch.all(sbuf[:guard] == 3.0) and torch.all(sbuf[-guard:] == 3.0)


# ----------------------------------------------------------------------------
# Argument errors that need a device to detect
# ----------------------------------------------------------------------------
def test_rejects_host_and_overlapping_pointers():
    spec = synth.small(B=1, H=1, F=2, S=16, D=32, dtype="bf16")
    inp = device_inputs(spec)
    ws = la.workspace_for(la.LA_MODE_GDN, 1, 1, 2, 16, 32)
    host = torch.zeros(1, 1, 2, 16, 32, dtype=torch.bfloat16).pin_memory()
    P = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    L = la.lib
    s = torch.cuda.current_stream().cuda_stream
    # unregistered host memory
    h = np.zeros(2 * 16 * 32, dtype=np.uint16)
    st = L.la_scan_gdn(P(inp["q"]), P(inp["k"]), P(inp["v"]), h.ctypes.data, la.LA_BF16,
                       P(inp["alpha"]), P(inp["beta"]), 0.1, None, None, 1, 1, 2, 16, 32,
                       P(ws), ws.numel(), s)
    assert st == la.LA_ERR_INVALID_ARG
    # output overlapping an input
    st = L.la_scan_gdn(P(inp["q"]), P(inp["k"]), P(inp["v"]), P(inp["q"]), la.LA_BF16,
                       P(inp["alpha"]), P(inp["beta"]), 0.1, None, None, 1, 1, 2, 16, 32,
                       P(ws), ws.numel(), s)
    assert st == la.LA_ERR_INVALID_ARG
    # misaligned pointer
    o = torch.empty(2 * 16 * 32 + 8, dtype=torch.bfloat16, device="cuda")
    st = L.la_scan_gdn(P(inp["q"]), P(inp["k"]), P(inp["v"]), o.data_ptr() + 2, la.LA_BF16,
                       P(inp["alpha"]), P(inp["beta"]), 0.1, None, None, 1, 1, 2, 16, 32,
                       P(ws), ws.numel(), s)
    assert st == la.LA_ERR_INVALID_ARG
    # a rejected call enqueues nothing; a valid call afterwards records LA_OK
    la.la_scan_gdn(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], 0.1, workspace=ws)
    assert la.la_query_device_status(ws) == la.LA_OK
    del host


# ----------------------------------------------------------------------------
# Both kernel paths agree (tensor-core path vs the float32 SIMT path)
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("mode", ["relu", "gdn"])
def test_tensor_core_path_matches_simt_path(mode, monkeypatch):
    spec = synth.small(B=1, H=3, F=5, S=333, D=128, dtype="bf16", seed=31, keys_l2=True)
    assert la.la_plan(la.LA_MODE_GDN if mode == "gdn" else la.LA_MODE_RELU, la.LA_BF16,
                      1, 3, 5, 333, 128)[0].startswith("tcgen05")
    inp = device_inputs(spec)
    o_tc, m_tc, _ = _run(spec, mode, inp)
    monkeypatch.setenv("LA_SCAN_FORCE_SIMT", "1")
    o_simt, m_simt, _ = _run(spec, mode, inp)
    torch.cuda.synchronize()
    assert rel_err(to_np(o_tc), to_np(o_simt)) <= TOL_BF16
    assert rel_err(to_np(m_tc), to_np(m_simt)) <= TOL_BF16


@pytest.mark.parametrize("mode", ["relu", "gdn"])
@pytest.mark.parametrize("D", [192, 256])
def test_wide_tensor_core_path_matches_simt_path(mode, D, monkeypatch):
    spec = synth.small(B=1, H=3, F=6, S=300, D=D, dtype="bf16", seed=41, keys_l2=True)
    m = la.LA_MODE_GDN if mode == "gdn" else la.LA_MODE_RELU
    assert la.la_plan(m, la.LA_BF16, 1, 3, 6, 300, D)[0] == "tcgen05_wide"
    inp = device_inputs(spec)
    o_tc, m_tc, _ = _run(spec, mode, inp)
    monkeypatch.setenv("LA_SCAN_FORCE_SIMT", "1")
    o_simt, m_simt, _ = _run(spec, mode, inp)
    torch.cuda.synchronize()
    assert rel_err(to_np(o_tc), to_np(o_simt)) <= TOL_BF16
    assert rel_err(to_np(m_tc), to_np(m_simt)) <= TOL_BF16


@pytest.mark.parametrize("mode", ["relu", "gdn", "gdn_token_beta"])
@pytest.mark.parametrize("D", [144, 192, 256])
def test_wide_gram_on_cta_pairs_matches_one_cta_kernel(mode, D, monkeypatch):
    """With LA_WIDE_PAIR=1 the wide gram runs on CTA pairs (M = 256 MMAs, each
    CTA holding its 128 key columns of K and V); the default one-CTA-per-key-row-
    block kernel computes the same products with M = 128 MMAs over whole tiles.  Both sum the same
    16-token slices in the same order into fp32, so they agree to rounding, and
    both match the oracle (ragged last token tile, key columns past D padded)."""
    spec = synth.small(B=2, H=2, F=7, S=200, D=D, dtype="bf16", seed=47, keys_l2=True,
                       alpha=("sigmoid_normal", 3.0, 1.0), beta=("sigmoid_normal", 0.0, 1.0))
    inp = device_inputs(spec)
    B, H, F, S = spec.B, spec.H, spec.F, spec.S
    m0n, z0n = synth.random_state(spec, 0.05)
    m0, z0 = torch.from_numpy(m0n).cuda(), torch.from_numpy(z0n).cuda()
    if mode == "gdn_token_beta":
        gates = torch.from_numpy(synth.token_gates(spec)).cuda()
        assert la.la_plan(la.LA_MODE_GDN_TOKEN_BETA, la.LA_BF16, B, H, F, S, D)[0] == "tcgen05_wide"

        def run():
            so = torch.empty((B, H, D, D), device="cuda")
            ws = la.workspace_for(la.LA_MODE_GDN_TOKEN_BETA, B, H, F, S, D)
            o = la.la_scan_gdn_token_beta(inp["q"], inp["k"], inp["v"], inp["alpha"], gates,
                                          spec.k_scale, state_in=m0, state_out=so, workspace=ws)
            _check_status(ws)
            return o, so, None
    else:
        m = la.LA_MODE_GDN if mode == "gdn" else la.LA_MODE_RELU
        assert la.la_plan(m, la.LA_BF16, B, H, F, S, D)[0] == "tcgen05_wide"

        def run():
            return _run(spec, mode, inp, m0, z0 if mode == "relu" else None)
    monkeypatch.setenv("LA_WIDE_PAIR", "1")
    o_p, m_p, z_p = run()
    monkeypatch.delenv("LA_WIDE_PAIR")
    o_1, m_1, z_1 = run()
    torch.cuda.synchronize()
    assert torch.isfinite(o_p.float()).all() and torch.isfinite(m_p).all()
    e_o = rel_err(to_np(o_p), to_np(o_1))
    e_m = rel_err(to_np(m_p), to_np(m_1))
    print(f"\n[pair vs one-CTA gram] {mode} D={D}: output {e_o:.3e} state {e_m:.3e}")
    assert e_o <= 1e-2 * TOL_BF16 and e_m <= 1e-2 * TOL_BF16
    if mode == "relu":
        assert rel_err(to_np(z_p), to_np(z_1)) < 1e-6
    if mode != "gdn_token_beta":
        _compare(spec, mode, with_state=True)


@pytest.mark.parametrize("mode", ["relu", "gdn"])
def test_wide_path_chunking_is_exact(mode, monkeypatch):
    """The wide path pipelines frame chunks and carries the fp32 state between
    them, so the chunk length changes nothing: every chunking gives the same
    bits, and matches the oracle (ragged last chunk, initial state)."""
    spec = synth.small(B=1, H=2, F=21, S=64, D=256, dtype="bf16", seed=43, keys_l2=True)
    inp = device_inputs(spec)
    m0n, z0n = synth.random_state(spec, 0.05)
    m0, z0 = torch.from_numpy(m0n).cuda(), torch.from_numpy(z0n).cuda()
    runs = []
    for chunk in ("1", "5", "21"):
        monkeypatch.setenv("LA_WIDE_CHUNK", chunk)
        runs.append(_run(spec, mode, inp, m0, z0 if mode == "relu" else None))
    torch.cuda.synchronize()
    for o, so, zo in runs[1:]:
        assert torch.equal(o.view(torch.int16), runs[0][0].view(torch.int16))
        assert torch.equal(so, runs[0][1])
        if mode == "relu":
            assert torch.equal(zo, runs[0][2])
    monkeypatch.delenv("LA_WIDE_CHUNK")
    _compare(spec, mode, with_state=True)


@pytest.mark.parametrize("mode", ["relu", "gdn"])
def test_three_kernel_chunk_pipeline_is_exact(mode, monkeypatch):
    """Long clips on the three-kernel path run as a pipeline of frame chunks
    (chain beside gram and output, fp32 state carried between chunk
    launches): any chunk length gives the same bits, and the oracle's values."""
    spec = synth.small(B=1, H=3, F=40, S=96, D=128, dtype="bf16", seed=71, keys_l2=True)
    monkeypatch.setenv("LA_SCAN_NO_FUSE", "1")
    m = la.LA_MODE_GDN if mode == "gdn" else la.LA_MODE_RELU
    assert la.la_plan(m, la.LA_BF16, 1, 3, 40, 96, 128) == ("tcgen05", 9)   # 3 chunks
    inp = device_inputs(spec)
    m0n, z0n = synth.random_state(spec, 0.05)
    m0, z0 = torch.from_numpy(m0n).cuda(), torch.from_numpy(z0n).cuda()
    runs = []
    for chunk in ("7", "16", "40"):
        monkeypatch.setenv("LA_TC_CHUNK", chunk)
        runs.append(_run(spec, mode, inp, m0, z0 if mode == "relu" else None))
    torch.cuda.synchronize()
    for o, so, zo in runs[1:]:
        assert torch.equal(o.view(torch.int16), runs[0][0].view(torch.int16))
        assert torch.equal(so, runs[0][1])
        if mode == "relu":
            assert torch.equal(zo, runs[0][2])
    monkeypatch.delenv("LA_TC_CHUNK")
    _compare(spec, mode, with_state=True)


def test_plan_of_the_workloads():
    assert la.la_plan(la.LA_MODE_GDN, la.LA_BF16, 1, 20, 181, 880, 128) == ("tcgen05_fused", 1)
    assert la.la_plan(la.LA_MODE_RELU, la.LA_BF16, 1, 20, 21, 1560, 112) == ("tcgen05_fused", 1)
    # 80 heads of 8 frames: one frame chunk, pipelined over two head groups
    assert la.la_plan(la.LA_MODE_GDN, la.LA_BF16, 4, 20, 8, 880, 128) == ("tcgen05", 6)
    assert la.la_plan(la.LA_MODE_GDN, la.LA_F32, 1, 2, 8, 64, 32)[0] == "simt_f32"
    # 8 pipeline chunks of 64 frames, three kernels each
    assert la.la_plan(la.LA_MODE_GDN, la.LA_BF16, 1, 16, 512, 1024, 256) == ("tcgen05_wide", 24)
    assert la.la_plan(la.LA_MODE_RELU, la.LA_BF16, 1, 16, 512, 1024, 256) == ("tcgen05_wide", 24)
    assert la.la_plan(la.LA_MODE_GDN, la.LA_F32, 1, 16, 512, 1024, 256)[0] == "simt_f32"


@pytest.mark.parametrize("mode", ["relu", "gdn"])
def test_fused_kernel_matches_three_kernel_path(mode, monkeypatch):
    spec = synth.small(B=2, H=5, F=13, S=250, D=112, dtype="bf16", seed=33, keys_l2=True)
    inp = device_inputs(spec)
    m0n, z0n = synth.random_state(spec, 0.05)
    m0, z0 = torch.from_numpy(m0n).cuda(), torch.from_numpy(z0n).cuda()
    o_f, m_f, z_f = _run(spec, mode, inp, m0, z0 if mode == "relu" else None)
    monkeypatch.setenv("LA_SCAN_NO_FUSE", "1")
    o_3, m_3, z_3 = _run(spec, mode, inp, m0, z0 if mode == "relu" else None)
    torch.cuda.synchronize()
    # The fused kernel adds each frame's increment as a bf16 operand of the
    # tensor core (the three-kernel path adds it in fp32), so the two agree to
    # bf16 rounding of the increments, well inside the bf16 parity bar.
    assert rel_err(to_np(o_f), to_np(o_3)) <= TOL_BF16
    assert rel_err(to_np(m_f), to_np(m_3)) <= TOL_BF16
    if mode == "relu":
        assert rel_err(to_np(z_f), to_np(z_3)) < 1e-5


@pytest.mark.parametrize("mode", ["relu", "gdn", "gdn_reverse", "gdn_token_beta"])
def test_fused_output_items_in_token_halves_are_exact(mode, monkeypatch):
    """Short clips split each output item into two token halves (two items
    read the frame's state image; the chain reuses the slot after both).  Each
    output tile is computed the same way either way, so the bits agree; 21
    frames reuse every hand-off slot; S = 650 leaves a ragged last tile."""
    spec = synth.small(B=2, H=6, F=21, S=650, D=112 if mode == "relu" else 128, dtype="bf16",
                       seed=75, keys_l2=True,
                       alpha=("sigmoid_normal", 3.0, 1.0), beta=("sigmoid_normal", 0.0, 1.0))
    B, H, F, S, D = spec.B, spec.H, spec.F, spec.S, spec.D
    inp = device_inputs(spec)
    m0n, z0n = synth.random_state(spec, 0.05)
    m0, z0 = torch.from_numpy(m0n).cuda(), torch.from_numpy(z0n).cuda()
    gates = torch.from_numpy(synth.token_gates(spec)).cuda() if mode == "gdn_token_beta" else None
    mcode = {"relu": la.LA_MODE_RELU, "gdn": la.LA_MODE_GDN, "gdn_reverse": la.LA_MODE_GDN_REVERSE,
             "gdn_token_beta": la.LA_MODE_GDN_TOKEN_BETA}[mode]
    assert la.la_plan(mcode, la.LA_BF16, B, H, F, S, D) == ("tcgen05_fused", 1)

    def run():
        ws = la.workspace_for(mcode, B, H, F, S, D)
        so = torch.empty((B, H, D, D), device="cuda")
        zo = torch.empty((B, H, D), device="cuda")
        if mode == "relu":
            o = la.la_scan_relu(inp["q"], inp["k"], inp["v"], state_in=m0, z_in=z0, state_out=so,
                                z_out=zo, eps=spec.eps, workspace=ws)
        elif mode == "gdn":
            o = la.la_scan_gdn(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                               spec.k_scale, state_in=m0, state_out=so, workspace=ws)
        elif mode == "gdn_reverse":
            o = la.la_scan_gdn_reverse(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                                       spec.k_scale, 8, workspace=ws)
            so = None
        else:
            o = la.la_scan_gdn_token_beta(inp["q"], inp["k"], inp["v"], inp["alpha"], gates,
                                          spec.k_scale, state_in=m0, state_out=so, workspace=ws)
        _check_status(ws)
        return o, so, zo

    runs = []
    for split in ("1", "0"):
        monkeypatch.setenv("LA_FUSED_OUT_SPLIT", split)
        runs.append(run())
    torch.cuda.synchronize()
    (o1, s1, z1), (o0, s0, z0_) = runs
    assert torch.isfinite(o1.float()).all()
    assert torch.equal(o1.view(torch.int16), o0.view(torch.int16))
    if s1 is not None:
        assert torch.equal(s1, s0)
    if mode == "relu":
        assert torch.equal(z1, z0_)
    if mode in ("relu", "gdn"):
        monkeypatch.setenv("LA_FUSED_OUT_SPLIT", "1")
        _compare(spec, mode, with_state=True, heads=[(0, 0), (1, 5)])


@pytest.mark.parametrize("mode", ["relu", "gdn"])
def test_fused_kernel_at_its_head_limit_with_slot_reuse(mode):
    # 49 (b, h) pairs: one chain block each on a 148-SM B200 (the fused
    # limit); F = 21 > 8 reuses every per-head hand-off slot.
    spec = synth.small(B=7, H=7, F=21, S=96, D=128, dtype="bf16", seed=35, keys_l2=True,
                       alpha=("sigmoid_normal", 3.0, 1.0), beta=("sigmoid_normal", 0.0, 1.0))
    assert la.la_plan(la.LA_MODE_GDN if mode == "gdn" else la.LA_MODE_RELU, la.LA_BF16,
                      7, 7, 21, 96, 128)[0] == "tcgen05_fused"
    _compare(spec, mode, with_state=True, heads=[(0, 0), (3, 4), (6, 6)])


def test_many_heads_use_the_three_kernel_path():
    spec = synth.small(B=15, H=20, F=2, S=64, D=64, dtype="bf16", seed=37)
    # 300 heads of 2 frames: two head groups of 150
    assert la.la_plan(la.LA_MODE_GDN, la.LA_BF16, 15, 20, 2, 64, 64) == ("tcgen05", 6)
    _compare(spec, "gdn", heads=[(0, 0), (7, 9), (7, 10), (14, 19)])


@pytest.mark.parametrize("mode", ["relu", "gdn"])
def test_three_kernel_head_groups_are_exact(mode, monkeypatch):
    """A one-chunk call on the three-kernel path runs as a pipeline of head
    groups (chain of one group beside the gram of the next and the output of
    the one before): any grouping gives the same bits, and the oracle's values
    on every head."""
    spec = synth.small(B=4, H=20, F=8, S=200, D=128, dtype="bf16", seed=73, keys_l2=True,
                       alpha=("sigmoid_normal", 3.0, 1.0), beta=("sigmoid_normal", 0.0, 1.0))
    m = la.LA_MODE_GDN if mode == "gdn" else la.LA_MODE_RELU
    assert la.la_plan(m, la.LA_BF16, 4, 20, 8, 200, 128) == ("tcgen05", 6)     # 2 groups
    inp = device_inputs(spec)
    m0n, z0n = synth.random_state(spec, 0.05)
    m0, z0 = torch.from_numpy(m0n).cuda(), torch.from_numpy(z0n).cuda()
    runs = []
    for groups in ("1", "3", "8"):
        monkeypatch.setenv("LA_TC_HEAD_GROUPS", groups)
        runs.append(_run(spec, mode, inp, m0, z0 if mode == "relu" else None))
    torch.cuda.synchronize()
    for o, so, zo in runs[1:]:
        assert torch.equal(o.view(torch.int16), runs[0][0].view(torch.int16))
        assert torch.equal(so, runs[0][1])
        if mode == "relu":
            assert torch.equal(zo, runs[0][2])
    monkeypatch.delenv("LA_TC_HEAD_GROUPS")
    _compare(spec, mode, with_state=True)


def test_device_wait_timeout_is_reported_and_the_context_stays_usable(monkeypatch):
    # A gram hand-off flag that nothing sets: the chain block's bounded wait
    # gives up, every block of the launch stops, the call's workspace records
    # LA_ERR_TIMEOUT, and the next call works normally.
    spec = synth.small(B=1, H=2, F=6, S=64, D=64, dtype="bf16", seed=39)
    inp = device_inputs(spec)
    ws = la.workspace_for(la.LA_MODE_GDN, 1, 2, 6, 64, 64)
    monkeypatch.setenv("LA_SCAN_TEST_SKIP_PUBLISH", "3")
    la.la_scan_gdn(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], spec.k_scale,
                   workspace=ws)
    assert la.la_query_device_status(ws) == la.LA_ERR_TIMEOUT
    monkeypatch.delenv("LA_SCAN_TEST_SKIP_PUBLISH")
    o = la.la_scan_gdn(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], spec.k_scale,
                       workspace=ws)
    assert la.la_query_device_status(ws) == la.LA_OK
    for h in range(2):
        ro, _, _ = _oracle(spec, "gdn", 0, h)
        assert rel_err(to_np(o[0, h]), ro) <= TOL_BF16
