"""GPU parity of the reversed GDN scan reset at chunk boundaries
(la_scan_gdn_reverse) against the CPU oracle.

Bars as for the forward scan: 1e-4 for float32 inputs, 2e-2 for bfloat16
inputs (max|gpu - ref| / max|ref|).  bf16 heads with 64 <= D <= 128 run on
the single-kernel tensor-core path (the three-kernel path for many heads),
128 < D <= 256 on the wide path, the rest on the SIMT kernel.
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


def _run(spec, inp, C):
    B, H, F, S, D = spec.B, spec.H, spec.F, spec.S, spec.D
    ws = la.workspace_for(la.LA_MODE_GDN_REVERSE, B, H, F, S, D)
    o = la.la_scan_gdn_reverse(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                               spec.k_scale, C, workspace=ws)
    assert la.la_query_device_status(ws) == la.LA_OK
    return o


def _compare(spec, C, heads=None):
    inp = device_inputs(spec)
    o = _run(spec, inp, C)
    torch.cuda.synchronize()
    pairs = heads or [(b, h) for b in range(spec.B) for h in range(spec.H)]
    got, ref = [], []
    for b, h in pairs:
        q, k, v, a, bt = oracle_slice(spec, b, h)
        ref.append(oracle.gdn_scan_reverse_chunked(q, k, v, a, bt, spec.k_scale, C)[0, 0])
        got.append(to_np(o[b, h]))
    e = rel_err(np.stack(got), np.stack(ref))
    print(f"\n[reverse] {spec.name} chunk={C}: output {e:.3e} (bar {tol_for(spec)})")
    assert e <= tol_for(spec)
    return o


@pytest.mark.parametrize("dtype,D,S,F,C", [
    ("bf16", 128, 130, 7, 3),      # tensor-core path, ragged last chunk
    ("bf16", 64, 64, 6, 1),        # one-frame chunks
    ("bf16", 112, 200, 5, 5),      # one chunk = the whole clip
    ("bf16", 128, 96, 9, 16),      # chunk longer than the clip
    ("f32", 32, 40, 7, 3),         # SIMT path
    ("f32", 128, 33, 5, 2),
    ("bf16", 256, 70, 5, 2),       # wide heads: wide tensor-core path
])
def test_reverse_scan_matches_oracle(dtype, D, S, F, C):
    spec = synth.small(B=2, H=2, F=F, S=S, D=D, dtype=dtype, seed=D + F, keys_l2=True)
    _compare(spec, C)


def test_reverse_scan_720p_gdn_all_heads():
    """The 720p 60 s GDN workload (B1 H20 D128 F181 S880) in chunks of 8 frames."""
    spec = synth.workload("gdn_720p_60s")
    assert la.la_plan(la.LA_MODE_GDN_REVERSE, la.LA_BF16, 1, 20, 181, 880, 128) == \
        ("tcgen05_fused", 1)
    _compare(spec, 8)


def test_reverse_tensor_core_path_matches_simt_path(monkeypatch):
    spec = synth.small(B=1, H=3, F=10, S=300, D=128, dtype="bf16", seed=51, keys_l2=True)
    inp = device_inputs(spec)
    o_tc = _run(spec, inp, 4)
    monkeypatch.setenv("LA_SCAN_FORCE_SIMT", "1")
    o_simt = _run(spec, inp, 4)
    torch.cuda.synchronize()
    assert rel_err(to_np(o_tc), to_np(o_simt)) <= TOL_BF16


def test_reverse_chunks_are_independent():
    """Changing one chunk's inputs leaves every other chunk's outputs bit-identical."""
    spec = synth.small(B=1, H=2, F=9, S=64, D=128, dtype="bf16", seed=53, keys_l2=True)
    inp = device_inputs(spec)
    o1 = _run(spec, inp, 3).clone()
    inp2 = {n: t.clone() for n, t in inp.items()}
    inp2["k"][:, :, 4] = -inp2["k"][:, :, 4]
    inp2["v"][:, :, 4] *= 3
    o2 = _run(spec, inp2, 3)
    torch.cuda.synchronize()
    same = [0, 1, 2, 6, 7, 8]
    assert torch.equal(o1[:, :, same].view(torch.int16), o2[:, :, same].view(torch.int16))
    assert not torch.equal(o1[:, :, 3].view(torch.int16), o2[:, :, 3].view(torch.int16))
    # inside the chunk {3, 4, 5} the reversed scan carries frame 4 back to frame 3, not on to 5
    assert torch.equal(o1[:, :, 5].view(torch.int16), o2[:, :, 5].view(torch.int16))


@pytest.mark.parametrize("C", [1, 4, 8])
def test_reverse_fused_kernel_matches_three_kernel_path(C, monkeypatch):
    """The single-kernel path (chunk resets as a zero decay at each chunk's
    first step) against the three-kernel path on the same inputs."""
    spec = synth.small(B=2, H=3, F=13, S=250, D=128, dtype="bf16", seed=61 + C, keys_l2=True,
                       alpha=("sigmoid_normal", 3.0, 1.0), beta=("sigmoid_normal", 0.0, 1.0))
    assert la.la_plan(la.LA_MODE_GDN_REVERSE, la.LA_BF16, 2, 3, 13, 250, 128)[0] == "tcgen05_fused"
    inp = device_inputs(spec)
    o_f = _run(spec, inp, C).clone()
    monkeypatch.setenv("LA_SCAN_NO_FUSE", "1")
    o_3 = _run(spec, inp, C)
    torch.cuda.synchronize()
    assert rel_err(to_np(o_f), to_np(o_3)) <= TOL_BF16
    monkeypatch.delenv("LA_SCAN_NO_FUSE")
    _compare(spec, C)


@pytest.mark.parametrize("wide_chunk", ["3", "7", "21"])
def test_reverse_wide_path_with_unaligned_pipeline_chunks(wide_chunk, monkeypatch):
    """D = 256 runs on the wide tensor-core path; its pipeline chunks (3, 7 or
    21 frames) need not line up with the reversed scan's 4-frame chunks, since
    a chunk start is a zero decay at that step."""
    spec = synth.small(B=1, H=2, F=21, S=100, D=256, dtype="bf16", seed=97, keys_l2=True)
    assert la.la_plan(la.LA_MODE_GDN_REVERSE, la.LA_BF16, 1, 2, 21, 100, 256)[0] == "tcgen05_wide"
    monkeypatch.setenv("LA_WIDE_CHUNK", wide_chunk)
    _compare(spec, 4)
