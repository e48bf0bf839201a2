"""The allocation-free GDN entry point, la_scan_gdn_noalloc.

It serves callers that cannot call cudaMalloc and so cannot hand the library
a workspace (a plug-in whose host framework owns all device memory, or a
real-time loop that must not allocate).  It runs the same kernels as
la_scan_gdn with the library's built-in 64 MiB scratch array in place of the
workspace; the tests cover each kernel path's layout of that array and the
status query that reads a device-side timeout back from it.  This file is
named to be collected last, so that a run stopping at its first failure has
already run every other test.
"""
import ctypes

import pytest
import torch

import linear_attention_video_frame_b200 as la
import synth
from helpers import TOL_BF16, TOL_F32, device_inputs, rel_err, to_np

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _two_calls_in_a_row(spec, path):
    """Two chunks of the clip, the second starting from the first's state:
    the no-alloc entry point against la_scan_gdn with its own workspace."""
    B, H, S, D = spec.B, spec.H, spec.S, spec.D
    half = spec.F // 2
    dt = la.LA_BF16 if spec.dtype == "bf16" else la.LA_F32
    assert la.la_plan(la.LA_MODE_GDN, dt, B, H, half, S, D)[0] == path
    tol = TOL_BF16 if spec.dtype == "bf16" else TOL_F32
    inp = device_inputs(spec)
    stream = torch.cuda.current_stream()
    ref_state = None
    state = None
    for call, sl in enumerate((slice(0, half), slice(half, 2 * half))):
        part = {n: inp[n][:, :, sl].contiguous() for n in ("q", "k", "v", "alpha", "beta")}
        # the existing entry point, with a caller-owned workspace
        ref_out = torch.empty((B, H, D, D), device="cuda")
        ref_o = la.la_scan_gdn(part["q"], part["k"], part["v"], part["alpha"], part["beta"],
                               spec.k_scale, state_in=ref_state, state_out=ref_out)
        # the allocation-free entry point, through the C ABI
        o = torch.full_like(part["q"], float("nan"))
        out = torch.full((B, H, D, D), float("nan"), device="cuda")
        st = la.lib.la_scan_gdn_noalloc(
            _p(part["q"]), _p(part["k"]), _p(part["v"]), _p(o), dt, _p(part["alpha"]),
            _p(part["beta"]), spec.k_scale, _p(state), _p(out), B, H, half, S, D,
            ctypes.c_void_p(stream.cuda_stream))
        assert st == la.LA_OK, la.la_status_string(st)
        assert la.la_query_noalloc_status() == la.LA_OK
        assert rel_err(to_np(o), to_np(ref_o)) <= tol, f"call {call}: outputs differ"
        assert rel_err(to_np(out), to_np(ref_out)) <= tol, f"call {call}: states differ"
        ref_state, state = ref_out, out


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    assert torch.cuda.is_available()
    # 720p-shaped GDN slice on the single-kernel path: 2 x 3 heads x 8 frames per call
    spec = synth.small(B=2, H=3, F=16, S=880, D=128, dtype="bf16", seed=41, keys_l2=True,
                       alpha=("sigmoid_normal", 3.0, 1.0), beta=("sigmoid_normal", 0.0, 1.0))
    _two_calls_in_a_row(spec, "tcgen05_fused")


def test_noalloc_three_kernel_layout_on_two_calls_in_a_row(monkeypatch):
    # The three-kernel path keeps per-frame buffers and the carried state at
    # other offsets of the shared array than the single-kernel path.
    monkeypatch.setenv("LA_SCAN_NO_FUSE", "1")
    spec = synth.small(B=1, H=4, F=12, S=300, D=128, dtype="bf16", seed=43, keys_l2=True,
                       alpha=("sigmoid_normal", 3.0, 1.0), beta=("sigmoid_normal", 0.0, 1.0))
    _two_calls_in_a_row(spec, "tcgen05")


def test_noalloc_float32_simt_layout_on_two_calls_in_a_row():
    spec = synth.small(B=1, H=2, F=8, S=64, D=32, dtype="f32", seed=45)
    _two_calls_in_a_row(spec, "simt_f32")


def test_noalloc_device_timeout_is_reported_by_its_status_query(monkeypatch):
    # A gram hand-off flag that nothing sets (the library's test hook): the
    # bounded wait gives up, the status word in the built-in array records
    # LA_ERR_TIMEOUT, and the next call starts from a clean status.
    spec = synth.small(B=1, H=2, F=6, S=64, D=64, dtype="bf16", seed=47)
    inp = device_inputs(spec)
    monkeypatch.setenv("LA_SCAN_TEST_SKIP_PUBLISH", "3")
    la.la_scan_gdn_noalloc(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                           spec.k_scale)
    assert la.la_query_noalloc_status() == la.LA_ERR_TIMEOUT
    monkeypatch.delenv("LA_SCAN_TEST_SKIP_PUBLISH")
    o = la.la_scan_gdn_noalloc(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"],
                               spec.k_scale)
    assert la.la_query_noalloc_status() == la.LA_OK
    ref = la.la_scan_gdn(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], spec.k_scale)
    torch.cuda.synchronize()
    assert rel_err(to_np(o), to_np(ref)) <= TOL_BF16


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # 4 x 20 heads of 128 x 128 state need more than 64 MiB of scratch:
    # refused before anything is enqueued (the pointers are never touched).
    fake = ctypes.c_void_p(0x10000)
    st = la.lib.la_scan_gdn_noalloc(fake, fake, fake, fake, la.LA_BF16, fake, fake, 0.01,
                                    None, None, 4, 20, 181, 880, 128, None)
    assert st == la.LA_ERR_UNSUPPORTED
    assert la.la_workspace_size(la.LA_MODE_GDN, 4, 20, 181, 880, 128) > la.LA_NOALLOC_SCRATCH_BYTES
