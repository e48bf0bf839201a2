"""The allocation-free GDN entry point, la_scan_gdn_noalloc.

It serves callers that cannot call cudaMalloc and so cannot hand the library
a workspace (a plug-in whose host framework owns all device memory, or a
real-time loop that must not allocate).  It runs the same kernels as
la_scan_gdn with the library's built-in 64 MiB scratch array in place of the
workspace.  This file is named to be collected last, so that a run stopping
at its first failure has already run every other test.
"""
import ctypes

import pytest
import torch

import linear_attention_video_frame_b200 as la
import synth
from helpers import TOL_BF16, device_inputs, rel_err, to_np

pytestmark = pytest.mark.gpu


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def test_noalloc_matches_workspace_entry_point_on_two_calls_in_a_row():
    assert torch.cuda.is_available()
    # 720p-shaped GDN slice on the tensor-core path: 2 x 3 heads x 8 frames per call
    spec = synth.small(B=2, H=3, F=16, S=880, D=128, dtype="bf16", seed=41, keys_l2=True,
                       alpha=("sigmoid_normal", 3.0, 1.0), beta=("sigmoid_normal", 0.0, 1.0))
    assert la.la_plan(la.LA_MODE_GDN, la.LA_BF16, 2, 3, 8, 880, 128)[0].startswith("tcgen05")
    inp = device_inputs(spec)
    B, H, S, D = spec.B, spec.H, spec.S, spec.D
    stream = torch.cuda.current_stream()
    ref_state = None
    state = None
    for call, sl in enumerate((slice(0, 8), slice(8, 16))):
        part = {n: inp[n][:, :, sl].contiguous() for n in ("q", "k", "v", "alpha", "beta")}
        # the existing entry point, with a caller-owned workspace
        ref_out = torch.empty((B, H, D, D), device="cuda")
        ref_o = la.la_scan_gdn(part["q"], part["k"], part["v"], part["alpha"], part["beta"],
                               spec.k_scale, state_in=ref_state, state_out=ref_out)
        # the allocation-free entry point, through the C ABI
        o = torch.full_like(part["q"], float("nan"))
        out = torch.full((B, H, D, D), float("nan"), device="cuda")
        st = la.lib.la_scan_gdn_noalloc(
            _p(part["q"]), _p(part["k"]), _p(part["v"]), _p(o), la.LA_BF16, _p(part["alpha"]),
            _p(part["beta"]), spec.k_scale, _p(state), _p(out), B, H, 8, S, D,
            ctypes.c_void_p(stream.cuda_stream))
        assert st == la.LA_OK, la.la_status_string(st)
        torch.cuda.synchronize()
        assert rel_err(to_np(o), to_np(ref_o)) <= TOL_BF16, f"call {call}: outputs differ"
        assert rel_err(to_np(out), to_np(ref_out)) <= TOL_BF16, f"call {call}: states differ"
        ref_state, state = ref_out, out


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # 4 x 20 heads of 128 x 128 state need more than 64 MiB of scratch:
    # refused before anything is enqueued (the pointers are never touched).
    fake = ctypes.c_void_p(0x10000)
    st = la.lib.la_scan_gdn_noalloc(fake, fake, fake, fake, la.LA_BF16, fake, fake, 0.01,
                                    None, None, 4, 20, 181, 880, 128, None)
    assert st == la.LA_ERR_UNSUPPORTED
    assert la.la_workspace_size(la.LA_MODE_GDN, 4, 20, 181, 880, 128) > la.LA_NOALLOC_SCRATCH_BYTES
