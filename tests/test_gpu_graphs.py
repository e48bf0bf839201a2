"""Calls captured into CUDA graphs replay with the same results as direct
calls: the fused kernel (one cooperative launch), the wide-head path (its
chunk pipeline forks to the library's own streams and joins back inside the
capture) and the three-kernel path."""
import pytest
import torch

import linear_attention_video_frame_b200 as la
import synth
from helpers import device_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    torch.cuda.init()


@pytest.mark.parametrize("shape,path", [
    (dict(B=1, H=4, F=12, S=200, D=128), "tcgen05_fused"),
    (dict(B=4, H=20, F=4, S=64, D=64), "tcgen05"),
    (dict(B=1, H=2, F=20, S=64, D=256), "tcgen05_wide"),
])
@pytest.mark.parametrize("mode", ["gdn", "relu"])
def test_graph_replay_equals_direct_call(shape, path, mode):
    spec = synth.small(dtype="bf16", seed=61, keys_l2=True, **shape)
    B, H, F, S, D = spec.B, spec.H, spec.F, spec.S, spec.D
    m = la.LA_MODE_GDN if mode == "gdn" else la.LA_MODE_RELU
    assert la.la_plan(m, la.LA_BF16, B, H, F, S, D)[0] == path
    inp = device_inputs(spec)
    ws = la.workspace_for(m, B, H, F, S, D)
    o = torch.empty_like(inp["q"])
    st = torch.empty((B, H, D, D), device="cuda")

    def call(stream=None):
        if mode == "gdn":
            la.la_scan_gdn(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], spec.k_scale,
                           o=o, state_out=st, workspace=ws, stream=stream)
        else:
            la.la_scan_relu(inp["q"], inp["k"], inp["v"], o=o, state_out=st, workspace=ws,
                            stream=stream)

    call()
    torch.cuda.synchronize()
    o_ref, st_ref = o.clone(), st.clone()
    o.zero_()
    st.zero_()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        call(stream=s)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert la.la_query_device_status(ws) == la.LA_OK
    assert torch.equal(o.view(torch.int16), o_ref.view(torch.int16))
    assert torch.equal(st, st_ref)
    del g
