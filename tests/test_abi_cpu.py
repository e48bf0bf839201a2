"""The C-ABI library on a machine without a GPU: it loads, exports every
declared symbol, and rejects bad arguments before touching CUDA."""
import ctypes
import os
import re

import pytest

import linear_attention_video_frame_b200 as la

HEADER = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                      "include", "la_scan.h")


def declared_symbols():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"LA_API\s+[\w\s\*]+?\b(la_\w+)\s*\(", txt)))


def test_header_declares_the_abi():
    assert declared_symbols() == sorted([
        "la_scan_relu", "la_scan_gdn", "la_state_step", "la_workspace_size",
        "la_query_device_status", "la_status_string", "la_plan", "la_scan_gdn_noalloc",
        "la_scan_host", "la_host_workspace_size", "la_host_chunk_frames",
        "la_scan_gdn_reverse", "la_scan_gdn_token_beta", "la_query_noalloc_status",
        "la_gdn_interval_composite", "la_gdn_compose_prefix", "la_scan_gdn_prep",
        "la_scan_relu_prep"])


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(la.LIB_PATH)
    for name in declared_symbols():
        assert hasattr(lib, name), name


def test_plan_reports_a_path_and_kernel_count():
    name, n = la.la_plan(la.LA_MODE_GDN, la.LA_BF16, 1, 20, 181, 880, 128)
    assert name in ("tcgen05_fused", "tcgen05", "tcgen05_wide", "simt_f32") and n >= 1
    name, n = la.la_plan(la.LA_MODE_RELU, la.LA_F32, 1, 2, 8, 64, 32)
    assert name == "simt_f32" and n == 1
    assert la.la_plan(la.LA_MODE_GDN, la.LA_BF16, 1, 1, 1, 1, 24) == (None, 0)


def test_status_strings():
    assert la.la_status_string(la.LA_OK) == "LA_OK"
    assert la.la_status_string(la.LA_ERR_TIMEOUT) == "LA_ERR_TIMEOUT"
    assert la.la_status_string(99) == "LA_ERR_UNKNOWN"


@pytest.mark.parametrize("D", [0, 8, 24, 100, 272])
def test_workspace_size_rejects_unsupported_head_dims(D):
    assert la.la_workspace_size(la.LA_MODE_GDN, 1, 1, 4, 64, D) == 0


@pytest.mark.parametrize("mode", [la.LA_MODE_RELU, la.LA_MODE_GDN])
@pytest.mark.parametrize("cfg", [(1, 2, 8, 64, 32), (1, 20, 21, 1560, 112),
                                 (1, 20, 181, 880, 128), (1, 16, 512, 1024, 256)])
def test_workspace_size_positive_and_aligned(mode, cfg):
    n = la.la_workspace_size(mode, *cfg)
    assert n >= 256 and n % 256 == 0


def _fake(addr=0x10000):
    return ctypes.c_void_p(addr)


def test_argument_errors_return_before_any_cuda_call():
    L = la.lib
    P = _fake
    ws = la.la_workspace_size(la.LA_MODE_GDN, 1, 1, 2, 8, 32)
    # unsupported head dim
    assert L.la_scan_gdn(P(), P(), P(), P(), la.LA_BF16, P(), P(), 0.1, None, None,
                         1, 1, 2, 8, 24, P(), ws, None) == la.LA_ERR_UNSUPPORTED
    # bad sizes
    assert L.la_scan_gdn(P(), P(), P(), P(), la.LA_BF16, P(), P(), 0.1, None, None,
                         0, 1, 2, 8, 32, P(), ws, None) == la.LA_ERR_INVALID_ARG
    assert L.la_scan_relu(P(), P(), P(), P(), la.LA_BF16, None, None, None, None,
                          1, 1, 2, 0, 32, 1e-6, P(), ws, None) == la.LA_ERR_INVALID_ARG
    # negative / non-finite eps, non-finite key scale
    assert L.la_scan_relu(P(), P(), P(), P(), la.LA_BF16, None, None, None, None,
                          1, 1, 2, 8, 32, -1.0, P(), ws, None) == la.LA_ERR_INVALID_ARG
    assert L.la_scan_gdn(P(), P(), P(), P(), la.LA_BF16, P(), P(), float("nan"), None, None,
                         1, 1, 2, 8, 32, P(), ws, None) == la.LA_ERR_INVALID_ARG
    # missing / misaligned / undersized workspace
    assert L.la_scan_gdn(P(), P(), P(), P(), la.LA_BF16, P(), P(), 0.1, None, None,
                         1, 1, 2, 8, 32, None, ws, None) == la.LA_ERR_INVALID_ARG
    assert L.la_scan_gdn(P(), P(), P(), P(), la.LA_BF16, P(), P(), 0.1, None, None,
                         1, 1, 2, 8, 32, P(0x10010), ws, None) == la.LA_ERR_INVALID_ARG
    assert L.la_scan_gdn(P(), P(), P(), P(), la.LA_BF16, P(), P(), 0.1, None, None,
                         1, 1, 2, 8, 32, P(), 16, None) == la.LA_ERR_INVALID_ARG
    # missing gates / inputs / output
    assert L.la_scan_gdn(P(), P(), P(), P(), la.LA_BF16, None, P(), 0.1, None, None,
                         1, 1, 2, 8, 32, P(), ws, None) == la.LA_ERR_INVALID_ARG
    assert L.la_scan_gdn(P(), None, P(), P(), la.LA_BF16, P(), P(), 0.1, None, None,
                         1, 1, 2, 8, 32, P(), ws, None) == la.LA_ERR_INVALID_ARG
    assert L.la_scan_relu(P(), P(), P(), None, la.LA_BF16, None, None, None, None,
                          1, 1, 2, 8, 32, 1e-6, P(), ws, None) == la.LA_ERR_INVALID_ARG
    # bad dtype / mode
    assert L.la_scan_relu(P(), P(), P(), P(), 7, None, None, None, None,
                          1, 1, 2, 8, 32, 1e-6, P(), ws, None) == la.LA_ERR_INVALID_ARG
    assert L.la_state_step(5, P(), P(), la.LA_BF16, None, None, 1.0, None, None, None, None,
                           1, 1, 2, 8, 32, P(), ws, None) == la.LA_ERR_INVALID_ARG


def test_reverse_scan_argument_errors_and_sizes():
    L = la.lib
    P = _fake
    ws = la.la_workspace_size(la.LA_MODE_GDN_REVERSE, 1, 1, 4, 16, 64)
    assert ws >= 256 and ws % 256 == 0
    # few heads: the reversed scan runs in the single fused kernel, with the
    # forward scan's per-head rings (no per-frame buffers)
    assert la.la_workspace_size(la.LA_MODE_GDN_REVERSE, 1, 20, 181, 880, 128) == \
        la.la_workspace_size(la.LA_MODE_GDN, 1, 20, 181, 880, 128)
    assert la.la_plan(la.LA_MODE_GDN_REVERSE, la.LA_BF16, 1, 20, 181, 880, 128) == \
        ("tcgen05_fused", 1)
    # many heads: the three-kernel path with per-frame buffers
    assert la.la_plan(la.LA_MODE_GDN_REVERSE, la.LA_BF16, 4, 20, 64, 880, 128)[0] == "tcgen05"
    assert la.la_plan(la.LA_MODE_GDN_REVERSE, la.LA_BF16, 1, 16, 512, 1024, 256)[0] == \
        "tcgen05_wide"
    args = lambda C, D=64, w=ws: (P(), P(), P(), P(), la.LA_BF16, P(), P(), 0.1, C,
                                  1, 1, 4, 16, D, P(), w, None)
    assert L.la_scan_gdn_reverse(*args(0)) == la.LA_ERR_INVALID_ARG
    assert L.la_scan_gdn_reverse(*args(-3)) == la.LA_ERR_INVALID_ARG
    assert L.la_scan_gdn_reverse(*args(2, D=24)) == la.LA_ERR_UNSUPPORTED
    assert L.la_scan_gdn_reverse(*args(2, w=16)) == la.LA_ERR_INVALID_ARG
    assert L.la_state_step(la.LA_MODE_GDN_REVERSE, P(), P(), la.LA_BF16, P(), P(), 0.1, None,
                           None, None, None, 1, 1, 4, 16, 64, P(), ws, None) == la.LA_ERR_INVALID_ARG


def test_token_gate_scan_argument_errors_and_plan():
    L = la.lib
    P = _fake
    ws = la.la_workspace_size(la.LA_MODE_GDN_TOKEN_BETA, 1, 1, 4, 16, 64)
    assert ws >= 256 and ws % 256 == 0
    assert la.la_plan(la.LA_MODE_GDN_TOKEN_BETA, la.LA_BF16, 1, 20, 181, 880, 128) == \
        ("tcgen05_fused", 1)
    assert la.la_plan(la.LA_MODE_GDN_TOKEN_BETA, la.LA_BF16, 4, 20, 64, 880, 128)[0] == "tcgen05"
    assert la.la_plan(la.LA_MODE_GDN_TOKEN_BETA, la.LA_F32, 1, 2, 8, 64, 32)[0] == "simt_f32"
    assert la.la_workspace_size(7, 1, 1, 4, 16, 64) == 0      # no mode 7
    args = lambda bt=P(), D=64, w=ws: (P(), P(), P(), P(), la.LA_BF16, P(), bt, 0.1, None, None,
                                       1, 1, 4, 16, D, P(), w, None)
    assert L.la_scan_gdn_token_beta(*args(bt=None)) == la.LA_ERR_INVALID_ARG
    assert L.la_scan_gdn_token_beta(*args(D=24)) == la.LA_ERR_UNSUPPORTED
    assert L.la_scan_gdn_token_beta(*args(w=16)) == la.LA_ERR_INVALID_ARG


def test_host_chunking_rule():
    assert la.la_host_chunk_frames(181) == 12          # about 16 chunks
    assert la.la_host_chunk_frames(8) == 1
    assert la.la_host_chunk_frames(0) == 1
    assert la.la_host_chunk_frames(21, 4) == 4
    assert la.la_host_chunk_frames(6, 50) == 6          # never longer than the clip
    assert la.la_host_chunk_frames(-1) == 0


def test_host_workspace_size():
    G, R = la.LA_MODE_GDN, la.LA_MODE_RELU
    n = la.la_host_workspace_size(G, la.LA_BF16, 1, 20, 181, 880, 128, 0)
    # three slots of q, k, v, o chunks (12 frames) dominate
    slot_q = 20 * 12 * 880 * 128 * 2
    assert n >= 3 * 4 * slot_q and n % 256 == 0
    assert n >= la.la_workspace_size(G, 1, 20, 12, 880, 128) + 3 * 4 * slot_q
    assert la.la_host_workspace_size(G, la.LA_F32, 1, 20, 181, 880, 128, 0) > n
    assert la.la_host_workspace_size(G, la.LA_BF16, 1, 20, 181, 880, 128, 24) > n
    assert la.la_host_workspace_size(R, la.LA_BF16, 1, 20, 21, 1560, 112, 0) > 0
    assert la.la_host_workspace_size(G, la.LA_BF16, 1, 1, 4, 64, 24, 0) == 0
    assert la.la_host_workspace_size(G, 5, 1, 1, 4, 64, 32, 0) == 0
    assert la.la_host_workspace_size(7, la.LA_BF16, 1, 1, 4, 64, 32, 0) == 0
    assert la.la_host_workspace_size(G, la.LA_BF16, 0, 1, 4, 64, 32, 0) == 0


def test_host_scan_argument_errors_return_before_any_cuda_call():
    L = la.lib
    P = _fake
    B, H, F, S, D = 1, 1, 4, 16, 32
    ws = la.la_host_workspace_size(la.LA_MODE_GDN, la.LA_BF16, B, H, F, S, D, 0)

    def call(mode=la.LA_MODE_GDN, dt=la.LA_BF16, shape=(B, H, F, S, D), w=P(), n=ws,
             ks=0.1, eps=1e-6, q=P()):
        return L.la_scan_host(mode, q, P(), P(), P(0x20000), dt, P(), P(), ks, eps,
                              None, None, None, None, *shape, 0, w, n, None)

    assert call(dt=3) == la.LA_ERR_INVALID_ARG
    assert call(mode=9) == la.LA_ERR_INVALID_ARG
    assert call(shape=(1, 1, 4, 16, 24)) == la.LA_ERR_UNSUPPORTED
    assert call(shape=(1, 0, 4, 16, 32)) == la.LA_ERR_INVALID_ARG
    assert call(shape=(1, 1, -1, 16, 32)) == la.LA_ERR_INVALID_ARG
    assert call(ks=float("inf")) == la.LA_ERR_INVALID_ARG
    assert call(mode=la.LA_MODE_RELU, eps=-1.0) == la.LA_ERR_INVALID_ARG
    assert call(w=None) == la.LA_ERR_INVALID_ARG
    assert call(w=P(0x10080)) == la.LA_ERR_INVALID_ARG
    assert call(n=ws - 1) == la.LA_ERR_INVALID_ARG
    assert call(q=None) == la.LA_ERR_INVALID_ARG


def test_python_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 1, 1, 16, 16, dtype=torch.bfloat16)
    a = torch.ones(1, 1, 1)
    with pytest.raises(ValueError):
        la.la_scan_gdn(x, x, x, a, a, 0.1, workspace=torch.zeros(1024, dtype=torch.uint8))


@pytest.mark.parametrize("F,chunks", [(8, 1), (31, 1), (32, 2), (40, 3), (181, 8), (512, 8)])
def test_three_kernel_path_chunk_count(F, chunks, monkeypatch):
    """Clips of 32+ frames with few heads run as a pipeline of frame chunks of
    max(16, ceil(F / 8)) frames, three kernels per chunk (two without output)
    (LA_SCAN_NO_FUSE keeps few heads off the single-kernel path)."""
    monkeypatch.setenv("LA_SCAN_NO_FUSE", "1")
    assert la.la_plan(la.LA_MODE_GDN_REVERSE, la.LA_BF16, 1, 4, F, 64, 128) == ("tcgen05", 3 * chunks)


def test_three_kernel_pipeline_needs_free_sms():
    # 80 heads would hold more than half of the SMs with chain CTAs: one frame
    # chunk, pipelined over two head groups instead
    assert la.la_plan(la.LA_MODE_GDN_REVERSE, la.LA_BF16, 4, 20, 64, 880, 128) == ("tcgen05", 6)


@pytest.mark.parametrize("B,H,F,groups", [(4, 20, 8, 2), (4, 20, 1, 1), (3, 20, 4, 1),
                                          (1, 60, 16, 2), (1, 80, 64, 2), (1, 7, 24, 1)])
def test_three_kernel_head_groups(B, H, F, groups, monkeypatch):
    """A one-chunk call with at least 8 heads and B H F >= 2 x 148 items runs
    its heads in two groups, three kernels per group."""
    monkeypatch.setenv("LA_SCAN_NO_FUSE", "1")
    assert la.la_plan(la.LA_MODE_GDN, la.LA_BF16, B, H, F, 880, 128) == ("tcgen05", 3 * groups)
    assert la.la_plan(la.LA_MODE_RELU, la.LA_BF16, B, H, F, 880, 128) == ("tcgen05", 3 * groups)


def test_three_kernel_head_groups_override(monkeypatch):
    monkeypatch.setenv("LA_SCAN_NO_FUSE", "1")
    monkeypatch.setenv("LA_TC_HEAD_GROUPS", "3")
    assert la.la_plan(la.LA_MODE_GDN, la.LA_BF16, 4, 20, 8, 880, 128) == ("tcgen05", 9)
    monkeypatch.setenv("LA_TC_HEAD_GROUPS", "1000")      # at most one group per head
    assert la.la_plan(la.LA_MODE_GDN, la.LA_BF16, 1, 5, 8, 880, 128) == ("tcgen05", 15)


def test_reversed_scan_chunks_align_with_pipeline_chunks(monkeypatch):
    # F = 181 -> pipeline chunks of 23 frames, rounded up to whole 8-frame reversed
    # chunks (24 frames): 8 launches of three kernels
    monkeypatch.setenv("LA_SCAN_NO_FUSE", "1")
    assert la.la_plan(la.LA_MODE_GDN_REVERSE, la.LA_BF16, 1, 20, 181, 880, 128) == ("tcgen05", 24)


@pytest.mark.parametrize("F,chunks", [(2, 1), (4, 1), (6, 2), (21, 6), (64, 8), (512, 8)])
def test_wide_path_chunk_count(F, chunks):
    """Wide heads run in chunks of max(4, ceil(F / 8)) frames."""
    assert la.la_plan(la.LA_MODE_GDN, la.LA_BF16, 1, 2, F, 64, 256) == ("tcgen05_wide", 3 * chunks)


def test_noalloc_scratch_limit_matches_its_documentation():
    """The built-in 64 MiB scratch holds the single-kernel path's per-head
    buffers (about 1.5 MiB per (b, h) pair whatever F is) for up to 42 pairs
    of 128 x 128 state; 43 pairs need more and are refused."""
    lim = la.LA_NOALLOC_SCRATCH_BYTES
    for F in (1, 181, 961):
        assert la.la_workspace_size(la.LA_MODE_GDN, 1, 42, F, 880, 128) <= lim
        assert la.la_workspace_size(la.LA_MODE_GDN, 1, 43, F, 880, 128) > lim
    # three-kernel path (more than 49 pairs): per-frame buffers, so F matters
    assert la.la_plan(la.LA_MODE_GDN, la.LA_BF16, 1, 63, 7, 880, 128)[0] == "tcgen05"
    assert la.la_workspace_size(la.LA_MODE_GDN, 1, 63, 7, 880, 128) <= lim
    assert la.la_workspace_size(la.LA_MODE_GDN, 1, 63, 8, 880, 128) > lim
    # float32 inputs and D < 64 need only the header
    assert la.la_workspace_size(la.LA_MODE_GDN, 4, 20, 181, 880, 32) < 4096


def test_composite_and_prefix_argument_errors_and_plan():
    L = la.lib
    P = _fake
    ws = la.la_workspace_size(la.LA_MODE_GDN_COMPOSITE, 1, 2, 5, 64, 128)
    assert ws >= 256 and ws % 256 == 0
    # one gram plus one chain launch of 2 B H blocks on the tensor-core path
    assert la.la_plan(la.LA_MODE_GDN_COMPOSITE, la.LA_BF16, 1, 20, 45, 880, 128) == ("tcgen05", 2)
    assert la.la_plan(la.LA_MODE_GDN_COMPOSITE, la.LA_F32, 1, 20, 45, 880, 128) == ("simt_f32", 1)
    assert la.la_plan(la.LA_MODE_GDN_COMPOSITE, la.LA_BF16, 1, 16, 8, 1024, 256)[0] == "simt_f32"
    # both outputs are required; they must not overlap; sizes and head dims are checked
    assert L.la_gdn_interval_composite(P(), P(), la.LA_BF16, P(), P(), 0.1, None, P(0x20000),
                                       1, 2, 5, 64, 128, P(), ws, None) == la.LA_ERR_INVALID_ARG
    assert L.la_gdn_interval_composite(P(), P(), la.LA_BF16, P(), P(), 0.1, P(0x20000),
                                       P(0x20000), 1, 2, 5, 64, 128, P(), ws, None) == \
        la.LA_ERR_INVALID_ARG
    assert L.la_gdn_interval_composite(P(), P(), la.LA_BF16, P(), P(), 0.1, P(0x20000),
                                       P(0x90000), 1, 2, 5, 64, 24, P(), ws, None) == \
        la.LA_ERR_UNSUPPORTED
    one = 2 * 3 * 64 * 64
    assert L.la_gdn_compose_prefix(P(), P(), one, None, P(), None, 0, 2, 3, 64, None) == \
        la.LA_ERR_INVALID_ARG
    assert L.la_gdn_compose_prefix(P(), P(), one - 1, None, P(), None, 2, 2, 3, 64, None) == \
        la.LA_ERR_INVALID_ARG
    assert L.la_gdn_compose_prefix(P(), P(), one, None, None, None, 2, 2, 3, 64, None) == \
        la.LA_ERR_INVALID_ARG
    assert L.la_gdn_compose_prefix(P(), P(), one, None, P(), None, 2, 2, 3, 40, None) == \
        la.LA_ERR_UNSUPPORTED


def test_prep_argument_errors_return_before_any_cuda_call():
    L = la.lib
    P = _fake
    ws = la.la_workspace_size(la.LA_MODE_GDN_PREP, 1, 2, 4, 12, 64)
    assert ws >= la.la_workspace_size(la.LA_MODE_GDN, 1, 2, 4, 12, 64)
    # single-kernel path for bf16 GDN with the preparation; ReLU with it on SIMT
    assert la.la_plan(la.LA_MODE_GDN_PREP, la.LA_BF16, 1, 20, 181, 880, 128) == ("tcgen05_fused", 1)
    assert la.la_plan(la.LA_MODE_RELU_PREP, la.LA_BF16, 1, 20, 21, 1560, 112) == ("simt_f32", 1)
    assert la.la_plan(la.LA_MODE_GDN_PREP, la.LA_F32, 1, 2, 4, 12, 64) == ("simt_f32", 1)

    def gdn(prep):
        return L.la_scan_gdn_prep(P(), P(), P(), P(), la.LA_BF16, P(), P(), 0.1,
                                  None if prep is None else ctypes.byref(prep), None, None,
                                  1, 2, 4, 12, 64, P(), ws, None)

    assert gdn(None) == la.LA_ERR_INVALID_ARG
    mk = lambda **kw: la.LaPrep(None, None, kw.get("eps", 1e-6), kw.get("rope", 1),
                                kw.get("gh", 3), kw.get("gw", 4), kw.get("off", 0),
                                kw.get("base", 1e4))
    assert gdn(mk(gh=5)) == la.LA_ERR_INVALID_ARG              # 5 x 4 != 12 tokens
    assert gdn(mk(gh=0, gw=12)) == la.LA_ERR_INVALID_ARG
    assert gdn(mk(base=0.5)) == la.LA_ERR_INVALID_ARG
    assert gdn(mk(eps=float("nan"))) == la.LA_ERR_INVALID_ARG
    assert gdn(mk(off=-3)) == la.LA_ERR_INVALID_ARG
    assert gdn(mk(off=1 << 24)) == la.LA_ERR_INVALID_ARG       # positions stay below 2^24
    assert L.la_scan_relu_prep(P(), P(), P(), P(), la.LA_BF16, None, None, None, None, None,
                               1, 2, 4, 12, 64, 1e-6, P(), ws, None) == la.LA_ERR_INVALID_ARG
