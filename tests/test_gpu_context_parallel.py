"""GPU parity of the context-parallel GDN steps (SANA-WM paper summary,
appendix C.1): interval composites, the exclusive prefix, and the whole
split scan, against the oracle.

One GPU plays every rank in turn (composites of each interval, one prefix,
a rescan of each interval from its recovered start); no kernel waits on
another.  The orchestration with real ranks is covered on CPU (gloo) in
tests/test_context_parallel_cpu.py.
"""
import numpy as np
import pytest
import torch

import linear_attention_video_frame_b200 as la
import oracle
import synth
from helpers import TOL_BF16, TOL_F32, device_inputs, oracle_slice, rel_err, to_np, tol_for
from linear_attention_video_frame_b200.context_parallel import cp_scan_gdn, frame_interval

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"


def _part(inp, f0, f1):
    return {n: inp[n][:, :, f0:f1].contiguous() for n in ("q", "k", "v", "alpha", "beta")}


@pytest.mark.parametrize("dtype,D,S,F,path", [
    ("bf16", 128, 130, 5, "tcgen05"),      # tensor-core path, ragged token tail
    ("bf16", 64, 64, 3, "tcgen05"),
    ("bf16", 112, 200, 6, "tcgen05"),
    ("f32", 32, 40, 4, "simt_f32"),
    ("f32", 48, 17, 3, "simt_f32"),
    ("bf16", 256, 70, 3, "simt_f32"),      # wide heads: SIMT path
])
def test_interval_composites_match_oracle(dtype, D, S, F, path):
    spec = synth.small(B=2, H=2, F=F, S=S, D=D, dtype=dtype, seed=D + F, keys_l2=True)
    assert la.la_plan(la.LA_MODE_GDN_COMPOSITE, la.LA_BF16 if dtype == "bf16" else la.LA_F32,
                      2, 2, F, S, D)[0] == path
    inp = device_inputs(spec)
    out = torch.full((2, 2, 2, D, D), float("nan"), device="cuda")
    la.la_gdn_interval_composite(inp["k"], inp["v"], inp["alpha"], inp["beta"], spec.k_scale,
                                 out=out)
    torch.cuda.synchronize()
    tol = tol_for(spec)
    for b in range(2):
        for h in range(2):
            _, k, v, a, bt = oracle_slice(spec, b, h)
            T, U = oracle.gdn_interval_composite(k[0, 0], v[0, 0], a[0, 0], bt[0, 0],
                                                 spec.k_scale)
            assert rel_err(to_np(out[0, b, h]), T) <= tol
            assert rel_err(to_np(out[1, b, h]), U) <= tol
            # the composite is the state map: T M + U equals the scan from M
            m0 = np.eye(D) * 0.5 + 0.01
            _, m_ref = oracle.gdn_scan(k, k, v, a, bt, spec.k_scale, m0[None, None],
                                       want_output=False)
            got = to_np(out[0, b, h]) @ m0 + to_np(out[1, b, h])
            assert rel_err(got, m_ref[0, 0]) <= tol


def test_zero_frame_interval_is_the_identity():
    spec = synth.small(B=1, H=2, F=0, S=16, D=64, dtype="bf16")
    inp = device_inputs(spec)
    out = torch.full((2, 1, 2, 64, 64), float("nan"), device="cuda")
    la.la_gdn_interval_composite(inp["k"], inp["v"], inp["alpha"], inp["beta"], 0.1, out=out)
    torch.cuda.synchronize()
    eye = torch.eye(64, device="cuda").expand(1, 2, 64, 64)
    assert torch.equal(out[0], eye) and torch.count_nonzero(out[1]) == 0


@pytest.mark.parametrize("n,D,with_state", [(1, 16, False), (3, 48, True), (5, 128, True),
                                            (4, 256, False), (2, 80, True)])
def test_compose_prefix_matches_oracle(n, D, with_state):
    rng = np.random.default_rng(n * 1000 + D)
    B, H = 2, 3
    comps = np.empty((n, 2, B, H, D, D), dtype=np.float32)
    comps[:, 0] = (np.eye(D) * 0.9 + rng.standard_normal((n, B, H, D, D)) * 0.3 / np.sqrt(D))
    comps[:, 1] = rng.standard_normal((n, B, H, D, D))
    m0 = rng.standard_normal((B, H, D, D)).astype(np.float32) if with_state else None
    dev = torch.from_numpy(comps).cuda()
    m0d = torch.from_numpy(m0).cuda() if with_state else None
    so = torch.full((B, H, D, D), float("nan"), device="cuda")
    starts = la.la_gdn_compose_prefix(dev, state_in=m0d, state_out=so)
    torch.cuda.synchronize()
    for b in range(B):
        for h in range(H):
            pairs = [(comps[r, 0, b, h].astype(np.float64), comps[r, 1, b, h].astype(np.float64))
                     for r in range(n)]
            ref = oracle.compose_exclusive_prefix(pairs, None if m0 is None else m0[b, h])
            for r in range(n):
                assert rel_err(to_np(starts[r, b, h]), ref[r]) <= 1e-5
            T, U = pairs[-1]
            assert rel_err(to_np(so[b, h]), T @ ref[-1] + U) <= 1e-5


def _split_scan(spec, inp, ranks, m0=None):
    """Every rank's step on one GPU: composites, one prefix, the rescans."""
    B, H, D = spec.B, spec.H, spec.D
    spans = [frame_interval(spec.F, ranks, r) for r in range(ranks)]
    comps = torch.empty((ranks, 2, B, H, D, D), device="cuda")
    for r, (f0, f1) in enumerate(spans):
        p = _part(inp, f0, f1)
        la.la_gdn_interval_composite(p["k"], p["v"], p["alpha"], p["beta"], spec.k_scale,
                                     out=comps[r])
    final = torch.empty((B, H, D, D), device="cuda")
    starts = la.la_gdn_compose_prefix(comps, state_in=m0, state_out=final)
    outs = []
    for r, (f0, f1) in enumerate(spans):
        p = _part(inp, f0, f1)
        outs.append(la.la_scan_gdn(p["q"], p["k"], p["v"], p["alpha"], p["beta"], spec.k_scale,
                                   state_in=starts[r]))
    return torch.cat(outs, dim=2), final


@pytest.mark.parametrize("dtype,D,ranks", [("bf16", 128, 3), ("f32", 32, 4), ("bf16", 64, 1)])
def test_split_scan_equals_the_single_scan(dtype, D, ranks):
    spec = synth.small(B=2, H=2, F=11, S=96, D=D, dtype=dtype, seed=71 + D, keys_l2=True)
    inp = device_inputs(spec)
    m0n, _ = synth.random_state(spec, 0.05)
    o, final = _split_scan(spec, inp, ranks, torch.from_numpy(m0n).cuda())
    torch.cuda.synchronize()
    tol = tol_for(spec)
    for b in range(2):
        for h in range(2):
            q, k, v, a, bt = oracle_slice(spec, b, h)
            ro, rm = oracle.gdn_scan(q, k, v, a, bt, spec.k_scale, m0n[b:b + 1, h:h + 1])
            assert rel_err(to_np(o[b, h]), ro[0, 0]) <= tol
            assert rel_err(to_np(final[b, h]), rm[0, 0]) <= tol


def test_split_scan_of_the_720p_clip_over_four_ranks():
    """The 720p 60 s GDN workload (B1 H20 D128 F181 S880) as four intervals
    of 46/45/45/45 frames, every head against the oracle's single scan."""
    spec = synth.workload("gdn_720p_60s")
    inp = device_inputs(spec)
    o, final = _split_scan(spec, inp, 4)
    torch.cuda.synchronize()
    num_o = den_o = num_m = den_m = 0.0
    for h in range(spec.H):
        q, k, v, a, bt = oracle_slice(spec, 0, h)
        ro, rm = oracle.gdn_scan(q, k, v, a, bt, spec.k_scale)
        go, gm = to_np(o[0, h]), to_np(final[0, h])
        num_o, den_o = max(num_o, np.abs(go - ro[0, 0]).max()), max(den_o, np.abs(ro).max())
        num_m, den_m = max(num_m, np.abs(gm - rm[0, 0]).max()), max(den_m, np.abs(rm).max())
    print(f"\n[cp] 720p over 4 ranks: output {num_o / den_o:.3e} state {num_m / den_m:.3e}")
    assert num_o / den_o <= TOL_BF16 and num_m / den_m <= TOL_BF16


def test_cp_scan_on_one_rank_runs_the_device_steps():
    # without a process group cp_scan_gdn is a single rank: composite,
    # prefix and rescan all run on this library's kernels
    spec = synth.small(B=1, H=3, F=6, S=200, D=128, dtype="bf16", seed=73, keys_l2=True)
    inp = device_inputs(spec)
    so = torch.empty((1, 3, 128, 128), device="cuda")
    o = cp_scan_gdn(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], spec.k_scale,
                    state_out=so)
    ref_so = torch.empty_like(so)
    ref = la.la_scan_gdn(inp["q"], inp["k"], inp["v"], inp["alpha"], inp["beta"], spec.k_scale,
                         state_out=ref_so)
    torch.cuda.synchronize()
    assert rel_err(to_np(o), to_np(ref)) <= TOL_BF16
    assert rel_err(to_np(so), to_np(ref_so)) <= TOL_BF16
