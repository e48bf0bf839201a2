"""Pins of the oracle's fused input preparation (RMSNorm, ReLU, 3D RoPE) and
of the scans on prepared features, against closed forms, hand-worked
examples and invariants that do not come from the oracle itself.

Readings pinned here (the pages give the order of the steps -- SANA-WM
digest, method details, "Context-Parallel + Fused Triton": RMSNorm + ReLU +
key scaling + UCPE/RoPE + GDN scan -- but no formulas): RMSNorm over the
head dimension with a per-head weight; 3D RoPE on adjacent channel pairs,
temporal group first, then height and width; in ReLU mode RoPE enters the
numerator only.
"""
import copy
import json
import math
import os

import numpy as np
import pytest

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _expr(x):
    """Value of a closed-form golden entry ('cos(1)', '3/4 + sin(2)/4', 2)."""
    if isinstance(x, list):
        return [_expr(e) for e in x]
    if isinstance(x, (int, float)):
        return float(x)
    return float(eval(x, {"__builtins__": {}}, {"cos": math.cos, "sin": math.sin}))


def _golden(name):
    d = json.load(open(os.path.join(GOLDEN, name)))
    arr = lambda key: np.array(d[key], dtype=np.float64)[None, None]
    return d, arr


# ----------------------------------------------------------------------------
# RMSNorm
# ----------------------------------------------------------------------------
def test_rms_norm_hand_example_and_closed_forms():
    # [3, 4]: mean square 12.5 -> [3, 4] / sqrt(12.5)
    y = oracle.rms_norm(np.array([3.0, 4.0]), eps=0.0)
    assert np.allclose(y, [3 / math.sqrt(12.5), 4 / math.sqrt(12.5)], rtol=0, atol=1e-15)
    # a constant row c maps to c / sqrt(c^2 + eps) in every channel
    for c in (-2.5, 0.3, 7.0):
        y = oracle.rms_norm(np.full(8, c), eps=1e-3)
        assert np.allclose(y, c / math.sqrt(c * c + 1e-3), rtol=1e-15)
    # the weight scales channel by channel
    w = np.array([2.0, 0.5, -1.0, 3.0])
    x = np.array([1.0, -2.0, 0.5, 4.0])
    assert np.allclose(oracle.rms_norm(x, w, 0.0), w * oracle.rms_norm(x, None, 0.0))


def test_rms_norm_unit_rms_and_scale_invariance():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 7, 48))
    y = oracle.rms_norm(x, eps=0.0)
    assert np.allclose(np.sqrt(np.mean(y * y, axis=-1)), 1.0, atol=1e-14)
    assert np.allclose(oracle.rms_norm(3.7 * x, eps=0.0), y, atol=1e-14)
    assert np.allclose(oracle.rms_norm(-0.2 * x, eps=0.0), -y, atol=1e-14)


# ----------------------------------------------------------------------------
# 3D RoPE
# ----------------------------------------------------------------------------
def test_rope_groups_split_the_pairs():
    assert oracle.rope3d_groups(128) == (22, 21, 21)
    assert oracle.rope3d_groups(112) == (20, 18, 18)
    assert oracle.rope3d_groups(6) == (1, 1, 1)
    assert oracle.rope3d_groups(2) == (1, 0, 0)
    for D in range(2, 258, 2):
        assert sum(oracle.rope3d_groups(D)) == D // 2


def test_rope_hand_examples():
    # D = 6: one pair per group, each turning by its position (base^0 = 1)
    ang = oracle.rope3d_angles(2, 2, 3, 6)                       # 2 frames of a 2 x 3 grid
    assert np.array_equal(ang[1, 2], [1.0, 0.0, 2.0])           # frame 1, row 0, column 2
    assert np.array_equal(ang[0, 4], [0.0, 1.0, 1.0])           # frame 0, row 1, column 1
    x = np.zeros((2, 6, 6))
    x[1, 2] = [1, 0, 1, 0, 1, 0]
    x[0, 3] = [0, 1, 0, 1, 0, 1]                                 # frame 0, row 1, column 0
    y = oracle.rope3d_apply(x, ang)
    c1, s1, c2, s2 = math.cos(1), math.sin(1), math.cos(2), math.sin(2)
    assert np.allclose(y[1, 2], [c1, s1, 1, 0, c2, s2], atol=1e-15)
    assert np.allclose(y[0, 3], [0, 1, -s1, c1, 0, 1], atol=1e-15)
    # D = 12: two pairs per group, frequencies base^0 and base^(-1/2)
    ang = oracle.rope3d_angles(4, 2, 5, 12, frame_offset=10, base=100.0)
    f, r, c = 3 + 10, 1, 4                                       # token 9 of frame 3
    assert np.allclose(ang[3, 9], [f, f / 10, r, r / 10, c, c / 10], rtol=1e-15)


def test_rope_is_a_rotation_of_each_pair():
    rng = np.random.default_rng(2)
    x = rng.standard_normal((3, 20, 16))
    ang = oracle.rope3d_angles(3, 4, 5, 16, frame_offset=5)
    y = oracle.rope3d_apply(x, ang)
    pair = lambda t: t[..., 0::2] ** 2 + t[..., 1::2] ** 2
    assert np.allclose(pair(y), pair(x), rtol=1e-13)
    # turning back by the same angles restores x; the origin token is untouched
    assert np.allclose(oracle.rope3d_apply(y, -ang), x, atol=1e-13)
    ang0 = oracle.rope3d_angles(3, 4, 5, 16)
    assert np.array_equal(oracle.rope3d_apply(x, ang0)[0, 0], x[0, 0])


def test_rope_dot_products_depend_on_relative_position_only():
    rng = np.random.default_rng(3)
    D = 24
    q, k = rng.standard_normal(D), rng.standard_normal(D)
    gh, gw = 4, 6
    ang_a = oracle.rope3d_angles(8, gh, gw, D, frame_offset=0)
    ang_b = oracle.rope3d_angles(8, gh, gw, D, frame_offset=13)

    def dot(ang, f1, s1, f2, s2):
        x = np.zeros((8, gh * gw, D))
        z = np.zeros((8, gh * gw, D))
        x[f1, s1], z[f2, s2] = q, k
        return oracle.rope3d_apply(x, ang)[f1, s1] @ oracle.rope3d_apply(z, ang)[f2, s2]

    tok = lambda r, c: r * gw + c
    ref = dot(ang_a, 5, tok(2, 3), 1, tok(0, 1))
    assert abs(dot(ang_b, 5, tok(2, 3), 1, tok(0, 1)) - ref) < 1e-12     # frame shift
    assert abs(dot(ang_a, 6, tok(3, 3), 2, tok(1, 1)) - ref) < 1e-12     # frame + row shift
    assert abs(dot(ang_a, 5, tok(2, 5), 1, tok(0, 3)) - ref) < 1e-12     # column shift
    assert abs(dot(ang_a, 5, tok(2, 4), 1, tok(0, 1)) - ref) > 1e-6      # a different offset


# ----------------------------------------------------------------------------
# Scans on prepared features
# ----------------------------------------------------------------------------
def test_golden_relu_rope_hand_example():
    d, arr = _golden("relu_rope_hand.json")
    gh, gw = d["grid"]
    o, m, z = oracle.relu_scan_prep(arr("q"), arr("k"), arr("v"), d["eps"], None, None,
                                    d["norm_eps"], gh, gw, base=d["base"])
    assert np.allclose(o[0, 0], _expr(d["expected_o"]), atol=1e-14)
    assert np.allclose(m[0, 0], _expr(d["expected_state"]), atol=1e-14)
    assert np.allclose(z[0, 0], _expr(d["expected_z"]), atol=1e-14)


def test_golden_gdn_rope_hand_example():
    d, arr = _golden("gdn_rope_hand.json")
    gh, gw = d["grid"]
    a = np.array(d["alpha"])[None, None]
    b = np.array(d["beta"])[None, None]
    o, m = oracle.gdn_scan_prep(arr("q"), arr("k"), arr("v"), a, b, d["k_scale"], None, None,
                                d["norm_eps"], gh, gw, base=d["base"])
    assert np.allclose(o[0, 0], _expr(d["expected_o"]), atol=1e-14)
    assert np.allclose(m[0, 0], _expr(d["expected_state"]), atol=1e-14)


def _inputs(seed, B=1, H=2, F=5, gh=3, gw=4, D=16):
    rng = np.random.default_rng(seed)
    S = gh * gw
    q, k, v = (rng.standard_normal((B, H, F, S, D)) for _ in range(3))
    a = rng.uniform(0.8, 1.0, (B, H, F))
    b = rng.uniform(0.0, 1.0, (B, H, F))
    wq, wk = rng.uniform(0.5, 1.5, (H, D)), rng.uniform(0.5, 1.5, (H, D))
    return q, k, v, a, b, wq, wk


def _temporal_rotation(D, delta, base=10000.0):
    """Key-side matrix of a uniform frame shift: x R^T turns every temporal
    pair of the row vector x by delta * base^(-i / n_t)."""
    n_t, _, _ = oracle.rope3d_groups(D)
    R = np.eye(D)
    for i in range(n_t):
        t = delta * base ** (-i / n_t)
        R[2 * i:2 * i + 2, 2 * i:2 * i + 2] = [[math.cos(t), -math.sin(t)],
                                               [math.sin(t), math.cos(t)]]
    return R


def test_gdn_prep_outputs_ignore_a_global_frame_shift():
    """q and k of every token turn by the same extra temporal angles, so the
    outputs Q~ M are unchanged and the state turns: M' = R M."""
    q, k, v, a, b, wq, wk = _inputs(4)
    D, S = 16, 12
    ks = 1 / math.sqrt(D * S)
    o0, m0 = oracle.gdn_scan_prep(q, k, v, a, b, ks, wq, wk, 1e-6, 3, 4, frame_offset=0)
    o1, m1 = oracle.gdn_scan_prep(q, k, v, a, b, ks, wq, wk, 1e-6, 3, 4, frame_offset=37)
    assert np.allclose(o1, o0, atol=1e-12 * np.abs(o0).max())
    R = _temporal_rotation(D, 37)
    for h in range(2):
        assert np.allclose(m1[0, h], R @ m0[0, h], atol=1e-12 * np.abs(m0).max())
        assert not np.allclose(m1[0, h], m0[0, h], atol=1e-3 * np.abs(m0).max())


def test_relu_prep_outputs_ignore_a_global_frame_shift():
    q, k, v, _, _, wq, wk = _inputs(5)
    o0, m0, z0 = oracle.relu_scan_prep(q, k, v, 1e-6, wq, wk, 1e-6, 3, 4, frame_offset=0)
    o1, m1, z1 = oracle.relu_scan_prep(q, k, v, 1e-6, wq, wk, 1e-6, 3, 4, frame_offset=11)
    assert np.allclose(o1, o0, atol=1e-12 * np.abs(o0).max())
    assert np.allclose(z1, z0, atol=1e-13)
    R = _temporal_rotation(16, 11)
    assert np.allclose(m1[0, 1], R @ m0[0, 1], atol=1e-12 * np.abs(m0).max())


def test_relu_prep_without_rope_is_the_relu_scan_of_normalised_inputs():
    q, k, v, _, _, wq, wk = _inputs(6)
    qn = np.stack([oracle.rms_norm(q[:, h], wq[h], 1e-6) for h in range(2)], axis=1)
    kn = np.stack([oracle.rms_norm(k[:, h], wk[h], 1e-6) for h in range(2)], axis=1)
    o_ref, m_ref, z_ref = oracle.relu_scan(qn, kn, v, 1e-6)
    o, m, z = oracle.relu_scan_prep(q, k, v, 1e-6, wq, wk, 1e-6, 3, 4, rope=False)
    assert np.allclose(o, o_ref, atol=1e-12) and np.allclose(m, m_ref, atol=1e-12)
    assert np.allclose(z, z_ref, atol=1e-12)


def test_prep_scans_ignore_the_scale_of_q_and_k():
    # RMSNorm removes a positive scale of every token (norm eps = 0)
    q, k, v, a, b, wq, wk = _inputs(7)
    ks = 1 / math.sqrt(16 * 12)
    o0, _ = oracle.gdn_scan_prep(q, k, v, a, b, ks, wq, wk, 0.0, 3, 4)
    o1, _ = oracle.gdn_scan_prep(4.0 * q, 0.3 * k, v, a, b, ks, wq, wk, 0.0, 3, 4)
    assert np.allclose(o1, o0, atol=1e-12 * np.abs(o0).max())
    r0 = oracle.relu_scan_prep(q, k, v, 1e-6, wq, wk, 0.0, 3, 4)[0]
    r1 = oracle.relu_scan_prep(2.5 * q, 0.1 * k, v, 1e-6, wq, wk, 0.0, 3, 4)[0]
    assert np.allclose(r1, r0, atol=1e-12 * np.abs(r0).max())


def test_prepared_keys_keep_the_spectral_bound():
    """RMSNorm (unit weight) bounds |k~|^2 by D; ReLU and the rotations only
    shrink or keep it; so with k_scale = 1/sqrt(D S) the frame gram has
    trace at most 1 and I - beta G is a contraction for beta in [0, 2]."""
    q, k, v, a, b, _, _ = _inputs(8, F=6, gh=4, gw=5, D=32)
    D, S = 32, 20
    kt, _ = oracle.prep_features(k, None, 1e-6, 4, 5, frame_offset=3)
    kh = kt / math.sqrt(D * S)
    for h in range(2):
        for f in range(6):
            G = kh[0, h, f].T @ kh[0, h, f]
            assert np.trace(G) <= 1.0 + 1e-12
            assert np.linalg.norm(np.eye(D) - 2.0 * G, 2) <= 1.0 + 1e-12


# ----------------------------------------------------------------------------
# Planted mistakes in copies of the oracle fail the pins
# ----------------------------------------------------------------------------
def _mutant(name):
    """A copy of the oracle module with one function replaced."""
    import importlib.util
    spec = importlib.util.spec_from_file_location("oracle_mutant", oracle.__file__)
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    if name == "half_split_pairs":        # pairs (i, i + D/2) instead of (2i, 2i + 1)
        def apply(x, angles):
            x = np.asarray(x, np.float64)
            P = x.shape[-1] // 2
            c, s = np.cos(angles), np.sin(angles)
            y = np.empty_like(x)
            y[..., :P] = x[..., :P] * c - x[..., P:] * s
            y[..., P:] = x[..., :P] * s + x[..., P:] * c
            return y
        mod.rope3d_apply = apply
    elif name == "reversed_turn":         # clockwise instead of counter-clockwise
        real = mod.rope3d_apply
        mod.rope3d_apply = lambda x, angles: real(x, -angles)
    elif name == "rope_in_normaliser":    # the normaliser reads rotated features
        real = mod.prep_features
        mod.prep_features = lambda *a, **kw: (real(*a, **kw)[0],) * 2
    elif name == "mean_abs_norm":         # mean |x| instead of the root mean square
        mod.rms_norm = lambda x, w=None, eps=1e-6: (
            np.asarray(x) / (np.mean(np.abs(x), axis=-1, keepdims=True) + eps)
            * (1 if w is None else w))
    elif name == "width_first":           # groups in the order width, height, time
        real = mod.rope3d_angles
        mod.rope3d_angles = lambda *a, **kw: real(*a, **kw)[..., ::-1]
    return mod


@pytest.mark.parametrize("name", ["half_split_pairs", "reversed_turn", "rope_in_normaliser",
                                  "mean_abs_norm", "width_first"])
def test_planted_mistakes_fail_the_pins(name, monkeypatch):
    mod = _mutant(name)
    failed = []
    for pin in (test_rope_hand_examples, test_golden_relu_rope_hand_example,
                test_golden_gdn_rope_hand_example, test_rms_norm_hand_example_and_closed_forms):
        with monkeypatch.context() as m:
            for fn in ("rope3d_apply", "rope3d_angles", "prep_features", "rms_norm"):
                m.setattr(oracle, fn, getattr(mod, fn))
            try:
                pin()
            except AssertionError:
                failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
