"""Pins for the CPU oracle: checks against what the pages and the mathematics
fix, computed by routes other than the oracle's own recurrence.

Each pin is chosen so that a plausible mistake in the oracle (a dropped term,
a wrong sign, a transposed operand, an off-by-one frame, exclusive instead of
inclusive causality, the key scale on the wrong operand) fails at least one
of them; ``test_pins_reject_planted_mistakes`` plants such mistakes in copies
of the oracle and shows the pins catch them.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rel(a, b):
    return float(np.max(np.abs(np.asarray(a) - np.asarray(b))) /
                 max(np.max(np.abs(np.asarray(b))), 1e-300))


def _inputs(spec):
    q = synth.full_values(spec, "q").astype(np.float64)
    k = synth.full_values(spec, "k").astype(np.float64)
    v = synth.full_values(spec, "v").astype(np.float64)
    a, bt = synth.gates(spec)
    return q, k, v, a.astype(np.float64), bt.astype(np.float64)


# ----------------------------------------------------------------------------
# Hand-worked fixtures (exact arithmetic)
# ----------------------------------------------------------------------------
def test_golden_gdn_hand_example():
    g = json.load(open(os.path.join(GOLDEN, "gdn_hand_2x2.json")))
    q = np.array(g["q"], float)[None, None]
    k = np.array(g["k"], float)[None, None]
    v = np.array(g["v"], float)[None, None]
    a = np.array(g["alpha"], float)[None, None]
    b = np.array(g["beta"], float)[None, None]
    o, m = oracle.gdn_scan(q, k, v, a, b, g["k_scale"])
    np.testing.assert_allclose(o[0, 0], np.array(g["expected_o"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(m[0, 0], np.array(g["expected_state"]), rtol=0, atol=1e-14)


def test_golden_relu_hand_example():
    g = json.load(open(os.path.join(GOLDEN, "relu_hand_2x2.json")))
    q = np.array(g["q"], float)[None, None]
    k = np.array(g["k"], float)[None, None]
    v = np.array(g["v"], float)[None, None]
    o, m, z = oracle.relu_scan(q, k, v, g["eps"])
    np.testing.assert_allclose(o[0, 0], np.array(g["expected_o"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(m[0, 0], np.array(g["expected_state"]), rtol=0, atol=1e-14)
    np.testing.assert_allclose(z[0, 0], np.array(g["expected_z"]), rtol=0, atol=1e-14)


# ----------------------------------------------------------------------------
# ReLU mode: explicit block-causal attention matrix (textbook linear attention)
# ----------------------------------------------------------------------------
def _relu_unrolled(q, k, v, eps, m0=None, z0=None):
    """O = (W V + phi(q) M0) / (W 1 + phi(q) z0 + eps), W[t,s] = phi(q_t).phi(k_s)
    for frame(s) <= frame(t), else 0.  Built as one explicit matrix per head."""
    B, H, F, S, D = k.shape
    out = np.zeros_like(q)
    fr = np.repeat(np.arange(F), S)
    mask = (fr[None, :] <= fr[:, None]).astype(float)      # [T, T], inclusive
    for b in range(B):
        for h in range(H):
            pq = np.maximum(q[b, h].reshape(F * S, D), 0)
            pk = np.maximum(k[b, h].reshape(F * S, D), 0)
            vv = v[b, h].reshape(F * S, D)
            W = (pq @ pk.T) * mask
            num = W @ vv
            den = W.sum(axis=1)
            if m0 is not None:
                num = num + pq @ m0[b, h]
                den = den + pq @ z0[b, h]
            out[b, h] = (num / (den + eps)[:, None]).reshape(F, S, D)
    return out


def test_relu_matches_unrolled_attention_tiny_config():
    spec = synth.workload("tiny_fp32")
    q, k, v, _, _ = _inputs(spec)
    o, _, _ = oracle.relu_scan(q, k, v, spec.eps)
    ref = _relu_unrolled(q, k, v, spec.eps)
    assert _rel(o, ref) < 1e-12


def test_relu_matches_unrolled_attention_with_state_in():
    spec = synth.small(B=2, H=1, F=3, S=5, D=4, dtype="f32", seed=11)
    q, k, v, _, _ = _inputs(spec)
    m0, z0 = synth.random_state(spec)
    o, m, z = oracle.relu_scan(q, k, v, 1e-6, m0, z0)
    ref = _relu_unrolled(q, k, v, 1e-6, m0.astype(float), z0.astype(float))
    assert _rel(o, ref) < 1e-12
    # final state: M0 + sum of all frames' phi(K)^T V, computed in one product
    for b in range(2):
        pk = np.maximum(k[b, 0].reshape(-1, 4), 0)
        np.testing.assert_allclose(m[b, 0], m0[b, 0] + pk.T @ v[b, 0].reshape(-1, 4),
                                   rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(z[b, 0], z0[b, 0] + pk.sum(0), rtol=1e-12, atol=1e-12)


def test_relu_output_is_convex_combination_of_visible_values():
    spec = synth.small(B=1, H=2, F=4, S=16, D=8, dtype="f32", seed=3)
    q, k, v, _, _ = _inputs(spec)
    with np.errstate(invalid="ignore"):          # rows with phi(q) = 0 give 0/0; skipped
        o, _, _ = oracle.relu_scan(q, k, v, 0.0)
    for h in range(2):
        for f in range(spec.F):
            vis = v[0, h, : f + 1].reshape(-1, spec.D)
            lo, hi = vis.min(0), vis.max(0)
            pq = np.maximum(q[0, h, f], 0)
            rows = pq.sum(1) > 0
            of = o[0, h, f][rows]
            assert np.all(of >= lo - 1e-12) and np.all(of <= hi + 1e-12)


def test_relu_block_causality_is_inclusive():
    spec = synth.small(B=1, H=1, F=4, S=6, D=4, dtype="f32", seed=5)
    q, k, v, _, _ = _inputs(spec)
    o, _, _ = oracle.relu_scan(q, k, v, 1e-6)
    k2, v2 = k.copy(), v.copy()
    k2[0, 0, 2] += 1.0
    v2[0, 0, 2] -= 2.0
    o2, _, _ = oracle.relu_scan(q, k2, v2, 1e-6)
    np.testing.assert_array_equal(o[0, 0, :2], o2[0, 0, :2])     # earlier frames blind
    assert np.max(np.abs(o[0, 0, 2] - o2[0, 0, 2])) > 1e-3       # frame sees itself
    assert np.max(np.abs(o[0, 0, 3] - o2[0, 0, 3])) > 1e-3       # later frames see it


# ----------------------------------------------------------------------------
# GDN mode: explicit unrolled product form
# ----------------------------------------------------------------------------
def _gdn_unrolled(q, k, v, alpha, beta, kappa, m0=None):
    """O_f = Q_f (A_f..A_1 M0 + sum_{j<=f} A_f..A_{j+1} B_j), with the block
    lower-triangular map assembled explicitly as an (F*S) x (F*S) matrix."""
    B, H, F, S, D = k.shape
    out = np.zeros_like(q)
    I = np.eye(D)
    for b in range(B):
        for h in range(H):
            A = [alpha[b, h, f] * (I - beta[b, h, f] * (kappa * k[b, h, f]).T @ (kappa * k[b, h, f]))
                 for f in range(F)]
            L = np.zeros((F * S, F * S))
            R = np.zeros((F * S, D))
            for f in range(F):
                phi = I.copy()                    # A_f ... A_{j+1}
                for j in range(f, -1, -1):
                    blk = q[b, h, f] @ phi @ (beta[b, h, j] * (kappa * k[b, h, j]).T)
                    L[f * S:(f + 1) * S, j * S:(j + 1) * S] = blk
                    phi = phi @ A[j]
                if m0 is not None:
                    R[f * S:(f + 1) * S] = q[b, h, f] @ phi @ m0[b, h]
            o = L @ v[b, h].reshape(F * S, D) + R
            out[b, h] = o.reshape(F, S, D)
    return out


def test_gdn_matches_unrolled_product_tiny_config():
    spec = synth.workload("tiny_fp32")
    q, k, v, a, bt = _inputs(spec)
    o, _ = oracle.gdn_scan(q, k, v, a, bt, spec.k_scale)
    ref = _gdn_unrolled(q, k, v, a, bt, spec.k_scale)
    assert _rel(o, ref) < 1e-12


def test_gdn_matches_unrolled_product_with_state_in():
    spec = synth.small(B=1, H=2, F=3, S=7, D=5, dtype="f32", seed=13)
    q, k, v, a, bt = _inputs(spec)
    m0, _ = synth.random_state(spec)
    o, _ = oracle.gdn_scan(q, k, v, a, bt, 0.4, m0)
    ref = _gdn_unrolled(q, k, v, a, bt, 0.4, m0.astype(float))
    assert _rel(o, ref) < 1e-12


# ----------------------------------------------------------------------------
# GDN closed forms
# ----------------------------------------------------------------------------
def test_gdn_alpha_zero_keeps_only_current_write():
    spec = synth.small(B=1, H=1, F=3, S=9, D=6, dtype="f32", seed=17)
    q, k, v, _, bt = _inputs(spec)
    m0, _ = synth.random_state(spec)
    a = np.zeros_like(bt)
    o, m = oracle.gdn_scan(q, k, v, a, bt, 0.3, m0)
    for f in range(spec.F):
        kh = 0.3 * k[0, 0, f]
        Mf = bt[0, 0, f] * kh.T @ v[0, 0, f]
        np.testing.assert_allclose(o[0, 0, f], q[0, 0, f] @ Mf, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(m[0, 0], Mf, rtol=1e-12, atol=1e-12)


def test_gdn_beta_zero_is_pure_decay():
    spec = synth.small(B=1, H=1, F=4, S=3, D=5, dtype="f32", seed=19)
    q, k, v, a, _ = _inputs(spec)
    m0, _ = synth.random_state(spec)
    bt = np.zeros_like(a)
    o, m = oracle.gdn_scan(q, k, v, a, bt, 0.7, m0)
    decay = 1.0
    for f in range(spec.F):
        decay *= a[0, 0, f]
        np.testing.assert_allclose(o[0, 0, f], q[0, 0, f] @ (decay * m0[0, 0]),
                                   rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(m[0, 0], decay * m0[0, 0], rtol=1e-12)


def test_gdn_scalar_recurrence_by_hand():
    # D = S = 1: m <- alpha (1 - beta kh^2) m + beta kh v ; o = q m ; kh = kappa k
    ks = [1.5, -0.5, 2.0, 0.25]
    vs = [2.0, 1.0, -3.0, 0.5]
    qs = [1.0, -2.0, 0.5, 3.0]
    al = [0.9, 0.5, 1.0, 0.75]
    be = [0.2, 1.0, 0.5, 0.4]
    kappa, m = 0.5, 1.25
    expect = []
    for f in range(4):
        kh = kappa * ks[f]
        m = al[f] * (1.0 - be[f] * kh * kh) * m + be[f] * kh * vs[f]
        expect.append(qs[f] * m)
    arr = lambda x: np.array(x, float).reshape(1, 1, 4, 1, 1)
    o, mf = oracle.gdn_scan(arr(qs), arr(ks), arr(vs), np.array(al).reshape(1, 1, 4),
                            np.array(be).reshape(1, 1, 4), kappa,
                            np.array([[[[1.25]]]]))
    np.testing.assert_allclose(o.ravel(), expect, rtol=1e-15)
    assert abs(mf.item() - m) < 1e-15


@pytest.mark.parametrize("alpha,beta", [(1.0, 1.0), (0.8, 1.0), (1.0, 0.3), (0.6, 0.7)])
def test_gdn_delta_rule_retrieval_with_orthonormal_keys(alpha, beta):
    # With orthonormal scaled keys (Kh Kh^T = I), querying the new state with
    # the frame's own keys gives Kh M_f = alpha (1 - beta) Kh M_{f-1} + beta V_f.
    # At alpha = beta = 1 the delta rule writes V exactly.
    rng = np.random.default_rng(0)
    S, D, kappa = 5, 8, 0.25
    Qo, _ = np.linalg.qr(rng.standard_normal((D, D)))
    kh = Qo[:S]                                   # orthonormal rows
    k = (kh / kappa)[None, None, None]
    v = rng.standard_normal((1, 1, 1, S, D))
    m0 = rng.standard_normal((1, 1, D, D))
    q = kh[None, None, None]
    o, _ = oracle.gdn_scan(q, k, v, np.full((1, 1, 1), alpha), np.full((1, 1, 1), beta),
                           kappa, m0)
    expect = alpha * (1 - beta) * kh @ m0[0, 0] + beta * v[0, 0, 0]
    np.testing.assert_allclose(o[0, 0, 0], expect, rtol=1e-12, atol=1e-12)


# ----------------------------------------------------------------------------
# Additive limit: GDN with alpha = 1, beta = delta, V / delta -> linear-attention cumsum
# ----------------------------------------------------------------------------
def test_gdn_additive_limit_is_linear_attention_cumsum():
    spec = synth.workload("tiny_fp32")
    q, k, v, _, _ = _inputs(spec)
    q, k, v = q[:, :1], k[:, :1], v[:, :1]
    kap = spec.k_scale
    F, S, D = spec.F, spec.S, spec.D
    ref = np.zeros((F, S, D))
    for f in range(F):                       # identity feature map, no normaliser
        acc = np.zeros((S, D))
        for j in range(f + 1):
            acc += (q[0, 0, f] @ (kap * k[0, 0, j]).T) @ v[0, 0, j]
        ref[f] = acc
    errs = []
    for delta in (1e-3, 1e-5, 1e-7):
        a = np.ones((1, 1, F))
        b = np.full((1, 1, F), delta)
        o, _ = oracle.gdn_scan(q, k, v / delta, a, b, kap)
        errs.append(_rel(o[0, 0], ref))
    assert errs[0] < 1e-2
    assert 30 < errs[0] / errs[1] < 300       # error falls in proportion to delta
    assert 30 < errs[1] / errs[2] < 300
    assert errs[2] < 1e-6


# ----------------------------------------------------------------------------
# Key scaling: spectral bound of the transition, contraction of the scan
# ----------------------------------------------------------------------------
@pytest.mark.parametrize("cfg", [0, "c2_like"])
def test_key_scaling_bounds_transition_norm(cfg):
    if cfg == "c2_like":
        spec = synth.workload("gdn_720p_60s").with_(B=1, H=2, F=6)   # same shape and recipe, fewer frames
    else:
        spec = synth.workload("tiny_fp32")
    k = synth.full_values(spec, "k").astype(np.float64)
    _, bt = synth.gates(spec)
    kap = spec.k_scale
    D = spec.D
    for h in range(spec.H):
        for f in range(spec.F):
            kh = kap * k[0, h, f]
            lam = np.linalg.eigvalsh(kh.T @ kh)
            assert lam.min() > -1e-12
            assert bt[0, h, f] * lam.max() <= 2.0
            A = np.eye(D) - bt[0, h, f] * kh.T @ kh
            assert np.linalg.norm(A, 2) <= 1.0 + 1e-12
            if spec.keys_l2:
                # unit-norm keys: lambda_max <= trace = S * kappa^2 * |k|^2 ~ 1/D
                assert lam.max() <= 1.0 / D * (1 + 1e-2)


def test_gdn_scan_is_a_contraction_in_the_initial_state():
    spec = synth.workload("tiny_fp32")
    q, k, v, a, bt = _inputs(spec)
    m0, _ = synth.random_state(spec)
    m1 = m0 + synth.random_state(spec.with_(seed=99))[0]
    _, ma = oracle.gdn_scan(q, k, v, a, bt, spec.k_scale, m0)
    _, mb = oracle.gdn_scan(q, k, v, a, bt, spec.k_scale, m1)
    for h in range(spec.H):
        bound = np.prod(a[0, h]) * np.linalg.norm((m1 - m0)[0, h].astype(float), 2)
        assert np.linalg.norm(ma[0, h] - mb[0, h], 2) <= bound * (1 + 1e-12)
        # and the gap is not trivially zero: the state really carries over
        assert np.linalg.norm(ma[0, h] - mb[0, h], 2) > 1e-3 * bound


# ----------------------------------------------------------------------------
# Chunked vs whole, and the composite route of context-parallel training
# ----------------------------------------------------------------------------
def test_chunked_equals_whole_bitwise():
    spec = synth.workload("tiny_fp32")
    q, k, v, a, bt = _inputs(spec)
    o, m = oracle.gdn_scan(q, k, v, a, bt, spec.k_scale)
    o1, m1 = oracle.gdn_scan(q[:, :, :3], k[:, :, :3], v[:, :, :3], a[:, :, :3], bt[:, :, :3],
                             spec.k_scale)
    o2, m2 = oracle.gdn_scan(q[:, :, 3:], k[:, :, 3:], v[:, :, 3:], a[:, :, 3:], bt[:, :, 3:],
                             spec.k_scale, m1)
    np.testing.assert_array_equal(np.concatenate([o1, o2], axis=2), o)
    np.testing.assert_array_equal(m2, m)
    r, rm, rz = oracle.relu_scan(q, k, v, spec.eps)
    r1, rm1, rz1 = oracle.relu_scan(q[:, :, :5], k[:, :, :5], v[:, :, :5], spec.eps)
    r2, rm2, rz2 = oracle.relu_scan(q[:, :, 5:], k[:, :, 5:], v[:, :, 5:], spec.eps, rm1, rz1)
    np.testing.assert_array_equal(np.concatenate([r1, r2], axis=2), r)
    np.testing.assert_array_equal(rm2, rm)
    np.testing.assert_array_equal(rz2, rz)


def test_state_step_matches_scan_state():
    spec = synth.workload("tiny_fp32")
    q, k, v, a, bt = _inputs(spec)
    m0, z0 = synth.random_state(spec)
    _, m = oracle.gdn_scan(q, k, v, a, bt, spec.k_scale, m0)
    np.testing.assert_array_equal(oracle.gdn_state_step(k, v, a, bt, spec.k_scale, m0), m)
    _, rm, rz = oracle.relu_scan(q, k, v, spec.eps, m0, z0)
    sm, sz = oracle.relu_state_step(k, v, m0, z0)
    np.testing.assert_array_equal(sm, rm)
    np.testing.assert_array_equal(sz, rz)


def test_composite_exclusive_prefix_recovers_interval_states():
    spec = synth.workload("tiny_fp32")
    q, k, v, a, bt = _inputs(spec)
    m0, _ = synth.random_state(spec)
    cuts = [0, 2, 3, 6, 8]
    for h in range(spec.H):
        comps = [oracle.gdn_interval_composite(k[0, h, s:e], v[0, h, s:e], a[0, h, s:e],
                                               bt[0, h, s:e], spec.k_scale)
                 for s, e in zip(cuts[:-1], cuts[1:])]
        starts = oracle.compose_exclusive_prefix(comps, m0[0, h])
        for (s, e), st in zip(zip(cuts[:-1], cuts[1:]), starts):
            _, ms = oracle.gdn_scan(q[:, h:h + 1, :s], k[:, h:h + 1, :s], v[:, h:h + 1, :s],
                                    a[:, h:h + 1, :s], bt[:, h:h + 1, :s], spec.k_scale,
                                    m0[:, h:h + 1])
            assert _rel(st, ms[0, 0]) < 1e-12
        # the last interval's end state from the composites equals the full scan
        T, U = comps[-1]
        _, mf = oracle.gdn_scan(q[:, h:h + 1], k[:, h:h + 1], v[:, h:h + 1], a[:, h:h + 1],
                                bt[:, h:h + 1], spec.k_scale, m0[:, h:h + 1])
        assert _rel(T @ starts[-1] + U, mf[0, 0]) < 1e-12


# ----------------------------------------------------------------------------
# The pins are sharp: planted mistakes in copies of the oracle are caught
# ----------------------------------------------------------------------------
def _gdn_mutant(kind):
    def scan(q, k, v, alpha, beta, kappa, m0=None):
        B, H, F, S, D = k.shape
        o = np.zeros_like(q, dtype=float)
        for b in range(B):
            for h in range(H):
                M = np.zeros((D, D)) if m0 is None else np.array(m0[b, h], float)
                for f in range(F):
                    a, bt = alpha[b, h, f], beta[b, h, f]
                    kh = kappa * k[b, h, f]
                    if kind == "erase_sign":
                        Mn = a * (M + bt * kh.T @ (kh @ M)) + bt * kh.T @ v[b, h, f]
                    elif kind == "alpha_on_write":
                        Mn = a * (M - bt * kh.T @ (kh @ M) + bt * kh.T @ v[b, h, f])
                    elif kind == "exclusive":
                        Mn = None
                    elif kind == "kappa_on_q":
                        Mn = a * (M - bt * kh.T @ (kh @ M)) + bt * kh.T @ v[b, h, f]
                    elif kind == "transposed_write":
                        Mn = a * (M - bt * kh.T @ (kh @ M)) + bt * (v[b, h, f].T @ kh)
                    elif kind == "gate_off_by_one":
                        fa = max(f - 1, 0)
                        Mn = alpha[b, h, fa] * (M - beta[b, h, fa] * kh.T @ (kh @ M)) + \
                            beta[b, h, fa] * kh.T @ v[b, h, f]
                    if kind == "exclusive":
                        o[b, h, f] = q[b, h, f] @ M
                        M = a * (M - bt * kh.T @ (kh @ M)) + bt * kh.T @ v[b, h, f]
                    else:
                        M = Mn
                        qq = kappa * q[b, h, f] if kind == "kappa_on_q" else q[b, h, f]
                        o[b, h, f] = qq @ M
        return o
    return scan


def _gdn_pins_pass(scan):
    """Run a subset of the GDN pins against a candidate scan; True if all pass."""
    try:
        g = json.load(open(os.path.join(GOLDEN, "gdn_hand_2x2.json")))
        arr = lambda x: np.array(x, float)[None, None]
        o = scan(arr(g["q"]), arr(g["k"]), arr(g["v"]), arr(g["alpha"]), arr(g["beta"]),
                 g["k_scale"])
        if np.max(np.abs(o[0, 0] - np.array(g["expected_o"]))) > 1e-12:
            return False
        spec = synth.workload("tiny_fp32")
        q, k, v, a, bt = _inputs(spec)
        o = scan(q, k, v, a, bt, spec.k_scale)
        if _rel(o, _gdn_unrolled(q, k, v, a, bt, spec.k_scale)) > 1e-12:
            return False
        return True
    except Exception:
        return False


@pytest.mark.parametrize("kind", ["erase_sign", "alpha_on_write", "exclusive", "kappa_on_q",
                                  "transposed_write", "gate_off_by_one"])
def test_pins_reject_planted_mistakes(kind):
    assert _gdn_pins_pass(lambda *a: oracle.gdn_scan(*a)[0])
    assert not _gdn_pins_pass(_gdn_mutant(kind))


# ----------------------------------------------------------------------------
# Reversed GDN scan, reset at chunk boundaries
# ----------------------------------------------------------------------------
def _gdn_reverse_unrolled(q, k, v, alpha, beta, kappa, C):
    """O_f = Q_f sum_{j = f .. e} A_f A_{f+1} .. A_{j-1} B_j within each chunk
    (e = the chunk's last frame), assembled as an explicit block
    upper-triangular (F*S) x (F*S) matrix per head."""
    B, H, F, S, D = k.shape
    out = np.zeros_like(q)
    I = np.eye(D)
    for b in range(B):
        for h in range(H):
            A = [alpha[b, h, f] * (I - beta[b, h, f] * (kappa * k[b, h, f]).T @ (kappa * k[b, h, f]))
                 for f in range(F)]
            L = np.zeros((F * S, F * S))
            for f in range(F):
                e = min((f // C + 1) * C, F) - 1
                phi = I.copy()                    # A_f ... A_{j-1}
                for j in range(f, e + 1):
                    L[f * S:(f + 1) * S, j * S:(j + 1) * S] = \
                        q[b, h, f] @ phi @ (beta[b, h, j] * (kappa * k[b, h, j]).T)
                    phi = phi @ A[j]
            out[b, h] = (L @ v[b, h].reshape(F * S, D)).reshape(F, S, D)
    return out


def _rev_inputs():
    spec = synth.small(B=1, H=2, F=7, S=6, D=5, dtype="f32", seed=17)
    return spec, _inputs(spec)


@pytest.mark.parametrize("C", [1, 2, 3, 7, 10])
def test_reverse_matches_unrolled_product(C):
    spec, (q, k, v, a, bt) = _rev_inputs()
    o = oracle.gdn_scan_reverse_chunked(q, k, v, a, bt, 0.35, C)
    assert _rel(o, _gdn_reverse_unrolled(q, k, v, a, bt, 0.35, C)) < 1e-12


def test_reverse_one_frame_chunks_are_single_writes():
    spec, (q, k, v, a, bt) = _rev_inputs()
    o = oracle.gdn_scan_reverse_chunked(q, k, v, a, bt, 0.35, 1)
    for f in range(spec.F):
        kh = 0.35 * k[0, 1, f]
        np.testing.assert_allclose(o[0, 1, f], q[0, 1, f] @ (bt[0, 1, f] * kh.T @ v[0, 1, f]),
                                   rtol=1e-12, atol=1e-12)


def test_reverse_does_not_leak_across_chunks():
    spec, (q, k, v, a, bt) = _rev_inputs()
    C = 3                                  # chunks {0,1,2} {3,4,5} {6}
    o = oracle.gdn_scan_reverse_chunked(q, k, v, a, bt, 0.35, C)
    for f_pert, inside in ((1, range(0, 3)), (4, range(3, 6)), (6, range(6, 7))):
        k2, v2, q2 = k.copy(), v.copy(), q.copy()
        k2[:, :, f_pert] += 0.7
        v2[:, :, f_pert] -= 1.3
        q2[:, :, f_pert] *= 2.0
        o2 = oracle.gdn_scan_reverse_chunked(q2, k2, v2, a, bt, 0.35, C)
        outside = [f for f in range(spec.F) if f not in inside]
        np.testing.assert_array_equal(o[:, :, outside], o2[:, :, outside])
        # within the chunk: frames up to the perturbed one see it, later ones do not
        later = [f for f in inside if f > f_pert]
        np.testing.assert_array_equal(o[:, :, later], o2[:, :, later])
        for f in inside:
            if f <= f_pert:
                assert np.max(np.abs(o[:, :, f] - o2[:, :, f])) > 1e-6


def test_reverse_of_whole_clip_is_forward_scan_of_reversed_frames():
    spec, (q, k, v, a, bt) = _rev_inputs()
    o = oracle.gdn_scan_reverse_chunked(q, k, v, a, bt, 0.35, spec.F)
    rev = lambda x: x[:, :, ::-1].copy()
    of, _ = oracle.gdn_scan(rev(q), rev(k), rev(v), rev(a), rev(bt), 0.35)
    assert _rel(o, rev(of)) < 1e-12


def _reverse_mutant(kind):
    def scan(q, k, v, alpha, beta, kappa, C):
        B, H, F, S, D = k.shape
        o = np.zeros_like(q, dtype=float)
        for b in range(B):
            for h in range(H):
                M = np.zeros((D, D))
                for start in range(0, F, C):
                    end = min(start + C, F)
                    if kind != "no_reset":
                        M = np.zeros((D, D))
                    frames = range(start, end) if kind == "forward_in_chunk" else \
                        range(end - 1, start - 1, -1)
                    for f in frames:
                        a, bt = alpha[b, h, f], beta[b, h, f]
                        kh = kappa * k[b, h, f]
                        if kind == "exclusive":
                            o[b, h, f] = q[b, h, f] @ M
                        M = a * (M - bt * kh.T @ (kh @ M)) + bt * kh.T @ v[b, h, f]
                        if kind != "exclusive":
                            o[b, h, f] = q[b, h, f] @ M
        return o
    return scan


@pytest.mark.parametrize("kind", ["no_reset", "forward_in_chunk", "exclusive"])
def test_reverse_pins_reject_planted_mistakes(kind):
    spec, (q, k, v, a, bt) = _rev_inputs()
    ref = _gdn_reverse_unrolled(q, k, v, a, bt, 0.35, 3)
    assert _rel(oracle.gdn_scan_reverse_chunked(q, k, v, a, bt, 0.35, 3), ref) < 1e-12
    assert _rel(_reverse_mutant(kind)(q, k, v, a, bt, 0.35, 3), ref) > 1e-3


# ----------------------------------------------------------------------------
# Per-token update gate
# ----------------------------------------------------------------------------
def _tok_inputs():
    spec = synth.small(B=1, H=2, F=4, S=6, D=5, dtype="f32", seed=19)
    q, k, v, a, _ = _inputs(spec)
    bt = synth.token_gates(spec).astype(np.float64)
    return spec, q, k, v, a, bt


def _gdn_token_unrolled(q, k, v, alpha, bt, kappa, m0):
    """O_f = Q_f (A_f..A_1 M0 + sum_j A_f..A_{j+1} B_j) with the explicit
    A_f = alpha_f (I - Kh^T diag(beta_f) Kh) and B_j = Kh^T diag(beta_j) V_j."""
    B, H, F, S, D = k.shape
    out = np.zeros_like(q)
    I = np.eye(D)
    for b in range(B):
        for h in range(H):
            kh = [kappa * k[b, h, f] for f in range(F)]
            A = [alpha[b, h, f] * (I - kh[f].T @ np.diag(bt[b, h, f]) @ kh[f]) for f in range(F)]
            Bm = [kh[f].T @ np.diag(bt[b, h, f]) @ v[b, h, f] for f in range(F)]
            for f in range(F):
                M = m0[b, h].copy()
                for j in range(f + 1):
                    M = A[j] @ M + Bm[j]
                out[b, h, f] = q[b, h, f] @ M
    return out


def test_token_gate_matches_unrolled_product():
    spec, q, k, v, a, bt = _tok_inputs()
    m0, _ = synth.random_state(spec)
    o, _ = oracle.gdn_scan_token_beta(q, k, v, a, bt, 0.3, m0)
    assert _rel(o, _gdn_token_unrolled(q, k, v, a, bt, 0.3, m0.astype(float))) < 1e-12


def test_token_gate_constant_over_tokens_is_the_frame_gate():
    spec, q, k, v, a, bt = _tok_inputs()
    _, _, _, _, bf = _inputs(spec)
    btok = np.repeat(bf[..., None], spec.S, axis=-1)
    o, m = oracle.gdn_scan_token_beta(q, k, v, a, btok, 0.3)
    of, mf = oracle.gdn_scan(q, k, v, a, bf, 0.3)
    assert _rel(o, of) < 1e-12 and _rel(m, mf) < 1e-12


def test_token_gate_zero_removes_the_token():
    """A token with beta = 0 neither erases nor writes: the scan equals the
    per-frame-gate scan of the frame without that token."""
    spec, q, k, v, a, _ = _tok_inputs()
    btok = np.full((spec.B, spec.H, spec.F, spec.S), 0.6)
    btok[..., 2] = 0.0
    o, m = oracle.gdn_scan_token_beta(q, k, v, a, btok, 0.3)
    keep = [t for t in range(spec.S) if t != 2]
    _, mf = oracle.gdn_scan(q[..., keep, :], k[..., keep, :], v[..., keep, :], a,
                            np.full((spec.B, spec.H, spec.F), 0.6), 0.3)
    assert _rel(m, mf) < 1e-12


@pytest.mark.parametrize("kind", ["write_only", "squared", "erase_only"])
def test_token_gate_pins_reject_planted_mistakes(kind):
    spec, q, k, v, a, bt = _tok_inputs()
    m0, _ = synth.random_state(spec)
    ref = _gdn_token_unrolled(q, k, v, a, bt, 0.3, m0.astype(float))
    B, H, F, S, D = k.shape
    o = np.zeros_like(q)
    for b in range(B):
        for h in range(H):
            M = m0[b, h].astype(float)
            for f in range(F):
                w = bt[b, h, f][:, None]
                kh = 0.3 * k[b, h, f]
                ew = {"write_only": 1.0, "squared": w * w, "erase_only": w}[kind]
                ww = {"write_only": w, "squared": w * w, "erase_only": 1.0}[kind]
                M = a[b, h, f] * (M - kh.T @ (ew * (kh @ M))) + kh.T @ (ww * v[b, h, f])
                o[b, h, f] = q[b, h, f] @ M
    assert _rel(o, ref) > 1e-3


# ----------------------------------------------------------------------------
# Hand-worked fixtures of the reversed scan and the per-token gate
# ----------------------------------------------------------------------------
def test_golden_token_gate_hand_example():
    g = json.load(open(os.path.join(GOLDEN, "gdn_token_gate_hand_2x2.json")))
    arr = lambda x: np.array(x, float)[None, None]
    o, m = oracle.gdn_scan_token_beta(arr(g["q"]), arr(g["k"]), arr(g["v"]), arr(g["alpha"]),
                                      arr(g["beta_token"]), g["k_scale"])
    np.testing.assert_allclose(o[0, 0], np.array(g["expected_o"], float), rtol=0, atol=1e-12)
    np.testing.assert_allclose(m[0, 0], np.array(g["expected_state"], float), rtol=0, atol=1e-12)


@pytest.mark.parametrize("chunk", [1, 2])
def test_golden_reverse_hand_example(chunk):
    g = json.load(open(os.path.join(GOLDEN, "gdn_reverse_hand_2x2.json")))
    arr = lambda x: np.array(x, float)[None, None]
    o = oracle.gdn_scan_reverse_chunked(arr(g["q"]), arr(g["k"]), arr(g["v"]), arr(g["alpha"]),
                                        arr(g["beta"]), g["k_scale"], chunk)
    np.testing.assert_allclose(o[0, 0], np.array(g[f"expected_o_chunk{chunk}"], float),
                               rtol=0, atol=1e-12)
