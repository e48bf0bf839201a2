"""The seeded input generator: determinism, rounding and workload recipes."""
import math

import numpy as np
import pytest
import torch

import synth


def test_bf16_rounding_matches_torch_round_to_nearest_even():
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(100000).astype(np.float32) * 10,
        np.array([0.0, -0.0, 1.0, -1.0, 1.00390625, 1.01171875, 3.0e38, -3.0e38,
                  1e-40, 65504.0], np.float32),
        # exact ties between two bf16 neighbours: both round-to-even directions
        (np.array([0x3F808000, 0x3F818000, 0xBF808000, 0xBF818000], np.uint32)
         .view(np.float32)),
    ])
    ours = synth.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    back = synth.bf16_bits_to_f32(ours)
    np.testing.assert_array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_slices_are_regenerable_and_deterministic():
    spec = synth.small(B=2, H=3, F=2, S=5, D=16, dtype="bf16", seed=4)
    full = synth.full_storage(spec, "k")
    assert full.dtype == np.uint16 and full.shape == (2, 3, 2, 5, 16)
    for b in range(2):
        for h in range(3):
            np.testing.assert_array_equal(full[b, h], synth.slice_storage(spec, "k", b, h))
    np.testing.assert_array_equal(full, synth.full_storage(spec, "k"))
    assert not np.array_equal(synth.full_storage(spec, "q"), full)


def test_fp32_config_is_plain_normal():
    spec = synth.workload("tiny_fp32")
    q = synth.full_storage(spec, "q")
    assert q.dtype == np.float32 and q.shape == (1, 2, 8, 64, 32)
    assert abs(q.mean()) < 0.05 and abs(q.std() - 1) < 0.05
    a, b = synth.gates(spec)
    assert a.shape == (1, 2, 8) and a.dtype == np.float32
    assert a.min() >= 0.9 and a.max() <= 1.0 and b.min() >= 0.0 and b.max() <= 1.0
    assert spec.k_scale == np.float32(1 / math.sqrt(32 * 64))


def test_l2_normalised_keys_recipe():
    spec = synth.workload("gdn_720p_60s").with_(H=1, F=3)
    k = synth.slice_values(spec, "k", 0, 0).astype(np.float64)
    n = np.linalg.norm(k, axis=-1)
    assert np.all(np.abs(n - 1) < 4e-3)          # unit norm up to bf16 rounding
    a, b = synth.gates(spec)
    # alpha = sigmoid(N(3,1)): median near sigmoid(3) = 0.9526
    assert 0.5 < a.min() and a.max() < 1.0


def test_outlier_tokens_recipe():
    spec = synth.workload("stress_d256").with_(F=4, S=256, D=32, H=2)
    rows = synth.outlier_rows(spec, 0)
    assert rows.size == round(0.01 * 4 * 256) and len(np.unique(rows)) == rows.size
    q0 = synth.slice_values(spec, "q", 0, 0).reshape(-1, 32)
    big = np.abs(q0[rows]).mean()
    rest = np.abs(np.delete(q0, rows, axis=0)).mean()
    assert 15 < big / rest < 25
    # the same positions are outliers in every head and in k and v
    k1 = synth.slice_values(spec, "k", 0, 1).reshape(-1, 32)
    assert np.abs(k1[rows]).mean() / np.abs(np.delete(k1, rows, axis=0)).mean() > 15


def test_config_table_shapes():
    assert [synth.workload(n).D for n in synth.WORKLOAD_NAMES] == [32, 112, 128, 128, 128, 256]
    for n in synth.WORKLOAD_NAMES:
        spec = synth.workload(n)
        assert spec.grid is None or spec.grid[0] * spec.grid[1] == spec.S, n
    raw, l2 = synth.workload("gdn_720p_60s_raw"), synth.workload("gdn_720p_60s")
    assert raw.with_(name=l2.name, keys_l2=True) == l2     # the same clip, raw keys
    assert synth.workload("relu_480p").S == 30 * 52 and synth.workload("gdn_720p_60s").S == 22 * 40
    assert synth.workload("gdn_stream").chunk_frames * 8 == synth.workload("gdn_stream").F


def test_token_gates_are_seeded_per_workload_and_follow_the_beta_recipe():
    spec = synth.small(B=1, H=2, F=3, S=50, D=32, seed=5, beta=("sigmoid_normal", 0.0, 1.0))
    a = synth.token_gates(spec)
    assert a.shape == (1, 2, 3, 50) and a.dtype == np.float32
    np.testing.assert_array_equal(a, synth.token_gates(spec))            # reproducible
    assert not np.array_equal(a, synth.token_gates(spec.with_(seed=6)))  # seed matters
    assert (a > 0).all() and (a < 1).all()                              # sigmoid of a normal
    # independent of the per-frame gates drawn for the same workload
    _, bt = synth.gates(spec)
    assert not np.allclose(a[..., 0], bt)
