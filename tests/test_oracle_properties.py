"""Property checks of the oracle on random tiny shapes (hypothesis): every
scan agrees with its independent brute-force product form, for any shape,
gates, key scale and chunking."""
import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

import oracle
from test_oracle_pins import (_gdn_reverse_unrolled, _gdn_token_unrolled, _gdn_unrolled, _rel)

shapes = st.tuples(st.integers(1, 2), st.integers(1, 2), st.integers(1, 5),
                   st.integers(1, 5), st.integers(1, 4))


def _draw(seed, B, H, F, S, D):
    r = np.random.default_rng(seed)
    q, k, v = (r.standard_normal((B, H, F, S, D)) for _ in range(3))
    a = r.uniform(0.0, 1.0, (B, H, F))
    bt = r.uniform(0.0, 1.0, (B, H, F))
    return q, k, v, a, bt, r


@settings(max_examples=25, deadline=None)
@given(shape=shapes, seed=st.integers(0, 2**31 - 1), kappa=st.floats(0.05, 1.0))
def test_forward_scan_equals_product_form(shape, seed, kappa):
    q, k, v, a, bt, r = _draw(seed, *shape)
    m0 = r.standard_normal((shape[0], shape[1], shape[4], shape[4]))
    o, _ = oracle.gdn_scan(q, k, v, a, bt, kappa, m0)
    assert _rel(o, _gdn_unrolled(q, k, v, a, bt, kappa, m0)) < 1e-10


@settings(max_examples=25, deadline=None)
@given(shape=shapes, seed=st.integers(0, 2**31 - 1), kappa=st.floats(0.05, 1.0),
       chunk=st.integers(1, 6))
def test_reversed_scan_equals_product_form(shape, seed, kappa, chunk):
    q, k, v, a, bt, _ = _draw(seed, *shape)
    o = oracle.gdn_scan_reverse_chunked(q, k, v, a, bt, kappa, chunk)
    assert _rel(o, _gdn_reverse_unrolled(q, k, v, a, bt, kappa, chunk)) < 1e-10


@settings(max_examples=25, deadline=None)
@given(shape=shapes, seed=st.integers(0, 2**31 - 1), kappa=st.floats(0.05, 1.0))
def test_token_gate_scan_equals_product_form(shape, seed, kappa):
    B, H, F, S, D = shape
    q, k, v, a, _, r = _draw(seed, *shape)
    btok = r.uniform(0.0, 1.0, (B, H, F, S))
    m0 = r.standard_normal((B, H, D, D))
    o, _ = oracle.gdn_scan_token_beta(q, k, v, a, btok, kappa, m0)
    assert _rel(o, _gdn_token_unrolled(q, k, v, a, btok, kappa, m0)) < 1e-10


@settings(max_examples=25, deadline=None)
@given(shape=shapes, seed=st.integers(0, 2**31 - 1), split=st.integers(0, 5))
def test_chunked_relu_scan_equals_whole(shape, seed, split):
    """Carrying (M, z) across any split point gives the whole-clip result."""
    B, H, F, S, D = shape
    q, k, v, _, _, _ = _draw(seed, *shape)
    c = min(split, F)
    o, m, z = oracle.relu_scan(q, k, v, 1e-6)
    o1, m1, z1 = oracle.relu_scan(q[:, :, :c], k[:, :, :c], v[:, :, :c], 1e-6)
    o2, m2, z2 = oracle.relu_scan(q[:, :, c:], k[:, :, c:], v[:, :, c:], 1e-6, m1, z1)
    np.testing.assert_array_equal(np.concatenate([o1, o2], axis=2), o)
    np.testing.assert_array_equal(m2, m)
    np.testing.assert_array_equal(z2, z)
