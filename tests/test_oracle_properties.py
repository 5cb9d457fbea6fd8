"""Property-based pins of the oracle (hypothesis, CPU): invariants that must
hold for every shape and value, checked on many small random cases.

* RoPE: q'.k' depends only on the position difference, for any head
  dimension and base; it is a rotation (norms of the pairs kept).
* Eq(2): the offset of the new row equals numpy's C-order offset for any
  region shape, and appending writes exactly that row.
* Attention: adding the same value to every score changes nothing (a key
  whose dot product with q is constant: K rows shifted along q); the output is
  a convex combination of the V rows (inside their per-column range).
* int8 format: weights already on the grid come back exactly, for any group
  count, scale exponent and sign pattern.
* Packing: a pure permutation of rows for any I and T (pack then unpack is the
  identity, and every row appears once)."""

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

import oracle
import oracle.attn as oa

FAST = settings(max_examples=40, deadline=None)


@FAST
@given(half=st.integers(1, 16), theta=st.floats(2.0, 1e6), m=st.integers(0, 5000),
       n=st.integers(0, 5000), shift=st.integers(0, 3000), seed=st.integers(0, 2**31 - 1))
def test_rope_relative_position(half, theta, m, n, shift, seed):
    rng = np.random.default_rng(seed)
    d = 2 * half
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    a = oa.rope(q, m, theta) @ oa.rope(k, n, theta)
    b = oa.rope(q, m + shift, theta) @ oa.rope(k, n + shift, theta)
    assert abs(a - b) <= 1e-9 * (1 + np.abs(q).sum() * np.abs(k).sum())
    y = oa.rope(q, m, theta)
    assert np.allclose(y[:half] ** 2 + y[half:] ** 2, q[:half] ** 2 + q[half:] ** 2,
                       rtol=1e-12, atol=1e-12)


@FAST
@given(H=st.integers(1, 6), n_p=st.integers(0, 300), n_r=st.integers(1, 40),
       d=st.integers(1, 64))
def test_gkvc_step_and_append(H, n_p, n_r, d):
    for h in range(H):
        assert oa.gkvc_step(h, n_p, n_r, d) == np.ravel_multi_index((h, n_p, 0), (H, n_p + n_r, d))
    cache = np.arange(H * (n_p + n_r) * d, dtype=np.float64).reshape(H, n_p + n_r, d)
    row = -np.ones((H, d))
    new = oa.kv_append(cache, row, n_p)
    changed = np.argwhere(new != cache)
    assert set(changed[:, 1].tolist()) == {n_p} and len(changed) == H * d


@FAST
@given(H_kv=st.integers(1, 3), group=st.integers(1, 4), n=st.integers(1, 40), d=st.integers(2, 24),
       c=st.floats(-30.0, 30.0), seed=st.integers(0, 2**31 - 1))
def test_attention_shift_invariance_and_convexity(H_kv, group, n, d, c, seed):
    rng = np.random.default_rng(seed)
    H = H_kv * group
    q = rng.standard_normal((H, d))
    K = rng.standard_normal((H_kv, n, d))
    V = rng.standard_normal((H_kv, n, d))
    scale = 1 / np.sqrt(d)
    base = oa.decode_attention(q, K, V, scale)
    # shift every key of KV head g along the direction of one of its queries:
    # with a single query per KV head this adds a constant to that head's scores
    if group == 1:
        Ks = K + (c * q / np.maximum(np.sum(q * q, axis=1, keepdims=True), 1e-12))[:, None, :] / scale
        assert np.allclose(oa.decode_attention(q, Ks, V, scale), base, atol=1e-9)
    lo = V.min(axis=1)[np.arange(H) // group] - 1e-12
    hi = V.max(axis=1)[np.arange(H) // group] + 1e-12
    assert np.all(base >= lo) and np.all(base <= hi)


@FAST
@given(rows=st.integers(1, 6), groups=st.integers(1, 6), exp=st.integers(-20, 4),
       seed=st.integers(0, 2**31 - 1))
def test_int8_grid_round_trip(rows, groups, exp, seed):
    rng = np.random.default_rng(seed)
    K = 64 * groups
    q = rng.integers(-127, 128, size=(rows, K))
    g = q.reshape(rows, groups, 64)
    g[:, :, 0] = np.where(rng.random((rows, groups)) < 0.5, 127, -127)   # max |q| = 127
    s = np.ldexp(1.0, exp + rng.integers(-2, 3, size=(rows, groups)))
    W = (g * s[:, :, None]).reshape(rows, K)
    q2, s2 = oracle.quantize_rows(W)
    assert np.array_equal(q2.astype(np.int64), q) and np.array_equal(s2.astype(np.float64), s)
    assert np.array_equal(oracle.dequantize_rows(q2, s2), W)


@FAST
@given(I=st.integers(1, 80), T=st.integers(1, 20), d=st.integers(1, 5))
def test_pack_is_a_permutation(I, T, d):
    Wg = np.arange(I * d, dtype=np.float64).reshape(I, d)
    Wu = -1.0 - np.arange(I * d, dtype=np.float64).reshape(I, d)
    P = oracle.pack_gate_up(Wg, Wu, T)
    assert P.shape == (2 * I, d)
    g2, u2 = oracle.unpack_gate_up(P, I, T)
    assert np.array_equal(g2, Wg) and np.array_equal(u2, Wu)
    assert sorted(P[:, 0].tolist()) == sorted(np.concatenate([Wg[:, 0], Wu[:, 0]]).tolist())
