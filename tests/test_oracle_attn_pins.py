"""Pins for the oracle's token-phase attention step (oracle/attn.py), each
tying it to something other than itself: numpy's own C-order offsets for the
Eq(2) address, complex multiplication for the RoPE pairing and signs, the
rotation's norm and relative-position invariants, scipy's softmax and
log-sum-exp, the one-row / equal-key / zero-query closed forms, the grouped
KV heads against explicitly repeated heads, and rows past the position that
must not be read.  Planted mutants each fail at least one pin."""

import numpy as np
import pytest
import scipy.special

import oracle.attn as oa
from oracle import round_to_bf16


def _bf16(rng, shape, std=1.0):
    return round_to_bf16(rng.standard_normal(shape) * std)


def pin_gkvc_step_is_the_c_order_offset(o):
    for H, n_p, n_r, d in [(1, 0, 5, 4), (8, 37, 11, 128), (32, 4095, 1, 96), (3, 2, 0, 2)]:
        for h in range(H):
            if n_r == 0:
                continue
            assert o.gkvc_step(h, n_p, n_r, d) == np.ravel_multi_index((h, n_p, 0), (H, n_p + n_r, d))


def pin_kv_append_replaces_one_row(o):
    rng = np.random.default_rng(3)
    cache = rng.standard_normal((4, 9, 8))
    row = rng.standard_normal((4, 8))
    for pos in (0, 5, 8):
        new = o.kv_append(cache, row, pos)
        want = cache.copy()
        want[:, pos, :] = row
        assert np.array_equal(new, want)
    with pytest.raises(ValueError):
        o.kv_append(cache, row, 9)


def pin_rope_is_complex_rotation(o):
    rng = np.random.default_rng(4)
    for d, theta, pos in [(2, 10000.0, 3), (8, 10000.0, 17), (96, 10000.0, 4095), (128, 500000.0, 8191)]:
        x = rng.standard_normal((3, d))
        z = x[:, : d // 2] + 1j * x[:, d // 2:]
        ang = pos / np.asarray([theta ** (2.0 * i / d) for i in range(d // 2)])
        w = z * np.exp(1j * ang)
        want = np.concatenate([w.real, w.imag], axis=-1)
        assert np.allclose(o.rope(x, pos, theta), want, rtol=0, atol=1e-12)
    # d = 2: the only frequency is theta^0 = 1, a rotation by pos radians
    x = np.array([[0.6, -0.8]])
    c, s = np.cos(5.0), np.sin(5.0)
    assert np.allclose(o.rope(x, 5, 1234.5), [[0.6 * c + 0.8 * s, 0.6 * s - 0.8 * c]], atol=1e-15)


def pin_rope_invariants(o):
    rng = np.random.default_rng(5)
    d = 64
    x = rng.standard_normal(d)
    assert np.array_equal(o.rope(x, 0, 10000.0), x)                  # position 0: identity
    y = o.rope(x, 123, 10000.0)
    assert np.allclose(y[: d // 2] ** 2 + y[d // 2:] ** 2, x[: d // 2] ** 2 + x[d // 2:] ** 2,
                       rtol=1e-13, atol=0)
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    for m, n in [(10, 3), (500, 499), (7, 40)]:
        a = o.rope(q, m, 10000.0) @ o.rope(k, n, 10000.0)
        b = o.rope(q, m + 77, 10000.0) @ o.rope(k, n + 77, 10000.0)
        assert abs(a - b) <= 1e-11 * (1 + abs(a))                   # depends on m - n only


def pin_attention_closed_forms(o):
    rng = np.random.default_rng(6)
    H, H_kv, d = 4, 2, 16
    q = rng.standard_normal((H, d))
    V = rng.standard_normal((H_kv, 7, d))
    K = rng.standard_normal((H_kv, 7, d))
    # one row: every head returns that row of its KV head
    one = o.decode_attention(q, K[:, :1], V[:, :1], 0.25)
    assert np.array_equal(one, V[np.arange(H) // 2, 0])
    # equal keys, or a zero query: uniform weights, the mean of V
    Keq = np.repeat(K[:, :1], 7, axis=1)
    assert np.allclose(o.decode_attention(q, Keq, V, 0.25), V[np.arange(H) // 2].mean(axis=1),
                       atol=1e-14)
    assert np.allclose(o.decode_attention(np.zeros((H, d)), K, V, 0.25),
                       V[np.arange(H) // 2].mean(axis=1), atol=1e-14)


def pin_attention_vs_scipy(o):
    rng = np.random.default_rng(7)
    H, H_kv, n, d = 6, 3, 50, 32
    q, K, V = rng.standard_normal((H, d)), rng.standard_normal((H_kv, n, d)), rng.standard_normal((H_kv, n, d))
    got = o.decode_attention(q, K, V, 1 / np.sqrt(d))
    for h in range(H):
        g = h // 2
        p = scipy.special.softmax(K[g] @ q[h] / np.sqrt(d))
        assert np.allclose(got[h], p @ V[g], rtol=0, atol=1e-13)
    # scores in the hundreds: exp overflows without the max subtraction
    big = o.decode_attention(q * 300.0, K, V, 1.0)
    for h in range(H):
        s = K[h // 2] @ (q[h] * 300.0)
        p = np.exp(s - scipy.special.logsumexp(s))
        assert np.all(np.isfinite(big[h])) and np.allclose(big[h], p @ V[h // 2], atol=1e-12)


def pin_grouped_heads_equal_repeated_heads(o):
    rng = np.random.default_rng(8)
    H, H_kv, n, d = 8, 2, 20, 8
    q, K, V = rng.standard_normal((H, d)), rng.standard_normal((H_kv, n, d)), rng.standard_normal((H_kv, n, d))
    rep = o.decode_attention(q, np.repeat(K, H // H_kv, axis=0), np.repeat(V, H // H_kv, axis=0), 0.3)
    assert np.allclose(o.decode_attention(q, K, V, 0.3), rep, atol=1e-15)


def pin_token_step(o):
    rng = np.random.default_rng(9)
    B, H, H_kv, d, n_max, theta = 3, 4, 2, 16, 12, 10000.0
    q = _bf16(rng, (B, H, d))
    kn, vn = _bf16(rng, (B, H_kv, d)), _bf16(rng, (B, H_kv, d))
    kc, vc = _bf16(rng, (B, H_kv, n_max, d)), _bf16(rng, (B, H_kv, n_max, d))
    pos = np.array([0, 5, 11])
    kc_nan, vc_nan = kc.copy(), vc.copy()
    for b in range(B):              # rows past the position must not be read
        kc_nan[b, :, pos[b] + 1:] = np.nan
        vc_nan[b, :, pos[b] + 1:] = np.nan
    out, ko, vo = o.token_attention(q, kn, vn, kc_nan, vc_nan, pos, theta)
    assert np.all(np.isfinite(out))
    # the stored rows: rotated k rounded to bf16, v as given; nothing else changes
    for b in range(B):
        p = pos[b]
        assert np.array_equal(ko[b, :, p], round_to_bf16(o.rope(kn[b], p, theta)))
        assert np.array_equal(vo[b, :, p], vn[b])
        keep = np.ones(n_max, bool)
        keep[p] = False
        assert np.array_equal(ko[b][:, keep][:, : p], kc[b][:, keep][:, : p])
    # position 0: the only row is the new one, so every head returns v
    assert np.array_equal(out[0], vn[0][np.arange(H) // 2])
    # against scipy's softmax with scale 1/sqrt(d), the new row included
    for b in (1, 2):
        p = pos[b]
        for h in range(H):
            g = h // 2
            Kb = np.concatenate([kc[b, g, :p], round_to_bf16(o.rope(kn[b], p, theta))[g][None]])
            Vb = np.concatenate([vc[b, g, :p], vn[b, g][None]])
            w = scipy.special.softmax(Kb @ o.rope(q[b, h], p, theta) / np.sqrt(d))
            assert np.allclose(out[b, h], w @ Vb, atol=1e-13)


PINS = [pin_gkvc_step_is_the_c_order_offset, pin_kv_append_replaces_one_row,
        pin_rope_is_complex_rotation, pin_rope_invariants, pin_attention_closed_forms,
        pin_attention_vs_scipy, pin_grouped_heads_equal_repeated_heads, pin_token_step]


@pytest.mark.parametrize("pin", PINS, ids=lambda p: p.__name__)
def test_attn_pin(pin):
    pin(oa)


# ---- planted mutants (in the oracle, on the CPU) ----

def _mut_rope_sign(x, pos, theta):
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    a = oa.rope_angles(pos, d, theta)
    lo, hi = x[..., : d // 2], x[..., d // 2:]
    return np.concatenate([lo * np.cos(a) + hi * np.sin(a), -lo * np.sin(a) + hi * np.cos(a)], axis=-1)


def _mut_rope_adjacent_pairs(x, pos, theta):
    x = np.asarray(x, dtype=np.float64)
    d = x.shape[-1]
    a = oa.rope_angles(pos, d, theta)
    ev, od = x[..., 0::2], x[..., 1::2]
    out = np.empty_like(x)
    out[..., 0::2] = ev * np.cos(a) - od * np.sin(a)
    out[..., 1::2] = ev * np.sin(a) + od * np.cos(a)
    return out


def _mut_step_off_by_one(h, n_p, n_r, d):
    return h * (n_p + n_r) * d + (n_p + 1) * d


def _mut_no_max(q_rot, K, V, scale):
    q_rot, K, V = (np.asarray(t, dtype=np.float64) for t in (q_rot, K, V))
    H = q_rot.shape[0]
    group = H // K.shape[0]
    out = np.empty(q_rot.shape)
    for h in range(H):
        w = np.exp(scale * (K[h // group] @ q_rot[h]))
        out[h] = (w / w.sum()) @ V[h // group]
    return out


def _mut_heads_modulo(q_rot, K, V, scale):
    q_rot, K, V = (np.asarray(t, dtype=np.float64) for t in (q_rot, K, V))
    out = np.empty(q_rot.shape)
    for h in range(q_rot.shape[0]):
        g = h % K.shape[0]
        s = scale * (K[g] @ q_rot[h])
        w = np.exp(s - s.max())
        out[h] = (w / w.sum()) @ V[g]
    return out


def _mut_unscaled(q, k_new, v_new, k_cache, v_cache, pos, theta, scale=None):
    return oa._orig_token_attention(q, k_new, v_new, k_cache, v_cache, pos, theta,
                                    1.0 if scale is None else scale)


def _mut_excludes_new_row(q, k_new, v_new, k_cache, v_cache, pos, theta, scale=None):
    q = np.asarray(q, dtype=np.float64)
    B, H, d = q.shape
    scale = 1.0 / np.sqrt(d) if scale is None else scale
    out, ko, vo = oa._orig_token_attention(q, k_new, v_new, k_cache, v_cache, pos, theta, scale)
    for b in range(B):
        p = int(pos[b])
        if p > 0:
            out[b] = oa.decode_attention(oa.rope(q[b], p, theta), ko[b][:, :p], vo[b][:, :p], scale)
        else:
            out[b] = np.nan
    return out, ko, vo


def _mut_unrounded_k(q, k_new, v_new, k_cache, v_cache, pos, theta, scale=None):
    saved = oa.round_to_bf16
    oa.round_to_bf16 = lambda v: np.asarray(v, dtype=np.float64)
    try:
        return oa._orig_token_attention(q, k_new, v_new, k_cache, v_cache, pos, theta, scale)
    finally:
        oa.round_to_bf16 = saved


MUTANTS = {"rope_sign": ("rope", _mut_rope_sign),
           "rope_adjacent_pairs": ("rope", _mut_rope_adjacent_pairs),
           "step_off_by_one": ("gkvc_step", _mut_step_off_by_one),
           "softmax_without_max": ("decode_attention", _mut_no_max),
           "heads_modulo": ("decode_attention", _mut_heads_modulo),
           "unscaled_scores": ("token_attention", _mut_unscaled),
           "excludes_new_row": ("token_attention", _mut_excludes_new_row),
           "unrounded_k_row": ("token_attention", _mut_unrounded_k)}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_attn_mutants_are_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(oa, "_orig_token_attention", oa.token_attention, raising=False)
    monkeypatch.setattr(oa, attr, fn)
    caught = []
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin(oa)
        except (AssertionError, ValueError, IndexError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, f"mutant {name} passed every pin"
