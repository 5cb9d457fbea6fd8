"""Pins for the fp64 oracle: each check ties it to something other than itself.

The pages print no worked numbers, so the pins are the mathematics the pages
fix: closed forms, exact invariants, limits of SiLU, brute force on tiny
shapes, library routines for special cases, and the row order the pages
describe for the gate/up interleave (tests/golden/interleave_rows.json).

Each ``pin_*`` takes the oracle module so that ``test_oracle_mutants`` can run
the same pins against deliberately broken copies of the oracle and show that
every plausible mistake (dropped term, wrong sign, swapped operand, misplaced
eps, wrong row order) is caught.
"""

import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
import oracle.fmlp as ofm

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16_values(rng, shape, scale=1.0, offset=0.0):
    """Random bf16-exact float64 values (drawn here, rounded with torch)."""
    v = torch.from_numpy((offset + scale * rng.standard_normal(shape)).astype(np.float32))
    return v.to(torch.bfloat16).to(torch.float64).numpy()


# ----------------------------------------------------------------------------
# bf16 decode / round
# ----------------------------------------------------------------------------

def pin_decode_bf16_exhaustive(o):
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    mine = o.decode_bf16(bits)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    same = (mine == ref) | (np.isnan(mine) & np.isnan(ref))
    assert same.all()
    # a few values by the IEEE definition
    assert o.decode_bf16(np.array([0x3F80], np.uint16))[0] == 1.0
    assert o.decode_bf16(np.array([0xC000], np.uint16))[0] == -2.0
    assert o.decode_bf16(np.array([0x3F81], np.uint16))[0] == 1.0 + 2.0 ** -7
    assert o.decode_bf16(np.array([0x0001], np.uint16))[0] == 2.0 ** -133
    assert o.decode_bf16(np.array([0x7F80], np.uint16))[0] == np.inf


def pin_round_to_bf16(o):
    # every finite bf16 value is a fixed point
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    vals = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    fin = np.isfinite(vals)
    assert np.array_equal(o.round_to_bf16(vals[fin]), vals[fin])
    # ties go to the even neighbour, just-above-tie goes up
    one = 1.0
    ulp = 2.0 ** -7
    assert o.round_to_bf16(np.array([one + ulp / 2]))[0] == one
    assert o.round_to_bf16(np.array([one + 3 * ulp / 2]))[0] == one + 2 * ulp
    assert o.round_to_bf16(np.array([one + ulp / 2 + 2.0 ** -30]))[0] == one + ulp
    assert o.round_to_bf16(np.array([-(one + ulp / 2)]))[0] == -one
    # overflow past the largest finite bf16 rounds to inf
    assert o.round_to_bf16(np.array([3.5e38]))[0] == np.inf
    # agreement with torch's binary32 -> bf16 rounding (inputs exact in binary32)
    rng = np.random.default_rng(7)
    f32 = np.concatenate([
        rng.standard_normal(200000).astype(np.float32),
        (rng.standard_normal(20000) * 1e-39).astype(np.float32),   # subnormals
        (rng.standard_normal(20000) * 1e37).astype(np.float32),
    ])
    ref = torch.from_numpy(f32).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(o.round_to_bf16(f32.astype(np.float64)), ref)


# ----------------------------------------------------------------------------
# RMSNorm
# ----------------------------------------------------------------------------

def pin_rms_inv_vs_norm(o):
    rng = np.random.default_rng(1)
    x = rng.standard_normal((5, 37))
    # eps = 0: r = sqrt(d) / ||x||_2 (numpy.linalg.norm is an independent routine)
    r = o.rms_inv(x, 0.0)
    ref = math.sqrt(37) / np.linalg.norm(x, axis=1)
    np.testing.assert_allclose(r, ref, rtol=1e-14)
    # eps sits inside the square root, with the mean (not the sum) of squares
    eps = 0.25
    ref_eps = 1.0 / np.sqrt((np.linalg.norm(x, axis=1) ** 2) / 37 + eps)
    np.testing.assert_allclose(o.rms_inv(x, eps), ref_eps, rtol=1e-14)


def pin_rmsnorm_scale_invariance(o):
    rng = np.random.default_rng(2)
    x = _bf16_values(rng, (3, 64))
    gamma = _bf16_values(rng, (64,), 0.1, 1.0)
    h = o.rmsnorm(x, gamma, 0.0)
    for k in (-3, 1, 5):
        hk = o.rmsnorm(x * 2.0 ** k, gamma, 0.0)
        assert np.array_equal(h, hk), k          # exact: powers of two scale exactly
    # with eps > 0 the drift is bounded by eps * |1 - c^-2| / (2 mean x^2)
    eps, c = 1e-5, 4.0
    h1 = o.rmsnorm(x, gamma, eps)
    h4 = o.rmsnorm(c * x, gamma, eps)
    ms = np.mean(x * x, axis=1)
    bound = eps * abs(1 - c ** -2) / (2 * ms) * 1.01 + 1e-15
    rel = np.max(np.abs(h4 - h1) / np.maximum(np.abs(h1), 1e-300), axis=1)
    assert np.all(rel <= bound)
    # gamma multiplies elementwise (gamma = 1 gives the plain normalised row)
    h_one = o.rmsnorm(x, np.ones(64), 0.0)
    np.testing.assert_allclose(h_one * gamma, h, rtol=1e-15)
    np.testing.assert_allclose(np.sqrt(np.mean(h_one ** 2, axis=1)), 1.0, rtol=1e-14)


# ----------------------------------------------------------------------------
# SiLU
# ----------------------------------------------------------------------------

def pin_silu(o):
    assert o.silu(np.array([0.0]))[0] == 0.0
    t = np.linspace(-30, 30, 6001)
    # SiLU(t) - SiLU(-t) = t  (t*sigma(t) + t*sigma(-t) = t)
    np.testing.assert_allclose(o.silu(t) - o.silu(-t), t, rtol=0, atol=1e-13)
    # against t * sigma(t) from scipy's logistic function
    from scipy.special import expit
    np.testing.assert_allclose(o.silu(t), t * expit(t), rtol=1e-14, atol=1e-300)
    # derivative 1/2 at 0, limits at +-inf
    dt = 1e-6
    assert abs((o.silu(np.array([dt]))[0] - o.silu(np.array([-dt]))[0]) / (2 * dt) - 0.5) < 1e-9
    assert o.silu(np.array([800.0]))[0] == 800.0
    assert o.silu(np.array([-800.0]))[0] == 0.0


# ----------------------------------------------------------------------------
# Eq(1)
# ----------------------------------------------------------------------------

def pin_closed_form_d1_I1(o):
    # d = 1, I = 1:  O = wd * SiLU(wg*h) * (wu*h),  h = gamma * x / sqrt(x^2 + eps)
    for (x, gamma, wg, wu, wd, eps) in [(1.5, 0.75, 0.5, -2.0, 3.0, 1e-5),
                                        (-0.25, 1.25, -4.0, 1.0, 0.5, 0.5),
                                        (2.0, 1.0, 3.0, 3.0, -1.0, 0.0)]:
        h = gamma * x / math.sqrt(x * x + eps)
        gv = wg * h
        expect = wd * (gv / (1.0 + math.exp(-gv))) * (wu * h)
        got = o.fused_mlp(np.array([[x]]), np.array([gamma]), eps,
                          np.array([[wg]]), np.array([[wu]]), np.array([[wd]]))
        assert got.shape == (1, 1)
        assert abs(got[0, 0] - expect) <= 1e-14 * max(1.0, abs(expect))


def pin_zero_invariants(o):
    rng = np.random.default_rng(3)
    M, d, I = 3, 24, 40
    x = _bf16_values(rng, (M, d))
    gamma = _bf16_values(rng, (d,), 0.1, 1.0)
    Wg = _bf16_values(rng, (I, d), 0.02)
    Wu = _bf16_values(rng, (I, d), 0.02)
    Wd = _bf16_values(rng, (d, I), 0.02)
    Z = np.zeros
    # SiLU(0) = 0 kills the block when the gate weights vanish
    assert np.array_equal(o.fused_mlp(x, gamma, 1e-5, Z((I, d)), Wu, Wd), Z((M, d)))
    assert np.array_equal(o.fused_mlp(x, gamma, 1e-5, Wg, Z((I, d)), Wd), Z((M, d)))
    assert np.array_equal(o.fused_mlp(x, gamma, 1e-5, Wg, Wu, Z((d, I))), Z((M, d)))
    # x = 0 with eps > 0: h = 0, so O = 0
    assert np.array_equal(o.fused_mlp(Z((M, d)), gamma, 1e-5, Wg, Wu, Wd), Z((M, d)))
    # a zero row only zeroes its own output row
    x2 = x.copy()
    x2[1] = 0
    O2 = o.fused_mlp(x2, gamma, 1e-5, Wg, Wu, Wd)
    assert np.array_equal(O2[1], np.zeros(d))
    np.testing.assert_allclose(O2[[0, 2]], o.fused_mlp(x[[0, 2]], gamma, 1e-5, Wg, Wu, Wd),
                               rtol=1e-13, atol=1e-15)
    # residual is added after the down projection: W_down = 0 leaves the residual
    R = _bf16_values(rng, (M, d))
    assert np.array_equal(o.fused_mlp(x, gamma, 1e-5, Wg, Wu, Z((d, I)), residual=R), R)


def _naive_exact(x, gamma, eps, Wg, Wu, Wd):
    """Independent evaluation with Python loops: exact rational dot products,
    math.sqrt / math.exp for the two transcendental steps."""
    M, d = len(x), len(x[0])
    I = len(Wg)
    out = []
    for m in range(M):
        ss = sum(Fraction(v) * Fraction(v) for v in x[m])
        r = 1.0 / math.sqrt(float(ss / d + Fraction(eps)))
        h = [Fraction(float(Fraction(x[m][k]) * Fraction(r) * Fraction(gamma[k]))) for k in range(d)]
        a = []
        for i in range(I):
            g = float(sum(Fraction(Wg[i][k]) * h[k] for k in range(d)))
            u = float(sum(Fraction(Wu[i][k]) * h[k] for k in range(d)))
            a.append(Fraction(g / (1.0 + math.exp(-g)) * u))
        out.append([float(sum(Fraction(Wd[n][i]) * a[i] for i in range(I))) for n in range(d)])
    return np.array(out)


def pin_bruteforce_tiny(o):
    rng = np.random.default_rng(4)
    for (M, d, I) in [(1, 1, 1), (2, 3, 5), (3, 8, 4), (1, 16, 16), (2, 5, 11)]:
        x = _bf16_values(rng, (M, d))
        gamma = _bf16_values(rng, (d,), 0.1, 1.0)
        Wg = _bf16_values(rng, (I, d), 0.7)
        Wu = _bf16_values(rng, (I, d), 0.7)
        Wd = _bf16_values(rng, (d, I), 0.7)
        eps = 1e-5
        got = o.fused_mlp(x, gamma, eps, Wg, Wu, Wd)
        ref = _naive_exact(x.tolist(), gamma.tolist(), eps, Wg.tolist(), Wu.tolist(), Wd.tolist())
        scale = max(1e-300, np.max(np.abs(ref)))
        assert np.max(np.abs(got - ref)) <= 1e-12 * scale, (M, d, I)


def pin_saturated_gate_is_bilinear(o):
    # all-positive rows and gate weights push W_gate h >> 0, where SiLU(t) -> t
    # within t*exp(-t); the block then reduces to a bilinear form evaluated here
    # with einsum and an independent norm.
    rng = np.random.default_rng(5)
    M, d, I = 2, 32, 24
    x = np.abs(_bf16_values(rng, (M, d))) + 0.5
    gamma = np.ones(d)
    Wg = np.abs(_bf16_values(rng, (I, d))) + 2.0
    Wu = _bf16_values(rng, (I, d))
    Wd = _bf16_values(rng, (d, I))
    h = x * (math.sqrt(d) / np.linalg.norm(x, axis=1))[:, None]
    g = np.einsum("ik,mk->mi", Wg, h)
    assert g.min() > 60
    ref = np.einsum("ni,mi,mi->mn", Wd, g, np.einsum("ik,mk->mi", Wu, h))
    got = o.fused_mlp(x, gamma, 0.0, Wg, Wu, Wd)
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12 * np.abs(ref).max())
    # the mirror case W_gate h << 0 drives every a to 0
    got_neg = o.fused_mlp(x, gamma, 0.0, -Wg, Wu, Wd)
    assert np.max(np.abs(got_neg)) < 1e-20


def pin_swiglu_intermediate(o):
    # a is what gated_mlp feeds the down projection: W_down = I recovers it
    rng = np.random.default_rng(11)
    M, d, I = 2, 6, 6
    h = _bf16_values(rng, (M, d))
    Wg, Wu = _bf16_values(rng, (I, d), 0.5), _bf16_values(rng, (I, d), 0.5)
    a = o.swiglu_intermediate(h, Wg, Wu)
    assert a.shape == (M, I)
    np.testing.assert_allclose(o.gated_mlp(h, Wg, Wu, np.eye(I)), a, rtol=1e-15, atol=0)
    for m in range(M):
        for i in range(I):
            g = float(sum(Fraction(Wg[i, k]) * Fraction(h[m, k]) for k in range(d)))
            u = float(sum(Fraction(Wu[i, k]) * Fraction(h[m, k]) for k in range(d)))
            assert abs(a[m, i] - g / (1 + math.exp(-g)) * u) <= 1e-14 * (1 + abs(a[m, i]))


def pin_intermediate_rounding(o):
    rng = np.random.default_rng(6)
    M, d, I = 2, 16, 12
    x = _bf16_values(rng, (M, d))
    gamma = _bf16_values(rng, (d,), 0.1, 1.0)
    Wg, Wu = _bf16_values(rng, (I, d), 0.3), _bf16_values(rng, (I, d), 0.3)
    Wd = np.eye(d, I)   # the down projection then copies a out
    O = o.fused_mlp(x, gamma, 1e-5, Wg, Wu, Wd)
    Ob = o.fused_mlp(x, gamma, 1e-5, Wg, Wu, Wd, intermediate="bf16")
    assert np.array_equal(Ob, o.round_to_bf16(O))
    assert not np.array_equal(Ob, O)


# ----------------------------------------------------------------------------
# The gate/up interleave
# ----------------------------------------------------------------------------

def pin_interleave_golden(o):
    with open(os.path.join(GOLDEN, "interleave_rows.json")) as f:
        cases = json.load(f)["cases"]
    for c in cases:
        I, T = c["I"], c["T"]
        # pack rows labelled by name and compare with the page-described order
        Wg = np.array([[f"g{i}"] for i in range(I)], dtype=object)
        Wu = np.array([[f"u{i}"] for i in range(I)], dtype=object)
        P = o.pack_gate_up(Wg, Wu, T)
        assert [row[0] for row in P] == c["order"], (I, T)


def pin_interleave_is_permutation(o):
    rng = np.random.default_rng(8)
    for (I, d, T) in [(688, 8, 16), (40, 16, 8), (45, 8, 16), (7, 3, 1), (64, 8, 64)]:
        Wg = rng.integers(0, 1 << 16, size=(I, d), dtype=np.uint16)
        Wu = rng.integers(0, 1 << 16, size=(I, d), dtype=np.uint16)
        P = o.pack_gate_up(Wg, Wu, T)
        assert P.shape == (2 * I, d) and P.dtype == np.uint16
        g2, u2 = o.unpack_gate_up(P, I, T)
        assert np.array_equal(g2, Wg) and np.array_equal(u2, Wu)
        # every source row lands exactly once
        gr, ur = o.interleaved_rows(I, T)
        assert np.array_equal(np.sort(np.concatenate([gr, ur])), np.arange(2 * I))
        # within a full tile: T gate rows, then the same T up rows
        if I % T == 0:
            for t in range(I // T):
                blk = P[2 * T * t: 2 * T * (t + 1)]
                assert np.array_equal(blk[:T], Wg[t * T:(t + 1) * T])
                assert np.array_equal(blk[T:], Wu[t * T:(t + 1) * T])


def pin_packed_forward_equals_plain(o):
    rng = np.random.default_rng(9)
    M, d, I, T = 3, 32, 48, 16
    x = _bf16_values(rng, (M, d))
    gamma = _bf16_values(rng, (d,), 0.1, 1.0)
    Wg, Wu = _bf16_values(rng, (I, d), 0.1), _bf16_values(rng, (I, d), 0.1)
    Wd = _bf16_values(rng, (d, I), 0.1)
    P = o.pack_gate_up(Wg, Wu, T)
    a = o.fused_mlp(x, gamma, 1e-5, Wg, Wu, Wd)
    b = o.fused_mlp_packed(x, gamma, 1e-5, P, T, Wd)
    assert np.array_equal(a, b)     # packing is layout only: bit-identical result


def pin_bf16_entry_decodes(o):
    rng = np.random.default_rng(10)
    M, d, I = 2, 16, 8
    t = lambda a: torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16)
    bits = lambda a: a.contiguous().view(torch.int16).numpy().view(np.uint16)
    x, gamma = t(rng.standard_normal((M, d))), t(1 + 0.1 * rng.standard_normal(d))
    Wg, Wu, Wd = (t(0.2 * rng.standard_normal(s)) for s in [(I, d), (I, d), (d, I)])
    got = o.fused_mlp_bf16(bits(x), bits(gamma), 1e-5, bits(Wg), bits(Wu), bits(Wd))
    f = lambda a: a.to(torch.float64).numpy()
    ref = _naive_exact(f(x).tolist(), f(gamma).tolist(), 1e-5, f(Wg).tolist(), f(Wu).tolist(),
                       f(Wd).tolist())
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-14)


def pin_bf16_output(o):
    """The bf16 output of the chained block: the binary64 result, residual
    included, rounded once.  Checked against torch's own binary64 -> bf16
    conversion of the block's binary64 output (an independent rounding), its
    half-step error bound, exact bf16 values, and the zero-weight case where
    the output is the (bf16) residual itself."""
    rng = np.random.default_rng(11)
    M, d, I = 3, 64, 48
    x = _bf16_values(rng, (M, d))
    gamma = _bf16_values(rng, (d,), 0.1, 1.0)
    Wg, Wu = _bf16_values(rng, (I, d), 0.2), _bf16_values(rng, (I, d), 0.2)
    Wd = _bf16_values(rng, (d, I), 0.2)
    res = _bf16_values(rng, (M, d))
    for r in (None, res):
        exact = o.fused_mlp(x, gamma, 1e-5, Wg, Wu, Wd, residual=r)
        got = o.fused_mlp(x, gamma, 1e-5, Wg, Wu, Wd, residual=r, output="bf16")
        ref = torch.from_numpy(exact).to(torch.bfloat16).to(torch.float64).numpy()
        assert np.array_equal(got, ref)
        # a bf16 value v in [2^(e-1), 2^e) has step 2^(e-8): within half a step
        step = np.ldexp(1.0, np.frexp(exact)[1] - 8)
        assert np.all(np.abs(got - exact) <= step / 2)
        assert np.array_equal(o.round_to_bf16(got), got)
    # the rounding happens after the residual add, not before it
    before = o.round_to_bf16(o.fused_mlp(x, gamma, 1e-5, Wg, Wu, Wd)) + res
    assert not np.array_equal(o.fused_mlp(x, gamma, 1e-5, Wg, Wu, Wd, residual=res,
                                          output="bf16"), before)
    # zero gate weights: SiLU(0) = 0, so the output is the residual exactly
    zero = o.fused_mlp(x, gamma, 1e-5, 0 * Wg, Wu, Wd, residual=res, output="bf16")
    assert np.array_equal(zero, res)


PINS = [pin_decode_bf16_exhaustive, pin_round_to_bf16, pin_rms_inv_vs_norm,
        pin_rmsnorm_scale_invariance, pin_silu, pin_closed_form_d1_I1, pin_zero_invariants,
        pin_bruteforce_tiny, pin_saturated_gate_is_bilinear, pin_swiglu_intermediate,
        pin_intermediate_rounding,
        pin_interleave_golden, pin_interleave_is_permutation, pin_packed_forward_equals_plain,
        pin_bf16_entry_decodes, pin_bf16_output]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_oracle_pin(pin):
    pin(ofm)


def test_package_exports_are_the_pinned_functions():
    for name in ["decode_bf16", "round_to_bf16", "rms_inv", "rmsnorm", "silu",
                 "swiglu_intermediate", "gated_mlp",
                 "fused_mlp", "interleaved_rows", "pack_gate_up", "unpack_gate_up",
                 "fused_mlp_packed", "fused_mlp_bf16"]:
        assert getattr(oracle, name) is getattr(ofm, name)


# ----------------------------------------------------------------------------
# Planted mistakes: every mutant of the oracle must fail at least one pin
# ----------------------------------------------------------------------------

def _mut_silu_sign(t):
    t = np.asarray(t, dtype=np.float64)
    with np.errstate(over="ignore"):
        return t / (1.0 + np.exp(t))


def _mut_silu_sigmoid(t):
    t = np.asarray(t, dtype=np.float64)
    with np.errstate(over="ignore"):
        return 1.0 / (1.0 + np.exp(-t))


def _mut_rms_eps_outside(x, eps):
    x = np.asarray(x, dtype=np.float64)
    return 1.0 / np.sqrt(np.mean(x * x, axis=-1)) + eps


def _mut_rms_sum(x, eps):
    x = np.asarray(x, dtype=np.float64)
    return 1.0 / np.sqrt(np.sum(x * x, axis=-1) + eps)


def _mut_rmsnorm_no_gamma(x, gamma, eps):
    x = np.asarray(x, dtype=np.float64)
    return x * ofm.rms_inv(x, eps)[..., None]


def _mut_gated_swap_branches(h, W_gate, W_up, W_down, intermediate=None):
    return ofm._orig_gated_mlp(h, W_up, W_gate, W_down, intermediate)


def _mut_gated_add(h, W_gate, W_up, W_down, intermediate=None):
    h = np.asarray(h, dtype=np.float64)
    a = ofm.silu(h @ W_gate.T) + h @ W_up.T
    return a @ np.asarray(W_down, dtype=np.float64).T


def _mut_gated_drop_last_term(h, W_gate, W_up, W_down, intermediate=None):
    h = np.asarray(h, dtype=np.float64).copy()
    h[..., -1] = 0.0
    return ofm._orig_gated_mlp(h, W_gate, W_up, W_down, intermediate)


def _mut_interleave_swapped(I, T):
    g, u = ofm._orig_interleaved_rows(I, T)
    return u, g


def _mut_interleave_plain_concat(I, T):
    i = np.arange(I, dtype=np.int64)
    return i, i + I


def _mut_round_truncate(v):
    v = np.asarray(v, dtype=np.float64)
    m, e = np.frexp(v)
    return np.ldexp(np.trunc(np.ldexp(m, 8)), e - 8)


def _mut_fused_round_before_residual(x, gamma, eps, W_gate, W_up, W_down, residual=None,
                                     intermediate=None, output=None):
    O = ofm._orig_fused_mlp(x, gamma, eps, W_gate, W_up, W_down, intermediate=intermediate,
                            output=output)
    if residual is not None:
        O = O + np.asarray(residual, dtype=np.float64)
    return O


MUTANTS = {
    "silu_sign": ("silu", _mut_silu_sign),
    "silu_is_sigmoid": ("silu", _mut_silu_sigmoid),
    "eps_outside_sqrt": ("rms_inv", _mut_rms_eps_outside),
    "sum_not_mean": ("rms_inv", _mut_rms_sum),
    "gamma_dropped": ("rmsnorm", _mut_rmsnorm_no_gamma),
    "silu_on_up_branch": ("gated_mlp", _mut_gated_swap_branches),
    "add_not_multiply": ("gated_mlp", _mut_gated_add),
    "dropped_last_k_term": ("gated_mlp", _mut_gated_drop_last_term),
    "gate_up_swapped_in_tile": ("interleaved_rows", _mut_interleave_swapped),
    "no_interleave": ("interleaved_rows", _mut_interleave_plain_concat),
    "bf16_truncates": ("round_to_bf16", _mut_round_truncate),
    "output_rounded_before_residual": ("fused_mlp", _mut_fused_round_before_residual),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_oracle_mutants_are_caught(name, monkeypatch):
    attr, fn = MUTANTS[name]
    monkeypatch.setattr(ofm, "_orig_gated_mlp", ofm.gated_mlp, raising=False)
    monkeypatch.setattr(ofm, "_orig_interleaved_rows", ofm.interleaved_rows, raising=False)
    monkeypatch.setattr(ofm, "_orig_fused_mlp", ofm.fused_mlp, raising=False)
    monkeypatch.setattr(ofm, attr, fn)
    caught = []
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin(ofm)
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"mutant {name} passed every pin"
