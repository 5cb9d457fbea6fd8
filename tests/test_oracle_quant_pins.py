"""Pins for the oracle's int8 weight format (oracle/quant.py): each ties it to
something other than itself -- exact round trips of weights already on the
grid, the rounding error bound, zero groups, exact power-of-two scale
invariance, the group maximum mapping to +-127, and the block on grid-exact
weights equal to the plain block.  Planted mutants (truncation, a 128
divisor, groups along the wrong axis) each fail a pin."""

import numpy as np
import pytest

import oracle
import oracle.quant as oq


def _grid(rng, rows, K, group=64, exp=-9):
    """Weights exactly on the int8 grid: q in [-127, 127] with +-127 in every
    group, times a power-of-two scale (so q * s is exact and max/127 = s)."""
    q = rng.integers(-127, 128, size=(rows, K))
    g = q.reshape(rows, K // group, group)
    g[:, :, 0] = np.where(rng.random((rows, K // group)) < 0.5, 127, -127)
    s = np.ldexp(1.0, exp + rng.integers(-3, 4, size=(rows, K // group)))
    return q, s, (g * s[:, :, None]).reshape(rows, K)


def pin_round_trip_on_grid(o):
    rng = np.random.default_rng(1)
    q, s, W = _grid(rng, 12, 256)
    q2, s2 = o.quantize_rows(W)
    assert np.array_equal(q2.astype(np.int64), q) and np.array_equal(s2.astype(np.float64), s)
    assert np.array_equal(o.dequantize_rows(q2, s2), W)


def pin_error_bound(o):
    rng = np.random.default_rng(2)
    W = (rng.standard_normal((16, 512)) * 0.02).astype(np.float32).astype(np.float64)
    q, s = o.quantize_rows(W)
    assert q.dtype == np.int8 and s.dtype == np.float32 and s.shape == (16, 8)
    err = np.abs(o.dequantize_rows(q, s) - W).reshape(16, 8, 64)
    bound = s.astype(np.float64)[:, :, None] / 2 + np.abs(W).reshape(16, 8, 64) * 2.0 ** -23
    assert np.all(err <= bound)
    # the scale is the group's largest magnitude over 127 (binary32), and that
    # element lands on +-127
    m = np.max(np.abs(W.reshape(16, 8, 64)), axis=2)
    assert np.array_equal(s, (m.astype(np.float32) / np.float32(127)).astype(np.float32))
    top = np.argmax(np.abs(W.reshape(16, 8, 64)), axis=2)
    qt = np.take_along_axis(q.reshape(16, 8, 64).astype(np.int64), top[:, :, None], 2)[:, :, 0]
    assert np.all(np.abs(qt) == 127)


def pin_zero_groups(o):
    W = np.zeros((2, 128))
    W[1, 64:] = 0.5
    q, s = o.quantize_rows(W)
    assert np.all(q[0] == 0) and np.all(q[1, :64] == 0) and s[0, 0] == 0 and s[1, 0] == 0
    assert np.all(q[1, 64:] == 127) and s[1, 1] == np.float32(0.5) / np.float32(127)


def pin_power_of_two_invariance(o):
    rng = np.random.default_rng(3)
    W = rng.standard_normal((8, 192)).astype(np.float32).astype(np.float64)
    q, s = o.quantize_rows(W)
    for k in (-5, 7):
        q2, s2 = o.quantize_rows(W * 2.0 ** k)
        assert np.array_equal(q2, q) and np.array_equal(s2, (s * np.float32(2.0 ** k)))


def pin_block_on_grid_weights(o):
    rng = np.random.default_rng(4)
    M, d, I = 3, 128, 192
    x = rng.standard_normal((M, d)).astype(np.float32).astype(np.float64)
    gamma = 1 + 0.1 * rng.standard_normal(d).astype(np.float32).astype(np.float64)
    _, _, Wg = _grid(rng, I, d, exp=-12)
    _, _, Wu = _grid(rng, I, d, exp=-12)
    _, _, Wd = _grid(rng, d, I, exp=-12)
    res = rng.standard_normal((M, d))
    qs = [o.quantize_rows(W) for W in (Wg, Wu, Wd)]
    got = o.fused_mlp_q8(x, gamma, 1e-5, *qs[0], *qs[1], *qs[2], residual=res)
    assert np.array_equal(got, oracle.fused_mlp(x, gamma, 1e-5, Wg, Wu, Wd, residual=res))
    # and quantization commutes with the gate/up interleave (it works row by row)
    qp, sp = o.quantize_rows(oracle.pack_gate_up(Wg, Wu, 16))
    assert np.array_equal(qp, oracle.pack_gate_up(qs[0][0], qs[1][0], 16))
    assert np.array_equal(sp, oracle.pack_gate_up(qs[0][1], qs[1][1], 16))


PINS = [pin_round_trip_on_grid, pin_error_bound, pin_zero_groups, pin_power_of_two_invariance,
        pin_block_on_grid_weights]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_quant_pin(pin):
    pin(oq)


def _mut_truncate(W, group=64):
    W = np.asarray(W, dtype=np.float64)
    rows, K = W.shape
    g = W.astype(np.float32).reshape(rows, K // group, group)
    s = (np.max(np.abs(g), axis=2) / np.float32(127)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(s[:, :, None] > 0, np.trunc(g / s[:, :, None]), 0)
    return q.reshape(rows, K).astype(np.int8), s


def _mut_div128(W, group=64):
    W = np.asarray(W, dtype=np.float64)
    rows, K = W.shape
    g = W.astype(np.float32).reshape(rows, K // group, group)
    s = (np.max(np.abs(g), axis=2) / np.float32(128)).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.where(s[:, :, None] > 0, np.clip(np.rint(g / s[:, :, None]), -127, 127), 0)
    return q.reshape(rows, K).astype(np.int8), s


def _mut_groups_across_rows(W, group=64):
    W = np.asarray(W, dtype=np.float64)
    q, s = oq._orig_quantize_rows(np.ascontiguousarray(W.T), group) if W.shape[0] % group == 0 \
        else oq._orig_quantize_rows(W, group)
    if W.shape[0] % group == 0:
        return np.ascontiguousarray(q.T), s
    return q, s


MUTANTS = {"truncates": _mut_truncate, "divides_by_128": _mut_div128,
           "groups_along_rows": _mut_groups_across_rows}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_quant_mutants_are_caught(name, monkeypatch):
    monkeypatch.setattr(oq, "_orig_quantize_rows", oq.quantize_rows, raising=False)
    monkeypatch.setattr(oq, "quantize_rows", MUTANTS[name])
    caught = []
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin(oq)
        except (AssertionError, ValueError, IndexError):
            caught.append(pin.__name__)
    assert caught, f"mutant {name} passed every pin"
