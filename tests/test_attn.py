"""Token-phase attention step on the GPU (fmlp_attn_decode) against the oracle
(oracle/attn.py): RoPE at each sequence's position, the GKVC append of the
rotated key and the value at the Eq(2) row, and the attention of every query
head over the held rows and the new one.

Bar (derived from the arithmetic, f32 throughout): every score is a D-term
f32 dot product (relative error ~1e-7 sqrt(D)), the softmax runs in base 2
with the hardware exp2 (relative error ~1e-7) and the sums over up to 4096
rows are f32, so the output should sit within ~1e-6 of the binary64 oracle;
the bar is normwise 1e-4 and per element 1e-3 max|o| (a wrong row, head,
scale or rotation costs 1e-2 and more).  The key written to the cache is
rounded from an f32 rotation on the GPU and from a binary64 one in the
oracle: the two may differ by one bf16 step where the value sits next to a
rounding boundary, so the test asks for every element within one step and
at least 99% of them equal; the value row is copied and must be bit-exact."""

import numpy as np
import pytest
import torch

import oracle
import workloads as wl

pytestmark = pytest.mark.gpu

TOL_NORM, TOL_ELEM = 1e-4, 1e-3


@pytest.fixture(scope="module")
def fm(cuda_device):
    import token_phase_swiglu_b200 as fm
    return fm


def _dec(t):
    return oracle.decode_bf16(wl.bf16_bits(t.cpu()))


def _setup(fm, dev, B, H, H_kv, D, n_max, seed):
    p = wl.make_attn_problem(B, H, H_kv, D, n_max, seed=seed)
    g = {k: v.to(dev) for k, v in p.items()}
    ws = torch.zeros(fm.fmlp_attn_workspace_bytes(B, H, H_kv, D), dtype=torch.uint8, device=dev)
    return p, g, ws


def _step(fm, dev, g, ws, pos, n_ctx, theta, expect=None):
    B, H, D = g["q"].shape
    out = torch.full((B, H, D), float("nan"), dtype=torch.float32, device=dev)
    n0 = fm.fmlp_kernel_launch_count()
    fm.fmlp_attn_decode(g["q"], g["k_new"], g["v_new"], g["k_cache"], g["v_cache"],
                        torch.tensor(pos, dtype=torch.int32, device=dev), n_ctx, theta, out, ws)
    launches = fm.fmlp_kernel_launch_count() - n0
    torch.cuda.synchronize()
    assert fm.fmlp_device_status(ws) == (fm.FMLP_OK if expect is None else expect)
    return out.cpu().double().numpy(), launches


def _oracle(p, pos, theta):
    return oracle.token_attention(_dec(p["q"]), _dec(p["k_new"]), _dec(p["v_new"]),
                                  _dec(p["k_cache"]), _dec(p["v_cache"]), np.asarray(pos), theta)


def _errors(got, ref):
    return (np.linalg.norm(got - ref) / np.linalg.norm(ref),
            np.max(np.abs(got - ref)) / np.max(np.abs(ref)))


def _check_cache(got_k, got_v, ref_k, ref_v, before_k, before_v, pos):
    """Appended rows as the bar above; every other row untouched."""
    for b, pb in enumerate(pos):
        kk, rk = got_k[b, :, pb], ref_k[b, :, pb]
        step = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(rk), 1e-30))) - 7)
        assert np.all(np.abs(kk - rk) <= step * 1.0001), "appended key off by more than a bf16 step"
        assert np.mean(kk == rk) >= 0.99
        assert np.array_equal(got_v[b, :, pb], ref_v[b, :, pb])
        keep = np.ones(got_k.shape[2], bool)
        keep[pb] = False
        assert np.array_equal(got_k[b][:, keep], before_k[b][:, keep])
        assert np.array_equal(got_v[b][:, keep], before_v[b][:, keep])


ATTN_CASES = [
    # B, H, H_kv, D, n_max, n_ctx, positions, theta
    (2, 4, 2, 64, 320, 300, [299, 0], 10000.0),
    (3, 8, 1, 128, 256, 200, [0, 63, 64], 500000.0),          # 8 query heads per KV head
    (1, 32, 32, 96, 1024, 1024, [1023], 10000.0),              # Phi-3-mini heads
    (2, 32, 8, 128, 512, 500, [137, 499], 500000.0),           # Llama-3.1-8B heads
    (4, 4, 4, 96, 130, 130, [129, 1, 64, 65], 10000.0),
    (5, 6, 3, 64, 700, 700, [699, 640, 639, 5, 400], 10000.0),
    (1, 2, 1, 64, 64, 64, [63], 10000.0),
]


@pytest.mark.parametrize("B,H,H_kv,D,n_max,n_ctx,pos,theta", ATTN_CASES)
def test_attn_matches_oracle(fm, cuda_device, B, H, H_kv, D, n_max, n_ctx, pos, theta):
    p, g, ws = _setup(fm, cuda_device, B, H, H_kv, D, n_max, seed=B * 7 + D)
    got, launches = _step(fm, cuda_device, g, ws, pos, n_ctx, theta)
    assert launches == 1
    ref, rk, rv = _oracle(p, pos, theta)
    norm, elem = _errors(got, ref)
    assert norm <= TOL_NORM and elem <= TOL_ELEM, (norm, elem)
    _check_cache(_dec(g["k_cache"]), _dec(g["v_cache"]), rk, rv, _dec(p["k_cache"]),
                 _dec(p["v_cache"]), pos)


@pytest.mark.parametrize("name", ["phi3_attn", "llama8b_attn"])
def test_attn_full_size(fm, cuda_device, name):
    w = wl.ATTN_WORKLOADS[name]
    p, g, ws = _setup(fm, cuda_device, w.B, w.H, w.H_kv, w.D, w.n_max, seed=0)
    pos = [w.n_ctx - 1] * w.B
    got, _ = _step(fm, cuda_device, g, ws, pos, w.n_ctx, w.theta)
    ref, rk, rv = _oracle(p, pos, w.theta)
    norm, elem = _errors(got, ref)
    print(f"{name}: normwise {norm:.2e}, per element {elem:.2e}")
    assert norm <= TOL_NORM and elem <= TOL_ELEM, (norm, elem)
    _check_cache(_dec(g["k_cache"]), _dec(g["v_cache"]), rk, rv, _dec(p["k_cache"]),
                 _dec(p["v_cache"]), pos)


def test_attn_two_steps_read_the_appended_row(fm, cuda_device):
    """The second token attends to the row the first one appended (GKVC: no
    Concat, the cache region is written in place and read back)."""
    B, H, H_kv, D, n_max, theta = 2, 8, 2, 128, 200, 10000.0
    p, g, ws = _setup(fm, cuda_device, B, H, H_kv, D, n_max, seed=41)
    pos1 = [70, 127]
    _step(fm, cuda_device, g, ws, pos1, n_max, theta)
    _, rk1, rv1 = _oracle(p, pos1, theta)
    p2 = wl.make_attn_problem(B, H, H_kv, D, n_max, seed=42)
    for key in ("q", "k_new", "v_new"):
        g[key] = p2[key].to(cuda_device)
    pos2 = [71, 128]
    got, _ = _step(fm, cuda_device, g, ws, pos2, n_max, theta)
    # the oracle's second step runs on the cache it produced itself
    ref, _, _ = oracle.token_attention(_dec(p2["q"]), _dec(p2["k_new"]), _dec(p2["v_new"]),
                                       rk1, rv1, np.asarray(pos2), theta)
    norm, elem = _errors(got, ref)
    assert norm <= TOL_NORM and elem <= TOL_ELEM, (norm, elem)


def test_attn_is_deterministic(fm, cuda_device):
    B, H, H_kv, D, n_max = 3, 16, 4, 128, 1500
    p, g, ws = _setup(fm, cuda_device, B, H, H_kv, D, n_max, seed=5)
    a, _ = _step(fm, cuda_device, g, ws, [1499, 700, 64], n_max, 10000.0)
    b, _ = _step(fm, cuda_device, g, ws, [1499, 700, 64], n_max, 10000.0)
    assert np.array_equal(a, b)   # pieces merged in a fixed order


def test_attn_position_out_of_range(fm, cuda_device):
    """A position at or past n_ctx is reported through the status word; the
    other sequences are still computed, and the bad one's rows stay as they were."""
    B, H, H_kv, D, n_max, n_ctx = 3, 4, 2, 64, 256, 200
    p, g, ws = _setup(fm, cuda_device, B, H, H_kv, D, n_max, seed=9)
    pos = [150, 200, 10]
    got, _ = _step(fm, cuda_device, g, ws, pos, n_ctx, 10000.0, expect=fm.FMLP_ERR_INVALID_ARG)
    ws.zero_()
    ref, _, _ = _oracle(p, [150, 0, 10], 10000.0)
    for b in (0, 2):
        norm, _ = _errors(got[b], ref[b])
        assert norm <= TOL_NORM
    assert np.all(np.isnan(got[1]))
    assert np.array_equal(_dec(g["k_cache"])[1], _dec(p["k_cache"])[1])


def test_attn_bounded_waits(fm, cuda_device):
    """Host-side fault injection withholds each CTA's last stage: the bounded
    waits expire, the call reports FMLP_ERR_TIMEOUT, and after zeroing the
    workspace the next call is correct."""
    B, H, H_kv, D, n_max = 2, 8, 2, 128, 2048
    p, g, ws = _setup(fm, cuda_device, B, H, H_kv, D, n_max, seed=13)
    pos = [2047, 1000]
    try:
        fm.fmlp_set_wait_timeout_ns(2_000_000)
        fm.fmlp_set_fault_injection(1)
        _step(fm, cuda_device, g, ws, pos, n_max, 10000.0, expect=fm.FMLP_ERR_TIMEOUT)
    finally:
        fm.fmlp_set_fault_injection(0)
        fm.fmlp_set_wait_timeout_ns(0)
    ws.zero_()
    got, _ = _step(fm, cuda_device, g, ws, pos, n_max, 10000.0)
    ref, _, _ = _oracle(p, pos, 10000.0)
    norm, elem = _errors(got, ref)
    assert norm <= TOL_NORM and elem <= TOL_ELEM


def test_attn_rejects_what_it_does_not_take(fm, cuda_device):
    L, A = fm.lib, 0x10000
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device=cuda_device)
    W = ws.data_ptr()
    assert L.fmlp_attn_workspace_bytes(1, 32, 32, 80) == 0          # D not taken
    assert L.fmlp_attn_workspace_bytes(1, 12, 8, 64) == 0           # H not a multiple of H_kv
    assert L.fmlp_attn_workspace_bytes(1, 48, 3, 64) == 0           # 16 heads per KV head
    bad = [dict(D=80), dict(n_ctx=300), dict(theta=0.0), dict(theta=float("nan")), dict(n_ctx=0)]
    for kw in bad:
        a = dict(B=1, H=4, H_kv=2, D=64, n_max=256, n_ctx=128, theta=10000.0) | kw
        st = L.fmlp_attn_decode(A, A, A, A, A, A, a["B"], a["H"], a["H_kv"], a["D"], a["n_max"],
                                a["n_ctx"], a["theta"], A, W, 1 << 20, None)
        assert st == fm.FMLP_ERR_INVALID_ARG, kw
