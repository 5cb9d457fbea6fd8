"""int8 weight streaming: this library's int8 format (groups of 64 along K,
one binary32 scale each) and the MLP block on it.

The quantizer must be bit-exact against the oracle's (oracle/quant.py), on
plain and on interleave-packed matrices.  fmlp_forward_q8 must match the
oracle's block on the dequantized weights at the stated bars (normwise
2e-3, per-element 1e-2 max|O_ref|), and the oracle with a rounded to bf16 at
the tight diagnostic bar, for every batch size it takes."""

import numpy as np
import pytest
import torch

import oracle
import workloads as wl

EPS = 1e-5
TOL_NORM, TOL_ELEM, TIGHT_FRAC = 2e-3, 1e-2, 0.25

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def fm(cuda_device):
    import token_phase_swiglu_b200 as fm
    return fm


def _bits(t):
    return wl.bf16_bits(t.cpu())


def _errors(got, ref):
    return (np.linalg.norm(got - ref) / np.linalg.norm(ref),
            np.max(np.abs(got - ref)) / np.max(np.abs(ref)))


def _quantize(fm, W):
    rows, K = W.shape
    q = torch.empty(rows, K, dtype=torch.int8, device=W.device)
    s = torch.empty(rows, K // 64, dtype=torch.float32, device=W.device)
    fm.fmlp_quantize_q8(W, q, s)
    return q, s


@pytest.mark.parametrize("rows,K", [(7, 64), (64, 4096), (256, 14336), (33, 8192)])
def test_quantize_bit_exact(fm, cuda_device, rows, K):
    W = wl.normal_bf16(rows, 2, (rows, K), std=0.02)
    W[0, :64] = 0                     # a group of zeros
    W[1, 5] = 3.0                     # a group with one large weight
    q, s = _quantize(fm, W.to(cuda_device))
    torch.cuda.synchronize()
    q_ref, s_ref = oracle.quantize_rows(oracle.decode_bf16(_bits(W)))
    assert np.array_equal(q.cpu().numpy(), q_ref)
    assert np.array_equal(s.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))


def _run(fm, dev, p, T=16, residual=False, expect=None):
    g = {k: v.to(dev) for k, v in p.items()}
    M, d = g["x"].shape
    I = g["W_gate"].shape[0]
    packed = torch.empty(2 * I, d, dtype=torch.bfloat16, device=dev)
    fm.fmlp_pack(g["W_gate"], g["W_up"], T, packed)
    pq, ps = _quantize(fm, packed)
    dq, ds = _quantize(fm, g["W_down"])
    ws = torch.zeros(fm.fmlp_workspace_bytes(M, d, I), dtype=torch.uint8, device=dev)
    out = torch.full((M, d), float("nan"), dtype=torch.float32, device=dev)
    n0 = fm.fmlp_kernel_launch_count()
    fm.fmlp_forward_q8(g["x"], g["gamma"], EPS, pq, ps, T, dq, ds, out, ws,
                       residual=g["residual"] if residual else None)
    launches = fm.fmlp_kernel_launch_count() - n0
    torch.cuda.synchronize()
    assert fm.fmlp_device_status(ws) == (fm.FMLP_OK if expect is None else expect)
    return out.cpu().double().numpy(), launches


def _oracle(p, residual, intermediate=None):
    b = {k: _bits(v) for k, v in p.items()}
    dec = oracle.decode_bf16
    qs = [oracle.quantize_rows(dec(b[k])) for k in ("W_gate", "W_up", "W_down")]
    return oracle.fused_mlp_q8(dec(b["x"]), dec(b["gamma"]), EPS, *qs[0], *qs[1], *qs[2],
                               residual=dec(b["residual"]) if residual else None,
                               intermediate=intermediate)


def _assert_parity(got, p, residual):
    ref = _oracle(p, residual)
    tight = _oracle(p, residual, "bf16")
    norm, elem = _errors(got, ref)
    assert norm <= TOL_NORM and elem <= TOL_ELEM, (norm, elem)
    rounding, _ = _errors(tight, ref)
    assert _errors(got, tight)[0] <= TIGHT_FRAC * rounding + 1e-6
    return norm


Q8_CASES = [(M, d, I, T) for M in (1, 2, 3, 4)
            for d, I, T in [(512, 1024, 16), (1536, 2560, 8), (4096, 14336, 16)]
            if M * I * 4 <= 200 * 1024]   # a of M rows (f32) in shared memory (4 x 14336: no)


@pytest.mark.parametrize("M,d,I,T", Q8_CASES)
def test_forward_q8(fm, cuda_device, M, d, I, T):
    p = wl.make_problem(M, d, I, sigma=0.02, seed=M * 13 + d, residual=True)
    for residual in (False, True):
        got, launches = _run(fm, cuda_device, p, T=T, residual=residual)
        assert launches == 2
        _assert_parity(got, p, residual)


@pytest.mark.parametrize("name", ["phi3_decode", "llama8b_decode_m1"])
def test_forward_q8_full_size(fm, cuda_device, name):
    w = wl.WORKLOADS[name]
    p = wl.make_problem(w.M, w.d, w.I, sigma=w.sigma, seed=0, residual=True)
    got, _ = _run(fm, cuda_device, p, residual=True)
    norm = _assert_parity(got, p, True)
    print(f"{name} int8 weights: normwise {norm:.3e}")


@pytest.mark.parametrize("M,d,I", [(1, 1024, 2048), (3, 4096, 14336)])
def test_forward_q8_bounded_waits(fm, cuda_device, M, d, I):
    """Host-side fault injection: each CTA's producer withholds its last stage,
    so the consumers' bounded waits (2 ms here) expire; the call reports
    FMLP_ERR_TIMEOUT through the workspace status word, the kernels return,
    and the next call on the same workspace is correct."""
    p = wl.make_problem(M, d, I, sigma=0.02, seed=77 + M, residual=True)
    try:
        fm.fmlp_set_wait_timeout_ns(2_000_000)
        fm.fmlp_set_fault_injection(1)
        _run(fm, cuda_device, p, residual=True, expect=fm.FMLP_ERR_TIMEOUT)
    finally:
        fm.fmlp_set_fault_injection(0)
        fm.fmlp_set_wait_timeout_ns(0)
    got, _ = _run(fm, cuda_device, p, residual=True)
    _assert_parity(got, p, True)


def test_forward_q8_is_deterministic(fm, cuda_device):
    p = wl.make_problem(2, 1024, 2048, seed=3, residual=True)
    a, _ = _run(fm, cuda_device, p, residual=True)
    b, _ = _run(fm, cuda_device, p, residual=True)
    assert np.array_equal(a, b)   # fixed summation order, one writer per element


def test_forward_q8_rejects_what_it_does_not_take(fm, cuda_device):
    dev = cuda_device
    for M, d, I in [(5, 512, 1024), (1, 256, 1024), (1, 512, 640), (4, 4096, 14336)]:
        x = torch.zeros(M, d, dtype=torch.bfloat16, device=dev)
        gamma = torch.ones(d, dtype=torch.bfloat16, device=dev)
        pq = torch.zeros(2 * I, d, dtype=torch.int8, device=dev)
        ps = torch.zeros(2 * I, d // 64, dtype=torch.float32, device=dev)
        dq = torch.zeros(d, I, dtype=torch.int8, device=dev)
        ds = torch.zeros(d, I // 64, dtype=torch.float32, device=dev)
        out = torch.empty(M, d, dtype=torch.float32, device=dev)
        ws = torch.zeros(fm.fmlp_workspace_bytes(M, d, I), dtype=torch.uint8, device=dev)
        with pytest.raises(fm.FmlpError) as e:
            fm.fmlp_forward_q8(x, gamma, EPS, pq, ps, 16, dq, ds, out, ws)
        assert e.value.status == fm.FMLP_ERR_UNSUPPORTED
