"""fmlp_forward_noalloc: the MLP block for callers that cannot allocate.

Some callers of this library are handed no device allocator -- a plug-in run
by an engine that owns all of device memory, or a serving loop that must not
call cudaMalloc/cudaFree because those can synchronise the device.  For them
fmlp_forward_noalloc runs the same kernels as fmlp_forward on a fixed scratch
buffer that the library keeps on each GPU, so the call needs no workspace.

The GPU tests call it through the C ABI, twice in a row (the second call finds
the buffer as the first one left it), over shapes whose order sends a fused
decode call with a wider d after calls that wrote the intermediate, and check
each output three ways: against the fp64 oracle at the parity bar, against
the oracle with a bf16 intermediate at the tight diagnostic bar, and against
fmlp_forward with a caller workspace at 1e-4 (the same kernels; only the
order of f32 sums differs, see TOL_SAME_KERNELS).  One more test makes a call
time out on purpose (host-controlled fault injection: the producers withhold
their last stage, so the bounded waits expire) and checks that the next call
is correct, because each call clears the buffer's control words first.
This file is collected last on purpose.
"""

import numpy as np
import pytest
import torch

import oracle
import workloads as wl

EPS = 1e-5
TOL_NORM, TOL_ELEM, TIGHT_FRAC = 2e-3, 1e-2, 0.25
# Both entry points run the same kernels, but a gate-up tile split between
# two thread blocks is finished by whichever arrives last, so the f32
# summation order of its accumulators, and with it the bf16 rounding of an
# occasional element of a, can differ from run to run.  One such element
# moves out by about a bf16 step of a / sqrt(M I) of the output norm (2e-5 to
# 4e-5 at these sizes); a dropped share of the contraction or a stale a costs
# orders of magnitude more.
TOL_SAME_KERNELS = 1e-4


def _errors(got, ref):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    return (np.linalg.norm(got - ref) / np.linalg.norm(ref),
            np.max(np.abs(got - ref)) / np.max(np.abs(ref)))


def _oracle(p, residual, intermediate=None):
    b = {k: wl.bf16_bits(v) for k, v in p.items()}
    return oracle.fused_mlp_bf16(b["x"], b["gamma"], EPS, b["W_gate"], b["W_up"], b["W_down"],
                                 residual_bits=b["residual"] if residual else None,
                                 intermediate=intermediate)


def _check_output(got, p, residual, ref_ws):
    ref = _oracle(p, residual)
    tight = _oracle(p, residual, "bf16")
    norm, elem = _errors(got, ref)
    assert norm <= TOL_NORM and elem <= TOL_ELEM, (norm, elem)
    rounding, _ = _errors(tight, ref)
    assert _errors(got, tight)[0] <= TIGHT_FRAC * rounding + 1e-6
    assert _errors(got, ref_ws)[0] <= TOL_SAME_KERNELS


def _setup(fm, dev, M, d, I, residual, seed):
    p = wl.make_problem(M, d, I, sigma=0.02, seed=seed, residual=residual)
    g = {k: v.to(dev) for k, v in p.items()}
    packed = torch.empty(2 * I, d, dtype=torch.bfloat16, device=dev)
    fm.fmlp_pack(g["W_gate"], g["W_up"], 16, packed)
    return p, g, packed


def _with_workspace(fm, dev, g, packed, M, d, I, res):
    ws = torch.zeros(fm.fmlp_workspace_bytes(M, d, I), dtype=torch.uint8, device=dev)
    out = torch.empty(M, d, dtype=torch.float32, device=dev)
    fm.fmlp_forward(g["x"], g["gamma"], EPS, packed, 16, g["W_down"], out, ws, residual=res)
    torch.cuda.synchronize()
    assert fm.fmlp_device_status(ws) == fm.FMLP_OK
    return out.cpu().double().numpy()


def test_noalloc_rejects_oversize_and_invalid_requests():
    # host-side checks only: these return before anything reaches a GPU
    import token_phase_swiglu_b200 as fm
    L, A = fm.lib, 0x10000
    # a prefill-sized intermediate (2048 x 14336 bf16) does not fit the scratch buffer
    assert L.fmlp_workspace_bytes(2048, 4096, 14336) > fm.NOALLOC_SCRATCH_BYTES
    assert L.fmlp_forward_noalloc(A, 2048, A, EPS, A, 16, A, 4096, 14336, None, A, None) == \
        fm.FMLP_ERR_UNSUPPORTED
    # the decode shapes the header lists as fitting do fit, the others do not
    for M, d, I, fits in [(4, 256, 688, True), (1, 3072, 8192, True), (1, 4096, 14336, True),
                          (8, 4096, 14336, True), (32, 4096, 14336, False),
                          (128, 8192, 28672, False)]:
        assert (L.fmlp_workspace_bytes(M, d, I) <= fm.NOALLOC_SCRATCH_BYTES) == fits, (M, d, I)
    assert L.fmlp_forward_noalloc(A, 4, A, 0.0, A, 16, A, 256, 688, None, A, None) == \
        fm.FMLP_ERR_INVALID_ARG
    assert L.fmlp_forward_noalloc(None, 4, A, EPS, A, 16, A, 256, 688, None, A, None) == \
        fm.FMLP_ERR_INVALID_ARG
    assert L.fmlp_forward_noalloc(A, 4, A, EPS, A, 16, A, 250, 688, None, A, None) == \
        fm.FMLP_ERR_INVALID_ARG


@pytest.mark.gpu
@pytest.mark.parametrize("M,d,I,residual", [(1, 3072, 8192, False), (4, 256, 688, True),
                                            (7, 1024, 2064, True), (12, 512, 1024, False),
                                            (8, 4096, 14336, True), (2, 2048, 1024, True)])
def test_noalloc_matches_oracle_and_workspace_entry_point(cuda_device, M, d, I, residual):
    import token_phase_swiglu_b200 as fm
    dev = cuda_device
    assert fm.fmlp_workspace_bytes(M, d, I) <= fm.NOALLOC_SCRATCH_BYTES
    p, g, packed = _setup(fm, dev, M, d, I, residual, seed=31 + M)
    res = g["residual"] if residual else None
    ref_ws = _with_workspace(fm, dev, g, packed, M, d, I, res)
    for call in range(2):
        out = torch.full((M, d), float("nan"), dtype=torch.float32, device=dev)
        fm.fmlp_forward_noalloc(g["x"], g["gamma"], EPS, packed, 16, g["W_down"], out,
                                residual=res)
        torch.cuda.synchronize()
        _check_output(out.cpu().double().numpy(), p, residual, ref_ws)


@pytest.mark.gpu
@pytest.mark.parametrize("M,d,I", [(2, 1024, 2048), (7, 1024, 2048), (4, 4096, 8192)])
def test_noalloc_recovers_after_a_timed_out_call(cuda_device, M, d, I):
    """A call whose bounded waits expire (the fused CUDA-core kernel at M=2,
    the three tensor-core launches at M=7, the one-launch tensor-core layer
    at M=4 on a 201 MB layer) leaves the scratch buffer's control words
    dirty; the next call clears them before its kernels run and is correct."""
    import token_phase_swiglu_b200 as fm
    dev = cuda_device
    p, g, packed = _setup(fm, dev, M, d, I, True, seed=50 + M)
    ref_ws = _with_workspace(fm, dev, g, packed, M, d, I, g["residual"])
    out = torch.empty(M, d, dtype=torch.float32, device=dev)
    try:
        fm.fmlp_set_wait_timeout_ns(2_000_000)
        fm.fmlp_set_fault_injection(1)
        fm.fmlp_forward_noalloc(g["x"], g["gamma"], EPS, packed, 16, g["W_down"], out,
                                residual=g["residual"])
        torch.cuda.synchronize()
    finally:
        fm.fmlp_set_fault_injection(0)
        fm.fmlp_set_wait_timeout_ns(0)
    for _ in range(2):
        out = torch.full((M, d), float("nan"), dtype=torch.float32, device=dev)
        fm.fmlp_forward_noalloc(g["x"], g["gamma"], EPS, packed, 16, g["W_down"], out,
                                residual=g["residual"])
        torch.cuda.synchronize()
        _check_output(out.cpu().double().numpy(), p, True, ref_ws)
