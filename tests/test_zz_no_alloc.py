"""fmlp_forward_noalloc: the MLP block for callers that cannot allocate.

Some callers of this library are handed no device allocator -- a plug-in run
by an engine that owns all of device memory, or a serving loop that must not
call cudaMalloc/cudaFree because those can synchronise the device.  For them
fmlp_forward_noalloc runs the same kernels as fmlp_forward on a fixed scratch
buffer that the library keeps on each GPU, so the call needs no workspace.

The GPU test checks it through the C ABI against fmlp_forward with a
caller-allocated workspace, on two calls in a row (the second call finds the
buffer as the first one left it), over shapes whose order sends a fused
decode call with a wider d after calls that wrote the intermediate.  This file is collected last on purpose.
"""

import numpy as np
import pytest
import torch

import workloads as wl

EPS = 1e-5
TOL_NORM, TOL_ELEM = 2e-3, 1e-2


def _errors(got, ref):
    got, ref = np.asarray(got, np.float64), np.asarray(ref, np.float64)
    return (np.linalg.norm(got - ref) / np.linalg.norm(ref),
            np.max(np.abs(got - ref)) / np.max(np.abs(ref)))


def test_noalloc_rejects_oversize_and_invalid_requests():
    # host-side checks only: these return before anything reaches a GPU
    import token_phase_swiglu_b200 as fm
    L, A = fm.lib, 0x10000
    # a prefill-sized intermediate (2048 x 14336 bf16) does not fit the scratch buffer
    assert L.fmlp_workspace_bytes(2048, 4096, 14336) > fm.NOALLOC_SCRATCH_BYTES
    assert L.fmlp_forward_noalloc(A, 2048, A, EPS, A, 16, A, 4096, 14336, None, A, None) == \
        fm.FMLP_ERR_UNSUPPORTED
    assert L.fmlp_forward_noalloc(A, 4, A, 0.0, A, 16, A, 256, 688, None, A, None) == \
        fm.FMLP_ERR_INVALID_ARG
    assert L.fmlp_forward_noalloc(None, 4, A, EPS, A, 16, A, 256, 688, None, A, None) == \
        fm.FMLP_ERR_INVALID_ARG
    assert L.fmlp_forward_noalloc(A, 4, A, EPS, A, 16, A, 250, 688, None, A, None) == \
        fm.FMLP_ERR_INVALID_ARG


@pytest.mark.gpu
@pytest.mark.parametrize("M,d,I,residual", [(1, 3072, 8192, False), (4, 256, 688, True),
                                            (7, 1024, 2064, True), (12, 512, 1024, False),
                                            (2, 2048, 1024, True)])
def test_noalloc_matches_workspace_entry_point(cuda_device, M, d, I, residual):
    import token_phase_swiglu_b200 as fm
    dev = cuda_device
    assert fm.fmlp_workspace_bytes(M, d, I) <= fm.NOALLOC_SCRATCH_BYTES
    p = wl.make_problem(M, d, I, sigma=0.02, seed=31 + M, residual=residual)
    g = {k: v.to(dev) for k, v in p.items()}
    res = g["residual"] if residual else None
    packed = torch.empty(2 * I, d, dtype=torch.bfloat16, device=dev)
    fm.fmlp_pack(g["W_gate"], g["W_up"], 16, packed)
    ws = torch.zeros(fm.fmlp_workspace_bytes(M, d, I), dtype=torch.uint8, device=dev)
    ref = torch.empty(M, d, dtype=torch.float32, device=dev)
    fm.fmlp_forward(g["x"], g["gamma"], EPS, packed, 16, g["W_down"], ref, ws, residual=res)
    torch.cuda.synchronize()
    assert fm.fmlp_device_status(ws) == fm.FMLP_OK
    ref_np = ref.cpu().double().numpy()
    for call in range(2):
        out = torch.full((M, d), float("nan"), dtype=torch.float32, device=dev)
        fm.fmlp_forward_noalloc(g["x"], g["gamma"], EPS, packed, 16, g["W_down"], out,
                                residual=res)
        torch.cuda.synchronize()
        norm, elem = _errors(out.cpu().double().numpy(), ref_np)
        assert norm <= TOL_NORM and elem <= TOL_ELEM, (call, norm, elem)
