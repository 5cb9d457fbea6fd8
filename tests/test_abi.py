"""The C ABI without a GPU: the library loads, exports every symbol the header
declares, and rejects invalid arguments on the host before any CUDA call."""

import ctypes
import os
import re

import pytest

import token_phase_swiglu_b200 as fm

HEADER = os.path.join(os.path.dirname(os.path.dirname(__file__)), "include", "fmlp.h")


def declared_functions():
    src = open(HEADER).read()
    return re.findall(r"FMLP_API\s+[\w\s\*]+?\b(fmlp_\w+)\s*\(", src)


def test_header_declares_the_binding_surface():
    names = declared_functions()
    assert len(names) == len(set(names))
    assert set(names) == set(fm.EXPORTED_SYMBOLS)


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(fm.LIB_PATH)
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_exports_nothing_else_from_the_library():
    # -fvisibility=hidden keeps internal kernels/launchers out of the dynamic table
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", fm.LIB_PATH], capture_output=True,
                         text=True).stdout
    ours = {ln.split()[-1] for ln in out.splitlines() if " T " in ln and "fmlp" in ln}
    assert ours == set(declared_functions())


def test_status_strings():
    for s in range(5):
        assert fm.fmlp_status_string(s).startswith("FMLP_")
    assert "unknown" in fm.fmlp_status_string(99)


def test_workspace_bytes():
    L = fm.lib
    assert L.fmlp_workspace_bytes(4, 256, 688) >= 256 + 4 * 688 * 2
    assert L.fmlp_workspace_bytes(0, 256, 688) >= 256
    assert L.fmlp_workspace_bytes(128, 8192, 28672) >= 128 * 28672 * 2
    # invalid sizes give 0
    assert L.fmlp_workspace_bytes(1, 255, 688) == 0
    assert L.fmlp_workspace_bytes(1, 256, 690) == 0
    assert L.fmlp_workspace_bytes(-1, 256, 688) == 0
    assert L.fmlp_workspace_bytes(1, 65536, 688) == 0
    assert L.fmlp_workspace_bytes(1, 4096, 65544) == 0
    assert L.fmlp_workspace_bytes(1, 32768, 65536) > 0
    for M in (1, 7, 2048):
        assert L.fmlp_workspace_bytes(M, 4096, 14336) % 256 == 0


def test_workspace_covers_the_tensor_core_path_from_two_rows():
    """2-4 rows may run on the tensor cores (large layers, or 4 rows): their
    workspace must hold that path's operand copy and stream-K partials, which
    a single row (always the fused kernel) does not need."""
    L = fm.lib
    tc_shape = L.fmlp_workspace_bytes(2, 4096, 14336)
    no_tc_shape = L.fmlp_workspace_bytes(2, 4096, 14344)  # I % 64 != 0: no tensor-core path
    assert tc_shape > no_tc_shape + (1 << 20)
    assert L.fmlp_workspace_bytes(4, 3072, 8192) > (1 << 20)
    assert L.fmlp_workspace_bytes(1, 4096, 14336) < (1 << 20)


# Fake, 16-byte aligned addresses: every call below fails validation and returns
# before touching the device, so nothing is dereferenced.
A = 0x10000
B = 0x20000
MIS = 0x30008


def _fwd(**kw):
    args = dict(x=A, M=4, gamma=A, eps=1e-5, P=A, T=16, Wd=A, d=256, I=688, res=None, out=B,
                ws=B, wsb=1 << 20, stream=None)
    args.update(kw)
    return fm.lib.fmlp_forward(args["x"], args["M"], args["gamma"], args["eps"], args["P"],
                               args["T"], args["Wd"], args["d"], args["I"], args["res"],
                               args["out"], args["ws"], args["wsb"], args["stream"])


@pytest.mark.parametrize("bad", [
    dict(x=None), dict(gamma=None), dict(P=None), dict(Wd=None), dict(out=None), dict(ws=None),
    dict(x=MIS), dict(out=MIS), dict(res=MIS), dict(ws=MIS),
    dict(eps=0.0), dict(eps=-1e-5), dict(eps=float("inf")), dict(eps=float("nan")),
    dict(T=12), dict(T=0), dict(T=32), dict(d=250), dict(I=690), dict(M=-1),
    dict(wsb=16), dict(d=40000),
])
def test_forward_rejects_invalid_arguments(bad):
    assert _fwd(**bad) == fm.FMLP_ERR_INVALID_ARG


def test_forward_m0_is_a_noop():
    assert _fwd(M=0) == fm.FMLP_OK


def test_pack_rejects_invalid_arguments():
    L = fm.lib
    assert L.fmlp_pack(None, A, 256, 688, 16, B, None) == fm.FMLP_ERR_INVALID_ARG
    assert L.fmlp_pack(A, A + 0x100000, 256, 688, 12, B + 0x10000000, None) == fm.FMLP_ERR_INVALID_ARG
    assert L.fmlp_pack(A, A + 0x100000, 256, 688, 32, B + 0x10000000, None) == fm.FMLP_ERR_INVALID_ARG
    # output overlapping an input
    assert L.fmlp_pack(A, A + 0x100000, 256, 688, 16, A + 0x80, None) == fm.FMLP_ERR_INVALID_ARG
    assert L.fmlp_pack(A, A + 0x100000, 250, 688, 16, B + 0x10000000, None) == fm.FMLP_ERR_INVALID_ARG


def test_stage_calls_reject_invalid_arguments():
    L = fm.lib
    assert L.fmlp_gate_up_swiglu(A, 4, A, 1e-5, A, 16, 256, 688, None, B, 1 << 20, None) == \
        fm.FMLP_ERR_INVALID_ARG
    assert L.fmlp_gate_up_swiglu(A, 4, A, 0.0, A, 16, 256, 688, A, B, 1 << 20, None) == \
        fm.FMLP_ERR_INVALID_ARG
    assert L.fmlp_down_proj(A, 4, A, 256, 688, MIS, B, B, 1 << 20, None) == fm.FMLP_ERR_INVALID_ARG
    assert L.fmlp_down_proj(A, 4, A, 256, 688, None, B, B, 8, None) == fm.FMLP_ERR_INVALID_ARG
    assert L.fmlp_gate_up_swiglu(A, 0, A, 1e-5, A, 16, 256, 688, A, B, 1 << 20, None) == fm.FMLP_OK
    assert L.fmlp_down_proj(A, 0, A, 256, 688, None, B, B, 1 << 20, None) == fm.FMLP_OK
    assert L.fmlp_device_status(None, None) == fm.FMLP_ERR_INVALID_ARG


def test_binding_checks_dtypes():
    import torch
    x = torch.zeros(2, 8, dtype=torch.float32)
    with pytest.raises(TypeError):
        fm.fmlp_pack(x, x, 8, x)


def test_binding_checks_shapes_and_device_before_the_library():
    """The Python wrappers reject a tensor of the wrong dtype (TypeError), shape
    or device (ValueError) before any pointer reaches the C ABI: a short or
    bf16 `out` would otherwise be written past its end."""
    import torch
    d, I, M = 16, 32, 2
    bf = lambda *s: torch.zeros(*s, dtype=torch.bfloat16)
    x, gamma, packed, Wd = bf(M, d), bf(d), bf(2 * I, d), bf(d, I)
    out = torch.zeros(M, d, dtype=torch.float32)
    ws = torch.zeros(1 << 16, dtype=torch.uint8)
    with pytest.raises(TypeError):
        fm.fmlp_forward(x, gamma, 1e-5, packed, 16, Wd, out.to(torch.bfloat16), ws)
    with pytest.raises(ValueError, match="shape"):
        fm.fmlp_forward(x, gamma, 1e-5, packed, 16, Wd, out[:1], ws)
    with pytest.raises(ValueError, match="shape"):
        fm.fmlp_forward(x, bf(d + 8), 1e-5, packed, 16, Wd, out, ws)
    with pytest.raises(ValueError, match="shape"):
        fm.fmlp_forward(x, gamma, 1e-5, bf(I, d), 16, Wd, out, ws)
    with pytest.raises(ValueError, match="shape"):
        fm.fmlp_forward(x, gamma, 1e-5, packed, 16, Wd, out, ws, residual=bf(M + 1, d))
    with pytest.raises(ValueError, match="rows"):
        fm.fmlp_forward(x, gamma, 1e-5, packed, 16, bf(d + 8, I), out, ws)
    with pytest.raises(ValueError, match="CUDA"):     # host memory is not device memory
        fm.fmlp_forward(x, gamma, 1e-5, packed, 16, Wd, out, ws)
    with pytest.raises(ValueError, match="CUDA"):
        fm.fmlp_forward_noalloc(x, gamma, 1e-5, packed, 16, Wd, out)
    with pytest.raises(ValueError, match="shape"):
        fm.fmlp_down_proj(bf(M, I), Wd, out[:, :8], ws)
    with pytest.raises(ValueError, match="shape"):
        fm.fmlp_gate_up_swiglu(x, gamma, 1e-5, packed, 16, bf(M + 1, I), ws)


def test_attention_workspace_and_rejections():
    """fmlp_attn_workspace_bytes / fmlp_attn_decode on the host: the shapes the
    kernel takes, the workspace it needs, and every argument it refuses before
    any CUDA call."""
    L = fm.lib
    # counters (one per sequence x KV head) + one f32 piece (m, l, acc[D]) per head per slot
    n = L.fmlp_attn_workspace_bytes(8, 32, 8, 128)
    assert n >= 256 + 8 * 8 * 4 + (148 + 64) * 4 * (2 + 128) * 4
    assert L.fmlp_attn_workspace_bytes(1, 32, 32, 96) > 0
    for B, H, H_kv, D in [(1, 32, 32, 80), (1, 12, 8, 64), (1, 48, 3, 64), (0, 8, 8, 64),
                          (1, 8, 8, 256), (1, 0, 1, 64)]:
        assert L.fmlp_attn_workspace_bytes(B, H, H_kv, D) == 0, (B, H, H_kv, D)
    W = 0x40000
    good = dict(q=A, k=A, v=A, kc=A, vc=A, pos=A, B=2, H=8, H_kv=2, D=64, n_max=256, n_ctx=200,
                theta=10000.0, out=A, ws=W, wsb=1 << 20)
    bad = [dict(D=80), dict(H=9), dict(n_ctx=300), dict(n_ctx=0), dict(theta=0.0),
           dict(theta=float("inf")), dict(q=None), dict(pos=A + 2), dict(out=MIS), dict(kc=MIS),
           dict(wsb=16), dict(B=0), dict(n_max=1 << 30, B=8, H=8, H_kv=8)]
    for kw in bad:
        a = good | kw
        st = L.fmlp_attn_decode(a["q"], a["k"], a["v"], a["kc"], a["vc"], a["pos"], a["B"], a["H"],
                                a["H_kv"], a["D"], a["n_max"], a["n_ctx"], a["theta"], a["out"],
                                a["ws"], a["wsb"], None)
        assert st == fm.FMLP_ERR_INVALID_ARG, kw


def test_attention_binding_checks_before_the_library():
    import torch
    bf = lambda *s: torch.zeros(*s, dtype=torch.bfloat16)
    B, H, H_kv, D, n_max = 2, 4, 2, 64, 128
    q, kn, vn = bf(B, H, D), bf(B, H_kv, D), bf(B, H_kv, D)
    kc, vc = bf(B, H_kv, n_max, D), bf(B, H_kv, n_max, D)
    pos = torch.zeros(B, dtype=torch.int32)
    out = torch.zeros(B, H, D)
    ws = torch.zeros(fm.fmlp_attn_workspace_bytes(B, H, H_kv, D), dtype=torch.uint8)
    with pytest.raises(TypeError):
        fm.fmlp_attn_decode(q, kn, vn, kc, vc, pos.to(torch.int64), n_max, 1e4, out, ws)
    with pytest.raises(ValueError, match="shape"):
        fm.fmlp_attn_decode(q, kn, vn, kc, bf(B, H_kv, n_max - 1, D), pos, n_max, 1e4, out, ws)
    with pytest.raises(ValueError, match="shape"):
        fm.fmlp_attn_decode(q, bf(B, H, D), vn, kc, vc, pos, n_max, 1e4, out, ws)
    with pytest.raises(ValueError, match="CUDA"):
        fm.fmlp_attn_decode(q, kn, vn, kc, vc, pos, n_max, 1e4, out, ws)
