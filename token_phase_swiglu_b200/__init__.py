"""Python binding of libfmlp.so, the B200 fused gated-MLP library.

Argument marshalling only: every step of the computation runs in the CUDA
kernels behind the C ABI declared in ``include/fmlp.h``.  Tensors are torch
CUDA tensors (torch provides device memory and streams); the functions pass
their device pointers and sizes through ctypes and raise ``FmlpError`` on any
status other than FMLP_OK.  There is no fallback: if the shared library has
not been built, importing this package raises ImportError.
"""

from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "FmlpError", "FMLP_OK", "FMLP_ERR_INVALID_ARG", "FMLP_ERR_UNSUPPORTED", "FMLP_ERR_CUDA",
    "FMLP_ERR_TIMEOUT", "LIB_PATH", "lib", "fmlp_pack", "fmlp_workspace_bytes", "fmlp_forward",
    "fmlp_gate_up_swiglu", "fmlp_down_proj", "fmlp_device_status", "fmlp_status_string",
    "fmlp_last_cuda_error", "fmlp_kernel_launch_count", "fmlp_set_wait_timeout_ns", "fmlp_set_fault_injection",
    "fmlp_forward_noalloc", "NOALLOC_SCRATCH_BYTES", "EXPORTED_SYMBOLS", "fmlp_forward_bf16",
    "fmlp_sum_partials", "fmlp_quantize_q8", "fmlp_forward_q8", "Q8_GROUP",
    "fmlp_attn_workspace_bytes", "fmlp_attn_decode",
]

FMLP_OK, FMLP_ERR_INVALID_ARG, FMLP_ERR_UNSUPPORTED, FMLP_ERR_CUDA, FMLP_ERR_TIMEOUT = range(5)

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libfmlp.so")

_i64, _sz, _vp, _int, _f32 = ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_int, ctypes.c_float

# name -> (restype, argtypes); mirrors include/fmlp.h
_SIGNATURES = {
    "fmlp_pack": (_int, [_vp, _vp, _i64, _i64, _int, _vp, _vp]),
    "fmlp_workspace_bytes": (_sz, [_i64, _i64, _i64]),
    "fmlp_forward": (_int, [_vp, _i64, _vp, _f32, _vp, _int, _vp, _i64, _i64, _vp, _vp, _vp, _sz, _vp]),
    "fmlp_gate_up_swiglu": (_int, [_vp, _i64, _vp, _f32, _vp, _int, _i64, _i64, _vp, _vp, _sz, _vp]),
    "fmlp_down_proj": (_int, [_vp, _i64, _vp, _i64, _i64, _vp, _vp, _vp, _sz, _vp]),
    "fmlp_device_status": (_int, [_vp, _vp]),
    "fmlp_status_string": (ctypes.c_char_p, [_int]),
    "fmlp_last_cuda_error": (_int, []),
    "fmlp_kernel_launch_count": (ctypes.c_uint64, []),
    "fmlp_set_wait_timeout_ns": (None, [ctypes.c_uint64]),
    "fmlp_set_fault_injection": (None, [_int]),
    "fmlp_forward_noalloc": (_int, [_vp, _i64, _vp, _f32, _vp, _int, _vp, _i64, _i64, _vp, _vp, _vp]),
    "fmlp_forward_bf16": (_int, [_vp, _i64, _vp, _f32, _vp, _int, _vp, _i64, _i64, _vp, _vp, _vp, _sz, _vp]),
    "fmlp_sum_partials": (_int, [ctypes.POINTER(_vp), _int, _i64, _i64, _vp, _vp, _int, _vp]),
    "fmlp_quantize_q8": (_int, [_vp, _i64, _i64, _vp, _vp, _vp]),
    "fmlp_forward_q8": (_int, [_vp, _i64, _vp, _f32, _vp, _vp, _int, _vp, _vp, _i64, _i64, _vp, _vp, _vp, _sz, _vp]),
    "fmlp_attn_workspace_bytes": (_sz, [_i64, _int, _int, _int]),
    "fmlp_attn_decode": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _int, _int, _int, _i64, _i64, _f32,
                                _vp, _vp, _sz, _vp]),
}
EXPORTED_SYMBOLS = tuple(_SIGNATURES)


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with `python -c 'import __graft_entry__ as g; g.build()'` "
            "(nvcc, sm_100a). There is no non-CUDA implementation.")
    handle = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(handle, name)
        fn.restype = res
        fn.argtypes = args
    return handle


lib = _load()


class FmlpError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib.fmlp_status_string(status).decode()
        if status == FMLP_ERR_CUDA:
            msg += f" (cudaError {lib.fmlp_last_cuda_error()})"
        super().__init__(f"{where}: {msg}")


def _check_status(status: int, where: str) -> None:
    if status != FMLP_OK:
        raise FmlpError(status, where)


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    if not t.is_contiguous():
        raise ValueError("tensors passed to libfmlp must be contiguous")
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


def _bf16(t, name):
    if t is not None and t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16, got {t.dtype}")


def _check(t, name, dtype, shape=None, optional=False):
    """Check one tensor argument before its pointer goes to the library: the
    dtype (TypeError), the exact shape and contiguity (ValueError).  Together
    with _on_device (the library launches on the current device), nothing
    malformed reaches the C ABI."""
    if t is None:
        if optional:
            return
        raise ValueError(f"{name} is required")
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor, got {type(t).__name__}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _on_device(**tensors):
    """Every given tensor lives on the current CUDA device (checked after the
    dtypes and shapes of all of them)."""
    for name, t in tensors.items():
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if t.device.index != torch.cuda.current_device():
            raise ValueError(f"{name} is on {t.device}, but the current device is "
                             f"cuda:{torch.cuda.current_device()}")


def _check_workspace(ws, need: int):
    _check(ws, "workspace", None)
    if ws.numel() * ws.element_size() < need:
        raise ValueError(f"workspace holds {ws.numel() * ws.element_size()} bytes, "
                         f"{need} needed")


def _dims2(t, name):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch tensor, got {type(t).__name__}")
    if t.dim() != 2:
        raise ValueError(f"{name} must be 2-D, got shape {tuple(t.shape)}")
    return t.shape


def _check_forward_args(x, gamma, packed, W_down, out, residual):
    """Shapes of the MLP block's tensors: (M, d, I)."""
    _bf16(x, "x")
    M, d = _dims2(x, "x")
    _bf16(W_down, "W_down")
    d2, I = _dims2(W_down, "W_down")
    if d2 != d:
        raise ValueError(f"W_down has {d2} rows, x has {d} columns")
    _check(x, "x", torch.bfloat16, (M, d))
    _check(gamma, "gamma", torch.bfloat16, (d,))
    _check(packed, "packed", torch.bfloat16, (2 * I, d))
    _check(W_down, "W_down", torch.bfloat16, (d, I))
    _check(residual, "residual", torch.bfloat16, (M, d), optional=True)
    return M, d, I


def fmlp_status_string(status: int) -> str:
    return lib.fmlp_status_string(status).decode()


def fmlp_last_cuda_error() -> int:
    return lib.fmlp_last_cuda_error()


def fmlp_kernel_launch_count() -> int:
    return int(lib.fmlp_kernel_launch_count())


def fmlp_set_wait_timeout_ns(ns: int) -> None:
    """Deadline of the kernels' bounded waits (0 = default, one second)."""
    lib.fmlp_set_wait_timeout_ns(int(ns))


def fmlp_set_fault_injection(mode: int) -> None:
    """Testing aid: nonzero makes kernels withhold their last stage (bounded waits expire)."""
    lib.fmlp_set_fault_injection(int(mode))


def fmlp_workspace_bytes(M: int, d: int, I: int) -> int:
    return int(lib.fmlp_workspace_bytes(M, d, I))


def fmlp_pack(W_gate, W_up, tile_T: int, packed, stream=None) -> None:
    """packed [2I x d] <- rows of W_gate / W_up [I x d] interleaved at tile tile_T."""
    _bf16(W_gate, "W_gate"); _bf16(W_up, "W_up"); _bf16(packed, "packed")
    I, d = _dims2(W_gate, "W_gate")
    _check(W_gate, "W_gate", torch.bfloat16, (I, d))
    _check(W_up, "W_up", torch.bfloat16, (I, d))
    _check(packed, "packed", torch.bfloat16, (2 * I, d))
    _on_device(W_gate=W_gate, W_up=W_up, packed=packed)
    _check_status(lib.fmlp_pack(_ptr(W_gate), _ptr(W_up), d, I, tile_T, _ptr(packed),
                                _stream(stream)), "fmlp_pack")


def fmlp_forward(x, gamma, eps: float, packed, tile_T: int, W_down, out, workspace,
                 residual=None, stream=None) -> None:
    """out [M x d] (f32) <- RMSNorm + gated MLP (+ residual) of x [M x d]."""
    M, d, I = _check_forward_args(x, gamma, packed, W_down, out, residual)
    _check(out, "out", torch.float32, (M, d))
    _check_workspace(workspace, fmlp_workspace_bytes(M, d, I))
    _on_device(x=x, gamma=gamma, packed=packed, W_down=W_down, residual=residual, out=out,
               workspace=workspace)
    _check_status(lib.fmlp_forward(_ptr(x), M, _ptr(gamma), eps, _ptr(packed), tile_T,
                                   _ptr(W_down), d, I, _ptr(residual), _ptr(out), _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(stream)),
                  "fmlp_forward")


def fmlp_forward_bf16(x, gamma, eps: float, packed, tile_T: int, W_down, out, workspace,
                      residual=None, stream=None) -> None:
    """out [M x d] (bf16) <- bf16(RMSNorm + gated MLP of x + residual): the output
    chained layers feed to each other.  out may be x or residual itself."""
    M, d, I = _check_forward_args(x, gamma, packed, W_down, out, residual)
    _check(out, "out", torch.bfloat16, (M, d))
    _check_workspace(workspace, fmlp_workspace_bytes(M, d, I))
    _on_device(x=x, gamma=gamma, packed=packed, W_down=W_down, residual=residual, out=out,
               workspace=workspace)
    _check_status(lib.fmlp_forward_bf16(_ptr(x), M, _ptr(gamma), eps, _ptr(packed), tile_T,
                                        _ptr(W_down), d, I, _ptr(residual), _ptr(out),
                                        _ptr(workspace),
                                        workspace.numel() * workspace.element_size(),
                                        _stream(stream)),
                  "fmlp_forward_bf16")


def fmlp_sum_partials(partials, out, residual=None, stream=None) -> None:
    """out [M x d] <- sum of the f32 partial outputs [M x d] (+ residual), out f32 or
    bf16: the reduction of a tensor-parallel MLP block (partials may be peer memory)."""
    if not partials:
        raise ValueError("at least one partial output is needed")
    M, d = _dims2(partials[0], "partials[0]")
    for r, t in enumerate(partials):
        _check(t, f"partials[{r}]", torch.float32, (M, d))
    if out.dtype not in (torch.float32, torch.bfloat16):
        raise TypeError(f"out must be float32 or bfloat16, got {out.dtype}")
    _check(out, "out", out.dtype, (M, d))
    _check(residual, "residual", torch.bfloat16, (M, d), optional=True)
    _on_device(out=out, residual=residual)
    arr = (_vp * len(partials))(*[t.data_ptr() for t in partials])
    _check_status(lib.fmlp_sum_partials(arr, len(partials), M, d, _ptr(residual), _ptr(out),
                                        int(out.dtype == torch.bfloat16), _stream(stream)),
                  "fmlp_sum_partials")


Q8_GROUP = 64   # elements per scale of the int8 weight format (include/fmlp.h)


def fmlp_quantize_q8(W, q, scales, stream=None) -> None:
    """q int8 [rows x K], scales f32 [rows x K/64] <- the int8 format of W bf16 [rows x K]."""
    _bf16(W, "W")
    rows, K = _dims2(W, "W")
    _check(W, "W", torch.bfloat16, (rows, K))
    _check(q, "q", torch.int8, (rows, K))
    _check(scales, "scales", torch.float32, (rows, K // Q8_GROUP))
    _on_device(W=W, q=q, scales=scales)
    _check_status(lib.fmlp_quantize_q8(_ptr(W), rows, K, _ptr(q), _ptr(scales), _stream(stream)),
                  "fmlp_quantize_q8")


def fmlp_forward_q8(x, gamma, eps: float, packed_q, packed_scales, tile_T: int, W_down_q,
                    W_down_scales, out, workspace, residual=None, stream=None) -> None:
    """out [M x d] (f32) <- the MLP block of x on int8 weights (fmlp_quantize_q8's)."""
    _bf16(x, "x")
    M, d = _dims2(x, "x")
    d2, I = _dims2(W_down_q, "W_down_q")
    if d2 != d:
        raise ValueError(f"W_down_q has {d2} rows, x has {d} columns")
    _check(x, "x", torch.bfloat16, (M, d))
    _check(gamma, "gamma", torch.bfloat16, (d,))
    _check(packed_q, "packed_q", torch.int8, (2 * I, d))
    _check(packed_scales, "packed_scales", torch.float32, (2 * I, d // Q8_GROUP))
    _check(W_down_q, "W_down_q", torch.int8, (d, I))
    _check(W_down_scales, "W_down_scales", torch.float32, (d, I // Q8_GROUP))
    _check(residual, "residual", torch.bfloat16, (M, d), optional=True)
    _check(out, "out", torch.float32, (M, d))
    _check_workspace(workspace, fmlp_workspace_bytes(M, d, I))
    _on_device(x=x, gamma=gamma, packed_q=packed_q, packed_scales=packed_scales,
               W_down_q=W_down_q, W_down_scales=W_down_scales, residual=residual, out=out,
               workspace=workspace)
    _check_status(lib.fmlp_forward_q8(_ptr(x), M, _ptr(gamma), eps, _ptr(packed_q),
                                      _ptr(packed_scales), tile_T, _ptr(W_down_q),
                                      _ptr(W_down_scales), d, I, _ptr(residual), _ptr(out),
                                      _ptr(workspace),
                                      workspace.numel() * workspace.element_size(),
                                      _stream(stream)),
                  "fmlp_forward_q8")


def fmlp_attn_workspace_bytes(B: int, H: int, H_kv: int, D: int) -> int:
    n = lib.fmlp_attn_workspace_bytes(B, H, H_kv, D)
    if n == 0:
        raise FmlpError(FMLP_ERR_INVALID_ARG, "fmlp_attn_workspace_bytes: shape not taken")
    return n


def fmlp_attn_decode(q, k_new, v_new, k_cache, v_cache, pos, n_ctx: int, theta: float, out,
                     workspace, stream=None) -> None:
    """One token-phase attention step (RoPE, in-place KV append, attention over
    the cache rows 0..pos); see include/fmlp.h for the layouts."""
    _bf16(q, "q")
    if q.dim() != 3 or k_cache.dim() != 4:
        raise ValueError("q must be [B, H, D] and the caches [B, H_kv, n_max, D]")
    B, H, D = q.shape
    H_kv, n_max = k_cache.shape[1], k_cache.shape[2]
    _check(q, "q", torch.bfloat16, (B, H, D))
    _check(k_new, "k_new", torch.bfloat16, (B, H_kv, D))
    _check(v_new, "v_new", torch.bfloat16, (B, H_kv, D))
    _check(k_cache, "k_cache", torch.bfloat16, (B, H_kv, n_max, D))
    _check(v_cache, "v_cache", torch.bfloat16, (B, H_kv, n_max, D))
    _check(pos, "pos", torch.int32, (B,))
    _check(out, "out", torch.float32, (B, H, D))
    _check_workspace(workspace, fmlp_attn_workspace_bytes(B, H, H_kv, D))
    _on_device(q=q, k_new=k_new, v_new=v_new, k_cache=k_cache, v_cache=v_cache, pos=pos, out=out,
               workspace=workspace)
    _check_status(lib.fmlp_attn_decode(_ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache),
                                       _ptr(v_cache), _ptr(pos), B, H, H_kv, D, n_max, n_ctx,
                                       theta, _ptr(out), _ptr(workspace),
                                       workspace.numel() * workspace.element_size(),
                                       _stream(stream)),
                  "fmlp_attn_decode")


NOALLOC_SCRATCH_BYTES = 8 << 20   # FMLP_NOALLOC_SCRATCH_BYTES in include/fmlp.h


def fmlp_forward_noalloc(x, gamma, eps: float, packed, tile_T: int, W_down, out, residual=None,
                         stream=None) -> None:
    """fmlp_forward without a workspace, for callers that cannot allocate device
    memory (the library's own fixed scratch buffer is used; see include/fmlp.h)."""
    M, d, I = _check_forward_args(x, gamma, packed, W_down, out, residual)
    _check(out, "out", torch.float32, (M, d))
    _on_device(x=x, gamma=gamma, packed=packed, W_down=W_down, residual=residual, out=out)
    _check_status(lib.fmlp_forward_noalloc(_ptr(x), M, _ptr(gamma), eps, _ptr(packed), tile_T,
                                           _ptr(W_down), d, I, _ptr(residual), _ptr(out),
                                           _stream(stream)),
                  "fmlp_forward_noalloc")


def fmlp_gate_up_swiglu(x, gamma, eps: float, packed, tile_T: int, a, workspace,
                        stream=None) -> None:
    """a [M x I] (bf16) <- SiLU(gate) * up of RMSNorm(x) against packed gate/up rows."""
    _bf16(x, "x"); _bf16(a, "a")
    M, d = _dims2(x, "x")
    _, I = _dims2(a, "a")
    _check(x, "x", torch.bfloat16, (M, d))
    _check(gamma, "gamma", torch.bfloat16, (d,))
    _check(packed, "packed", torch.bfloat16, (2 * I, d))
    _check(a, "a", torch.bfloat16, (M, I))
    _check_workspace(workspace, fmlp_workspace_bytes(M, d, I))
    _on_device(x=x, gamma=gamma, packed=packed, a=a, workspace=workspace)
    _check_status(lib.fmlp_gate_up_swiglu(_ptr(x), M, _ptr(gamma), eps, _ptr(packed), tile_T, d,
                                          I, _ptr(a), _ptr(workspace),
                                          workspace.numel() * workspace.element_size(),
                                          _stream(stream)),
                  "fmlp_gate_up_swiglu")


def fmlp_down_proj(a, W_down, out, workspace, residual=None, stream=None) -> None:
    """out [M x d] (f32) <- a [M x I] W_down^T (+ residual)."""
    _bf16(a, "a"); _bf16(W_down, "W_down")
    M, I = _dims2(a, "a")
    d, _ = _dims2(W_down, "W_down")
    _check(a, "a", torch.bfloat16, (M, I))
    _check(W_down, "W_down", torch.bfloat16, (d, I))
    _check(residual, "residual", torch.bfloat16, (M, d), optional=True)
    _check(out, "out", torch.float32, (M, d))
    _check_workspace(workspace, fmlp_workspace_bytes(M, d, I))
    _on_device(a=a, W_down=W_down, residual=residual, out=out, workspace=workspace)
    _check_status(lib.fmlp_down_proj(_ptr(a), M, _ptr(W_down), d, I, _ptr(residual), _ptr(out),
                                     _ptr(workspace), workspace.numel() * workspace.element_size(),
                                     _stream(stream)),
                  "fmlp_down_proj")


def fmlp_device_status(workspace, stream=None) -> int:
    """Synchronise, read and clear the workspace's device status word; returns the status."""
    _check(workspace, "workspace", None)
    _on_device(workspace=workspace)
    return int(lib.fmlp_device_status(_ptr(workspace), _stream(stream)))
