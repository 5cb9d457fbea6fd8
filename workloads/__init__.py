"""Seeded synthetic inputs for the fused gated MLP (shared by the tests, the
benchmark and the oracle's callers).

This module only draws numbers: it holds none of the MLP's arithmetic.  It
turns a (workload, seed) pair into bf16 tensors on the host with the shapes
and value distributions of the decoder layers the workloads stand in for:

* x      ~ N(0, 1)              [M x d]   token rows entering the MLP block
* gamma  = 1 + N(0, 0.1)        [d]       RMSNorm weight
* W_gate ~ N(0, sigma)          [I x d]   nn.Linear layout (out, in)
* W_up   ~ N(0, sigma)          [I x d]
* W_down ~ N(0, sigma)          [d x I]

Every value is drawn as a binary32 normal, scaled in binary32 and rounded to
bf16 (round to nearest, ties to even).  The draw for tensor ``k`` of a
problem with seed ``s`` is split into fixed chunks of 2**22 values; chunk
``c`` comes from numpy's PCG64 seeded with ``SeedSequence([s, k, c])``, so
the bytes do not depend on how many threads fill them.

No trained weights are used: the model names in WORKLOADS only give shapes.
"""

from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass

import numpy as np
import torch

CHUNK = 1 << 22

# tensor ids inside one problem's seed space
TID_X, TID_GAMMA, TID_WGATE, TID_WUP, TID_WDOWN, TID_RESID = 0, 1, 2, 3, 4, 5


@dataclass(frozen=True)
class Workload:
    name: str
    M: int          # token rows
    d: int          # hidden size
    I: int          # intermediate size
    sigma: float    # weight standard deviation
    layers: int = 1  # independent layers (own weights each)

    @property
    def weight_bytes(self) -> int:
        return 6 * self.d * self.I


# The five workload families (token count M, hidden d, intermediate I).
# `layers` independent layers (own weights each) run back to back in one
# step, as a model's layers do: the Phi-3-mini model's 32, and a slice of 4
# (8B) or 2 (70B) layers of the others, so that every workload measures
# layers that follow each other on the GPU rather than one layer per launch.
WORKLOADS = {
    "tiny": Workload("tiny", 4, 256, 688, 0.02),
    "phi3_decode": Workload("phi3_decode", 1, 3072, 8192, 0.02, layers=32),
    "llama8b_decode_m1": Workload("llama8b_decode_m1", 1, 4096, 14336, 0.02, layers=4),
    "llama8b_decode_m8": Workload("llama8b_decode_m8", 8, 4096, 14336, 0.02, layers=4),
    "llama8b_decode_m32": Workload("llama8b_decode_m32", 32, 4096, 14336, 0.02, layers=4),
    "llama70b_verify": Workload("llama70b_verify", 128, 8192, 28672, 0.01, layers=2),
    "llama8b_prefill": Workload("llama8b_prefill", 2048, 4096, 14336, 0.02, layers=2),
}


def _threads() -> int:
    return max(1, min(32, os.cpu_count() or 1))


def normal_f32(seed: int, tid: int, n: int) -> np.ndarray:
    """n standard-normal binary32 values for tensor ``tid`` of problem ``seed``."""
    out = np.empty(n, dtype=np.float32)
    nchunks = (n + CHUNK - 1) // CHUNK

    def fill(c: int) -> None:
        lo = c * CHUNK
        hi = min(n, lo + CHUNK)
        rng = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, tid, c])))
        rng.standard_normal(hi - lo, dtype=np.float32, out=out[lo:hi])

    if nchunks <= 1:
        if n:
            fill(0)
    else:
        with ThreadPoolExecutor(_threads()) as ex:
            list(ex.map(fill, range(nchunks)))
    return out


def normal_bf16(seed: int, tid: int, shape, mean: float = 0.0, std: float = 1.0) -> torch.Tensor:
    """bf16 host tensor of ``shape`` holding round(mean + std * z) with z ~ N(0,1)."""
    n = int(np.prod(shape)) if len(shape) else 1
    z = torch.from_numpy(normal_f32(seed, tid, n))
    if std != 1.0:
        z.mul_(np.float32(std))
    if mean != 0.0:
        z.add_(np.float32(mean))
    return z.to(torch.bfloat16).reshape(shape)


def make_activations(M: int, d: int, seed: int = 0) -> dict:
    """x [M x d] and gamma [d] for one problem."""
    return {
        "x": normal_bf16(seed, TID_X, (M, d)),
        "gamma": normal_bf16(seed, TID_GAMMA, (d,), mean=1.0, std=0.1),
    }


def make_weights(d: int, I: int, sigma: float, seed: int = 0) -> dict:
    """W_gate, W_up [I x d] and W_down [d x I] for one layer."""
    return {
        "W_gate": normal_bf16(seed, TID_WGATE, (I, d), std=sigma),
        "W_up": normal_bf16(seed, TID_WUP, (I, d), std=sigma),
        "W_down": normal_bf16(seed, TID_WDOWN, (d, I), std=sigma),
    }


def make_residual(M: int, d: int, seed: int = 0) -> torch.Tensor:
    """A residual stream [M x d] (bf16), drawn like x but from its own stream."""
    return normal_bf16(seed, TID_RESID, (M, d))


def make_problem(M: int, d: int, I: int, sigma: float = 0.02, seed: int = 0,
                 residual: bool = False) -> dict:
    p = make_activations(M, d, seed)
    p.update(make_weights(d, I, sigma, seed))
    if residual:
        p["residual"] = make_residual(M, d, seed)
    return p


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """The raw bf16 bit patterns of a host tensor, as uint16 (a view, no arithmetic)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)
