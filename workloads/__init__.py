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

The token-phase attention workloads (ATTN_WORKLOADS) draw, from tensor ids of
their own: the new token's q [B x H x D], k and v [B x H_kv x D], and the
KV-cache regions [B x H_kv x N_max x D] that earlier tokens filled, all
N(0, 1) in bf16 (unit-variance projections, so scores q.k/sqrt(D) are of
order one); every sequence's new token sits at position n_ctx - 1.
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
TID_Q, TID_KNEW, TID_VNEW, TID_KCACHE, TID_VCACHE = 6, 7, 8, 9, 10


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


@dataclass(frozen=True)
class AttnWorkload:
    name: str
    B: int          # sequences, one new token each
    H: int          # query heads
    H_kv: int       # KV heads (H / H_kv queries share one)
    D: int          # head dimension
    n_ctx: int      # rows held after the step (the new token is row n_ctx - 1)
    n_max: int      # rows of each head's cache region (N_p + N_r)
    theta: float    # RoPE base
    layers: int = 1  # independent layers (own caches each)

    @property
    def kv_bytes(self) -> int:
        """K and V rows the step reads (bf16), the new row included."""
        return 2 * self.B * self.H_kv * self.n_ctx * self.D * 2


# Shapes of the attention side of the same models: Phi-3-mini-4k (32 heads of
# 96, no grouping, a full 4k context) and Llama-3.1-8B (32 query heads over 8
# KV heads of 128) with eight 4k sequences in flight.
ATTN_WORKLOADS = {
    "attn_tiny": AttnWorkload("attn_tiny", 2, 4, 2, 64, 300, 320, 10000.0),
    "phi3_attn": AttnWorkload("phi3_attn", 1, 32, 32, 96, 4096, 4096, 10000.0, layers=32),
    "llama8b_attn": AttnWorkload("llama8b_attn", 8, 32, 8, 128, 4096, 4096, 500000.0, layers=8),
}


def make_attn_problem(B: int, H: int, H_kv: int, D: int, n_max: int, seed: int = 0) -> dict:
    """q, k_new, v_new and the two cache regions of one attention step (bf16, host)."""
    return {
        "q": normal_bf16(seed, TID_Q, (B, H, D)),
        "k_new": normal_bf16(seed, TID_KNEW, (B, H_kv, D)),
        "v_new": normal_bf16(seed, TID_VNEW, (B, H_kv, D)),
        "k_cache": normal_bf16(seed, TID_KCACHE, (B, H_kv, n_max, D)),
        "v_cache": normal_bf16(seed, TID_VCACHE, (B, H_kv, n_max, D)),
    }

