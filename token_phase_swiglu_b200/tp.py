"""Tensor-parallel split of the MLP block (host side).

The block's output is linear in the columns of the intermediate a: with the
intermediate dimension I cut into rank shards, rank r computes the block on
W_gate[i0:i1], W_up[i0:i1] and W_down[:, i0:i1] and gets a partial output;
their sum is the block's output (Eq(1) of "FastTPS: An Optimized Method for
LLM Token Phase for AI Accelerators", xllm-io review, section 三; the
tensor-parallel layers of "Together AI 的推测解码内核融合优化", blog.hotdry.top,
reduce the partial outputs across GPUs before the next norm).  Each shard is
a whole number of interleave tiles, so gate row i and up row i stay on one
rank and the packed shard is the plain fmlp_pack of the shard's rows; shard
widths are also multiples of 64 so that every rank's layer can take the
tensor-core paths.

This module only slices and dispatches; the arithmetic runs in the library's
kernels (fmlp_forward per shard, then fmlp_sum_partials or an NCCL
all-reduce of the f32 partial outputs).
"""

from __future__ import annotations

import torch

from . import (fmlp_forward, fmlp_pack, fmlp_sum_partials, fmlp_workspace_bytes)

__all__ = ["shard_bounds", "shard_layer", "TPShard", "forward_shards_local"]


def shard_bounds(I: int, world: int, align: int = 64) -> list:
    """[(i0, i1)] of each rank: equal shards of the intermediate dimension,
    each a multiple of `align` columns (the interleave tile, and 64 for the
    tensor-core paths)."""
    if world < 1:
        raise ValueError("world must be >= 1")
    if I % (world * align) != 0:
        raise ValueError(f"I = {I} does not split into {world} shards of whole "
                         f"{align}-column blocks")
    w = I // world
    return [(r * w, (r + 1) * w) for r in range(world)]


def shard_layer(W_gate, W_up, W_down, rank: int, world: int, align: int = 64):
    """Rank `rank`'s (W_gate, W_up, W_down) shard, contiguous: rows [i0, i1)
    of W_gate and W_up [I x d], columns [i0, i1) of W_down [d x I].  Works on
    torch tensors and numpy arrays alike (it only slices)."""
    I = W_gate.shape[0]
    i0, i1 = shard_bounds(I, world, align)[rank]
    cont = (lambda t: t.contiguous()) if isinstance(W_gate, torch.Tensor) else \
        (lambda t: t.copy())
    return cont(W_gate[i0:i1]), cont(W_up[i0:i1]), cont(W_down[:, i0:i1])


class TPShard:
    """One rank's share of a layer on the current CUDA device: its packed
    gate/up rows and W_down columns, a workspace and its f32 partial output.

    forward() runs fmlp_forward on the shard (the residual is added by rank 0
    only) and then reduces the partials: with a torch.distributed process
    group, an all-reduce of the f32 partial over it (NCCL on GPUs); out then
    holds the block's output on every rank."""

    def __init__(self, W_gate, W_up, W_down, gamma, rank: int, world: int, tile_T: int = 16,
                 align: int = 64, eps: float = 1e-5):
        dev = torch.device("cuda", torch.cuda.current_device())
        wg, wu, wd = shard_layer(W_gate, W_up, W_down, rank, world, align)
        self.rank, self.world, self.tile_T, self.eps = rank, world, tile_T, eps
        self.d, self.I = wg.shape[1], wg.shape[0]
        self.packed = torch.empty(2 * self.I, self.d, dtype=torch.bfloat16, device=dev)
        fmlp_pack(wg.to(dev), wu.to(dev), tile_T, self.packed)
        self.W_down = wd.to(dev)
        self.gamma = gamma.to(dev)
        self.ws = None

    def partial(self, x, out, residual=None):
        """out (f32 [M x d]) <- this rank's partial output (+ residual on rank 0)."""
        M = x.shape[0]
        need = fmlp_workspace_bytes(M, self.d, self.I)
        if self.ws is None or self.ws.numel() < need:
            self.ws = torch.zeros(need, dtype=torch.uint8, device=x.device)
        fmlp_forward(x, self.gamma, self.eps, self.packed, self.tile_T, self.W_down, out,
                     self.ws, residual=residual if self.rank == 0 else None)

    def forward(self, x, out, residual=None, group=None):
        """out (f32 [M x d]) <- the whole block's output, on every rank."""
        import torch.distributed as dist
        self.partial(x, out, residual)
        if self.world > 1:
            dist.all_reduce(out, op=dist.ReduceOp.SUM, group=group)


def forward_shards_local(shards, x, out, residual=None):
    """All ranks' shards on this one GPU (one process): each shard's partial
    output, then fmlp_sum_partials over them; out is f32 or bf16 [M x d].
    The same reduction kernel reads peer memory when the partials live on
    other GPUs."""
    M, d = x.shape
    parts = [torch.empty(M, d, dtype=torch.float32, device=x.device) for _ in shards]
    for s, p in zip(shards, parts):
        s.partial(x, p)
    fmlp_sum_partials(parts, out, residual=residual)
