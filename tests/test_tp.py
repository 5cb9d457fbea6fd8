"""Tensor-parallel split of the MLP block.

CPU: the split itself, against the fp64 oracle -- world_size-2 gloo ranks
each evaluate the oracle on their shard of the intermediate dimension and
all-reduce the partial outputs; the sum equals the oracle on the whole layer
(the block is linear in the columns of a, and rounding a to bf16 is
elementwise, so it holds with the bf16 intermediate too).

GPU (one device, ranks emulated as shards in one process): each shard's
fmlp_forward partial, reduced by fmlp_sum_partials to f32 and to bf16,
against the oracle at the parity bars.
"""

import datetime
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import oracle
import workloads as wl
from token_phase_swiglu_b200 import tp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
EPS = 1e-5


def test_shard_bounds():
    assert tp.shard_bounds(14336, 2) == [(0, 7168), (7168, 14336)]
    assert tp.shard_bounds(28672, 8)[7] == (25088, 28672)
    with pytest.raises(ValueError):
        tp.shard_bounds(688, 2)            # not whole 64-column blocks
    assert tp.shard_bounds(688, 1, align=16) == [(0, 688)]
    wg = np.arange(12 * 2).reshape(12, 2)
    wd = np.arange(2 * 12).reshape(2, 12)
    g, u, d = tp.shard_layer(wg, wg + 100, wd, 1, 3, align=4)
    assert np.array_equal(g, wg[4:8]) and np.array_equal(u, wg[4:8] + 100)
    assert np.array_equal(d, wd[:, 4:8]) and d.flags["C_CONTIGUOUS"]


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle as orc
        import workloads as wlm
        from token_phase_swiglu_b200 import tp as tpm
        M, d, I = 3, 64, 256
        p = wlm.make_problem(M, d, I, sigma=0.05, seed=5, residual=True)
        b = {k: wlm.bf16_bits(v) for k, v in p.items()}
        res = []
        for inter in (None, "bf16"):
            wg, wu, wd = tpm.shard_layer(b["W_gate"], b["W_up"], b["W_down"], rank, world)
            part = orc.fused_mlp_bf16(b["x"], b["gamma"], EPS, wg, wu, wd,
                                      residual_bits=b["residual"] if rank == 0 else None,
                                      intermediate=inter)
            t = torch.from_numpy(part)
            dist.all_reduce(t)
            full = orc.fused_mlp_bf16(b["x"], b["gamma"], EPS, b["W_gate"], b["W_up"],
                                      b["W_down"], residual_bits=b["residual"],
                                      intermediate=inter)
            res.append(float(np.max(np.abs(t.numpy() - full)) / np.max(np.abs(full))))
        q.put((rank, res))
    finally:
        dist.destroy_process_group()


def test_tensor_parallel_split_matches_oracle_on_two_gloo_ranks():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    got = sorted(q.get(timeout=10) for _ in range(world))
    for rank, errs in got:
        assert all(e < 1e-12 for e in errs), (rank, errs)


@pytest.mark.gpu
@pytest.mark.parametrize("M,d,I,world", [(1, 3072, 8192, 4), (8, 4096, 14336, 2),
                                         (32, 1024, 4096, 8), (5, 512, 1024, 2)])
def test_tensor_parallel_shards_on_one_gpu(cuda_device, M, d, I, world):
    import token_phase_swiglu_b200 as fm
    torch.cuda.set_device(cuda_device)
    p = wl.make_problem(M, d, I, sigma=0.02, seed=90 + world, residual=True)
    g = {k: v.to(cuda_device) for k, v in p.items()}
    shards = [tp.TPShard(p["W_gate"], p["W_up"], p["W_down"], p["gamma"], r, world)
              for r in range(world)]
    b = {k: wl.bf16_bits(v) for k, v in p.items()}
    ref = oracle.fused_mlp_bf16(b["x"], b["gamma"], EPS, b["W_gate"], b["W_up"], b["W_down"],
                                residual_bits=b["residual"])
    out = torch.empty(M, d, dtype=torch.float32, device=cuda_device)
    tp.forward_shards_local(shards, g["x"], out, residual=g["residual"])
    torch.cuda.synchronize()
    # the same partials reduced to f32 and to bf16 (a second run of the shards
    # would add into its outputs in another order)
    parts = [torch.empty(M, d, dtype=torch.float32, device=cuda_device) for _ in shards]
    for sh, pt in zip(shards, parts):
        sh.partial(g["x"], pt)
    out32 = torch.empty(M, d, dtype=torch.float32, device=cuda_device)
    out16 = torch.empty(M, d, dtype=torch.bfloat16, device=cuda_device)
    fm.fmlp_sum_partials(parts, out32, residual=g["residual"])
    fm.fmlp_sum_partials(parts, out16, residual=g["residual"])
    torch.cuda.synchronize()
    got = out.cpu().double().numpy()
    norm = np.linalg.norm(got - ref) / np.linalg.norm(ref)
    elem = np.max(np.abs(got - ref)) / np.max(np.abs(ref))
    assert norm <= 2e-3 and elem <= 1e-2, (norm, elem)
    # the bf16 output is the f32 sum rounded once
    rounded = out32.cpu().to(torch.bfloat16).double().numpy()
    assert np.array_equal(oracle.decode_bf16(wl.bf16_bits(out16.cpu())), rounded)
    got32 = out32.cpu().double().numpy()
    assert np.linalg.norm(got32 - ref) / np.linalg.norm(ref) <= 2e-3
    for s in shards:
        assert fm.fmlp_device_status(s.ws) == fm.FMLP_OK


@pytest.mark.gpu
def test_sum_partials_rejects_overlap_and_sizes(cuda_device):
    import token_phase_swiglu_b200 as fm
    a = torch.zeros(4, 64, dtype=torch.float32, device=cuda_device)
    b = torch.zeros(4, 64, dtype=torch.float32, device=cuda_device)
    fm.fmlp_sum_partials([a, b], a)      # an f32 out may be one of the partials
    with pytest.raises(fm.FmlpError):    # but a bf16 out may not overlap them
        fm.fmlp_sum_partials([a, b], a.view(torch.bfloat16).view(-1)[:256].view(4, 64))
    with pytest.raises(fm.FmlpError):    # more than 16 partials
        fm.fmlp_sum_partials([a] * 17, b)
    torch.cuda.synchronize()
