"""The N > 1 host logic of bench.py, on CPU: two gloo ranks.

The MLP block does not shard across GPUs: bench.py --gpus N runs N independent
replicas (weak scaling) with no collective on the data path.  The only
cross-rank steps are the barriers around the timed region and the max over
ranks of the device time; those run here as world_size-2 gloo process groups.
"""

import json
import os
import socket
import subprocess
import sys

import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    import datetime

    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        # rank r's device time for the timed steps; the slowest rank sets the job time
        elapsed = 10.0 + 5.0 * rank
        worst = bench.reduce_max(elapsed)
        dist.barrier()
        gbs = bench.job_gbs(1_000_000, 4, world, worst)
        q.put((rank, worst, gbs))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_whole_job_throughput():
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
    for rank, worst, gbs in got:
        assert worst == 15.0                      # both ranks see the slowest rank's time
        # 2 replicas x 4 steps x 1 MB over 15 ms
        assert gbs == pytest.approx(2 * 4 * 1_000_000 / 0.015 / 1e9)


def test_reduce_max_without_process_group_is_identity():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.25) == 3.25
    assert bench.job_gbs(2_000_000, 10, 1, 20.0) == pytest.approx(1.0)


def test_reference_arm_under_torchrun_prints_once():
    """bench.py --impl reference launched as two ranks: rank 0 prints one JSON
    line, rank 1 exits 0 without work."""
    port = _free_port()
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr", "127.0.0.1", "--master-port", str(port), "bench.py",
           "--impl", "reference", "--gpus", "2", "--steps", "1", "--warmup", "3",
           "--workload", "tiny"]
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run(cmd, cwd=ROOT, capture_output=True, text=True, timeout=300, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, r.stdout
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == 2
    assert line["cpu_baseline"]["kind"] == "oracle"
