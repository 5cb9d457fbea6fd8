"""Host-side logic of bench.py: algorithmic byte counts and the reference arm's JSON line."""

import json
import subprocess
import sys
import os

import bench
import workloads as wl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_algorithmic_bytes_match_the_workload_table():
    # 6dI weights + 2Md x + 2d gamma + 4Md f32 out
    assert bench.algorithmic_bytes(1, 3072, 8192) == 151_019_520
    assert round(bench.algorithmic_bytes(1, 4096, 14336) / 1e6, 2) == 352.35
    assert bench.algorithmic_bytes(32, 4096, 14336) == 353_116_160
    assert round(bench.algorithmic_bytes(128, 8192, 28672) / 1e6, 2) == 1415.59
    assert bench.algorithmic_bytes(2, 8, 8, residual=True) - bench.algorithmic_bytes(2, 8, 8) == 32
    assert bench.gateup_bytes(1, 3072, 8192) == 4 * 3072 * 8192 + 2 * 3072 + 2 * 3072 + 2 * 8192


def test_reference_arm_prints_one_json_line():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--steps", "3", "--warmup", "3"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert out.returncode == 0, out.stderr
    lines = [ln for ln in out.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1
    rec = json.loads(lines[0])
    assert rec["impl"] == "reference" and rec["unit"] == "GB/s" and rec["value"] > 0
    assert rec["cpu_baseline"]["kind"] == "oracle" and rec["cpu_baseline"]["cores"] >= 1
    assert rec["e2e"]["h2d_bytes_per_step"] == 0 and rec["config"]["workload"] == "tiny"


def test_reference_arm_nonzero_ranks_exit_quietly():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny", "--steps", "3", "--warmup", "3"],
                         capture_output=True, text=True, timeout=300, cwd=ROOT, env=env)
    assert out.returncode == 0 and out.stdout.strip() == ""


def test_warmup_floor():
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--warmup", "2"], capture_output=True, text=True, timeout=120, cwd=ROOT)
    assert out.returncode != 0


def test_bench_oracle_check_rows_reach_every_token_tile():
    # all rows up to 128; else rows in every 128-row gate-up and 256-row down
    # token tile, first and last row included
    assert bench.check_rows(128) == list(range(128))
    rows = bench.check_rows(2048)
    assert rows[0] == 0 and rows[-1] == 2047 and len(rows) <= 80
    assert {r // 128 for r in rows} == set(range(16))
    assert {r // 256 for r in rows} == set(range(8))


def test_int8_and_attention_byte_models():
    # int8 layer: codes 3dI + scales 3dI/16 (one f32 per 64) + x, gamma, a, out
    assert bench.q8_bytes(1, 4096, 14336) == 187_203_584
    assert bench.q8_bytes(1, 3072, 8192) == 80_240_640
    # attention step: the held K and V rows (n_ctx - 1 of them) + q, k, v, positions, new rows, out
    w = wl.ATTN_WORKLOADS["llama8b_attn"]
    held = 2 * w.B * w.H_kv * (w.n_ctx - 1) * w.D * 2
    assert bench.attn_bytes(w) == held + w.B * w.H * w.D * 2 + 4 * w.B * w.H_kv * w.D * 2 \
        + 4 * w.B + w.B * w.H * w.D * 4
    assert round(bench.attn_bytes(wl.ATTN_WORKLOADS["phi3_attn"]) / 1e6, 2) == 50.36
    assert w.kv_bytes == 2 * w.B * w.H_kv * w.n_ctx * w.D * 2


def test_default_run_covers_every_workload_family():
    """`--workloads all` (the default) measures the bf16 workloads, the int8 ones
    and the attention step; every kernel with a traffic record has its sources listed."""
    names = list(wl.WORKLOADS) + [n + "_q8" for n in bench.Q8_WORKLOADS] + bench.ATTN_BENCH
    assert {"phi3_decode_q8", "llama8b_decode_m1_q8", "phi3_attn", "llama8b_attn"} <= set(names)
    rec = json.load(open(os.path.join(ROOT, "profiles", "traffic.json")))
    for kernel in rec:
        assert kernel in bench.KERNEL_SOURCES
        for name in bench.KERNEL_SOURCES[kernel]:
            assert os.path.exists(os.path.join(ROOT, "token_phase_swiglu_b200", "csrc", name))
