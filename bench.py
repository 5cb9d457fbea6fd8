#!/usr/bin/env python3
"""Benchmark of the fused gated-MLP hot path on B200.

One step = the whole MLP block (RMSNorm -> interleaved gate-up -> SiLU*up ->
down projection) over one batch of token rows for every layer of the
workload, through the library's C ABI.  Default workload: a Phi-3-mini-shaped
decode layer (M=1, d=3072, I=8192, bf16) over 32 independent layers' weights,
4.8 GB of weights per GPU, far beyond the 126 MB L2, so no L2 flush is needed.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
  python bench.py --impl reference ...     # the fp64 CPU oracle, timed alone

Multi-GPU: launched by torch.distributed.run, one rank per GPU; the path has
no exchange step, so every rank runs its own replica of the workload (weak
scaling) and the reported time is the max over ranks.

Prints one JSON line on rank 0.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import workloads as wl  # noqa: E402

EPS = 1e-5
TILE_T = 16
METRIC = "fused-MLP weight-stream GB/s (% B200 HBM peak) and tokens/s per layer at 1 GPU"
# decode workloads also measured on this library's int8 weights (entries "<name>_q8")
Q8_WORKLOADS = ["phi3_decode", "llama8b_decode_m1"]
# the token-phase attention step on the same models' attention shapes
ATTN_BENCH = ["phi3_attn", "llama8b_attn"]
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_BF16_TFLOPS_SUSTAINED = 1400.0


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------

def algorithmic_bytes(M: int, d: int, I: int, residual: bool = False) -> int:
    """Bytes the MLP block must move once: weights 6dI, x 2Md, gamma 2d, out 4Md (+ residual 2Md)."""
    return 6 * d * I + 2 * M * d + 2 * d + 4 * M * d + (2 * M * d if residual else 0)


def q8_bytes(M: int, d: int, I: int) -> int:
    """Algorithmic bytes of the block on int8 weights: 3dI int8 weights and one f32
    scale per 64 of them, x 2Md, gamma 2d, out 4Md."""
    return 3 * d * I + 3 * d * I // 64 * 4 + 2 * M * d + 2 * d + 4 * M * d


def gateup_bytes(M: int, d: int, I: int) -> int:
    """Algorithmic bytes of the gate-up kernel: packed weights 4dI, x, gamma, a written 2MI."""
    return 4 * d * I + 2 * M * d + 2 * d + 2 * M * I


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            return json.load(f)
    except (OSError, ValueError):
        return {}


# the source files each kernel is built from (its traffic record goes stale
# when any of them changes)
KERNEL_SOURCES = {
    "fused_decode": ["stream.cu", "ring.cuh", "common.cuh", "internal.h"],
    "q8_stream": ["q8.cu", "ring.cuh", "common.cuh", "internal.h"],
    "attn_decode": ["attn.cu", "ring.cuh", "common.cuh", "internal.h", "tmap.cu", "tmap.h"],
    "tc_gemm": ["tc.cu", "tcgen05.cuh", "common.cuh", "internal.h", "tmap.cu", "tmap.h"],
    "tc_layer": ["layer.cu", "tcgen05.cuh", "common.cuh", "internal.h", "tmap.cu", "tmap.h"],
}


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "token_phase_swiglu_b200", "csrc")
    for name in KERNEL_SOURCES[kernel]:
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode() + f.read())
    return h.hexdigest()[:16]


def recorded_traffic(kernel: str, workload: str):
    """DRAM bytes per launch from the committed ncu summary, if taken on this kernel source."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(kernel, {}).get(workload)
    except (OSError, ValueError):
        return None
    if not rec or kernel not in KERNEL_SOURCES or rec.get("source_hash") != kernel_source_hash(kernel):
        return None
    return rec.get("dram_bytes_per_launch")


class ClockSampler:
    """Samples SM clock and throttle reasons through NVML while the GPU works."""

    REASONS = {
        "gpu_idle": 0x1, "applications_clocks_setting": 0x2, "sw_power_cap": 0x4,
        "hw_slowdown": 0x8, "sync_boost": 0x10, "sw_thermal_slowdown": 0x20,
        "hw_thermal_slowdown": 0x40, "hw_power_brake_slowdown": 0x80,
        "display_clock_setting": 0x100,
    }

    def __init__(self, device_index: int, period_s: float = 0.002):
        self.samples = []
        self.reasons = 0
        self.max_mhz = None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        self._handle = None
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            if not uuid.startswith("GPU-"):
                uuid = "GPU-" + uuid
            self._nvml = pynvml
            self._handle = pynvml.nvmlDeviceGetHandleByUUID(uuid.encode())
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._handle, pynvml.NVML_CLOCK_SM)
        except Exception as e:  # noqa: BLE001 -- clocks are reported as unavailable
            self.error = repr(e)
            self._handle = None

    def _run(self):
        nv = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self._handle, nv.NVML_CLOCK_SM))
                self.reasons |= nv.nvmlDeviceGetCurrentClocksEventReasons(self._handle)
            except Exception:  # noqa: BLE001
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._handle is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
        return self

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self) -> dict:
        if self._handle is None or not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"],
                    "samples": 0}
        names = sorted(n for n, bit in self.REASONS.items() if self.reasons & bit)
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": names, "samples": len(self.samples)}


def dist_env():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def reduce_max(v: float, device=None) -> float:
    """The maximum of `v` over all ranks (the value itself without a process group)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return v
    t = torch.tensor([v], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbs(bytes_per_step_per_rank: int, steps: int, world: int, elapsed_ms: float) -> float:
    """Whole-job throughput: the bytes every replica streamed over the slowest
    rank's device time (replicas do equal work, so weak scaling)."""
    return bytes_per_step_per_rank * steps * world / (elapsed_ms / 1e3) / 1e9


def host_cores() -> int:
    """Host cores this process may run on."""
    try:
        return len(os.sched_getaffinity(0))
    except (AttributeError, OSError):
        return os.cpu_count() or 1


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:  # noqa: BLE001
        return os.cpu_count() or 1


# ----------------------------------------------------------------------------
# the fp64 oracle as a CPU baseline (a bounded sample of the workload)
# ----------------------------------------------------------------------------

def layer_bits(w: wl.Workload, seed: int, layer: int) -> dict:
    act = wl.make_activations(w.M, w.d, seed=seed)
    wts = wl.make_weights(w.d, w.I, w.sigma, seed=seed + layer)
    return {k: wl.bf16_bits(v) for k, v in {**act, **wts}.items()}


def oracle_call(w: wl.Workload, b: dict, ic: int, keep: bool = False):
    """One oracle evaluation of the MLP block on an I-slice of `ic` columns.

    Gate/up/down columns are independent terms of Eq(1), so a slice of the
    intermediate dimension is a proportional share of the layer's work.
    Returns (algorithmic bytes, seconds), and the output if `keep`.
    """
    import oracle
    wg, wu = b["W_gate"][:ic], b["W_up"][:ic]
    wd = np.ascontiguousarray(b["W_down"][:, :ic])
    t0 = time.perf_counter()
    out = oracle.fused_mlp_bf16(b["x"], b["gamma"], EPS, wg, wu, wd)
    dt = time.perf_counter() - t0
    if keep:
        return algorithmic_bytes(w.M, w.d, ic), dt, out
    return algorithmic_bytes(w.M, w.d, ic), dt


def oracle_sample(w: wl.Workload, seconds: float, seed: int = 0):
    """The oracle on whole layers of the workload for about `seconds` of CPU time.

    Returns (GB/s, description, the oracle's output of layer 0): layer 0 has
    the same inputs as the benchmark's first layer, so its output checks the
    timed kernels' result."""
    done, t_total, calls, ref0 = 0, 0.0, 0, None
    while True:
        b = layer_bits(w, seed, calls % w.layers)
        if calls == 0:
            nb, dt, ref0 = oracle_call(w, b, w.I, keep=True)
        else:
            nb, dt = oracle_call(w, b, w.I)
        done += nb
        t_total += dt
        calls += 1
        if t_total >= seconds:
            break
    desc = (f"{calls} whole layer(s) of {w.name} (M={w.M}, d={w.d}, I={w.I}) through the fp64 "
            f"oracle (bf16 decode + numpy), {t_total:.1f} s")
    return done / t_total / 1e9, desc, ref0


def run_reference(args) -> None:
    rank, world, _ = dist_env()
    if rank != 0:
        return
    w = wl.WORKLOADS[args.workload]
    b = layer_bits(w, 0, 0)
    # size one step so that warm-up + timed steps finish within about two minutes
    budget = 120.0 / max(1, args.steps + args.warmup)
    _, t_full = oracle_call(w, b, w.I)
    ic = w.I
    if t_full > budget:
        ic = min(w.I, max(8, int(w.I * budget / t_full) // 8 * 8))
    for _ in range(args.warmup):
        oracle_call(w, b, ic)
    t, nbytes = 0.0, 0
    for _ in range(args.steps):
        nb, dt = oracle_call(w, b, ic)
        t += dt
        nbytes += nb
    gbs = nbytes / t / 1e9
    cores = blas_threads()
    sample = (f"each step: the fp64 oracle (bf16 decode + numpy) on layer 0 of {w.name} "
              f"(M={w.M}, d={w.d}) restricted to an I-slice of {ic} of {w.I} columns")
    line = {
        "impl": "reference", "metric": METRIC, "value": round(gbs, 4), "unit": "GB/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(t / args.steps * 1e3, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": config_of(w, args),
        "cpu_baseline": {"value": round(gbs, 4), "unit": "GB/s", "cores": cores,
                         "host_cores": host_cores(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": round(gbs, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def config_of(w: wl.Workload, args) -> dict:
    layers = getattr(args, "layers", 0) or w.layers
    return {"workload": w.name, "M": w.M, "d": w.d, "I": w.I, "layers": layers,
            "tile_T": TILE_T, "dtype_in": "bf16", "out": "f32",
            "weights_per_gpu_GB": round(layers * 6 * w.d * w.I / 1e9, 3),
            "l2": "no flush: weights streamed per step exceed the 126 MB L2",
            "parallelism": f"replicas x{args.gpus}"}


# ----------------------------------------------------------------------------
# the CUDA path
# ----------------------------------------------------------------------------

def check_rows(M: int) -> list:
    """Token rows compared with the oracle inside the benchmark: all of them up
    to 128, else 64 spread over every token tile plus the last row (the
    parity tests compare every row)."""
    if M <= 128:
        return list(range(M))
    return sorted(set(range(0, M, max(1, M // 64))) | {M - 1})


class WorkloadRun:
    """One workload resident on the GPU: every layer's packed gate/up and
    W_down (+ gamma), the token rows x, one output slice per layer and a
    workspace; step() runs the whole hot path once through the C ABI."""

    def __init__(self, fm, w: wl.Workload, dev, seed0: int, layers: int = 0, quant: bool = False):
        self.fm, self.w, self.dev, self.quant = fm, w, dev, quant
        self.M, self.d, self.I = w.M, w.d, w.I
        self.L = layers or w.layers
        self.seed0 = seed0
        self.act = wl.make_activations(w.M, w.d, seed=seed0)
        self.x = self.act["x"].to(dev)
        self.outs = torch.empty(self.L, w.M, w.d, dtype=torch.float32, device=dev)
        self.layers = []
        for l in range(self.L):
            wts = wl.make_weights(w.d, w.I, w.sigma, seed=seed0 + l)
            gamma = wl.normal_bf16(seed0 + l, wl.TID_GAMMA, (w.d,), mean=1.0, std=0.1).to(dev)
            wg, wu = wts["W_gate"].to(dev), wts["W_up"].to(dev)
            packed = torch.empty(2 * w.I, w.d, dtype=torch.bfloat16, device=dev)
            fm.fmlp_pack(wg, wu, TILE_T, packed)
            torch.cuda.synchronize()
            del wg, wu
            layer = {"packed": packed, "W_down": wts["W_down"].to(dev), "gamma": gamma,
                     "out": self.outs[l]}
            if quant:   # this library's int8 format of the packed gate/up rows and W_down
                for k in ("packed", "W_down"):
                    W = layer.pop(k)
                    q = torch.empty(W.shape, dtype=torch.int8, device=dev)
                    sc = torch.empty(W.shape[0], W.shape[1] // fm.Q8_GROUP, dtype=torch.float32,
                                     device=dev)
                    fm.fmlp_quantize_q8(W, q, sc)
                    layer[k + "_q"], layer[k + "_s"] = q, sc
                torch.cuda.synchronize()
            self.layers.append(layer)
        self.ws = torch.zeros(fm.fmlp_workspace_bytes(w.M, w.d, w.I), dtype=torch.uint8,
                              device=dev)
        self.stream = torch.cuda.current_stream()
        self.graph = None
        self.per_step = None

    def step(self, x=None, outs=None, stream=None):
        fm = self.fm
        x = self.x if x is None else x
        for li, ly in enumerate(self.layers):
            out = ly["out"] if outs is None else outs[li]
            if self.quant:
                fm.fmlp_forward_q8(x, ly["gamma"], EPS, ly["packed_q"], ly["packed_s"], TILE_T,
                                   ly["W_down_q"], ly["W_down_s"], out, self.ws, stream=stream)
            else:
                fm.fmlp_forward(x, ly["gamma"], EPS, ly["packed"], TILE_T, ly["W_down"], out,
                                self.ws, stream=stream)

    def capture(self, warmup: int, use_graph: bool = True) -> None:
        """Warm-up from the host (also the library's one-time set-up, before
        any capture), then a CUDA graph of one step."""
        fm = self.fm
        for _ in range(max(1, warmup)):
            self.step()
        torch.cuda.synchronize()
        if not use_graph:
            return
        try:
            self.graph = torch.cuda.CUDAGraph()
            c0 = fm.fmlp_kernel_launch_count()
            with torch.cuda.graph(self.graph):
                self.step()
            self.per_step = fm.fmlp_kernel_launch_count() - c0
            torch.cuda.synchronize()
            for _ in range(warmup):
                self.graph.replay()
            torch.cuda.synchronize()
        except Exception as e:  # noqa: BLE001 -- report and launch from the host instead
            print(f"bench: CUDA graph capture failed ({e}); launching from the host",
                  file=sys.stderr)
            self.graph = None
            torch.cuda.synchronize()

    def run_steps(self, n: int) -> None:
        for _ in range(n):
            if self.graph is not None:
                self.graph.replay()
            else:
                self.step()

    def timed(self, steps: int, barrier, max_over_ranks) -> tuple:
        """Device time of exactly `steps` steps between CUDA events on the
        launching stream, with a barrier and a synchronize on both sides, max
        over ranks; clocks sampled during it.  Returns (ms, launches, clocks)."""
        fm = self.fm
        sampler = ClockSampler(self.dev.index)
        launches0 = fm.fmlp_kernel_launch_count()
        with sampler:
            barrier()
            torch.cuda.synchronize()
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(self.stream)
            self.run_steps(steps)
            e1.record(self.stream)
            torch.cuda.synchronize()
            barrier()
        ms = max_over_ranks(e0.elapsed_time(e1))
        launches = fm.fmlp_kernel_launch_count() - launches0
        if self.graph is not None:
            launches = self.per_step * steps   # each replay launches the captured kernels
        return ms, launches, sampler.summary()

    def step_estimate_ms(self) -> float:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(self.stream)
        self.run_steps(3)
        e1.record(self.stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / 3

    def isolated_calls(self, steps: int, max_over_ranks) -> dict:
        """Per-call durations, each call bracketed by events on the launching
        stream: fmlp_forward, then the same step through the two stage calls."""
        fm, stream, L = self.fm, self.stream, self.L
        a_buf = torch.empty(self.M, self.I, dtype=torch.bfloat16, device=self.dev)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(L)]
        fw_ms = []
        for _ in range(steps):
            for ly, (a0, a1) in zip(self.layers, ev):
                a0.record(stream)
                fm.fmlp_forward(self.x, ly["gamma"], EPS, ly["packed"], TILE_T, ly["W_down"],
                                ly["out"], self.ws, stream=stream)
                a1.record(stream)
            torch.cuda.synchronize()
            fw_ms.extend(a0.elapsed_time(a1) for a0, a1 in ev)
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(L)]
        gu_ms, dn_ms = [], []
        for _ in range(steps):
            for ly, (a0, a1, a2) in zip(self.layers, ev):
                a0.record(stream)
                fm.fmlp_gate_up_swiglu(self.x, ly["gamma"], EPS, ly["packed"], TILE_T, a_buf,
                                       self.ws, stream=stream)
                a1.record(stream)
                fm.fmlp_down_proj(a_buf, ly["W_down"], ly["out"], self.ws, stream=stream)
                a2.record(stream)
            torch.cuda.synchronize()
            for a0, a1, a2 in ev:
                gu_ms.append(a0.elapsed_time(a1))
                dn_ms.append(a1.elapsed_time(a2))
        return {"fmlp_forward_ms": max_over_ranks(statistics.mean(fw_ms)),
                "fmlp_gate_up_swiglu_ms": max_over_ranks(statistics.mean(gu_ms)),
                "fmlp_down_proj_ms": max_over_ranks(statistics.mean(dn_ms))}

    def e2e(self, steps: int, barrier, max_over_ranks) -> tuple:
        """The same step end to end, the way a serving loop runs it: every step
        copies its input from pinned host memory and its outputs (every layer's
        out) back to pinned host memory, both on copy streams and
        double-buffered, so that step i's copies overlap the layers of its
        neighbours.  The timed region starts before the first input copy and
        ends after the last output copy.  Returns (ms, h2d bytes, d2h bytes)."""
        dev, stream, L, M, d = self.dev, self.stream, self.L, self.M, self.d
        x_host = self.act["x"].pin_memory()
        outs_host = [torch.empty(L, M, d, dtype=torch.float32).pin_memory() for _ in range(2)]
        x_dev = [torch.empty_like(self.x) for _ in range(2)]
        outs_dev = [self.outs, torch.empty_like(self.outs)]
        copy_in, copy_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_step(i):
            b = i & 1
            copy_in.wait_event(ev_done[b])       # step i - 2 has read x_dev[b]
            with torch.cuda.stream(copy_in):
                x_dev[b].copy_(x_host, non_blocking=True)
            ev_in[b].record(copy_in)
            stream.wait_event(ev_in[b])
            stream.wait_event(ev_out[b])         # step i - 2's outputs have left outs_dev[b]
            self.step(x=x_dev[b], outs=outs_dev[b], stream=stream)
            ev_done[b].record(stream)
            copy_out.wait_event(ev_done[b])
            with torch.cuda.stream(copy_out):
                outs_host[b].copy_(outs_dev[b], non_blocking=True)
            ev_out[b].record(copy_out)

        e2e_step(0)
        e2e_step(1)
        torch.cuda.synchronize()
        barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        copy_in.wait_stream(stream)
        for i in range(steps):
            e2e_step(i)
        stream.wait_event(ev_out[0])
        stream.wait_event(ev_out[1])
        f1.record(stream)
        torch.cuda.synchronize()
        barrier()
        # the last pass wrote layer 0's output of buffer 0 last when steps is even
        self.outs_last = outs_dev[(steps - 1) & 1]
        return (max_over_ranks(f0.elapsed_time(f1)), x_host.numel() * x_host.element_size(),
                outs_host[0].numel() * outs_host[0].element_size())

    def release(self) -> None:
        self.graph = None
        self.layers = []
        self.outs = self.outs_last = None
        torch.cuda.synchronize()
        torch.cuda.empty_cache()


def peaks_of(sustained: bool = False) -> tuple:
    """(HBM GB/s, source), (bf16 TFLOP/s, source): the measured copy bandwidth
    and cuBLAS bf16 throughput, the burst figure for a kernel timed alone and
    the sustained one (seconds under the power cap) for work timed for a
    second or more."""
    peaks = measured_peaks()
    if "hbm_gbs" in peaks:
        hbm = (float(peaks["hbm_gbs"]), "measured")
    else:
        hbm = (FALLBACK_HBM_GBS, "fallback")
    key = "bf16_tflops_sustained" if sustained and "bf16_tflops_sustained" in peaks else \
        "bf16_tflops"
    if key in peaks:
        tc = (float(peaks[key]), "measured" + (" sustained" if key.endswith("sustained") else
                                                " burst"))
    else:
        tc = (FALLBACK_BF16_TFLOPS_SUSTAINED if sustained else FALLBACK_BF16_TFLOPS, "fallback")
    return hbm, tc


def roofline_entry(run: WorkloadRun, ms_step: float, gu_ms, sustained: bool = False) -> dict:
    """The dominant kernel against its roofline.  One kernel per layer (the
    single-launch paths): its average launch duration is the timed region over
    the launches in it.  Otherwise the gate-up call, timed with events around
    each isolated call (it includes the small prologue kernel)."""
    M, d, I, L, w = run.M, run.d, run.I, run.L, run.w
    (peak, peak_src), (tpeak, tpeak_src) = peaks_of(sustained)
    single = run.per_step is not None and run.per_step == L
    if run.quant:
        # the int8 path: two launches per layer, both weight streams
        kname, kms = "q8_stream", ms_step / L
        timing = "timed region / layers (two launches per layer, back to back in a CUDA graph)"
        kbytes, kflops = q8_bytes(M, d, I), 6 * M * d * I
    elif single:
        kname = "fused_decode" if M <= 4 else "tc_layer"
        kms = ms_step / L
        timing = "timed region / launches (the step's only kernel, back to back in a CUDA graph)"
        kbytes, kflops = algorithmic_bytes(M, d, I), 6 * M * d * I
    else:
        kname, kms = "gate-up (fmlp_gate_up_swiglu)", gu_ms
        timing = "isolated: events around each call"
        kbytes, kflops = gateup_bytes(M, d, I), 4 * M * d * I
    if kflops / kbytes > tpeak * 1e12 / (peak * 1e9):
        bound, kpeak, src, unit, work = "tensor", tpeak, tpeak_src, "TFLOP/s", kflops
    else:
        bound, kpeak, src, unit, work = "hbm", peak, peak_src, "GB/s", kbytes
    achieved = work / (kms / 1e3) / (1e12 if unit == "TFLOP/s" else 1e9)
    # DRAM bytes of one layer (the two int8 launches summed) or of the gate-up launch
    traffic = recorded_traffic(
        kname if kname in ("fused_decode", "tc_layer", "q8_stream") else "tc_gemm",
        w.name + ("_q8" if run.quant else ""))
    return {"bound": bound, "kernel": kname, "achieved": round(achieved, 2), "peak": kpeak,
            "peak_source": src, "unit": unit, "frac": round(achieved / kpeak, 4),
            "traffic": traffic, "algorithmic_per_launch": work, "avg_launch_ms": round(kms, 5),
            "launch_timing": timing}


def oracle_check(run: WorkloadRun, got_outs) -> dict:
    """The timed kernels' output of layer 0 (written by the last end-to-end
    pass, same inputs) against the oracle on the rows of check_rows."""
    w = run.w
    rows = check_rows(w.M)
    b = layer_bits(w, run.seed0, 0)
    import oracle
    t0 = time.perf_counter()
    if run.quant:   # the block on the dequantized int8 weights (quantization included)
        dec = oracle.decode_bf16
        qs = [oracle.quantize_rows(dec(b[k])) for k in ("W_gate", "W_up", "W_down")]
        ref = oracle.fused_mlp_q8(dec(b["x"][rows]), dec(b["gamma"]), EPS, *qs[0], *qs[1],
                                  *qs[2])
    else:
        ref = oracle.fused_mlp_bf16(b["x"][rows], b["gamma"], EPS, b["W_gate"], b["W_up"],
                                    b["W_down"])
    dt = time.perf_counter() - t0
    got = got_outs[0].cpu().double().numpy()[rows]
    norm = float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-300))
    elem = float(np.max(np.abs(got - ref)) / max(np.max(np.abs(ref)), 1e-300))
    nbytes = (q8_bytes if run.quant else algorithmic_bytes)(len(rows), w.d, w.I)
    run.cpu_baseline = {
        "value": round(nbytes / dt / 1e9, 4), "unit": "GB/s", "cores": blas_threads(),
        "host_cores": host_cores(), "kind": "oracle",
        "sample": f"this check: layer 0, {len(rows)} token row(s), through the fp64 oracle, {dt:.2f} s"}
    return {"layer": 0, "rows": len(rows), "normwise": float(f"{norm:.3e}"),
            "per_element": float(f"{elem:.3e}"), "within_bar": bool(norm <= 2e-3 and elem <= 1e-2)}


def measure_sub_workload(fm, w: wl.Workload, dev, args, barrier, max_over_ranks, rank: int,
                         world: int, quant: bool = False) -> dict:
    """One entry of the line's `workloads` object: the workload timed for at
    least --min-seconds of device time, its own clocks, roofline, end-to-end
    pass and oracle check (quant: on this library's int8 weights)."""
    run = WorkloadRun(fm, w, dev, seed0=1000 * rank, quant=quant)
    run.capture(args.warmup, use_graph=not args.no_graph)
    est = run.step_estimate_ms()
    steps = max(args.steps, int(np.ceil(args.min_seconds * 1e3 / max(est, 1e-3))))
    ms, launches, clocks = run.timed(steps, barrier, max_over_ranks)
    ms_step = ms / steps
    gu_ms = None
    if not quant and not (run.per_step is not None and run.per_step == run.L):
        gu_ms = run.isolated_calls(max(3, min(20, steps)), max_over_ranks)["fmlp_gate_up_swiglu_ms"]
    e2e_steps = max(2, min(4000, int(np.ceil(0.5e3 / max(est, 1e-3)))))
    e2e_ms, h2d, d2h = run.e2e(e2e_steps, barrier, max_over_ranks)
    bytes_step = run.L * (q8_bytes(w.M, w.d, w.I) if quant else algorithmic_bytes(w.M, w.d, w.I))
    (peak, _), (tpeak, _) = peaks_of(sustained=True)
    gbs = job_gbs(bytes_step, steps, world, ms)
    tflops = 6 * w.M * w.d * w.I * run.L * steps * world / (ms / 1e3) / 1e12
    wbytes = run.L * (q8_bytes(w.M, w.d, w.I) - q8_bytes(w.M, w.d, 0) if quant else w.weight_bytes)
    entry = {
        "config": {"M": w.M, "d": w.d, "I": w.I, "layers": run.L, "tile_T": TILE_T,
                   "weights": "int8, one f32 scale per 64 (this library's format)" if quant
                   else "bf16", "weights_per_gpu_GB": round(wbytes / 1e9, 3)},
        "value": round(gbs, 2), "unit": "GB/s", "hbm_frac": round(gbs / world / peak, 4),
        "tflops": round(tflops, 2), "tensor_frac": round(tflops / world / tpeak, 4),
        "tokens_per_s_per_layer": round(w.M * run.L * steps * world / (ms / 1e3), 1),
        "ms_per_layer": round(ms_step / run.L, 5), "steps": steps, "timed_ms": round(ms, 2),
        "roofline": roofline_entry(run, ms_step, gu_ms, sustained=True),
        "e2e": {"value": round(job_gbs(bytes_step, e2e_steps, world, e2e_ms), 2), "unit": "GB/s",
                "steps": e2e_steps, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches, "cuda_graph": run.graph is not None,
        "device_status": fm.fmlp_status_string(fm.fmlp_device_status(run.ws)),
        "clocks": clocks,
    }
    if rank == 0 and not args.no_oracle_check:
        entry["check_vs_oracle"] = oracle_check(run, run.outs_last)
        entry["cpu_baseline"] = run.cpu_baseline
    run.release()
    return entry


def attn_bytes(w: wl.AttnWorkload) -> int:
    """Algorithmic bytes of one attention step of one layer: the held K and V
    rows read, the new rows written, q / k / v / positions read and out written."""
    B, H, Hk, D = w.B, w.H, w.H_kv, w.D
    return (2 * B * Hk * (w.n_ctx - 1) * D * 2 + B * H * D * 2 + 2 * B * Hk * D * 2 + 4 * B
            + 2 * B * Hk * D * 2 + B * H * D * 4)


class AttnRun:
    """One attention workload resident on the GPU: every layer's K and V cache
    regions, the new token's q / k / v and positions, one output per layer;
    step() runs fmlp_attn_decode once per layer."""

    def __init__(self, fm, w: wl.AttnWorkload, dev, seed0: int):
        self.fm, self.w, self.dev, self.L = fm, w, dev, w.layers
        p0 = wl.make_attn_problem(w.B, w.H, w.H_kv, w.D, w.n_max, seed=seed0)
        self.host = p0                                  # layer 0's inputs, for the oracle
        self.q, self.k_new, self.v_new = (p0[k].to(dev) for k in ("q", "k_new", "v_new"))
        self.pos_host = torch.full((w.B,), w.n_ctx - 1, dtype=torch.int32)
        self.pos = self.pos_host.to(dev)
        self.caches = [(p0["k_cache"].to(dev), p0["v_cache"].to(dev))]
        for l in range(1, self.L):
            pl = wl.make_attn_problem(w.B, w.H, w.H_kv, w.D, w.n_max, seed=seed0 + l)
            self.caches.append((pl["k_cache"].to(dev), pl["v_cache"].to(dev)))
        self.outs = torch.empty(self.L, w.B, w.H, w.D, dtype=torch.float32, device=dev)
        self.ws = torch.zeros(fm.fmlp_attn_workspace_bytes(w.B, w.H, w.H_kv, w.D),
                              dtype=torch.uint8, device=dev)
        self.stream = torch.cuda.current_stream()
        self.graph, self.per_step, self.outs_last = None, None, None

    def step(self, ins=None, outs=None, stream=None):
        q, k, v, pos = ins if ins is not None else (self.q, self.k_new, self.v_new, self.pos)
        outs = self.outs if outs is None else outs
        for l, (kc, vc) in enumerate(self.caches):
            self.fm.fmlp_attn_decode(q, k, v, kc, vc, pos, self.w.n_ctx, self.w.theta, outs[l],
                                     self.ws, stream=stream)

    capture = WorkloadRun.capture
    run_steps = WorkloadRun.run_steps
    timed = WorkloadRun.timed
    step_estimate_ms = WorkloadRun.step_estimate_ms

    def e2e(self, steps: int, barrier, max_over_ranks) -> tuple:
        """As WorkloadRun.e2e: every step copies q, k, v and the positions in
        from pinned host memory and every layer's out back, double-buffered on
        copy streams.  Returns (ms, h2d bytes, d2h bytes)."""
        stream = self.stream
        host_in = [t.pin_memory() for t in (self.host["q"], self.host["k_new"], self.host["v_new"],
                                            self.pos_host)]
        dev_in = [[torch.empty_like(t, device=self.dev) for t in host_in] for _ in range(2)]
        outs_host = [torch.empty(self.outs.shape, dtype=torch.float32).pin_memory()
                     for _ in range(2)]
        outs_dev = [self.outs, torch.empty_like(self.outs)]
        copy_in, copy_out = torch.cuda.Stream(self.dev), torch.cuda.Stream(self.dev)
        ev_in = [torch.cuda.Event() for _ in range(2)]
        ev_done = [torch.cuda.Event() for _ in range(2)]
        ev_out = [torch.cuda.Event() for _ in range(2)]

        def e2e_step(i):
            b = i & 1
            copy_in.wait_event(ev_done[b])
            with torch.cuda.stream(copy_in):
                for d, h in zip(dev_in[b], host_in):
                    d.copy_(h, non_blocking=True)
            ev_in[b].record(copy_in)
            stream.wait_event(ev_in[b])
            stream.wait_event(ev_out[b])
            self.step(ins=dev_in[b], outs=outs_dev[b], stream=stream)
            ev_done[b].record(stream)
            copy_out.wait_event(ev_done[b])
            with torch.cuda.stream(copy_out):
                outs_host[b].copy_(outs_dev[b], non_blocking=True)
            ev_out[b].record(copy_out)

        e2e_step(0)
        e2e_step(1)
        torch.cuda.synchronize()
        barrier()
        f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        f0.record(stream)
        copy_in.wait_stream(stream)
        for i in range(steps):
            e2e_step(i)
        stream.wait_event(ev_out[0])
        stream.wait_event(ev_out[1])
        f1.record(stream)
        torch.cuda.synchronize()
        barrier()
        self.outs_last = outs_dev[(steps - 1) & 1]
        return (max_over_ranks(f0.elapsed_time(f1)),
                sum(t.numel() * t.element_size() for t in host_in),
                outs_host[0].numel() * outs_host[0].element_size())

    def release(self) -> None:
        self.graph = None
        self.caches = []
        self.outs = self.outs_last = None
        torch.cuda.synchronize()
        torch.cuda.empty_cache()


def attn_oracle_check(run: AttnRun, outs) -> dict:
    """Layer 0's output of the last end-to-end pass against the oracle's step on
    the same inputs (every sequence and head)."""
    import oracle
    dec = lambda t: oracle.decode_bf16(wl.bf16_bits(t))  # noqa: E731
    h = run.host
    args = (dec(h["q"]), dec(h["k_new"]), dec(h["v_new"]), dec(h["k_cache"]), dec(h["v_cache"]),
            run.pos_host.numpy(), run.w.theta)
    t0 = time.perf_counter()
    ref, _, _ = oracle.token_attention(*args)
    dt = time.perf_counter() - t0
    run.cpu_baseline = {
        "value": round(attn_bytes(run.w) / dt / 1e9, 4), "unit": "GB/s", "cores": blas_threads(),
        "host_cores": host_cores(), "kind": "oracle",
        "sample": f"this check: layer 0's whole step through the fp64 oracle, {dt:.2f} s"}
    got = outs[0].cpu().double().numpy()
    norm = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
    elem = float(np.max(np.abs(got - ref)) / np.max(np.abs(ref)))
    return {"layer": 0, "normwise": float(f"{norm:.3e}"), "per_element": float(f"{elem:.3e}"),
            "within_bar": bool(norm <= 1e-4 and elem <= 1e-3), "bar": "normwise 1e-4, per element 1e-3"}


def measure_attn_workload(fm, w: wl.AttnWorkload, dev, args, barrier, max_over_ranks, rank: int,
                          world: int) -> dict:
    """A `workloads` entry for the token-phase attention step: timed for at
    least --min-seconds, one fmlp_attn_decode per layer back to back in a CUDA
    graph (one kernel per layer), with its roofline, end-to-end pass, oracle
    check and clocks."""
    run = AttnRun(fm, w, dev, seed0=1000 * rank)
    run.capture(args.warmup, use_graph=not args.no_graph)
    est = run.step_estimate_ms()
    steps = max(args.steps, int(np.ceil(args.min_seconds * 1e3 / max(est, 1e-3))))
    ms, launches, clocks = run.timed(steps, barrier, max_over_ranks)
    ms_step = ms / steps
    e2e_steps = max(2, min(4000, int(np.ceil(0.5e3 / max(est, 1e-3)))))
    e2e_ms, h2d, d2h = run.e2e(e2e_steps, barrier, max_over_ranks)
    bytes_step = run.L * attn_bytes(w)
    (peak, src), _ = peaks_of(sustained=True)
    gbs = job_gbs(bytes_step, steps, world, ms)
    kms = ms_step / run.L
    achieved = attn_bytes(w) / (kms / 1e3) / 1e9
    entry = {
        "config": {"B": w.B, "H": w.H, "H_kv": w.H_kv, "D": w.D, "n_ctx": w.n_ctx, "n_max": w.n_max,
                   "rope_theta": w.theta, "layers": run.L,
                   "kv_cache_per_gpu_GB": round(2 * w.B * w.H_kv * w.n_max * w.D * 2 * run.L / 1e9, 3)},
        "value": round(gbs, 2), "unit": "GB/s", "hbm_frac": round(gbs / world / peak, 4),
        "tokens_per_s_per_layer": round(w.B * run.L * steps * world / (ms / 1e3), 1),
        "ms_per_layer": round(kms, 5), "steps": steps, "timed_ms": round(ms, 2),
        "roofline": {"bound": "hbm", "kernel": "attn_decode", "achieved": round(achieved, 2),
                     "peak": peak, "peak_source": src, "unit": "GB/s",
                     "frac": round(achieved / peak, 4),
                     "traffic": recorded_traffic("attn_decode", w.name),
                     "algorithmic_per_launch": attn_bytes(w), "avg_launch_ms": round(kms, 5),
                     "launch_timing": "timed region / launches (one kernel per layer, back to back "
                                      "in a CUDA graph)"},
        "e2e": {"value": round(job_gbs(bytes_step, e2e_steps, world, e2e_ms), 2), "unit": "GB/s",
                "steps": e2e_steps, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "gpu_launches": launches, "cuda_graph": run.graph is not None,
        "device_status": fm.fmlp_status_string(fm.fmlp_device_status(run.ws)),
        "clocks": clocks,
    }
    if rank == 0 and not args.no_oracle_check:
        entry["check_vs_oracle"] = attn_oracle_check(run, run.outs_last)
        entry["cpu_baseline"] = run.cpu_baseline
    run.release()
    return entry


def run_ours(args) -> None:
    rank, world, local = dist_env()
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    dev = torch.device("cuda", torch.cuda.current_device())
    import token_phase_swiglu_b200 as fm

    def barrier():
        if world > 1:
            import torch.distributed as dist
            dist.barrier()

    def max_over_ranks(v: float) -> float:
        return reduce_max(v, dev)

    w = wl.WORKLOADS[args.workload]
    run = WorkloadRun(fm, w, dev, seed0=1000 * rank, layers=args.layers)
    M, d, I, L = run.M, run.d, run.I, run.L
    run.capture(args.warmup, use_graph=not args.no_graph)

    # the headline: exactly K timed steps
    elapsed_ms, launches, clocks = run.timed(args.steps, barrier, max_over_ranks)
    fm_status = fm.fmlp_device_status(run.ws)
    bytes_step = L * algorithmic_bytes(M, d, I)
    gbs = job_gbs(bytes_step, args.steps, world, elapsed_ms)
    ms_step = elapsed_ms / args.steps
    tok_per_s_layer = M * L * args.steps * world / (elapsed_ms / 1e3)

    iso = run.isolated_calls(max(1, min(args.steps, 50)), max_over_ranks)
    e2e_steps = max(2, min(args.steps, 200))
    e2e_ms, h2d, d2h = run.e2e(e2e_steps, barrier, max_over_ranks)
    e2e_gbs = job_gbs(bytes_step, e2e_steps, world, e2e_ms)
    roof = roofline_entry(run, ms_step, iso["fmlp_gate_up_swiglu_ms"])
    (peak, _), _ = peaks_of()

    cpu, check = None, None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, desc, _ = oracle_sample(w, args.cpu_seconds, seed=run.seed0)
        cpu = {"value": round(v, 4), "unit": "GB/s", "cores": blas_threads(),
               "host_cores": host_cores(), "kind": "oracle", "sample": desc}
    if rank == 0 and not args.no_oracle_check:
        check = oracle_check(run, run.outs_last)
    graph_used = run.graph is not None
    run.release()
    del run

    # every other workload (and the headline's own, timed for a second), one
    # entry each
    subs = {}
    names = [] if args.workloads == "none" else (
        list(wl.WORKLOADS) + [n + "_q8" for n in Q8_WORKLOADS] + ATTN_BENCH
        if args.workloads == "all" else args.workloads.split(","))
    for name in names:
        if name in wl.ATTN_WORKLOADS:
            subs[name] = measure_attn_workload(fm, wl.ATTN_WORKLOADS[name], dev, args, barrier,
                                               max_over_ranks, rank, world)
            continue
        quant = name.endswith("_q8")
        subs[name] = measure_sub_workload(fm, wl.WORKLOADS[name[:-3] if quant else name], dev,
                                          args, barrier, max_over_ranks, rank, world, quant=quant)

    if rank == 0:
        gu_ms, dn_ms = iso["fmlp_gate_up_swiglu_ms"], iso["fmlp_down_proj_ms"]
        line = {
            "metric": METRIC, "value": round(gbs, 2), "unit": "GB/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": config_of(w, args),
            "hbm_frac": round(gbs / world / peak, 4),
            "tokens_per_s_per_layer": round(tok_per_s_layer, 1),
            "roofline": roof,
            "tflops": round(6 * M * d * I * L * args.steps * world / (elapsed_ms / 1e3) / 1e12, 2),
            "isolated_calls": {
                "note": "each call bracketed by its own events (no overlap with its neighbours)",
                "fmlp_forward_ms": round(iso["fmlp_forward_ms"], 5),
                "fmlp_gate_up_swiglu_ms": round(gu_ms, 5),
                "fmlp_gate_up_swiglu_GBps": round(gateup_bytes(M, d, I) / (gu_ms / 1e3) / 1e9, 2),
                "fmlp_down_proj_ms": round(dn_ms, 5),
                "fmlp_down_proj_GBps": round((2 * d * I + 2 * M * I + 4 * M * d) /
                                             (dn_ms / 1e3) / 1e9, 2)},
            "cpu_baseline": cpu,
            "check_vs_oracle": check,
            "e2e": {"value": round(e2e_gbs, 2), "unit": "GB/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "copies": "pinned host buffers, copy streams, double-buffered across steps"},
            "gpu_launches": launches,
            "cuda_graph": graph_used,
            "device_status": fm.fmlp_status_string(fm_status),
            "clocks": clocks,
            "workloads": subs,
        }
        print(json.dumps(line), flush=True)

    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def main() -> None:
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="phi3_decode", choices=sorted(wl.WORKLOADS))
    ap.add_argument("--no-graph", action="store_true", help="launch each step from the host")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--layers", type=int, default=0,
                    help="override the workload's layer count (small profiling captures only)")
    ap.add_argument("--workloads", default="all",
                    help="comma list of workloads measured as entries of the line's `workloads` "
                         "object, 'all' (default) or 'none'")
    ap.add_argument("--min-seconds", type=float, default=1.0,
                    help="device time each `workloads` entry is timed for, at least")
    ap.add_argument("--no-oracle-check", action="store_true")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
