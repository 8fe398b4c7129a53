#!/usr/bin/env python
"""Throughput of the quantized W8A8 linear layer on B200.

Default workload (the headline): the LLM.int8 DiT MLP at 1024^2 -- the
up-projection X[4352,3072] W[12288,3072]^T and the down-projection
X'[4352,12288] W'[3072,12288]^T, bf16 activations, threshold 6.0, seeded
synthetic inputs (N(0,1) activations with outlier channels and massive text
tokens, N(0,0.02) weights). One step = one pass of the whole hot path over
both linears: outlier detection, activation quantisation, outlier gathers,
and the tcgen05 int8 GEMM with its fused epilogue.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl qlin|reference]

Prints one JSON line (rank 0). `value` is whole-job TOPS (2*M*N*K per
linear; the outlier sub-GEMM is not counted) over the device time of the K
timed steps, max over ranks. L2 is flushed (a 256 MiB write) before every
timed step, outside the timed events. Multi-GPU runs are independent
replicas (the layer has no data-parallel exchange): weak scaling.

`--impl reference` times the CPU oracle (plain C, fp64) on a bounded sample
of rows of the same workload, on the host cores, rank 0 only.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "quantized-linear TOPS at DiT 1024² shapes; % of B200 int8/fp8 tensor peak"
WORKLOAD = "dit1024_int8_mlp"
L2_FLUSH_BYTES = 256 << 20
# nominal dense int8 (and fp8) : bf16 tensor-core ratio of B200 (4.5 : 2.25 POPS)
INT8_PER_BF16 = 2.0
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def parse_args():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=["qlin", "reference"], default="qlin")
    ap.add_argument("--e2e-steps", type=int, default=10)
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="CPU-baseline sample budget")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-secondary", action="store_true", help="skip the secondary workloads")
    ap.add_argument("--workload", default=WORKLOAD,
                    help="workload timed as the main line (default: the 1024^2 LLM.int8 DiT MLP)")
    return ap.parse_args()


# ---------------------------------------------------------------------------
# environment
# ---------------------------------------------------------------------------

def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def source_sha(files):
    h = hashlib.sha256()
    for f in files:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


GEMM_SOURCES = ["quantized_w8a8_linear_b200/csrc/gemm.cuh", "quantized_w8a8_linear_b200/csrc/common.cuh"]


def profiled_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if the kernel's
    source is unchanged since the counters were taken; else None."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None, None
    with open(p) as f:
        d = json.load(f)
    e = d.get(kernel)
    if not e or e.get("source_sha") != source_sha(GEMM_SOURCES):
        return None, None
    return e.get("dram_bytes_per_launch"), e.get("note")


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""
    FIELDS = ["clocks.sm", "clocks.max.sm", "power.draw", "clocks_event_reasons.hw_slowdown",
              "clocks_event_reasons.hw_thermal_slowdown", "clocks_event_reasons.sw_thermal_slowdown",
              "clocks_event_reasons.sw_power_cap"]

    def __init__(self, device_index: int):
        self.proc = None
        self.dev = device_index

    def _gpu_id(self):
        import torch
        try:
            return "GPU-" + str(torch.cuda.get_device_properties(self.dev).uuid)
        except Exception:
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            return vis.split(",")[self.dev] if vis else str(self.dev)

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", self._gpu_id(), "--query-gpu=" + ",".join(self.FIELDS),
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        time.sleep(0.06)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, reasons, power = [], [], set(), []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != len(self.FIELDS):
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
                power.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": sorted(reasons), "samples": len(sm),
                "power_w_max": max(power) if power else None}


# ---------------------------------------------------------------------------
# workloads on the GPU
# ---------------------------------------------------------------------------

class LinearRun:
    """One quantized linear, resident on the device, split into its two stages."""

    def __init__(self, q, wl, lin, index, device):
        import torch
        import workloads
        self.q, self.lin, self.mode = q, lin, wl.mode
        X, W, bias = workloads.make_linear(wl, lin, index=index)
        self.X_cpu, self.W_cpu = X, W
        self.X = X.to(device)
        Wd = W.to(device)
        M, K, N = lin.M, lin.K, lin.N
        self.M, self.K, self.N = M, K, N
        self.dtype = X.dtype
        self.Y = torch.empty((M, N), dtype=X.dtype, device=device)
        self.ops = 2.0 * M * N * K
        if self.mode == "int8_outlier":
            self.Wq, self.s_w = q.qlin_quantize_weight(Wd, q.QLIN_W_INT8_ROW)
            n = q.qlin_workspace_bytes(q.QLIN_OP_INT8_OUTLIER, M, N, K)
            self.ws = torch.empty(n, dtype=torch.uint8, device=device)
            # algorithmic prep bytes: X read (2 B) + Xq write (1 B) per element
            self.prep_bytes = 3.0 * M * K
        elif self.mode == "w4a8":
            self.Wq, self.s_w = q.qlin_quantize_weight(Wd, q.QLIN_W_INT4_G128)
            self.Xq = torch.empty((M, K), dtype=torch.int8, device=device)
            self.s_x = torch.empty((M,), dtype=torch.float32, device=device)
            self.prep_bytes = 3.0 * M * K
        elif self.mode == "fp8_weight_only":
            self.Wq, self.s_w = q.qlin_quantize_weight(Wd, q.QLIN_W_FP8_CHANNEL)
            self.prep_bytes = 0.0
        elif self.mode == "nvfp4_weight_only":
            self.Wq, self.s_w = q.qlin_quantize_weight(Wd, q.QLIN_W_NVFP4)
            self.prep_bytes = 0.0
        elif self.mode == "fp_linear":
            self.Wq, self.s_w = Wd.clone(), None
            self.prep_bytes = 0.0
        else:
            wmode = q.QLIN_W_FP8_TENSOR if self.mode == "fp8_static" else q.QLIN_W_FP8_CHANNEL
            self.wmode = wmode
            self.Wq, self.s_w = q.qlin_quantize_weight(Wd, wmode)
            self.x_scale = None
            if self.mode == "fp8_static":
                self.x_scale = q.qlin_calibrate_input_scale(workloads.make_calibration(wl, lin, index=index).to(device))
            self.Xq = torch.empty((M, K), dtype=torch.uint8, device=device)
            self.s_x = torch.empty((M,), dtype=torch.float32, device=device)
            self.gws = torch.empty(max(256, q.qlin_workspace_bytes(q.QLIN_OP_FP8_GEMM, M, N, K)), dtype=torch.uint8,
                                   device=device)
            self.prep_bytes = 3.0 * M * K
        del Wd

    def prepare(self):
        q = self.q
        if self.mode in ("fp8_weight_only", "fp_linear", "nvfp4_weight_only"):
            return   # one kernel: the activations are not quantised
        if self.mode == "int8_outlier":
            q.qlin_int8_outlier_prepare(self.X, self.Wq, self.s_w, 6.0, self.ws)
        elif self.mode == "w4a8":
            q.qlin_w4a8_prep(self.X, self.Xq, self.s_x)
        else:
            q._check(q.lib.qlin_fp8_prep(q._ptr(self.X), q._dt(self.X), self.M, self.K, q._ptr(self.x_scale),
                                         q._ptr(self.Xq), q._ptr(self.s_x), q._stream(self.X.device)))

    def gemm(self):
        q = self.q
        if self.mode == "fp8_weight_only":
            q.qlin_fp8_weight_only_forward(self.X, self.Wq, self.s_w, Y=self.Y)
            return
        if self.mode == "nvfp4_weight_only":
            q.qlin_nvfp4_weight_only_forward(self.X, self.Wq, self.s_w, Y=self.Y)
            return
        if self.mode == "fp_linear":
            q.qlin_fp_linear_forward(self.X, self.Wq, Y=self.Y)
            return
        if self.mode == "int8_outlier":
            q.qlin_int8_outlier_gemm(self.dtype, self.M, self.K, self.Wq, self.s_w, self.Y, self.ws)
        elif self.mode == "w4a8":
            q.qlin_w4a8_gemm(self.Xq, self.s_x, self.Wq, self.s_w, self.dtype, Y=self.Y)
        else:
            q.qlin_fp8_gemm(self.Xq, self.s_x, self.Wq, self.s_w, self.wmode, self.dtype, x_scale=self.x_scale,
                            Y=self.Y, ws=self.gws)

    def forward(self):
        self.prepare()
        self.gemm()

    def forward_one_call(self):
        """The public one-call forward of this linear's format (the C ABI's
        qlin_int8_outlier_forward, qlin_w4a8_forward or qlin_fp8_forward)."""
        q = self.q
        if self.mode == "int8_outlier":
            q.qlin_int8_outlier_forward(self.X, self.Wq, self.s_w, 6.0, Y=self.Y, ws=self.ws)
        elif self.mode == "w4a8":
            q.qlin_w4a8_forward(self.X, self.Wq, self.s_w, Y=self.Y)
        elif self.mode in ("fp8_weight_only", "fp_linear", "nvfp4_weight_only"):
            self.gemm()
        else:
            q.qlin_fp8_forward(self.X, self.Wq, self.s_w, self.wmode, x_scale=self.x_scale, Y=self.Y)

    # kernels of ours launched per forward: LLM.int8 reset, streaming pass,
    # finishing kernel and GEMM; the FP8 and W4A8 forwards a prep kernel and
    # the GEMM; the weight-only FP8 and 16-bit linears one GEMM
    def launches(self):
        if self.mode == "int8_outlier":
            return 4
        if self.mode in ("fp8_weight_only", "fp_linear", "nvfp4_weight_only"):
            return 1
        return 2


def max_over_ranks(value, device, world):
    """The largest of the ranks' values (all_reduce MAX over the default
    process group); the local value when there is one rank."""
    if world <= 1:
        return float(value)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(value)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_tops(world, steps, ops_step, total_ms_max):
    """Throughput of all ranks together: each rank ran `steps` steps of
    `ops_step` ops; the job took the slowest rank's time."""
    return world * steps * ops_step / (total_ms_max * 1e-3) / 1e12


def time_steps(runs, steps, warmup, flush):
    """Device time of `steps` steps (each: every linear's prepare + gemm), L2
    flushed before each step outside the events. Returns per-part sums (ms)."""
    import torch
    st = torch.cuda.current_stream()
    for _ in range(warmup):
        flush.zero_()
        for r in runs:
            r.forward()
    torch.cuda.synchronize()
    evs = []
    for _ in range(steps):
        flush.zero_()
        step = []
        for r in runs:
            e0, e1, e2 = (torch.cuda.Event(enable_timing=True) for _ in range(3))
            e0.record(st)
            r.prepare()
            e1.record(st)
            r.gemm()
            e2.record(st)
            step.append((e0, e1, e2))
        evs.append(step)
    torch.cuda.synchronize()
    prep = [0.0] * len(runs)
    gemm = [0.0] * len(runs)
    for step in evs:
        for i, (e0, e1, e2) in enumerate(step):
            prep[i] += e0.elapsed_time(e1)
            gemm[i] += e1.elapsed_time(e2)
    return prep, gemm


def time_whole(runs, steps, warmup, flush):
    """Device time of `steps` whole steps (every linear's prepare + gemm, no
    events in between), replayed from one CUDA graph when the launches can be
    captured. L2 flushed before each step outside the events. Returns
    (total ms, "graph" | "stream")."""
    import torch
    st = torch.cuda.current_stream()
    replay = None
    mode = "stream"
    try:
        g = torch.cuda.CUDAGraph()
        side = torch.cuda.Stream()
        side.wait_stream(st)
        with torch.cuda.stream(side):
            with torch.cuda.graph(g, stream=side):
                for r in runs:
                    r.forward()
        st.wait_stream(side)
        torch.cuda.synchronize()
        replay = g.replay
        mode = "graph"
    except Exception:
        torch.cuda.synchronize()

    def one():
        if replay is not None:
            replay()
        else:
            for r in runs:
                r.forward()
    for _ in range(warmup):
        flush.zero_()
        one()
    torch.cuda.synchronize()
    evs = []
    for _ in range(steps):
        flush.zero_()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(st)
        one()
        e1.record(st)
        evs.append((e0, e1))
    torch.cuda.synchronize()
    return sum(a.elapsed_time(b) for a, b in evs), mode


def time_e2e(runs, steps):
    """Same work through the public one-call forward of the C ABI
    (qlin_int8_outlier_forward for the headline) with host buffers: per step
    and linear, the pinned H2D copy of X, the one-call forward, and the D2H
    copy of Y, all inside the timed events."""
    import torch
    st = torch.cuda.current_stream()
    h_in = [r.X_cpu.pin_memory() for r in runs]
    h_out = [torch.empty(r.Y.shape, dtype=r.Y.dtype).pin_memory() for r in runs]
    for _ in range(2):
        for r, hi, ho in zip(runs, h_in, h_out):
            r.X.copy_(hi, non_blocking=True)
            r.forward_one_call()
            ho.copy_(r.Y, non_blocking=True)
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(st)
    for _ in range(steps):
        for r, hi, ho in zip(runs, h_in, h_out):
            r.X.copy_(hi, non_blocking=True)
            r.forward_one_call()
            ho.copy_(r.Y, non_blocking=True)
    e1.record(st)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    h2d = sum(h.numel() * h.element_size() for h in h_in)
    d2h = sum(h.numel() * h.element_size() for h in h_out)
    return ms, h2d, d2h


# ---------------------------------------------------------------------------
# CPU oracle (baseline leg / reference arm)
# ---------------------------------------------------------------------------

class OracleSample:
    """The CPU oracle on a bounded sample of rows of the headline workload.
    Outlier detection and row scales still run over every token; the
    contraction runs for `rows` rows of each linear."""

    def __init__(self, lin_data):
        import oracle
        self.oracle = oracle
        self.items = []
        for X, W, lin in lin_data:
            Wq, s_w = oracle.quantize_weight(W, "int8_row")     # offline, not timed
            self.items.append((X, Wq, s_w, lin))

    def run(self, rows: int) -> float:
        t0 = time.perf_counter()
        for X, Wq, s_w, lin in self.items:
            self.oracle.int8_outlier_forward(X, Wq, s_w, 6.0, rows=list(range(rows)), want_c=False)
        return time.perf_counter() - t0

    def ops(self, rows: int) -> float:
        return sum(2.0 * rows * lin.N * lin.K for _, _, _, lin in self.items)

    def calibrate(self, budget_s: float, max_rows: int) -> int:
        """Rows whose run takes about budget_s: double until a run takes a
        quarter of the budget, then scale linearly (first call warms up)."""
        self.run(1)
        rows = 8
        while True:
            t = self.run(rows)
            if t >= budget_s / 4 or rows >= max_rows:
                break
            rows *= 2
        return int(max(1, min(max_rows, rows * budget_s / max(t, 1e-6))))


def cpu_sample_inputs():
    import workloads
    wl = workloads.get_workload(WORKLOAD)
    out = []
    for i, lin in enumerate(wl.linears):
        X, W, _ = workloads.make_linear(wl, lin, index=i)
        out.append((X, W, lin))
    return out


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    oracle.build()
    data = cpu_sample_inputs()
    sample = OracleSample(data)
    budget = max(0.05, min(10.0, 150.0 / max(1, args.steps + args.warmup)))
    rows = sample.calibrate(budget, data[0][2].M)
    for _ in range(args.warmup):
        sample.run(rows)
    t = 0.0
    for _ in range(args.steps):
        t += sample.run(rows)
    ops = sample.ops(rows) * args.steps
    value = ops / t / 1e12
    cores = oracle.num_threads()
    desc = (f"{rows} token rows of each linear per step (outlier detection and row scales over all "
            f"{data[0][2].M} tokens), {args.steps} steps")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * t / args.steps,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "int64+f64",
        "data": "synthetic", "config": workload_config(),
        "cpu_baseline": {"value": value, "unit": "TOPS", "cores": cores, "kind": "oracle", "sample": desc},
        "e2e": {"value": value, "unit": "TOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def workload_config(name=WORKLOAD, wl=None):
    l2 = "flushed before every timed step (256 MiB write, outside the timed events)"
    if name == WORKLOAD:
        return {"workload": "LLM.int8 DiT MLP at 1024^2: up [4352x3072]x[12288x3072]^T + down "
                            "[4352x12288]x[3072x12288]^T, bf16, threshold 6.0",
                "name": WORKLOAD, "tokens": 4352, "hidden": 3072, "mlp": 12288, "threshold": 6.0,
                "l2": l2, "parallelism": "replicas"}
    shapes = " + ".join(f"{l.name} [{l.M}x{l.K}]x[{l.N}x{l.K}]^T" for l in wl.linears)
    return {"workload": f"{wl.mode}: {shapes}", "name": name, "l2": l2, "parallelism": "replicas"}


# ---------------------------------------------------------------------------
# main (qlin arm)
# ---------------------------------------------------------------------------

def main():
    args = parse_args()
    if args.impl == "reference":
        return run_reference(args)

    import torch
    import torch.distributed as dist

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)

    import quantized_w8a8_linear_b200 as q
    import workloads

    wl = workloads.get_workload(args.workload)
    runs = [LinearRun(q, wl, lin, i, device) for i, lin in enumerate(wl.linears)]
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    torch.cuda.synchronize()

    # -------- timed region --------
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    t_wall0 = time.perf_counter()
    # whole steps (the headline), then the same steps with an event between
    # every stage (the per-kernel split and the roofline)
    whole_ms, step_mode = time_whole(runs, args.steps, max(3, args.warmup), flush)
    prep_ms, gemm_ms = time_steps(runs, args.steps, max(3, args.warmup), flush)
    t_wall = time.perf_counter() - t_wall0
    clk = clocks.stop()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    total_ms_max = max_over_ranks(whole_ms, device, world)
    ops_step = sum(r.ops for r in runs)
    value = whole_job_tops(world, args.steps, ops_step, total_ms_max)
    ms_per_step = total_ms_max / args.steps

    # -------- roofline of the dominant kernel (the tcgen05 GEMM) --------
    peaks, peak_src = load_peaks()
    peak_tops = INT8_PER_BF16 * float(peaks["bf16_tflops"])
    gemm_launches = len(runs) * args.steps
    gemm_avg_ms = sum(gemm_ms) / gemm_launches
    gemm_ops_avg = ops_step / len(runs)
    achieved = gemm_ops_avg / (gemm_avg_ms * 1e-3) / 1e12
    # the ncu DRAM counters exist for the headline workload's GEMM only
    traffic = None
    if wl.name == "dit1024_int8_mlp":
        traffic, _ = profiled_traffic("k_gemm_int8_outlier_dit1024")
    kernel_name = {"int8_outlier": "k_gemm<kind::i8, LLM.int8 epilogue>",
                   "w4a8": "k_gemm_w4a8<kind::i8, per-group promotion>",
                   "fp8_static": "k_gemm<kind::f8f6f4, per-tensor epilogue>",
                   "fp8_dynamic": "k_gemm<kind::f8f6f4, per-token x per-channel epilogue>"}.get(wl.mode, wl.mode)
    unit_kind = "fp8 TFLOPS" if wl.mode.startswith("fp8") else "int8 TOPS"
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak_tops, "unit": "TFLOP/s",
                "frac": achieved / peak_tops, "traffic": traffic, "kernel": kernel_name,
                "peak_source": f"{peak_src} bf16 burst {peaks['bf16_tflops']} TFLOP/s x {INT8_PER_BF16} "
                               f"(nominal int8|fp8:bf16 dense ratio); unit is {unit_kind}"}
    hbm = float(peaks["hbm_gbs"])
    prep_bytes = sum(r.prep_bytes for r in runs)
    prep_gbs = prep_bytes * args.steps / (sum(prep_ms) * 1e-3) / 1e9
    kernels = {
        "gemm": {"avg_us_per_launch": 1e3 * gemm_avg_ms, "TOPS": achieved,
                 "per_linear_us": [1e3 * g / args.steps for g in gemm_ms]},
        "prepare": {"avg_us_per_linear": 1e3 * sum(prep_ms) / gemm_launches, "GBps_algorithmic": prep_gbs,
                    "hbm_peak_GBps": hbm, "frac": prep_gbs / hbm,
                    "per_linear_us": [1e3 * p / args.steps for p in prep_ms]},
    }

    # -------- end to end through the one-call forward with host buffers --------
    e2e_ms, h2d, d2h = time_e2e(runs, args.e2e_steps)
    e2e = {"value": ops_step / (e2e_ms * 1e-3) / 1e12 * world, "unit": "TOPS", "h2d_bytes_per_step": h2d,
           "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms}

    # -------- secondary workloads (FP8, 2048^2 DiT block), rank-local, reported beside --------
    secondary = {}
    if not args.no_secondary:
        for name in ("dit1024_fp8_static_qkv", "te_fp8_dynamic_mlp", "dit2048_block_int8", "dit2048_block_w4a8",
                     "te_fp8_weight_only_mlp", "te_nvfp4_weight_only_mlp", "dit1024_bf16_mlp"):
            w2 = workloads.get_workload(name)
            r2 = [LinearRun(q, w2, lin, i, device) for i, lin in enumerate(w2.linears)]
            steps2 = max(20, args.steps // 5)
            p2, g2 = time_steps(r2, steps2, 3, flush)
            ops2 = sum(r.ops for r in r2)
            tot2 = sum(p2) + sum(g2)
            # the 16-bit contractions (kind::f16) against the bf16 peak, the rest against int8/fp8
            pk = (float(peaks["bf16_tflops"]) if w2.mode in ("fp8_weight_only", "fp_linear", "nvfp4_weight_only")
                  else peak_tops)
            secondary[name] = {"TOPS": steps2 * ops2 / (tot2 * 1e-3) / 1e12,
                               "gemm_TOPS": steps2 * ops2 / (sum(g2) * 1e-3) / 1e12,
                               "gemm_frac_of_peak": steps2 * ops2 / (sum(g2) * 1e-3) / 1e12 / pk,
                               "peak_TOPS": pk,
                               "ms_per_step": tot2 / steps2,
                               "prep_GBps": (steps2 * sum(r.prep_bytes for r in r2) / (sum(p2) * 1e-3) / 1e9
                                             if sum(p2) > 0 else None),
                               "gemm_TOPS_per_linear": {r.lin.name: steps2 * r.ops / (g * 1e-3) / 1e12
                                                        for r, g in zip(r2, g2)}}
            blocks = w2.extra.get("blocks") if w2.extra else None
            if blocks:
                secondary[name]["ms_per_sweep_of_%d_blocks" % blocks] = blocks * tot2 / steps2
            del r2
            torch.cuda.empty_cache()

    # -------- CPU baseline (rank 0, N = 1) --------
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline and args.workload == WORKLOAD:
        import oracle
        data = [(r.X_cpu, r.W_cpu, r.lin) for r in runs]
        sample = OracleSample(data)
        rows = sample.calibrate(args.cpu_seconds, runs[0].M)
        t = sample.run(rows)
        cpu = {"value": sample.ops(rows) / t / 1e12, "unit": "TOPS", "cores": oracle.num_threads(),
               "kind": "oracle", "seconds": t,
               "sample": f"{rows} token rows of each linear (outlier detection and row scales over all "
                         f"{runs[0].M} tokens)"}

    assert q.qlin_get_device_status() == 0, "a device-side wait timed out"
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TOPS", "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": ms_per_step, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "int8", "data": "synthetic",
            "config": workload_config(args.workload, wl), "impl": "qlin",
            "pct_of_int8_peak": 100.0 * value / world / peak_tops,
            "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e,
            "gpu_launches": sum(r.launches() for r in runs) * args.steps,
            "clocks": clk, "kernels": kernels, "secondary": secondary, "wall_s_timed_region": t_wall,
            "timing": {"value": f"whole steps with no event between stages ({step_mode} replay)",
                       "kernels": "a second pass of the same steps with an event between every stage"},
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
