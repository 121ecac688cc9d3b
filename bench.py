#!/usr/bin/env python
"""Throughput of the EQ-Linear forward on B200, one JSON line on rank 0.

Default workload: the p4 (T=4) FP16 ViT-B MLP pair, N = 12608 rows (64 images x
197 tokens), layer 1 C=192 -> D=768 (768 -> 3072 features), layer 2 C=768 ->
D=192 (3072 -> 768) applied to layer 1's output.  One step = both forward
launches.  `value` = rows (tokens) per second over the whole job, inputs
resident in HBM; `e2e` = the same through the C ABI with the step's input copied
from pinned host memory and the result read back, inside the timed region.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
       [--workload p4_vitb_mlp_f16|p4_vitb_proj_f32|p4_vith_fc1_f16|c8_1024_f16]
Under torchrun (N > 1) every rank runs its own copy of the workload (weak
scaling; rows are independent, so no collective is on the data path).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from group_circulant_gemm_b200.synth import WORKLOADS, make_inputs  # noqa: E402

METRIC = "EQ-Linear fwd tokens/s + TFLOP/s (T=4, fp16/fp32) and % of tensor roofline"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# workload name -> list of layer workloads applied in sequence (output feeds the next)
PIPELINES = {
    "p4_vitb_mlp_f16": ["p4_vitb_fc1_f16", "p4_vitb_fc2_f16"],
    "p4_vitb_proj_f32": ["p4_vitb_proj_f32"],
    "p4_vith_fc1_f16": ["p4_vith_fc1_f16"],
    "c8_1024_f16": ["c8_1024_f16"],
}
DESCR = {
    "p4_vitb_mlp_f16": "p4 EQ-Linear fp16 ViT-B MLP pair: N=12608, C=192->D=768 then "
                       "C=768->D=192, T=4",
    "p4_vitb_proj_f32": "p4 EQ-Linear fp32 ViT-B projection: N=12608, C=D=192, T=4",
    "p4_vith_fc1_f16": "p4 EQ-Linear fp16 ViT-H fc1: N=8224, C=320->D=1280, T=4",
    "c8_1024_f16": "cyclic T=8 EQ-Linear fp16: N=16384, C=D=128",
}


def layer_flops(w) -> float:
    """Algorithmic FLOPs of one forward: 2 * (real GEMMs per frequency plan) * N*C*D."""
    nr = 2 if w.T % 2 == 0 else 1
    nc = (w.T - nr) // 2
    return 2.0 * (nr + 4 * nc) * w.N * w.C * w.D


def layer_bytes(w) -> float:
    """Algorithmic HBM bytes of one forward: read X, prepared weights, bias; write Y."""
    es = 2 if w.dtype == "f16" else 4
    nr = 2 if w.T % 2 == 0 else 1
    planes = w.T + (w.T - nr) // 2
    return es * (w.N * w.C * w.T + w.N * w.D * w.T + planes * w.C * w.D + w.D)


# DRAM traffic per forward launch (dram__bytes_read.sum + dram__bytes_write.sum),
# from the ncu captures summarised in profiles/, valid only for the kernel source
# they were taken on (SHA-256 prefix of csrc/eql_tc_fwd.cu); any other source
# reports null.
NCU_TRAFFIC = {
    "86ba56eb36e4696e": {"p4_vitb_mlp_f16": 64.73e6, "c8_1024_f16": 34.20e6},
}


def kernel_traffic(workload: str):
    import hashlib
    path = os.path.join(ROOT, "group_circulant_gemm_b200", "csrc", "eql_tc_fwd.cu")
    try:
        with open(path, "rb") as f:
            h = hashlib.sha256(f.read()).hexdigest()[:16]
    except OSError:
        return None
    return NCU_TRAFFIC.get(h, {}).get(workload)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled during the timed region."""

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None

    def stop(self):
        out = {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        if self.proc is None:
            return out
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [x.strip() for x in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    sm.append(float(parts[1]))
                    mx.append(float(parts[2]))
                except ValueError:
                    continue
                for nm, v in zip(names, parts[5:9]):
                    if v.lower() == "active":
                        reasons.add(nm)
        os.unlink(self.path)
        if sm:
            out = {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                   "reasons": sorted(reasons), "samples": len(sm)}
        return out


def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def oracle_sample(pipeline, rows: int):
    """Time the float64 oracle on `rows` rows of the pipeline; returns (seconds, rows)."""
    import oracle
    oracle.build()
    layers = [(WORKLOADS[name], make_inputs(WORKLOADS[name], rows=rows)) for name in pipeline]
    x = layers[0][1]["X"].astype(np.float64)
    t0 = time.perf_counter()
    for w, inp in layers:
        x = oracle.forward(w.T, x, inp["W"], inp["bias"])
    return time.perf_counter() - t0, rows


def calibrated_oracle_rows(pipeline, target_s: float) -> int:
    t, r = oracle_sample(pipeline, 16)
    n_full = WORKLOADS[pipeline[0]].N
    return int(max(16, min(n_full, 16 * target_s / max(t, 1e-6))))


def run_reference(args, workload):
    """Reference arm: the float64 oracle on the host cores, bounded sample per step."""
    import oracle
    world, rank, _ = dist_init()
    if rank != 0:
        return 0
    pipeline = PIPELINES[workload]
    per_step_s = max(1.0, 120.0 / max(1, args.steps + args.warmup))
    rows = calibrated_oracle_rows(pipeline, min(per_step_s, 20.0))
    for _ in range(args.warmup):
        oracle_sample(pipeline, rows)
    times = [oracle_sample(pipeline, rows)[0] for _ in range(args.steps)]
    total = sum(times)
    value = rows * args.steps / total
    w0 = WORKLOADS[pipeline[0]]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": DESCR[workload], "rows_per_step": rows, "global_batch": w0.N,
                   "seq_len": None, "parallelism": "none (host oracle)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.threads_used(),
                         "kind": "oracle",
                         "sample": f"{rows} of {w0.N} rows per step through every layer"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_ours(args, workload):
    import torch
    import torch.distributed as dist

    world, rank, local = dist_init()
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    from group_circulant_gemm_b200 import EqLinearPlan

    pipeline = [WORKLOADS[n] for n in PIPELINES[workload]]
    dt = torch.float16 if pipeline[0].dtype == "f16" else torch.float32
    N = pipeline[0].N
    es = 2 if dt == torch.float16 else 4
    stream = torch.cuda.current_stream()

    # weights: prepared once, outside the timed region
    plans, whats, biases = [], [], []
    for w in pipeline:
        inp = make_inputs(w.with_(seed=w.seed + 1000 * rank), rows=1)
        p = EqLinearPlan(w.T, w.C, w.D, dt)
        W = torch.from_numpy(inp["W"]).cuda()
        plans.append(p)
        whats.append(p.prepare_weights(W))
        biases.append(torch.from_numpy(inp["bias"]).cuda() if w.bias else None)
    x_host = make_inputs(pipeline[0].with_(seed=pipeline[0].seed + 1000 * rank))["X"]

    # rotating input/output sets so the step's working set leaves L2 between steps
    per_set = sum(N * w.C * w.T * es + N * w.D * w.T * es for w in pipeline)
    nsets = max(2, int(np.ceil(2 * L2_BYTES / per_set)))
    xs = [torch.from_numpy(x_host).cuda() for _ in range(nsets)]
    outs = [[torch.empty((N, w.D * w.T), dtype=dt, device="cuda") for w in pipeline]
            for _ in range(nsets)]

    def step(i, events=None):
        x = xs[i % nsets]
        for li, (p, wh, b) in enumerate(zip(plans, whats, biases)):
            if events is not None:
                events.append(torch.cuda.Event(enable_timing=True))
                events[-1].record(stream)
            p.forward(x, wh, b, out=outs[i % nsets][li])
            if events is not None:
                events.append(torch.cuda.Event(enable_timing=True))
                events[-1].record(stream)
            x = outs[i % nsets][li]

    kernel_names = [p.forward_kernel_name(N) for p in plans]
    # the clock sampler runs from the start of warm-up to the end of the timed region
    clocks = ClockSampler(local)
    if rank == 0:
        clocks.start()
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    for p in plans:
        assert p.status() == 0

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    ev = []
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        step(args.warmup + i, ev)
    t1.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop() if rank == 0 else {}
    elapsed_ms = t0.elapsed_time(t1)
    launch_ms = [ev[2 * j].elapsed_time(ev[2 * j + 1]) for j in range(len(ev) // 2)]

    # end to end through the ABI: pinned host input -> device, both layers, result -> host
    x_pin = torch.from_numpy(x_host).pin_memory()
    y_pin = torch.empty((N, pipeline[-1].D * pipeline[-1].T), dtype=dt).pin_memory()
    for _ in range(2):
        xs[0].copy_(x_pin, non_blocking=True)
        step(0)
        y_pin.copy_(outs[0][-1], non_blocking=True)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for i in range(args.steps):
        xs[0].copy_(x_pin, non_blocking=True)
        step(0)
        y_pin.copy_(outs[0][-1], non_blocking=True)
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    for p in plans:
        assert p.status() == 0

    times = torch.tensor([elapsed_ms, e2e_ms], dtype=torch.float64, device="cuda")
    if world > 1:
        dist.all_reduce(times, op=dist.ReduceOp.MAX)
    elapsed_ms, e2e_ms = times.tolist()

    if rank == 0:
        peaks, peak_src = load_peaks()
        flops = sum(layer_flops(w) for w in pipeline)
        value = world * N * args.steps / (elapsed_ms / 1e3)
        e2e_value = world * N * args.steps / (e2e_ms / 1e3)
        # dominant kernel: the per-layer forward kernel (same kernel for every layer)
        per_layer = np.array(launch_ms).reshape(args.steps, len(pipeline))
        mean_launch_ms = float(per_layer.mean())
        flops_per_launch = flops / len(pipeline)
        bytes_per_launch = sum(layer_bytes(w) for w in pipeline) / len(pipeline)
        if kernel_names[0] == "tcgen05":
            peak = peaks["bf16_tflops"]
            achieved = flops_per_launch / (mean_launch_ms / 1e3) / 1e12
            roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": kernel_traffic(workload),
                    "peak_source": f"{peak_src} dense bf16 burst (fp16 runs at the same rate)"}
        else:
            # CUDA-core FP32 FMA peak: 148 SMs x 128 FMA/clk x 2 FLOP x max SM clock
            peak = 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
            achieved = flops_per_launch / (mean_launch_ms / 1e3) / 1e12
            roof = {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": None,
                    "peak_source": "derived: 148 SM x 128 FP32 FMA/clk x 2 x max SM clock"}
        hbm = bytes_per_launch / (mean_launch_ms / 1e3) / 1e9
        roof["hbm_gbs"] = hbm
        roof["hbm_frac"] = hbm / peaks["hbm_gbs"]
        roof["launch_ms"] = mean_launch_ms
        roof["kernel"] = f"eqlinear_forward[{kernel_names[0]}]"
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            import oracle
            rows = calibrated_oracle_rows(PIPELINES[workload], 10.0)
            secs, rows = oracle_sample(PIPELINES[workload], rows)
            cpu = {"value": rows / secs, "unit": "tokens/s", "cores": oracle.threads_used(),
                   "kind": "oracle",
                   "sample": f"{rows} of {N} rows through every layer, float64, {secs:.1f} s"}
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "f16" if dt == torch.float16 else "f32", "data": "synthetic",
            "tflops": flops * args.steps * world / (elapsed_ms / 1e3) / 1e12,
            "config": {"workload": DESCR[workload], "global_batch": N * world, "seq_len": None,
                       "parallelism": f"replicas x{world} (rows independent)",
                       "l2": f"{nsets} rotating input/output sets of {per_set / 2**20:.0f} MiB "
                             "(> 2x L2)",
                       "kernels": kernel_names},
            "roofline": roof,
            "cpu_baseline": cpu,
            "e2e": {"value": e2e_value, "unit": "tokens/s",
                    "h2d_bytes_per_step": int(x_host.nbytes),
                    "d2h_bytes_per_step": int(y_pin.numel() * y_pin.element_size())},
            "gpu_launches": args.steps * len(pipeline),
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    for p in plans:
        p.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=list(PIPELINES), default="p4_vitb_mlp_f16")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps, reported as run
    if args.impl == "reference":
        return run_reference(args, args.workload)
    return run_ours(args, args.workload)


if __name__ == "__main__":
    sys.exit(main())
