#!/usr/bin/env python
"""Throughput of the EQ-Linear forward on B200, one JSON line on rank 0.

Default workload: the p4 (T=4) FP16 ViT-B MLP pair, N = 12608 rows (64 images x
197 tokens), layer 1 C=192 -> D=768 (768 -> 3072 features), layer 2 C=768 ->
D=192 (3072 -> 768) applied to layer 1's output.  One step = the group DFT of X
into tiled spectral planes, then both layers as one chained launch on SM pairs
(the first layer's epilogue writes the second layer's planes).  `value` = rows (tokens) per second over the whole job, inputs
resident in HBM; `e2e` = the same through the C ABI with the step's input copied
from pinned host memory and the result read back, inside the timed region.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
       [--workload p4_vitb_mlp_f16|p4_vitb_mlp_fused_f16|p4_vitb_mlp_2calls_f16|
                   p4_vitb_proj_f32|p4_vitb_proj_f32_simt|p4_vith_fc1_f16|
                   c8_1024_f16|c8_1024_tiled_f16|p4_vith_fc1_fwd_bwd_f16|
                   p4_vitb_mlp_block_f16|p4_vitb_mlp_spectral_f16|p4m_vitb_mlp_f16|
                   p4m_vitb_mlp_fused_f16|p4_conv3x3_f16] [--dp-path]
       [--wgrad-transform] [--no-dense] [--no-cpu-baseline] [--eager]
The training workload (p4_vith_fc1_fwd_bwd_f16) is forward, dX and dW; the
forward and dX kernels save the group spectra of X and dY, which dW multiplies
directly (--wgrad-transform: dW transforms X and dY itself).
Under torchrun (N > 1) every rank runs its own copy of the workload (weak
scaling; rows are independent, so no collective is on the forward path).  The
training workload is then data parallel: each rank's FP32 weight gradient is
summed over ranks by one NCCL all-reduce and rounded once.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from group_circulant_gemm_b200.synth import (CONV_WORKLOADS, WORKLOADS,  # noqa: E402
                                             make_conv_inputs, make_inputs)

METRIC = "EQ-Linear fwd tokens/s + TFLOP/s (T=4, fp16/fp32) and % of tensor roofline"
L2_BYTES = 126 * 1024 * 1024
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# workload name -> list of layer workloads applied in sequence (output feeds the next)
PIPELINES = {
    "p4_vitb_mlp_f16": ["p4_vitb_fc1_f16", "p4_vitb_fc2_f16"],
    "p4_vitb_mlp_fused_f16": ["p4_vitb_fc1_f16", "p4_vitb_fc2_f16"],
    "p4_vitb_mlp_2calls_f16": ["p4_vitb_fc1_f16", "p4_vitb_fc2_f16"],
    "p4_vitb_proj_f32": ["p4_vitb_proj_f32"],
    "p4_vitb_proj_f32_simt": ["p4_vitb_proj_f32"],
    "p4_vith_fc1_f16": ["p4_vith_fc1_f16"],
    "c8_1024_f16": ["c8_1024_f16"],
    "c8_1024_tiled_f16": ["c8_1024_f16"],
    "p4_vith_fc1_fwd_bwd_f16": ["p4_vith_fc1_f16"],
    "p4_vith_fc1_fwd_bwd_tiled_f16": ["p4_vith_fc1_f16"],
    "p4_vitb_mlp_block_f16": ["p4_vitb_fc1_f16", "p4_vitb_fc2_f16"],
    "p4_vitb_mlp_spectral_f16": ["p4_vitb_fc1_f16", "p4_vitb_fc2_f16"],
    "p4m_vitb_mlp_f16": ["p4m_vitb_fc1_f16", "p4m_vitb_fc2_f16"],
    "p4m_vitb_mlp_fused_f16": ["p4m_vitb_fc1_f16", "p4m_vitb_fc2_f16"],
}
# pipelines whose layers are over the dihedral group D4 (T = 8 elements) instead
# of the cyclic group
DIHEDRAL = {"p4m_vitb_mlp_f16", "p4m_vitb_mlp_fused_f16"}
# two-layer pipelines whose intermediate stays in the frequency domain (the first
# layer's epilogue writes the second layer's operand planes)
SPECTRAL = {"p4_vitb_mlp_block_f16", "p4_vitb_mlp_spectral_f16"}
BACKWARD = {"p4_vith_fc1_fwd_bwd_f16", "p4_vith_fc1_fwd_bwd_tiled_f16"}
# training steps in the frequency-domain form: one group-DFT launch for X (it
# serves the forward and dW) and one for dY (dX and dW), the products on SM pairs
# (eqlinear_forward_tiled, eqlinear_backward_input_tiled) and the weight gradient
# from the two tiled planes (eqlinear_backward_weight_tiled)
TILED_TRAIN = {"p4_vith_fc1_fwd_bwd_tiled_f16"}
# two-layer pipelines run as one chained launch (eqlinear_forward_chain: both
# layers' tiles in one dynamic queue; bitwise the two separate calls)
CHAINED = {"p4_vitb_mlp_fused_f16", "p4_vitb_mlp_block_f16", "p4_vitb_mlp_spectral_f16"}
# two-layer pipelines run on tiled spectral planes: one group-DFT launch, then both
# layers in one chained launch on SM pairs (eqlinear_group_dft +
# eqlinear_forward_chain_tiled; bitwise the per-layer tiled calls)
TILED = {"p4_vitb_mlp_f16"}
# layers in the frequency-domain form, one layer at a time: per layer a group
# Fourier transform launch (tiled planes; TF32 hi/lo planes for FP32), then the
# pair kernel (eqlinear_forward_tiled): the FP32 layer with 3xTF32 split
# precision, the cyclic T = 8 layer and the D4 layers with eight planes
TILED_LAYERS = {"p4_vitb_proj_f32", "c8_1024_tiled_f16", "p4m_vitb_mlp_f16"}
# of those, pipelines whose layers after the first take their input planes from
# the previous layer's epilogue (eqlinear_forward_tiled_next): one group-DFT
# launch per step
TILED_NEXT = {"p4m_vitb_mlp_f16"}
# per-layer output activation (fused into that layer's epilogue); default none
ACTS = {"p4_vitb_mlp_block_f16": ["gelu", "none"]}


def acts_of(workload):
    return ACTS.get(workload, ["none"] * len(PIPELINES[workload]))
DESCR = {
    "p4_vitb_mlp_f16": "p4 EQ-Linear fp16 ViT-B MLP pair: N=12608, C=192->D=768 then "
                       "C=768->D=192, T=4; group DFT of X to tiled planes, then both layers "
                       "in one chained launch on SM pairs",
    "p4_vitb_mlp_fused_f16": "p4 EQ-Linear fp16 ViT-B MLP pair: N=12608, C=192->D=768 then "
                             "C=768->D=192, T=4; both layers in one chained launch, the "
                             "group transforms fused into the GEMM kernel",
    "p4_vitb_mlp_2calls_f16": "p4 EQ-Linear fp16 ViT-B MLP pair: N=12608, C=192->D=768 then "
                              "C=768->D=192, T=4; one launch per layer",
    "p4_vitb_proj_f32": "p4 EQ-Linear fp32 ViT-B projection: N=12608, C=D=192, T=4; group DFT "
                        "to TF32 hi/lo planes, then 3xTF32 products on SM-pair tensor cores",
    "p4_vitb_proj_f32_simt": "p4 EQ-Linear fp32 ViT-B projection: N=12608, C=D=192, T=4; FP32 FMA "
                             "on the CUDA cores",
    "p4_vith_fc1_f16": "p4 EQ-Linear fp16 ViT-H fc1: N=8224, C=320->D=1280, T=4",
    "c8_1024_f16": "cyclic T=8 EQ-Linear fp16: N=16384, C=D=128; group DFT fused into the "
                   "one-CTA GEMM kernel",
    "c8_1024_tiled_f16": "cyclic T=8 EQ-Linear fp16: N=16384, C=D=128; group DFT to eight tiled "
                         "planes, then the products on SM pairs",
    "p4_vith_fc1_fwd_bwd_f16": "p4 EQ-Linear fp16 ViT-H fc1 forward + dX + dW: N=8224, "
                               "C=320->D=1280, T=4; forward and dX in the one-CTA kernel, "
                               "saving the group spectra that dW reads",
    "p4_vith_fc1_fwd_bwd_tiled_f16": "p4 EQ-Linear fp16 ViT-H fc1 forward + dX + dW: N=8224, "
                                     "C=320->D=1280, T=4; group DFTs of X and dY to tiled "
                                     "planes, forward and dX on SM pairs, dW from the planes",
    "p4_vitb_mlp_block_f16": "p4 EQ-MLP block fp16 ViT-B: N=12608, EQ-Linear 192->768 + bias + "
                             "GELU (fused), EQ-Linear 768->192 + bias, T=4; intermediate kept as "
                             "the second layer's spectral planes; one chained launch",
    "p4_vitb_mlp_spectral_f16": "p4 EQ-Linear fp16 ViT-B MLP pair: N=12608, C=192->D=768 then "
                                "C=768->D=192, T=4; intermediate kept as the second layer's "
                                "spectral planes; one chained launch",
    "p4m_vitb_mlp_f16": "p4m (dihedral D4, 8 elements) EQ-Linear fp16 ViT-B MLP pair: N=12608, "
                        "C=96->D=384 then C=384->D=96 per group element (768->3072->768 "
                        "features); the group Fourier transform of X to eight tiled "
                        "planes, fc1 on SM pairs writing fc2's planes from its epilogue, "
                        "fc2 on SM pairs",
    "p4m_vitb_mlp_fused_f16": "p4m (dihedral D4, 8 elements) EQ-Linear fp16 ViT-B MLP pair: "
                              "N=12608, C=96->D=384 then C=384->D=96 per group element; one "
                              "launch of the fused one-CTA kernel per layer",
}


def is_d4(w) -> bool:
    return w.name.startswith("p4m_")


def layer_flops(w) -> float:
    """Algorithmic FLOPs of one forward: 2 * (real GEMMs per frequency plan) * N*C*D
    (D4: four characters and a 2 x 2 block, 4 + 8 real GEMMs)."""
    if is_d4(w):
        return 2.0 * 12 * w.N * w.C * w.D
    nr = 2 if w.T % 2 == 0 else 1
    nc = (w.T - nr) // 2
    return 2.0 * (nr + 4 * nc) * w.N * w.C * w.D


def layer_bytes(w) -> float:
    """Algorithmic HBM bytes of one forward: read X, prepared weights, bias; write Y."""
    es = 2 if w.dtype == "f16" else 4
    nr = 2 if w.T % 2 == 0 else 1
    planes = 8 if is_d4(w) else w.T + (w.T - nr) // 2
    return es * (w.N * w.C * w.T + w.N * w.D * w.T + planes * w.C * w.D + w.D)


# DRAM bytes (read + write) per launch of the step's dominant kernel, from the
# ncu captures summarised under profiles/, keyed by a hash of the kernel's
# sources: a changed kernel reports null until it is captured again.
KERNEL_SOURCES = {
    "forward": ("eql_tc_fwd.cu", "eql_tc_fwd_parts.cuh", "eql_tc_common.cuh"),
    "forward_chain": ("eql_tc_chain.cu", "eql_tc_fwd_parts.cuh", "eql_tc_common.cuh"),
    "conv": ("eql_tc_conv.cu", "eql_tc_fwd_parts.cuh", "eql_tc_common.cuh"),
    "backward_weight": ("eql_tc_wgrad.cu", "eql_tc_common.cuh"),
    "forward_chain_tiled": ("eql_tc_pair.cu", "eql_tc_pair_common.cuh", "eql_tc_fwd_parts.cuh",
                            "eql_tc_common.cuh"),
    "forward_tiled": ("eql_tc_pair32.cu", "eql_tc_pair8.cu", "eql_tc_pair_common.cuh",
                      "eql_tc_fwd_parts.cuh", "eql_tc_common.cuh"),
    "forward_pair": ("eql_tc_pair.cu", "eql_tc_pair_common.cuh", "eql_tc_fwd_parts.cuh",
                     "eql_tc_common.cuh"),
}
NCU_TRAFFIC = {
    ("forward", "443ba94f5b306a59"): {"p4_vitb_mlp_2calls_f16": 58.96e6, "c8_1024_f16": 34.20e6, "p4_vith_fc1_f16": 51.20e6, "p4_vith_fc1_fwd_bwd_f16": 109.13e6, "p4m_vitb_mlp_fused_f16": 57.79e6},
    ("forward_chain", "246b0f491b3357c1"): {"p4_vitb_mlp_fused_f16": 89.59e6, "p4_vitb_mlp_spectral_f16": 80.93e6, "p4_vitb_mlp_block_f16": 81.74e6},
    ("conv", "ae4ea6f4164e2f9d"): {"p4_conv3x3_f16": 161.54e6},
    ("forward_chain_tiled", "6ade53bcfcfaa10b"): {"p4_vitb_mlp_f16": 99.44e6},
    ("forward_pair", "6ade53bcfcfaa10b"): {"p4_vith_fc1_fwd_bwd_tiled_f16": 96.53e6},
    ("forward_tiled", "2fe2ac1739cebc38"): {"p4_vitb_proj_f32": 85.81e6, "p4m_vitb_mlp_f16": 59.08e6, "c8_1024_tiled_f16": 34.38e6},
}

def kernel_traffic(family: str, workload: str):
    import hashlib
    files = KERNEL_SOURCES.get(family)
    if not files:
        return None
    m = hashlib.sha256()
    try:
        for f in files:
            with open(os.path.join(ROOT, "group_circulant_gemm_b200", "csrc", f), "rb") as fh:
                m.update(fh.read())
    except OSError:
        return None
    return NCU_TRAFFIC.get((family, m.hexdigest()[:16]), {}).get(workload)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            return json.load(f), "measured"
    return dict(FALLBACK_PEAKS), "fallback"


class ClockSampler:
    """SM clocks and clock-event (throttle) reasons, polled through NVML every ~2 ms.

    `mark()` brackets the timed region (called with the GPU idle, right before the
    timed launches are queued and right after they completed), so only samples
    taken while the timed kernels ran are reported.
    """

    REASONS = {"hw_slowdown": 0x8, "hw_thermal_slowdown": 0x40,
               "sw_thermal_slowdown": 0x20, "sw_power_cap": 0x4}

    def __init__(self, cuda_index: int):
        self.cuda_index = cuda_index
        self.samples = []  # (host time, sm MHz, max sm MHz, reason bits)
        self.window = [None, None]
        self._stop = threading.Event()
        self._thread = None
        self._nvml = None

    def _handle(self, nv):
        import torch
        try:
            uuid = str(torch.cuda.get_device_properties(self.cuda_index).uuid)
            return nv.nvmlDeviceGetHandleByUUID(uuid if uuid.startswith("GPU-") else "GPU-" + uuid)
        except Exception:
            return nv.nvmlDeviceGetHandleByIndex(self.cuda_index)

    def start(self):
        try:
            import pynvml as nv
            nv.nvmlInit()
            h = self._handle(nv)
            mx = float(nv.nvmlDeviceGetMaxClockInfo(h, nv.NVML_CLOCK_SM))
            reasons = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
                nv.nvmlDeviceGetCurrentClocksThrottleReasons
        except Exception:
            return
        self._nvml = nv

        def one():
            try:
                sm = float(nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM))
                self.samples.append((time.perf_counter(), sm, mx, int(reasons(h))))
            except Exception:
                pass
        self._one = one

        def run():
            while not self._stop.is_set():
                one()
                time.sleep(0.002)

        self._thread = threading.Thread(target=run, daemon=True)
        self._thread.start()

    def mark(self, which: int):
        self.window[which] = time.perf_counter()

    def sample_now(self):
        """One sample from the calling thread (the timed loop calls this every few
        launches, while the GPU works through the queue, so a short timed region
        is covered even when the polling thread is not scheduled)."""
        one = getattr(self, "_one", None)
        if one is not None:
            one()

    def stop(self):
        out = {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0,
               "source": "nvml, 2 ms polling, samples inside the timed region"}
        if self._thread is None:
            out["source"] = "unavailable (NVML could not be opened)"
            return out
        self._stop.set()
        self._thread.join(timeout=5)
        t0, t1 = self.window
        inside = [s for s in self.samples if t0 is not None and t1 is not None and t0 <= s[0] <= t1]
        if inside:
            bits = 0
            for s in inside:
                bits |= s[3]
            out.update(sm_mhz=statistics.median(s[1] for s in inside),
                       sm_max_mhz=max(s[2] for s in inside),
                       reasons=sorted(k for k, v in self.REASONS.items() if bits & v),
                       samples=len(inside))
        try:
            self._nvml.nvmlShutdown()
        except Exception:
            pass
        return out


def capture_graphs(step, nsets):
    """One CUDA graph per rotating input/output set, each holding one step's
    launches, so the timed region replays them without per-launch host work."""
    import torch
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for k in range(nsets):
            step(k)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graphs = []
    for k in range(nsets):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            step(k)
        graphs.append(g)
    for g in graphs:
        g.replay()
    torch.cuda.synchronize()
    return graphs


def graph_op_times(step, nsets, op_steps, first):
    """Per-launch device times of each op of a step, from CUDA graphs that hold
    the step with event-record nodes around every launch (one graph per rotating
    set).  Each replay runs alone (synchronised after it), so a launch's time
    holds no host work: in eager launches the event before a kernel can complete
    while the host is still encoding that kernel's arguments.  Returns an array
    [op_steps, ops], or None when events cannot be captured (then the caller
    times eager launches)."""
    import torch
    try:
        gs, evs = [], []
        for k in range(nsets):
            e = []
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                step(first + k, e, external=True)
            gs.append(g)
            evs.append(e)
        rows = []
        for i in range(op_steps):
            k = i % nsets
            gs[k].replay()
            torch.cuda.synchronize()
            e = evs[k]
            rows.append([e[2 * j].elapsed_time(e[2 * j + 1]) for j in range(len(e) // 2)])
        return np.array(rows)
    except Exception as exc:  # noqa: BLE001 - fall back to eager timing, say so
        print(f"per-launch timing inside graphs unavailable ({exc}); timing eager launches",
              file=sys.stderr)
        return None


def new_event(external: bool = False):
    """A timing event recorded on the current stream (inside a graph capture,
    `external` makes the record a node of the graph)."""
    import torch
    e = torch.cuda.Event(enable_timing=True, external=external)
    e.record()
    return e


def dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return world, rank, local


def oracle_sample(pipeline, rows: int, backward: bool = False, acts=None):
    """Time the float64 oracle on `rows` rows of the step's ops; returns (seconds, rows)."""
    import oracle
    oracle.build()
    layers = [(WORKLOADS[name], make_inputs(WORKLOADS[name], rows=rows, need_dy=backward))
              for name in pipeline]
    acts = acts or ["none"] * len(layers)
    x = layers[0][1]["X"].astype(np.float64)
    t0 = time.perf_counter()
    for (w, inp), act in zip(layers, acts):
        if is_d4(w):
            x = oracle.d4_forward(x, inp["W"], inp["bias"], act=act)
        else:
            x = oracle.forward(w.T, x, inp["W"], inp["bias"], act=act)
    if backward:
        w, inp = layers[0]
        oracle.backward_input(w.T, inp["dY"], inp["W"])
        oracle.backward_weight(w.T, inp["X"], inp["dY"], w.D)
    return time.perf_counter() - t0, rows


def calibrated_oracle_rows(pipeline, target_s: float, backward: bool = False, acts=None) -> int:
    t, r = oracle_sample(pipeline, 16, backward, acts)
    n_full = WORKLOADS[pipeline[0]].N
    return int(max(16, min(n_full, 16 * target_s / max(t, 1e-6))))


def reference_step_seconds(args) -> float:
    """Host-oracle seconds per step of the reference arm: the whole run (warm-up
    + timed steps) takes about two minutes, at most 20 s a step, unless
    --ref-seconds sets it."""
    if args.ref_seconds is not None:
        return max(1e-3, args.ref_seconds)
    return min(20.0, max(1.0, 120.0 / max(1, args.steps + args.warmup)))


def layer_cpu_baseline(workload, backward: bool, N: int) -> dict:
    """The oracle on the host cores, a calibrated sample (~15 s with all threads,
    ~5 s with one) through every op of the step; rows/s."""
    import oracle
    pipeline, acts = PIPELINES[workload], acts_of(workload)
    rows = calibrated_oracle_rows(pipeline, 15.0, backward, acts)
    secs, rows = oracle_sample(pipeline, rows, backward, acts)
    cores = oracle.threads_used()
    oracle.set_threads(1)
    try:
        rows1 = calibrated_oracle_rows(pipeline, 5.0, backward, acts)
        secs1, rows1 = oracle_sample(pipeline, rows1, backward, acts)
    finally:
        oracle.set_threads(None)
    return {"value": rows / secs, "unit": "tokens/s", "cores": cores,
            "cpu_model": oracle.cpu_model(), "kind": "oracle",
            "sample": f"{rows} of {N} rows through every op of the step, float64, "
                      f"{secs:.1f} s",
            "value_1thread": rows1 / secs1,
            "sample_1thread": f"{rows1} rows, 1 thread, {secs1:.1f} s"}


def conv_cpu_baseline(w) -> dict:
    """The convolution oracle on the host cores (~15 s) and on one thread (~5 s)."""
    import oracle
    images = conv_oracle_images(w, 15.0)
    secs = conv_oracle_sample(w, images)
    cores = oracle.threads_used()
    oracle.set_threads(1)
    try:
        images1 = conv_oracle_images(w, 5.0)
        secs1 = conv_oracle_sample(w, images1)
    finally:
        oracle.set_threads(None)
    return {"value": images * w.Ho * w.Wo / secs, "unit": "tokens/s", "cores": cores,
            "cpu_model": oracle.cpu_model(), "kind": "oracle",
            "sample": f"{images} of {w.N} images, float64, {secs:.1f} s",
            "value_1thread": images1 * w.Ho * w.Wo / secs1,
            "sample_1thread": f"{images1} images, 1 thread, {secs1:.1f} s"}


def use_all_host_cores(world: int) -> None:
    """Under a launcher with several ranks (torchrun sets OMP_NUM_THREADS=1 per
    rank) rank 0 runs the host oracle alone, so it gets every core it may use."""
    if world > 1:
        import oracle
        oracle.set_threads(len(os.sched_getaffinity(0)))


def run_reference(args, workload):
    """Reference arm: the float64 oracle on the host cores, bounded sample per step."""
    import oracle
    world, rank, _ = dist_init()
    if rank != 0:
        return 0
    use_all_host_cores(world)
    pipeline = PIPELINES[workload]
    backward = workload in BACKWARD
    acts = acts_of(workload)
    rows = calibrated_oracle_rows(pipeline, reference_step_seconds(args), backward, acts)
    for _ in range(args.warmup):
        oracle_sample(pipeline, rows, backward, acts)
    times = [oracle_sample(pipeline, rows, backward, acts)[0] for _ in range(args.steps)]
    total = sum(times)
    value = rows * args.steps / total
    w0 = WORKLOADS[pipeline[0]]
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": DESCR[workload], "rows_per_step": rows, "global_batch": w0.N,
                   "seq_len": None, "parallelism": "none (host oracle)"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.threads_used(),
                         "cpu_model": oracle.cpu_model(), "kind": "oracle",
                         "sample": f"{rows} of {w0.N} rows per step through every layer"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def wgrad_flops(w) -> float:
    return layer_flops(w)  # same per-frequency products, reduced over rows


def dense_flops(w) -> float:
    return 2.0 * w.N * (w.C * w.T) * (w.D * w.T)


def dense_comparator(pipeline, backward, xs, dys, nsets, steps, rank, acts=None, eager=False):
    """Same-GPU dense baseline: torch F.linear (cuBLAS) on the replicated
    (D*T x C*T) matrix M[(d,s),(c,t)] = W[d,c,(t-s) mod T] in the same dtype, GEMM
    time only (M built outside the timed region); for the training step also
    dX = dY M and the dense weight-gradient GEMM dY^T X."""
    import torch
    import torch.nn.functional as F
    stream = torch.cuda.current_stream()
    Ms, bs = [], []
    for w in pipeline:
        inp = make_inputs(w.with_(seed=w.seed + 1000 * rank), rows=1)
        W = torch.from_numpy(inp["W"]).cuda()
        M = torch.empty((w.D, w.T, w.C, w.T), dtype=W.dtype, device="cuda")
        if is_d4(w):
            # M[(d,g),(c,h)] = W[d, c, g^-1 h] with g = a + 4b for r^a m^b (m r m = r^-1)
            def mul(g, h):
                a, bb, c, e = g & 3, g >> 2, h & 3, h >> 2
                return ((a + (-c if bb else c)) & 3) + 4 * (bb ^ e)

            def inv(g):
                return ((g & 3) if g >> 2 else (-(g & 3)) & 3) + 4 * (g >> 2)
            for g in range(8):
                idx = torch.tensor([mul(inv(g), h) for h in range(8)], device="cuda")
                M[:, g] = W[:, :, idx]
        else:
            for sh in range(w.T):
                M[:, sh] = torch.roll(W, shifts=sh, dims=2)
        Ms.append(M.reshape(w.D * w.T, w.C * w.T))
        bs.append(torch.from_numpy(inp["bias"]).cuda().repeat_interleave(w.T) if w.bias else None)
    outs = []

    def step(i, events=None, external=False):
        def mark():
            if events is not None:
                events.append(new_event(external))
        x = xs[i % nsets]
        for li in range(len(pipeline)):
            mark()
            x = F.linear(x, Ms[li], bs[li])
            if acts and acts[li] == "gelu":
                x = F.gelu(x)
            mark()
        if backward:
            dy = dys[i % nsets]
            mark()
            dx = dy @ Ms[0]
            mark()
            mark()
            dw = dy.t() @ xs[i % nsets]
            mark()
            del dx, dw
        del x

    for i in range(3):
        step(i)
    torch.cuda.synchronize()
    # timed the same way as our step: CUDA graph replays, per-op times from an
    # eager pass with events
    graphs = None if eager else capture_graphs(step, nsets)
    ev = []
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(steps):
        if graphs is not None:
            graphs[(3 + i) % nsets].replay()
        else:
            step(3 + i, ev)
    t1.record(stream)
    torch.cuda.synchronize()
    ms = t0.elapsed_time(t1) / steps
    op_steps = steps
    per_op = None
    if graphs is not None:
        op_steps = min(steps, 50)
        per_op = graph_op_times(step, nsets, op_steps, 3)
        if per_op is None:
            for i in range(op_steps):
                step(3 + i, ev)
            torch.cuda.synchronize()
    if per_op is None:
        nops = len(ev) // 2 // op_steps
        per_op = np.array([ev[2 * j].elapsed_time(ev[2 * j + 1])
                           for j in range(len(ev) // 2)]).reshape(op_steps, nops)
    op_ms = per_op.mean(axis=0)
    flops = sum(dense_flops(w) for w in pipeline) + (2 * dense_flops(pipeline[0]) if backward else 0)
    return {"kind": "dense F.linear on the replicated (D*T x C*T) matrix, cuBLAS, same dtype, "
                    "GEMM time only" + ("; training step adds dY@M and dY^T@X" if backward else "")
                    + ("; F.gelu after the layers that fuse it" if acts and "gelu" in acts else ""),
            "value": pipeline[0].N / (ms / 1e3), "unit": "tokens/s", "ms_per_step": ms,
            "op_ms": [round(float(m), 5) for m in op_ms],
            "tflops": flops / (ms / 1e3) / 1e12}


def run_ours(args, workload):
    import torch
    import torch.distributed as dist

    world, rank, local = dist_init()
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    from group_circulant_gemm_b200 import EqLinearPlan, forward_chain, native
    from group_circulant_gemm_b200.layer import forward_chain_tiled
    from group_circulant_gemm_b200.parallel import allreduce_grad_buffer

    backward = workload in BACKWARD
    pipeline = [WORKLOADS[n] for n in PIPELINES[workload]]
    dt = torch.float16 if pipeline[0].dtype == "f16" else torch.float32
    N = pipeline[0].N
    es = 2 if dt == torch.float16 else 4
    stream = torch.cuda.current_stream()

    # weights: prepared once, outside the timed region
    plans, whats, biases = [], [], []
    for w in pipeline:
        inp = make_inputs(w.with_(seed=w.seed + 1000 * rank), rows=1)
        p = EqLinearPlan(w.T, w.C, w.D, dt, group="dihedral4" if is_d4(w) else "cyclic")
        W = torch.from_numpy(inp["W"]).cuda()
        plans.append(p)
        whats.append(p.prepare_weights(W))
        biases.append(torch.from_numpy(inp["bias"]).cuda() if w.bias else None)
    first = make_inputs(pipeline[0].with_(seed=pipeline[0].seed + 1000 * rank), need_dy=backward)
    x_host = first["X"]
    dy_host = first.get("dY")

    # rotating input/output sets so the step's working set leaves L2 between steps
    per_set = sum(N * w.C * w.T * es + N * w.D * w.T * es for w in pipeline)
    tiled = workload in TILED
    tiled_layers = workload in TILED_LAYERS
    if tiled_layers:
        # every layer input's tiled planes (rows padded to the 128-row tile)
        per_set += sum(int(np.prod(plans[li].tiled_shape(N, w.C))) * es
                       for li, w in enumerate(pipeline))
    if tiled:
        # X's tiled planes (rows padded to the kernel's 128-row tile)
        per_set += int(np.prod(plans[0].tiled_shape(N, pipeline[0].C))) * es
    if backward:
        per_set += sum(N * w.D * w.T * es + N * w.C * w.T * es for w in pipeline)
    # training: the forward and dX kernels save the group spectra of X and dY
    # (the same sizes) for the weight gradient, unless --wgrad-transform
    tiled_train = workload in TILED_TRAIN
    if tiled_train:
        # the tiled planes of X and of dY
        per_set += sum(int(np.prod(plans[0].tiled_shape(N, c))) * es
                       for c in (pipeline[0].C, pipeline[0].D))
    saved = backward and not args.wgrad_transform and not tiled_train
    if saved:
        per_set += sum(N * w.C * w.T * es + N * w.D * w.T * es for w in pipeline[:1])
    nsets = max(2, int(np.ceil(2 * L2_BYTES / per_set)))
    xs = [torch.from_numpy(x_host).cuda() for _ in range(nsets)]
    outs = [[torch.empty((N, w.D * w.T), dtype=dt, device="cuda") for w in pipeline]
            for _ in range(nsets)]
    # data parallel: every rank trains on its own rows; the weight gradient is
    # summed over ranks in FP32 (one NCCL all-reduce) and rounded once
    dp = backward and (world > 1 or args.dp_path)
    if backward:
        w0 = pipeline[0]
        dys = [torch.from_numpy(dy_host).cuda() for _ in range(nsets)]
        dxs = [torch.empty((N, w0.C * w0.T), dtype=dt, device="cuda") for _ in range(nsets)]
        # two gradient buffers (set i uses i % 2) so that the end-to-end loop can
        # copy one step's dW out while the next step computes
        gbufs = [plans[0].grad_buffer(dt) for _ in range(2)]
        gbuf = gbufs[0]
        gbuf32 = plans[0].grad_buffer(torch.float32) if dp else None
        ws = torch.empty(max(16, plans[0].workspace_bytes(N)), dtype=torch.uint8, device="cuda")
        if saved:
            xhats = [torch.empty((4, N, w0.C), dtype=dt, device="cuda") for _ in range(nsets)]
            ghats = [torch.empty((4, N, w0.D), dtype=dt, device="cuda") for _ in range(nsets)]

    # the ops of one step: (label, kernel, flops, algorithmic bytes, callable(set index))
    ops = []
    acts = acts_of(workload)
    spectral = workload in SPECTRAL
    if spectral:
        # the first layer writes the second layer's input planes [4, N, H]
        outs = [[torch.empty((4, N, pipeline[0].D), dtype=dt, device="cuda"), o[1]]
                for o in outs]
    chained = workload in CHAINED
    if tiled:
        # the intermediate is the second layer's tiled planes, written by the first
        # layer's epilogue
        w1, w2 = pipeline
        xts = [torch.empty(plans[0].tiled_shape(N, w1.C), dtype=dt, device="cuda")
               for _ in range(nsets)]
        outs = [[torch.empty(plans[0].tiled_shape(N, w1.D), dtype=dt, device="cuda"), o[1]]
                for o in outs]
        ws_tiled = torch.zeros(max(16, native.eqlinear_chain_tiled_workspace_bytes(
            plans[0].handle, plans[1].handle, N)), dtype=torch.uint8, device="cuda")

        def group_dft(i):
            plans[0].group_dft(xs[i % nsets], out=xts[i % nsets])

        def fwd_chain_tiled(i):
            o = outs[i % nsets]
            forward_chain_tiled(plans[0], plans[1], xts[i % nsets], N, whats[0], biases[0],
                                whats[1], biases[1], act=acts[0], Ht=o[0], Y=o[1],
                                workspace=ws_tiled)
        # the transform reads X and writes its planes (the same bytes); its
        # additions are not counted as the method's FLOPs
        ops.append(("group_dft", "simt", 0.0, 2.0 * es * N * w1.C * w1.T, group_dft))
        ops.append(("forward_chain_tiled", "tcgen05", sum(layer_flops(w) for w in pipeline),
                    sum(layer_bytes(w) for w in pipeline), fwd_chain_tiled))
    if chained:
        ws_chain = torch.zeros(max(16, native.eqlinear_chain_workspace_bytes(
            plans[0].handle, plans[1].handle, N)), dtype=torch.uint8, device="cuda")

        def fwd_chain(i):
            o = outs[i % nsets]
            forward_chain(plans[0], plans[1], xs[i % nsets], whats[0], biases[0], whats[1],
                          biases[1], act=acts[0], spectral=spectral, H=o[0], Y=o[1],
                          workspace=ws_chain)
        ops.append(("forward_chain", "tcgen05", sum(layer_flops(w) for w in pipeline),
                    sum(layer_bytes(w) for w in pipeline), fwd_chain))
    if tiled_layers:
        # planes / input bytes: the FP32 form stores TF32 hi and lo parts
        pf = 2 if dt == torch.float32 else 1
        tkern = "tcgen05-3xtf32" if dt == torch.float32 else "tcgen05"
        xts = [[torch.empty(plans[li].tiled_shape(N, w.C), dtype=dt, device="cuda")
                for li, w in enumerate(pipeline)] for _ in range(nsets)]
        chained_next = workload in TILED_NEXT
        for li, w in enumerate(pipeline):
            def dft_l(i, li=li):
                x = xs[i % nsets] if li == 0 else outs[i % nsets][li - 1]
                plans[li].group_dft(x, out=xts[i % nsets][li])

            def fwd_l(i, li=li):
                if chained_next and li + 1 < len(pipeline):
                    # the next layer's input planes straight from this epilogue
                    plans[li].forward_tiled_next(xts[i % nsets][li], N, whats[li], biases[li],
                                                 act=acts[li], out=xts[i % nsets][li + 1])
                else:
                    plans[li].forward_tiled(xts[i % nsets][li], N, whats[li], biases[li],
                                            act=acts[li], out=outs[i % nsets][li])
            # the transform reads the input and writes its planes; the products read
            # the planes and the weight stages and write the output (or the next
            # layer's planes, the same bytes at T = 8)
            if li == 0 or not chained_next:
                ops.append(("group_dft", "simt", 0.0, (1 + pf) * es * N * w.C * w.T, dft_l))
            ops.append(("forward_tiled", tkern, layer_flops(w),
                        layer_bytes(w) + (pf - 1) * es * N * w.C * w.T, fwd_l))
    if tiled_train:
        w0 = pipeline[0]
        xts = [torch.empty(plans[0].tiled_shape(N, w0.C), dtype=dt, device="cuda")
               for _ in range(nsets)]
        dyts = [torch.empty(plans[0].tiled_shape(N, w0.D), dtype=dt, device="cuda")
                for _ in range(nsets)]

        def dft_x(i):
            plans[0].group_dft(xs[i % nsets], out=xts[i % nsets])

        def fwd_t(i):
            plans[0].forward_tiled(xts[i % nsets], N, whats[0], biases[0], act=acts[0],
                                   out=outs[i % nsets][0])
        ops.append(("group_dft", "simt", 0.0, 2.0 * es * N * w0.C * w0.T, dft_x))
        ops.append(("forward_pair", "tcgen05", layer_flops(w0), layer_bytes(w0), fwd_t))
    for li, w in enumerate([] if chained or tiled or tiled_layers or tiled_train
                           else pipeline):
        def fwd(i, li=li):
            x = xs[i % nsets] if li == 0 else outs[i % nsets][li - 1]
            if spectral and li == 0:
                plans[li].forward_to_spectral(x, whats[li], biases[li], act=acts[li],
                                              out=outs[i % nsets][li])
            elif spectral and li == 1:
                plans[li].forward_from_spectral(x, whats[li], biases[li], act=acts[li],
                                                out=outs[i % nsets][li])
            elif saved and li == 0:
                plans[li].forward_save_spectrum(x, whats[li], biases[li], act=acts[li],
                                                out=outs[i % nsets][li], Xhat=xhats[i % nsets])
            else:
                plans[li].forward(x, whats[li], biases[li], out=outs[i % nsets][li],
                                  act=acts[li])
        # a saved spectrum is one more write of X's size
        extra = es * w.N * w.C * w.T if saved and li == 0 else 0
        ops.append(("forward", plans[li].forward_kernel_name(N), layer_flops(w),
                    layer_bytes(w) + extra, fwd))
    if backward:
        w0 = pipeline[0]
        pending = []

        def dft_dy(i):
            plans[0].group_dft(dys[i % nsets], out=dyts[i % nsets])

        def bwd_x(i):
            if tiled_train:
                plans[0].backward_input_tiled(dyts[i % nsets], N, whats[0], out=dxs[i % nsets])
            elif saved:
                plans[0].backward_input_save_spectrum(dys[i % nsets], whats[0],
                                                      out=dxs[i % nsets], dYhat=ghats[i % nsets])
            else:
                plans[0].backward_input(dys[i % nsets], whats[0], out=dxs[i % nsets])

        def bwd_w(i):
            # the weight gradient reads the spectra (or X and dY: the same bytes)
            a = xhats[i % nsets] if saved else xs[i % nsets]
            g = ghats[i % nsets] if saved else dys[i % nsets]
            if tiled_train:
                a, g = xts[i % nsets], dyts[i % nsets]
            if dp:
                if tiled_train:
                    plans[0].backward_weight_tiled_f32(a, g, N, buf=gbuf32, workspace=ws)
                elif saved:
                    plans[0].backward_weight_from_spectra_f32(a, g, buf=gbuf32, workspace=ws)
                else:
                    plans[0].backward_weight_f32(a, g, buf=gbuf32, workspace=ws)
                # queued behind dW; dX runs on the compute stream meanwhile
                pending.append(allreduce_grad_buffer(gbuf32, async_op=True))
            else:
                dW, db = plans[0].split_grad(gbufs[i % 2])
                if tiled_train:
                    plans[0].backward_weight_tiled(a, g, N, dW=dW, dbias=db, workspace=ws)
                elif saved:
                    plans[0].backward_weight_from_spectra(a, g, dW=dW, dbias=db, workspace=ws)
                else:
                    plans[0].backward_weight(a, g, dW=dW, dbias=db, workspace=ws)

        def grad_sync(i):
            handle = pending.pop()
            if handle is not None:  # None: one rank, nothing was reduced
                handle.wait()
            plans[0].cast_from_f32(gbuf32, out=gbuf)
        nb = es * (N * w0.C * w0.T + N * w0.D * w0.T)
        op_dx = ("backward_input", plans[0].forward_kernel_name(N), layer_flops(w0),
                 nb + es * 1.25 * w0.C * w0.D * w0.T + (es * N * w0.D * w0.T if saved else 0),
                 bwd_x)
        if tiled_train:
            # dX reads dY's planes (dY's bytes) and the adjoint weight stages
            op_dx = ("backward_input_pair", "tcgen05", layer_flops(w0),
                     nb + es * 1.25 * w0.C * w0.D * w0.T, bwd_x)
        op_dw = ("backward_weight", plans[0].backward_weight_kernel_name(N), wgrad_flops(w0),
                 nb + es * w0.D * w0.C * w0.T, bwd_w)
        if dp:
            # dW from saved spectra needs dX's saved dY spectrum, so it follows dX;
            # the transforming dW (and dW from tiled planes, which needs only dY's
            # transform) goes first and its all-reduce overlaps dX
            first_two = [op_dx, op_dw] if saved else [op_dw, op_dx]
            ops += first_two + [("weight_grad_allreduce", "nccl+cast", 0.0,
                                 (4 + es) * gbuf.numel(), grad_sync)]
        else:
            ops += [op_dx, op_dw]
        if tiled_train:
            ops.insert(len(ops) - (3 if dp else 2),
                       ("group_dft", "simt", 0.0, 2.0 * es * N * w0.D * w0.T, dft_dy))

    def step(i, events=None, external=False):
        for _, _, _, _, fn in ops:
            if events is not None:
                events.append(new_event(external))
            fn(i)
            if events is not None:
                events.append(new_event(external))

    kernel_names = [k for _, k, _, _, _ in ops]
    # the clock sampler runs from the start of warm-up to the end of the timed region
    clocks = ClockSampler(local)
    if rank == 0:
        clocks.start()
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    for p in plans:
        assert p.status() == 0

    # the timed steps replay CUDA graphs (one per rotating set); the data-parallel
    # training step, whose all-reduce is queued asynchronously, runs eagerly
    graphs = None if (dp or args.eager) else capture_graphs(step, nsets)
    for p in plans:
        assert p.status() == 0

    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.mark(0)
    ev = []
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        if graphs is not None:
            graphs[(args.warmup + i) % nsets].replay()
        else:
            step(args.warmup + i, ev)
        if rank == 0 and i % 16 == 15:
            clocks.sample_now()
    t1.record(stream)
    torch.cuda.synchronize()
    clocks.mark(1)
    if world > 1:
        dist.barrier()
    clk = clocks.stop() if rank == 0 else {}
    elapsed_ms = t0.elapsed_time(t1)
    op_steps = args.steps
    launch_ms = None
    if graphs is not None:
        # per-launch times: the step's graphs again, with event nodes around every
        # launch (eager launches if events cannot be captured)
        op_steps = min(args.steps, 100)
        launch_ms = graph_op_times(step, nsets, op_steps, args.warmup)
        if launch_ms is None:
            for i in range(op_steps):
                step(args.warmup + i, ev)
            torch.cuda.synchronize()
        for p in plans:
            assert p.status() == 0
    in_graph = launch_ms is not None
    if launch_ms is None:
        launch_ms = np.array([ev[2 * j].elapsed_time(ev[2 * j + 1])
                              for j in range(len(ev) // 2)]).reshape(op_steps, len(ops))
    timing = ("CUDA graph replay of each step (one graph per rotating set); per-launch times "
              + (f"from {op_steps} replays of the step's graphs with event nodes around each "
                 "launch" if in_graph else
                 f"from {op_steps} eager steps with events around each launch")
              if graphs is not None else "eager launches with events around each launch")

    # end to end through the ABI: pinned host inputs -> device, the step, results -> host
    x_pin = torch.from_numpy(x_host).pin_memory()
    y_pin = torch.empty((N, pipeline[-1].D * pipeline[-1].T), dtype=dt).pin_memory()
    h2d = x_pin.numel() * x_pin.element_size()
    d2h = y_pin.numel() * y_pin.element_size()
    if backward:
        dy_pin = torch.from_numpy(dy_host).pin_memory()
        dx_pin = torch.empty(tuple(dxs[0].shape), dtype=dt).pin_memory()
        dw_pin = torch.empty(tuple(gbuf.shape), dtype=dt).pin_memory()
        h2d += dy_pin.numel() * dy_pin.element_size()
        d2h += (dx_pin.numel() + dw_pin.numel()) * dx_pin.element_size()

    # Each step's copies overlap the neighbouring steps' compute: copy-in,
    # compute and copy-out streams over two device input/output sets, ordered by
    # events (a set is refilled only after the step two back has read it, and
    # its outputs are overwritten only after that step's copy-out).  The
    # data-parallel training step keeps its copies and kernels in order on one
    # stream (its all-reduce and cast share one buffer).
    piped = not dp
    s_in = torch.cuda.Stream() if piped else stream
    s_out = torch.cuda.Stream() if piped else stream
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_c = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(k):
        if not piped:
            xs[0].copy_(x_pin, non_blocking=True)
            dys[0].copy_(dy_pin, non_blocking=True)
            step(0)
            y_pin.copy_(outs[0][-1], non_blocking=True)
            dx_pin.copy_(dxs[0], non_blocking=True)
            dw_pin.copy_(gbuf, non_blocking=True)
            return
        j = k % 2
        with torch.cuda.stream(s_in):
            if k >= 2:
                s_in.wait_event(ev_c[j])
            xs[j].copy_(x_pin, non_blocking=True)
            if backward:
                dys[j].copy_(dy_pin, non_blocking=True)
            ev_in[j].record(s_in)
        stream.wait_event(ev_in[j])
        if k >= 2:
            stream.wait_event(ev_out[j])
        step(j)
        ev_c[j].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_c[j])
            y_pin.copy_(outs[j][-1], non_blocking=True)
            if backward:
                dx_pin.copy_(dxs[j], non_blocking=True)
                dw_pin.copy_(gbufs[j], non_blocking=True)
            ev_out[j].record(s_out)

    for k in range(2):
        e2e_step(k)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for k in range(args.steps):
        e2e_step(k)
    e1.record(s_out)
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
        flops = sum(f for _, _, f, _, _ in ops)
        value = world * N * args.steps / (elapsed_ms / 1e3)
        e2e_value = world * N * args.steps / (e2e_ms / 1e3)
        # dominant kernel: the kernel family with the largest share of the step
        mean_ms = launch_ms.mean(axis=0)
        fam = {}
        for j, (label, kern, f, nbytes, _) in enumerate(ops):
            key = ({"backward_input": "forward", "backward_input_pair": "forward_pair"}
                   .get(label, label), kern)
            a = fam.setdefault(key, [0.0, 0.0, 0.0, 0])
            a[0] += mean_ms[j]
            a[1] += f
            a[2] += nbytes
            a[3] += 1
        (dlabel, dkern), (dms, dflops, dbytes, dcount) = max(fam.items(), key=lambda kv: kv[1][0])
        mean_launch_ms = dms / dcount
        flops_per_launch = dflops / dcount
        bytes_per_launch = dbytes / dcount
        achieved = flops_per_launch / (mean_launch_ms / 1e3) / 1e12
        if dkern == "tcgen05-3xtf32":
            # TF32 peak from the measured BF16 one and the nominal TF32:BF16 ratio
            # (1.1 : 2.25 PFLOP/s dense); the split precision runs three TF32
            # products per product of the method, so 1/3 is this path's ceiling
            peak = peaks["bf16_tflops"] * 1.1 / 2.25
            roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": kernel_traffic(dlabel, workload),
                    "peak_source": f"{peak_src} dense bf16 burst x 1.1/2.25 (TF32)",
                    "mma_flops_per_method_flop": 3}
        elif dkern == "tcgen05":
            peak = peaks["bf16_tflops"]
            roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak,
                    # the training step's forward family stores spectra unless
                    # --wgrad-transform: its counters were taken in that mode only
                    "traffic": (None if backward and args.wgrad_transform
                                else kernel_traffic(dlabel, workload)),
                    "peak_source": f"{peak_src} dense bf16 burst (fp16 runs at the same rate)"}
        else:
            # CUDA-core FP32 FMA peak: 148 SMs x 128 FMA/clk x 2 FLOP x max SM clock
            peak = 148 * 128 * 2 * peaks.get("sm_max_mhz", 1965.0) * 1e6 / 1e12
            roof = {"bound": "alu", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                    "frac": achieved / peak, "traffic": None,
                    "peak_source": "derived: 148 SM x 128 FP32 FMA/clk x 2 x max SM clock"}
        hbm = bytes_per_launch / (mean_launch_ms / 1e3) / 1e9
        roof["hbm_gbs"] = hbm
        roof["hbm_frac"] = hbm / peaks["hbm_gbs"]
        roof["launch_ms"] = mean_launch_ms
        roof["kernel"] = f"eqlinear_{dlabel}[{dkern}]"
        roof["step_share"] = dms / float(mean_ms.sum())
        comparator = None
        if not args.no_dense:
            comparator = dense_comparator(pipeline, backward, xs, dys if backward else None,
                                          nsets, min(args.steps, 200), rank, acts, args.eager)
            comparator["ours_over_dense"] = value / comparator["value"]
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cpu = layer_cpu_baseline(workload, backward, N)
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None,
            "dtype": "f16" if dt == torch.float16 else "f32", "data": "synthetic",
            "tflops": flops * args.steps * world / (elapsed_ms / 1e3) / 1e12,
            "tflops_dense_equiv": (sum(dense_flops(w) for w in pipeline)
                                   + (2 * dense_flops(pipeline[0]) if backward else 0))
                                  * args.steps * world / (elapsed_ms / 1e3) / 1e12,
            "config": {"workload": DESCR[workload], "global_batch": N * world, "seq_len": None,
                       "parallelism": (f"data parallel x{world}: rows sharded, dW/dbias "
                                       "FP32 NCCL all-reduce overlapped with dX"
                                       if dp else f"replicas x{world} (rows independent)"),
                       "l2": f"{nsets} rotating input/output sets of {per_set / 2**20:.0f} MiB "
                             "(> 2x L2)",
                       "kernels": [f"{label}[{k}]" for label, k, _, _, _ in ops],
                       "timing": timing},
            "op_ms": [round(float(m), 5) for m in mean_ms],
            "roofline": roof,
            "cpu_baseline": cpu,
            "dense_comparator": comparator,
            "e2e": {"value": e2e_value, "unit": "tokens/s",
                    "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
                    "copies": ("in order with the kernels on one stream" if dp else
                               "overlapped with the neighbouring steps' kernels (copy-in, "
                               "compute, copy-out streams; two device sets)")},
            "gpu_launches": args.steps * sum(2 if label == "backward_weight" else 1
                                             for label, _, _, _, _ in ops),
            # (the all-reduce op counts its cast kernel; NCCL's own kernel is not ours)
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    for p in plans:
        p.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


CONV_DESCR = {
    "p4_conv3x3_f16": "p4 group-circulant convolution fp16: 64 images 56x56, C=64->D=64 per "
                      "group element (256 -> 256 features), 3x3 taps, stride 1, zero padding 1, "
                      "T=4",
    "p4_conv3x3_fwd_bwd_f16": "p4 group-circulant convolution fp16 training step (forward, dX, "
                              "dWc + dbias): 64 images 56x56, C=64->D=64 per group element, "
                              "3x3 taps, stride 1, zero padding 1, T=4",
}


def conv_flops(w) -> float:
    """Algorithmic FLOPs of one pass (forward, dX or dWc): the layer's 12*C*D per
    output pixel and tap (6 real GEMMs)."""
    return 12.0 * w.N * w.Ho * w.Wo * w.C * w.D * w.KH * w.KW


def conv_dense_flops(w) -> float:
    return 2.0 * w.N * w.Ho * w.Wo * (w.C * w.T) * (w.D * w.T) * w.KH * w.KW


def conv_oracle_sample(w, images: int):
    import oracle
    oracle.build()
    inp = make_conv_inputs(w, images=images, need_dy=w.backward)
    t0 = time.perf_counter()
    oracle.conv_forward(w.T, inp["X"], inp["Wc"], inp["bias"], pad=(w.ph, w.pw))
    if w.backward:
        oracle.conv_backward_input(w.T, inp["dY"], inp["Wc"], w.H, w.W, pad=(w.ph, w.pw))
        oracle.conv_backward_weight(w.T, inp["X"], inp["dY"], w.KH, w.KW, pad=(w.ph, w.pw))
    return time.perf_counter() - t0


def conv_oracle_images(w, target_s: float) -> int:
    t1 = conv_oracle_sample(w, 1)
    return int(max(1, min(w.N, target_s / max(t1, 1e-6))))


def run_conv_reference(args, workload):
    import oracle
    world, rank, _ = dist_init()
    if rank != 0:
        return 0
    use_all_host_cores(world)
    w = CONV_WORKLOADS[workload]
    images = conv_oracle_images(w, reference_step_seconds(args))
    for _ in range(args.warmup):
        conv_oracle_sample(w, images)
    times = [conv_oracle_sample(w, images) for _ in range(args.steps)]
    total = sum(times)
    value = images * w.Ho * w.Wo * args.steps / total
    sample = f"{images} of {w.N} images per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": CONV_DESCR[workload], "images_per_step": images,
                   "global_batch": w.N, "seq_len": None, "parallelism": "none (host oracle)",
                   "tokens": "output pixels"},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.threads_used(),
                         "cpu_model": oracle.cpu_model(), "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_conv(args, workload):
    """The convolution step: one eqlinear_conv_forward (planes pre-pass + tap-loop
    kernel) over the whole batch; tokens = output pixels."""
    import torch
    import torch.distributed as dist
    import torch.nn.functional as F

    world, rank, local = dist_init()
    torch.cuda.set_device(local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    from group_circulant_gemm_b200 import EqLinearPlan

    w = CONV_WORKLOADS[workload]
    bwd = w.backward
    inp = make_conv_inputs(w.with_(seed=w.seed + 1000 * rank), need_dy=bwd)
    p = EqLinearPlan(w.T, w.C, w.D, torch.float16)
    Wc = torch.from_numpy(inp["Wc"]).cuda()
    Wh = p.conv_prepare_weights(Wc)
    bias = torch.from_numpy(inp["bias"]).cuda()
    x_host = inp["X"]
    pixels = w.N * w.Ho * w.Wo
    per_set = x_host.nbytes + pixels * w.D * w.T * 2
    if bwd:
        per_set += inp["dY"].nbytes + x_host.nbytes  # dY in, dX out
    nsets = max(2, int(np.ceil(2 * L2_BYTES / per_set)))
    xs = [torch.from_numpy(x_host).cuda() for _ in range(nsets)]
    ys = [torch.empty((w.N, w.Ho, w.Wo, w.D * w.T), dtype=torch.float16, device="cuda")
          for _ in range(nsets)]
    from group_circulant_gemm_b200 import native
    ws = torch.empty(native.eqlinear_conv_workspace_bytes(p.handle, w.N, w.H, w.W),
                     dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream()

    def fwd(i):
        p.conv_forward(xs[i % nsets], Wh, w.KH, w.KW, bias, pad=(w.ph, w.pw),
                       out=ys[i % nsets], workspace=ws)
    # (label, kernel family, FLOPs, launches, callable)
    ops = [("conv_forward", "conv", conv_flops(w), 2, fwd)]
    if bwd:
        dys = [torch.from_numpy(inp["dY"]).cuda() for _ in range(nsets)]
        dxs = [torch.empty_like(xs[0]) for _ in range(nsets)]
        gW = torch.empty((w.KH, w.KW, w.D, w.C, w.T), dtype=torch.float16, device="cuda")
        gb = torch.empty((w.D,), dtype=torch.float16, device="cuda")
        wsb = torch.empty(native.eqlinear_conv_backward_workspace_bytes(
            p.handle, w.N, w.H, w.W, w.KH, w.KW, w.ph, w.pw), dtype=torch.uint8, device="cuda")

        def bwd_x(i):
            p.conv_backward_input(dys[i % nsets], Wh, w.KH, w.KW, w.H, w.W, pad=(w.ph, w.pw),
                                  out=dxs[i % nsets], workspace=wsb)

        def bwd_w(i):
            p.conv_backward_weight(xs[i % nsets], dys[i % nsets], w.KH, w.KW, pad=(w.ph, w.pw),
                                   workspace=wsb, dW=gW, dbias=gb)
        # dX: the planes pre-pass of dY and the tap-loop kernel; dWc: X and dY onto
        # the padded grid (and their group spectra), then per tap the layer's
        # weight gradient and its finalize
        ops += [("conv_backward_input", "conv", conv_flops(w), 2, bwd_x),
                ("conv_backward_weight", "conv_wgrad", conv_flops(w),
                 # two copies onto the padded grid; with C and D multiples of 64 two
                 # spectra passes and one weight gradient + finalize for all taps,
                 # else per tap a weight gradient + finalize
                 2 + (4 if w.C % 64 == 0 and w.D % 64 == 0 else 2 * w.KH * w.KW),
                 bwd_w)]

    def step(i, events=None, external=False):
        for _, _, _, _, fn in ops:
            if events is not None:
                events.append(new_event(external))
            fn(i)
            if events is not None:
                events.append(new_event(external))

    clocks = ClockSampler(local)
    if rank == 0:
        clocks.start()
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    graphs = None if args.eager else capture_graphs(step, nsets)
    assert p.status() == 0
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    clocks.mark(0)
    ev = []
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    for i in range(args.steps):
        if graphs is not None:
            graphs[(args.warmup + i) % nsets].replay()
        else:
            step(args.warmup + i, ev)
        if rank == 0 and i % 16 == 15:
            clocks.sample_now()
    t1.record(stream)
    torch.cuda.synchronize()
    clocks.mark(1)
    if world > 1:
        dist.barrier()
    clk = clocks.stop() if rank == 0 else {}
    elapsed_ms = t0.elapsed_time(t1)
    op_steps = args.steps
    per_call = None
    if graphs is not None:
        op_steps = min(args.steps, 100)
        per_call = graph_op_times(step, nsets, op_steps, args.warmup)
        if per_call is None:
            for i in range(op_steps):
                step(args.warmup + i, ev)
            torch.cuda.synchronize()
    in_graph = per_call is not None
    if per_call is None:
        per_call = np.array([ev[2 * j].elapsed_time(ev[2 * j + 1])
                             for j in range(len(ev) // 2)]).reshape(-1, len(ops))
    op_ms = per_call.mean(axis=0)
    timing = ("CUDA graph replay of each step (one graph per rotating set); per-call time "
              + (f"from {op_steps} replays of the step's graphs with event nodes around the "
                 "call" if in_graph else f"from {op_steps} eager steps with events around each call")
              if graphs is not None else "eager launches with events around each call")

    x_pin = torch.from_numpy(x_host).pin_memory()
    y_pin = torch.empty(tuple(ys[0].shape), dtype=torch.float16).pin_memory()
    h2d, d2h = x_pin.numel() * 2, y_pin.numel() * 2
    if bwd:
        dy_pin = torch.from_numpy(inp["dY"]).pin_memory()
        dx_pin = torch.empty(tuple(dxs[0].shape), dtype=torch.float16).pin_memory()
        dw_pin = torch.empty(tuple(gW.shape), dtype=torch.float16).pin_memory()
        h2d += dy_pin.numel() * 2
        d2h += (dx_pin.numel() + dw_pin.numel()) * 2

    # copies overlap the neighbouring steps' calls, as in the layer workloads
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_c = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def e2e_step(k):
        j = k % 2
        with torch.cuda.stream(s_in):
            if k >= 2:
                s_in.wait_event(ev_c[j])
            xs[j].copy_(x_pin, non_blocking=True)
            if bwd:
                dys[j].copy_(dy_pin, non_blocking=True)
            ev_in[j].record(s_in)
        stream.wait_event(ev_in[j])
        if k >= 2:
            stream.wait_event(ev_out[j])
        step(j)
        ev_c[j].record(stream)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_c[j])
            y_pin.copy_(ys[j], non_blocking=True)
            if bwd:
                dx_pin.copy_(dxs[j], non_blocking=True)
                dw_pin.copy_(gW, non_blocking=True)
            ev_out[j].record(s_out)
    for k in range(2):
        e2e_step(k)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for k in range(args.steps):
        e2e_step(k)
    e1.record(s_out)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1)
    assert p.status() == 0
    times = torch.tensor([elapsed_ms, e2e_ms], dtype=torch.float64, device="cuda")
    if world > 1:
        dist.all_reduce(times, op=dist.ReduceOp.MAX)
    elapsed_ms, e2e_ms = times.tolist()

    if rank == 0:
        peaks, peak_src = load_peaks()
        flops = sum(f for _, _, f, _, _ in ops)
        value = world * pixels * args.steps / (elapsed_ms / 1e3)
        # dominant kernel family: the forward and dX run the same convolution kernel
        fam = {}
        for j, (_, fk, f, _, _) in enumerate(ops):
            a = fam.setdefault(fk, [0.0, 0.0, 0])
            a[0] += op_ms[j]
            a[1] += f
            a[2] += 1
        dfam, (fam_ms, dflops, dcount) = max(fam.items(), key=lambda kv: kv[1][0])
        launch_ms = fam_ms / dcount
        achieved = dflops / dcount / (launch_ms / 1e3) / 1e12
        # one convolution pass reads its input and the weights and writes its output
        nbytes = x_host.nbytes + pixels * w.D * w.T * 2 + inp["Wc"].nbytes
        hbm = nbytes / (launch_ms / 1e3) / 1e9
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
                "traffic": kernel_traffic("conv", workload) if dfam == "conv" else None,
                "peak_source": f"{peak_src} dense bf16 burst (fp16 runs at the same rate)",
                "hbm_gbs": hbm, "hbm_frac": hbm / peaks["hbm_gbs"], "launch_ms": launch_ms,
                "kernel": ("eqlinear_conv_forward / conv_backward_input[planes pre-pass + "
                           "tcgen05 tap loop]" if dfam == "conv" else
                           "eqlinear_conv_backward_weight[padded grid + per-tap layer dW]"),
                "step_share": fam_ms / float(op_ms.sum())}
        comparator = None
        if not args.no_dense:
            # cuDNN on the replicated dense kernel K[(d,s),(c,t),i,j] = Wc[i,j,d,c,(t-s) mod T]
            K = torch.stack([torch.roll(Wc, shifts=sh, dims=4) for sh in range(w.T)])
            K = K.permute(3, 0, 4, 5, 1, 2).reshape(w.D * w.T, w.C * w.T, w.KH, w.KW)
            K = K.contiguous(memory_format=torch.channels_last)
            brep = bias.repeat_interleave(w.T)

            def dense(i):
                x = xs[i % nsets].permute(0, 3, 1, 2)
                y = F.conv2d(x, K, brep, padding=(w.ph, w.pw))
                if bwd:
                    g = dys[i % nsets].permute(0, 3, 1, 2)
                    torch.nn.grad.conv2d_input(x.shape, K, g, padding=(w.ph, w.pw))
                    torch.nn.grad.conv2d_weight(x, K.shape, g, padding=(w.ph, w.pw))
                    g.sum(dim=(0, 2, 3))
                return y
            for i in range(3):
                dense(i)
            torch.cuda.synchronize()
            dgraphs = None if args.eager else capture_graphs(lambda i: dense(i), nsets)
            d0 = torch.cuda.Event(enable_timing=True)
            d1 = torch.cuda.Event(enable_timing=True)
            nd = min(args.steps, 100)
            d0.record(stream)
            for i in range(nd):
                if dgraphs is not None:
                    dgraphs[i % nsets].replay()
                else:
                    dense(i)
            d1.record(stream)
            torch.cuda.synchronize()
            dms = d0.elapsed_time(d1) / nd
            comparator = {"kind": "dense F.conv2d (cuDNN, channels-last) with the replicated "
                                  "(D*T x C*T x KH x KW) kernel, same dtype"
                                  + ("; plus cuDNN's input and weight gradients and the bias "
                                     "sum" if bwd else ""),
                          "value": pixels / (dms / 1e3), "unit": "tokens/s",
                          "ms_per_step": dms,
                          "tflops": conv_dense_flops(w) * (3 if bwd else 1) / (dms / 1e3)
                                    / 1e12}
            comparator["ours_over_dense"] = value / world / comparator["value"]
        cpu = None
        if world == 1 and not args.no_cpu_baseline:
            cpu = conv_cpu_baseline(w)
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": elapsed_ms / args.steps, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
            "tflops": flops * args.steps * world / (elapsed_ms / 1e3) / 1e12,
            "tflops_dense_equiv": conv_dense_flops(w) * (3 if bwd else 1) * args.steps * world
                                  / (elapsed_ms / 1e3) / 1e12,
            "config": {"workload": CONV_DESCR[workload], "global_batch": w.N * world,
                       "seq_len": None, "tokens": "output pixels",
                       "parallelism": f"replicas x{world} (images independent)",
                       "l2": f"{nsets} rotating input/output sets of {per_set / 2**20:.0f} MiB "
                             "(> 2x L2)",
                       "kernels": [f"{label}[{fk}]" for label, fk, _, _, _ in ops],
                       "timing": timing},
            "op_ms": [round(float(m), 5) for m in op_ms],
            "roofline": roof,
            "cpu_baseline": cpu,
            "dense_comparator": comparator,
            "e2e": {"value": world * pixels * args.steps / (e2e_ms / 1e3), "unit": "tokens/s",
                    "h2d_bytes_per_step": int(h2d),
                    "d2h_bytes_per_step": int(d2h),
                    "copies": "overlapped with the neighbouring steps' calls (copy-in, "
                              "compute, copy-out streams; two device sets)"},
            "gpu_launches": sum(n for _, _, _, n, _ in ops) * args.steps,
            "clocks": clk,
        }
        print(json.dumps(line), flush=True)
    p.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def spawn_ranks(n: int) -> int:
    """Run this same command as n ranks on this node (torch.distributed.run,
    rendezvous on 127.0.0.1), so that --gpus N without a launcher still runs N
    ranks; rank 0 prints the result line.  Returns the launcher's exit code."""
    import socket
    import subprocess
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n}", "--master-addr", "127.0.0.1", f"--master-port={port}",
           os.path.abspath(__file__), *sys.argv[1:]]
    return subprocess.call(cmd)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=500)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", choices=list(PIPELINES) + list(CONV_WORKLOADS),
                    default="p4_vitb_mlp_f16")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-dense", action="store_true", help="skip the dense F.linear comparator")
    ap.add_argument("--eager", action="store_true",
                    help="time eager launches instead of replaying CUDA graphs of the step")
    ap.add_argument("--wgrad-transform", action="store_true",
                    help="training workload: the weight gradient transforms X and dY itself "
                         "instead of reading the spectra the forward and dX kernels saved")
    ap.add_argument("--dp-path", action="store_true",
                    help="training workload: take the data-parallel weight-gradient path "
                         "(FP32 sums, reduction over ranks, one cast) even on one rank")
    ap.add_argument("--ref-seconds", type=float, default=None,
                    help="reference arm: host-oracle seconds per step (default: about two "
                         "minutes for the whole run, at most 20 s a step)")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)  # at least 3 untimed warm-up steps, reported as run
    env_world = os.environ.get("WORLD_SIZE")
    if env_world is None and args.gpus > 1:
        # not launched by torchrun: start one rank per GPU ourselves
        return spawn_ranks(args.gpus)
    if env_world is not None and int(env_world) != args.gpus:
        print(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={env_world}; launch one rank per "
              "GPU (torchrun --nproc-per-node N) with --gpus N", file=sys.stderr, flush=True)
        return 2
    if args.workload in CONV_WORKLOADS:
        if args.impl == "reference":
            return run_conv_reference(args, args.workload)
        return run_conv(args, args.workload)
    if args.impl == "reference":
        return run_reference(args, args.workload)
    return run_ours(args, args.workload)


if __name__ == "__main__":
    sys.exit(main())
