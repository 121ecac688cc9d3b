"""The bench's workload tables and algorithmic accounting (CPU only).

The FLOP counts are the method's (per row: two real GEMMs per real frequency
and four per complex frequency, "Algorithmic approach" item 2; D4: four
characters and the 2 x 2 block), the dense comparator's are 2·N·(C·T)·(D·T);
the traffic table must point at existing kernel sources.
"""
import os
import sys

import bench
from group_circulant_gemm_b200.synth import WORKLOADS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_every_pipeline_resolves_and_chains():
    for name, layers in bench.PIPELINES.items():
        ws = [WORKLOADS[n] for n in layers]
        for a, b in zip(ws, ws[1:]):
            assert a.D == b.C and a.T == b.T and a.N == b.N, name
        assert name in bench.DESCR, name
    for name in bench.CHAINED | bench.SPECTRAL | bench.TILED:
        assert len(bench.PIPELINES[name]) == 2, name
    for name in bench.BACKWARD:
        assert name in bench.PIPELINES
    # the frequency-domain training step is a training step; a pipeline chained
    # through next-layer planes runs in the frequency-domain form
    assert bench.TILED_TRAIN <= bench.BACKWARD
    assert bench.TILED_NEXT <= bench.TILED_LAYERS


def test_every_convolution_workload_is_described():
    from group_circulant_gemm_b200.synth import CONV_WORKLOADS, make_conv_inputs
    for name, w in CONV_WORKLOADS.items():
        assert name in bench.CONV_DESCR, name
        assert w.Ho >= 1 and w.Wo >= 1
    # the training step's upstream gradient has the output's shape
    w = CONV_WORKLOADS["p4_conv3x3_fwd_bwd_f16"]
    assert w.backward
    inp = make_conv_inputs(w, images=2, need_dy=True)
    assert inp["dY"].shape == (2, w.Ho, w.Wo, w.D * w.T)
    # the forward's inputs do not depend on whether dY is drawn (it comes last)
    base = make_conv_inputs(CONV_WORKLOADS["p4_conv3x3_f16"], images=2)
    for k in ("X", "Wc", "bias"):
        assert (base[k] == inp[k]).all(), k


def test_flop_counts():
    w4 = WORKLOADS["p4_vitb_fc1_f16"]      # T = 4: 2 real + 1 complex frequency
    assert bench.layer_flops(w4) == 2.0 * 6 * w4.N * w4.C * w4.D
    w8 = WORKLOADS["c8_1024_f16"]          # T = 8: 2 real + 3 complex
    assert bench.layer_flops(w8) == 2.0 * 14 * w8.N * w8.C * w8.D
    wd = WORKLOADS["p4m_vitb_fc1_f16"]     # D4: 4 characters + 2 x 2 block
    assert bench.layer_flops(wd) == 2.0 * 12 * wd.N * wd.C * wd.D
    # the dense layer the method replaces: 16·N·C·D multiply-adds at T = 4 against
    # the method's 6·N·C·D
    assert bench.dense_flops(w4) == 2.0 * w4.N * (w4.C * 4) * (w4.D * 4)
    assert bench.wgrad_flops(w4) == bench.layer_flops(w4)


def test_layer_bytes_counts_inputs_weights_outputs():
    w = WORKLOADS["p4_vith_fc1_f16"]
    planes = 4 + 1  # T = 4: frequencies 0 and 2, Re/Im of frequency 1, and -Im
    assert bench.layer_bytes(w) == 2 * (w.N * w.C * 4 + w.N * w.D * 4 + planes * w.C * w.D + w.D)


def test_traffic_table_refers_to_existing_sources():
    csrc = os.path.join(bench.ROOT, "group_circulant_gemm_b200", "csrc")
    for family, files in bench.KERNEL_SOURCES.items():
        for f in files:
            assert os.path.exists(os.path.join(csrc, f)), (family, f)
    for (family, _), per_workload in bench.NCU_TRAFFIC.items():
        assert family in bench.KERNEL_SOURCES
        for workload, nbytes in per_workload.items():
            assert workload in bench.PIPELINES or workload in bench.CONV_WORKLOADS
            assert 1e6 < nbytes < 1e9


def _run_bench(args, env_extra=None, timeout=300):
    import json
    import subprocess
    env = dict(os.environ)
    env.pop("WORLD_SIZE", None)
    env.update(env_extra or {})
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], env=env,
                       capture_output=True, text=True, timeout=timeout, cwd=ROOT)
    lines = [json.loads(x) for x in r.stdout.splitlines() if x.startswith("{")]
    return r.returncode, lines, r.stderr


def test_gpus_flag_launches_that_many_ranks():
    """--gpus 2 without a launcher starts two ranks itself (torch.distributed.run on
    127.0.0.1); the host-oracle reference arm needs no GPU, so the path runs here:
    rank 0 prints one line for a world of two, the other rank prints nothing."""
    rc, lines, err = _run_bench(["--gpus", "2", "--impl", "reference", "--steps", "1",
                                 "--warmup", "3", "--ref-seconds", "0.01"])
    assert rc == 0, err[-2000:]
    assert len(lines) == 1 and lines[0]["impl"] == "reference"
    assert lines[0]["n_gpus"] == 2
    assert lines[0]["cpu_baseline"]["cores"] >= 1 and lines[0]["cpu_baseline"]["cpu_model"]


def test_gpus_flag_disagreeing_with_the_launcher_fails_loudly():
    rc, lines, err = _run_bench(["--gpus", "2", "--impl", "reference", "--steps", "1",
                                 "--ref-seconds", "0.01"], {"WORLD_SIZE": "3"}, timeout=120)
    assert rc != 0 and not lines
    assert "WORLD_SIZE=3" in err
