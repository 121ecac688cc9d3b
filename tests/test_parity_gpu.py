"""Parity of the CUDA library against the float64 oracle (GPU required).

Every comparison is element by element on the same seeded, dtype-cast inputs,
with the error metric max|gpu - oracle| / max|oracle| per output tensor and the
bars of the layer's accuracy target: 1e-5 for FP32, 2e-3 for FP16.  All calls
go through the C ABI (group_circulant_gemm_b200.native via EqLinearPlan).
"""
import numpy as np
import pytest
import torch

import oracle
from group_circulant_gemm_b200.synth import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-5, "f16": 2e-3}
TDT = {"f32": torch.float32, "f16": torch.float16}


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def _plan(w: Workload, kernel="auto"):
    from group_circulant_gemm_b200 import EqLinearPlan
    return EqLinearPlan(w.T, w.C, w.D, TDT[w.dtype], kernel=kernel)


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _gpu_forward(w, inp, kernel="auto", bias=True):
    p = _plan(w, kernel)
    W = _dev(inp["W"])
    Wh = p.prepare_weights(W)
    Y = p.forward(_dev(inp["X"]), Wh, _dev(inp["bias"]) if bias else None)
    assert p.status() == 0
    return Y.double().cpu().numpy(), p


def _kernels_for(w, N):
    ks = ["simt"]
    p = _plan(w, "tcgen05")
    if p.forward_kernel_name(N) == "tcgen05":
        ks.append("tcgen05")
    return ks


# --- the five workloads, element by element at sizes the oracle finishes in seconds

SMALL = {
    "p4_small_f32": 256,
    "p4_vitb_proj_f32": 333,
    "p4_vitb_fc1_f16": 333,
    "p4_vitb_fc2_f16": 333,
    "p4_vith_fc1_f16": 261,
    "c8_1024_f16": 389,
}


@pytest.mark.parametrize("name", list(SMALL))
def test_forward_workloads_small(name):
    w = WORKLOADS[name]
    inp = make_inputs(w, rows=SMALL[name])
    ref = oracle.forward(w.T, inp["X"], inp["W"], inp["bias"])
    for k in _kernels_for(w, SMALL[name]):
        Y, _ = _gpu_forward(w, inp, k)
        assert _rel(Y, ref) <= TOL[w.dtype], (name, k, _rel(Y, ref))


def test_small_f32_against_dense_replicated_matrix():
    """Workload 1 also checked against the replicated dense 64x64 matrix."""
    w = WORKLOADS["p4_small_f32"]
    inp = make_inputs(w)
    W = inp["W"].astype(np.float64)
    D, C, T = W.shape
    M = np.zeros((D * T, C * T))
    for d in range(D):
        for s in range(T):
            for c in range(C):
                M[d * T + s, c * T:(c + 1) * T] = np.roll(W[d, c], s)
    ref = inp["X"].astype(np.float64) @ M.T + np.repeat(inp["bias"].astype(np.float64), T)
    Y, _ = _gpu_forward(w, inp)
    assert _rel(Y, ref) <= TOL["f32"]


@pytest.mark.parametrize("name", ["p4_small_f32", "p4_vitb_proj_f32", "p4_vith_fc1_f16",
                                  "c8_1024_f16"])
def test_backward_small(name):
    w = WORKLOADS[name]
    rows = min(SMALL[name], 200)
    inp = make_inputs(w, need_dy=True, rows=rows)
    p = _plan(w)
    Wh = p.prepare_weights(_dev(inp["W"]))
    dX = p.backward_input(_dev(inp["dY"]), Wh).double().cpu().numpy()
    dW, db = p.backward_weight(_dev(inp["X"]), _dev(inp["dY"]))
    assert p.status() == 0
    ref_dX = oracle.backward_input(w.T, inp["dY"], inp["W"])
    ref_dW, ref_db = oracle.backward_weight(w.T, inp["X"], inp["dY"], w.D)
    assert _rel(dX, ref_dX) <= TOL[w.dtype]
    assert _rel(dW.double().cpu().numpy(), ref_dW) <= TOL[w.dtype]
    assert _rel(db.double().cpu().numpy(), ref_db) <= TOL[w.dtype]


# --- edge shapes: ragged tails, tiny sizes, every T ---------------------------------

EDGE = [
    # T, N, C, D
    (1, 7, 5, 3), (2, 65, 9, 17), (3, 129, 7, 33), (4, 1, 1, 1), (4, 63, 17, 65),
    (4, 130, 64, 64), (5, 77, 11, 9), (6, 50, 8, 40), (7, 33, 3, 5), (8, 97, 13, 31),
]


@pytest.mark.parametrize("dtype", ["f32", "f16"])
@pytest.mark.parametrize("T,N,C,D", EDGE)
def test_edge_shapes_all_ops(T, N, C, D, dtype):
    w = Workload("edge", T, N, C, D, dtype, True, 77 + T + N)
    inp = make_inputs(w, need_dy=True)
    ref = oracle.forward(T, inp["X"], inp["W"], inp["bias"])
    Y, p = _gpu_forward(w, inp, "simt")
    assert _rel(Y, ref) <= TOL[dtype]
    Wh = p.prepare_weights(_dev(inp["W"]))
    dX = p.backward_input(_dev(inp["dY"]), Wh).double().cpu().numpy()
    assert _rel(dX, oracle.backward_input(T, inp["dY"], inp["W"])) <= TOL[dtype]
    dW, db = p.backward_weight(_dev(inp["X"]), _dev(inp["dY"]))
    rdW, rdb = oracle.backward_weight(T, inp["X"], inp["dY"], D)
    assert _rel(dW.double().cpu().numpy(), rdW) <= TOL[dtype]
    assert _rel(db.double().cpu().numpy(), rdb) <= TOL[dtype]


TC_EDGE = [
    # T, N, C, D : ragged rows, channels and out-channels for the tcgen05 path
    (4, 1, 16, 16), (4, 127, 48, 144), (4, 129, 80, 208), (4, 300, 208, 16), (4, 513, 64, 384),
    (4, 260, 336, 80),
    (8, 1, 16, 16), (8, 129, 48, 80), (8, 300, 128, 128), (8, 257, 32, 208), (8, 200, 176, 48),
]


@pytest.mark.parametrize("T,N,C,D", TC_EDGE)
def test_tcgen05_edge_shapes(T, N, C, D):
    w = Workload("tcedge", T, N, C, D, "f16", True, 500 + N + C + D)
    inp = make_inputs(w, need_dy=True)
    p = _plan(w, "tcgen05")
    assert p.forward_kernel_name(N) == "tcgen05"
    Wh = p.prepare_weights(_dev(inp["W"]))
    Y = p.forward(_dev(inp["X"]), Wh, _dev(inp["bias"])).double().cpu().numpy()
    assert _rel(Y, oracle.forward(T, inp["X"], inp["W"], inp["bias"])) <= TOL["f16"]
    dX = p.backward_input(_dev(inp["dY"]), Wh).double().cpu().numpy()
    assert _rel(dX, oracle.backward_input(T, inp["dY"], inp["W"])) <= TOL["f16"]
    if T == 4:
        assert p.backward_weight_kernel_name(N) == "tcgen05"
        dW, db = p.backward_weight(_dev(inp["X"]), _dev(inp["dY"]))
        rdW, rdb = oracle.backward_weight(T, inp["X"], inp["dY"], D)
        assert _rel(dW.double().cpu().numpy(), rdW) <= TOL["f16"]
        assert _rel(db.double().cpu().numpy(), rdb) <= TOL["f16"]
    assert p.status() == 0


def test_tcgen05_weight_gradient_matches_simt():
    """Both weight-gradient kernels on the same inputs (several row splits)."""
    w = Workload("wgsimt", 4, 2000, 144, 272, "f16", True, 41)
    inp = make_inputs(w, need_dy=True)
    out = {}
    for k in ("tcgen05", "simt"):
        p = _plan(w, k)
        assert p.backward_weight_kernel_name(w.N) == k
        dW, db = p.backward_weight(_dev(inp["X"]), _dev(inp["dY"]))
        assert p.status() == 0
        out[k] = (dW.double().cpu().numpy(), db.double().cpu().numpy())
    assert _rel(out["tcgen05"][0], out["simt"][0]) <= 1e-3
    assert _rel(out["tcgen05"][1], out["simt"][1]) <= 1e-3


def test_tcgen05_weight_gradient_many_units():
    """More work units than SMs: each CTA runs several units back to back."""
    w = Workload("wgmany", 4, 96, 2048, 2048, "f16", True, 43)
    inp = make_inputs(w, need_dy=True)
    p = _plan(w, "tcgen05")
    dW, db = p.backward_weight(_dev(inp["X"]), _dev(inp["dY"]))
    assert p.status() == 0
    rng = np.random.default_rng(3)
    dd = np.concatenate([rng.integers(0, w.D, 160), [0, w.D - 1]])
    cc = np.concatenate([rng.integers(0, w.C, 160), [w.C - 1, 0]])
    ref = oracle.backward_weight_pairs(w.T, inp["X"], inp["dY"], w.D, dd, cc)
    assert _rel(dW.double().cpu().numpy()[dd, cc, :], ref) <= TOL["f16"]
    ref_db = inp["dY"].astype(np.float64).reshape(w.N, w.D, w.T).sum(axis=(0, 2))
    assert _rel(db.double().cpu().numpy(), ref_db) <= TOL["f16"]


def test_tcgen05_matches_simt_bitwise_structure():
    """Same inputs through both kernel families agree to FP16 output rounding."""
    w = Workload("tcsimt", 4, 1000, 96, 256, "f16", True, 31)
    inp = make_inputs(w)
    a, _ = _gpu_forward(w, inp, "tcgen05")
    b, _ = _gpu_forward(w, inp, "simt")
    assert _rel(a, b) <= 1e-3


def test_no_bias_and_zero_rows():
    w = Workload("nb", 4, 40, 8, 8, "f32", True, 5)
    inp = make_inputs(w, need_dy=True)
    Y, p = _gpu_forward(w, inp, bias=False)
    assert _rel(Y, oracle.forward(4, inp["X"], inp["W"], None)) <= 1e-5
    Wh = p.prepare_weights(_dev(inp["W"]))
    X0 = torch.empty((0, 32), dtype=torch.float32, device="cuda")
    Y0 = p.forward(X0, Wh)
    assert Y0.shape == (0, 32)
    dW, db = p.backward_weight(X0, torch.empty((0, 32), dtype=torch.float32, device="cuda"))
    assert float(dW.abs().max()) == 0.0 and float(db.abs().max()) == 0.0


# --- full sizes, the launch configuration the benchmark times, sampled rows ----------

FULL = ["p4_vitb_proj_f32", "p4_vitb_fc1_f16", "p4_vitb_fc2_f16", "p4_vith_fc1_f16",
        "c8_1024_f16"]


@pytest.mark.parametrize("name", FULL)
def test_forward_full_size_sampled_rows(name):
    w = WORKLOADS[name]
    inp = make_inputs(w)
    rng = np.random.default_rng(99)
    rows = np.unique(np.concatenate([rng.choice(w.N, 48, replace=False),
                                     np.arange(w.N - 16, w.N), np.arange(16)]))
    ref = oracle.forward(w.T, inp["X"][rows], inp["W"], inp["bias"])
    for k in _kernels_for(w, w.N):
        Y, _ = _gpu_forward(w, inp, k)
        assert _rel(Y[rows], ref) <= TOL[w.dtype], (name, k)


def test_backward_full_size_sampled():
    w = WORKLOADS["p4_vith_fc1_f16"]
    inp = make_inputs(w, need_dy=True)
    p = _plan(w)
    assert p.backward_weight_kernel_name(w.N) == "tcgen05"
    Wh = p.prepare_weights(_dev(inp["W"]))
    dX = p.backward_input(_dev(inp["dY"]), Wh).double().cpu().numpy()
    dW, db = p.backward_weight(_dev(inp["X"]), _dev(inp["dY"]))
    assert p.status() == 0
    rng = np.random.default_rng(7)
    rows = np.unique(np.concatenate([rng.choice(w.N, 32, replace=False), [w.N - 1]]))
    ref_dX = oracle.backward_input(w.T, inp["dY"][rows], inp["W"])
    assert _rel(dX[rows], ref_dX) <= TOL["f16"]
    dd = rng.integers(0, w.D, 96)
    cc = rng.integers(0, w.C, 96)
    ref_pairs = oracle.backward_weight_pairs(w.T, inp["X"], inp["dY"], w.D, dd, cc)
    got = dW.double().cpu().numpy()[dd, cc, :]
    # scale of the whole dW (the metric's denominator) from a cheap exact proxy:
    # the sampled pairs' own max, which is a lower bound, makes the check stricter
    assert _rel(got, ref_pairs) <= TOL["f16"]
    ref_db = inp["dY"].astype(np.float64).reshape(w.N, w.D, w.T).sum(axis=(0, 2))
    assert _rel(db.double().cpu().numpy(), ref_db) <= TOL["f16"]


@pytest.mark.parametrize("name", ["p4_vitb_fc1_f16", "c8_1024_f16"])
def test_full_size_equivariance_of_gpu_output(name):
    """Rolling X's group axis by r rolls the GPU's Y by r (any size; GPU vs GPU)."""
    w = WORKLOADS[name]
    inp = make_inputs(w)
    p = _plan(w)
    Wh = p.prepare_weights(_dev(inp["W"]))
    b = _dev(inp["bias"])
    X = _dev(inp["X"])
    Y = p.forward(X, Wh, b).view(w.N, w.D, w.T)
    for r in range(1, w.T):
        Xr = torch.roll(X.view(w.N, w.C, w.T), r, dims=-1).contiguous().view(w.N, -1)
        Yr = p.forward(Xr, Wh, b).view(w.N, w.D, w.T)
        err = (Yr.float() - torch.roll(Y, r, dims=-1).float()).abs().max().item()
        assert err <= TOL[w.dtype] * Y.float().abs().max().item()


# --- error paths through the ABI -------------------------------------------------------

def test_error_paths():
    from group_circulant_gemm_b200 import native as n
    w = Workload("err", 4, 32, 8, 8, "f32", True, 3)
    p = _plan(w)
    X = torch.zeros(32 * 32 + 1, dtype=torch.float32, device="cuda")
    Wh = torch.zeros(n.eqlinear_prepared_weight_bytes(p.handle) // 4, device="cuda")
    Y = torch.zeros(32 * 32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    s = n.raw_status("eqlinear_forward", p.handle, X.data_ptr() + 4, 32, Wh.data_ptr(), None,
                     Y.data_ptr(), st)
    assert s == n.EQL_ERR_ALIGNMENT
    s = n.raw_status("eqlinear_forward", p.handle, X.data_ptr(), -1, Wh.data_ptr(), None,
                     Y.data_ptr(), st)
    assert s == n.EQL_ERR_INVALID_ARG
    ws = torch.zeros(16, dtype=torch.uint8, device="cuda")
    s = n.raw_status("eqlinear_backward_weight", p.handle, X.data_ptr(), Y.data_ptr(), 32,
                     Wh.data_ptr(), None, ws.data_ptr(), 16, st)
    assert s == n.EQL_ERR_WORKSPACE
    assert p.status() == 0


# --- fused activation (EQ-MLP block: EQ-Linear + bias + GELU in the epilogue) ------

ACT_CASES = [
    # T, N, C, D, dtype, kernel
    (4, 333, 192, 768, "f16", "tcgen05"),
    (4, 261, 80, 208, "f16", "tcgen05"),
    (8, 389, 128, 128, "f16", "tcgen05"),
    (4, 256, 16, 16, "f32", "simt"),
    (3, 129, 7, 33, "f16", "simt"),
]


@pytest.mark.parametrize("T,N,C,D,dtype,kernel", ACT_CASES)
def test_forward_gelu_matches_oracle(T, N, C, D, dtype, kernel):
    w = Workload("act", T, N, C, D, dtype, True, 900 + T + N)
    inp = make_inputs(w)
    p = _plan(w, kernel)
    assert p.forward_kernel_name(N) == kernel
    Wh = p.prepare_weights(_dev(inp["W"]))
    Y = p.forward(_dev(inp["X"]), Wh, _dev(inp["bias"]), act="gelu")
    assert p.status() == 0
    ref = oracle.forward(T, inp["X"], inp["W"], inp["bias"], act="gelu")
    assert _rel(Y.double().cpu().numpy(), ref) <= TOL[dtype]


def test_forward_gelu_equivariant_on_gpu():
    w = Workload("acteq", 4, 512, 64, 128, "f16", True, 77)
    inp = make_inputs(w)
    p = _plan(w)
    Wh = p.prepare_weights(_dev(inp["W"]))
    N, C, D, T = w.N, w.C, w.D, w.T
    X = inp["X"]
    Y = p.forward(_dev(X), Wh, _dev(inp["bias"]), act="gelu").float().cpu().numpy()
    for r in range(1, T):
        Xr = np.roll(X.reshape(N, C, T), r, axis=2).reshape(N, C * T)
        Yr = p.forward(_dev(Xr), Wh, _dev(inp["bias"]), act="gelu").float().cpu().numpy()
        Yroll = np.roll(Y.reshape(N, D, T), r, axis=2).reshape(N, D * T)
        assert np.max(np.abs(Yr - Yroll)) <= TOL["f16"] * np.max(np.abs(Y))


def test_forward_act_rejects_unknown_activation():
    from group_circulant_gemm_b200 import native as n
    w = Workload("actbad", 4, 16, 16, 16, "f16", True, 3)
    p = _plan(w)
    X = torch.zeros((16, 64), dtype=torch.float16, device="cuda")
    Y = torch.empty((16, 64), dtype=torch.float16, device="cuda")
    Wh = p.prepare_weights(_dev(make_inputs(w)["W"]))
    s = n.raw_status("eqlinear_forward_act", p.handle, X.data_ptr(), 16, Wh.data_ptr(), None, 7,
                     Y.data_ptr(), None)
    assert s == 1  # EQL_ERR_INVALID_ARG


# --- two-layer block with the intermediate in the frequency domain -------------------

def _planes_of(Y, H):
    """float64 group DFT of a [N, H*4] activation: planes [4, N, H] in the kernel's order,
    times 1/4 (the scale of every stored plane)."""
    g = Y.reshape(Y.shape[0], H, 4)
    return 0.25 * np.stack([g.sum(axis=2), g[..., 0] - g[..., 1] + g[..., 2] - g[..., 3],
                            g[..., 0] - g[..., 2], g[..., 3] - g[..., 1]])


BLOCK_CASES = [
    # N, C, H (hidden), D2, act
    (333, 192, 768, 192, "gelu"),
    (300, 48, 144, 80, "none"),
    (129, 16, 16, 32, "gelu"),
    (1, 32, 64, 48, "none"),
]


@pytest.mark.parametrize("N,C,H,D2,act", BLOCK_CASES)
def test_spectral_block_matches_oracle(N, C, H, D2, act):
    w1 = Workload("blk1", 4, N, C, H, "f16", True, 1300 + N + C)
    w2 = Workload("blk2", 4, N, H, D2, "f16", True, 1400 + N + H)
    in1, in2 = make_inputs(w1), make_inputs(w2, rows=1)
    p1, p2 = _plan(w1), _plan(w2)
    Wh1, Wh2 = p1.prepare_weights(_dev(in1["W"])), p2.prepare_weights(_dev(in2["W"]))
    Xh = p1.forward_to_spectral(_dev(in1["X"]), Wh1, _dev(in1["bias"]), act=act)
    assert tuple(Xh.shape) == (4, N, H)
    Y1 = oracle.forward(4, in1["X"], in1["W"], in1["bias"], act=act)
    assert _rel(Xh.double().cpu().numpy(), _planes_of(Y1, H)) <= TOL["f16"]
    Y = p2.forward_from_spectral(Xh, Wh2, _dev(in2["bias"]))
    assert p1.status() == 0 and p2.status() == 0
    ref = oracle.forward(4, Y1, in2["W"], in2["bias"])
    assert _rel(Y.double().cpu().numpy(), ref) <= TOL["f16"]


def test_spectral_block_full_size_sampled_rows():
    w1, w2 = WORKLOADS["p4_vitb_fc1_f16"], WORKLOADS["p4_vitb_fc2_f16"]
    in1, in2 = make_inputs(w1), make_inputs(w2, rows=1)
    p1, p2 = _plan(w1), _plan(w2)
    Wh1, Wh2 = p1.prepare_weights(_dev(in1["W"])), p2.prepare_weights(_dev(in2["W"]))
    Xh = p1.forward_to_spectral(_dev(in1["X"]), Wh1, _dev(in1["bias"]), act="gelu")
    Y = p2.forward_from_spectral(Xh, Wh2, _dev(in2["bias"])).double().cpu().numpy()
    assert p1.status() == 0 and p2.status() == 0
    rng = np.random.default_rng(5)
    rows = np.unique(np.concatenate([rng.choice(w1.N, 40, replace=False),
                                     np.arange(w1.N - 8, w1.N), np.arange(8)]))
    Y1 = oracle.forward(4, in1["X"][rows], in1["W"], in1["bias"], act="gelu")
    ref = oracle.forward(4, Y1, in2["W"], in2["bias"])
    assert _rel(Y[rows], ref) <= TOL["f16"]


def test_spectral_entry_points_reject_unsupported_plans():
    from group_circulant_gemm_b200 import native as n
    w = Workload("blkbad", 8, 16, 16, 16, "f16", True, 3)  # T = 8: no spectral form
    p = _plan(w)
    X = torch.zeros((16, 128), dtype=torch.float16, device="cuda")
    Xh = torch.zeros((4, 16, 16), dtype=torch.float16, device="cuda")
    Wh = p.prepare_weights(_dev(make_inputs(w)["W"]))
    s = n.raw_status("eqlinear_forward_to_spectral", p.handle, X.data_ptr(), 16, Wh.data_ptr(),
                     None, 0, Xh.data_ptr(), None)
    assert s == 2  # EQL_ERR_UNSUPPORTED


@pytest.mark.parametrize("N,C,D", [(151 * 128 - 51, 64, 128), (150 * 128, 32, 256), (300, 64, 128)])
def test_last_wave_half_units_match_oracle(N, C, D):
    """Tiles of the last partial wave run as two 64-row halves (M = 64 MMAs): every row
    of the split tiles, and a sample of whole-tile rows, against the oracle."""
    w = Workload("halves", 4, N, C, D, "f16", True, 700 + N)
    inp = make_inputs(w)
    p = _plan(w, "tcgen05")
    Wh = p.prepare_weights(_dev(inp["W"]))
    Y = p.forward(_dev(inp["X"]), Wh, _dev(inp["bias"])).double().cpu().numpy()
    assert p.status() == 0
    n_dt = (D + 127) // 128
    tiles = ((N + 127) // 128) * n_dt
    rem = tiles % 148 if tiles >= 148 else tiles
    first_split_row = ((tiles - rem) // n_dt) * 128
    rng = np.random.default_rng(1)
    rows = np.unique(np.concatenate([np.arange(first_split_row, N),
                                     rng.integers(0, max(first_split_row, 1), 64)]))
    ref = oracle.forward(4, inp["X"][rows], inp["W"], inp["bias"])
    assert _rel(Y[rows], ref) <= TOL["f16"]
