"""Backward of the layer over the dihedral group D4 (GPU required).

The gradients of Y[n,d,g] = bias[d] + sum_{c,h} W[d,c,g^-1 h] X[n,c,h]:
  * dX[n,c,h] = sum_{d,g} W[d,c,g^-1 h] dY[n,d,g] is the D4 layer of dY with
    W'[c][d][v] = W[d][c][v^-1]. It runs as eqlinear_group_dft of dY, then
    eqlinear_backward_input_tiled on SM-pair tensor cores. The adjoint weight
    stages are the forward Fourier planes transposed, with the 2 x 2 block's
    off-diagonal entries exchanged.
  * dW[d,c,u] = sum_{n,g} dY[n,d,g] X[n,c,g u] and dbias run on CUDA cores
    (eqlinear_backward_weight, FP32 partials per row split, fixed-order sum).
Checked against the float64 oracle's gradients (themselves pinned to autograd of
the dense matrix built from the 2 x 2 matrix group), FP16 bar 2e-3 of max|ref|:
  * at shapes with ragged rows and partial channel tiles;
  * at the ViT-B fc1 shape of the D4 MLP (12608 x 96 -> 384). dX is checked on
    sampled rows. dW is checked on every output from inputs that are zero except
    a row set holding one row of every 16-row stage and the last rows (the
    gradient is a sum over rows).
"""
import numpy as np
import pytest
import torch

import oracle
from group_circulant_gemm_b200.synth import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu

TOL16 = 2e-3


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _plan(C, D):
    from group_circulant_gemm_b200 import EqLinearPlan
    return EqLinearPlan(8, C, D, torch.float16, group="dihedral4")


CASES = [
    # N, C, D
    (300, 16, 16),
    (129, 48, 80),
    (1000, 64, 128),
    (1, 16, 32),
    (700, 96, 208),
]


@pytest.mark.parametrize("N,C,D", CASES)
def test_d4_gradients_match_the_oracle(N, C, D):
    inp = make_inputs(Workload("d4b", 8, N, C, D, "f16", True, 9100 + N + C), need_dy=True)
    p = _plan(C, D)
    assert p.backward_weight_kernel_name(N) == "simt"
    Wh = p.prepare_weights(_dev(inp["W"]))
    dX = p.backward_input_tiled(p.group_dft(_dev(inp["dY"])), N, Wh)
    dW, db = p.backward_weight(_dev(inp["X"]), _dev(inp["dY"]))
    buf = p.backward_weight_f32(_dev(inp["X"]), _dev(inp["dY"]))
    assert p.status() == 0
    assert _rel(dX.double().cpu().numpy(), oracle.d4_backward_input(inp["dY"], inp["W"])) <= TOL16
    ref_dW, ref_db = oracle.d4_backward_weight(inp["X"], inp["dY"], D)
    assert _rel(dW.double().cpu().numpy(), ref_dW) <= TOL16
    assert _rel(db.double().cpu().numpy(), ref_db) <= TOL16
    w32, b32 = p.split_grad(buf)
    assert _rel(w32.double().cpu().numpy(), ref_dW) <= 1e-5
    assert _rel(b32.double().cpu().numpy(), ref_db) <= 1e-5


def test_d4_gradients_full_size():
    w = WORKLOADS["p4m_vitb_fc1_f16"]
    N, C, D = w.N, w.C, w.D
    inp = make_inputs(w, need_dy=True)
    p = _plan(C, D)
    Wh = p.prepare_weights(_dev(inp["W"]))
    dX = p.backward_input_tiled(p.group_dft(_dev(inp["dY"])), N, Wh).double().cpu().numpy()
    rng = np.random.default_rng(91)
    rows = np.unique(np.concatenate([rng.choice(N, 40, replace=False), np.arange(N - 8, N),
                                     np.arange(8), np.arange(252, 260)]))
    assert _rel(dX[rows], oracle.d4_backward_input(inp["dY"][rows], inp["W"])) <= TOL16
    k = np.arange(N // 16)
    S = np.unique(np.concatenate([16 * k + (5 * k) % 16, np.arange(N - 24, N)]))
    X = np.zeros_like(inp["X"])
    dY = np.zeros_like(inp["dY"])
    X[S], dY[S] = inp["X"][S], inp["dY"][S]
    dW, db = p.backward_weight(_dev(X), _dev(dY))
    assert p.status() == 0
    ref_dW, ref_db = oracle.d4_backward_weight(inp["X"][S], inp["dY"][S], D)
    assert _rel(dW.double().cpu().numpy(), ref_dW) <= TOL16
    assert _rel(db.double().cpu().numpy(), ref_db) <= TOL16
