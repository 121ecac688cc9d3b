"""Weight gradient from tiled planes (eqlinear_backward_weight_tiled), GPU required.

"Implementation", bullet 1: the backward pass is the same per-frequency product,
transposed and summed over rows. eqlinear_group_dft writes the group DFT of X
and of dY once (planes X0, X2, Xr, Xi times 1/4, 32-byte swizzled rows). The
tensor-core weight gradient reads those planes as MN-major operands, with no
transform of its own. So one transform of X serves the forward and dW, and one
of dY serves dX and dW.

Checks against the float64 oracle (FP16 bar 2e-3 of max|ref|, FP32 output the
same operands so the same bar):
  * ragged rows and channel counts that are multiples of 16 but not of 64;
  * FP32 output (the data-parallel gradient buffer);
  * the full-size ViT-H fc1 training shape, every output, by the sparse-row
    construction of the row-set test: the planes are zero except on rows that
    walk through every 32-row stage and the last 40 rows;
  * plans the entry does not take are rejected.
"""
import numpy as np
import pytest
import torch

import oracle
from group_circulant_gemm_b200 import native
from group_circulant_gemm_b200.synth import Workload, make_inputs

pytestmark = pytest.mark.gpu

TOL16 = 2e-3


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _plan(C, D, dtype=torch.float16, group="cyclic"):
    from group_circulant_gemm_b200 import EqLinearPlan
    return EqLinearPlan(8 if group == "dihedral4" else 4, C, D, dtype, group=group)


CASES = [
    # N, C, D
    (333, 48, 80),      # ragged rows; a 128-channel tile that is mostly padding
    (1, 16, 16),
    (700, 192, 48),
    (129, 64, 128),
    (1000, 320, 1280),  # the ViT-H fc1 channels, two row blocks
]


@pytest.mark.parametrize("N,C,D", CASES)
def test_tiled_weight_gradient_matches_the_oracle(N, C, D):
    inp = make_inputs(Workload("wt", 4, N, C, D, "f16", True, 8100 + N + C), need_dy=True)
    p = _plan(C, D)
    X, dY = _dev(inp["X"]), _dev(inp["dY"])
    Xt, dYt = p.group_dft(X), p.group_dft(dY)
    dW, db = p.backward_weight_tiled(Xt, dYt, N)
    buf = p.backward_weight_tiled_f32(Xt, dYt, N)
    assert p.status() == 0
    ref_dW, ref_db = oracle.backward_weight(4, inp["X"], inp["dY"], D)
    assert _rel(dW.double().cpu().numpy(), ref_dW) <= TOL16
    assert _rel(db.double().cpu().numpy(), ref_db) <= TOL16
    dW32, db32 = p.split_grad(buf)
    assert _rel(dW32.double().cpu().numpy(), ref_dW) <= TOL16
    assert _rel(db32.double().cpu().numpy(), ref_db) <= TOL16
    # the FP16 result is the FP32 one rounded
    assert torch.equal(dW.view(torch.int16), dW32.half().view(torch.int16))


def test_tiled_weight_gradient_full_size_every_output():
    N, C, D = 8224, 320, 1280
    inp = make_inputs(Workload("wr", 4, N, C, D, "f16", True, 6100), need_dy=True)
    k = np.arange(N // 32)
    S = np.unique(np.concatenate([32 * k + (7 * k) % 32, np.arange(N - 40, N)]))
    X = np.zeros_like(inp["X"])
    dY = np.zeros_like(inp["dY"])
    X[S], dY[S] = inp["X"][S], inp["dY"][S]
    p = _plan(C, D)
    dW, db = p.backward_weight_tiled(p.group_dft(_dev(X)), p.group_dft(_dev(dY)), N)
    assert p.status() == 0
    ref_dW, ref_db = oracle.backward_weight(4, inp["X"][S], inp["dY"][S], D)
    assert _rel(dW.double().cpu().numpy(), ref_dW) <= TOL16
    assert _rel(db.double().cpu().numpy(), ref_db) <= TOL16


def test_tiled_weight_gradient_rejects_what_it_does_not_take():
    p = _plan(16, 16)
    Xt = torch.zeros(p.tiled_shape(4, 16), dtype=torch.float16, device="cuda")
    dW = torch.zeros(16, 16, 4, dtype=torch.float16, device="cuda")
    ws = torch.zeros(max(p.workspace_bytes(4), 16), dtype=torch.uint8, device="cuda")

    def call(plan):
        return native.raw_status("eqlinear_backward_weight_tiled", plan.handle, Xt.data_ptr(),
                                 Xt.data_ptr(), 4, dW.data_ptr(), None, ws.data_ptr(),
                                 ws.numel(), None)
    assert call(p) == native.EQL_OK
    assert call(_plan(16, 16, torch.float32)) == native.EQL_ERR_UNSUPPORTED
    assert call(_plan(16, 16, group="dihedral4")) == native.EQL_ERR_UNSUPPORTED
    simt = _plan(16, 16)
    simt.set_kernel("simt")
    assert call(simt) == native.EQL_ERR_UNSUPPORTED
    assert native.raw_status("eqlinear_backward_weight_tiled", p.handle, Xt.data_ptr(),
                             Xt.data_ptr(), 4, dW.data_ptr(), None, ws.data_ptr(), 8,
                             None) == native.EQL_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert p.status() == 0
