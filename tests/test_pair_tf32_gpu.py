"""The FP32 p4 layer on the tensor cores with 3xTF32 split precision (GPU required).

For FP32 plans, eqlinear_group_dft writes the group DFT of the input (planes X0,
X2, Xr, Xi times 1/4, "Algorithmic approach" items 1-2) as TF32 hi parts and
residual lo parts. eqlinear_forward_tiled and eqlinear_backward_input_tiled form
each per-frequency product as hi*hi + lo*hi + hi*lo on TF32 tensor cores with
FP32 accumulation, then apply the inverse DFT in FP32 (item 3).

The FP32 bar is max|err| / max|ref| <= 1e-5 against the float64 oracle.

Checks:
  * hi holds TF32 values (low 13 mantissa bits zero), and hi + lo is the
    oracle's transform within FP32 rounding; the padding rows are zero;
  * Y and dX against the oracle, at the two FP32 configurations (256 x 16 -> 16
    and the full ViT-B projection, 12608 x 192 -> 192) and at ragged shapes;
  * agreement with the FP32 CUDA-core kernel;
  * requests the path does not take are rejected.
"""
import numpy as np
import pytest
import torch

import oracle
from group_circulant_gemm_b200 import native
from group_circulant_gemm_b200.synth import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu

TOL32 = 1e-5


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _plan(C, D, kernel="auto"):
    from group_circulant_gemm_b200 import EqLinearPlan
    return EqLinearPlan(4, C, D, torch.float32, kernel=kernel)


def _untile32(t, N, c):
    """Tiled FP32 planes (8, c/8, Np, 8) -> float64 [8, N, c] and the padding rows.
    Row n's 16-byte halves are swapped when (n / 4) % 2."""
    a = t.double().cpu().numpy().reshape(8, c // 8, -1, 2, 4)
    Np = a.shape[2]
    sw = (np.arange(Np) >> 2) & 1
    idx = np.stack([sw, 1 - sw], axis=1)
    a = np.take_along_axis(a, idx[None, None, :, :, None], axis=3)
    a = a.reshape(8, c // 8, Np, 8).transpose(0, 2, 1, 3).reshape(8, Np, c)
    return a[:, :N, :], a[:, N:, :]


def _planes_ref(rows, channels):
    F, _ = oracle.p4_transform_matrices()
    x = rows.astype(np.float64).reshape(rows.shape[0], channels, 4)
    return 0.25 * np.einsum("pt,nct->pnc", F, x)


CASES = [
    # N, C, D, act, bias
    (256, 16, 16, "none", True),       # the small FP32 configuration
    (333, 64, 128, "none", True),      # ragged rows: the second half of a pair tile past N
    (257, 48, 80, "gelu", True),       # a 64-channel tile and a 16-channel one
    (1, 8, 8, "none", False),
    (700, 192, 56, "none", True),
]


@pytest.mark.parametrize("N,C,D,act,bias", CASES)
def test_tf32_forward_and_dx_match_the_oracle(N, C, D, act, bias):
    w = Workload("t3", 4, N, C, D, "f32", True, 7100 + N + C)
    inp = make_inputs(w, need_dy=True)
    p = _plan(C, D)
    Wh = p.prepare_weights(_dev(inp["W"]))
    b = _dev(inp["bias"]) if bias else None
    Xt = p.group_dft(_dev(inp["X"]))
    assert tuple(Xt.shape) == p.tiled_shape(N, C)
    got, pad = _untile32(Xt, N, C)
    hi, lo = got[:4], got[4:]
    hi_bits = Xt.view(torch.int32).cpu().numpy().reshape(8, -1)[:4]
    assert np.all((hi_bits & 0x1FFF) == 0)                    # TF32 values
    ref_planes = _planes_ref(inp["X"], C)
    # FP32 sums of four terms, then the TF32 rounding of lo: a few 2^-24 of the
    # terms' magnitude (the plane coefficients are all +-1/4)
    scale = 0.25 * np.abs(inp["X"].astype(np.float64)).reshape(N, C, 4).sum(axis=2)[None]
    assert np.all(np.abs(hi + lo - ref_planes) <= scale * 2.0 ** -21)
    assert np.all(pad == 0.0)
    Y = p.forward_tiled(Xt, N, Wh, b, act=act)
    dYt = p.group_dft(_dev(inp["dY"]))
    dX = p.backward_input_tiled(dYt, N, Wh)
    assert p.status() == 0
    ref = oracle.forward(4, inp["X"], inp["W"], inp["bias"] if bias else None, act=act)
    assert _rel(Y.double().cpu().numpy(), ref) <= TOL32
    assert _rel(dX.double().cpu().numpy(), oracle.backward_input(4, inp["dY"], inp["W"])) <= TOL32


def test_tf32_full_vitb_projection_matches_the_oracle():
    """The FP32 ViT-B projection (N = 12608, C = D = 192), every output."""
    w = WORKLOADS["p4_vitb_proj_f32"]
    inp = make_inputs(w)
    p = _plan(w.C, w.D)
    Wh = p.prepare_weights(_dev(inp["W"]))
    Y = p.forward_tiled(p.group_dft(_dev(inp["X"])), w.N, Wh, _dev(inp["bias"]))
    assert p.status() == 0
    ref = oracle.forward(4, inp["X"], inp["W"], inp["bias"])
    assert _rel(Y.double().cpu().numpy(), ref) <= TOL32


def test_tf32_agrees_with_the_cuda_core_kernel():
    w = Workload("t3s", 4, 1500, 192, 192, "f32", True, 7300)
    inp = make_inputs(w)
    p = _plan(192, 192)
    Wh = p.prepare_weights(_dev(inp["W"]))
    X, b = _dev(inp["X"]), _dev(inp["bias"])
    y_simt = p.forward(X, Wh, b).double().cpu().numpy()
    y_tc = p.forward_tiled(p.group_dft(X), 1500, Wh, b).double().cpu().numpy()
    assert _rel(y_tc, y_simt) <= TOL32


def test_tf32_tiled_rejects_what_it_does_not_take():
    n = native
    p = _plan(16, 16)
    Wh = p.prepare_weights(torch.zeros(16, 16, 4, device="cuda"))
    Xt = torch.zeros(p.tiled_shape(4, 16), device="cuda")
    assert n.eqlinear_tiled_spectrum_bytes(p.handle, 4, 16) == 8 * 128 * 16 * 4
    # the next layer's planes: an FP16 chain only
    assert n.raw_status("eqlinear_forward_tiled_next", p.handle, Xt.data_ptr(), 4, Wh.data_ptr(),
                        None, 0, Xt.data_ptr(), None) == n.EQL_ERR_UNSUPPORTED
    # channel counts that are not multiples of 8
    odd = _plan(12, 16)
    X = torch.zeros(4, 48, device="cuda")
    assert n.raw_status("eqlinear_group_dft", odd.handle, X.data_ptr(), 4, 12, Xt.data_ptr(),
                        None) == n.EQL_ERR_UNSUPPORTED
    # a plan forced to the CUDA cores has no tiled form
    p.set_kernel("simt")
    Y = torch.zeros(4, 64, device="cuda")
    assert n.raw_status("eqlinear_forward_tiled", p.handle, Xt.data_ptr(), 4, Wh.data_ptr(),
                        None, 0, Y.data_ptr(), None) == n.EQL_ERR_UNSUPPORTED
