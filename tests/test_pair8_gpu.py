"""Eight-plane layers in the frequency domain on SM pairs (GPU required).

The cyclic T = 8 layer and the layer over the dihedral group D4. In both,
eqlinear_group_dft forms the group Fourier transform of the input as eight FP16
planes (each times 1/8) in the tiled layout. eqlinear_forward_tiled (and, for
the cyclic group, eqlinear_backward_input_tiled) then takes the per-frequency
products on two SMs per 256-row tile and applies the inverse transform + bias
in the epilogue ("Algorithmic approach" items 1-3; the D4 form as read in
"Limitations and future work").

Checks against the float64 oracle on the same FP16 inputs (FP16 bar 2e-3 of
max|ref|):
  * the cyclic planes equal numpy's DFT of the rows times 1/8, within one FP16
    rounding; the padding rows are zero;
  * Y and dX at shapes spanning several tiles, ragged rows and out-channel
    counts that leave a partial 64-channel tile, with and without GELU;
  * the T = 8 workload (16384 x 128 -> 128) and the D4 ViT-B MLP layers at full
    size, on sampled rows;
  * agreement with the fused one-CTA kernels;
  * requests the path does not take are rejected (D4 dX in this form is checked
    in test_d4_backward_gpu.py).
"""
import numpy as np
import pytest
import torch

import oracle
from group_circulant_gemm_b200 import native
from group_circulant_gemm_b200.synth import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu

TOL16 = 2e-3


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _plan(C, D, group="cyclic"):
    from group_circulant_gemm_b200 import EqLinearPlan
    return EqLinearPlan(8, C, D, torch.float16, group=group)


def _untile8(t, N, c):
    """Tiled planes (8, c/16, Np, 16) -> float64 [8, N, c] and the padding rows."""
    a = t.double().cpu().numpy().reshape(8, c // 16, -1, 2, 8)
    Np = a.shape[2]
    sw = (np.arange(Np) >> 2) & 1
    idx = np.stack([sw, 1 - sw], axis=1)
    a = np.take_along_axis(a, idx[None, None, :, :, None], axis=3)
    a = a.reshape(8, c // 16, Np, 16).transpose(0, 2, 1, 3).reshape(8, Np, c)
    return a[:, :N, :], a[:, N:, :]


def _cyclic_planes_ref(rows, c):
    """V0, V4, Re/Im V1, V2, V3 of the DFT over the group axis, times 1/8."""
    V = np.fft.fft(rows.astype(np.float64).reshape(rows.shape[0], c, 8), axis=2) / 8
    order = [V[..., 0].real, V[..., 4].real, V[..., 1].real, V[..., 1].imag,
             V[..., 2].real, V[..., 2].imag, V[..., 3].real, V[..., 3].imag]
    return np.stack(order)


CASES = [
    # N, C, D, act
    (333, 32, 64, "none"),
    (257, 48, 80, "gelu"),     # a 64-channel tile and a 16-channel one
    (1, 16, 16, "none"),
    (1000, 128, 128, "none"),
    (700, 96, 208, "none"),
]


@pytest.mark.parametrize("N,C,D,act", CASES)
def test_cyclic_t8_tiled_matches_the_oracle(N, C, D, act):
    w = Workload("e8", 8, N, C, D, "f16", True, 8100 + N + C)
    inp = make_inputs(w, need_dy=True)
    p = _plan(C, D)
    Wh = p.prepare_weights(_dev(inp["W"]))
    Xt = p.group_dft(_dev(inp["X"]))
    assert tuple(Xt.shape) == p.tiled_shape(N, C)
    got, pad = _untile8(Xt, N, C)
    ref_planes = _cyclic_planes_ref(inp["X"], C)
    scale = np.abs(inp["X"].astype(np.float64)).reshape(N, C, 8).sum(axis=2)[None] / 8
    assert np.all(np.abs(got - ref_planes) <= np.abs(ref_planes) * 2.0 ** -10 + scale * 2.0 ** -20)
    assert np.all(pad == 0.0)
    Y = p.forward_tiled(Xt, N, Wh, _dev(inp["bias"]), act=act)
    dX = p.backward_input_tiled(p.group_dft(_dev(inp["dY"])), N, Wh)
    assert p.status() == 0
    ref = oracle.forward(8, inp["X"], inp["W"], inp["bias"], act=act)
    assert _rel(Y.double().cpu().numpy(), ref) <= TOL16
    assert _rel(dX.double().cpu().numpy(), oracle.backward_input(8, inp["dY"], inp["W"])) <= TOL16


@pytest.mark.parametrize("N,C,D,act", CASES)
def test_d4_tiled_matches_the_oracle(N, C, D, act):
    w = Workload("e4", 8, N, C, D, "f16", True, 8200 + N + C)
    inp = make_inputs(w)
    p = _plan(C, D, "dihedral4")
    Wh = p.prepare_weights(_dev(inp["W"]))
    Y = p.forward_tiled(p.group_dft(_dev(inp["X"])), N, Wh, _dev(inp["bias"]), act=act)
    assert p.status() == 0
    ref = oracle.d4_forward(inp["X"], inp["W"], inp["bias"], act=act)
    assert _rel(Y.double().cpu().numpy(), ref) <= TOL16


def _sampled(N, seed):
    rng = np.random.default_rng(seed)
    return np.unique(np.concatenate([rng.choice(N, 48, replace=False), np.arange(N - 8, N),
                                     np.arange(8), np.arange(252, 260)]))


def test_t8_workload_full_size_sampled_rows():
    w = WORKLOADS["c8_1024_f16"]
    inp = make_inputs(w)
    p = _plan(w.C, w.D)
    Wh = p.prepare_weights(_dev(inp["W"]))
    Y = p.forward_tiled(p.group_dft(_dev(inp["X"])), w.N, Wh, _dev(inp["bias"]))
    assert p.status() == 0
    rows = _sampled(w.N, 81)
    ref = oracle.forward(8, inp["X"][rows], inp["W"], inp["bias"])
    assert _rel(Y.double().cpu().numpy()[rows], ref) <= TOL16
    # the fused one-CTA kernel computes the same layer
    Y2 = p.forward(_dev(inp["X"]), Wh, _dev(inp["bias"])).double().cpu().numpy()
    assert _rel(Y.double().cpu().numpy(), Y2) <= TOL16


@pytest.mark.parametrize("layer", ["p4m_vitb_fc1_f16", "p4m_vitb_fc2_f16"])
def test_d4_vitb_layers_full_size_sampled_rows(layer):
    w = WORKLOADS[layer]
    inp = make_inputs(w)
    p = _plan(w.C, w.D, "dihedral4")
    Wh = p.prepare_weights(_dev(inp["W"]))
    Y = p.forward_tiled(p.group_dft(_dev(inp["X"])), w.N, Wh, _dev(inp["bias"]))
    assert p.status() == 0
    rows = _sampled(w.N, 82)
    ref = oracle.d4_forward(inp["X"][rows], inp["W"], inp["bias"])
    assert _rel(Y.double().cpu().numpy()[rows], ref) <= TOL16


def test_eight_plane_tiled_rejects_what_it_does_not_take():
    n = native
    p = _plan(16, 16, "dihedral4")
    Wh = p.prepare_weights(torch.zeros(16, 16, 8, dtype=torch.float16, device="cuda"))
    Xt = torch.zeros(p.tiled_shape(4, 16), dtype=torch.float16, device="cuda")
    X = torch.zeros(4, 128, dtype=torch.float16, device="cuda")
    assert n.eqlinear_tiled_spectrum_bytes(p.handle, 4, 16) == 8 * 128 * 16 * 2
    # no next-layer planes for D4 either
    assert n.raw_status("eqlinear_forward_tiled_next", p.handle, Xt.data_ptr(), 4,
                        Wh.data_ptr(), None, 0, Xt.data_ptr(), None) == n.EQL_ERR_UNSUPPORTED
    # channels that are not the plan's C or D
    assert n.raw_status("eqlinear_group_dft", p.handle, X.data_ptr(), 4, 32, Xt.data_ptr(),
                        None) == n.EQL_ERR_INVALID_ARG
    # the next layer's planes: p4 only
    c = _plan(16, 16)
    Wc = c.prepare_weights(torch.zeros(16, 16, 8, dtype=torch.float16, device="cuda"))
    assert n.raw_status("eqlinear_forward_tiled_next", c.handle, Xt.data_ptr(), 4,
                        Wc.data_ptr(), None, 0, Xt.data_ptr(), None) == n.EQL_ERR_UNSUPPORTED
