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
  * eqlinear_forward_tiled_next (the next layer's planes from the epilogue)
    equals eqlinear_group_dft of eqlinear_forward_tiled's output, padding rows
    zero: bitwise for D4 (its inverse transform is adds only); for the cyclic
    group the compiler may fuse the sqrt(2)/2 twiddle products of the inverse
    into the following adds differently in the two kernels, so a value of Y
    can differ by one FP16 rounding; and the D4 MLP pair chained that way
    matches the oracle;
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
    # a plan forced to the CUDA cores has no tiled form
    p.set_kernel("simt")
    assert n.raw_status("eqlinear_forward_tiled_next", p.handle, Xt.data_ptr(), 4,
                        Wh.data_ptr(), None, 0, Xt.data_ptr(), None) == n.EQL_ERR_UNSUPPORTED
    p.set_kernel("auto")
    # channels that are not the plan's C or D
    assert n.raw_status("eqlinear_group_dft", p.handle, X.data_ptr(), 4, 32, Xt.data_ptr(),
                        None) == n.EQL_ERR_INVALID_ARG
    # misaligned output planes
    bad = torch.zeros(8 * 128 * 16 + 8, dtype=torch.float16, device="cuda")[1:]
    assert n.raw_status("eqlinear_forward_tiled_next", p.handle, Xt.data_ptr(), 4,
                        Wh.data_ptr(), None, 0, bad.data_ptr(), None) == n.EQL_ERR_ALIGNMENT


NEXT_CASES = [
    # N, C, D, group, act
    (333, 32, 64, "dihedral4", "none"),
    (257, 48, 80, "cyclic", "gelu"),
    (1000, 96, 384, "dihedral4", "gelu"),
    (129, 16, 16, "cyclic", "none"),
]


@pytest.mark.parametrize("N,C,D,group,act", NEXT_CASES)
def test_next_layer_planes_are_the_group_dft_of_the_output(N, C, D, group, act):
    w = Workload("n8", 8, N, C, D, "f16", True, 8500 + N + C)
    inp = make_inputs(w)
    p = _plan(C, D, group)
    Wh = p.prepare_weights(_dev(inp["W"]))
    b = _dev(inp["bias"])
    Xt = p.group_dft(_dev(inp["X"]))
    Y = p.forward_tiled(Xt, N, Wh, b, act=act)
    nxt = _plan(D, 16, group)  # a plan whose input width is D
    ref = nxt.group_dft(Y)
    got = torch.full(p.tiled_shape(N, D), float("nan"), dtype=torch.float16, device="cuda")
    p.forward_tiled_next(Xt, N, Wh, b, act=act, out=got)
    assert p.status() == 0 and nxt.status() == 0
    if group == "dihedral4":
        assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
    else:
        g, r = got.double().cpu().numpy(), ref.double().cpu().numpy()
        assert np.all(np.isfinite(g))
        # one FP16 rounding of a Y value (2^-10 of |Y|) moves a plane (a signed
        # mean of the eight) by at most that much, plus the plane's own rounding
        assert np.max(np.abs(g - r)) <= 2.0 ** -9 * float(Y.abs().max())
        Np = g.shape[2]
        assert np.all(g[:, :, N:Np, :] == 0.0)


def test_d4_mlp_pair_through_next_layer_planes_matches_the_oracle():
    """The p4m ViT-B MLP pair (C = 96 -> 384 -> 96 per group element) with the
    intermediate kept as tiled planes, on sampled rows of the full N = 12608."""
    w1, w2 = WORKLOADS["p4m_vitb_fc1_f16"], WORKLOADS["p4m_vitb_fc2_f16"]
    inp1, inp2 = make_inputs(w1), make_inputs(w2)
    p1, p2 = _plan(w1.C, w1.D, "dihedral4"), _plan(w2.C, w2.D, "dihedral4")
    W1, W2 = p1.prepare_weights(_dev(inp1["W"])), p2.prepare_weights(_dev(inp2["W"]))
    b1, b2 = _dev(inp1["bias"]), _dev(inp2["bias"])
    Ht = p1.forward_tiled_next(p1.group_dft(_dev(inp1["X"])), w1.N, W1, b1)
    Y = p2.forward_tiled(Ht, w1.N, W2, b2)
    assert p1.status() == 0 and p2.status() == 0
    rows = _sampled(w1.N, 83)
    H = oracle.d4_forward(inp1["X"][rows], inp1["W"], inp1["bias"])
    ref = oracle.d4_forward(H.astype(np.float16), inp2["W"], inp2["bias"])
    assert _rel(Y.double().cpu().numpy()[rows], ref) <= TOL16
