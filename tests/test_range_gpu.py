"""FP16 range of the frequency-domain operands (GPU required).

A group DFT coefficient can reach T times the largest input magnitude (a
constant group vector puts all of it into frequency 0), so an FP16 plane that
held the plain DFT would overflow to inf for legal FP16 inputs above 65504 / T
(about 16 K at T = 4, 8 K at T = 8) while the layer's true outputs stay
finite.  The library stores every plane times 1/Tp (Tp = T for T = 4, 8; the
next power of two otherwise), which is exact and bounds each stored value by
the largest input.  These cases feed group vectors of magnitude up to 6e4,
planted in the patterns that maximise one frequency ("Specialisation for p4":
the transforms' coefficients 0, +-1; the constant and alternating groups reach
T times the amplitude), through every path that stores or forms planes:
forward, dX and dW on tensor cores, the spectral intermediate, the two-layer
chain, saved spectra, T = 8, D4, the convolution, and the CUDA-core path's
prepared weights.  Each output is compared with the float64 oracle on the same
FP16 inputs, with the FP16 bar max|err| / max|ref| <= 2e-3; each case also
checks that its reference is finite in FP16 (the test is about the operands'
range, not about outputs that cannot be represented).
"""
import numpy as np
import pytest
import torch

import oracle
from group_circulant_gemm_b200.synth import make_range_inputs

pytestmark = pytest.mark.gpu

TOL = 2e-3
AMP = 6.0e4  # largest planted magnitude (FP16 max is 65504)


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _plan(T, C, D, kernel="auto", group="cyclic"):
    from group_circulant_gemm_b200 import EqLinearPlan
    return EqLinearPlan(T, C, D, torch.float16, kernel=kernel, group=group)


def _check(got, ref):
    assert np.max(np.abs(ref)) < 65504.0, "case design: reference outside the FP16 range"
    got = got.double().cpu().numpy() if torch.is_tensor(got) else got
    assert np.all(np.isfinite(got))
    assert _rel(got, ref) <= TOL


def _planes_ref(rows, channels):
    """float64 p4 planes [4, N, channels] of rows [N, channels * 4], times 1/4 (the
    library's stored scale)."""
    F, _ = oracle.p4_transform_matrices()
    x = rows.astype(np.float64).reshape(rows.shape[0], channels, 4)
    return 0.25 * np.einsum("pt,nct->pnc", F, x)


def _planted_max(a, T):
    """Largest |sum over a group| of an array whose last axis holds c*T+t groups."""
    g = a.astype(np.float64).reshape(a.shape[0], -1, T)
    return float(np.max(np.abs(g.sum(axis=-1))))


@pytest.mark.parametrize("kernel", ["tcgen05", "simt"])
def test_forward_large_inputs_p4(kernel):
    inp = make_range_inputs(2001, 4, 333, 64, 128, x=(AMP, AMP), w=(0.2, 0.0))
    assert _planted_max(inp["X"], 4) > 65504.0  # the plain DFT would overflow
    p = _plan(4, 64, 128, kernel)
    Wh = p.prepare_weights(_dev(inp["W"]))
    Y = p.forward(_dev(inp["X"]), Wh, _dev(inp["bias"]))
    assert p.status() == 0
    _check(Y, oracle.forward(4, inp["X"], inp["W"], inp["bias"]))


@pytest.mark.parametrize("kernel", ["tcgen05", "simt"])
def test_forward_and_dx_large_weights_p4(kernel):
    inp = make_range_inputs(2002, 4, 200, 64, 128, x=(1e-3, 0.0), w=(0.0, AMP),
                            dy=(1e-3, 0.0), need_dy=True)
    assert float(np.max(np.abs(inp["W"].astype(np.float64).sum(axis=-1)))) > 65504.0
    p = _plan(4, 64, 128, kernel)
    Wh = p.prepare_weights(_dev(inp["W"]))
    assert torch.isfinite(Wh.float()).all()  # every stored plane is finite
    Y = p.forward(_dev(inp["X"]), Wh, _dev(inp["bias"]))
    dX = p.backward_input(_dev(inp["dY"]), Wh)
    assert p.status() == 0
    _check(Y, oracle.forward(4, inp["X"], inp["W"], inp["bias"]))
    _check(dX, oracle.backward_input(4, inp["dY"], inp["W"]))


@pytest.mark.parametrize("kernel", ["tcgen05", "simt"])
def test_dx_large_upstream_gradient_p4(kernel):
    inp = make_range_inputs(2003, 4, 333, 128, 64, w=(0.2, 0.0), dy=(AMP, AMP), need_dy=True)
    assert _planted_max(inp["dY"], 4) > 65504.0
    p = _plan(4, 128, 64, kernel)
    Wh = p.prepare_weights(_dev(inp["W"]))
    dX = p.backward_input(_dev(inp["dY"]), Wh)
    assert p.status() == 0
    _check(dX, oracle.backward_input(4, inp["dY"], inp["W"]))


def test_dw_large_inputs_p4_tensor_cores():
    # large X with a small upstream gradient, then a large upstream gradient with
    # small X (dbias then exceeds FP16 by construction and is not requested)
    p = _plan(4, 64, 128, "tcgen05")
    assert p.backward_weight_kernel_name(333) == "tcgen05"
    a = make_range_inputs(2004, 4, 333, 64, 128, x=(AMP, AMP), dy=(1e-3, 0.0), need_dy=True)
    dW, db = p.backward_weight(_dev(a["X"]), _dev(a["dY"]))
    assert p.status() == 0
    ref_w, ref_b = oracle.backward_weight(4, a["X"], a["dY"], 128)
    _check(dW, ref_w)
    _check(db, ref_b)
    b = make_range_inputs(2005, 4, 333, 64, 128, x=(1e-3, 0.0), dy=(AMP, AMP), need_dy=True)
    assert _planted_max(b["dY"], 4) > 65504.0
    dW, db = p.backward_weight(_dev(b["X"]), _dev(b["dY"]), want_bias=False)
    assert db is None and p.status() == 0
    _check(dW, oracle.backward_weight(4, b["X"], b["dY"], 128)[0])


def _identity_weights(C, scale):
    """W[d][c][u] = scale if d == c and u == 0: Y = scale * X (+ bias), so a large
    input passes through to a large intermediate."""
    W = np.zeros((C, C, 4), dtype=np.float16)
    W[np.arange(C), np.arange(C), 0] = scale
    return W


@pytest.mark.parametrize("act", ["none", "gelu"])
def test_spectral_intermediate_and_chain_large_activations(act):
    from group_circulant_gemm_b200.layer import forward_chain
    N, C1, C2 = 333, 64, 128
    a = make_range_inputs(2006, 4, N, C1, C1, x=(AMP, AMP))
    W1 = _identity_weights(C1, 0.875)
    b1 = a["bias"]
    l2 = make_range_inputs(2007, 4, 1, C1, C2, w=(0.2, 0.0))
    W2, b2 = l2["W"], l2["bias"]
    Y1 = oracle.forward(4, a["X"], W1, b1, act=act)
    assert _planted_max(Y1, 4) > 65504.0 and np.max(np.abs(Y1)) < 65504.0
    p1, p2 = _plan(4, C1, C1, "tcgen05"), _plan(4, C1, C2, "tcgen05")
    Wh1, Wh2 = p1.prepare_weights(_dev(W1)), p2.prepare_weights(_dev(W2))
    Xh = p1.forward_to_spectral(_dev(a["X"]), Wh1, _dev(b1), act=act)
    assert p1.status() == 0
    _check(Xh, _planes_ref(Y1, C1))
    Y = p2.forward_from_spectral(Xh, Wh2, _dev(b2))
    assert p2.status() == 0
    _check(Y, oracle.forward(4, Y1, W2, b2))
    for spectral in (False, True):
        H, Yc = forward_chain(p1, p2, _dev(a["X"]), Wh1, _dev(b1), Wh2, _dev(b2), act=act,
                              spectral=spectral)
        assert p1.status() == 0 and p2.status() == 0
        if not spectral:
            # the spatial intermediate is the FP16 first-layer output; the second
            # layer's in-kernel transform of it reaches 4 x 5e4
            _check(H, Y1)
            ref = oracle.forward(4, H.double().cpu().numpy(), W2, b2)
        else:
            ref = oracle.forward(4, Y1, W2, b2)
        _check(Yc, ref)


def test_saved_spectra_large_inputs():
    N, C, D = 333, 64, 128
    p = _plan(4, C, D, "tcgen05")
    a = make_range_inputs(2008, 4, N, C, D, x=(AMP, AMP), w=(0.2, 0.0), dy=(1e-3, 0.0),
                          need_dy=True)
    Wh = p.prepare_weights(_dev(a["W"]))
    Y, Xhat = p.forward_save_spectrum(_dev(a["X"]), Wh, _dev(a["bias"]))
    dX, dYhat = p.backward_input_save_spectrum(_dev(a["dY"]), Wh)
    dW, db = p.backward_weight_from_spectra(Xhat, dYhat)
    assert p.status() == 0
    _check(Y, oracle.forward(4, a["X"], a["W"], a["bias"]))
    _check(Xhat, _planes_ref(a["X"], C))
    ref_w, ref_b = oracle.backward_weight(4, a["X"], a["dY"], D)
    _check(dW, ref_w)
    _check(db, ref_b)
    # large upstream gradient: its saved spectrum, dX, and dW against small X
    b = make_range_inputs(2009, 4, N, C, D, x=(1e-3, 0.0), w=(0.2, 0.0), dy=(AMP, AMP),
                          need_dy=True)
    Wh = p.prepare_weights(_dev(b["W"]))
    _, Xhat = p.forward_save_spectrum(_dev(b["X"]), Wh, _dev(b["bias"]))
    dX, dYhat = p.backward_input_save_spectrum(_dev(b["dY"]), Wh)
    dW, _ = p.backward_weight_from_spectra(Xhat, dYhat, want_bias=False)
    assert p.status() == 0
    _check(dYhat, _planes_ref(b["dY"], D))
    _check(dX, oracle.backward_input(4, b["dY"], b["W"]))
    _check(dW, oracle.backward_weight(4, b["X"], b["dY"], D)[0])


def test_t8_large_inputs():
    T, N, C, D = 8, 389, 128, 64
    p = _plan(T, C, D, "tcgen05")
    assert p.forward_kernel_name(N) == "tcgen05"
    a = make_range_inputs(2010, T, N, C, D, x=(AMP, AMP), w=(0.2, 0.0), dy=(AMP, AMP),
                          need_dy=True)
    assert _planted_max(a["X"], T) > 65504.0
    Wh = p.prepare_weights(_dev(a["W"]))
    Y = p.forward(_dev(a["X"]), Wh, _dev(a["bias"]))
    dX = p.backward_input(_dev(a["dY"]), Wh)
    assert p.status() == 0
    _check(Y, oracle.forward(T, a["X"], a["W"], a["bias"]))
    _check(dX, oracle.backward_input(T, a["dY"], a["W"]))
    # large weights
    w = make_range_inputs(2011, T, N, C, D, x=(1e-3, 0.0), w=(0.0, AMP))
    Wh = p.prepare_weights(_dev(w["W"]))
    Y = p.forward(_dev(w["X"]), Wh, _dev(w["bias"]))
    assert p.status() == 0
    _check(Y, oracle.forward(T, w["X"], w["W"], w["bias"]))


def test_d4_large_inputs():
    N, C, D = 300, 32, 48
    p = _plan(8, C, D, "auto", group="dihedral4")
    a = make_range_inputs(2012, 8, N, C, D, x=(AMP, AMP), w=(0.2, 0.0))
    Wh = p.prepare_weights(_dev(a["W"]))
    Y = p.forward(_dev(a["X"]), Wh, _dev(a["bias"]))
    assert p.status() == 0
    _check(Y, oracle.d4_forward(a["X"], a["W"], a["bias"]))


def test_cuda_core_general_t_large_weights():
    # T = 3 runs on CUDA cores; its prepared FP16 planes held 3 max|W| before scaling
    T, N, C, D = 3, 97, 16, 24
    p = _plan(T, C, D, "auto")
    a = make_range_inputs(2013, T, N, C, D, x=(1e-3, 0.0), w=(0.0, AMP), dy=(1e-3, 0.0),
                          need_dy=True)
    Wh = p.prepare_weights(_dev(a["W"]))
    assert torch.isfinite(Wh.float()).all()
    Y = p.forward(_dev(a["X"]), Wh, _dev(a["bias"]))
    dX = p.backward_input(_dev(a["dY"]), Wh)
    assert p.status() == 0
    _check(Y, oracle.forward(T, a["X"], a["W"], a["bias"]))
    _check(dX, oracle.backward_input(T, a["dY"], a["W"]))


def test_convolution_large_inputs():
    T, Nimg, H, W, C, D = 4, 2, 9, 11, 16, 32
    r = make_range_inputs(2014, T, Nimg * H * W, C, 9 * D, x=(AMP, AMP), w=(0.1, 0.0))
    X = r["X"].reshape(Nimg, H, W, C * T)
    Wc = r["W"].reshape(3, 3, D, C, T)
    bias = r["bias"][:D].copy()
    p = _plan(T, C, D, "tcgen05")
    Wch = p.conv_prepare_weights(_dev(Wc))
    Y = p.conv_forward(_dev(X), Wch, 3, 3, _dev(bias), pad=(1, 1))
    assert p.status() == 0
    _check(Y, oracle.conv_forward(T, X, Wc, bias, pad=(1, 1)))
