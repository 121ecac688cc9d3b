"""Gradients of the group-circulant convolution on the GPU against the float64
oracle (oracle.conv_backward_input / conv_backward_weight), GPU required.

The convolution applies the layer ("Algorithmic approach": per frequency, a
product of the input's group spectrum with the weight's) at every tap of a
KH x KW window, so
  * dX is the same convolution run on dY with the kernel flipped in space and
    every tap replaced by its adjoint (the layer's dX weights), with padding
    (KH-1-ph, KW-1-pw): eqlinear_conv_backward_input runs the forward
    convolution kernel on those prepared tiles;
  * dWc[i, j] is the layer's weight gradient over the rows of X shifted by tap
    (i, j) and the rows of dY; dbias is the layer's, once. The library puts X
    and dY on the padded pixel grid once, so that each tap is a row offset.

FP16 bar: max|gpu - oracle| / max|oracle| <= 2e-3 (the layer's).
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

TOL16 = 2e-3


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def _inputs(N, H, W, C, D, KH, KW, ph, pw, seed):
    rng = np.random.default_rng(seed)
    Ho, Wo = H + 2 * ph - KH + 1, W + 2 * pw - KW + 1
    X = rng.standard_normal((N, H, W, C * 4)).astype(np.float16)
    Wc = (rng.standard_normal((KH, KW, D, C, 4)) / np.sqrt(C * 4 * KH * KW)).astype(np.float16)
    dY = (rng.standard_normal((N, Ho, Wo, D * 4)) * 0.1).astype(np.float16)
    return X, Wc, dY


def _plan(C, D):
    from group_circulant_gemm_b200 import EqLinearPlan
    return EqLinearPlan(4, C, D, torch.float16)


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


CASES = [
    # N, H, W, C, D, KH, KW, ph, pw
    (2, 10, 13, 16, 32, 3, 3, 1, 1),
    (1, 17, 33, 48, 16, 3, 3, 1, 1),
    (1, 9, 20, 64, 64, 5, 5, 2, 2),
    (2, 7, 7, 16, 16, 3, 3, 0, 0),      # no padding: dX pads by KH-1
    (1, 6, 40, 32, 144, 3, 1, 1, 0),
    (1, 1, 1, 16, 16, 3, 3, 1, 1),      # one pixel: only the centre tap sees data
    (3, 8, 16, 80, 208, 2, 2, 1, 0),    # even kernel, asymmetric padding
    (1, 6, 10, 192, 64, 3, 3, 1, 1),    # two 128-channel tiles per tap in dWc's single launch
    (2, 5, 7, 128, 192, 3, 2, 1, 0),    # two out-channel tiles, a 3 x 2 kernel
]


@pytest.mark.parametrize("N,H,W,C,D,KH,KW,ph,pw", CASES)
def test_conv_backward_matches_the_oracle(N, H, W, C, D, KH, KW, ph, pw):
    X, Wc, dY = _inputs(N, H, W, C, D, KH, KW, ph, pw, 5000 + H * W + C)
    p = _plan(C, D)
    Wh = p.conv_prepare_weights(_dev(Wc))
    dX = p.conv_backward_input(_dev(dY), Wh, KH, KW, H, W, pad=(ph, pw))
    dW, db = p.conv_backward_weight(_dev(X), _dev(dY), KH, KW, pad=(ph, pw))
    assert p.status() == 0
    ref_dX = oracle.conv_backward_input(4, dY, Wc, H, W, pad=(ph, pw))
    ref_dW, ref_db = oracle.conv_backward_weight(4, X, dY, KH, KW, pad=(ph, pw))
    assert tuple(dX.shape) == ref_dX.shape and tuple(dW.shape) == ref_dW.shape
    assert _rel(dX.double().cpu().numpy(), ref_dX) <= TOL16
    assert _rel(dW.double().cpu().numpy(), ref_dW) <= TOL16
    assert _rel(db.double().cpu().numpy(), ref_db) <= TOL16


def test_conv_backward_1x1_is_the_layer_backward():
    """A 1 x 1 kernel without padding is the layer on N*H*W rows. With C and D
    multiples of 64 the convolution's weight gradient multiplies the rows' group
    spectra, exactly as the layer's weight gradient from saved spectra does."""
    N, H, W, C, D = 2, 9, 21, 64, 128
    X, Wc, dY = _inputs(N, H, W, C, D, 1, 1, 0, 0, 5100)
    p = _plan(C, D)
    Xd, dYd = _dev(X), _dev(dY)
    dX = p.conv_backward_input(dYd, p.conv_prepare_weights(_dev(Wc)), 1, 1, H, W)
    dW, db = p.conv_backward_weight(Xd, dYd, 1, 1)
    Wh = p.prepare_weights(_dev(Wc[0, 0]))
    rows = N * H * W
    dX_l = p.backward_input(dYd.view(rows, D * 4), Wh)
    _, Xhat = p.forward_save_spectrum(Xd.view(rows, C * 4), Wh)
    _, dYhat = p.backward_input_save_spectrum(dYd.view(rows, D * 4), Wh)
    dW_l, db_l = p.backward_weight_from_spectra(Xhat, dYhat)
    assert p.status() == 0
    assert _rel(dX.double().cpu().numpy().reshape(rows, -1), dX_l.double().cpu().numpy()) <= 1e-3
    assert torch.equal(dW[0, 0].view(torch.int16), dW_l.view(torch.int16))
    assert torch.equal(db.view(torch.int16), db_l.view(torch.int16))


def test_conv_backward_full_size_batch():
    """The bench's shape (a batch of 16 56 x 56 images, 64 -> 64 channels, 3 x 3,
    padding 1). dX: two whole images against the oracle. dW: X and dY are zero
    except on images 0 and 15, so the full-size launch must give exactly the
    gradient of those two images, which the oracle computes for every output."""
    N, H, W, C, D = 16, 56, 56, 64, 64
    X, Wc, dY = _inputs(N, H, W, C, D, 3, 3, 1, 1, 5200)
    keep = [0, N - 1]
    Xs, dYs = np.zeros_like(X), np.zeros_like(dY)
    Xs[keep], dYs[keep] = X[keep], dY[keep]
    p = _plan(C, D)
    Wh = p.conv_prepare_weights(_dev(Wc))
    dX = p.conv_backward_input(_dev(dY), Wh, 3, 3, H, W, pad=(1, 1)).double().cpu().numpy()
    dW, db = p.conv_backward_weight(_dev(Xs), _dev(dYs), 3, 3, pad=(1, 1))
    assert p.status() == 0
    for n in keep:
        ref = oracle.conv_backward_input(4, dY[n:n + 1], Wc, H, W, pad=(1, 1))
        assert _rel(dX[n:n + 1], ref) <= TOL16
    ref_dW, ref_db = oracle.conv_backward_weight(4, X[keep], dY[keep], 3, 3, pad=(1, 1))
    assert _rel(dW.double().cpu().numpy(), ref_dW) <= TOL16
    assert _rel(db.double().cpu().numpy(), ref_db) <= TOL16


def test_conv_backward_error_paths():
    from group_circulant_gemm_b200 import EqLinearPlan, native
    p = _plan(16, 16)
    f32 = EqLinearPlan(4, 16, 16, torch.float32)
    assert native.eqlinear_conv_backward_workspace_bytes(f32.handle, 1, 4, 4, 3, 3, 1, 1) == 0
    assert native.eqlinear_conv_backward_workspace_bytes(p.handle, 1, 4, 4, 7, 7, 0, 0) == 0
    Wh = p.conv_prepare_weights(torch.zeros(3, 3, 16, 16, 4, dtype=torch.float16, device="cuda"))
    X = torch.zeros(1, 4, 4, 64, dtype=torch.float16, device="cuda")
    dY = torch.zeros(1, 4, 4, 64, dtype=torch.float16, device="cuda")
    dX = torch.zeros_like(X)
    dW = torch.zeros(3, 3, 16, 16, 4, dtype=torch.float16, device="cuda")
    nb = native.eqlinear_conv_backward_workspace_bytes(p.handle, 1, 4, 4, 3, 3, 1, 1)
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")

    def bin_(plan=p, ph=1, nbytes=nb):
        return native.raw_status("eqlinear_conv_backward_input", plan.handle, dY.data_ptr(), 1,
                                 4, 4, 3, 3, ph, 1, Wh.data_ptr(), dX.data_ptr(), ws.data_ptr(),
                                 nbytes, None)

    def bw_(plan=p, ph=1, nbytes=nb):
        return native.raw_status("eqlinear_conv_backward_weight", plan.handle, X.data_ptr(), 1,
                                 4, 4, dY.data_ptr(), 3, 3, ph, 1, dW.data_ptr(), None,
                                 ws.data_ptr(), nbytes, None)
    assert bin_() == native.EQL_OK and bw_() == native.EQL_OK
    assert bin_(plan=f32) == native.EQL_ERR_UNSUPPORTED
    assert bw_(plan=f32) == native.EQL_ERR_UNSUPPORTED
    assert bin_(ph=-1) == native.EQL_ERR_INVALID_ARG and bw_(ph=-1) == native.EQL_ERR_INVALID_ARG
    assert bin_(nbytes=8) == native.EQL_ERR_WORKSPACE
    assert bw_(nbytes=8) == native.EQL_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert p.status() == 0
