"""Group-circulant convolution on the GPU (eqlinear_conv_forward) against the
float64 oracle (oracle.conv_forward), GPU required.

Inputs are the oracle's own seeded, FP16-cast arrays; the error metric is the
layer's, max|gpu - oracle| / max|oracle| <= 2e-3 for FP16.
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

TOL16 = 2e-3


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def _inputs(N, H, W, C, D, KH, KW, seed):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((N, H, W, C * 4)).astype(np.float16)
    Wc = (rng.standard_normal((KH, KW, D, C, 4)) / np.sqrt(C * 4 * KH * KW)).astype(np.float16)
    b = (rng.standard_normal(D) * 0.1).astype(np.float16)
    return X, Wc, b


def _plan(C, D):
    from group_circulant_gemm_b200 import EqLinearPlan
    return EqLinearPlan(4, C, D, torch.float16)


CASES = [
    # N, H, W, C, D, KH, KW, ph, pw, act
    (2, 10, 13, 16, 32, 3, 3, 1, 1, "none"),
    (1, 17, 33, 48, 16, 3, 3, 1, 1, "gelu"),
    (1, 9, 20, 64, 64, 5, 5, 2, 2, "none"),
    (2, 7, 7, 16, 16, 3, 3, 0, 0, "none"),
    (1, 6, 40, 32, 144, 3, 1, 1, 0, "none"),
    (1, 1, 1, 16, 16, 3, 3, 1, 1, "none"),
    (3, 8, 16, 80, 208, 2, 2, 1, 0, "gelu"),
]


@pytest.mark.parametrize("N,H,W,C,D,KH,KW,ph,pw,act", CASES)
def test_conv_matches_oracle(N, H, W, C, D, KH, KW, ph, pw, act):
    X, Wc, b = _inputs(N, H, W, C, D, KH, KW, 3000 + H * W + C)
    p = _plan(C, D)
    Wh = p.conv_prepare_weights(torch.from_numpy(Wc).cuda())
    Y = p.conv_forward(torch.from_numpy(X).cuda(), Wh, KH, KW, torch.from_numpy(b).cuda(),
                       pad=(ph, pw), act=act)
    assert p.status() == 0
    ref = oracle.conv_forward(4, X, Wc, b, pad=(ph, pw))
    if act == "gelu":
        ref = oracle.gelu(ref)
    assert tuple(Y.shape) == ref.shape
    assert _rel(Y.double().cpu().numpy(), ref) <= TOL16


def test_conv_1x1_is_the_layer_forward_bitwise():
    N, H, W, C, D = 2, 9, 21, 64, 128
    X, Wc, b = _inputs(N, H, W, C, D, 1, 1, 3100)
    p = _plan(C, D)
    Xd, bd = torch.from_numpy(X).cuda(), torch.from_numpy(b).cuda()
    Yc = p.conv_forward(Xd, p.conv_prepare_weights(torch.from_numpy(Wc).cuda()), 1, 1, bd)
    Yl = p.forward(Xd.view(N * H * W, C * 4), p.prepare_weights(torch.from_numpy(Wc[0, 0]).cuda()),
                   bd)
    assert p.status() == 0
    assert torch.equal(Yc.view(-1).view(torch.int16), Yl.view(-1).view(torch.int16))


def test_conv_full_size_images_against_oracle():
    """The bench's shape (56 x 56 images, 64 -> 64 channels, 3 x 3): two whole images
    of a 16-image batch against the oracle."""
    N, H, W, C, D = 16, 56, 56, 64, 64
    X, Wc, b = _inputs(N, H, W, C, D, 3, 3, 3200)
    p = _plan(C, D)
    Wh = p.conv_prepare_weights(torch.from_numpy(Wc).cuda())
    Y = p.conv_forward(torch.from_numpy(X).cuda(), Wh, 3, 3, torch.from_numpy(b).cuda(),
                       pad=(1, 1)).double().cpu().numpy()
    assert p.status() == 0
    for n in (0, N - 1):
        ref = oracle.conv_forward(4, X[n:n + 1], Wc, b, pad=(1, 1))
        assert _rel(Y[n:n + 1], ref) <= TOL16


def test_conv_group_shift_equivariance_on_gpu():
    N, H, W, C, D = 1, 12, 18, 32, 48
    X, Wc, b = _inputs(N, H, W, C, D, 3, 3, 3300)
    p = _plan(C, D)
    Wh = p.conv_prepare_weights(torch.from_numpy(Wc).cuda())
    bd = torch.from_numpy(b).cuda()
    Y = p.conv_forward(torch.from_numpy(X).cuda(), Wh, 3, 3, bd, pad=(1, 1))
    Xr = np.roll(X.reshape(N, H, W, C, 4), 1, axis=4).reshape(N, H, W, C * 4)
    Yr = p.conv_forward(torch.from_numpy(np.ascontiguousarray(Xr)).cuda(), Wh, 3, 3, bd,
                        pad=(1, 1))
    y = Y.double().cpu().numpy().reshape(N, H, W, D, 4)
    yr = Yr.double().cpu().numpy().reshape(N, H, W, D, 4)
    assert _rel(yr, np.roll(y, 1, axis=4)) <= 1e-3


def test_conv_error_paths():
    from group_circulant_gemm_b200 import EqLinearPlan, native
    p = _plan(16, 16)
    p8 = EqLinearPlan(8, 16, 16, torch.float16)
    f32 = EqLinearPlan(4, 16, 16, torch.float32)
    assert native.eqlinear_conv_prepared_weight_bytes(p8.handle, 3, 3) == 0
    assert native.eqlinear_conv_prepared_weight_bytes(f32.handle, 3, 3) == 0
    assert native.eqlinear_conv_prepared_weight_bytes(p.handle, 0, 3) == 0
    X = torch.zeros(1, 4, 4, 64, dtype=torch.float16, device="cuda")
    Y = torch.zeros(1, 4, 4, 64, dtype=torch.float16, device="cuda")
    Wh = p.conv_prepare_weights(torch.zeros(3, 3, 16, 16, 4, dtype=torch.float16, device="cuda"))
    ws = torch.zeros(native.eqlinear_conv_workspace_bytes(p.handle, 1, 4, 4), dtype=torch.uint8,
                     device="cuda")

    def call(plan=p, H=4, W=4, KH=3, KW=3, ph=1, pw=1, act=0, nbytes=None, ws_=ws):
        nb = ws_.numel() if nbytes is None else nbytes
        return native.raw_status("eqlinear_conv_forward", plan.handle, X.data_ptr(), 1, H, W, KH,
                                 KW, ph, pw, Wh.data_ptr(), None, act, Y.data_ptr(),
                                 ws_.data_ptr(), nb, None)
    assert call() == native.EQL_OK
    assert call(plan=p8) == native.EQL_ERR_UNSUPPORTED
    assert call(plan=f32) == native.EQL_ERR_UNSUPPORTED
    assert call(act=5) == native.EQL_ERR_INVALID_ARG
    assert call(ph=-1) == native.EQL_ERR_INVALID_ARG
    assert call(KH=7, KW=7, ph=0, pw=0) == native.EQL_ERR_INVALID_ARG  # empty output
    assert call(ph=3) == native.EQL_ERR_UNSUPPORTED                    # padding >= kernel
    assert call(nbytes=8) == native.EQL_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert p.status() == 0
