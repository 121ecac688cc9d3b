"""Training with saved group spectra on the GPU, GPU required.

The forward and dX kernels can also store the group DFTs they form (of X and
of dY); the weight gradient then multiplies those planes directly.  Checks:
  * Y and dX are bitwise those of the plain calls;
  * the saved planes are the real 4-point DFT of the input rows times 1/4 (the oracle's
    p4 transform matrix, float64) up to the one FP16 rounding;
  * dW and dbias from the spectra match the float64 oracle (FP16 tolerance
    2e-3 of max|ref|) and the transforming weight-gradient kernel;
  * rows past N and channels past C are never written (guard sentinels).
"""
import numpy as np
import pytest
import torch

import oracle
from group_circulant_gemm_b200.synth import Workload, make_inputs

pytestmark = pytest.mark.gpu

TOL16 = 2e-3


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _setup(N, C, D, seed):
    from group_circulant_gemm_b200 import EqLinearPlan
    w = Workload("sv", 4, N, C, D, "f16", True, seed)
    inp = make_inputs(w, need_dy=True)
    p = EqLinearPlan(4, C, D, torch.float16)
    Wh = p.prepare_weights(_dev(inp["W"]))
    return inp, p, Wh


def _planes_ref(rows, channels):
    """float64 planes [4, N, channels] of rows [N, channels * 4], times 1/4 (the scale
    of every stored plane)."""
    F, _ = oracle.p4_transform_matrices()
    x = rows.astype(np.float64).reshape(rows.shape[0], channels, 4)
    return 0.25 * np.einsum("pt,nct->pnc", F, x)


def _check_planes(got, ref):
    # FP32 arithmetic, one rounding to FP16: within one FP16 ulp of the exact value
    err = np.abs(got.astype(np.float64) - ref)
    assert np.all(err <= np.abs(ref) * 2.0 ** -10 + 2.0 ** -24)


def _guarded(shape, dtype=torch.float16, pad=4096):
    """A tensor of `shape` inside a buffer whose margins hold a sentinel."""
    n = int(np.prod(shape))
    buf = torch.full((n + 2 * pad,), -77.0, dtype=dtype, device="cuda")
    return buf, buf[pad:pad + n].view(shape), pad


def _margins_intact(buf, pad, n):
    b = buf.float().cpu().numpy()
    return bool(np.all(b[:pad] == -77.0) and np.all(b[pad + n:] == -77.0))


CASES = [
    # N, C, D, act
    (333, 64, 128, "none"),
    (4096, 16, 48, "none"),     # the smallest widths the save calls take, whole row tiles
    (129, 128, 64, "gelu"),
    (1000, 192, 768, "none"),
    (1, 64, 64, "none"),
    (777, 80, 208, "gelu"),     # C, D not multiples of 64: the save calls only
]


@pytest.mark.parametrize("N,C,D,act", CASES)
def test_save_spectrum_calls(N, C, D, act):
    inp, p, Wh = _setup(N, C, D, 5000 + N + C)
    X, dY, b = _dev(inp["X"]), _dev(inp["dY"]), _dev(inp["bias"])
    xbuf, Xhat, pad = _guarded((4, N, C))
    Y, _ = p.forward_save_spectrum(X, Wh, b, act=act, Xhat=Xhat)
    gbuf, dYhat, gpad = _guarded((4, N, D))
    dX, _ = p.backward_input_save_spectrum(dY, Wh, dYhat=dYhat)
    assert p.status() == 0
    assert torch.equal(Y.view(torch.int16), p.forward(X, Wh, b, act=act).view(torch.int16))
    assert torch.equal(dX.view(torch.int16), p.backward_input(dY, Wh).view(torch.int16))
    _check_planes(Xhat.cpu().numpy(), _planes_ref(inp["X"], C))
    _check_planes(dYhat.cpu().numpy(), _planes_ref(inp["dY"], D))
    assert _margins_intact(xbuf, pad, 4 * N * C)
    assert _margins_intact(gbuf, gpad, 4 * N * D)


WG_CASES = [
    # N, C, D
    (333, 64, 128),
    (129, 128, 64),
    (1000, 192, 768),
    (1, 64, 64),
    (4097, 320, 192),
    (2000, 64, 384),
    (8223, 64, 64),      # many row blocks, a ragged last stage
    (129, 1024, 64),     # wide input: 8 in-channel tiles
]


@pytest.mark.parametrize("N,C,D", WG_CASES)
def test_backward_weight_from_spectra_matches_oracle(N, C, D):
    inp, p, Wh = _setup(N, C, D, 5100 + N + D)
    X, dY, b = _dev(inp["X"]), _dev(inp["dY"]), _dev(inp["bias"])
    _, Xhat = p.forward_save_spectrum(X, Wh, b)
    _, dYhat = p.backward_input_save_spectrum(dY, Wh)
    dW, db = p.backward_weight_from_spectra(Xhat, dYhat)
    dW_t, db_t = p.backward_weight(X, dY)
    assert p.status() == 0
    ref_w, ref_b = oracle.backward_weight(4, inp["X"], inp["dY"], D)
    got_w, got_b = dW.double().cpu().numpy(), db.double().cpu().numpy()
    assert _rel(got_w, ref_w) <= TOL16
    assert _rel(got_b, ref_b) <= TOL16
    # dW: the same FP16 operands as the transforming kernel, so the two agree to
    # well inside the FP16 tolerance; dbias here sums plane 0 after its FP16
    # rounding (the transforming kernel sums it in FP32), so only the tolerance
    assert _rel(got_w, dW_t.double().cpu().numpy()) <= 2e-4
    assert _rel(got_b, db_t.double().cpu().numpy()) <= TOL16


def test_backward_weight_from_spectra_f32_then_cast_is_the_fp16_call():
    N, C, D = 1500, 128, 256
    inp, p, Wh = _setup(N, C, D, 5200)
    X, dY = _dev(inp["X"]), _dev(inp["dY"])
    _, Xhat = p.forward_save_spectrum(X, Wh)
    _, dYhat = p.backward_input_save_spectrum(dY, Wh)
    dW, db = p.backward_weight_from_spectra(Xhat, dYhat)
    buf = p.backward_weight_from_spectra_f32(Xhat, dYhat)
    cast = p.cast_from_f32(buf)
    w16, b16 = p.split_grad(cast)
    assert p.status() == 0
    assert torch.equal(w16.reshape(-1).view(torch.int16), dW.reshape(-1).view(torch.int16))
    assert torch.equal(b16.view(torch.int16), db.view(torch.int16))


def test_training_step_full_size_from_spectra():
    """ViT-H fc1 shape (N = 8224, 320 -> 1280), the training step the bench
    times: sampled (d, c) pairs of dW and all of dbias against the oracle."""
    N, C, D = 8224, 320, 1280
    inp, p, Wh = _setup(N, C, D, 5300)
    X, dY, b = _dev(inp["X"]), _dev(inp["dY"]), _dev(inp["bias"])
    _, Xhat = p.forward_save_spectrum(X, Wh, b)
    _, dYhat = p.backward_input_save_spectrum(dY, Wh)
    dW, db = p.backward_weight_from_spectra(Xhat, dYhat)
    assert p.status() == 0
    # both saved spectra in full (the last partial wave runs as 64-row half units)
    _check_planes(Xhat.cpu().numpy(), _planes_ref(inp["X"], C))
    _check_planes(dYhat.cpu().numpy(), _planes_ref(inp["dY"], D))
    rng = np.random.default_rng(5301)
    d_idx = np.concatenate([[0, D - 1, 127, 128], rng.integers(0, D, 28)]).astype(np.int64)
    c_idx = np.concatenate([[0, C - 1, 255, 256], rng.integers(0, C, 28)]).astype(np.int64)
    ref = oracle.backward_weight_pairs(4, inp["X"], inp["dY"], D, d_idx, c_idx)
    got = dW.double().cpu().numpy()[d_idx, c_idx]
    assert _rel(got, ref) <= TOL16
    ref_b = inp["dY"].astype(np.float64).reshape(N, D, 4).sum(axis=(0, 2))
    assert _rel(db.double().cpu().numpy(), ref_b) <= TOL16


def test_saved_spectra_error_paths():
    from group_circulant_gemm_b200 import EqLinearPlan, native
    p = EqLinearPlan(4, 64, 128, torch.float16)
    odd = EqLinearPlan(4, 80, 128, torch.float16)       # C % 64 != 0: no dW from spectra
    p8 = EqLinearPlan(8, 64, 64, torch.float16)
    f32 = EqLinearPlan(4, 64, 64, torch.float32)
    N = 40
    Xh = torch.zeros(4, N, 80, dtype=torch.float16, device="cuda")
    Gh = torch.zeros(4, N, 128, dtype=torch.float16, device="cuda")
    dW = torch.empty(128, 80, 4, dtype=torch.float16, device="cuda")
    ws = torch.empty(max(odd.workspace_bytes(N), 16), dtype=torch.uint8, device="cuda")

    def wg(plan, n=N, x=Xh, g=Gh, dw=dW):
        return native.raw_status("eqlinear_backward_weight_from_spectra", plan.handle,
                                 x.data_ptr(), g.data_ptr(), n, dw.data_ptr(), None,
                                 ws.data_ptr(), ws.numel(), None)
    assert wg(odd) == native.EQL_ERR_UNSUPPORTED
    assert wg(p8) == native.EQL_ERR_UNSUPPORTED
    assert wg(f32) == native.EQL_ERR_UNSUPPORTED
    p.set_kernel("simt")
    assert wg(p) == native.EQL_ERR_UNSUPPORTED
    p.set_kernel("auto")
    X = torch.zeros(N, 64 * 4, dtype=torch.float16, device="cuda")
    Wh = p.prepare_weights(torch.zeros(128, 64, 4, dtype=torch.float16, device="cuda"))
    Y = torch.empty(N, 128 * 4, dtype=torch.float16, device="cuda")
    S = torch.empty(4, N, 64, dtype=torch.float16, device="cuda")

    def fwd(plan=p, spec=S, act=0):
        return native.raw_status("eqlinear_forward_save_spectrum", plan.handle, X.data_ptr(), N,
                                 Wh.data_ptr(), None, act, Y.data_ptr(),
                                 spec.data_ptr() if spec is not None else None, None)
    assert fwd() == native.EQL_OK
    assert fwd(spec=None) == native.EQL_ERR_INVALID_ARG
    assert fwd(act=9) == native.EQL_ERR_INVALID_ARG
    assert fwd(plan=p8) == native.EQL_ERR_UNSUPPORTED
    Sodd = torch.zeros(4 * N * 64 * 2 + 8, dtype=torch.uint8, device="cuda")[8:]
    assert native.raw_status("eqlinear_forward_save_spectrum", p.handle, X.data_ptr(), N,
                             Wh.data_ptr(), None, 0, Y.data_ptr(), Sodd.data_ptr(),
                             None) == native.EQL_ERR_ALIGNMENT
    # N = 0: the saves do nothing, the weight gradient writes zeros
    dW0 = torch.full((128, 64, 4), 5.0, dtype=torch.float16, device="cuda")
    db0 = torch.full((128,), 5.0, dtype=torch.float16, device="cuda")
    ws0 = torch.empty(max(p.workspace_bytes(0), 16), dtype=torch.uint8, device="cuda")
    assert native.raw_status("eqlinear_backward_weight_from_spectra", p.handle, None, None, 0,
                             dW0.data_ptr(), db0.data_ptr(), ws0.data_ptr(), ws0.numel(),
                             None) == native.EQL_OK
    torch.cuda.synchronize()
    assert float(dW0.abs().sum()) == 0.0 and float(db0.abs().sum()) == 0.0
    assert p.status() == 0


def test_dw_from_the_spectral_intermediate():
    """A layer whose input arrives as the previous layer's spectral planes
    (eqlinear_forward_to_spectral) passes those planes as its Xhat: dW then
    equals the oracle's on the spatial input they represent (the inverse p4
    transform of the planes, float64)."""
    from group_circulant_gemm_b200 import EqLinearPlan
    N, C0, C1, C2 = 777, 64, 128, 64
    w1 = Workload("sp1", 4, N, C0, C1, "f16", True, 5400)
    w2 = Workload("sp2", 4, N, C1, C2, "f16", True, 5401)
    in1, in2 = make_inputs(w1), make_inputs(w2, need_dy=True)
    p1 = EqLinearPlan(4, C0, C1, torch.float16)
    p2 = EqLinearPlan(4, C1, C2, torch.float16)
    Wh1, Wh2 = p1.prepare_weights(_dev(in1["W"])), p2.prepare_weights(_dev(in2["W"]))
    H = p1.forward_to_spectral(_dev(in1["X"]), Wh1, _dev(in1["bias"]), act="gelu")
    _, g2 = p2.backward_input_save_spectrum(_dev(in2["dY"]), Wh2)
    dW, db = p2.backward_weight_from_spectra(H, g2)
    assert p1.status() == 0 and p2.status() == 0
    _, G = oracle.p4_transform_matrices()
    # the planes carry 1/4: four times them are the plain DFT that G inverts
    Hs = np.einsum("tp,pnc->nct", G, 4.0 * H.double().cpu().numpy()).reshape(N, C1 * 4)
    ref_w, ref_b = oracle.backward_weight(4, Hs, in2["dY"], C2)
    assert _rel(dW.double().cpu().numpy(), ref_w) <= TOL16
    assert _rel(db.double().cpu().numpy(), ref_b) <= TOL16
