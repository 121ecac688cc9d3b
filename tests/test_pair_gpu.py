"""The frequency-domain form of the p4 layer on a pair of SMs (GPU required).

eqlinear_group_dft forms the group DFT of the input once (planes X0, X2, Xr, Xi
times 1/4, stored tiled: the tensor cores' operand image); eqlinear_forward_tiled
/ eqlinear_forward_tiled_next / eqlinear_backward_input_tiled multiply those
planes on the tensor cores of two SMs per 256-row tile ("Algorithmic approach"
items 1-3: forward DFT, per-frequency products, inverse DFT).  Checks, element
by element against the float64 oracle on the same FP16 inputs (FP16 bar 2e-3 of
max|ref|):
  * the planes, read back through the documented tiled layout, are the oracle's
    p4 transform times 1/4 within one FP16 rounding, padding rows zero;
  * Y, the next layer's planes, and dX, at shapes that span several tiles, ragged
    row counts (a pair tile whose second half lies past N), out-channel counts
    that leave a partial 128-channel tile, with and without bias and GELU;
  * the two-layer MLP pair kept in the frequency domain, full ViT-B size on
    sampled rows;
  * unsupported plans and misaligned buffers are rejected.
"""
import numpy as np
import pytest
import torch

import oracle
from group_circulant_gemm_b200 import native
from group_circulant_gemm_b200.synth import WORKLOADS, Workload, make_inputs

pytestmark = pytest.mark.gpu

TOL = 2e-3


def _rel(a, b):
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _plan(T, C, D, kernel="auto"):
    from group_circulant_gemm_b200 import EqLinearPlan
    return EqLinearPlan(T, C, D, torch.float16, kernel=kernel)


def _planes_ref(rows, channels):
    F, _ = oracle.p4_transform_matrices()
    x = rows.astype(np.float64).reshape(rows.shape[0], channels, 4)
    return 0.25 * np.einsum("pt,nct->pnc", F, x)


def _untile(t, N, c):
    """Tiled planes (4, c/16, Np, 16) -> float64 planes [4, N, c], following the
    layout of the header: row n's 16-byte halves are swapped when (n / 4) % 2."""
    a = t.double().cpu().numpy().reshape(4, c // 16, -1, 2, 8)
    Np = a.shape[2]
    sw = (np.arange(Np) >> 2) & 1
    idx = np.stack([sw, 1 - sw], axis=1)  # stored piece of logical half 0 and 1
    a = np.take_along_axis(a, idx[None, None, :, :, None], axis=3)
    a = a.reshape(4, c // 16, Np, 16).transpose(0, 2, 1, 3).reshape(4, Np, c)
    return a[:, :N, :], a[:, N:, :]


CASES = [
    # N, C, D, act, bias
    (333, 64, 128, "none", True),
    (257, 192, 768, "none", True),     # two pair rows, the second almost empty
    (256, 48, 80, "gelu", True),       # partial out-channel tile (80 of 128)
    (1, 16, 16, "none", False),
    (129, 768, 192, "gelu", True),     # long K, a 64-wide last tile
    (1000, 128, 256, "none", False),
    (700, 320, 1280, "none", True),
]


@pytest.mark.parametrize("N,C,D,act,bias", CASES)
def test_tiled_forward_and_dx_match_the_oracle(N, C, D, act, bias):
    w = Workload("pr", 4, N, C, D, "f16", True, 3100 + N + C)
    inp = make_inputs(w, need_dy=True)
    p = _plan(4, C, D)
    Wh = p.prepare_weights(_dev(inp["W"]))
    b = _dev(inp["bias"]) if bias else None
    Xt = p.group_dft(_dev(inp["X"]))
    got, pad = _untile(Xt, N, C)
    ref_planes = _planes_ref(inp["X"], C)
    assert np.all(np.abs(got - ref_planes) <= np.abs(ref_planes) * 2.0 ** -10 + 2.0 ** -24)
    assert np.all(pad == 0.0)
    Y = p.forward_tiled(Xt, N, Wh, b, act=act)
    Yt = p.forward_tiled_next(Xt, N, Wh, b, act=act)
    dYt = p.group_dft(_dev(inp["dY"]))
    dX = p.backward_input_tiled(dYt, N, Wh)
    assert p.status() == 0
    ref = oracle.forward(4, inp["X"], inp["W"], inp["bias"] if bias else None, act=act)
    assert _rel(Y.double().cpu().numpy(), ref) <= TOL
    assert _rel(_untile(Yt, N, D)[0], _planes_ref(ref, D)) <= TOL
    assert _rel(dX.double().cpu().numpy(), oracle.backward_input(4, inp["dY"], inp["W"])) <= TOL


def test_tiled_form_agrees_with_the_fused_kernel():
    """The tiled entry points and eqlinear_forward_act compute the same layer:
    within the FP16 bar of each other (they round the input planes at different
    points of the same FP32 arithmetic)."""
    w = Workload("pf", 4, 1500, 192, 768, "f16", True, 3300)
    inp = make_inputs(w)
    p = _plan(4, 192, 768)
    Wh = p.prepare_weights(_dev(inp["W"]))
    X = _dev(inp["X"])
    Y1 = p.forward(X, Wh, _dev(inp["bias"])).double().cpu().numpy()
    Y2 = p.forward_tiled(p.group_dft(X), 1500, Wh, _dev(inp["bias"])).double().cpu().numpy()
    assert _rel(Y2, Y1) <= TOL


def test_mlp_pair_in_the_frequency_domain_full_size_sampled_rows():
    w1, w2 = WORKLOADS["p4_vitb_fc1_f16"], WORKLOADS["p4_vitb_fc2_f16"]
    in1, in2 = make_inputs(w1), make_inputs(w2, rows=1)
    p1, p2 = _plan(4, w1.C, w1.D), _plan(4, w2.C, w2.D)
    Wh1, Wh2 = p1.prepare_weights(_dev(in1["W"])), p2.prepare_weights(_dev(in2["W"]))
    N = w1.N
    Xt = p1.group_dft(_dev(in1["X"]))
    Ht = p1.forward_tiled_next(Xt, N, Wh1, _dev(in1["bias"]), act="gelu")
    Y = p2.forward_tiled(Ht, N, Wh2, _dev(in2["bias"])).double().cpu().numpy()
    assert p1.status() == 0 and p2.status() == 0
    rng = np.random.default_rng(7)
    rows = np.unique(np.concatenate([rng.choice(N, 48, replace=False),
                                     np.arange(N - 8, N), np.arange(8),
                                     np.arange(252, 260)]))  # a pair-tile seam
    H = oracle.forward(4, in1["X"][rows], in1["W"], in1["bias"], act="gelu")
    ref = oracle.forward(4, H, in2["W"], in2["bias"])
    assert _rel(Y[rows], ref) <= TOL


def test_tiled_entries_reject_what_they_do_not_take():
    w = Workload("pb", 4, 64, 32, 32, "f16", True, 3400)
    inp = make_inputs(w)
    p = _plan(4, 32, 32)
    Wh = p.prepare_weights(_dev(inp["W"]))
    X = _dev(inp["X"])
    Xt = torch.empty(p.tiled_shape(64, 32), dtype=torch.float16, device="cuda")
    Y = torch.empty((64, 128), dtype=torch.float16, device="cuda")
    n = native
    assert n.eqlinear_tiled_spectrum_bytes(p.handle, 64, 32) == 4 * 128 * 32 * 2
    # channels must be the plan's C or D
    assert n.raw_status("eqlinear_group_dft", p.handle, X.data_ptr(), 64, 48, Xt.data_ptr(),
                        None) == n.EQL_ERR_INVALID_ARG
    # misaligned planes
    bad = torch.empty(4 * 128 * 32 + 8, dtype=torch.float16, device="cuda")[1:]
    assert n.raw_status("eqlinear_forward_tiled", p.handle, bad.data_ptr(), 64,
                        Wh.data_ptr(), None, 0, Y.data_ptr(), None) == n.EQL_ERR_ALIGNMENT
    # a plan forced to the CUDA cores has no tiled form
    p.set_kernel("simt")
    assert n.raw_status("eqlinear_forward_tiled_next", p.handle, Xt.data_ptr(), 64,
                        Wh.data_ptr(), None, 0, Xt.data_ptr(), None) == n.EQL_ERR_UNSUPPORTED
    # T = 3 plans neither (T = 4 and 8 only)
    p3 = _plan(3, 16, 16)
    assert n.raw_status("eqlinear_group_dft", p3.handle, X.data_ptr(), 64, 16, Xt.data_ptr(),
                        None) == n.EQL_ERR_UNSUPPORTED
    # N = 0 is a no-op
    p.set_kernel("auto")
    assert n.raw_status("eqlinear_forward_tiled", p.handle, None, 0, Wh.data_ptr(), None, 0,
                        None, None) == n.EQL_OK


CHAIN_CASES = [
    # N, C0, C1, C2, act
    (333, 64, 128, 64, "none"),
    (1000, 192, 768, 192, "gelu"),
    (257, 48, 80, 32, "none"),
    (1, 16, 32, 16, "gelu"),
    (2600, 128, 256, 128, "none"),   # more tasks than pairs: the queue wraps
]


@pytest.mark.parametrize("N,C0,C1,C2,act", CHAIN_CASES)
def test_tiled_chain_equals_two_calls_bitwise(N, C0, C1, C2, act):
    from group_circulant_gemm_b200.layer import forward_chain_tiled
    w1 = Workload("c1", 4, N, C0, C1, "f16", True, 3500 + N)
    w2 = Workload("c2", 4, N, C1, C2, "f16", True, 3600 + N)
    in1, in2 = make_inputs(w1), make_inputs(w2, rows=1)
    p1, p2 = _plan(4, C0, C1), _plan(4, C1, C2)
    Wh1, Wh2 = p1.prepare_weights(_dev(in1["W"])), p2.prepare_weights(_dev(in2["W"]))
    b1, b2 = _dev(in1["bias"]), _dev(in2["bias"])
    Xt = p1.group_dft(_dev(in1["X"]))
    ws = torch.zeros(native.eqlinear_chain_tiled_workspace_bytes(p1.handle, p2.handle, N) + 64,
                     dtype=torch.uint8, device="cuda")
    for _ in range(2):  # the second call reuses the workspace the first left zero
        Ht, Y = forward_chain_tiled(p1, p2, Xt, N, Wh1, b1, Wh2, b2, act=act, workspace=ws)
        assert p1.status() == 0 and p2.status() == 0
        assert int(ws.abs().sum()) == 0
    Ht_ref = p1.forward_tiled_next(Xt, N, Wh1, b1, act=act)
    Y_ref = p2.forward_tiled(Ht_ref, N, Wh2, b2)
    got_h, _ = _untile(Ht, N, C1)
    ref_h, _ = _untile(Ht_ref, N, C1)
    assert np.array_equal(got_h, ref_h)
    assert torch.equal(Y, Y_ref)
    if N <= 1000:
        H = oracle.forward(4, in1["X"], in1["W"], in1["bias"], act=act)
        assert _rel(Y.double().cpu().numpy(), oracle.forward(4, H, in2["W"], in2["bias"])) <= TOL


def test_tiled_chain_full_size_sampled_rows():
    from group_circulant_gemm_b200.layer import forward_chain_tiled
    w1, w2 = WORKLOADS["p4_vitb_fc1_f16"], WORKLOADS["p4_vitb_fc2_f16"]
    in1, in2 = make_inputs(w1), make_inputs(w2, rows=1)
    p1, p2 = _plan(4, w1.C, w1.D), _plan(4, w2.C, w2.D)
    Wh1, Wh2 = p1.prepare_weights(_dev(in1["W"])), p2.prepare_weights(_dev(in2["W"]))
    N = w1.N
    Xt = p1.group_dft(_dev(in1["X"]))
    _, Y = forward_chain_tiled(p1, p2, Xt, N, Wh1, _dev(in1["bias"]), Wh2, _dev(in2["bias"]))
    Y = Y.double().cpu().numpy()
    assert p1.status() == 0 and p2.status() == 0
    rng = np.random.default_rng(11)
    rows = np.unique(np.concatenate([rng.choice(N, 48, replace=False), np.arange(N - 8, N),
                                     np.arange(8), np.arange(252, 260)]))
    H = oracle.forward(4, in1["X"][rows], in1["W"], in1["bias"])
    assert _rel(Y[rows], oracle.forward(4, H, in2["W"], in2["bias"])) <= TOL


def test_tiled_chain_rejects_bad_arguments():
    p1, p2, p3 = _plan(4, 32, 64), _plan(4, 64, 32), _plan(4, 48, 32)
    N = 100
    Xt = torch.zeros(p1.tiled_shape(N, 32), dtype=torch.float16, device="cuda")
    Ht = torch.zeros(p1.tiled_shape(N, 64), dtype=torch.float16, device="cuda")
    Y = torch.zeros((N, 128), dtype=torch.float16, device="cuda")
    W1 = torch.zeros(native.eqlinear_prepared_weight_bytes(p1.handle) // 2, dtype=torch.float16,
                     device="cuda")
    W2 = torch.zeros(native.eqlinear_prepared_weight_bytes(p2.handle) // 2, dtype=torch.float16,
                     device="cuda")
    nb = native.eqlinear_chain_tiled_workspace_bytes(p1.handle, p2.handle, N)
    ws = torch.zeros(nb, dtype=torch.uint8, device="cuda")

    def call(a, b, wsb=nb):
        return native.raw_status("eqlinear_forward_chain_tiled", a.handle, b.handle, Xt.data_ptr(),
                                 N, W1.data_ptr(), None, 0, W2.data_ptr(), None, Ht.data_ptr(),
                                 Y.data_ptr(), ws.data_ptr(), wsb, None)

    assert call(p1, p3) == native.EQL_ERR_INVALID_ARG      # widths do not chain
    assert call(p1, p2, nb - 4) == native.EQL_ERR_WORKSPACE
